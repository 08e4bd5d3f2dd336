// kvq_card.cuh -- CacheCard kernels: gather the used rows of many views into
// one contiguous card image in device memory (pack), and scatter a card image
// back into views (unpack).
//
// "QKVShare: Quantized KV-Cache Handoff for Multi-Agent On-Device LLMs",
// Metodologia (CacheCard representation): one compact artifact carries the
// quantized KV groups, their width assignment and the metadata a receiver
// needs (sequence length, model id, position offset).  "Agent Memory Below the
// Prompt: Persistent Q4 KV Cache ...", Abstract: per-agent 4-bit caches are
// persisted and reloaded straight into attention.
//
// Card layout (little-endian), all offsets from the card start:
//   [0, 64)            CardHeader
//   [64, 64 + 64 n)    one CardView record per view
//   then per view, at its data_offset (256-byte aligned), six sections, each
//   16-byte aligned: K codes [H][n_packed][row_bytes], V codes, K scale/min
//   [H][n_packed][D/64][2] fp32, V scale/min, K window [H][n_window][D] bf16
//   in logical order (oldest first), V window.
#pragma once

#include <cstdint>

#include "kvq_debug.cuh"

namespace kvq {

constexpr int kCardMaxViews = 96;  // views per pack/unpack launch
constexpr uint32_t kCardVersion = 1;

struct CardHeader {
    char magic[8];          // "KVQCARD1"
    uint32_t version;
    uint32_t n_views;
    uint32_t n_kv_heads;
    uint32_t head_dim;
    uint64_t model_id;      // caller's tag of the model the cache belongs to
    uint64_t total_bytes;
    uint8_t pad[24];
};
static_assert(sizeof(CardHeader) == 64, "card header");

struct CardView {
    uint32_t bits;
    uint32_t n_window;
    uint64_t n_packed;
    int64_t position_offset;  // position of the view's first token in the sequence
    uint64_t data_offset;
    uint64_t data_bytes;
    uint64_t seq_len;         // n_packed + n_window
    uint8_t pad[16];
};
static_assert(sizeof(CardView) == 64, "card view record");

// One view's side of a pack/unpack launch, resolved on the host.
struct CardSide {
    uint8_t *codes[2];        // K, V packed rows [H][cap_packed][RB]
    float *scalemin[2];       // [H][cap_packed][NG][2]
    uint16_t *window[2];      // bf16 [H][cap_window][D]
    int64_t cap_packed;
    int64_t n_packed;
    int32_t cap_window;
    int32_t n_window;
    int32_t window_head;      // pack: ring slot of the oldest token; unpack: 0
    int32_t row_bytes;
    uint64_t sect_off[6];     // card offsets of the six sections
    CardView record;          // written by pack
};

// Sections are cut into pieces of whole rows of one KV head, about
// kCardPieceBytes each; one CTA copies one piece.  Host and kernel both derive
// a section's piece count from its row size with these two functions.
constexpr int64_t kCardPieceBytes = 32 * 1024;
constexpr int kCardSections = 6;

__host__ __device__ inline int64_t card_piece_rows(int64_t row) {
    return row >= kCardPieceBytes ? 1 : kCardPieceBytes / row;
}
__host__ __device__ inline int64_t card_pieces_per_head(int64_t rows, int64_t row) {
    const int64_t r = card_piece_rows(row);
    return (rows + r - 1) / r;
}

struct CardArgs {
    uint8_t *card;            // device card image
    uint64_t card_bytes;      // its size (the debug build's checks)
    int32_t n_views;
    int32_t n_kv_heads;
    int32_t head_dim;
    int32_t write_header;     // pack: this launch also writes the card header
    CardHeader header;
    uint64_t records_off;     // card offset of this launch's first record
    // first CTA of each (view, section) entry, entry = view * 6 + section;
    // entry_cta[6 * n_views] is the number of copying CTAs
    uint32_t entry_cta[kCardMaxViews * kCardSections + 1];
    CardSide views[kCardMaxViews];
};

// Copy n bytes from src to dst with one CTA, T-sized accesses (n and both
// addresses multiples of sizeof(T)); four loads in flight per thread.
template <typename T>
__device__ __forceinline__ void cta_copy(uint8_t *dst, const uint8_t *src, int64_t n) {
    const T *s = reinterpret_cast<const T *>(src);
    T *d = reinterpret_cast<T *>(dst);
    const int64_t nv = n / (int64_t)sizeof(T), bd = blockDim.x;
    int64_t i = threadIdx.x;
    for (; i + 3 * bd < nv; i += 4 * bd) {
        const T a0 = __ldcs(s + i), a1 = __ldcs(s + i + bd), a2 = __ldcs(s + i + 2 * bd), a3 = __ldcs(s + i + 3 * bd);
        __stcs(d + i, a0);
        __stcs(d + i + bd, a1);
        __stcs(d + i + 2 * bd, a2);
        __stcs(d + i + 3 * bd, a3);
    }
    for (; i < nv; i += bd) __stcs(d + i, __ldcs(s + i));
}

// Every row size is a multiple of 8 bytes; 16-byte accesses when both ends
// allow them.
__device__ __forceinline__ void cta_copy_rows(uint8_t *dst, const uint8_t *src, int64_t n) {
    if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | (uintptr_t)n) & 15) == 0)
        cta_copy<uint4>(dst, src, n);
    else
        cta_copy<uint2>(dst, src, n);
}

// One CTA per piece.  PACK: views -> card (CTA 0 also writes this launch's
// records and, on the first launch, the header); otherwise card -> views, the
// window landing in slots 0 .. n_window-1.
template <bool PACK>
__global__ void __launch_bounds__(256, 4) card_kernel(const __grid_constant__ CardArgs a) {
    if (PACK && blockIdx.x == 0) {
        CardView *rec = reinterpret_cast<CardView *>(a.card + a.records_off);
        for (int i = threadIdx.x; i < a.n_views; i += blockDim.x) rec[i] = a.views[i].record;
        if (a.write_header && threadIdx.x == 0) *reinterpret_cast<CardHeader *>(a.card) = a.header;
    }
    const uint32_t cta = blockIdx.x;
    const int n_entries = a.n_views * kCardSections;
    if (cta >= a.entry_cta[n_entries]) return;
    // the entry holding this CTA: the last one whose first CTA is <= cta
    int lo = 0, hi = n_entries - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.entry_cta[mid] <= cta) lo = mid;
        else hi = mid - 1;
    }
    const CardSide &v = a.views[lo / kCardSections];
    const int sect = lo % kCardSections, kv = sect & 1;
    const int D = a.head_dim;
    const bool window = sect >= 4;
    const int64_t row = sect < 2 ? v.row_bytes : sect < 4 ? (int64_t)(D / 64) * 8 : (int64_t)D * 2;
    const int64_t rows = window ? v.n_window : v.n_packed;
    const int64_t pph = card_pieces_per_head(rows, row);
    const int64_t local = cta - a.entry_cta[lo];
    const int64_t h = local / pph, r0 = (local % pph) * card_piece_rows(row);
    const int64_t r1 = min(rows, r0 + card_piece_rows(row));
    uint8_t *card_p = a.card + v.sect_off[sect] + (h * rows + r0) * row;
    // the piece lies in the card and in the view's rows or ring (debug build)
    if (!dcheck(h < a.n_kv_heads && r0 >= 0 && r0 <= r1 &&
                    v.sect_off[sect] + (uint64_t)((h * rows + r1) * row) <= a.card_bytes &&
                    (window ? r1 <= v.cap_window : r1 <= v.cap_packed),
                kDbgCard))
        return;
    if (!window) {
        uint8_t *base = sect < 2 ? v.codes[kv] : reinterpret_cast<uint8_t *>(v.scalemin[kv]);
        uint8_t *view_p = base + (h * v.cap_packed + r0) * row;
        if (PACK) cta_copy_rows(card_p, view_p, (r1 - r0) * row);
        else cta_copy_rows(view_p, card_p, (r1 - r0) * row);
    } else {
        // logical rows r0..r1 of the ring: slots (window_head + r) mod cap, at
        // most two contiguous runs
        uint8_t *ring = reinterpret_cast<uint8_t *>(v.window[kv]) + h * v.cap_window * row;
        const int64_t s0 = (v.window_head + r0) % v.cap_window;
        const int64_t first = min(r1 - r0, (int64_t)v.cap_window - s0);
        if (PACK) {
            cta_copy_rows(card_p, ring + s0 * row, first * row);
            if (first < r1 - r0) cta_copy_rows(card_p + first * row, ring, (r1 - r0 - first) * row);
        } else {
            cta_copy_rows(ring + s0 * row, card_p, first * row);
            if (first < r1 - r0) cta_copy_rows(ring, card_p + first * row, (r1 - r0 - first) * row);
        }
    }
}

}  // namespace kvq
