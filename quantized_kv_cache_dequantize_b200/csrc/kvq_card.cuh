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

struct CardArgs {
    uint8_t *card;            // device card image
    int32_t n_views;
    int32_t n_kv_heads;
    int32_t head_dim;
    int32_t write_header;     // pack: this launch also writes the card header
    CardHeader header;
    uint64_t records_off;     // card offset of this launch's first record
    CardSide views[kCardMaxViews];
};

// Copy n bytes (multiple of 8, both ends 8-byte aligned) with one CTA.
__device__ __forceinline__ void cta_copy8(uint8_t *dst, const uint8_t *src, int64_t n) {
    const uint2 *s = reinterpret_cast<const uint2 *>(src);
    uint2 *d = reinterpret_cast<uint2 *>(dst);
    const int64_t n8 = n >> 3;
    for (int64_t i = threadIdx.x; i < n8; i += blockDim.x) __stcs(d + i, __ldcs(s + i));
}

// Grid (view, KV head, section).  PACK: views -> card; otherwise card -> views
// (the window lands in slots 0 .. n_window-1).
template <bool PACK>
__global__ void __launch_bounds__(256) card_kernel(const __grid_constant__ CardArgs a) {
    const CardSide &v = a.views[blockIdx.x];
    const int h = blockIdx.y, sect = blockIdx.z;
    const int D = a.head_dim, NG = D / 64;
    if (PACK && threadIdx.x == 0 && h == 0 && sect == 0) {
        reinterpret_cast<CardView *>(a.card + a.records_off)[blockIdx.x] = v.record;
        if (a.write_header && blockIdx.x == 0) *reinterpret_cast<CardHeader *>(a.card) = a.header;
    }
    const int kv = sect & 1;
    if (sect < 4) {
        // packed rows of head h: contiguous in the view and in the card
        const bool codes = sect < 2;
        const int64_t row = codes ? v.row_bytes : (int64_t)NG * 8;
        const int64_t n = v.n_packed * row;
        uint8_t *view_p = codes ? v.codes[kv] + (int64_t)h * v.cap_packed * row
                                : reinterpret_cast<uint8_t *>(v.scalemin[kv]) + (int64_t)h * v.cap_packed * row;
        uint8_t *card_p = a.card + v.sect_off[sect] + (int64_t)h * n;
        if (PACK) cta_copy8(card_p, view_p, n);
        else cta_copy8(view_p, card_p, n);
    } else {
        // window rows of head h: the ring's logical order (two pieces when it wraps)
        if (v.n_window == 0) return;
        const int64_t row = (int64_t)D * 2;
        uint8_t *ring = reinterpret_cast<uint8_t *>(v.window[kv]) + (int64_t)h * v.cap_window * row;
        uint8_t *card_p = a.card + v.sect_off[sect] + (int64_t)h * v.n_window * row;
        const int first = min(v.n_window, v.cap_window - v.window_head);
        if (PACK) {
            cta_copy8(card_p, ring + (int64_t)v.window_head * row, first * row);
            if (first < v.n_window) cta_copy8(card_p + first * row, ring, (v.n_window - first) * row);
        } else {
            cta_copy8(ring + (int64_t)v.window_head * row, card_p, first * row);
            if (first < v.n_window) cta_copy8(ring, card_p + first * row, (v.n_window - first) * row);
        }
    }
}

}  // namespace kvq
