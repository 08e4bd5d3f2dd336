// kvq.cu -- C-ABI entry points of libkvq (declared in include/kvq.h):
// argument validation on the host, work planning, and kernel launches for
// sm_100a.  Nothing here allocates device memory or synchronizes.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <limits>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "kvq.h"
#include "kvq_alloc.cuh"
#include "kvq_attn.cuh"
#include "kvq_card.cuh"
#include "kvq_codec.cuh"
#include "kvq_sparse.cuh"

#define KVQ_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kAbiVersion = 1;
constexpr int kMaxDevices = 64;

bool bits_supported(int32_t bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }
bool head_dim_supported(int32_t d) { return d >= 64 && d <= KVQ_MAX_HEAD_DIM && d % 64 == 0; }
bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
int64_t row_bytes(int32_t head_dim, int32_t bits) { return (int64_t)head_dim / 8 * bits; }

int device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return 148;
    }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        (void)cudaGetLastError();
        return 148;
    }
    return sms;
}

template <int B, int NG>
void launch_codec(bool quant, const kvq::CodecArgs &a, cudaStream_t st) {
    // one flat sweep over the rows of all heads; blocks of 8 warps, a few
    // resident per SM, the grid several waves deep (the sweep's tail balances
    // better).  Quantize: 16 groups per warp at a time, 16 blocks per SM (on
    // the handoff's K cache 591.6 us against 604.0 with 8 per SM, 614.2 with
    // one wave of 5); dequantize: kDeqUnroll units of RPU rows per warp at a
    // time, 24 blocks per SM (536.3 against 543.5 us with 8).
    const int64_t rows = a.n_tokens * a.n_heads;
    const int64_t per_block = quant ? 8 * 16 / NG : 8 * kvq::kDeqUnroll * kvq::DeqShape<NG>::RPU;
    const int64_t max_blocks = std::max<int64_t>(1, (rows + per_block - 1) / per_block);
    const int64_t blocks =
        std::max<int64_t>(1, std::min<int64_t>(max_blocks, (int64_t)device_sm_count() * (quant ? 16 : 24)));
    if (quant)
        kvq::quantize_kernel<B, NG><<<(unsigned)blocks, 256, 0, st>>>(a);
    else
        kvq::dequantize_kernel<B, NG><<<(unsigned)blocks, 256, 0, st>>>(a);
}

template <int B>
void launch_codec_ng(bool quant, int ng, const kvq::CodecArgs &a, cudaStream_t st) {
    switch (ng) {
        case 1: launch_codec<B, 1>(quant, a, st); break;
        case 2: launch_codec<B, 2>(quant, a, st); break;
        case 3: launch_codec<B, 3>(quant, a, st); break;
        default: launch_codec<B, 4>(quant, a, st); break;
    }
}

kvq_status codec(bool quant, const void *x, int64_t hs, int64_t ts, int32_t n_heads, int64_t n_tokens,
                 int32_t head_dim, int32_t bits, const void *codes, const float *scalemin, int64_t cap,
                 void *stream) {
    if (!bits_supported(bits) || !head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (n_heads < 0 || n_tokens < 0 || cap < n_tokens || n_heads > 65535) return KVQ_ERR_INVALID_ARG;
    if (n_heads == 0 || n_tokens == 0) return KVQ_OK;
    if (!x || !codes || !scalemin) return KVQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scalemin, 8)) return KVQ_ERR_INVALID_ARG;
    if (hs < 0 || ts < 0 || hs % 8 || ts % 8) return KVQ_ERR_INVALID_ARG;
    // dequantize writes rows: consecutive tokens and heads may not share a row
    if (!quant && ((n_tokens > 1 && ts < head_dim) || (n_heads > 1 && hs < head_dim))) return KVQ_ERR_INVALID_ARG;
    kvq::CodecArgs a;
    a.x = static_cast<const uint16_t *>(x);
    a.x_head_stride = hs;
    a.x_tok_stride = ts;
    a.n_tokens = n_tokens;
    a.n_heads = n_heads;
    a.codes = static_cast<uint8_t *>(const_cast<void *>(codes));
    a.scalemin = const_cast<float *>(scalemin);
    a.head_cap = cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int ng = head_dim / 64;
    switch (bits) {
        case 2: launch_codec_ng<2>(quant, ng, a, st); break;
        case 3: launch_codec_ng<3>(quant, ng, a, st); break;
        case 4: launch_codec_ng<4>(quant, ng, a, st); break;
        default: launch_codec_ng<8>(quant, ng, a, st); break;
    }
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// ------------------------------------------------------ decode planning ---

struct AttnLaunch {
    int v0, v1;          // views order[v0 .. v1) of the plan
    int total_chunks;
    int bits;            // the width of every view of the launch with packed tokens
    int ring_bytes = 0;  // per warp, and the launch's dynamic shared memory:
    size_t smem = 0;     // sized for this launch's own blocks
};

struct ViewChunks {
    int32_t n_packed, n_window;  // chunks of the packed part and of the window
};

struct AttnPlan {
    int ring_bytes = 0;
    size_t smem = 0;
    int head_blocks = 0;
    std::vector<int> order;  // views with tokens, grouped by width (stable), as the launches take them
    std::vector<AttnLaunch> launches;
    std::vector<ViewChunks> chunks;
    std::vector<int32_t> seq_of, part_begin;        // per view: its sequence, partial slot of its chunk 0
    std::vector<int32_t> seq_part_begin, seq_chunks;  // per sequence
    size_t counters_off = 0, partials_off = 0;
    size_t zero_bytes = 0, total = 0;
    int64_t n_slots = 0;                            // partial slots of the call (every unit)
};

int env_int(const char *name, int dflt) {
    const char *s = std::getenv(name);
    if (!s || !*s) return dflt;
    const long v = std::strtol(s, nullptr, 10);
    return v > 0 ? (int)v : dflt;
}

kvq_status validate_views(const kvq_view *views, int32_t n_views, bool need_nonempty) {
    if (!views || n_views <= 0 || n_views > KVQ_MAX_VIEWS) return KVQ_ERR_INVALID_ARG;
    for (int i = 0; i < n_views; ++i) {
        const kvq_view &v = views[i];
        if (v.n_packed < 0 || v.cap_packed < v.n_packed || (v.cap_packed & 1)) return KVQ_ERR_INVALID_ARG;
        if (v.cap_packed > INT32_MAX) return KVQ_ERR_INVALID_ARG;
        if (v.cap_window < 0 || v.n_window < 0 || v.n_window > v.cap_window) return KVQ_ERR_INVALID_ARG;
        if (v.cap_window > 0 && (v.window_head < 0 || v.window_head >= v.cap_window)) return KVQ_ERR_INVALID_ARG;
        if (need_nonempty && v.n_packed + v.n_window <= 0) return KVQ_ERR_INVALID_ARG;
        if (v.cap_packed > 0 || v.n_packed > 0) {
            if (!bits_supported(v.bits)) return KVQ_ERR_UNSUPPORTED;
            if (!v.k_codes || !v.v_codes || !v.k_scalemin || !v.v_scalemin) return KVQ_ERR_INVALID_ARG;
            if (!aligned(v.k_codes, 16) || !aligned(v.v_codes, 16) || !aligned(v.k_scalemin, 16) ||
                !aligned(v.v_scalemin, 16))
                return KVQ_ERR_INVALID_ARG;
        }
        if (v.cap_window > 0) {
            if (!v.k_window || !v.v_window || !aligned(v.k_window, 16) || !aligned(v.v_window, 16))
                return KVQ_ERR_INVALID_ARG;
        }
    }
    return KVQ_OK;
}

int attn_ctas_per_sm(int ng) {
    switch (ng) {
        case 1: return kvq::attn_ctas_per_sm<1>();
        case 2: return kvq::attn_ctas_per_sm<2>();
        case 3: return kvq::attn_ctas_per_sm<3>();
        default: return kvq::attn_ctas_per_sm<4>();
    }
}

int attn_team_warps(int ng) {
    switch (ng) {
        case 1: return kvq::attn_team_warps<1>();
        case 2: return kvq::attn_team_warps<2>();
        case 3: return kvq::attn_team_warps<3>();
        default: return kvq::attn_team_warps<4>();
    }
}

int attn_header_bytes(int ng) {
    switch (ng) {
        case 1: return kvq::attn_header_bytes<1>();
        case 2: return kvq::attn_header_bytes<2>();
        case 3: return kvq::attn_header_bytes<3>();
        default: return kvq::attn_header_bytes<4>();
    }
}

// Bytes of one unit's packed token (K and V codes + scale/min) and window token.
int64_t packed_token_bytes(int32_t head_dim, int32_t bits) { return 2 * row_bytes(head_dim, bits) + 16 * (head_dim / 64); }
int64_t window_token_bytes(int32_t head_dim) { return 4 * (int64_t)head_dim; }

// Planner cost of a packed token, in byte-equivalents: its bytes, or a floor
// for its arithmetic (unpacking, MMAs and the affine fold do not shrink with
// the width), whichever is more.  Without the floor a 2-bit token looks 40 %
// cheaper than a 4-bit one, and a mixed-width call gives its narrow views
// too few CTAs.  The floor, 80 bytes per 64-dim group, is the largest that
// leaves the 4-bit plans as they were: Qwen3-32B-shape layer 82.1 -> 72.0
// us; Llama-3.1-8B and Gemma-3-12B layers unchanged (120 and more moved the
// Gemma plan off its best, 74 -> 80 us).
constexpr double kTokComputePerGroup = 80.0;
double packed_token_cost(int32_t head_dim, int32_t bits) {
    return std::max((double)packed_token_bytes(head_dim, bits), kTokComputePerGroup * (head_dim / 64));
}

// Cost model of a work item, in byte-equivalents: its tokens' costs (packed:
// packed_token_cost; window: bytes) plus a fixed per-CTA cost (set-up,
// pipeline fill, partial merge).  A
// launch's predicted time is its number of waves times (largest item +
// per-CTA cost).
// Items are kept between kMinItem and kBigItem (larger items measured slower
// on the 32K-token dense layer: 127.6 vs 123.5 us at 1 MB).
constexpr double kCtaCost = 96.0 * 1024;
constexpr double kMinItem = 16.0 * 1024, kBigItem = 512.0 * 1024;

// Cost of the largest of n chunks of equal step counts over n_tok tokens.
double largest_chunk(int64_t n_tok, int step, int64_t n, double tok_cost) {
    if (n <= 0) return 0.0;
    const int64_t steps = (n_tok + step - 1) / step;
    return (double)std::min<int64_t>((steps + n - 1) / n * step, n_tok) * tok_cost;
}

// Free chunking of the views idx[0 .. n): each part (packed, window) of a
// view is cut into chunks of equal step counts (+-1 step) costing about W
// each, W picked by the smallest predicted time over whole waves of `slots`
// resident CTAs.  Stores the chunk counts, returns the predicted time;
// *chunks = the launch's chunk count per unit.
double plan_free(const kvq_view *views, const int *idx, int n_idx, int64_t units, int32_t head_dim, int64_t slots,
                 std::vector<ViewChunks> &out, int64_t *chunks, double big_item = kBigItem) {
    const int forced = env_int("KVQ_CHUNK_TOKENS", 0);  // tests: force a chunk length
    double total = 0;
    for (int k = 0; k < n_idx; ++k) {
        const kvq_view &v = views[idx[k]];
        total += (double)units * ((double)v.n_packed * packed_token_cost(head_dim, v.bits) +
                                  (double)v.n_window * window_token_bytes(head_dim));
    }
    auto split = [&](int64_t n_tok, int step, double tok_cost, double W) -> int64_t {
        if (n_tok <= 0) return 0;
        const int64_t steps = (n_tok + step - 1) / step;
        const int64_t n = forced > 0 ? (n_tok + forced - 1) / forced : std::llround((double)n_tok * tok_cost / W);
        return std::max<int64_t>(1, std::min<int64_t>(n, steps));
    };
    auto count = [&](double W, bool store, double *max_item) -> int64_t {
        int64_t items = 0;
        double mx = 0;
        for (int k = 0; k < n_idx; ++k) {
            const int i = idx[k];
            const kvq_view &v = views[i];
            const double cp = packed_token_cost(head_dim, v.bits), cw = (double)window_token_bytes(head_dim);
            int64_t np = split(v.n_packed, 2 * kvq::kTile, cp, W), nw = split(v.n_window, kvq::kTile, cw, W);
            // the unit combine holds at most kMaxChunksPerUnit chunks per unit
            while (np + nw > kvq::kMaxChunksPerUnit) {
                if (np >= nw) np = std::max<int64_t>(1, np * 3 / 4);
                else nw = std::max<int64_t>(1, nw * 3 / 4);
            }
            mx = std::max(mx, std::max(largest_chunk(v.n_packed, 2 * kvq::kTile, np, cp),
                                       largest_chunk(v.n_window, kvq::kTile, nw, cw)));
            items += np + nw;
            if (store) out[i] = ViewChunks{(int32_t)np, (int32_t)nw};
        }
        if (max_item) *max_item = mx;
        return items;
    };
    double best_W = std::max(kMinItem, std::min(big_item, total / (double)slots)), best_cost = 1e300;
    const double fs[] = {0.5, 0.6, 0.7, 0.8, 0.9, 1.0, 1.15, 1.3, 1.5, 1.75, 2.0, 2.5, 3.0, 4.0,
                         5.0, 6.0, 8.0, 12.0, 16.0, 24.0, 32.0};
    for (double f : fs) {
        const double W = std::max(kMinItem, std::min(big_item, total / ((double)slots * f)));
        double mx = 0;
        const int64_t items = count(W, false, &mx) * units;
        const double cost = (double)((items + slots - 1) / slots) * (mx + kCtaCost);
        if (cost < best_cost * 0.999) {
            best_cost = cost;
            best_W = W;
        }
    }
    *chunks = count(best_W, true, nullptr);
    return best_cost;
}

template <int NG, int BSEL, bool SCORE = false>
kvq_status ensure_attn_smem(size_t smem) {
    // the attention (or score) kernel's dynamic shared-memory limit, raised once per device
    static std::mutex mu;
    static int configured[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return KVQ_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= kMaxDevices || configured[dev] < (int)smem) {
        cudaError_t e;
        if constexpr (SCORE)
            e = cudaFuncSetAttribute(kvq::score_attn_kernel<NG, BSEL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
        else
            e = cudaFuncSetAttribute(kvq::decode_attn_kernel<NG, BSEL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return KVQ_ERR_CUDA;
        }
        if (dev < kMaxDevices) configured[dev] = (int)smem;
    }
    return KVQ_OK;
}

// seq_begin == nullptr: every view is a sequence of its own (and must hold a
// token).  Otherwise sequence s is views seq_begin[s] .. seq_begin[s+1]-1, its
// tokens the concatenation of theirs; empty views are allowed and skipped.
// allow_empty (internal callers): sequences without tokens are planned as
// nothing at all.
kvq_status plan_attn(const kvq_view *views, int32_t n_views, const int32_t *seq_begin, int32_t n_seqs,
                     int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, AttnPlan &plan,
                     bool allow_empty = false, double big_item = kBigItem) {
    if (!head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads || n_kv_heads > 65535)
        return KVQ_ERR_INVALID_ARG;
    const kvq_status vs = validate_views(views, n_views, seq_begin == nullptr);
    if (vs != KVQ_OK) return vs;
    plan.seq_of.assign(n_views, 0);
    if (!seq_begin) {
        n_seqs = n_views;
        for (int i = 0; i < n_views; ++i) plan.seq_of[i] = i;
    } else {
        if (n_seqs <= 0 || seq_begin[0] != 0 || seq_begin[n_seqs] != n_views) return KVQ_ERR_INVALID_ARG;
        for (int s = 0; s < n_seqs; ++s) {
            if (seq_begin[s + 1] <= seq_begin[s]) return KVQ_ERR_INVALID_ARG;
            int64_t tokens = 0;
            int used = 0;
            for (int i = seq_begin[s]; i < seq_begin[s + 1]; ++i) {
                plan.seq_of[i] = s;
                tokens += views[i].n_packed + views[i].n_window;
                used += views[i].n_packed + views[i].n_window > 0 ? 1 : 0;
            }
            if (tokens <= 0 && !allow_empty) return KVQ_ERR_INVALID_ARG;
            if (used > KVQ_MAX_SEGMENTS) return KVQ_ERR_UNSUPPORTED;
        }
    }
    const int ng = head_dim / 64;
    const int group = n_q_heads / n_kv_heads;
    plan.head_blocks = (group + kvq::kHeadsPerCta - 1) / kvq::kHeadsPerCta;
    if (plan.head_blocks > 65535) return KVQ_ERR_UNSUPPORTED;
    const int64_t units = (int64_t)n_kv_heads * plan.head_blocks;

    // shared memory: the CTA's share of the SM at the kernel's target occupancy
    const int ctas = attn_ctas_per_sm(ng);
    const int smem_cta = std::min(227 * 1024, (228 * 1024) / ctas - 1024);
    const int header = attn_header_bytes(ng);
    const int ring_fit = (smem_cta - header) / kvq::kAttnWarps / 128 * 128;
    // Ring and shared memory of a launch over views[order[v0 .. v1)]: a
    // team's ring (its warps' rings together) holds two of the launch's
    // largest blocks, and later the team's partial (m, l, O of 8 heads); all
    // rings together hold the unit combine's scratch.  Per launch, so that a
    // mixed-width call's 8-bit blocks do not take the narrower launches'
    // CTAs per SM.
    const uint32_t tw = (uint32_t)attn_team_warps(ng);
    const uint32_t combine_scratch = (2 * kvq::kMaxChunksPerUnit * kvq::kHeadsPerCta + kvq::kHeadsPerCta) * 4;
    auto size_launch = [&](AttnLaunch &L) -> bool {
        uint32_t blk_max = 0;
        for (int k = L.v0; k < L.v1; ++k) {
            const kvq_view &v = views[plan.order[k]];
            if (v.n_packed > 0)
                blk_max = std::max<uint32_t>(blk_max, (uint32_t)(64 * row_bytes(head_dim, v.bits) + 512 * ng));
            if (v.n_window > 0) blk_max = std::max<uint32_t>(blk_max, (uint32_t)(32 * head_dim));
        }
        const int ring_min = (int)std::max<uint32_t>(
            std::max<uint32_t>((2 * blk_max + tw - 1) / tw, (64 + 32 * (uint32_t)head_dim + tw - 1) / tw),
            (combine_scratch + kvq::kAttnWarps - 1) / kvq::kAttnWarps);
        int ring = ring_fit;
        if (ring < ring_min) ring = (ring_min + 127) / 128 * 128;  // fewer CTAs per SM, still correct
        L.ring_bytes = ring;
        L.smem = (size_t)header + (size_t)kvq::kAttnWarps * ring;
        return L.smem <= 227 * 1024;
    };

    const int64_t slots = (int64_t)device_sm_count() * ctas;
    plan.chunks.assign(n_views, ViewChunks{0, 0});
    // Views grouped by width (stable; views without packed tokens join the
    // first width), at most kAttnMaxViews per launch: each launch then runs
    // the kernel built for its width alone.  All launches of a call run
    // concurrently, each on its own workspace regions, so each is planned for
    // its byte share of the GPU.
    int first_bits = 4;
    for (int i = 0; i < n_views; ++i)
        if (views[i].n_packed > 0) { first_bits = views[i].bits; break; }
    auto key = [&](int i) { return views[i].n_packed > 0 ? views[i].bits : first_bits; };
    plan.order.clear();
    for (int i = 0; i < n_views; ++i)
        if (views[i].n_packed + views[i].n_window > 0) plan.order.push_back(i);
    const int n_used = (int)plan.order.size();
    std::stable_sort(plan.order.begin(), plan.order.end(), [&](int a, int b) { return key(a) < key(b); });
    double bytes_all = 0;
    for (int i = 0; i < n_views; ++i)
        bytes_all += (double)views[i].n_packed * packed_token_cost(head_dim, views[i].bits) +
                     (double)views[i].n_window * window_token_bytes(head_dim);
    // A call of several width launches is planned for 5/4 of the resident
    // slots: the launches run side by side, and smaller items let them share
    // the SMs more evenly (Qwen3-32B-shape layer, widths 2/3/4/8: 68.5 vs
    // 73.0 us).  A single-width call keeps whole waves of its own (planned
    // for 5/4, the Gemma-3-12B and Llama-3.1-8B layers lost 20-25 %).
    bool mixed = false;
    for (int k = 1; k < n_used; ++k) mixed |= key(plan.order[k]) != key(plan.order[0]);
    const int64_t plan_slots = mixed ? slots * 5 / 4 : slots;
    for (int v0 = 0; v0 < n_used;) {
        int v1 = v0 + 1;
        while (v1 < n_used && v1 - v0 < kvq::kAttnMaxViews && key(plan.order[v1]) == key(plan.order[v0])) ++v1;
        double bytes = 0;
        for (int k = v0; k < v1; ++k) {
            const kvq_view &v = views[plan.order[k]];
            bytes += (double)v.n_packed * packed_token_cost(head_dim, v.bits) +
                     (double)v.n_window * window_token_bytes(head_dim);
        }
        const int64_t share = std::max<int64_t>(
            1, (int64_t)std::llround((double)plan_slots * (bytes_all > 0 ? bytes / bytes_all : 1.0)));
        int64_t chunks = 0;
        plan_free(views, plan.order.data() + v0, v1 - v0, units, head_dim, share, plan.chunks, &chunks, big_item);
        if (chunks > INT32_MAX) return KVQ_ERR_UNSUPPORTED;
        AttnLaunch L{v0, v1, (int)chunks, key(plan.order[v0])};
        if (!size_launch(L)) return KVQ_ERR_UNSUPPORTED;
        plan.ring_bytes = std::max(plan.ring_bytes, L.ring_bytes);
        plan.smem = std::max(plan.smem, L.smem);
        plan.launches.push_back(L);
        v0 = v1;
    }
    // A sequence's unit combine holds at most kMaxChunksPerUnit chunks: trim
    // the largest parts of the sequences above that.
    const int32_t *sb = seq_begin;
    auto seq_first = [&](int s) { return sb ? sb[s] : s; };
    auto seq_end = [&](int s) { return sb ? sb[s + 1] : s + 1; };
    for (int s = 0; s < n_seqs; ++s) {
        for (;;) {
            int64_t total = 0;
            int32_t *big = nullptr;
            for (int i = seq_first(s); i < seq_end(s); ++i) {
                ViewChunks &c = plan.chunks[i];
                total += c.n_packed + c.n_window;
                if (!big || c.n_packed > *big) big = &c.n_packed;
                if (c.n_window > *big) big = &c.n_window;
            }
            if (total <= kvq::kMaxChunksPerUnit) break;
            *big = std::max<int32_t>(1, *big * 3 / 4);
        }
    }
    for (AttnLaunch &L : plan.launches) {
        int64_t chunks = 0;
        for (int k = L.v0; k < L.v1; ++k)
            chunks += plan.chunks[plan.order[k]].n_packed + plan.chunks[plan.order[k]].n_window;
        L.total_chunks = (int)chunks;
    }
    // partial slots: sequences in order, each one's views in order, each
    // view's chunks in order (the order the unit combine merges them in)
    plan.part_begin.assign(n_views, 0);
    plan.seq_part_begin.assign(n_seqs, 0);
    plan.seq_chunks.assign(n_seqs, 0);
    int64_t slot = 0;
    for (int s = 0; s < n_seqs; ++s) {
        plan.seq_part_begin[s] = (int32_t)slot;
        for (int i = seq_first(s); i < seq_end(s); ++i) {
            plan.part_begin[i] = (int32_t)slot;
            slot += plan.chunks[i].n_packed + plan.chunks[i].n_window;
        }
        plan.seq_chunks[s] = (int32_t)(slot - plan.seq_part_begin[s]);
        if (slot > INT32_MAX) return KVQ_ERR_UNSUPPORTED;
    }
    plan.n_slots = slot * units;
    size_t off = 256;  // bytes [0, 4): the device status word
    plan.counters_off = off;  // one arrival counter per (sequence, KV head, head block)
    off += ((size_t)n_seqs * units * 4 + 255) / 256 * 256;
    plan.zero_bytes = off;  // status word and counters: the part that must start at zero
    plan.partials_off = off;
    off += ((size_t)slot * units * kvq::kHeadsPerCta * (head_dim + 2) * 4 + 255) / 256 * 256;
    plan.total = off;
    return KVQ_OK;
}

// The attention grid of one launch: the kernel specialized for its width
// (or its score-only variant).
template <int NG, int BSEL, bool SCORE>
kvq_status launch_attn_width(size_t smem, const cudaLaunchConfig_t &cfg, const kvq::AttnParams &prm) {
    const kvq_status es = ensure_attn_smem<NG, BSEL, SCORE>(smem);
    if (es != KVQ_OK) return es;
    cudaError_t e;
    if constexpr (SCORE) e = cudaLaunchKernelEx(&cfg, kvq::score_attn_kernel<NG, BSEL>, prm);
    else e = cudaLaunchKernelEx(&cfg, kvq::decode_attn_kernel<NG, BSEL>, prm);
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

template <int NG, bool SCORE>
kvq_status launch_attn_grid(int bits, size_t smem, const cudaLaunchConfig_t &cfg, const kvq::AttnParams &prm) {
    switch (bits) {
        case 2: return launch_attn_width<NG, 2, SCORE>(smem, cfg, prm);
        case 3: return launch_attn_width<NG, 3, SCORE>(smem, cfg, prm);
        case 4: return launch_attn_width<NG, 4, SCORE>(smem, cfg, prm);
        default: return launch_attn_width<NG, 8, SCORE>(smem, cfg, prm);
    }
}

// scores != nullptr: the score-only grids (views without windows, one head
// block), each view's scores at scores + score_off[view]
template <int NG>
kvq_status launch_attn_ng(const AttnPlan &plan, const kvq_view *views, int32_t n_q_heads, int32_t n_kv_heads,
                          const void *q, float scale, float *out, uint8_t *ws, cudaStream_t st,
                          const int32_t *dep = nullptr, float *scores = nullptr, const int64_t *score_off = nullptr,
                          bool prefetch = true, int64_t n_scores = 0, const int32_t *const *gather = nullptr) {
    kvq::AttnParams prm;
    std::memset(&prm, 0, sizeof prm);
    prm.n_seqs = (int32_t)plan.seq_chunks.size();
    prm.n_part_slots = plan.n_slots;
    prm.n_scores = n_scores;
    prm.q = static_cast<const uint16_t *>(q);
    prm.out = out;
    prm.status = reinterpret_cast<uint32_t *>(ws);
    prm.timeout_ns = 2000000000ull;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.n_q_heads = n_q_heads;
    prm.n_kv_heads = n_kv_heads;
    prm.group = n_q_heads / n_kv_heads;
    prm.head_blocks = plan.head_blocks;

    prm.counters = reinterpret_cast<uint32_t *>(ws + plan.counters_off);
    prm.partials = reinterpret_cast<float *>(ws + plan.partials_off);
    for (const AttnLaunch &L : plan.launches) {
        prm.n_views = L.v1 - L.v0;
        // The first launch fills its first ring stages, then waits for the
        // preceding work (behind a fused append, the blocks holding appended
        // rows are copied only after that wait) and releases the next launch.
        // Later launches of the call start as soon as the one before has
        // released them, so all run concurrently on their own workspace
        // regions; each waits for its predecessor before it exits, so the
        // call's last grid completes after all of them.
        prm.chain = &L != &plan.launches[0] ? 1 : 0;
        prm.fused = (dep != nullptr && !prm.chain) ? 1 : 0;
        prm.prefetch = prefetch ? 1 : 0;
        int begin = 0;
        for (int k = L.v0; k < L.v1; ++k) {
            const int i = plan.order[k];
            const kvq_view &v = views[i];
            const ViewChunks &c = plan.chunks[i];
            kvq::AttnView &d = prm.views[k - L.v0];
            d.codes[0] = static_cast<const uint8_t *>(v.k_codes);
            d.codes[1] = static_cast<const uint8_t *>(v.v_codes);
            d.scalemin[0] = v.k_scalemin;
            d.scalemin[1] = v.v_scalemin;
            d.window[0] = static_cast<const uint16_t *>(v.k_window);
            d.window[1] = static_cast<const uint16_t *>(v.v_window);
            d.cap_packed = v.cap_packed;
            d.n_packed = (int32_t)v.n_packed;
            d.n_window = v.n_window;
            d.cap_window = v.cap_window;
            d.window_head = v.window_head;
            d.bits = v.n_packed > 0 ? v.bits : 4;
            d.n_chunks_packed = c.n_packed;
            d.n_chunks = c.n_packed + c.n_window;
            d.chunk_begin = begin;
            d.seq_index = plan.seq_of[i];
            d.part_begin = plan.part_begin[i];
            d.seq_part_begin = plan.seq_part_begin[plan.seq_of[i]];
            d.seq_chunks = plan.seq_chunks[plan.seq_of[i]];
            d.dep_step[0] = prm.fused ? dep[2 * i] : -1;
            d.dep_step[1] = prm.fused ? dep[2 * i + 1] : -1;
            d.score_off = scores ? score_off[i] : 0;
            d.gather = gather ? gather[i] : nullptr;
            begin += d.n_chunks;
        }
        // The grid carries a programmatic dependency on the preceding work in
        // the stream: before griddepcontrol.wait it only copies packed rows
        // and windows (prefetch), so its launch, CTA scheduling and first
        // copies overlap the predecessor's tail.
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof cfg);
        cfg.gridDim = dim3((unsigned)L.total_chunks, (unsigned)n_kv_heads, (unsigned)plan.head_blocks);
        cfg.blockDim = dim3(kvq::kAttnThreads);
        cfg.dynamicSmemBytes = L.smem;
        prm.ring_bytes = L.ring_bytes;
        cfg.stream = st;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        prm.scores = scores;
        const kvq_status es = scores ? launch_attn_grid<NG, true>(L.bits, L.smem, cfg, prm)
                                     : launch_attn_grid<NG, false>(L.bits, L.smem, cfg, prm);
        if (es != KVQ_OK) return es;
    }
    return KVQ_OK;
}

// ------------------------------------------------------------- append ---

kvq_status validate_append(const kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                           const void *k_new, const void *v_new) {
    if (!head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (n_kv_heads <= 0 || n_kv_heads > 65535) return KVQ_ERR_INVALID_ARG;
    const kvq_status vs = validate_views(views, n_views, false);
    if (vs != KVQ_OK) return vs;
    if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return KVQ_ERR_INVALID_ARG;
    // every view must be able to take the token
    for (int i = 0; i < n_views; ++i) {
        const kvq_view &v = views[i];
        const bool flush = v.cap_window == 0 || v.n_window == v.cap_window;
        if (flush) {
            if (!bits_supported(v.bits)) return KVQ_ERR_UNSUPPORTED;
            if (v.n_packed >= v.cap_packed) return KVQ_ERR_CAPACITY;
        }
    }
    return KVQ_OK;
}

// Enqueue the append grids (validated arguments); host counters unchanged.
kvq_status launch_append(const kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                         const void *k_new, const void *v_new, cudaStream_t st, bool early = false) {
    const int ng = head_dim / 64;
    for (int v0 = 0; v0 < n_views; v0 += kvq::kAppendMaxViews) {
        const int v1 = std::min<int>(n_views, v0 + kvq::kAppendMaxViews);
        kvq::AppendArgs a;
        std::memset(&a, 0, sizeof a);
        a.k_new = static_cast<const uint16_t *>(k_new) + (int64_t)v0 * n_kv_heads * head_dim;
        a.v_new = static_cast<const uint16_t *>(v_new) + (int64_t)v0 * n_kv_heads * head_dim;
        a.n_views = v1 - v0;
        a.n_kv_heads = n_kv_heads;
        a.early = early ? 1 : 0;
        for (int i = v0; i < v1; ++i) {
            const kvq_view &v = views[i];
            kvq::AppendView &d = a.views[i - v0];
            d.codes[0] = static_cast<uint8_t *>(v.k_codes);
            d.codes[1] = static_cast<uint8_t *>(v.v_codes);
            d.scalemin[0] = v.k_scalemin;
            d.scalemin[1] = v.v_scalemin;
            d.window[0] = static_cast<uint16_t *>(v.k_window);
            d.window[1] = static_cast<uint16_t *>(v.v_window);
            d.cap_packed = v.cap_packed;
            d.cap_window = v.cap_window;
            d.bits = v.bits;
            d.packed_row = v.n_packed;
            if (v.cap_window == 0) {
                d.flush = 1;
                d.slot = -1;
            } else if (v.n_window == v.cap_window) {
                d.flush = 1;
                d.slot = v.window_head;
            } else {
                d.flush = 0;
                d.slot = (v.window_head + v.n_window) % v.cap_window;
            }
        }
        // programmatic dependency: the kernel starts with griddepcontrol.wait
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof cfg);
        cfg.gridDim = dim3((unsigned)(v1 - v0), (unsigned)n_kv_heads, 2);
        cfg.blockDim = dim3(32);
        cfg.stream = st;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        cudaError_t e;
        switch (ng) {
            case 1: e = cudaLaunchKernelEx(&cfg, kvq::append_kernel<1>, a); break;
            case 2: e = cudaLaunchKernelEx(&cfg, kvq::append_kernel<2>, a); break;
            case 3: e = cudaLaunchKernelEx(&cfg, kvq::append_kernel<3>, a); break;
            default: e = cudaLaunchKernelEx(&cfg, kvq::append_kernel<4>, a); break;
        }
        if (e != cudaSuccess) return KVQ_ERR_CUDA;
    }
    return KVQ_OK;
}

// A view's counters after one append.
void advance_view(kvq_view &v) {
    if (v.cap_window == 0) {
        v.n_packed += 1;
    } else if (v.n_window == v.cap_window) {
        v.n_packed += 1;
        v.window_head = (v.window_head + 1) % v.cap_window;
    } else {
        v.n_window += 1;
    }
}

// ------------------------------------------------------------ CacheCard ---

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Byte layout of a card for these per-view (bits, n_packed, n_window).
struct CardLayout {
    size_t total = 0;
    std::vector<uint64_t> data_off, data_bytes;
    std::vector<std::vector<uint64_t>> sect;  // six section offsets per view
};

void card_layout(int32_t n_views, int32_t n_kv_heads, int32_t head_dim, const int32_t *bits, const int64_t *n_packed,
                 const int32_t *n_window, CardLayout &L) {
    const int ng = head_dim / 64;
    size_t off = align_up(sizeof(kvq::CardHeader) + sizeof(kvq::CardView) * (size_t)n_views, 256);
    L.data_off.resize(n_views);
    L.data_bytes.resize(n_views);
    L.sect.assign(n_views, std::vector<uint64_t>(6, 0));
    for (int i = 0; i < n_views; ++i) {
        const size_t codes = n_packed[i] > 0 ? (size_t)n_kv_heads * n_packed[i] * row_bytes(head_dim, bits[i]) : 0;
        const size_t sm = (size_t)n_kv_heads * (size_t)std::max<int64_t>(n_packed[i], 0) * ng * 8;
        const size_t win = (size_t)n_kv_heads * (size_t)std::max(n_window[i], 0) * head_dim * 2;
        const size_t sizes[6] = {codes, codes, sm, sm, win, win};
        L.data_off[i] = off;
        for (int k = 0; k < 6; ++k) {
            L.sect[i][k] = off;
            off = align_up(off + sizes[k], 16);
        }
        L.data_bytes[i] = off - L.data_off[i];
        off = align_up(off, 256);
    }
    L.total = off;
}

void card_layout_of_views(const kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                          CardLayout &L) {
    std::vector<int32_t> b(n_views), w(n_views);
    std::vector<int64_t> p(n_views);
    for (int i = 0; i < n_views; ++i) {
        b[i] = views[i].bits;
        p[i] = views[i].n_packed;
        w[i] = views[i].n_window;
    }
    card_layout(n_views, n_kv_heads, head_dim, b.data(), p.data(), w.data(), L);
}

kvq_status card_launch(bool pack, const kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                       const CardLayout &L, const kvq::CardHeader *header, const int64_t *position_offsets,
                       uint8_t *card, cudaStream_t st) {
    for (int v0 = 0; v0 < n_views; v0 += kvq::kCardMaxViews) {
        const int v1 = std::min<int>(n_views, v0 + kvq::kCardMaxViews);
        kvq::CardArgs a;
        std::memset(&a, 0, sizeof a);
        a.card = card;
        a.card_bytes = L.total;
        a.n_views = v1 - v0;
        a.n_kv_heads = n_kv_heads;
        a.head_dim = head_dim;
        a.write_header = (pack && v0 == 0) ? 1 : 0;
        if (header) a.header = *header;
        a.records_off = sizeof(kvq::CardHeader) + sizeof(kvq::CardView) * (uint64_t)v0;
        for (int i = v0; i < v1; ++i) {
            const kvq_view &v = views[i];
            kvq::CardSide &d = a.views[i - v0];
            d.codes[0] = static_cast<uint8_t *>(v.k_codes);
            d.codes[1] = static_cast<uint8_t *>(v.v_codes);
            d.scalemin[0] = v.k_scalemin;
            d.scalemin[1] = v.v_scalemin;
            d.window[0] = static_cast<uint16_t *>(v.k_window);
            d.window[1] = static_cast<uint16_t *>(v.v_window);
            d.cap_packed = v.cap_packed;
            d.n_packed = v.n_packed;
            d.cap_window = v.cap_window;
            d.n_window = v.n_window;
            d.window_head = pack ? v.window_head : 0;
            d.row_bytes = v.n_packed > 0 ? (int32_t)row_bytes(head_dim, v.bits) : 0;
            for (int k = 0; k < 6; ++k) d.sect_off[k] = L.sect[i][k];
            d.record.bits = (uint32_t)v.bits;
            d.record.n_window = (uint32_t)v.n_window;
            d.record.n_packed = (uint64_t)v.n_packed;
            d.record.position_offset = position_offsets ? position_offsets[i] : 0;
            d.record.data_offset = L.data_off[i];
            d.record.data_bytes = L.data_bytes[i];
            d.record.seq_len = (uint64_t)v.n_packed + (uint64_t)v.n_window;
        }
        // one CTA per piece of every (view, section), views in order
        uint64_t ctas = 0;
        for (int i = v0; i < v1; ++i) {
            const kvq_view &v = views[i];
            const int64_t rows[6] = {v.n_packed, v.n_packed, v.n_packed, v.n_packed, v.n_window, v.n_window};
            const int64_t row[6] = {a.views[i - v0].row_bytes, a.views[i - v0].row_bytes, (int64_t)(head_dim / 64) * 8,
                                    (int64_t)(head_dim / 64) * 8, (int64_t)head_dim * 2, (int64_t)head_dim * 2};
            for (int k = 0; k < 6; ++k) {
                a.entry_cta[(i - v0) * 6 + k] = (uint32_t)ctas;
                if (rows[k] > 0) ctas += (uint64_t)n_kv_heads * (uint64_t)kvq::card_pieces_per_head(rows[k], row[k]);
            }
        }
        if (ctas > (uint64_t)INT32_MAX) return KVQ_ERR_INVALID_ARG;
        a.entry_cta[(v1 - v0) * 6] = (uint32_t)ctas;
        const unsigned grid = (unsigned)std::max<uint64_t>(ctas, pack ? 1 : 0);
        if (grid == 0) continue;
        if (pack) kvq::card_kernel<true><<<grid, 256, 0, st>>>(a);
        else kvq::card_kernel<false><<<grid, 256, 0, st>>>(a);
        if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
    }
    return KVQ_OK;
}

// Validate a card held in host memory; fills its header and records.
kvq_status card_parse(const void *card_host, size_t card_bytes, kvq::CardHeader &h,
                      std::vector<kvq::CardView> &recs) {
    if (!card_host || card_bytes < sizeof(kvq::CardHeader)) return KVQ_ERR_INVALID_ARG;
    std::memcpy(&h, card_host, sizeof h);
    if (std::memcmp(h.magic, "KVQCARD1", 8) != 0 || h.version != kvq::kCardVersion) return KVQ_ERR_INVALID_ARG;
    if (!head_dim_supported((int32_t)h.head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (h.n_views == 0 || h.n_views > (1u << 24) || h.n_kv_heads == 0 || h.n_kv_heads > 65535)
        return KVQ_ERR_INVALID_ARG;
    const size_t rec_end = sizeof(kvq::CardHeader) + sizeof(kvq::CardView) * (size_t)h.n_views;
    if (h.total_bytes > card_bytes || rec_end > h.total_bytes) return KVQ_ERR_INVALID_ARG;
    recs.resize(h.n_views);
    std::memcpy(recs.data(), static_cast<const uint8_t *>(card_host) + sizeof(kvq::CardHeader),
                sizeof(kvq::CardView) * (size_t)h.n_views);
    std::vector<int32_t> b(h.n_views), w(h.n_views);
    std::vector<int64_t> p(h.n_views);
    for (uint32_t i = 0; i < h.n_views; ++i) {
        const kvq::CardView &r = recs[i];
        if (r.n_packed > (uint64_t)INT32_MAX || r.n_window > (uint32_t)INT32_MAX) return KVQ_ERR_INVALID_ARG;
        if (r.n_packed > 0 && !bits_supported((int32_t)r.bits)) return KVQ_ERR_UNSUPPORTED;
        if (r.seq_len != r.n_packed + r.n_window) return KVQ_ERR_INVALID_ARG;
        b[i] = (int32_t)r.bits;
        p[i] = (int64_t)r.n_packed;
        w[i] = (int32_t)r.n_window;
    }
    // the data must sit exactly where this version's layout puts it
    CardLayout L;
    card_layout((int32_t)h.n_views, (int32_t)h.n_kv_heads, (int32_t)h.head_dim, b.data(), p.data(), w.data(), L);
    if (L.total != h.total_bytes) return KVQ_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < h.n_views; ++i)
        if (recs[i].data_offset != L.data_off[i] || recs[i].data_bytes != L.data_bytes[i]) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

// ------------------------------------------- fixed scratch (no allocation) ---

// Scratch of kvq_decode_attn_noalloc: one array per device, laid out like a
// kvq_decode_attn workspace (status word at byte 0, partials from byte 256).
static __device__ __align__(256) uint8_t g_noalloc_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device.  It is looked up on
// every call (a host-side query of the runtime, no device work), so a reset
// or re-created primary context never leaves a stale address behind; the
// first lookup on a device also loads the library's device code there.
kvq_status noalloc_scratch(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p || !aligned(p, 256)) {
        (void)cudaGetLastError();
        return KVQ_ERR_CUDA;
    }
    *out = p;
    return KVQ_OK;
}

// The attention (or score) grids of a plan, for the view's head_dim; dep and
// scores/score_off as launch_attn_ng.
kvq_status launch_attn(const AttnPlan &plan, const kvq_view *views, int32_t n_q_heads, int32_t n_kv_heads,
                       int32_t head_dim, const void *q, float scale, float *out, uint8_t *ws, cudaStream_t st,
                       const int32_t *dep = nullptr, float *scores = nullptr, const int64_t *score_off = nullptr,
                       bool prefetch = true, int64_t n_scores = 0, const int32_t *const *gather = nullptr) {
    switch (head_dim / 64) {
        case 1: return launch_attn_ng<1>(plan, views, n_q_heads, n_kv_heads, q, scale, out, ws, st, dep, scores, score_off, prefetch, n_scores, gather);
        case 2: return launch_attn_ng<2>(plan, views, n_q_heads, n_kv_heads, q, scale, out, ws, st, dep, scores, score_off, prefetch, n_scores, gather);
        case 3: return launch_attn_ng<3>(plan, views, n_q_heads, n_kv_heads, q, scale, out, ws, st, dep, scores, score_off, prefetch, n_scores, gather);
        default: return launch_attn_ng<4>(plan, views, n_q_heads, n_kv_heads, q, scale, out, ws, st, dep, scores, score_off, prefetch, n_scores, gather);
    }
}

// ------------------------------------------------------ sparse decode ---

// Top-K sparse decode: every (view, KV head) becomes a view of its own (one
// KV head, the group's query heads): its packed part is the K selected rows,
// read in place through the selection list (gather), or every packed row
// when the view has no more than K; its window is the view's bf16 window for
// that head.  Workspace: the attention's region first (its zero part stays
// at offset 0 from call to call), then scores and selections.
struct SparsePlan {
    std::vector<kvq_view> compact;     // [n_views * H_kv]: per (view, KV head)
    std::vector<int64_t> score_off;    // per view, floats from scores_off; -1: no scoring
    AttnPlan attn;
    size_t scores_off = 0, sel_off = 0, total = 0;
};

kvq_status plan_sparse(const kvq_view *views, int32_t n_views, int32_t n_q_heads, int32_t n_kv_heads,
                       int32_t head_dim, int32_t top_k, SparsePlan &sp) {
    sp = SparsePlan();
    if (!head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads || n_kv_heads > 65535)
        return KVQ_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > (1 << 24)) return KVQ_ERR_INVALID_ARG;
    const kvq_status vs = validate_views(views, n_views, true);
    if (vs != KVQ_OK) return vs;
    const int ng = head_dim / 64, group = n_q_heads / n_kv_heads;
    sp.score_off.assign(n_views, -1);
    int64_t n_scores = 0;
    for (int i = 0; i < n_views; ++i) {
        const kvq_view &v = views[i];
        if (v.n_packed <= top_k) continue;
        sp.score_off[i] = n_scores;
        n_scores += (int64_t)n_kv_heads * v.n_packed;
    }
    sp.compact.assign((size_t)n_views * n_kv_heads, kvq_view{});
    for (int i = 0; i < n_views; ++i) {
        const kvq_view &v = views[i];
        const int64_t rb = row_bytes(head_dim, v.bits);
        for (int hk = 0; hk < n_kv_heads; ++hk) {
            kvq_view &c = sp.compact[(size_t)i * n_kv_heads + hk];
            c.bits = v.bits;
            c.n_window = v.n_window;
            c.cap_window = v.cap_window;
            c.window_head = v.window_head;
            if (v.cap_window > 0) {
                const size_t w = (size_t)hk * v.cap_window * head_dim * 2;
                c.k_window = static_cast<uint8_t *>(v.k_window) + w;
                c.v_window = static_cast<uint8_t *>(v.v_window) + w;
            }
            // the head's own rows, every one or the selected ones
            c.n_packed = std::min<int64_t>(v.n_packed, top_k);
            c.cap_packed = v.cap_packed;
            if (v.cap_packed > 0) {
                c.k_codes = static_cast<uint8_t *>(v.k_codes) + (size_t)hk * v.cap_packed * rb;
                c.v_codes = static_cast<uint8_t *>(v.v_codes) + (size_t)hk * v.cap_packed * rb;
                c.k_scalemin = v.k_scalemin + (size_t)hk * v.cap_packed * ng * 2;
                c.v_scalemin = v.v_scalemin + (size_t)hk * v.cap_packed * ng * 2;
            }
        }
    }
    const kvq_status ps = plan_attn(sp.compact.data(), n_views * n_kv_heads, nullptr, 0, group, 1, head_dim, sp.attn);
    if (ps != KVQ_OK) return ps;
    size_t off = align_up(sp.attn.total, 256);
    sp.scores_off = off;
    off = align_up(off + (size_t)n_scores * 4, 256);
    sp.sel_off = off;
    sp.total = align_up(off + (size_t)n_views * n_kv_heads * top_k * 4, 256);
    return KVQ_OK;
}

// A launch with a programmatic dependency on the preceding work in the stream
// (the kernel starts with griddepcontrol.wait).
template <typename Args>
kvq_status launch_pdl(void (*kernel)(Args), dim3 grid, unsigned block, size_t smem, cudaStream_t st,
                      const Args &a) {
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

// The same with thread-block clusters of `cluster` CTAs along x.
template <typename Args>
kvq_status launch_pdl_cluster(void (*kernel)(Args), dim3 grid, unsigned block, unsigned cluster, size_t smem,
                              cudaStream_t st, const Args &a) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, a) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

template <int NG, int B>
kvq_status launch_score_grid(const kvq::ScoreArgs &a, unsigned ctas, size_t smem, cudaStream_t st) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kvq::score_kernel<NG, B>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess) {
        (void)cudaGetLastError();
        return KVQ_ERR_UNSUPPORTED;
    }
    return launch_pdl(kvq::score_kernel<NG, B>, dim3(ctas), kvq::kScoreTok, smem, st, a);
}

template <int NG>
kvq_status launch_score_ng(int bits, const kvq::ScoreArgs &a, unsigned ctas, size_t smem, cudaStream_t st) {
    switch (bits) {
        case 2: return launch_score_grid<NG, 2>(a, ctas, smem, st);
        case 3: return launch_score_grid<NG, 3>(a, ctas, smem, st);
        case 4: return launch_score_grid<NG, 4>(a, ctas, smem, st);
        default: return launch_score_grid<NG, 8>(a, ctas, smem, st);
    }
}

kvq_status launch_sparse(const SparsePlan &sp, const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                         int32_t n_kv_heads, int32_t head_dim, const void *q, float scale, int32_t top_k, float *out,
                         int32_t *sel, uint8_t *ws, cudaStream_t st) {
    const int ng = head_dim / 64, group = n_q_heads / n_kv_heads;
    float *scores = reinterpret_cast<float *>(ws + sp.scores_off);
    // 1. scores of the views with more than K packed tokens.  A group of at
    // most 8 query heads: the attention grid's QK path (tensor cores) over the
    // packed parts, scores in base-2 logit units (the order is that of the
    // logits); wider groups: the SIMT score kernel.
    std::vector<int> scored;
    for (int i = 0; i < n_views; ++i)
        if (sp.score_off[i] >= 0) scored.push_back(i);
    if (group <= kvq::kHeadsPerCta && !scored.empty()) {
        // every view its own sequence (q row = view index); views not scored
        // are left empty, windows are left out
        std::vector<kvq_view> packed(views, views + n_views);
        std::vector<int32_t> seq(n_views + 1);
        for (int i = 0; i < n_views; ++i) {
            kvq_view &v = packed[i];
            v.n_window = v.cap_window = v.window_head = 0;
            v.k_window = v.v_window = nullptr;
            if (sp.score_off[i] < 0) v.n_packed = 0;
            seq[i] = i;
        }
        seq[n_views] = n_views;
        AttnPlan splan;
        // (a score item reads the K half of the bytes the item model counts:
        // twice the attention's largest item)
        const kvq_status ps = plan_attn(packed.data(), n_views, seq.data(), n_views, n_q_heads, n_kv_heads, head_dim,
                                        splan, true, 2 * kBigItem);
        if (ps != KVQ_OK) return ps;
        const kvq_status es = launch_attn(splan, packed.data(), n_q_heads, n_kv_heads, head_dim, q, scale, nullptr,
                                          ws, st, nullptr, scores, sp.score_off.data(), true,
                                          (int64_t)((sp.sel_off - sp.scores_off) / sizeof(float)));
        if (es != KVQ_OK) return es;
        scored.clear();  // nothing left for the SIMT kernel
    }
    std::stable_sort(scored.begin(), scored.end(), [&](int x, int y) { return views[x].bits < views[y].bits; });
    const size_t smem = (size_t)group * head_dim * 4 + (size_t)group * ng * 4;
    if (smem > 227 * 1024) return KVQ_ERR_UNSUPPORTED;
    for (size_t v0 = 0; v0 < scored.size();) {
        size_t v1 = v0 + 1;
        while (v1 < scored.size() && v1 - v0 < (size_t)kvq::kSparseMaxViews &&
               views[scored[v1]].bits == views[scored[v0]].bits)
            ++v1;
        kvq::ScoreArgs a;
        std::memset(&a, 0, sizeof a);
        a.q = static_cast<const uint16_t *>(q);
        a.scores = scores;
        a.n_scores = (int64_t)((sp.sel_off - sp.scores_off) / sizeof(float));
        a.scale = scale;
        a.n_views = (int)(v1 - v0);
        a.n_q_heads = n_q_heads;
        a.group = group;
        int64_t ctas = 0;
        for (size_t k = v0; k < v1; ++k) {
            const int i = scored[k];
            const kvq_view &v = views[i];
            kvq::ScoreView &d = a.views[k - v0];
            d.k_codes = static_cast<const uint8_t *>(v.k_codes);
            d.k_sm = v.k_scalemin;
            d.cap_packed = v.cap_packed;
            d.score_off = sp.score_off[i];
            d.n_packed = (int32_t)v.n_packed;
            d.blocks = (int32_t)((v.n_packed + kvq::kScoreTok * kvq::kScoreBlocks - 1) /
                                 (kvq::kScoreTok * kvq::kScoreBlocks));
            d.cta_begin = (int32_t)ctas;
            d.q_row = i;
            ctas += (int64_t)n_kv_heads * d.blocks;
        }
        if (ctas > INT32_MAX) return KVQ_ERR_UNSUPPORTED;
        kvq_status es;
        switch (ng) {
            case 1: es = launch_score_ng<1>(views[scored[v0]].bits, a, (unsigned)ctas, smem, st); break;
            case 2: es = launch_score_ng<2>(views[scored[v0]].bits, a, (unsigned)ctas, smem, st); break;
            case 3: es = launch_score_ng<3>(views[scored[v0]].bits, a, (unsigned)ctas, smem, st); break;
            default: es = launch_score_ng<4>(views[scored[v0]].bits, a, (unsigned)ctas, smem, st); break;
        }
        if (es != KVQ_OK) return es;
        v0 = v1;
    }
    // 2. selections of every view (ascending row indices): views of up to
    // kSelFastMax packed tokens on select_cluster_kernel, longer ones on
    // select_kernel (keys staged in shared memory or read from the scores)
    for (int large = 0; large < 2; ++large) {
        std::vector<int> idx;
        for (int i = 0; i < n_views; ++i)
            if ((views[i].n_packed > kvq::kSelFastMax) == (large != 0)) idx.push_back(i);
        for (size_t v0 = 0; v0 < idx.size(); v0 += kvq::kSparseMaxViews) {
            const size_t v1 = std::min(idx.size(), v0 + kvq::kSparseMaxViews);
            kvq::SelectArgs a;
            std::memset(&a, 0, sizeof a);
            a.scores = scores;
            a.sel = sel;
            a.n_scores = (int64_t)((sp.sel_off - sp.scores_off) / sizeof(float));
            a.n_sel_rows = n_views;
            a.top_k = top_k;
            a.n_kv_heads = n_kv_heads;
            size_t smem = 0;
            int64_t max_n = 0;
            for (size_t k = v0; k < v1; ++k) {
                const int i = idx[k];
                const kvq_view &v = views[i];
                kvq::SelectView &d = a.views[k - v0];
                d.score_off = std::max<int64_t>(sp.score_off[i], 0);
                d.n_packed = (int32_t)v.n_packed;
                d.out_row = i;
                if (sp.score_off[i] < 0) continue;
                max_n = std::max<int64_t>(max_n, v.n_packed);
                d.staged = v.n_packed <= kvq::kSelectStageMax ? 1 : 0;
                if (d.staged) smem = std::max(smem, (size_t)v.n_packed * 4);
            }
            kvq_status es;
            if (!large) {
                // `cl` CTAs per (view, KV head), a thread-block cluster when
                // more than one: the fewest that leave a lane at most 32 keys
                // (KVQ_SELECT_CLUSTER = 2 or 4 asks for more)
                constexpr int64_t T = kvq::kSelClusterThreads;
                int cl = 1;
                const int forced = env_int("KVQ_SELECT_CLUSTER", 0);
                if (forced == 2 || forced == 4) cl = forced;
                while (cl < kvq::kSelMaxCluster && max_n > cl * T * 32) cl *= 2;
                int64_t cap = 0;  // keys of the largest slice: T * keys per lane
                for (size_t k = v0; k < v1; ++k)
                    if (sp.score_off[idx[k]] >= 0)
                        cap = std::max(cap, T * ((views[idx[k]].n_packed + cl * T - 1) / (cl * T)));
                a.key_cap = (int32_t)cap;
                const size_t keys = (size_t)cap * 6;  // keys and first-pass bins
                const dim3 grid((unsigned)((v1 - v0) * cl), (unsigned)n_kv_heads);
                auto kernel = cl > 1 ? kvq::select_cluster_kernel<kvq::kSelClusterThreads, true>
                                     : kvq::select_cluster_kernel<kvq::kSelClusterThreads, false>;
                // (the opt-in above 48 KiB counts the kernel's ~25 KiB of
                // static shared memory too)
                if (keys + 26 * 1024 > 48 * 1024 &&
                    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)keys) !=
                        cudaSuccess) {
                    (void)cudaGetLastError();
                    return KVQ_ERR_CUDA;
                }
                es = cl > 1 ? launch_pdl_cluster(kernel, grid, kvq::kSelClusterThreads, (unsigned)cl, keys, st, a)
                            : launch_pdl(kernel, grid, kvq::kSelClusterThreads, keys, st, a);
            } else {
                if (smem + 2 * 1024 > 48 * 1024 &&  // (with its 1 KiB of static shared memory)
                    cudaFuncSetAttribute(kvq::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                        cudaSuccess) {
                    (void)cudaGetLastError();
                    return KVQ_ERR_CUDA;
                }
                const dim3 grid((unsigned)(v1 - v0), (unsigned)n_kv_heads);
                es = launch_pdl(kvq::select_kernel, grid, kvq::kSelectThreads, smem, st, a);
            }
            if (es != KVQ_OK) return es;
        }
    }
    // 3. attention over the per-head views: one KV head each, the group's
    // query heads; a view with more than K packed rows reads the selected
    // ones through its selection list, which the select grid writes, so no
    // copy starts before the dependency wait
    std::vector<const int32_t *> gather((size_t)n_views * n_kv_heads, nullptr);
    for (int i = 0; i < n_views; ++i)
        if (sp.score_off[i] >= 0)
            for (int hk = 0; hk < n_kv_heads; ++hk)
                gather[(size_t)i * n_kv_heads + hk] = sel + ((int64_t)i * n_kv_heads + hk) * top_k;
    return launch_attn(sp.attn, sp.compact.data(), group, 1, head_dim, q, scale, out, ws, st, nullptr, nullptr,
                       nullptr, false, 0, gather.data());
}

}  // namespace

// ================================================================ C ABI ===

KVQ_API const char *kvq_status_string(int32_t status) {
    switch (status) {
        case KVQ_OK: return "KVQ_OK";
        case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
        case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
        case KVQ_ERR_CAPACITY: return "KVQ_ERR_CAPACITY";
        case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
        default: return "unknown status";
    }
}

KVQ_API int32_t kvq_abi_version(void) { return kAbiVersion; }

KVQ_API int32_t kvq_debug_build(void) {
#ifdef KVQ_DEBUG
    return 1;
#else
    return 0;
#endif
}

KVQ_API kvq_status kvq_debug_flags(uint32_t *flags, int32_t clear, void *stream) {
#ifdef KVQ_DEBUG
    if (!flags || !aligned(flags, 4)) return KVQ_ERR_INVALID_ARG;
    void *word = nullptr;
    if (cudaGetSymbolAddress(&word, kvq::g_debug_flags) != cudaSuccess || !word) {
        (void)cudaGetLastError();
        return KVQ_ERR_CUDA;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(flags, word, sizeof(uint32_t), cudaMemcpyDefault, st) != cudaSuccess ||
        (clear && cudaMemsetAsync(word, 0, sizeof(uint32_t), st) != cudaSuccess)) {
        (void)cudaGetLastError();
        return KVQ_ERR_CUDA;
    }
    return KVQ_OK;
#else
    (void)flags;
    (void)clear;
    (void)stream;
    return KVQ_ERR_UNSUPPORTED;
#endif
}

KVQ_API kvq_status kvq_quantize(const void *x, int64_t x_head_stride, int64_t x_tok_stride, int32_t n_heads,
                                int64_t n_tokens, int32_t head_dim, int32_t bits, void *codes, float *scalemin,
                                int64_t out_head_cap, void *stream) {
    return codec(true, x, x_head_stride, x_tok_stride, n_heads, n_tokens, head_dim, bits, codes, scalemin,
                 out_head_cap, stream);
}

KVQ_API kvq_status kvq_dequantize(const void *codes, const float *scalemin, int64_t in_head_cap, int32_t n_heads,
                                  int64_t n_tokens, int32_t head_dim, int32_t bits, void *y, int64_t y_head_stride,
                                  int64_t y_tok_stride, void *stream) {
    return codec(false, y, y_head_stride, y_tok_stride, n_heads, n_tokens, head_dim, bits, codes, scalemin,
                 in_head_cap, stream);
}

KVQ_API kvq_status kvq_append(kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                              const void *k_new, const void *v_new, void *stream) {
    const kvq_status vs = validate_append(views, n_views, n_kv_heads, head_dim, k_new, v_new);
    if (vs != KVQ_OK) return vs;
    const kvq_status ls =
        launch_append(views, n_views, n_kv_heads, head_dim, k_new, v_new, static_cast<cudaStream_t>(stream));
    if (ls != KVQ_OK) return ls;
    // the launch is enqueued: advance the host-side counters
    for (int i = 0; i < n_views; ++i) advance_view(views[i]);
    return KVQ_OK;
}

KVQ_API size_t kvq_decode_attn_workspace_size(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                              int32_t n_kv_heads, int32_t head_dim) {
    AttnPlan plan;
    if (plan_attn(views, n_views, nullptr, 0, n_q_heads, n_kv_heads, head_dim, plan) != KVQ_OK) return 0;
    return plan.total;
}

KVQ_API kvq_status kvq_decode_attn(const kvq_view *views, int32_t n_views, int32_t n_q_heads, int32_t n_kv_heads,
                                   int32_t head_dim, const void *q, float softmax_scale, float *out, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    AttnPlan plan;
    const kvq_status ps = plan_attn(views, n_views, nullptr, 0, n_q_heads, n_kv_heads, head_dim, plan);
    if (ps != KVQ_OK) return ps;
    if (!q || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (workspace_bytes < plan.total) return KVQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    return launch_attn(plan, views, n_q_heads, n_kv_heads, head_dim, q, softmax_scale, out, ws, st);
}

KVQ_API size_t kvq_decode_attn_seq_workspace_size(const kvq_view *views, int32_t n_views, const int32_t *seq_begin,
                                                  int32_t n_seqs, int32_t n_q_heads, int32_t n_kv_heads,
                                                  int32_t head_dim) {
    if (!seq_begin) return 0;
    AttnPlan plan;
    if (plan_attn(views, n_views, seq_begin, n_seqs, n_q_heads, n_kv_heads, head_dim, plan) != KVQ_OK) return 0;
    return plan.total;
}

KVQ_API kvq_status kvq_decode_attn_seq(const kvq_view *views, int32_t n_views, const int32_t *seq_begin,
                                       int32_t n_seqs, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                       const void *q, float softmax_scale, float *out, void *workspace,
                                       size_t workspace_bytes, void *stream) {
    if (!seq_begin) return KVQ_ERR_INVALID_ARG;
    AttnPlan plan;
    const kvq_status ps = plan_attn(views, n_views, seq_begin, n_seqs, n_q_heads, n_kv_heads, head_dim, plan);
    if (ps != KVQ_OK) return ps;
    if (!q || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (workspace_bytes < plan.total) return KVQ_ERR_INVALID_ARG;
    return launch_attn(plan, views, n_q_heads, n_kv_heads, head_dim, q, softmax_scale, out,
                       static_cast<uint8_t *>(workspace), static_cast<cudaStream_t>(stream));
}

KVQ_API kvq_status kvq_decode_attn_noalloc(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                           int32_t n_kv_heads, int32_t head_dim, const void *q, float softmax_scale,
                                           float *out, void *stream) {
    AttnPlan plan;
    const kvq_status ps = plan_attn(views, n_views, nullptr, 0, n_q_heads, n_kv_heads, head_dim, plan);
    if (ps != KVQ_OK) return ps;
    if (!q || !out) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16)) return KVQ_ERR_INVALID_ARG;
    if (plan.total > (size_t)KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_CAPACITY;
    void *scratch = nullptr;
    const kvq_status ss = noalloc_scratch(&scratch);
    if (ss != KVQ_OK) return ss;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word and the arrival counters must start at zero; the
    // partials are written before they are read
    if (cudaMemsetAsync(scratch, 0, plan.zero_bytes, st) != cudaSuccess) return KVQ_ERR_CUDA;
    return launch_attn(plan, views, n_q_heads, n_kv_heads, head_dim, q, softmax_scale, out,
                       static_cast<uint8_t *>(scratch), st);
}

KVQ_API kvq_status kvq_decode_attn_noalloc_status(uint32_t *status, void *stream) {
    if (!status || !aligned(status, 4)) return KVQ_ERR_INVALID_ARG;
    void *scratch = nullptr;
    const kvq_status ss = noalloc_scratch(&scratch);
    if (ss != KVQ_OK) return ss;
    // stream-ordered: the word as the last call enqueued before this one on
    // the stream left it
    if (cudaMemcpyAsync(status, scratch, sizeof(uint32_t), cudaMemcpyDefault, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return KVQ_ERR_CUDA;
    }
    return KVQ_OK;
}

KVQ_API kvq_status kvq_append_decode_attn(kvq_view *views, int32_t n_views, int32_t n_q_heads, int32_t n_kv_heads,
                                          int32_t head_dim, const void *k_new, const void *v_new, const void *q,
                                          float softmax_scale, float *out, void *workspace, size_t workspace_bytes,
                                          void *stream) {
    const kvq_status vs = validate_append(views, n_views, n_kv_heads, head_dim, k_new, v_new);
    if (vs != KVQ_OK) return vs;
    // plan the attention over the views as they will be after the append
    std::vector<kvq_view> post(views, views + n_views);
    for (kvq_view &v : post) advance_view(v);
    AttnPlan plan;
    const kvq_status ps = plan_attn(post.data(), n_views, nullptr, 0, n_q_heads, n_kv_heads, head_dim, plan);
    if (ps != KVQ_OK) return ps;
    if (!q || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (workspace_bytes < plan.total) return KVQ_ERR_INVALID_ARG;
    // the steps whose rows the append writes: the flushed packed row, the new window token
    std::vector<int32_t> dep(2 * (size_t)n_views);
    for (int i = 0; i < n_views; ++i) {
        const kvq_view &a = views[i], &b = post[i];
        const bool flush = a.cap_window == 0 || a.n_window == a.cap_window;
        dep[2 * i] = flush ? (int32_t)((b.n_packed - 1) / (2 * kvq::kTile)) : -1;
        dep[2 * i + 1] = a.cap_window > 0 ? (b.n_window - 1) / kvq::kTile : -1;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const kvq_status ls = launch_append(views, n_views, n_kv_heads, head_dim, k_new, v_new, st, true);
    if (ls != KVQ_OK) return ls;
    for (int i = 0; i < n_views; ++i) views[i] = post[i];  // enqueued: advance the counters
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    return launch_attn(plan, post.data(), n_q_heads, n_kv_heads, head_dim, q, softmax_scale, out, ws, st, dep.data());
}

KVQ_API size_t kvq_sparse_decode_attn_workspace_size(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                                     int32_t n_kv_heads, int32_t head_dim, int32_t top_k) {
    SparsePlan sp;
    if (plan_sparse(views, n_views, n_q_heads, n_kv_heads, head_dim, top_k, sp) != KVQ_OK) return 0;
    return sp.total;
}

KVQ_API kvq_status kvq_sparse_decode_attn(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                          int32_t n_kv_heads, int32_t head_dim, const void *q, float softmax_scale,
                                          int32_t top_k, float *out, int32_t *selected, void *workspace,
                                          size_t workspace_bytes, void *stream) {
    SparsePlan sp;
    const kvq_status ps = plan_sparse(views, n_views, n_q_heads, n_kv_heads, head_dim, top_k, sp);
    if (ps != KVQ_OK) return ps;
    if (!q || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
    if (selected && !aligned(selected, 4)) return KVQ_ERR_INVALID_ARG;
    if (workspace_bytes < sp.total) return KVQ_ERR_INVALID_ARG;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *sel = selected ? selected : reinterpret_cast<int32_t *>(ws + sp.sel_off);
    return launch_sparse(sp, views, n_views, n_q_heads, n_kv_heads, head_dim, q, softmax_scale, top_k, out, sel, ws,
                         static_cast<cudaStream_t>(stream));
}

KVQ_API kvq_status kvq_width_sensitivity(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                         int32_t n_kv_heads, int32_t head_dim, const void *q, float softmax_scale,
                                         float *sens, void *stream) {
    if (!head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (n_kv_heads <= 0 || n_q_heads <= 0 || n_q_heads % n_kv_heads || n_kv_heads > 65535)
        return KVQ_ERR_INVALID_ARG;
    const kvq_status vs = validate_views(views, n_views, false);
    if (vs != KVQ_OK) return vs;
    if (!q || !sens || !aligned(q, 16) || !aligned(sens, 4)) return KVQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int v0 = 0; v0 < n_views; v0 += kvq::kSensMaxViews) {
        const int v1 = std::min<int>(n_views, v0 + kvq::kSensMaxViews);
        kvq::SensArgs a;
        std::memset(&a, 0, sizeof a);
        a.q = static_cast<const uint16_t *>(q);
        a.sens = sens;
        a.n_rows = n_views;
        a.scale = softmax_scale;
        a.n_q_heads = n_q_heads;
        a.n_kv_heads = n_kv_heads;
        a.group = n_q_heads / n_kv_heads;
        for (int i = v0; i < v1; ++i) {
            kvq::SensView &d = a.views[i - v0];
            d.k_window = static_cast<const uint16_t *>(views[i].k_window);
            d.v_window = static_cast<const uint16_t *>(views[i].v_window);
            d.cap_window = views[i].cap_window;
            d.n_window = views[i].n_window;
            d.window_head = views[i].window_head;
            d.row = i;
        }
        const unsigned grid = (unsigned)(v1 - v0);
        switch (head_dim / 64) {
            case 1: kvq::sensitivity_kernel<1><<<grid, 32 * kvq::kSensWarps, 0, st>>>(a); break;
            case 2: kvq::sensitivity_kernel<2><<<grid, 32 * kvq::kSensWarps, 0, st>>>(a); break;
            case 3: kvq::sensitivity_kernel<3><<<grid, 32 * kvq::kSensWarps, 0, st>>>(a); break;
            default: kvq::sensitivity_kernel<4><<<grid, 32 * kvq::kSensWarps, 0, st>>>(a); break;
        }
        if (cudaGetLastError() != cudaSuccess) return KVQ_ERR_CUDA;
    }
    return KVQ_OK;
}

KVQ_API kvq_status kvq_allocate_widths(const float *sens, const int64_t *capacity, int32_t n_views, int32_t n_kv_heads,
                                       int32_t head_dim, uint64_t budget_bytes, int32_t units, int32_t *bits,
                                       double *total_error) {
    if (!head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (!sens || !capacity || !bits || n_views <= 0 || n_kv_heads <= 0 || n_kv_heads > 65535) return KVQ_ERR_INVALID_ARG;
    if (units < 1 || units > (1 << 20)) return KVQ_ERR_INVALID_ARG;
    static const int kWidths[4] = {8, 4, 3, 2};  // equal totals keep the earlier (wider) choice
    for (int i = 0; i < n_views; ++i)
        if (capacity[i] < 0 || capacity[i] > ((int64_t)1 << 40) || !(sens[i] >= 0.f) || std::isinf(sens[i]))
            return KVQ_ERR_INVALID_ARG;
    // ceil(budget / units) without forming budget + units - 1, which wraps
    // for budgets near 2^64
    const uint64_t unit = budget_bytes > 0 ? budget_bytes / (uint64_t)units + (budget_bytes % (uint64_t)units != 0)
                                           : 1;
    const size_t cap_units = (size_t)(budget_bytes / unit);
    // the back-pointers take one byte per (view, unit): at most 1 GiB
    if ((uint64_t)n_views * (uint64_t)(cap_units + 1) > (1ull << 30)) return KVQ_ERR_UNSUPPORTED;
    const double inf = std::numeric_limits<double>::infinity();
    std::vector<double> best(cap_units + 1, inf), next(cap_units + 1);
    std::vector<int8_t> choice((size_t)n_views * (cap_units + 1), 0);
    std::vector<uint64_t> cost((size_t)n_views * 4);
    best[0] = 0.0;
    for (int i = 0; i < n_views; ++i) {
        std::fill(next.begin(), next.end(), inf);
        int8_t *pick = choice.data() + (size_t)i * (cap_units + 1);
        for (int j = 0; j < 4; ++j) {
            const int b = kWidths[j];
            // up to 2^40 * 2 * 65535 * 288 bytes: wider than 64 bits, so in
            // 128-bit arithmetic; a cost above the whole budget is simply not
            // affordable (cap_units + 1 units)
            const unsigned __int128 bytes = (unsigned __int128)capacity[i] * 2u * (unsigned __int128)n_kv_heads *
                                            (unsigned __int128)(head_dim * b / 8 + head_dim / 64 * 8);
            const unsigned __int128 c128 = (bytes + unit - 1) / unit;
            const uint64_t c = c128 > (unsigned __int128)cap_units ? (uint64_t)cap_units + 1 : (uint64_t)c128;
            cost[(size_t)i * 4 + j] = c;
            const double err = (double)sens[i] / (double)((1 << b) - 1);
            for (size_t u = (size_t)std::min<uint64_t>(c, cap_units + 1); u <= cap_units; ++u) {
                const double cand = best[u - c] + err;
                if (cand < next[u]) {
                    next[u] = cand;
                    pick[u] = (int8_t)j;
                }
            }
        }
        best.swap(next);
    }
    size_t u = 0;
    for (size_t k = 1; k <= cap_units; ++k)
        if (best[k] < best[u]) u = k;
    if (best[u] == inf) return KVQ_ERR_CAPACITY;
    if (total_error) *total_error = best[u];
    for (int i = n_views - 1; i >= 0; --i) {
        const int j = choice[(size_t)i * (cap_units + 1) + u];
        bits[i] = kWidths[j];
        u -= (size_t)cost[(size_t)i * 4 + j];
    }
    return KVQ_OK;
}

KVQ_API size_t kvq_card_bytes(const kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim) {
    if (!head_dim_supported(head_dim) || n_kv_heads <= 0 || n_kv_heads > 65535) return 0;
    if (validate_views(views, n_views, false) != KVQ_OK) return 0;
    CardLayout L;
    card_layout_of_views(views, n_views, n_kv_heads, head_dim, L);
    return L.total;
}

KVQ_API kvq_status kvq_card_pack(const kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                                 uint64_t model_id, const int64_t *position_offsets, void *card, size_t card_bytes,
                                 void *stream) {
    if (!head_dim_supported(head_dim)) return KVQ_ERR_UNSUPPORTED;
    if (n_kv_heads <= 0 || n_kv_heads > 65535) return KVQ_ERR_INVALID_ARG;
    const kvq_status vs = validate_views(views, n_views, false);
    if (vs != KVQ_OK) return vs;
    if (!card || !aligned(card, 256)) return KVQ_ERR_INVALID_ARG;
    CardLayout L;
    card_layout_of_views(views, n_views, n_kv_heads, head_dim, L);
    if (card_bytes < L.total) return KVQ_ERR_INVALID_ARG;
    kvq::CardHeader h;
    std::memset(&h, 0, sizeof h);
    std::memcpy(h.magic, "KVQCARD1", 8);
    h.version = kvq::kCardVersion;
    h.n_views = (uint32_t)n_views;
    h.n_kv_heads = (uint32_t)n_kv_heads;
    h.head_dim = (uint32_t)head_dim;
    h.model_id = model_id;
    h.total_bytes = L.total;
    return card_launch(true, views, n_views, n_kv_heads, head_dim, L, &h, position_offsets,
                       static_cast<uint8_t *>(card), static_cast<cudaStream_t>(stream));
}

KVQ_API kvq_status kvq_card_read_header(const void *card_host, size_t card_bytes, int32_t *n_views,
                                        int32_t *n_kv_heads, int32_t *head_dim, uint64_t *model_id) {
    kvq::CardHeader h;
    std::vector<kvq::CardView> recs;
    const kvq_status ps = card_parse(card_host, card_bytes, h, recs);
    if (ps != KVQ_OK) return ps;
    if (n_views) *n_views = (int32_t)h.n_views;
    if (n_kv_heads) *n_kv_heads = (int32_t)h.n_kv_heads;
    if (head_dim) *head_dim = (int32_t)h.head_dim;
    if (model_id) *model_id = h.model_id;
    return KVQ_OK;
}

KVQ_API kvq_status kvq_card_view_info(const void *card_host, size_t card_bytes, int32_t index, int32_t *bits,
                                      int64_t *n_packed, int32_t *n_window, int64_t *position_offset) {
    kvq::CardHeader h;
    std::vector<kvq::CardView> recs;
    const kvq_status ps = card_parse(card_host, card_bytes, h, recs);
    if (ps != KVQ_OK) return ps;
    if (index < 0 || (uint32_t)index >= h.n_views) return KVQ_ERR_INVALID_ARG;
    const kvq::CardView &r = recs[index];
    if (bits) *bits = (int32_t)r.bits;
    if (n_packed) *n_packed = (int64_t)r.n_packed;
    if (n_window) *n_window = (int32_t)r.n_window;
    if (position_offset) *position_offset = r.position_offset;
    return KVQ_OK;
}

KVQ_API kvq_status kvq_card_unpack(const void *card_host, const void *card, size_t card_bytes, kvq_view *views,
                                   int32_t n_views, int32_t n_kv_heads, int32_t head_dim, void *stream) {
    kvq::CardHeader h;
    std::vector<kvq::CardView> recs;
    const kvq_status ps = card_parse(card_host, card_bytes, h, recs);
    if (ps != KVQ_OK) return ps;
    if (!card || !aligned(card, 256)) return KVQ_ERR_INVALID_ARG;
    if (n_views != (int32_t)h.n_views || n_kv_heads != (int32_t)h.n_kv_heads || head_dim != (int32_t)h.head_dim)
        return KVQ_ERR_INVALID_ARG;
    // the views as they will be: the card's counts, window from slot 0
    std::vector<kvq_view> post(views, views + n_views);
    for (int i = 0; i < n_views; ++i) {
        const kvq::CardView &r = recs[i];
        kvq_view &v = post[i];
        if (r.n_packed > 0 && v.bits != (int32_t)r.bits) return KVQ_ERR_INVALID_ARG;  // rows are laid out per width
        if ((int64_t)r.n_packed > v.cap_packed || (int32_t)r.n_window > v.cap_window) return KVQ_ERR_CAPACITY;
        v.n_packed = (int64_t)r.n_packed;
        v.n_window = (int32_t)r.n_window;
        v.window_head = 0;
    }
    const kvq_status vs = validate_views(post.data(), n_views, false);
    if (vs != KVQ_OK) return vs;
    CardLayout L;
    card_layout_of_views(post.data(), n_views, n_kv_heads, head_dim, L);
    const kvq_status ls = card_launch(false, post.data(), n_views, n_kv_heads, head_dim, L, nullptr, nullptr,
                                      const_cast<uint8_t *>(static_cast<const uint8_t *>(card)),
                                      static_cast<cudaStream_t>(stream));
    if (ls != KVQ_OK) return ls;
    for (int i = 0; i < n_views; ++i) views[i] = post[i];
    return KVQ_OK;
}
