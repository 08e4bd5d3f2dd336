// kvq_sparse.cuh -- top-K sparse decode attention over the packed cache:
// score every packed token against the query group, select the K best per
// (view, KV head), gather their rows into a compact per-head view; the
// attention kernel then runs over the compact rows plus the bf16 window.
//
// "Reasoning-Aware Error-Bounded KV-Cache Compression and Sparse Attention
// for Long-Context LLMs", Metodologia C (dynamic sparse decode attention: the
// top-K entries by a query-aware score form the active set; the rest stay in
// the cache for later steps).  Score of a packed token for KV head hk: the
// largest logit scale * q_h . k over the query heads h of hk's group, with k
// the exact affine value mn + s*c.  Ties go to the lower token index.  The
// bf16 recent window is always active.
#pragma once

#include <cstdint>

namespace kvq {

constexpr int kSparseMaxViews = 96;  // views per score / select / gather launch
constexpr int kScoreTok = 128;       // tokens per score CTA, one per thread
constexpr int kScoreHeads = 8;       // query heads per register batch
constexpr int kSelectThreads = 512;
constexpr int kGatherRows = 32;      // selected rows per gather CTA

struct ScoreView {
    const uint8_t *k_codes;   // [H_kv][cap][RB]
    const float *k_sm;        // [H_kv][cap][NG][2]
    int64_t cap_packed;
    int64_t score_off;        // float offset of head 0's scores; head hk at + hk * n_packed
    int32_t n_packed;
    int32_t blocks;           // token blocks of kScoreTok per head
    int32_t cta_begin;        // first CTA of this view in the launch
    int32_t q_row;            // row of q: [q_row][H_q][D]
};

struct ScoreArgs {
    const uint16_t *q;        // bf16 [n_views][H_q][D]
    float *scores;
    float scale;
    int32_t n_views;
    int32_t n_q_heads;
    int32_t group;            // query heads per KV head
    ScoreView views[kSparseMaxViews];
};

// One thread per packed token: the token's K codes are unpacked group by
// group into exact floats, dotted with each query head's 64 q values (fp32,
// fixed order), scaled by s and offset by mn times the q group sum.
template <int NG, int B>
__global__ void __launch_bounds__(kScoreTok) score_kernel(const __grid_constant__ ScoreArgs a) {
    constexpr int D = 64 * NG;
    constexpr int RB = 8 * B * NG;
    extern __shared__ __align__(16) float score_smem[];
    const int bx = blockIdx.x, tid = threadIdx.x;
    int lo = 0, hi = a.n_views - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.views[mid].cta_begin <= bx) lo = mid; else hi = mid - 1;
    }
    const ScoreView &v = a.views[lo];
    const int local = bx - v.cta_begin;
    const int hk = local / v.blocks, tb = local - hk * v.blocks;
    const int G = a.group;
    float *qs = score_smem;          // [G][D]
    float *qsum = qs + G * D;        // [G][NG]
    const uint16_t *qp = a.q + ((int64_t)v.q_row * a.n_q_heads + (int64_t)hk * G) * D;
    for (int i = tid; i < G * D; i += kScoreTok) qs[i] = __uint_as_float((uint32_t)qp[i] << 16);
    __syncthreads();
    for (int i = tid; i < G * NG; i += kScoreTok) {
        const float *x = qs + (i / NG) * D + (i % NG) * 64;
        float t = 0.f;
        for (int j = 0; j < 64; ++j) t += x[j];
        qsum[i] = t;
    }
    __syncthreads();
    const int t = tb * kScoreTok + tid;
    if (t >= v.n_packed) return;
    const uint8_t *row = v.k_codes + ((int64_t)hk * v.cap_packed + t) * RB;
    const float2 *smr = reinterpret_cast<const float2 *>(v.k_sm + ((int64_t)hk * v.cap_packed + t) * NG * 2);
    float best = -INFINITY;
    for (int h0 = 0; h0 < G; h0 += kScoreHeads) {
        float l[kScoreHeads];
#pragma unroll
        for (int h = 0; h < kScoreHeads; ++h) l[h] = 0.f;
#pragma unroll 1
        for (int g = 0; g < NG; ++g) {
            // the group's 64 codes: 8*B bytes, LSB-first little-endian
            uint64_t w[B];
#pragma unroll
            for (int i = 0; i < B; ++i) w[i] = __ldg(reinterpret_cast<const unsigned long long *>(row + g * 8 * B) + i);
            float cf[64];
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const int bit = j * B, wi = bit >> 6, sh = bit & 63;
                uint32_t c = (uint32_t)(w[wi] >> sh);
                if (sh + B > 64) c |= (uint32_t)(w[wi + 1] << (64 - sh));
                c &= (1u << B) - 1u;
                cf[j] = __uint_as_float(0x4B000000u | c) - 8388608.0f;  // exact: c < 2^23
            }
            const float2 sm = __ldg(smr + g);
#pragma unroll
            for (int h = 0; h < kScoreHeads; ++h) {
                if (h0 + h < G) {
                    const float4 *q4 = reinterpret_cast<const float4 *>(qs + (h0 + h) * D + g * 64);
                    float acc = 0.f;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float4 x = q4[j];
                        acc = fmaf(x.x, cf[4 * j], acc);
                        acc = fmaf(x.y, cf[4 * j + 1], acc);
                        acc = fmaf(x.z, cf[4 * j + 2], acc);
                        acc = fmaf(x.w, cf[4 * j + 3], acc);
                    }
                    l[h] = fmaf(sm.x, acc, fmaf(sm.y, qsum[(h0 + h) * NG + g], l[h]));
                }
            }
        }
#pragma unroll
        for (int h = 0; h < kScoreHeads; ++h)
            if (h0 + h < G) best = fmaxf(best, a.scale * l[h]);
    }
    a.scores[v.score_off + (int64_t)hk * v.n_packed + t] = best;
}

struct SelectView {
    int64_t score_off;        // as ScoreView::score_off
    int32_t n_packed;         // n_packed <= top_k: every token, no scores read
    int32_t out_row;          // row of the selection: [out_row][H_kv][top_k]
};

struct SelectArgs {
    const float *scores;
    int32_t *sel;             // int32 [n_views][H_kv][top_k], ascending, -1 padded
    int32_t top_k;
    int32_t n_kv_heads;
    SelectView views[kSparseMaxViews];
};

// Monotone map of a finite float onto uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the block's threads (kSelectThreads), in thread order.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t *warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        uint32_t t = lane < kSelectThreads / 32 ? warp_tot[lane] : 0u;
        uint32_t ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, ti, o);
            if (lane >= o) ti += y;
        }
        if (lane < kSelectThreads / 32) warp_tot[lane] = ti - t;
    }
    __syncthreads();
    const uint32_t r = warp_tot[warp] + inc - x;
    __syncthreads();  // warp_tot is reused by the next scan
    return r;
}

// One CTA per (view, KV head): radix select of the K largest scores (four
// 8-bit digit passes from the top), then an ordered compaction that writes
// the selected indices in ascending order, equal scores at the threshold
// taken from the lowest index up.
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const __grid_constant__ SelectArgs a) {
    __shared__ uint32_t hist[256];
    __shared__ uint32_t warp_tot[kSelectThreads / 32];
    __shared__ uint32_t pick[2];
    const SelectView &v = a.views[blockIdx.x];
    const int hk = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
    const int n = v.n_packed, K = a.top_k;
    int32_t *out = a.sel + ((int64_t)v.out_row * a.n_kv_heads + hk) * K;
    if (n <= K) {
        for (int i = tid; i < K; i += kSelectThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float *sc = a.scores + v.score_off + (int64_t)hk * n;
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)K;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelectThreads) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += kSelectThreads) {
            const uint32_t k = order_key(sc[i]);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // lane l holds bins 255-8l .. 248-8l, highest first
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[255 - 8 * lane - j];
                tot += c[j];
            }
            uint32_t inc = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
                if (lane >= o) inc += y;
            }
            uint32_t above = inc - tot;  // keys in higher bins
            if (above < remaining && remaining <= inc) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (above + c[j] >= remaining) {
                        pick[0] = 255u - 8u * lane - j;
                        pick[1] = above;
                        break;
                    }
                    above += c[j];
                }
            }
        }
        __syncthreads();
        prefix |= pick[0] << shift;
        mask |= 255u << shift;
        remaining -= pick[1];
        __syncthreads();
    }
    // keys above the threshold key `prefix`, and the first `remaining` equal to it
    const int per = (n + kSelectThreads - 1) / kSelectThreads;
    const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
    uint32_t gt = 0, eq = 0;
    for (int i = b0; i < b1; ++i) {
        const uint32_t k = order_key(sc[i]);
        gt += k > prefix;
        eq += k == prefix;
    }
    const uint32_t eq_before = block_excl_scan(eq, warp_tot);
    const uint32_t take = eq_before >= remaining ? 0u : min(eq, remaining - eq_before);
    uint32_t pos = block_excl_scan(gt + take, warp_tot);
    uint32_t taken = 0;
    for (int i = b0; i < b1; ++i) {
        const uint32_t k = order_key(sc[i]);
        if (k > prefix || (k == prefix && taken < take)) {
            out[pos++] = i;
            if (k == prefix) ++taken;
        }
    }
}

struct GatherView {
    const uint8_t *codes[2];  // source K, V codes [H_kv][cap][RB]
    const float *sm[2];       // source K, V scale/min [H_kv][cap][NG][2]
    uint8_t *dst_codes[2];    // compact [H_kv][cap_c][RB]
    float *dst_sm[2];         // compact [H_kv][cap_c][NG][2]
    int64_t cap_packed;
    int64_t cap_compact;
    int32_t row_bytes;
    int32_t sel_row;
};

struct GatherArgs {
    const int32_t *sel;       // [n_views][H_kv][top_k]
    int32_t top_k;
    int32_t n_kv_heads;
    int32_t sm_bytes;         // scale/min bytes per row: (D/64) * 8
    GatherView views[kSparseMaxViews];
};

// Grid (view, KV head, block of kGatherRows selections): copy the selected
// packed rows (K and V codes and scale/min) to consecutive compact rows, 8
// bytes per thread and access.
__global__ void __launch_bounds__(256) gather_kernel(const __grid_constant__ GatherArgs a) {
    const GatherView &v = a.views[blockIdx.x];
    const int hk = blockIdx.y;
    const int r0 = blockIdx.z * kGatherRows;
    const int rows = min(kGatherRows, a.top_k - r0);
    const int32_t *sel = a.sel + ((int64_t)v.sel_row * a.n_kv_heads + hk) * a.top_k + r0;
    const int wc = v.row_bytes / 8, ws = a.sm_bytes / 8, W = 2 * wc + 2 * ws;
    for (int i = threadIdx.x; i < rows * W; i += blockDim.x) {
        const int r = i / W, w = i - r * W;
        const int64_t src_row = (int64_t)hk * v.cap_packed + sel[r];
        const int64_t dst_row = (int64_t)hk * v.cap_compact + r0 + r;
        const uint2 *src;
        uint2 *dst;
        if (w < 2 * wc) {
            const int kv = w >= wc, x = w - kv * wc;
            src = reinterpret_cast<const uint2 *>(v.codes[kv] + src_row * v.row_bytes) + x;
            dst = reinterpret_cast<uint2 *>(v.dst_codes[kv] + dst_row * v.row_bytes) + x;
        } else {
            const int y = w - 2 * wc, kv = y >= ws, x = y - kv * ws;
            src = reinterpret_cast<const uint2 *>(reinterpret_cast<const uint8_t *>(v.sm[kv]) + src_row * a.sm_bytes) + x;
            dst = reinterpret_cast<uint2 *>(reinterpret_cast<uint8_t *>(v.dst_sm[kv]) + dst_row * a.sm_bytes) + x;
        }
        *dst = __ldg(src);
    }
}

}  // namespace kvq
