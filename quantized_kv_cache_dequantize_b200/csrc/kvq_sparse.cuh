// kvq_sparse.cuh -- top-K sparse decode attention over the packed cache:
// score every packed token against the query group, select the K best per
// (view, KV head) as a list of ascending row indices; the attention kernel
// then reads those rows through the list, plus the bf16 window.
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

#include "kvq_debug.cuh"
#include "kvq_ptx.cuh"

namespace kvq {

constexpr int kSparseMaxViews = 96;  // views per score / select launch
constexpr int kScoreTok = 128;       // threads of a score CTA, one token each at a time
constexpr int kScoreBlocks = 4;      // blocks of kScoreTok tokens per score CTA
constexpr int kScoreHeads = 8;       // query heads per register batch
constexpr int kSelectThreads = 512;
constexpr int kSelectStageMax = 45056;  // keys a select CTA stages in shared memory (176 KiB)
constexpr int kSelFastMax = 32768;      // select_fast_kernel: views of up to 32 keys per thread
constexpr int kSelBins = 2048;          // histogram bins of a select_fast_kernel pass

struct ScoreView {
    const uint8_t *k_codes;   // [H_kv][cap][RB]
    const float *k_sm;        // [H_kv][cap][NG][2]
    int64_t cap_packed;
    int64_t score_off;        // float offset of head 0's scores; head hk at + hk * n_packed
    int32_t n_packed;
    int32_t blocks;           // score CTAs per head (kScoreBlocks * kScoreTok tokens each)
    int32_t cta_begin;        // first CTA of this view in the launch
    int32_t q_row;            // row of q: [q_row][H_q][D]
};

struct ScoreArgs {
    const uint16_t *q;        // bf16 [n_views][H_q][D]
    float *scores;
    int64_t n_scores;         // floats of the score array (the debug build's checks)
    float scale;
    int32_t n_views;
    int32_t n_q_heads;
    int32_t group;            // query heads per KV head
    ScoreView views[kSparseMaxViews];
};

// One thread per packed token, kScoreBlocks blocks of kScoreTok tokens per
// CTA: the token's K codes are unpacked 16 at a time into exact floats and
// dotted with each query head's q values (fp32, fixed order); per group the
// sum is scaled by s and offset by mn times the q group sum.
template <int NG, int B>
__global__ void __launch_bounds__(kScoreTok) score_kernel(const __grid_constant__ ScoreArgs a) {
    constexpr int D = 64 * NG;
    constexpr int RB = 8 * B * NG;
    extern __shared__ __align__(16) float score_smem[];
    // q and the cache may come from the preceding grid; the next stage may be
    // scheduled as slots free up (it waits for this grid in turn)
    pdl_wait();
    pdl_launch_dependents();
    const int bx = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    int lo = 0, hi = a.n_views - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.views[mid].cta_begin <= bx) lo = mid; else hi = mid - 1;
    }
    const ScoreView &v = a.views[lo];
    const int local = bx - v.cta_begin;
    const int hk = local / v.blocks, tb0 = (local - hk * v.blocks) * kScoreBlocks;
    const int G = a.group;
    float *qs = score_smem;          // [G][D]
    float *qsum = qs + G * D;        // [G][NG]
    const uint16_t *qp = a.q + ((int64_t)v.q_row * a.n_q_heads + (int64_t)hk * G) * D;
    // q to fp32, and each (head, group) sum of 64 values: 4 values per lane,
    // then 16 lanes by shuffles (fixed order)
    for (int i0 = 0; i0 < G * D; i0 += 4 * kScoreTok) {
        const int i = i0 + 4 * tid;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (i < G * D) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[j] = __uint_as_float((uint32_t)qp[i + j] << 16);
                qs[i + j] = x[j];
            }
        }
        float t = (x[0] + x[1]) + (x[2] + x[3]);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
        if ((lane & 15) == 0 && i < G * D) qsum[i / 64] = t;
    }
    __syncthreads();
    for (int tb = tb0; tb < tb0 + kScoreBlocks; ++tb) {
        const int t = tb * kScoreTok + tid;
        if (t >= v.n_packed) break;
        const int64_t si = v.score_off + (int64_t)hk * v.n_packed + t;
        if (!dcheck(t < v.cap_packed && si >= 0 && si < a.n_scores, kDbgScore)) break;
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
                for (int i = 0; i < B; ++i)
                    w[i] = __ldg(reinterpret_cast<const unsigned long long *>(row + g * 8 * B) + i);
                float acc[kScoreHeads];
#pragma unroll
                for (int h = 0; h < kScoreHeads; ++h) acc[h] = 0.f;
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 16) {
                    float cf[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int bit = (c0 + j) * B, wi = bit >> 6, sh = bit & 63;
                        uint32_t c = (uint32_t)(w[wi] >> sh);
                        if (sh + B > 64) c |= (uint32_t)(w[wi + 1] << (64 - sh));
                        c &= (1u << B) - 1u;
                        cf[j] = __uint_as_float(0x4B000000u | c) - 8388608.0f;  // exact: c < 2^23
                    }
#pragma unroll
                    for (int h = 0; h < kScoreHeads; ++h) {
                        if (h0 + h < G) {
                            const float4 *q4 = reinterpret_cast<const float4 *>(qs + (h0 + h) * D + g * 64 + c0);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float4 x = q4[j];
                                acc[h] = fmaf(x.x, cf[4 * j], acc[h]);
                                acc[h] = fmaf(x.y, cf[4 * j + 1], acc[h]);
                                acc[h] = fmaf(x.z, cf[4 * j + 2], acc[h]);
                                acc[h] = fmaf(x.w, cf[4 * j + 3], acc[h]);
                            }
                        }
                    }
                }
                const float2 sm = __ldg(smr + g);
#pragma unroll
                for (int h = 0; h < kScoreHeads; ++h)
                    if (h0 + h < G) l[h] = fmaf(sm.x, acc[h], fmaf(sm.y, qsum[(h0 + h) * NG + g], l[h]));
            }
#pragma unroll
            for (int h = 0; h < kScoreHeads; ++h)
                if (h0 + h < G) best = fmaxf(best, a.scale * l[h]);
        }
        a.scores[si] = best;
    }
}

struct SelectView {
    int64_t score_off;        // as ScoreView::score_off
    int32_t n_packed;         // n_packed <= top_k: every token, no scores read
    int32_t out_row;          // row of the selection: [out_row][H_kv][top_k]
    int32_t staged;           // 1: the head's keys fit the launch's shared-memory stage
};

struct SelectArgs {
    const float *scores;
    int32_t *sel;             // int32 [n_views][H_kv][top_k], ascending, -1 padded
    int64_t n_scores;         // floats of the score array,
    int32_t n_sel_rows;       // rows of sel (the debug build's checks)
    int32_t top_k;
    int32_t n_kv_heads;
    SelectView views[kSparseMaxViews];
};

// Monotone map of a finite float onto uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One CTA per (view, KV head): radix select of the K largest scores (four
// 8-bit digit passes from the top, over keys staged in shared memory when
// they fit), an ordered compaction that writes the selected indices in
// ascending order (equal scores at the threshold taken from the lowest index
// up).  The attention grid reads the selected rows through that list.
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const __grid_constant__ SelectArgs a) {
    extern __shared__ uint32_t skeys[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t pick[2];
    pdl_wait();  // the scores of the preceding grid
    pdl_launch_dependents();
    const SelectView &v = a.views[blockIdx.x];
    const int hk = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
    const int n = v.n_packed, K = a.top_k;
    int32_t *out = a.sel + ((int64_t)v.out_row * a.n_kv_heads + hk) * K;
    // the selection row and the head's scores exist (debug
    // build; uniform over the CTA, so a refused CTA returns whole)
    if (!dcheck(v.out_row >= 0 && v.out_row < a.n_sel_rows && hk < a.n_kv_heads &&
                    (n <= K || (v.score_off >= 0 && v.score_off + (int64_t)(hk + 1) * n <= a.n_scores)),
                kDbgSelect))
        return;
    if (n <= K) {
        for (int i = tid; i < K; i += kSelectThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float *sc = a.scores + v.score_off + (int64_t)hk * n;
    const bool staged = v.staged != 0;
    if (staged) {
        // eight loads in flight per thread
        for (int i0 = tid; i0 < n; i0 += 8 * kSelectThreads) {
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = i0 + j * kSelectThreads < n ? __ldcg(sc + i0 + j * kSelectThreads) : 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (i0 + j * kSelectThreads < n) skeys[i0 + j * kSelectThreads] = order_key(x[j]);
        }
        __syncthreads();
    }
    auto key_at = [&](int i) { return staged ? skeys[i] : order_key(sc[i]); };
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)K;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelectThreads) hist[i] = 0u;
        __syncthreads();
        // scores cluster in few bins (the top digit holds the sign and most of
        // the exponent): lanes with the same bin add once, with their count
        for (int i0 = 0; i0 < n; i0 += kSelectThreads) {
            const int i = i0 + tid;
            const uint32_t k = i < n ? key_at(i) : 0u;
            const bool in = i < n && (k & mask) == prefix;
            const uint32_t bin = (k >> shift) & 255u;
            const uint32_t act = __ballot_sync(0xFFFFFFFFu, in);
            if (in) {
                const uint32_t peers = __match_any_sync(act, bin);
                if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
            }
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
    // keys above the threshold key `prefix`, and the first `remaining` equal
    // to it.  Warp w owns one contiguous segment of the keys and walks it 32
    // keys at a time (lane = key): counts first, then positions from ballots.
    const int warp = tid >> 5;
    constexpr int kWarps = kSelectThreads / 32;
    const int seg = (n + kWarps - 1) / kWarps;
    const int w0 = min(n, warp * seg), w1 = min(n, w0 + seg);
    uint32_t gt = 0, eq = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < w1 ? key_at(i) : 0u;
        gt += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && k > prefix));
        eq += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && k == prefix));
    }
    if (lane == 0) {
        hist[warp] = gt;
        hist[kWarps + warp] = eq;
    }
    __syncthreads();
    if (tid == 0) {
        // per warp: the equal keys it takes and its first output position
        uint32_t eq_before = 0, pos = 0;
        for (int w = 0; w < kWarps; ++w) {
            const uint32_t e = hist[kWarps + w];
            const uint32_t take = eq_before >= remaining ? 0u : min(e, remaining - eq_before);
            hist[2 * kWarps + w] = take;
            hist[3 * kWarps + w] = pos;
            pos += hist[w] + take;
            eq_before += e;
        }
    }
    __syncthreads();
    {
        const uint32_t take = hist[2 * kWarps + warp];
        uint32_t pos = hist[3 * kWarps + warp], taken = 0;
        const uint32_t below = (1u << lane) - 1u;
        for (int i0 = w0; i0 < w1; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t k = i < w1 ? key_at(i) : 0u;
            const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, i < w1 && k == prefix);
            const bool pick_me = i < w1 && (k > prefix || (k == prefix && taken + __popc(eqm & below) < take));
            const uint32_t pm = __ballot_sync(0xFFFFFFFFu, pick_me);
            if (pick_me) out[pos + __popc(pm & below)] = i;
            pos += __popc(pm);
            taken += min((uint32_t)__popc(eqm), take - min(take, taken));
        }
    }
}

// ---- select with a float-range first pass (views of up to 32768 tokens)

// Inverse of order_key.
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Bin of order key k among kSelBins equal-width bins over [lo, lo + kSelBins
// / scl], keys below and above the range in the end bins: monotone in the
// key's float value, computed without contraction so that every use agrees.
__device__ __forceinline__ uint32_t float_bin(uint32_t k, float lo, float scl) {
    const float y = __fmul_rn(__fsub_rn(key_float(k), lo), scl);
    return y <= 0.f ? 0u : min((uint32_t)(kSelBins - 1), (uint32_t)y);
}

// One CTA of THREADS per (view, KV head) with 32 * THREADS packed tokens at
// most.  Keys (order keys of the scores) are staged in shared memory; thread
// t owns keys t, t + kSelFastThreads, ... and marks which of them are still
// candidates in one register.  The K-th largest key T comes from histogram
// passes over the candidates: first kSelBins equal-width bins over the
// scores' float range (scores spread evenly there, so the counters rarely
// collide), then 11-bit digits of the candidates' keys below the bits they
// all share.  The keys in the bins above the boundary bin are taken; those
// in it stay candidates.  Each warp then walks one contiguous segment of the
// keys and writes every key above T and the first (by index) of those equal
// to T in ascending order.
template <int THREADS>
__global__ void __launch_bounds__(THREADS) select_fast_kernel(const __grid_constant__ SelectArgs a) {
    static_assert(THREADS >= 64 && THREADS <= 1024 && kSelBins % THREADS == 0, "threads");
    constexpr int kSelFastThreads = THREADS;
    extern __shared__ uint32_t fkeys[];
    __shared__ uint32_t hist[kSelBins];
    __shared__ uint32_t red[5 * 32];
    __shared__ uint32_t pick[2];
    constexpr int kWarps = THREADS / 32;
    constexpr int kKeys = 32;                         // keys per thread at most
    constexpr int kBpt = kSelBins / THREADS;          // bins per thread of the boundary search
    pdl_wait();  // the scores of the preceding grid
    pdl_launch_dependents();
    const SelectView &v = a.views[blockIdx.x];
    const int hk = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = v.n_packed, K = a.top_k;
    int32_t *out = a.sel + ((int64_t)v.out_row * a.n_kv_heads + hk) * K;
    // the selection row and the head's scores exist, and the keys fit (debug
    // build; uniform over the CTA, so a refused CTA returns whole)
    if (!dcheck(v.out_row >= 0 && v.out_row < a.n_sel_rows && hk < a.n_kv_heads &&
                    (n <= K || (v.score_off >= 0 && v.score_off + (int64_t)(hk + 1) * n <= a.n_scores &&
                                n <= kKeys * THREADS)),
                kDbgSelect))
        return;
    if (n <= K) {
        for (int i = tid; i < K; i += kSelFastThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float *sc = a.scores + v.score_off + (int64_t)hk * n;
    const int nk = tid < n ? (n - tid + kSelFastThreads - 1) / kSelFastThreads : 0;  // keys of this thread
    uint32_t cand = 0;  // bit j: key tid + j * kSelFastThreads is a candidate
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
    float s1 = 0.f, s2 = 0.f;  // sum and sum of squares of the finite scores
#pragma unroll 8
    for (int j = 0; j < kKeys; ++j) {
        const int i = tid + j * kSelFastThreads;
        if (i < n) {
            const float x = __ldcg(sc + i);
            const uint32_t k = order_key(x);
            fkeys[i] = k;
            cand |= 1u << j;
            mn = min(mn, k);
            mx = max(mx, k);
            if (isfinite(x)) {
                s1 += x;
                s2 = fmaf(x, x, s2);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
        s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
    }
    if (lane == 0) {
        reinterpret_cast<float *>(red)[96 + warp] = s1;
        reinterpret_cast<float *>(red)[128 + warp] = s2;
    }
    __syncthreads();
    s1 = lane < kWarps ? reinterpret_cast<const float *>(red)[96 + lane] : 0.f;
    s2 = lane < kWarps ? reinterpret_cast<const float *>(red)[128 + lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
        s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
    }
    // the first pass's range: mean +- 6 standard deviations within [min, max]
    // (any range gives the exact selection: scores outside it fall into the
    // end bins; a range that leaves out a few outliers keeps the bins where
    // the K-th score lies from collapsing into one)
    const float mean = s1 / (float)n, sd = sqrtf(fmaxf(s2 / (float)n - mean * mean, 0.f));
    uint32_t rem = (uint32_t)K;
    bool first = true, done = false, failed = false;
    // at most one float pass and three digit passes; the bound and the
    // boundary check only guard against a broken count
    for (int pass = 0; pass < 5; ++pass) {
        // block-wide min and max of the candidates (shuffles, then warp 0's
        // partials in shared memory)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
            mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        }
        if (lane == 0) {
            red[warp] = mn;
            red[32 + warp] = mx;
        }
        __syncthreads();
        mn = lane < kWarps ? red[lane] : 0xFFFFFFFFu;
        mx = lane < kWarps ? red[32 + lane] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
            mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        }
        if (mn == mx) {  // the candidates are all T (uniform)
            done = true;
            break;
        }
        // this pass's bins: the float range on the first pass when its ends
        // are finite and distinct, else 11-bit digits below the shared bits
        // (every candidate finite: the smallest and largest are)
        const bool ends_finite = isfinite(key_float(mn)) && isfinite(key_float(mx));
        float lo = key_float(mn), hi = key_float(mx);
        if (first && ends_finite && isfinite(mean) && isfinite(sd) && sd > 0.f) {
            lo = fmaxf(lo, mean - 6.f * sd);
            hi = fminf(hi, mean + 6.f * sd);
        }
        const float span = hi - lo;
        const float scl = (float)kSelBins / span;
        const bool use_float = first && ends_finite && isfinite(span) && span > 0.f && isfinite(scl);
        first = false;
        const int top_bit = 31 - __clz(mn ^ mx);
        const int shift = top_bit > 10 ? top_bit - 10 : 0;
        for (int i = tid; i < kSelBins; i += kSelFastThreads) hist[i] = 0u;
        if (tid == 0) {
            pick[0] = 0xFFFFFFFFu;  // stays so if no bin holds the boundary
            pick[1] = 0u;
        }
        __syncthreads();
        // the candidates: on the first pass every key of the thread (an
        // unrolled loop, several in flight), later the set bits
        if (pass == 0) {
#pragma unroll 8
            for (int j = 0; j < nk; ++j) {
                const uint32_t k = fkeys[tid + j * kSelFastThreads];
                const uint32_t b = use_float ? float_bin(k, lo, scl) : (k >> shift) & (uint32_t)(kSelBins - 1);
                atomicAdd(&hist[b], 1u);
            }
        } else {
            for (uint32_t cb = cand; cb != 0u; cb &= cb - 1u) {
                const int j = __ffs(cb) - 1;
                const uint32_t k = fkeys[tid + j * kSelFastThreads];
                const uint32_t b = use_float ? float_bin(k, lo, scl) : (k >> shift) & (uint32_t)(kSelBins - 1);
                atomicAdd(&hist[b], 1u);
            }
        }
        __syncthreads();
        // boundary bin: thread t sums bins kSelBins - (t+1)*kBpt .. kSelBins
        // - t*kBpt - 1 (the highest bins first), one block scan of the sums
        const int top = kSelBins - tid * kBpt;
        uint32_t c = 0;
#pragma unroll
        for (int i = 1; i <= kBpt; ++i) c += hist[top - i];
        uint32_t inc = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) red[64 + warp] = inc;
        __syncthreads();
        uint32_t wtot = lane < kWarps ? red[64 + lane] : 0u, winc = wtot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, winc, o);
            if (lane >= o) winc += y;
        }
        uint32_t above = __shfl_sync(0xFFFFFFFFu, winc - wtot, warp) + inc - c;
        if (above < rem && rem <= above + c) {
#pragma unroll
            for (int i = 1; i <= kBpt; ++i) {
                const uint32_t h = hist[top - i];
                if (above + h >= rem) {
                    pick[0] = (uint32_t)(top - i);
                    pick[1] = above;
                    break;
                }
                above += h;
            }
        }
        __syncthreads();
        const uint32_t pb = pick[0], pabove = pick[1];
        if (pb >= (uint32_t)kSelBins) {
            failed = true;
            break;
        }
        rem -= pabove;
        mn = 0xFFFFFFFFu;
        mx = 0u;
        if (pass == 0) {
#pragma unroll 8
            for (int j = 0; j < nk; ++j) {
                const uint32_t k = fkeys[tid + j * kSelFastThreads];
                const uint32_t b = use_float ? float_bin(k, lo, scl) : (k >> shift) & (uint32_t)(kSelBins - 1);
                if (b != pb) {
                    cand &= ~(1u << j);
                } else {
                    mn = min(mn, k);
                    mx = max(mx, k);
                }
            }
        } else {
            for (uint32_t cb = cand; cb != 0u; cb &= cb - 1u) {
                const int j = __ffs(cb) - 1;
                const uint32_t k = fkeys[tid + j * kSelFastThreads];
                const uint32_t b = use_float ? float_bin(k, lo, scl) : (k >> shift) & (uint32_t)(kSelBins - 1);
                if (b != pb) {
                    cand &= ~(1u << j);
                } else {
                    mn = min(mn, k);
                    mx = max(mx, k);
                }
            }
        }
        __syncthreads();  // red, hist and pick are rewritten by the next pass
    }
    if (!dcheck(done && !failed && rem >= 1u && rem <= (uint32_t)K, kDbgSelect) || !done || failed) {
        for (int i = tid; i < K; i += kSelFastThreads) out[i] = -1;
        return;
    }
    const uint32_t T = mn;  // rem keys equal to T remain to be taken
    // ordered compaction: warp w walks keys [w0, w1), 32 at a time
    const int seg = (n + kWarps - 1) / kWarps;
    const int w0 = min(n, warp * seg), w1 = min(n, w0 + seg);
    uint32_t gt = 0, eq = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < w1 ? fkeys[i] : 0u;
        gt += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && k > T));
        eq += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && k == T));
    }
    if (lane == 0) {
        red[96 + warp] = gt;
        red[128 + warp] = eq;
    }
    __syncthreads();
    // this warp's first output position and the equal keys it takes
    uint32_t g_before = 0, e_before = 0;
    for (int w = 0; w < warp; ++w) {
        g_before += red[96 + w];
        e_before += red[128 + w];
    }
    const uint32_t take = e_before >= rem ? 0u : min(eq, rem - e_before);
    uint32_t pos = g_before + min(e_before, rem), taken = 0;
    const uint32_t below = (1u << lane) - 1u;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < w1 ? fkeys[i] : 0u;
        const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, i < w1 && k == T);
        const bool pick_me = i < w1 && (k > T || (k == T && taken + __popc(eqm & below) < take));
        const uint32_t pm = __ballot_sync(0xFFFFFFFFu, pick_me);
        const uint32_t at = pos + __popc(pm & below);
        if (pick_me && dcheck(at < (uint32_t)K, kDbgSelect)) out[at] = i;
        pos += __popc(pm);
        taken += min((uint32_t)__popc(eqm), take - min(take, taken));
    }
}

}  // namespace kvq
