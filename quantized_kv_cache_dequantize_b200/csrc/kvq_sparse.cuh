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

// ---- inline PTX used by the select only

// Per-thread asynchronous 4-byte copy global -> shared (both addresses
// 4-byte aligned), completed for the issuing thread by cp_async_wait_all.
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Wait until every cp.async this thread issued has landed (visible to it).
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;\n" : "=r"(r));
    return r;
}

// Barrier over every thread of the cluster: shared-memory writes before it
// (this CTA's and the peers') are visible to the cluster's reads after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\nbarrier.cluster.wait.acquire;\n" ::: "memory");
}

// Load of the 32-bit word at `p` in the shared memory of the cluster's CTA
// `rank` (p: this CTA's address of the same variable).
__device__ __forceinline__ uint32_t ld_cluster_u32(const void *p, uint32_t rank) {
    uint32_t a, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(a) : "memory");
    return v;
}

// 16-byte load from the cluster's CTA `rank` (p 16-byte aligned).
__device__ __forceinline__ uint4 ld_cluster_v4(const void *p, uint32_t rank) {
    uint32_t a;
    uint4 v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a)
                 : "memory");
    return v;
}

constexpr int kSparseMaxViews = 96;  // views per score / select launch
constexpr int kScoreTok = 128;       // threads of a score CTA, one token each at a time
constexpr int kScoreBlocks = 4;      // blocks of kScoreTok tokens per score CTA
constexpr int kScoreHeads = 8;       // query heads per register batch
constexpr int kSelectThreads = 512;     // select_kernel CTA (views longer than kSelFastMax)
constexpr int kSelectStageMax = 45056;  // keys a select_kernel CTA stages in shared memory (176 KiB)
constexpr int kSelClusterThreads = 1024;  // select_cluster_kernel CTA
constexpr int kSelMaxCluster = 4;         // CTAs per (view, KV head) at most
// views of up to kSelFastMax packed tokens select in shared memory (32 keys a
// thread at most)
constexpr int kSelFastMax = kSelMaxCluster * kSelClusterThreads * 32;
constexpr int kSelBins = 2048;            // histogram bins of a select_cluster_kernel pass
constexpr int kSelWarpMax = 64;           // candidates one warp finishes

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
    int32_t key_cap;          // keys a select_cluster_kernel CTA's dynamic shared memory holds
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

// ---- select over keys in shared memory (views of up to kSelFastMax tokens)

// Bin of a score x (order key k) on the first pass: kSelBins equal-width bins
// over [lo, lo + kSelBins / scl] with scores below and above the range in the
// end bins, or, without a usable range, the key's top 11 bits.  Monotone in
// the key (NaNs sort beyond the infinities of their sign); computed without
// contraction so that every use agrees.
__device__ __forceinline__ uint32_t first_bin(float x, uint32_t k, bool use_float, float lo, float scl) {
    if (!use_float) return k >> 21;
    // clamped into [0, kSelBins - 1] (the infinities into the end bins), then
    // truncated; a NaN goes to the end bin of its sign
    const float y = fminf(fmaxf(__fmul_rn(__fsub_rn(x, lo), scl), 0.f), (float)(kSelBins - 1));
    return x != x ? ((k >> 31) ? (uint32_t)(kSelBins - 1) : 0u) : (uint32_t)y;
}

// Butterfly sum over a warp (every lane ends with the same result).
__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    return x;
}

// Top-K selection of one (view, KV head) by one CTA, or, with CLUSTER, by a
// thread-block cluster of CL CTAs (CL from the launch).  CTA r owns the keys
// [r*S, (r+1)*S) of the view, warp w of it the 32*kpt keys from r*S +
// 32*kpt*w, lane l the keys l, l+32, ... of those, kpt <= 32 per lane (bit j
// of a lane's masks: its key j).  The scores arrive by asynchronous 4-byte
// copies straight into shared memory, where they become order keys; the
// first-pass bins are kept beside them.
//   1. 256 scores of the CTA in 8 evenly spaced runs (of each CTA of the
//      cluster) give the first pass's range (mean +- 6 standard deviations
//      within their min and max; any range gives the exact selection: scores
//      outside it go to the end bins).
//   2. First pass: counts of every key's bin; the boundary bin from the
//      counts (of the whole cluster: each CTA sums its peers' histograms), the
//      same in every CTA.  Keys in higher bins are taken ("above"); those in
//      it stay candidates.
//   3. While more than kSelWarpMax candidates remain and they differ: 11-bit
//      digit passes below the bits they share.  Then the candidates are
//      gathered into one list, where one warp finds the K-th largest key T:
//      the candidate with fewer than rem larger ones and at least rem not
//      smaller (rem: K less the keys already taken above the candidates).
//   4. Ordered compaction: the keys above T and the first (by index) of
//      those equal to T; each warp's output position from the counts of the
//      warps and CTAs before it, each key's from one ballot per row of its
//      warp's keys.
// In a cluster, every decision that gates a cluster barrier is taken on
// cluster-wide values, so all its CTAs pass the same barriers; values from
// the peers are read by one warp and handed on in shared memory.
template <int THREADS, bool CLUSTER>
__global__ void __launch_bounds__(THREADS, 1) select_cluster_kernel(const __grid_constant__ SelectArgs a) {
    static_assert(THREADS % 32 == 0 && THREADS >= 128 && THREADS <= 1024 && kSelBins % THREADS == 0 &&
                      kSelBins / 4 <= THREADS && (THREADS / 32) * 64 <= kSelBins, "threads");
    constexpr int kWarps = THREADS / 32;
    constexpr int kBpt = kSelBins / THREADS;  // bins per thread of the boundary search
    constexpr int kSample = 8;                // scores per lane of warp 0 behind the first pass's range
    constexpr uint32_t kFull = 0xFFFFFFFFu;
    extern __shared__ __align__(16) uint32_t skeys[];  // [S] scores, then keys; then [S] uint16 first-pass bins
    __shared__ __align__(16) uint32_t hist[2][kSelBins];  // this CTA's counts, by pass parity
    __shared__ __align__(16) uint32_t hm[CLUSTER ? kSelBins : 4];  // the cluster's counts
    __shared__ uint32_t lst[kSelWarpMax];                 // this CTA's candidates at the end
    __shared__ uint32_t gl[CLUSTER ? kSelWarpMax : 4];    // the cluster's candidates
    __shared__ uint32_t xch[12];                          // what the cluster's CTAs read from each other
    __shared__ uint32_t red[5][32];
    __shared__ uint32_t bc[6];                            // values handed on to the CTA
    __shared__ uint32_t pick[2];
    __shared__ uint32_t pc[3];                            // the candidates' min, max and count
    pdl_wait();  // the scores of the preceding grid
    pdl_launch_dependents();
    const uint32_t CL = CLUSTER ? cluster_nctarank() : 1u, rank = CLUSTER ? cluster_ctarank() : 0u;
    const SelectView &v = a.views[blockIdx.x / CL];
    const int hk = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = v.n_packed, K = a.top_k;
    int32_t *out = a.sel + ((int64_t)v.out_row * a.n_kv_heads + hk) * K;
    const int kpt = (n + (int)CL * THREADS - 1) / ((int)CL * THREADS);
    const int seg = 32 * kpt, S = kWarps * seg;
    // the selection row and the head's scores exist, and the keys fit (debug
    // build; uniform over the cluster, so a refused cluster returns whole)
    if (!dcheck(v.out_row >= 0 && v.out_row < a.n_sel_rows && hk < a.n_kv_heads &&
                    (n <= K || (v.score_off >= 0 && v.score_off + (int64_t)(hk + 1) * n <= a.n_scores &&
                                kpt <= 32 && S <= a.key_cap)),
                kDbgSelect))
        return;
    if (n <= K) {
        for (int i = (int)rank * THREADS + tid; i < K; i += (int)CL * THREADS) out[i] = i < n ? i : -1;
        return;
    }
    auto csync = [&]() {
        if constexpr (CLUSTER)
            cluster_sync();
        else
            __syncthreads();
    };
    uint16_t *sbin = reinterpret_cast<uint16_t *>(skeys + S);
    const float *sc = a.scores + v.score_off + (int64_t)hk * n;
    const int base = (int)rank * S + warp * seg + lane;  // index of this lane's key 0; key j at + 32 j
    const int lbase = warp * seg + lane;                 // its place in skeys
    const int nk = base < n ? min(kpt, (n - base + 31) / 32) : 0;
    // every score of this lane in flight at once
    for (int j = 0; j < nk; ++j) cp_async4(skeys + lbase + 32 * j, sc + base + 32 * j);
    for (int i = tid; i < kSelBins; i += THREADS) hist[0][i] = 0u;
    cp_async_wait_all();
    __syncthreads();  // every lane's scores have landed

    // 1. the range, from kSample evenly spaced scores per lane of warp 0 (the
    //    cluster's CTAs: their samples together)
    float s1 = 0.f, s2 = 0.f, smin = INFINITY, smax = -INFINITY;
    uint32_t ns = 0;
    auto reduce5 = [&]() {  // butterfly: the same result in every lane
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s1 += __shfl_xor_sync(kFull, s1, o);
            s2 += __shfl_xor_sync(kFull, s2, o);
            smin = fminf(smin, __shfl_xor_sync(kFull, smin, o));
            smax = fmaxf(smax, __shfl_xor_sync(kFull, smax, o));
            ns += __shfl_xor_sync(kFull, ns, o);
        }
    };
    if (warp == 0) {
        const int nloc = min(max(n - (int)rank * S, 0), S);  // keys of this CTA
#pragma unroll
        for (int i = 0; i < kSample; ++i) {  // kSample runs of 32 consecutive scores
            const int li = (int)((((int64_t)i * nloc) / kSample) & ~31) + lane;
            const float x = __uint_as_float(skeys[min(li, S - 1)]);
            if (li < nloc && isfinite(x)) {
                s1 += x;
                s2 = fmaf(x, x, s2);
                smin = fminf(smin, x);
                smax = fmaxf(smax, x);
                ++ns;
            }
        }
        reduce5();
    }
    if constexpr (CLUSTER) {
        if (tid == 0) {
            xch[0] = __float_as_uint(s1);
            xch[1] = __float_as_uint(s2);
            xch[2] = __float_as_uint(smin);
            xch[3] = __float_as_uint(smax);
            xch[4] = ns;
        }
        cluster_sync();
        if (warp == 0) {  // lane q < CL: CTA q's values
            const bool in = (uint32_t)lane < CL;
            s1 = in ? __uint_as_float(ld_cluster_u32(&xch[0], lane)) : 0.f;
            s2 = in ? __uint_as_float(ld_cluster_u32(&xch[1], lane)) : 0.f;
            smin = in ? __uint_as_float(ld_cluster_u32(&xch[2], lane)) : INFINITY;
            smax = in ? __uint_as_float(ld_cluster_u32(&xch[3], lane)) : -INFINITY;
            ns = in ? ld_cluster_u32(&xch[4], lane) : 0u;
            reduce5();
        }
    }
    if (tid == 0) {
        bc[0] = __float_as_uint(s1);
        bc[1] = __float_as_uint(s2);
        bc[2] = __float_as_uint(smin);
        bc[3] = __float_as_uint(smax);
        bc[4] = ns;
    }
    __syncthreads();
    s1 = __uint_as_float(bc[0]);
    s2 = __uint_as_float(bc[1]);
    smin = __uint_as_float(bc[2]);
    smax = __uint_as_float(bc[3]);
    ns = bc[4];
    const float mean = s1 / (float)max(ns, 1u);
    const float sd = sqrtf(fmaxf(s2 / (float)max(ns, 1u) - mean * mean, 0.f));
    const float lo = fmaxf(smin, mean - 6.f * sd), hi = fminf(smax, mean + 6.f * sd);
    const float span = hi - lo, scl = (float)kSelBins / span;
    const bool use_float = ns > 0 && isfinite(mean) && isfinite(sd) && isfinite(span) && span > 0.f && isfinite(scl);

    // 2. first pass: keys in place of the scores, bins beside them, counts
#pragma unroll 8
    for (int j = 0; j < nk; ++j) {
        const float x = __uint_as_float(skeys[lbase + 32 * j]);
        const uint32_t k = order_key(x);
        const uint32_t b = first_bin(x, k, use_float, lo, scl);
        skeys[lbase + 32 * j] = k;
        sbin[lbase + 32 * j] = (uint16_t)b;
        atomicAdd(&hist[0][b], 1u);
    }
    csync();  // every CTA's counts are complete

    // boundary bin of this pass's counts (the cluster's: summed from the
    // peers' histograms with 16-byte loads): thread t sums bins kSelBins -
    // (t+1)*kBpt .. kSelBins - t*kBpt - 1 (highest first), one block scan of
    // the sums; pick = {bin, keys in higher bins}, or {kSelBins, 0} when no
    // bin holds the rem-th key (a broken count)
    uint32_t rem = (uint32_t)K;
    auto boundary = [&](int p) {
        const uint32_t *h = hist[p];
        if constexpr (CLUSTER) {
            if (tid < kSelBins / 4) {
                uint4 s = make_uint4(0u, 0u, 0u, 0u);
                for (uint32_t q = 0; q < CL; ++q) {
                    const uint4 y = ld_cluster_v4(&hist[p][4 * tid], q);
                    s.x += y.x;
                    s.y += y.y;
                    s.z += y.z;
                    s.w += y.w;
                }
                *reinterpret_cast<uint4 *>(&hm[4 * tid]) = s;
            }
            __syncthreads();
            h = hm;
        }
        const int top = kSelBins - tid * kBpt;
        uint32_t hc[kBpt], c = 0;
#pragma unroll
        for (int i = 0; i < kBpt; ++i) {
            hc[i] = h[top - 1 - i];
            c += hc[i];
        }
        uint32_t inc = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, inc, o);
            if (lane >= o) inc += y;
        }
        if (tid == 0) {
            pick[0] = (uint32_t)kSelBins;
            pick[1] = 0u;
            pc[0] = 0xFFFFFFFFu;  // for the next pass's candidate counts
            pc[1] = 0u;
            pc[2] = 0u;
        }
        if (lane == 31) red[0][warp] = inc;
        __syncthreads();
        const uint32_t wtot = lane < kWarps ? red[0][lane] : 0u;
        uint32_t winc = wtot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, winc, o);
            if (lane >= o) winc += y;
        }
        uint32_t above = __shfl_sync(kFull, winc - wtot, warp) + inc - c;
        if (above < rem && rem <= above + c) {
#pragma unroll
            for (int i = 0; i < kBpt; ++i) {
                if (above + hc[i] >= rem) {
                    pick[0] = (uint32_t)(top - 1 - i);
                    pick[1] = above;
                    break;
                }
                above += hc[i];
            }
        }
        __syncthreads();
    };
    boundary(0);
    uint32_t pb = pick[0];
    bool failed = pb >= (uint32_t)kSelBins, done = false;
    rem -= pick[1];
    uint32_t above = 0u, cand = 0u;  // bit j: key j is above the candidates / a candidate
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll 8
    for (int j = 0; j < nk; ++j) {
        const uint32_t b = sbin[lbase + 32 * j];
        above |= (b > pb ? 1u : 0u) << j;
        if (b == pb) {
            cand |= 1u << j;
            const uint32_t k = skeys[lbase + 32 * j];
            mn = min(mn, k);
            mx = max(mx, k);
        }
    }

    // 3. digit passes while many candidates differ, then the warp finish
    for (int pass = 1; pass <= 4 && !failed; ++pass) {
        // the CTA's candidates' min, max and count: shared atomics of the
        // lanes that hold any (few after the first pass)
        if (cand != 0u) {
            atomicMin(&pc[0], mn);
            atomicMax(&pc[1], mx);
            atomicAdd(&pc[2], (uint32_t)__popc(cand));
        }
        __syncthreads();
        mn = pc[0];
        mx = pc[1];
        uint32_t cnt = pc[2];
        if constexpr (CLUSTER) {
            if (tid == 0) {
                xch[5] = mn;
                xch[6] = mx;
                xch[7] = cnt;
            }
            cluster_sync();
            if (warp == 0) {
                const bool in = (uint32_t)lane < CL;
                mn = in ? ld_cluster_u32(&xch[5], lane) : 0xFFFFFFFFu;
                mx = in ? ld_cluster_u32(&xch[6], lane) : 0u;
                cnt = in ? ld_cluster_u32(&xch[7], lane) : 0u;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mn = min(mn, __shfl_xor_sync(kFull, mn, o));
                    mx = max(mx, __shfl_xor_sync(kFull, mx, o));
                    cnt += __shfl_xor_sync(kFull, cnt, o);
                }
                if (lane == 0) {
                    bc[0] = mn;
                    bc[1] = mx;
                    bc[2] = cnt;
                }
            }
            __syncthreads();
            mn = bc[0];
            mx = bc[1];
            cnt = bc[2];
        }
        if (mn == mx) {  // the candidates are all T
            done = true;
            break;
        }
        if (cnt <= (uint32_t)kSelWarpMax) {
            // this CTA's candidates to its list (and the cluster's lists
            // into one), then warp 0: lane l tests candidates l and l + 32
            if (tid == 0) pick[0] = 0u;
            __syncthreads();
            const uint32_t my = __popc(cand);
            if (my) {
                uint32_t at = atomicAdd(&pick[0], my);
                for (uint32_t cb = cand; cb != 0u; cb &= cb - 1u) {
                    const uint32_t k = skeys[lbase + 32 * (__ffs(cb) - 1)];
                    if (dcheck(at < (uint32_t)kSelWarpMax, kDbgSelect)) lst[at] = k;
                    ++at;
                }
            }
            __syncthreads();
            const uint32_t *g = lst;
            uint32_t m = min(pick[0], (uint32_t)kSelWarpMax);
            if constexpr (CLUSTER) {
                if (tid == 0) xch[8] = pick[0];
                cluster_sync();
                g = gl;
                m = 0;
                if (warp == 0)
                    for (uint32_t q = 0; q < CL; ++q) {
                        const uint32_t cq = min(ld_cluster_u32(&xch[8], q), (uint32_t)kSelWarpMax);
                        for (uint32_t i = lane; i < cq; i += 32)
                            if (dcheck(m + i < (uint32_t)kSelWarpMax, kDbgSelect)) gl[m + i] = ld_cluster_u32(&lst[i], q);
                        m = min(m + cq, (uint32_t)kSelWarpMax);
                    }
                __syncwarp();
            }
            if (warp == 0) {
#pragma unroll
                for (int h = 0; h < kSelWarpMax / 32; ++h) {
                    const uint32_t i0 = (uint32_t)(lane + 32 * h);
                    const uint32_t c = i0 < m ? g[i0] : 0u;
                    uint32_t n_gt = 0, n_ge = 0;
                    for (uint32_t i = 0; i < m; ++i) {
                        const uint32_t y = g[i];
                        n_gt += y > c ? 1u : 0u;
                        n_ge += y >= c ? 1u : 0u;
                    }
                    // T: fewer than rem candidates above it, at least rem not
                    // below it (equal candidates write the same values)
                    if (i0 < m && n_gt < rem && rem <= n_ge) {
                        pick[0] = c;
                        pick[1] = rem - n_gt;  // keys equal to T still to take (>= 1)
                    }
                }
            }
            __syncthreads();
            mn = pick[0];
            rem = pick[1];
            done = true;
            break;
        }
        // a digit pass: 11 bits below the bits the candidates share
        const int p = pass & 1;
        const int top_bit = 31 - __clz(mn ^ mx);
        const int shift = top_bit > 10 ? top_bit - 10 : 0;
        for (int i = tid; i < kSelBins; i += THREADS) hist[p][i] = 0u;
        __syncthreads();
        for (uint32_t cb = cand; cb != 0u; cb &= cb - 1u) {
            const uint32_t k = skeys[lbase + 32 * (__ffs(cb) - 1)];
            atomicAdd(&hist[p][(k >> shift) & (uint32_t)(kSelBins - 1)], 1u);
        }
        csync();
        boundary(p);
        pb = pick[0];
        if (pb >= (uint32_t)kSelBins) {
            failed = true;
            break;
        }
        rem -= pick[1];
        mn = 0xFFFFFFFFu;
        mx = 0u;
        for (uint32_t cb = cand; cb != 0u; cb &= cb - 1u) {
            const int j = __ffs(cb) - 1;
            const uint32_t k = skeys[lbase + 32 * j];
            const uint32_t b = (k >> shift) & (uint32_t)(kSelBins - 1);
            if (b != pb) {
                cand &= ~(1u << j);
                if (b > pb) above |= 1u << j;
            } else {
                mn = min(mn, k);
                mx = max(mx, k);
            }
        }
    }

    // 4. ordered compaction (T = mn; rem keys equal to T to take).  Per lane
    //    the masks of its keys above T (gtm) and equal to T (eqm).  Row j of
    //    a warp (its keys j of every lane, in index order) is one ballot,
    //    kept by lane j; the rows give the warp's counts, and the counts of
    //    the warps (and CTAs) before it give its first output position and
    //    the equal keys it takes.  A key's position is its warp's, plus the
    //    keys taken in the rows before its own, plus the lanes before it in
    //    its row.
    if (!dcheck(done && !failed && rem >= 1u && rem <= (uint32_t)K, kDbgSelect) || !done || failed) {
        for (int i = (int)rank * THREADS + tid; i < K; i += (int)CL * THREADS) out[i] = -1;
    } else {
        const uint32_t T = mn;
        uint32_t gtm = above, eqm = 0u;
        for (uint32_t cb = cand; cb != 0u; cb &= cb - 1u) {
            const int j = __ffs(cb) - 1;
            const uint32_t k = skeys[lbase + 32 * j];
            gtm |= (k > T ? 1u : 0u) << j;
            eqm |= (k == T ? 1u : 0u) << j;
        }
        // this lane's rows, and the warp's counts from a scan of the rows
        uint32_t rgt = 0u, req = 0u, eq = 0u;
#pragma unroll 8
        for (int j = 0; j < kpt; ++j) {
            const uint32_t r = __ballot_sync(kFull, (gtm >> j) & 1u);
            rgt = lane == j ? r : rgt;
        }
        if (__any_sync(kFull, eqm != 0u)) {
            for (int j = 0; j < kpt; ++j) {
                const uint32_t r = __ballot_sync(kFull, (eqm >> j) & 1u);
                req = lane == j ? r : req;
            }
            eq = warp_sum_u32(__popc(req));
        }
        const uint32_t rcg = __popc(rgt);
        uint32_t rig = rcg;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, rig, o);
            if (lane >= o) rig += y;
        }
        const uint32_t gt = __shfl_sync(kFull, rig, 31);
        uint32_t *wcnt = hist[1];  // [0, 32): warps' keys above T, [32, 64): equal; [64, 128): before them
        if (lane == 0) {
            wcnt[warp] = gt;
            wcnt[32 + warp] = eq;
        }
        __syncthreads();
        if (warp == 0) {
            const uint32_t g = lane < kWarps ? wcnt[lane] : 0u, e = lane < kWarps ? wcnt[32 + lane] : 0u;
            uint32_t gi = g, ei = e;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t yg = __shfl_up_sync(kFull, gi, o), ye = __shfl_up_sync(kFull, ei, o);
                if (lane >= o) {
                    gi += yg;
                    ei += ye;
                }
            }
            wcnt[64 + lane] = gi - g;
            wcnt[96 + lane] = ei - e;
            if constexpr (CLUSTER) {
                const uint32_t cta_gt = __shfl_sync(kFull, gi, 31), cta_eq = __shfl_sync(kFull, ei, 31);
                if (lane == 0) {
                    xch[9] = cta_gt;
                    xch[10] = cta_eq;
                }
            }
        }
        if constexpr (CLUSTER) {
            cluster_sync();
            if (warp == 0) {  // the CTAs before this one
                const bool in = (uint32_t)lane < rank;
                const uint32_t cg = warp_sum_u32(in ? ld_cluster_u32(&xch[9], lane) : 0u);
                const uint32_t ce = warp_sum_u32(in ? ld_cluster_u32(&xch[10], lane) : 0u);
                if (lane == 0) {
                    bc[0] = cg;
                    bc[1] = ce;
                }
            }
        }
        __syncthreads();
        uint32_t gt_before = wcnt[64 + warp], eq_before = wcnt[96 + warp];
        if constexpr (CLUSTER) {
            gt_before += bc[0];
            eq_before += bc[1];
        }
        const uint32_t take = eq_before >= rem ? 0u : min(eq, rem - eq_before);
        const uint32_t pos = gt_before + min(eq_before, rem);
        const uint32_t below = (1u << lane) - 1u;
        // the equal keys taken: the warp's first `take`, by row then lane
        uint32_t keep = 0u;
        if (take >= eq) {
            keep = req;
        } else if (take > 0u) {
            const uint32_t ec = __popc(req);
            uint32_t ei = ec;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFull, ei, o);
                if (lane >= o) ei += y;
            }
            const uint32_t epre = ei - ec;
            uint32_t kk = take > epre ? min(ec, take - epre) : 0u, m = req;
            for (; kk > 0u; --kk) {  // the lowest kk lanes of the row
                keep |= m & (0u - m);
                m &= m - 1u;
            }
        }
        const uint32_t myrow = rgt | keep;
        uint32_t rc = rcg, ri = rig;  // the rows' counts, again when equal keys join them
        if (__any_sync(kFull, keep != 0u)) {
            rc = __popc(myrow);
            ri = rc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFull, ri, o);
                if (lane >= o) ri += y;
            }
        }
        uint32_t *wrow = hist[0] + 64 * warp;  // [row masks | keys in the rows before], kWarps * 64 <= kSelBins
        wrow[lane] = myrow;
        wrow[32 + lane] = ri - rc;
        __syncwarp();
        uint32_t selm = gtm;  // this lane's keys taken
        for (uint32_t eb = take > 0u ? eqm : 0u; eb != 0u; eb &= eb - 1u) {
            const int j = __ffs(eb) - 1;
            selm |= ((wrow[j] >> lane) & 1u) << j;
        }
        for (uint32_t sb = selm; sb != 0u; sb &= sb - 1u) {
            const int j = __ffs(sb) - 1;
            const uint32_t at = pos + wrow[32 + j] + __popc(wrow[j] & below);
            if (dcheck(at < (uint32_t)K, kDbgSelect)) out[at] = base + 32 * j;
        }
    }
    if constexpr (CLUSTER) cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace kvq
