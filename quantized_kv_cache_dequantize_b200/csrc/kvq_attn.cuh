// kvq_attn.cuh -- batched split-K decode attention straight over packed b-bit
// KV caches plus a bf16 recent window.
//
// "Agent Memory Below the Prompt: Persistent Q4 KV Cache for Multi-Agent LLM
// Inference on Edge Devices", Abstract: quantized caches go directly into the
// attention layer and several agents' caches are attended at once
// (BatchQuantizedKVCache).  "QKVShare ...", Significato e Affermazioni: a
// fused quantized attention kernel in place of dequantize-then-attend.
// "Coordinated Mixed-Precision KV Cache Quantization ...", Abstract: a width
// per (agent, layer) and recent states kept in native precision.
//
// Work unit: (view, KV head, block of <= 8 query heads, chunk of tokens).
// A CTA of 4 warps owns one unit; each warp streams 16-token tiles of the
// chunk through its own ring of shared-memory stages filled by 1-D bulk async
// copies (one elected lane issues them; an mbarrier per stage counts the
// bytes).  Per tile, on tensor cores (mma.m16n8k16 bf16 -> fp32):
//   QK:  S^T[token][head] = codes[token][d] . q[d][head], one accumulator per
//        64-element group; the affine dequantisation is folded into the
//        epilogue:  logit = sum_g s_g * acc_g + mn_g * sum_{d in g} q_d.
//        Codes become exact bf16 integers with a LOP3 "magic exponent"
//        (128 + c) and one bf16x2 FMA; q is bf16 already, so every product is
//        exact.
//   softmax: online (running max and sum per head, base 2).
//   PV:  O^T[d][head] += codes^T[d][token] . (p * s)[token][head] plus the
//        min term sum_t p_t * mn_t per group; p*s is split into two bf16
//        terms (hi + lo, relative error <= 2^-17), and the 16x8 probability
//        tile is moved from the QK accumulator layout to the B-operand layout
//        with movmatrix.
// Window tiles (bf16 K/V) use the same tile loop with the values as operands.
// Each CTA merges its warps in a fixed order and writes its chunk's partial
// (m, l, O); the CTA that finishes a unit's last chunk (an atomic arrival
// counter, never a wait) merges the unit's chunks in chunk order, so results
// are bitwise reproducible and no CTA waits on another.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "kvq_debug.cuh"
#include "kvq_ptx.cuh"

namespace kvq {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kTile = 16;
constexpr int kMaxStages = 12;
constexpr int kHeadsPerCta = 8;
constexpr int kAttnMaxViews = 96;
constexpr int kMaxChunksPerUnit = 256;  // combine scratch: 2 * 256 * 8 + 8 floats in the ring area

struct AttnView {
    const uint8_t *codes[2];     // K, V packed rows [H_kv][cap][RB]
    const float *scalemin[2];    // [H_kv][cap][NG][2]
    const uint16_t *window[2];   // bf16 [H_kv][cap_w][D]
    int64_t cap_packed;
    int32_t n_packed;
    int32_t n_window;
    int32_t cap_window;
    int32_t window_head;
    int32_t bits;
    int32_t n_chunks_packed;     // the packed part's 32-token steps, split evenly
    int32_t n_chunks;            // packed + window chunks (window: 16-token steps)
    int32_t chunk_begin;         // first chunk index of this view in the launch
    int32_t seq_index;           // its sequence: row of q / out, arrival counter
    int32_t part_begin;          // partial slot of the view's chunk 0 (call-wide)
    int32_t seq_part_begin;      // partial slot of the sequence's first chunk
    int32_t seq_chunks;          // chunks of the whole sequence (all its views)
    int32_t dep_step[2];         // packed / window step whose rows the preceding append grid
                                 // writes (-1: none); with AttnParams::fused its copy waits
                                 // for that grid, every other copy starts at once
    int64_t score_off;           // score grids: float offset of the view's head-0 scores
    const int32_t *gather;       // packed position j holds row gather[j] of the head's rows
                                 // (written by the preceding grid); nullptr: row j
};

struct AttnParams {
    const uint16_t *q;           // bf16 [n_seqs][Hq][D]
    float *out;                  // fp32 [n_seqs][Hq][D]
    float *partials;             // workspace: chunk partials of the whole call
    uint32_t *counters;          // workspace: per (sequence, KV head, head block), chunks finished
    uint32_t *status;            // workspace word 0
    uint64_t timeout_ns;
    float scale_log2;            // softmax_scale * log2(e)
    int32_t n_views;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t group;               // n_q_heads / n_kv_heads
    int32_t head_blocks;         // ceil(group / 8)
    int32_t ring_bytes;          // shared-memory ring per warp
    int32_t fused;               // 1: launched right behind this step's append grid (see dep_step)
    int32_t chain;               // 1: a later launch of a call: no wait at entry, wait before exit
    int32_t prefetch;            // 1: no grid that may still run before this one writes the packed
                                 // rows or windows (dep_step blocks aside), so the first ring
                                 // stages are filled before the dependency wait
    float *scores;               // score grids: [view][H_kv][n_packed] largest logit of the CTA's heads
    int64_t n_part_slots;        // extents for the debug build's checks: partial slots of the call,
    int64_t n_scores;            // floats of the score array,
    int32_t n_seqs;              // rows of q and out
    AttnView views[kAttnMaxViews];
};

// ------------------------------------------------------- code unpacking ---
//
// Codes enter the tensor cores as fp16 subnormals: a b-bit code moved, with
// LOP3/PRMT only, to bit offset o (o + b <= 10) of a 16-bit half whose
// exponent field is zero is the fp16 value c * 2^(o - 24), exactly.  The MMA
// multiplies it exactly with an fp16 operand and accumulates in fp32, so no
// conversion instruction and no offset constant is needed; the weight 2^o
// is compensated in the other operand (QK: in q) or in the output rows (PV).
//
// QK operand: lane (gid, tig) holds, for one token row and one group, the 16
// codes [16*tig, 16*tig + 16) of the group (2*B bytes at byte 2*B*tig).  They
// become 8 registers r = 0..7; half e of register r holds code qk_code<B>(r, e)
// at bit qk_off<B>(r, e), and register r feeds k-step r/2, half r%2 of the
// group's four m16n8k16 steps.  The same map places q (times 2^-offset) in the
// B operand, so the dot product sums matching elements.

template <int B>
__host__ __device__ constexpr int qk_code(int r, int e) {
    return B == 4 ? 8 * (r / 4) + (r % 4) + 4 * e
         : B == 8 ? 4 * (r / 2) + (r & 1) + 2 * e
         : B == 2 ? r + 8 * e
                  : (r == 7 ? 7 + e : r + 9 * e);
}

template <int B>
__host__ __device__ constexpr int qk_off(int r, int e) {
    return B == 4 ? 4 * (r & 1)
         : B == 8 ? 0
         : B == 2 ? (r < 5 ? 2 * r : 2 * (r - 3))
                  : (r == 7 ? (e ? 6 : 3) : 3 * (r % 3));
}

template <int B>
__device__ __forceinline__ void qk_unpack(const uint8_t *seg, uint32_t (&r)[8]);

template <>
__device__ __forceinline__ void qk_unpack<4>(const uint8_t *seg, uint32_t (&r)[8]) {
    // two words of 8 nibbles; per word: nibbles (0,4) and (1,5) in place at
    // offsets 0 and 4, bytes 1 and 3 moved down for nibbles (2,6) and (3,7)
    const uint2 w = *reinterpret_cast<const uint2 *>(seg);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t wk = k ? w.y : w.x;
        const uint32_t x = prmt(wk, 0u, 0x4341u);
        r[4 * k + 0] = wk & 0x000F000Fu;
        r[4 * k + 1] = wk & 0x00F000F0u;
        r[4 * k + 2] = x & 0x000F000Fu;
        r[4 * k + 3] = x & 0x00F000F0u;
    }
}

template <>
__device__ __forceinline__ void qk_unpack<8>(const uint8_t *seg, uint32_t (&r)[8]) {
    // four words of 4 bytes: bytes (0,2) in place, bytes (1,3) moved down
    // (the zero second source clears the high bytes)
    const uint4 w = *reinterpret_cast<const uint4 *>(seg);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        r[2 * k] = ws[k] & 0x00FF00FFu;
        r[2 * k + 1] = prmt(ws[k], 0u, 0x4341u);
    }
}

template <>
__device__ __forceinline__ void qk_unpack<2>(const uint8_t *seg, uint32_t (&r)[8]) {
    // one word, code j at bit 2j (halves: codes 0..7 and 8..15): codes 0..4 of
    // each half in place at offsets 0..8, codes 5..7 at offsets 4..8 after >> 6
    const uint32_t w = *reinterpret_cast<const uint32_t *>(seg);
    const uint32_t y = w >> 6;
    r[0] = w & 0x00030003u;
    r[1] = w & 0x000C000Cu;
    r[2] = w & 0x00300030u;
    r[3] = w & 0x00C000C0u;
    r[4] = w & 0x03000300u;
    r[5] = y & 0x00300030u;
    r[6] = y & 0x00C000C0u;
    r[7] = y & 0x03000300u;
}

template <>
__device__ __forceinline__ void qk_unpack<3>(const uint8_t *seg, uint32_t (&r)[8]) {
    // 16 codes x 3 bits = 6 bytes at a 2-byte-aligned address, code j at bit
    // 3j.  16-bit windows at bits 9k hold codes 3k..3k+2 at offsets 0, 3, 6;
    // windows k and k+3 are paired into one word.
    const uintptr_t addr = reinterpret_cast<uintptr_t>(seg);
    const uint32_t *wp = reinterpret_cast<const uint32_t *>(addr & ~uintptr_t(3));
    const uint32_t sh = (uint32_t)(addr & 3u) * 8u;  // 0 or 16
    const uint32_t w0 = wp[0], w1 = wp[1];
    const uint32_t lo = __funnelshift_r(w0, w1, sh);  // bits 0..31 of the segment
    const uint32_t hi = w1 >> sh;                     // bits 32..47 (above: not used)
    const uint32_t p0 = prmt(lo, __funnelshift_r(lo, hi, 27), 0x5410u);            // codes 0..2 | 9..11
    const uint32_t x9 = __funnelshift_r(lo, hi, 9);
    const uint32_t p1 = prmt(x9, hi >> 4, 0x5410u);                                  // codes 3..5 | 12..14
    const uint32_t x18 = __funnelshift_r(lo, hi, 18);
    const uint32_t p2 = prmt(x18, hi >> 13, 0x5410u);                                // codes 6..8 | 15
    r[0] = p0 & 0x00070007u;
    r[1] = p0 & 0x00380038u;
    r[2] = p0 & 0x01C001C0u;
    r[3] = p1 & 0x00070007u;
    r[4] = p1 & 0x00380038u;
    r[5] = p1 & 0x01C001C0u;
    r[6] = p2 & 0x00070007u;
    r[7] = prmt(x18, x18, 0x1010u) & 0x01C00038u;  // codes 7 (offset 3) | 8 (offset 6)
}

// PV operand: O^T rows d, columns heads; the A fragment pairs two tokens per
// register.  Lane (gid, tig) loads, for tokens 2tig, 2tig+1, 2tig+8, 2tig+9 of
// a 16-token tile, the 8 codes d = 8*gid .. 8*gid+7 of the group (B bytes at
// byte B*gid).  d-tile t's row gid is d = 8*gid + 2t, its row gid+8 is
// d = 8*gid + 2t + 1; their codes sit at bit pv_off<B>(t, odd) of fp16
// subnormals, so output row d accumulates 2^(pv_off - 24) times its value.
template <int B>
__host__ __device__ constexpr int pv_off(int t, int odd) {
    return B == 4 ? 4 * odd
         : B == 8 ? 0
         : B == 2 ? (odd ? (t == 0 ? 2 : t == 1 ? 6 : t == 2 ? 4 : 8) : (t == 0 ? 0 : t == 1 ? 4 : t == 2 ? 8 : 6))
                  : (odd ? (t == 0 ? 3 : t == 1 ? 0 : t == 2 ? 0 : 6) : (t == 0 ? 0 : t == 1 ? 6 : 3));
}

__device__ __forceinline__ uint32_t load24(const uint8_t *s) {
    // 3 bytes at any address, as the low 24 bits of a word
    const uintptr_t a = reinterpret_cast<uintptr_t>(s);
    const uint32_t *wp = reinterpret_cast<const uint32_t *>(a & ~uintptr_t(3));
    return __funnelshift_r(wp[0], wp[1], (uint32_t)(a & 3u) * 8u);
}

// The 8 codes of one token row for this lane (see above), low bits.
template <int B>
__device__ __forceinline__ uint2 pv_row(const uint8_t *s) {
    if constexpr (B == 8) return *reinterpret_cast<const uint2 *>(s);
    else if constexpr (B == 4) return make_uint2(*reinterpret_cast<const uint32_t *>(s), 0u);
    else if constexpr (B == 2) return make_uint2(*reinterpret_cast<const uint16_t *>(s), 0u);
    else return make_uint2(load24(s), 0u);
}

// Registers of d-tile t for the token pair (a, b): x[0] = row gid (even d),
// x[1] = row gid+8 (odd d).
template <int B>
__device__ __forceinline__ void pv_pair(uint2 a, uint2 b, uint32_t (&x)[4][2]) {
    if constexpr (B == 4) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint32_t p = prmt(a.x, b.x, (uint32_t)(t | ((4 + t) << 8)));  // byte t of a | of b
            x[t][0] = p & 0x000F000Fu;
            x[t][1] = p & 0x00F000F0u;
        }
    } else if constexpr (B == 8) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint32_t sa = t < 2 ? a.x : a.y, sb = t < 2 ? b.x : b.y;
            const uint32_t k = (uint32_t)(2 * t) & 3u;
            x[t][0] = prmt(sa, sb, k | ((4u + k) << 8)) & 0x00FF00FFu;
            x[t][1] = prmt(sa, sb, (k + 1u) | ((5u + k) << 8)) & 0x00FF00FFu;
        }
    } else if constexpr (B == 2) {
        const uint32_t p = prmt(a.x, b.x, 0x5410u);  // the 16 bits of a | of b
        const uint32_t y = p >> 6;
        x[0][0] = p & 0x00030003u;
        x[0][1] = p & 0x000C000Cu;
        x[1][0] = p & 0x00300030u;
        x[1][1] = p & 0x00C000C0u;
        x[2][0] = p & 0x03000300u;
        x[2][1] = y & 0x00300030u;
        x[3][0] = y & 0x00C000C0u;
        x[3][1] = y & 0x03000300u;
    } else {
        const uint32_t p = prmt(a.x, b.x, 0x5410u);                // codes 0..4 of a | of b
        const uint32_t y = p >> 9;                                  // codes 3, 4 at offsets 0, 3
        const uint32_t q = prmt(a.x >> 15, b.x >> 15, 0x5410u);    // codes 5..7 at offsets 0, 3, 6
        x[0][0] = p & 0x00070007u;
        x[0][1] = p & 0x00380038u;
        x[1][0] = p & 0x01C001C0u;
        x[1][1] = y & 0x00070007u;
        x[2][0] = y & 0x00380038u;
        x[2][1] = q & 0x00070007u;
        x[3][0] = q & 0x00380038u;
        x[3][1] = q & 0x01C001C0u;
    }
}

// ------------------------------------------------------------ per-warp ----

// 2^x on the special-function unit (relative error about 2^-22; 2^-inf = 0)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

template <int NG>
struct WarpState {
    float o[NG][4][4];      // O^T tiles: group g, d-tile t; (row gid|gid+8) x (head 2tig|2tig+1)
    float mt[NG][2];        // min-term partial sums, heads 2tig, 2tig+1
    float m[2];             // running max (log2 units), heads 2tig, 2tig+1
    float l[2];             // running sum (partial over this lane's rows)
    uint32_t bq[NG][4][2];  // q as B operand: group, k-step, (b0b1, b2b3); fp16 (packed items) or bf16 (window)
    float qsum[NG][2];      // packed items: sum of q over each group / 2^(10 + eq), heads 2tig, 2tig+1
    float pscale;           // packed items: p*s enters the PV MMA times pscale (a power of two) ...
    float plimit;           // ... chosen so that p*s*pscale < 2^15 while V scales stay below plimit
};

// Online-softmax step over R row-sets (R = 2: one 16-token tile, rows gid and
// gid+8; R = 4: two tiles).  lg[r][j] are base-2 logits of this lane's rows
// for heads 2tig, 2tig+1; they are replaced by the probabilities relative to
// the new running max.
// The running max is only moved when a tile exceeds it by more than
// kLazyMax (log2 units): probabilities relative to a stale max stay below
// 2^kLazyMax, harmless in fp32 sums and bf16 hi/lo operands, and the O rescale
// (32+ multiplies) becomes rare instead of firing on most early tiles.  One
// warp vote decides whether any lane's rows exceed it; only then are the
// per-head maxima reduced across the warp (most tiles skip the shuffles).
constexpr float kLazyMax = 8.0f;

template <int NG, int R>
__device__ __forceinline__ void softmax_step_n(WarpState<NG> &st, float (&lg)[R][2]) {
    float alpha[2] = {1.f, 1.f};
    float tl[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        tl[j] = lg[0][j];
#pragma unroll
        for (int r = 1; r < R; ++r) tl[j] = fmaxf(tl[j], lg[r][j]);
    }
    const bool move = __any_sync(0xFFFFFFFFu, tl[0] > st.m[0] + kLazyMax || tl[1] > st.m[1] + kLazyMax);
    if (move) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float t = tl[j];
            t = fmaxf(t, __shfl_xor_sync(0xFFFFFFFFu, t, 4));
            t = fmaxf(t, __shfl_xor_sync(0xFFFFFFFFu, t, 8));
            t = fmaxf(t, __shfl_xor_sync(0xFFFFFFFFu, t, 16));
            const float mnew = (t > st.m[j] + kLazyMax) ? t : st.m[j];
            alpha[j] = fast_exp2(st.m[j] - mnew);
            st.m[j] = mnew;
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float mnew = st.m[j];
        float sum = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            lg[r][j] = fast_exp2(lg[r][j] - mnew);
            sum += lg[r][j];
        }
        st.l[j] = fmaf(st.l[j], alpha[j], sum);
    }
    if (move && __any_sync(0xFFFFFFFFu, alpha[0] != 1.0f || alpha[1] != 1.0f)) {
#pragma unroll
        for (int g = 0; g < NG; ++g) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                st.o[g][t][0] *= alpha[0];
                st.o[g][t][1] *= alpha[1];
                st.o[g][t][2] *= alpha[0];
                st.o[g][t][3] *= alpha[1];
            }
            st.mt[g][0] *= alpha[0];
            st.mt[g][1] *= alpha[1];
        }
    }
}

// hi/lo bf16 split of the 16x8 tile (rows gid, gid+8; heads 2tig, 2tig+1)
// and transpose of both halves to the B-operand layout (tokens along k).
__device__ __forceinline__ void split_transpose(float a0, float a1, float b0, float b1, uint32_t &bh0,
                                                uint32_t &bh1, uint32_t &bl0, uint32_t &bl1) {
    const uint32_t h0 = pack_bf16x2(a0, a1);
    const uint32_t h1 = pack_bf16x2(b0, b1);
    const uint32_t l0 = pack_bf16x2(a0 - bf16lo_to_f32(h0), a1 - bf16hi_to_f32(h0));
    const uint32_t l1 = pack_bf16x2(b0 - bf16lo_to_f32(h1), b1 - bf16hi_to_f32(h1));
    bh0 = movmatrix_trans(h0);
    bh1 = movmatrix_trans(h1);
    bl0 = movmatrix_trans(l0);
    bl1 = movmatrix_trans(l1);
}

// QK of one 16-token tile of packed codes: codes rows at `kc` (row stride RB),
// K scale/min rows at `ks` ([row][NG] float2), over the warp's groups g0 ..
// g0+NGW-1.  The fp16 MMA accumulates sum_d c_d q_d 2^(-10-eq) per group
// exactly scaled, so the group's contribution is s*acc + mn*qsum (qsum carries
// the same factor).  Writes the raw sums of rows gid, gid+8 (l[0], l[1]) for
// heads 2tig, 2tig+1; the caller adds a team partner's groups, scales to
// base-2 logits and masks rows past the valid count.
template <int B, int NG, int NGW>
__device__ __forceinline__ void packed_qk_tile(const WarpState<NGW> &st, const uint8_t *kc, const uint8_t *ks_bytes,
                                               int gid, int tig, int g0, float (&l)[2][2]) {
    constexpr int RB = 8 * B * NG;
    const float2 *sm = reinterpret_cast<const float2 *>(ks_bytes);
    const uint8_t *row0 = kc + gid * RB + 2 * B * tig;
    const uint8_t *row1 = row0 + 8 * RB;
    float l00 = 0.f, l01 = 0.f, l10 = 0.f, l11 = 0.f;
#pragma unroll
    for (int gg = 0; gg < NGW; ++gg) {
        const int g = g0 + gg;
        uint32_t a0[8], a1[8];
        qk_unpack<B>(row0 + g * 8 * B, a0);
        qk_unpack<B>(row1 + g * 8 * B, a1);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_f16_16816(acc, a0[2 * s], a1[2 * s], a0[2 * s + 1], a1[2 * s + 1], st.bq[gg][s][0], st.bq[gg][s][1]);
        const float2 k0 = sm[gid * NG + g], k1 = sm[(gid + 8) * NG + g];
        l00 = fmaf(k0.x, acc[0], fmaf(k0.y, st.qsum[gg][0], l00));
        l01 = fmaf(k0.x, acc[1], fmaf(k0.y, st.qsum[gg][1], l01));
        l10 = fmaf(k1.x, acc[2], fmaf(k1.y, st.qsum[gg][0], l10));
        l11 = fmaf(k1.x, acc[3], fmaf(k1.y, st.qsum[gg][1], l11));
    }
    l[0][0] = l00;
    l[0][1] = l01;
    l[1][0] = l10;
    l[1][1] = l11;
}

// QK of both (full) tiles of a packed block, raw sums; l rows: tile A gid,
// tile A gid+8, tile B gid, tile B gid+8.  The two tiles' MMA chains
// interleave.
template <int B, int NG, int NGW>
__device__ __forceinline__ void packed_qk_block(const WarpState<NGW> &st, const uint8_t *blk, int gid, int tig, int g0,
                                                float (&l)[4][2]) {
    constexpr int RB = 8 * B * NG;
    const float2 *sm = reinterpret_cast<const float2 *>(blk + 4 * kTile * RB);
    const uint8_t *row0 = blk + gid * RB + 2 * B * tig;
#pragma unroll
    for (int r = 0; r < 4; ++r) l[r][0] = l[r][1] = 0.f;
#pragma unroll
    for (int gg = 0; gg < NGW; ++gg) {
        const int g = g0 + gg;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            uint32_t a0[8], a1[8];
            qk_unpack<B>(row0 + tt * kTile * RB + g * 8 * B, a0);
            qk_unpack<B>(row0 + tt * kTile * RB + 8 * RB + g * 8 * B, a1);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16_16816(acc, a0[2 * s], a1[2 * s], a0[2 * s + 1], a1[2 * s + 1], st.bq[gg][s][0],
                              st.bq[gg][s][1]);
            const float2 k0 = sm[(tt * kTile + gid) * NG + g], k1 = sm[(tt * kTile + gid + 8) * NG + g];
            l[2 * tt][0] = fmaf(k0.x, acc[0], fmaf(k0.y, st.qsum[gg][0], l[2 * tt][0]));
            l[2 * tt][1] = fmaf(k0.x, acc[1], fmaf(k0.y, st.qsum[gg][1], l[2 * tt][1]));
            l[2 * tt + 1][0] = fmaf(k1.x, acc[2], fmaf(k1.y, st.qsum[gg][0], l[2 * tt + 1][0]));
            l[2 * tt + 1][1] = fmaf(k1.x, acc[3], fmaf(k1.y, st.qsum[gg][1], l[2 * tt + 1][1]));
        }
    }
}

// Before the PV of a packed block: V scales of up to `rows` rows of the block
// (sm rows [row][NG] float2) against the warp's limit.  p (<= 2^8 under the
// lazy max) times s times pscale must stay below the fp16 range; when a scale
// reaches plimit, pscale drops to 2^(6 - floor(log2 s_max)) and the O
// accumulators (in p*s*pscale units) follow.  One warp reduction per block.
template <int NG, int NGW>
__device__ __forceinline__ void track_pscale(WarpState<NGW> &st, const uint8_t *vs_bytes, int rows, int gid, int g0) {
    const float2 *sm = reinterpret_cast<const float2 *>(vs_bytes);
    float mx = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int row = gid + 8 * q;  // rows gid, gid+8 of both tiles
        if (row < rows) {
#pragma unroll
            for (int gg = 0; gg < NGW; ++gg) mx = fmaxf(mx, sm[row * NG + g0 + gg].x);
        }
    }
    // scales are >= 0: their bit patterns order like the values
    const uint32_t wmax = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mx));
    if (__uint_as_float(wmax) >= st.plimit) {
        const int ex = max(-100, min(120, (int)(max(wmax, 0x0D800000u) >> 23) - 127));  // floor(log2 s_max)
        const float ps = __uint_as_float((uint32_t)(127 + 6 - ex) << 23);
        const float f = ps / st.pscale;  // a power of two: exact
#pragma unroll
        for (int g = 0; g < NGW; ++g)
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) st.o[g][t][e] *= f;
        st.pscale = ps;
        st.plimit = __uint_as_float((uint32_t)(127 + ex + 1) << 23);
    }
}

// hi/lo split of x for two fp16 terms: hi keeps 11 significant bits (exact
// in fp16 in its normal range), lo = x - hi is exact in fp32 and rounds once
// in fp16, so hi + lo carries x to about 2^-22.
__device__ __forceinline__ void split_f16(float x, float &hi, float &lo) {
    hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    lo = x - hi;
}

// O += a block's PV sums (one d-tile).  The tensor cores add an MMA's
// products to its fp32 accumulator after aligning them to the largest term
// and dropping the bits below, so chaining thousands of tiles through O
// (whose code terms are all >= 0) loses a little at every MMA, always
// downward; at 32K tokens in one chunk that came to about 2e-2 relative in
// the output, where the code and min terms cancel.  Each block's MMAs start
// from zero instead and O takes the block sum in round-to-nearest fp32 adds:
// the error no longer grows with the tokens a warp accumulates.
__device__ __forceinline__ void add_block(float (&o)[4], const float (&acc)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] += acc[e];
}

// PV of one packed block (two 16-token tiles): V codes rows at `vc` (row
// stride RB), V scale/min rows at `vs` ([row][NG] float2); p[2tt], p[2tt+1]
// are this lane's probabilities of tile tt's rows gid, gid+8.
// O^T[d][h] += codes^T[d][t] . (p s pscale)[t][h] on the fp16 tensor cores
// (codes as exact subnormals, p*s*pscale as a hi + lo pair of fp16 terms,
// relative error about 2^-22), group by group, both tiles into one zeroed
// accumulator that joins O through add_block; plus the min term
// sum_t p_t mn_t per group in fp32.  FULL == false: only the first n_valid
// rows hold tokens; a tile past them is skipped, and the scale/min of rows
// at or past n_valid are zeroed (stale stage bytes; p is 0 there but 0 * NaN
// would not be).
template <int B, int NG, int NGW, bool FULL>
__device__ __forceinline__ void packed_pv_block(WarpState<NGW> &st, const uint8_t *vc, const uint8_t *vs_bytes,
                                                int n_valid, const float (&p)[4][2], int gid, int tig, int g0) {
    constexpr int RB = 8 * B * NG;
    const float2 *sm = reinterpret_cast<const float2 *>(vs_bytes);
    const uint8_t *ta = vc + (2 * tig) * RB + B * gid;
#pragma unroll
    for (int gg = 0; gg < NGW; ++gg) {
        const int g = g0 + gg;
        float acc[4][4] = {};
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            if (!FULL && tt * kTile >= n_valid) break;  // warp-uniform
            const int r0 = tt * kTile + gid;
            float2 m0 = sm[r0 * NG + g], m1 = sm[(r0 + 8) * NG + g];
            if (!FULL) {
                if (r0 >= n_valid) m0 = make_float2(0.f, 0.f);
                if (r0 + 8 >= n_valid) m1 = make_float2(0.f, 0.f);
            }
            const float(&p0)[2] = p[2 * tt];
            const float(&p1)[2] = p[2 * tt + 1];
            st.mt[gg][0] = fmaf(p0[0], m0.y, fmaf(p1[0], m1.y, st.mt[gg][0]));
            st.mt[gg][1] = fmaf(p0[1], m0.y, fmaf(p1[1], m1.y, st.mt[gg][1]));
            const float s0 = m0.x * st.pscale, s1 = m1.x * st.pscale;
            // (p s pscale) of rows gid, gid+8 (heads 2tig, 2tig+1) as hi + lo,
            // moved to the B-operand layout (tokens along k)
            float h[4], l[4];
            split_f16(p0[0] * s0, h[0], l[0]);
            split_f16(p0[1] * s0, h[1], l[1]);
            split_f16(p1[0] * s1, h[2], l[2]);
            split_f16(p1[1] * s1, h[3], l[3]);
            const uint32_t bh0 = movmatrix_trans(pack_f16x2(h[0], h[1]));
            const uint32_t bh1 = movmatrix_trans(pack_f16x2(h[2], h[3]));
            const uint32_t bl0 = movmatrix_trans(pack_f16x2(l[0], l[1]));
            const uint32_t bl1 = movmatrix_trans(pack_f16x2(l[2], l[3]));
            const uint8_t *tr = ta + tt * kTile * RB + g * 8 * B;
            uint32_t xab[4][2], xcd[4][2];
            pv_pair<B>(pv_row<B>(tr), pv_row<B>(tr + RB), xab);
            pv_pair<B>(pv_row<B>(tr + 8 * RB), pv_row<B>(tr + 9 * RB), xcd);
#pragma unroll
            for (int t = 0; t < 4; ++t) mma_f16_16816(acc[t], xab[t][0], xab[t][1], xcd[t][0], xcd[t][1], bh0, bh1);
#pragma unroll
            for (int t = 0; t < 4; ++t) mma_f16_16816(acc[t], xab[t][0], xab[t][1], xcd[t][0], xcd[t][1], bl0, bl1);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) add_block(st.o[gg][t], acc[t]);
    }
}

// K half of a window tile: block = K rows [16][D] bf16, over the warp's
// groups g0 .. g0+NGW-1; raw sums of rows gid, gid+8 (l[0], l[1]) for heads
// 2tig, 2tig+1 (the caller adds a team partner's groups, scales and masks).
template <int NG, int NGW>
__device__ __forceinline__ void window_qk(const WarpState<NGW> &st, const uint8_t *blk, int gid, int tig, int g0,
                                          float (&l)[2][2]) {
    constexpr int D = 64 * NG;
    const uint16_t *k = reinterpret_cast<const uint16_t *>(blk);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int gg = 0; gg < NGW; ++gg) {
        const int g = g0 + gg;
        const uint4 *p0 = reinterpret_cast<const uint4 *>(k + gid * D + 64 * g + 16 * tig);
        const uint4 *p1 = reinterpret_cast<const uint4 *>(k + (gid + 8) * D + 64 * g + 16 * tig);
        const uint4 x0 = p0[0], x1 = p0[1], y0 = p1[0], y1 = p1[1];
        const uint32_t a0[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const uint32_t a1[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_bf16_16816(acc, a0[2 * s], a1[2 * s], a0[2 * s + 1], a1[2 * s + 1], st.bq[gg][s][0], st.bq[gg][s][1]);
    }
    l[0][0] = acc[0];
    l[0][1] = acc[1];
    l[1][0] = acc[2];
    l[1][1] = acc[3];
}

// V half of a window tile: block = V rows [16][D] bf16, the warp's groups.
template <int NG, int NGW, bool FULL>
__device__ __forceinline__ void window_pv(WarpState<NGW> &st, const uint8_t *blk, int n_valid,
                                          const float (&p)[2][2], int gid, int tig, int g0) {
    constexpr int D = 64 * NG;
    const uint16_t *v = reinterpret_cast<const uint16_t *>(blk);
    uint32_t bh0, bh1, bl0, bl1;
    split_transpose(p[0][0], p[0][1], p[1][0], p[1][1], bh0, bh1, bl0, bl1);
    const int ta = 2 * tig, tb = 2 * tig + 1, tc = 2 * tig + 8, td = 2 * tig + 9;
#pragma unroll
    for (int gg = 0; gg < NGW; ++gg) {
        const int col = 64 * (g0 + gg) + 8 * gid;
        uint4 xa = *reinterpret_cast<const uint4 *>(v + ta * D + col);
        uint4 xb = *reinterpret_cast<const uint4 *>(v + tb * D + col);
        uint4 xc = *reinterpret_cast<const uint4 *>(v + tc * D + col);
        uint4 xd = *reinterpret_cast<const uint4 *>(v + td * D + col);
        if (!FULL) {
            // stale rows may hold non-finite bit patterns: zero them (p is 0 there)
            if (ta >= n_valid) xa = make_uint4(0, 0, 0, 0);
            if (tb >= n_valid) xb = make_uint4(0, 0, 0, 0);
            if (tc >= n_valid) xc = make_uint4(0, 0, 0, 0);
            if (td >= n_valid) xd = make_uint4(0, 0, 0, 0);
        }
        const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
        const uint32_t wc[4] = {xc.x, xc.y, xc.z, xc.w}, wd[4] = {xd.x, xd.y, xd.z, xd.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint32_t a0 = prmt(wa[t], wb[t], 0x5410u), a1 = prmt(wa[t], wb[t], 0x7632u);
            const uint32_t a2 = prmt(wc[t], wd[t], 0x5410u), a3 = prmt(wc[t], wd[t], 0x7632u);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16_16816(acc, a0, a1, a2, a3, bh0, bh1);
            mma_bf16_16816(acc, a0, a1, a2, a3, bl0, bl1);
            add_block(st.o[gg][t], acc);
        }
    }
}

// Named barrier 1 + team for the two warps (64 threads) of a team, with the
// id as an immediate.
__device__ __forceinline__ void team_bar(int team) {
    if (team == 0) asm volatile("bar.sync 1, 64;\n" ::: "memory");
    else asm volatile("bar.sync 2, 64;\n" ::: "memory");
}

// Two warps of a team hold halves of head_dim: each has summed the QK terms
// of its groups; this adds the partner's (addition commutes, so both warps
// hold the same sums) and ANDs the two warps' copy-wait results.  xb: the
// team's exchange area, [2 parities][2 halves][32 lanes][8 floats] then
// [2 parities][2 halves] flags; alternating parities keep a write from racing
// the partner's read of the block before.  `bar` is the team's named barrier.
template <int R>
__device__ __forceinline__ bool team_add(float (&l)[R][2], float *xb, int parity, int half, int lane, int bar,
                                         bool ok) {
    static_assert(R == 2 || R == 4, "rows");
    float4 *mine = reinterpret_cast<float4 *>(xb + ((parity * 2 + half) * 32 + lane) * 8);
    const float4 *theirs = reinterpret_cast<const float4 *>(xb + ((parity * 2 + (half ^ 1)) * 32 + lane) * 8);
    int *flags = reinterpret_cast<int *>(xb + 2 * 2 * 32 * 8);
    mine[0] = make_float4(l[0][0], l[0][1], l[1][0], l[1][1]);
    if (R == 4) mine[1] = make_float4(l[R - 2][0], l[R - 2][1], l[R - 1][0], l[R - 1][1]);
    if (lane == 0) flags[parity * 2 + half] = ok ? 1 : 0;
    team_bar(bar - 1);
    const float4 a = theirs[0];
    l[0][0] += a.x;
    l[0][1] += a.y;
    l[1][0] += a.z;
    l[1][1] += a.w;
    if (R == 4) {
        const float4 b = theirs[1];
        l[R - 2][0] += b.x;
        l[R - 2][1] += b.y;
        l[R - 1][0] += b.z;
        l[R - 1][1] += b.w;
    }
    return ok && flags[parity * 2 + (half ^ 1)] != 0;
}

// The two warps' copy-wait results ANDed at the team barrier (flags after
// team_add's, same parity scheme).
__device__ __forceinline__ bool team_and(bool ok, float *xb, int parity, int half, int lane, int bar) {
    int *flags = reinterpret_cast<int *>(xb + 2 * 2 * 32 * 8) + 4;
    if (lane == 0) flags[parity * 2 + half] = ok ? 1 : 0;
    team_bar(bar - 1);
    return ok && flags[parity * 2 + (half ^ 1)] != 0;
}

// ---------------------------------------------------------------- kernel ---

__device__ __forceinline__ uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

// Warps per team: a team streams one sequence of steps through one ring and
// its warps split head_dim (head_dim 256: two warps of 128 each, so that a
// warp's accumulators and q operands stay within 128 registers).
template <int NG>
__host__ __device__ constexpr int attn_team_warps() {
    return NG == 4 ? 2 : 1;
}

template <int NG>
__host__ __device__ constexpr int attn_ctas_per_sm() {
    return NG == 3 ? 3 : 4;
}

// per team: [2 parities][2 halves][32 lanes][8 floats] of QK sums, then two
// sets of [2 parities][2 halves] flags
constexpr int kXchgFloats = 2 * 2 * 32 * 8 + 8;

template <int NG>
__host__ __device__ constexpr int attn_xchg_offset() {
    return (8 * 64 * NG * 2 + kAttnWarps * kMaxStages * 8 + 16 + 15) & ~15;
}

template <int NG>
__host__ __device__ constexpr int attn_header_bytes() {
    return (attn_xchg_offset<NG>() +
            (attn_team_warps<NG>() > 1 ? kAttnWarps / attn_team_warps<NG>() * kXchgFloats * 4 : 0) + 127) &
           ~127;
}

// Split-K combine of one unit (sequence, KV head, head block) whose n > 1
// chunk partials are in the workspace (the chunks of all the sequence's views,
// in view order, contiguous), run by the CTA that finished the unit's last
// chunk.  A partial is [O: 8 heads x D][m: 8][l: 8] floats.  Up to 8 chunks:
// every thread loads all chunks' (m, l) of its head and O of its 4 outputs in
// one round and merges them in chunk order.  More chunks: the CTA gathers
// every chunk's (m, l), reduces per head with warp shuffles, then sums the
// chunks' O in chunk order, 4 elements per thread and 8 chunks per batch of
// independent loads.  Fixed orders throughout: results are bitwise
// reproducible.  `scratch` holds 2 * kMaxChunksPerUnit * 8 + 8 floats.
template <int NG>
__device__ __forceinline__ void combine_unit(const AttnParams &p, const AttnView &V, int hk, int z,
                                             float *scratch) {
    constexpr int D = 64 * NG;
    constexpr int kSlot = kHeadsPerCta * (D + 2);  // floats per partial
    float *sm_w = scratch;                                        // m, then weight
    float *sm_l = scratch + kMaxChunksPerUnit * kHeadsPerCta;
    float *sm_L = scratch + 2 * kMaxChunksPerUnit * kHeadsPerCta;
    const int n = V.seq_chunks;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h0 = hk * p.group + z * kHeadsPerCta;
    const int nh = min(kHeadsPerCta, p.group - z * kHeadsPerCta);
    const int64_t slot0 = ((int64_t)V.seq_part_begin * p.n_kv_heads + hk) * p.head_blocks + z;
    const int64_t stride = (int64_t)p.n_kv_heads * p.head_blocks * kSlot;  // between chunks
    const float *part0 = p.partials + slot0 * kSlot;
    float4 *out4 = reinterpret_cast<float4 *>(p.out + ((int64_t)V.seq_index * p.n_q_heads + h0) * D);
    // the unit's chunk slots and output rows (debug build)
    if (!dcheck(n >= 1 && n <= kMaxChunksPerUnit && slot0 >= 0 &&
                    slot0 + (int64_t)(n - 1) * p.n_kv_heads * p.head_blocks < p.n_part_slots,
                kDbgAttnWorkspace) ||
        !dcheck(V.seq_index < p.n_seqs && h0 + nh <= p.n_q_heads, kDbgAttnIo))
        return;
    if (n <= 8) {
        // one round of loads: each thread fetches every chunk's (m, l) of its
        // head and O of its 4 outputs at once, then merges in chunk order
        const float4 *o4 = reinterpret_cast<const float4 *>(part0);
        for (int f = tid; f < nh * (D / 4); f += kAttnThreads) {
            const int j = f / (D / 4);
            float m[8], l[8];
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool ok = u < n;
                const float *pc = part0 + u * stride + kHeadsPerCta * D;
                m[u] = ok ? __ldcg(pc + j) : -INFINITY;
                l[u] = ok ? __ldcg(pc + kHeadsPerCta + j) : 0.f;
                v[u] = ok ? __ldcg(o4 + u * (stride / 4) + f) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float M = m[0];
#pragma unroll
            for (int u = 1; u < 8; ++u) M = fmaxf(M, m[u]);
            float L = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float w = (m[u] == -INFINITY) ? 0.f : fast_exp2(m[u] - M);
                L = fmaf(w, l[u], L);
                acc.x = fmaf(w, v[u].x, acc.x);
                acc.y = fmaf(w, v[u].y, acc.y);
                acc.z = fmaf(w, v[u].z, acc.z);
                acc.w = fmaf(w, v[u].w, acc.w);
            }
            out4[f] = make_float4(acc.x / L, acc.y / L, acc.z / L, acc.w / L);
        }
        return;
    }
    for (int i = tid; i < n * nh; i += kAttnThreads) {
        const int cc = i / nh, j = i - cc * nh;
        const float *pc = part0 + cc * stride + kHeadsPerCta * D;
        sm_w[cc * kHeadsPerCta + j] = __ldcg(pc + j);
        sm_l[cc * kHeadsPerCta + j] = __ldcg(pc + kHeadsPerCta + j);
    }
    __syncthreads();
    for (int j = warp; j < nh; j += kAttnWarps) {
        float M = -INFINITY;
        for (int cc = lane; cc < n; cc += 32) M = fmaxf(M, sm_w[cc * kHeadsPerCta + j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        float L = 0.f;
        for (int cc = lane; cc < n; cc += 32) {
            const float mc = sm_w[cc * kHeadsPerCta + j];
            const float w = (mc == -INFINITY) ? 0.f : fast_exp2(mc - M);
            sm_w[cc * kHeadsPerCta + j] = w;
            L = fmaf(w, sm_l[cc * kHeadsPerCta + j], L);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xFFFFFFFFu, L, o);
        if (lane == 0) sm_L[j] = L;
    }
    __syncthreads();
    const float4 *o4 = reinterpret_cast<const float4 *>(part0);
    const int64_t stride4 = stride / 4;
    for (int f = tid; f < nh * (D / 4); f += kAttnThreads) {
        const int j = f / (D / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c0 = 0; c0 < n; c0 += 8) {
            float4 v[8];
            float w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool ok = c0 + u < n;
                v[u] = ok ? __ldcg(o4 + (c0 + u) * stride4 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
                w[u] = ok ? sm_w[(c0 + u) * kHeadsPerCta + j] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc.x = fmaf(w[u], v[u].x, acc.x);
                acc.y = fmaf(w[u], v[u].y, acc.y);
                acc.z = fmaf(w[u], v[u].z, acc.z);
                acc.w = fmaf(w[u], v[u].w, acc.w);
            }
        }
        const float L = sm_L[j];
        out4[f] = make_float4(acc.x / L, acc.y / L, acc.z / L, acc.w / L);
    }
}

// BYTES (a multiple of 8) from src to dst as cp.async pieces: 16 bytes when
// BYTES is a multiple of 16, else 8 (both addresses aligned to the piece).
template <int BYTES>
__device__ __forceinline__ void cp_async_row(uint8_t *dst, const uint8_t *src) {
    constexpr int P = BYTES % 16 == 0 ? 16 : 8;
    // both addresses aligned to the piece (debug build; a refused row is skipped)
    if (!dcheck((((uintptr_t)dst | (uintptr_t)src) & (P - 1)) == 0, kDbgAttnPacked)) return;
#pragma unroll
    for (int i = 0; i < BYTES / P; ++i) cp_async<P>(dst + i * P, src + i * P);
}

// One work item: (view, KV head hk, query-head block z, chunk of tokens).
// The chunk is cut into steps (32 packed tokens, or 16 window tokens).  The
// CTA's warps form T = 4 / TW teams of TW warps; team t takes steps t, t+T,
// ...  A packed step is one block holding both halves of two 16-token tiles
// (K codes, V codes, K scale/min, V scale/min); a window step is two blocks
// (K rows, then V rows).  Blocks stream through the team's own ring of S
// equal slots, each with an mbarrier that counts the bytes of the block's
// bulk copies; lane 0 of the team's first warp issues them.  With TW = 1 a
// slot is refilled as soon as the warp has consumed it.  With TW = 2 the two
// warps split the head's groups: each computes the QK sums of its groups,
// they add each other's through shared memory at a named barrier (team_add),
// both run the same softmax, and each does the PV of its groups; a slot is
// refilled at that barrier, once both warps are past the block it held.
// SCORE: the packed part's K rows only (no V copies, no softmax, no PV): each
// token's largest logit over the CTA's query heads (base-2 units, scale_log2
// applied) goes to p.scores; no partials, no combine.
template <int NG, int B, bool WINDOW, bool SCORE = false>
__device__ __forceinline__ void attn_item(const AttnParams &p, const AttnView &V, int c, int hk, int z,
                                          uint8_t *smem) {
    constexpr int D = 64 * NG;
    constexpr int RB = 8 * B * NG;
    constexpr int TW = attn_team_warps<NG>();
    constexpr int T = kAttnWarps / TW;    // teams per CTA
    constexpr int NGW = NG / TW;          // groups per warp
    constexpr int kStepTok = WINDOW ? kTile : 2 * kTile;
    constexpr int kBlkPerStep = WINDOW ? 2 : 1;
    // packed block: [K codes 32*RB][V codes 32*RB][K sm 32*NG*8][V sm 32*NG*8]
    constexpr uint32_t kOffV = 2 * kTile * RB, kOffKs = 4 * kTile * RB, kOffVs = kOffKs + 2 * kTile * NG * 8;
    constexpr uint32_t kBlk = WINDOW ? (uint32_t)(kTile * D * 2) : (uint32_t)(kOffVs + 2 * kTile * NG * 8);
    uint16_t *q_s = reinterpret_cast<uint16_t *>(smem);                              // [8][D]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 8 * D * 2);                // [4][kMaxStages]
    uint8_t *rings = smem + attn_header_bytes<NG>();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const int team = warp / TW, half = warp % TW, g0 = half * NGW;
    float *xb = reinterpret_cast<float *>(smem + attn_xchg_offset<NG>()) + team * kXchgFloats;
    const int h0 = hk * p.group + z * kHeadsPerCta;
    const int nh = min(kHeadsPerCta, p.group - z * kHeadsPerCta);
    // this chunk's steps: the part's steps split into equal runs (+-1 step)
    const int n_part = WINDOW ? V.n_window : V.n_packed;
    const int steps_part = (n_part + kStepTok - 1) / kStepTok;
    const int chunks_part = WINDOW ? V.n_chunks - V.n_chunks_packed : V.n_chunks_packed;
    const int ci = WINDOW ? c - V.n_chunks_packed : c;
    const int s0 = (int)((int64_t)ci * steps_part / chunks_part);
    const int s1 = (int)((int64_t)(ci + 1) * steps_part / chunks_part);
    const int64_t tok0 = (int64_t)s0 * kStepTok;
    const int n_tok = (int)min((int64_t)(s1 - s0) * kStepTok, (int64_t)n_part - tok0);
    const int n_steps = s1 - s0;
    const int n_my = (team < n_steps) ? (n_steps - team + T - 1) / T : 0;
    const int n_blocks = kBlkPerStep * n_my;
    const int team_ring = TW * p.ring_bytes;
    const int S = min(kMaxStages, (int)(team_ring / kBlk));
    uint8_t *ring = rings + (size_t)team * team_ring;
    uint64_t *wbar = bars + team * kMaxStages;
    constexpr int kAdvTok = T * kStepTok;  // tokens between a team's steps

    // Copy sources at this team's first step; incremental from then on (no
    // integer division on the per-block path).
    const uint8_t *src_kc = nullptr, *src_vc = nullptr;
    const float *src_ks = nullptr, *src_vs = nullptr;
    const uint16_t *win_k = nullptr, *win_v = nullptr;
    int win_phys = 0;
    if (!WINDOW) {
        const int64_t row = (int64_t)hk * V.cap_packed + tok0 + kStepTok * team;
        src_kc = V.codes[0] + row * RB;
        src_vc = V.codes[1] + row * RB;
        src_ks = V.scalemin[0] + row * NG * 2;
        src_vs = V.scalemin[1] + row * NG * 2;
    } else {
        win_k = V.window[0] + (int64_t)hk * V.cap_window * D;
        win_v = V.window[1] + (int64_t)hk * V.cap_window * D;
        win_phys = V.cap_window > 0 ? (int)(((int64_t)V.window_head + tok0 + kStepTok * team) % V.cap_window) : 0;
    }
    // Copy issue: every lane of the team's first warp keeps the (warp-uniform)
    // bookkeeping and runs issue_next; only its lane 0's async instructions are
    // predicated on.
    const bool issuer = lane == 0 && half == 0;
    int issue_blk = 0, issue_slot = 0, issue_left = n_tok - kStepTok * team;
    int issue_step = s0 + team;  // step index within the part
    // gathered packed rows: position of the next block's first row in the
    // gather list; lane r of the issuing warp copies row r of a block
    const int32_t *gather = (WINDOW || SCORE) ? nullptr : V.gather;
    int64_t issue_pos = tok0 + kStepTok * team;
    const int dep_step = p.fused ? V.dep_step[WINDOW ? 1 : 0] : -1;
    auto issue_next = [&]() {
        // the block the preceding append grid writes: wait for that grid first
        if (issue_step == dep_step && (!WINDOW || (issue_blk & 1) == 0)) pdl_wait();
        uint8_t *dst = ring + (size_t)issue_slot * kBlk;
        uint64_t *bar = &wbar[issue_slot];
        const int n = min(kStepTok, issue_left);
        const bool stage_ok = dcheck((size_t)(issue_slot + 1) * kBlk <= (size_t)team_ring, kDbgAttnStage);
        if (!WINDOW && gather != nullptr) {
            // K and V codes and scale/min of up to 32 selected rows, one row
            // per lane; the slot's barrier counts one arrival per lane, made
            // once that lane's copies have landed (rows past n stay stale
            // and are masked like a ragged tail)
            if (stage_ok && lane < n) {
                const int64_t pos = issue_pos + lane;
                const int32_t row = dcheck(pos < V.n_packed, kDbgAttnPacked) ? __ldcg(gather + pos) : -1;
                if (dcheck(row >= 0 && row < V.cap_packed, kDbgAttnPacked)) {
                    const int64_t r = (int64_t)hk * V.cap_packed + row;
                    cp_async_row<RB>(dst + lane * RB, V.codes[0] + r * RB);
                    cp_async_row<RB>(dst + kOffV + lane * RB, V.codes[1] + r * RB);
                    cp_async_row<NG * 8>(dst + kOffKs + lane * NG * 8,
                                         reinterpret_cast<const uint8_t *>(V.scalemin[0] + r * NG * 2));
                    cp_async_row<NG * 8>(dst + kOffVs + lane * NG * 8,
                                         reinterpret_cast<const uint8_t *>(V.scalemin[1] + r * NG * 2));
                }
            }
            cp_async_mbar_arrive(bar);
            issue_pos += kAdvTok;
            issue_left -= kAdvTok;
            issue_step += T;
        } else if (!WINDOW) {
            const bool full = n == kStepTok;
            const uint32_t bc = full ? (uint32_t)(kStepTok * RB) : round16((uint32_t)(n * RB));
            const uint32_t bs = full ? (uint32_t)(kStepTok * NG * 8) : round16((uint32_t)(n * NG * 8));
            // the copies stay inside the view's rows of this head (debug build)
            const int64_t hrows = (int64_t)hk * V.cap_packed;
            const bool ok = stage_ok &&
                            dcheck(n > 0 && within(src_kc, bc, V.codes[0] + hrows * RB, V.cap_packed * RB) &&
                                       within(src_ks, bs, V.scalemin[0] + hrows * NG * 2, V.cap_packed * NG * 8) &&
                                       (SCORE || (within(src_vc, bc, V.codes[1] + hrows * RB, V.cap_packed * RB) &&
                                                  within(src_vs, bs, V.scalemin[1] + hrows * NG * 2,
                                                         V.cap_packed * NG * 8))),
                                   kDbgAttnPacked);
            // a refused block completes its barrier without bytes (its stage is garbage)
            mbar_arrive_expect_tx_if(issuer, bar, !ok ? 0u : SCORE ? bc + bs : 2 * (bc + bs));
            bulk_copy_g2s_if(issuer && ok, dst, src_kc, bc, bar);
            if (!SCORE) bulk_copy_g2s_if(issuer && ok, dst + kOffV, src_vc, bc, bar);
            bulk_copy_g2s_if(issuer && ok, dst + kOffKs, src_ks, bs, bar);
            if (!SCORE) bulk_copy_g2s_if(issuer && ok, dst + kOffVs, src_vs, bs, bar);
            src_kc += (int64_t)kAdvTok * RB;
            src_vc += (int64_t)kAdvTok * RB;
            src_ks += (int64_t)kAdvTok * NG * 2;
            src_vs += (int64_t)kAdvTok * NG * 2;
            issue_left -= kAdvTok;
            issue_step += T;
        } else {
            const int kv = issue_blk & 1;
            const uint16_t *base = kv ? win_v : win_k;
            const int first = min(n, V.cap_window - win_phys);
            const bool ok = stage_ok && dcheck(n > 0 && win_phys >= 0 && first > 0 && n - first <= V.cap_window,
                                               kDbgAttnWindow);
            mbar_arrive_expect_tx_if(issuer, bar, ok ? (uint32_t)(n * D * 2) : 0u);
            bulk_copy_g2s_if(issuer && ok, dst, base + (int64_t)win_phys * D, (uint32_t)(first * D * 2), bar);
            if (n > first)
                bulk_copy_g2s_if(issuer && ok, dst + first * D * 2, base, (uint32_t)((n - first) * D * 2), bar);
            if (kv == 1) {
                win_phys = (win_phys + kAdvTok) % V.cap_window;
                issue_left -= kAdvTok;
                issue_step += T;
            }
        }
        ++issue_blk;
        if (++issue_slot == S) issue_slot = 0;
    };

    // ---- prologue: barriers and the first copies, then the dependency wait
    // (q, the partials, the counters and out belong to the stream's order),
    // then q.  The packed rows and windows of the layer do not depend on the
    // grid before (prefetch; the blocks an append of the same step writes
    // wait inside issue_next), so their first ring stages are already in
    // flight while that grid drains.
    const int n_pro = min(S, n_blocks);
    if (!p.chain && (!p.prefetch || gather != nullptr)) pdl_wait();  // a gather list comes from the grid before
    if (half == 0) {
        if (lane == 0) {
            for (int s = 0; s < S; ++s) mbar_init(&wbar[s], gather != nullptr ? 32u : 1u);
            fence_mbar_init();
        }
        __syncwarp();
        for (int b = 0; b < n_pro; ++b) issue_next();
    }
    if (!p.chain) {
        pdl_wait();
        pdl_launch_dependents();  // the next grid may be scheduled as slots free up (it waits in turn)
    }
    for (int i = tid; i < kHeadsPerCta * D / 8; i += kAttnThreads) {
        const int j = i / (D / 8), d8 = i - j * (D / 8);
        uint4 val = make_uint4(0, 0, 0, 0);
        if (j < nh && dcheck(V.seq_index < p.n_seqs && h0 + j < p.n_q_heads, kDbgAttnIo))
            val = __ldcg(reinterpret_cast<const uint4 *>(p.q + ((int64_t)V.seq_index * p.n_q_heads + h0 + j) * D) + d8);
        reinterpret_cast<uint4 *>(q_s)[i] = val;
    }
    __syncthreads();  // also publishes the barriers' initialization to the team's other warp

    WarpState<NGW> st;
    // base-2 logits per unit of the QK accumulators (window items: bf16 q
    // as it is; packed items: the factor q was scaled by, see below)
    float qk_scale = p.scale_log2;
    {
        // q as B operand (column n = gid) for the warp's groups, k-slots from
        // the unpack map; the per-group sums of q come from the same values:
        // each lane adds its 16 elements, lanes of one gid combine, then lanes
        // fetch the sums of heads 2tig, 2tig+1.
        const uint16_t *qr = q_s + gid * D;
        auto qf = [&](int g, int k) { return __uint_as_float((uint32_t)qr[64 * g + 16 * tig + k] << 16); };
        // packed items: q * 2^(14 - off - eq) in fp16, with 2^eq > max|q| over
        // the CTA's heads and this warp's groups, so that |B| < 2^14 and the
        // products with the codes' 2^(off - 24) carry 2^(-10 - eq)
        int eq = 0;
        if (!WINDOW) {
            float mx = 0.f;
#pragma unroll
            for (int gg = 0; gg < NGW; ++gg)
#pragma unroll
                for (int k = 0; k < 16; ++k) mx = fmaxf(mx, fabsf(qf(g0 + gg, k)));
            const uint32_t wm = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mx));
            eq = wm == 0u ? 0 : max(-100, min(110, (int)(wm >> 23) - 126));
            qk_scale = p.scale_log2 * __uint_as_float((uint32_t)(127 + 10 + eq) << 23);
        }
#pragma unroll
        for (int gg = 0; gg < NGW; ++gg) {
            const int g = g0 + gg;
            float part = 0.f;
#pragma unroll
            for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = 2 * s + j;
                    const float q0 = qf(g, WINDOW ? 2 * r : qk_code<B>(r, 0));
                    const float q1 = qf(g, WINDOW ? 2 * r + 1 : qk_code<B>(r, 1));
                    if (WINDOW) {
                        st.bq[gg][s][j] = pack_bf16x2(q0, q1);
                    } else {
                        // exact: a power-of-two scaling of a bf16 value (fp16 normal range)
                        const float c0 = __uint_as_float((uint32_t)(127 + 14 - qk_off<B>(r, 0) - eq) << 23);
                        const float c1 = __uint_as_float((uint32_t)(127 + 14 - qk_off<B>(r, 1) - eq) << 23);
                        st.bq[gg][s][j] = pack_f16x2(q0 * c0, q1 * c1);
                    }
                    part += q0 + q1;
                }
            part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
            part += __shfl_xor_sync(0xFFFFFFFFu, part, 2);
            const float qs = WINDOW ? 1.f : __uint_as_float((uint32_t)(127 - 10 - eq) << 23);
            st.qsum[gg][0] = qs * __shfl_sync(0xFFFFFFFFu, part, 4 * (2 * tig));
            st.qsum[gg][1] = qs * __shfl_sync(0xFFFFFFFFu, part, 4 * (2 * tig + 1));
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) st.o[gg][t][e] = 0.f;
            st.mt[gg][0] = st.mt[gg][1] = 0.f;
        }
        st.m[0] = st.m[1] = -INFINITY;
        st.l[0] = st.l[1] = 0.f;
        st.pscale = 1.f;
        st.plimit = 0.f;  // the first packed block sets pscale
    }
    // the two warps of a team use different logit scales (eq) only inside
    // their QK sums; those are added in logit units
    float team_scale = qk_scale;

    // consumer position: the current block is in slot `slot`, phase `phase`
    int slot = 0;
    uint32_t phase = 0;
    const uint8_t *stage = ring;
    int consumed = 0;
    auto wait_cur = [&]() -> bool {
        // warp-uniform result: one lane giving up makes the warp give up
        if (__all_sync(0xFFFFFFFFu, mbar_try_wait(&wbar[slot], phase))) return true;
        return __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&wbar[slot], phase, p.timeout_ns));
    };
    auto advance_cur = [&]() {
        ++consumed;
        if (++slot == S) {
            slot = 0;
            phase ^= 1u;
            stage = ring;
        } else {
            stage += kBlk;
        }
    };
    // TW = 1: a consumed slot is refilled at once
    auto release_cur = [&]() {
        if (TW == 1) {
            __syncwarp();
            if (consumed + S < n_blocks) {  // warp-uniform
                fence_proxy_async_shared();
                issue_next();
            }
        }
        advance_cur();
    };
    // TW = 2, at the team barrier: blocks [0, both) are done in both warps
    auto refill_team = [&](int both) {
        if (TW == 2 && half == 0) {
            bool fenced = false;
            while (issue_blk < n_blocks && issue_blk < both + S) {
                if (!fenced) {
                    fence_proxy_async_shared();
                    fenced = true;
                }
                issue_next();
            }
        }
    };
    // QK sums of the warp's groups -> logits of the team's heads: the
    // partner's groups added (TW = 2), scale, rows past `valid` masked
    auto finish_qk = [&](auto &l, int i, bool ok, int valid) -> bool {
        constexpr int R = sizeof(l) / sizeof(l[0]);
        if constexpr (TW == 2) {
            // the partner's sums carry its own eq: bring them to logit units first
#pragma unroll
            for (int r = 0; r < R; ++r) {
                l[r][0] *= team_scale;
                l[r][1] *= team_scale;
            }
            ok = team_add<R>(l, xb, i & 1, half, lane, 1 + team, ok);
        } else {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                l[r][0] *= team_scale;
                l[r][1] *= team_scale;
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int row = (r >> 1) * kTile + gid + (r & 1) * 8;
            if (row >= valid) l[r][0] = l[r][1] = -INFINITY;
        }
        return ok;
    };

    // ---- main loop
    bool failed = false;
    int left = n_tok - kStepTok * team;
    for (int i = 0; i < n_my; ++i, left -= kAdvTok) {
        const bool ok = wait_cur();
        if (TW == 1 && !ok) { failed = true; break; }
        // TW = 2: a failed wait still takes part in the team barrier below,
        // so that both warps leave the loop together
        if constexpr (!WINDOW) {
            float lg[4][2];
            if (left >= kStepTok) {
                packed_qk_block<B, NG, NGW>(st, stage, gid, tig, g0, lg);
            } else {
                float a[2][2], b[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
                packed_qk_tile<B, NG, NGW>(st, stage, stage + kOffKs, gid, tig, g0, a);
                if (left > kTile)
                    packed_qk_tile<B, NG, NGW>(st, stage + kTile * RB, stage + kOffKs + kTile * NG * 8, gid, tig, g0,
                                               b);
                lg[0][0] = a[0][0]; lg[0][1] = a[0][1]; lg[1][0] = a[1][0]; lg[1][1] = a[1][1];
                lg[2][0] = b[0][0]; lg[2][1] = b[0][1]; lg[3][0] = b[1][0]; lg[3][1] = b[1][1];
            }
            if (!finish_qk(lg, i, ok, min(left, kStepTok))) { failed = true; break; }
            refill_team(i);  // TW = 2: the blocks before this one are done in both warps
            if constexpr (SCORE) {
                release_cur();
                // largest logit over the CTA's heads (2 per lane, 8 per quad)
                const int64_t dst_i = V.score_off + (int64_t)hk * V.n_packed + tok0 + (int64_t)kStepTok * (team + i * T);
                float *dst = p.scores + dst_i;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float m = fmaxf(2 * tig < nh ? lg[r][0] : -INFINITY, 2 * tig + 1 < nh ? lg[r][1] : -INFINITY);
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                    const int row = (r >> 1) * kTile + gid + (r & 1) * 8;
                    if (half == 0 && tig == 0 && row < left &&
                        dcheck(dst_i + row >= 0 && dst_i + row < p.n_scores, kDbgAttnIo))
                        dst[row] = m;
                }
                continue;
            }
            softmax_step_n<NGW, 4>(st, lg);
            if (left >= kStepTok) {
                // two full 16-token tiles, one softmax update over 32 tokens
                track_pscale<NG, NGW>(st, stage + kOffVs, 2 * kTile, gid, g0);
                packed_pv_block<B, NG, NGW, true>(st, stage + kOffV, stage + kOffVs, 2 * kTile, lg, gid, tig, g0);
            } else {
                // the chunk's ragged end: one or two partial tiles
                const int n_valid = min(left, 2 * kTile);
                track_pscale<NG, NGW>(st, stage + kOffVs, n_valid, gid, g0);  // the block's valid rows
                packed_pv_block<B, NG, NGW, false>(st, stage + kOffV, stage + kOffVs, n_valid, lg, gid, tig, g0);
            }
            release_cur();
        } else {
            const int n_valid = min(kTile, left);
            float lg[2][2];
            window_qk<NG, NGW>(st, stage, gid, tig, g0, lg);
            if (!finish_qk(lg, i, ok, n_valid)) { failed = true; break; }
            release_cur();
            refill_team(2 * i + 1);  // TW = 2: up to this step's K block, done in both warps
            softmax_step_n<NGW, 2>(st, lg);
            bool vok = wait_cur();
            if constexpr (TW == 2) vok = team_and(vok, xb, i & 1, half, lane, 1 + team);
            if (!vok) { failed = true; break; }
            if (n_valid == kTile) window_pv<NG, NGW, true>(st, stage, n_valid, lg, gid, tig, g0);
            else window_pv<NG, NGW, false>(st, stage, n_valid, lg, gid, tig, g0);
            release_cur();
        }
    }
    if (failed) {
        // let every copy this team issued land before the CTA can exit
        if (half == 0) {
            const int issued = __shfl_sync(0xFFFFFFFFu, issue_blk, 0);
            for (; consumed < issued; ++consumed) {
                (void)__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&wbar[slot], phase, p.timeout_ns));
                if (++slot == S) { slot = 0; phase ^= 1u; }
            }
        }
        if (lane == 0) atomicExch(p.status, 1u);
    }
    if constexpr (SCORE) return;

    // ---- team partial -> the team's ring area (all its copies have landed):
    // m and l from the team's first warp, each warp's groups of O
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        float l = st.l[j];
        l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
        l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
        l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
        st.l[j] = l;
#pragma unroll
        for (int g = 0; g < NGW; ++g) {
            float m = st.mt[g][j];
            m += __shfl_xor_sync(0xFFFFFFFFu, m, 4);
            m += __shfl_xor_sync(0xFFFFFFFFu, m, 8);
            m += __shfl_xor_sync(0xFFFFFFFFu, m, 16);
            st.mt[g][j] = m;
        }
    }
    if (TW == 2) team_bar(team);  // both warps past the ring
    __syncwarp();
    float *wpart = reinterpret_cast<float *>(ring);  // m[8], l[8], o[8][D]
    if (gid == 0 && half == 0) {
        wpart[2 * tig] = st.m[0];
        wpart[2 * tig + 1] = st.m[1];
        wpart[8 + 2 * tig] = st.l[0];
        wpart[8 + 2 * tig + 1] = st.l[1];
    }
    float *wo = wpart + 16;
    // packed items: O row d accumulated 2^(pv_off - 24) * pscale times its value
    const float inv_ps = 1.f / st.pscale;  // a power of two: exact
#pragma unroll
    for (int gg = 0; gg < NGW; ++gg)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int d0 = 64 * (g0 + gg) + 8 * gid + 2 * t;
            const float fe = WINDOW ? 1.f : inv_ps * __uint_as_float((uint32_t)(127 + 24 - pv_off<B>(t, 0)) << 23);
            const float fo = WINDOW ? 1.f : inv_ps * __uint_as_float((uint32_t)(127 + 24 - pv_off<B>(t, 1)) << 23);
            *reinterpret_cast<float2 *>(&wo[(2 * tig) * D + d0]) =
                make_float2(fmaf(st.o[gg][t][0], fe, st.mt[gg][0]), fmaf(st.o[gg][t][2], fo, st.mt[gg][0]));
            *reinterpret_cast<float2 *>(&wo[(2 * tig + 1) * D + d0]) =
                make_float2(fmaf(st.o[gg][t][1], fe, st.mt[gg][1]), fmaf(st.o[gg][t][3], fo, st.mt[gg][1]));
        }
    __syncthreads();

    // ---- merge the T teams (fixed order)
    const bool single = V.seq_chunks == 1;
    const int64_t pslot = ((int64_t)(V.part_begin + c) * p.n_kv_heads + hk) * p.head_blocks + z;
    float *part = p.partials + pslot * (kHeadsPerCta * (D + 2));
    const bool io_ok = single ? dcheck(V.seq_index < p.n_seqs && h0 + nh <= p.n_q_heads, kDbgAttnIo)
                              : dcheck(pslot >= 0 && pslot < p.n_part_slots, kDbgAttnWorkspace);
    for (int idx = io_ok ? tid : nh * D; idx < nh * D; idx += kAttnThreads) {
        const int j = idx / D, d = idx - j * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < T; ++w)
            M = fmaxf(M, reinterpret_cast<const float *>(rings + (size_t)w * team_ring)[j]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < T; ++w) {
            const float *wp = reinterpret_cast<const float *>(rings + (size_t)w * team_ring);
            const float mw = wp[j];
            const float e = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
            L = fmaf(e, wp[8 + j], L);
            O = fmaf(e, wp[16 + j * D + d], O);
        }
        if (single) {
            p.out[((int64_t)V.seq_index * p.n_q_heads + h0 + j) * D + d] = O / L;
        } else {
            part[j * D + d] = O;
            if (d == 0) {
                part[kHeadsPerCta * D + j] = M;
                part[kHeadsPerCta * D + kHeadsPerCta + j] = L;
            }
        }
    }
    if (single) return;
    // ---- the CTA that finishes a unit's last chunk combines the unit (an
    // arrival counter, never a wait); it resets the counter for the next call
    int *last_flag = reinterpret_cast<int *>(bars + kAttnWarps * kMaxStages);
    __threadfence();  // this thread's partial stores, before the arrival below
    __syncthreads();
    if (tid == 0) {
        const int64_t ci = ((int64_t)V.seq_index * p.n_kv_heads + hk) * p.head_blocks + z;
        bool last = false;
        if (dcheck(ci >= 0 && ci < (int64_t)p.n_seqs * p.n_kv_heads * p.head_blocks, kDbgAttnWorkspace)) {
            uint32_t *ctr = p.counters + ci;
            const uint32_t before = atomicAdd(ctr, 1u);
            last = before + 1 == (uint32_t)V.seq_chunks;
            if (last) *ctr = 0u;
        }
        *last_flag = last ? 1 : 0;
    }
    __syncthreads();
    if (*last_flag) {
        __threadfence();  // the other chunks' partials, after their arrivals
        combine_unit<NG>(p, V, hk, z, reinterpret_cast<float *>(rings));
    }
}

// BSEL = 2, 3, 4 or 8: every view of the launch that has packed tokens has
// that width, and only that width's code is compiled into the kernel (the
// host groups the views of a call by width, one launch per group).  With all
// four widths compiled into one kernel and dispatched per CTA, the Qwen3-32B
// layer (8 views, up to four widths) took 72 us against 64 us for the
// per-width launches (more spills, one fetch in five missing the
// instruction cache).
template <int NG, int BSEL, bool SCORE = false>
__device__ __forceinline__ void decode_attn_body(const AttnParams &p, uint8_t *smem) {
    // The first launch of a call waits for the preceding grid inside the
    // item, after its first copies (see attn_item) and releases the next grid
    // right after that wait.  A later launch of a call is released by the one
    // before it once that one has waited, so it needs no wait at entry and
    // releases the next grid at once.
    if (p.chain) pdl_launch_dependents();
    // ---- which item: view by binary search over chunk ranges
    const int bx = blockIdx.x;
    int lo = 0, hi = p.n_views - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.views[mid].chunk_begin <= bx) lo = mid; else hi = mid - 1;
    }
    const AttnView &V = p.views[lo];
    const int c = bx - V.chunk_begin;
    const int hk = blockIdx.y, z = blockIdx.z;
    if (c >= V.n_chunks) return;  // never launched by the host planner; defensive
    if constexpr (SCORE) {
        if (c < V.n_chunks_packed) attn_item<NG, BSEL, false, true>(p, V, c, hk, z, smem);
    } else {
        if (c >= V.n_chunks_packed) attn_item<NG, 4, true>(p, V, c, hk, z, smem);
        else attn_item<NG, BSEL, false>(p, V, c, hk, z, smem);
    }
}

template <int NG, int BSEL>
__global__ void __launch_bounds__(kAttnThreads, attn_ctas_per_sm<NG>())
    decode_attn_kernel(const __grid_constant__ AttnParams p) {
    static_assert(BSEL == 2 || BSEL == 3 || BSEL == 4 || BSEL == 8, "width");
    extern __shared__ __align__(128) uint8_t smem[];
    decode_attn_body<NG, BSEL>(p, smem);
    // a later launch of a call completes only after the one before it, so
    // the call's last grid completes after all of them
    if (p.chain) pdl_wait();
}

// Scores of packed tokens for the top-K selection: the attention grid's QK
// path alone over views without windows, one query-head block per KV head.
template <int NG, int BSEL>
__global__ void __launch_bounds__(kAttnThreads, attn_ctas_per_sm<NG>())
    score_attn_kernel(const __grid_constant__ AttnParams p) {
    static_assert(BSEL == 2 || BSEL == 3 || BSEL == 4 || BSEL == 8, "width");
    extern __shared__ __align__(128) uint8_t smem[];
    decode_attn_body<NG, BSEL, true>(p, smem);
    if (p.chain) pdl_wait();
}

}  // namespace kvq
