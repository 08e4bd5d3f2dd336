// kvq_codec.cuh -- group-wise affine quantization of bf16 K/V rows into packed
// b-bit codes with a per-group {scale, min}, and its inverse into bf16.
//
// "QKVShare: Quantized KV-Cache Handoff for Multi-Agent On-Device LLMs",
// Metodologia: quantized KV groups form the handoff card and the receiver
// rebuilds full-precision past_key_values from them.  "Agent Memory Below the
// Prompt ...", Abstract: 4-bit format.  "Coordinated Mixed-Precision KV Cache
// Quantization ...", Abstract: widths 2/3/4 (and 8) per (agent, layer).
//
// Both kernels stream HBM: two lanes share one 64-element group (32 elements,
// 64 bytes of bf16 each), loads and stores are 16-byte vectors, and every
// result is a bit-exact function of the input (fp32 round-to-nearest steps in
// the order of the format definition).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <type_traits>

#include "kvq_debug.cuh"
#include "kvq_ptx.cuh"

namespace kvq {

constexpr int kGroup = 64;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: y + magic rounds y to an integer (RNE)
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// The packed words of 32 fields that all hold kRoundMagicBits (field j at bit
// j*B, mod 2^32): the fast path packs the magic sums' raw bits, 0x4B400000 +
// c, and removes this constant once per word (shifts and sums are linear mod
// 2^32, and c < 2^22 never carries into the magic bits).
template <int B>
__host__ __device__ constexpr uint32_t magic_pack_word(int w) {
    uint32_t acc = 0;
    for (int i = 0; i < 32; ++i) {
        const int bit = i * B;
        if ((bit >> 5) == w) acc += kRoundMagicBits << (bit & 31);
        if ((bit & 31) + B > 32 && (bit >> 5) + 1 == w) acc += kRoundMagicBits >> (32 - (bit & 31));
    }
    return acc;
}

// Quantize one half (32 elements) of a 64-element group held as 16 bf16x2
// words (also readable at `src`, read again only for the exact re-check of
// near-tie elements); the
// partner half lives in lane ^ 1, which must execute this call in the same
// instruction stream (full-warp shuffles).  Writes the packed codes of this
// half (32*B bits = B words, code j at bit j*B) and the group's s, mn.
template <int B>
__device__ __forceinline__ void quantize_half_group(const uint32_t (&x)[16], const uint16_t *src,
                                                    uint32_t (&packed)[B], float &s_out, float &mn_out) {
    __nv_bfloat162 lo2 = *reinterpret_cast<const __nv_bfloat162 *>(&x[0]);
    __nv_bfloat162 hi2 = lo2;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&x[i]);
        lo2 = __hmin2(lo2, v);
        hi2 = __hmax2(hi2, v);
    }
    const uint32_t lo_bits = *reinterpret_cast<uint32_t *>(&lo2);
    const uint32_t hi_bits = *reinterpret_cast<uint32_t *>(&hi2);
    float mn = fminf(bf16lo_to_f32(lo_bits), bf16hi_to_f32(lo_bits));
    float mx = fmaxf(bf16lo_to_f32(hi_bits), bf16hi_to_f32(hi_bits));
    mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
    if ((__float_as_uint(mn) << 1) == 0u) mn = 0.0f;  // +0 for either zero
    if ((__float_as_uint(mx) << 1) == 0u) mx = 0.0f;

    constexpr uint32_t qmax = (1u << B) - 1u;
    const float s = (mx != mn) ? __fdiv_rn(__fsub_rn(mx, mn), (float)qmax) : 0.0f;

#pragma unroll
    for (int w = 0; w < B; ++w) packed[w] = 0u;

    if (s != 0.0f && !(s >= 0x1p-100f && s <= 0x1p100f)) {
        // extreme scales (subnormal ranges): IEEE division for every element
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float xf = (i & 1) ? bf16hi_to_f32(x[i >> 1]) : bf16lo_to_f32(x[i >> 1]);
            const uint32_t c = min(__float2uint_rn(__fdiv_rn(__fsub_rn(xf, mn), s)), qmax);
            const int bit = i * B;
            packed[bit >> 5] += c << (bit & 31);
            if ((bit & 31) + B > 32) packed[(bit >> 5) + 1] += c >> (32 - (bit & 31));
        }
    } else if (s != 0.0f) {
        // Fast path: y = fma(x, r, -RN(mn*r)) with r = RN(1/s) lies within
        // 2^(B-23) + |mn*r|*2^-24 of the quotient (x - mn)/s (quotients are
        // <= 2^B).  A group whose min is large against its scale (|mn*r| >=
        // 2^(B+2)) takes y = (x - mn) * r instead (within 3*2^(B-24) of the
        // quotient), which keeps y > -1/2 there.  With W = 2^(B-21) (plus
        // |mn*r|*2^-21 on the fma form), at least four times that error, y1
        // and y2 are y shifted by +W and -W (on the fma form: the addend
        // -mn*r +- W): they bracket the quotient strictly, so when they round
        // to the same integer the quotient lies strictly inside that
        // integer's interval and the correctly rounded RN((x - mn)/s) is it
        // (and every code is in range).  Elements whose brackets round apart
        // (bf16 grids make exact ties common) are redone exactly below,
        // without a division.
        const float r = __frcp_rn(s);
        const float mr = __fmul_rn(mn, r);
        const bool fma_ok = fabsf(mr) < __uint_as_float((uint32_t)(127 + B + 2) << 23);
        const float win = __fadd_rn(__uint_as_float((uint32_t)(127 + B - 21) << 23),
                                    fma_ok ? __fmul_rn(fabsf(mr), 0x1p-21f) : 0.0f);
        const float c1 = __fsub_rn(win, mr), c2 = __fsub_rn(-win, mr);
        // codes of y1 packed, and those of y2 in `apart`, which then becomes
        // the difference: per element y1's code minus y2's (0 or 1) in its
        // field (B = 3: fields straddle words, so a 32-bit mask of the
        // elements instead)
        uint32_t apart[B == 3 ? 1 : B];
#pragma unroll
        for (int w = 0; w < (B == 3 ? 1 : B); ++w) apart[w] = 0u;
        auto fast = [&](auto use_fma) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float xf = (i & 1) ? bf16hi_to_f32(x[i >> 1]) : bf16lo_to_f32(x[i >> 1]);
                float y1, y2;
                if constexpr (decltype(use_fma)::value) {
                    y1 = __fmaf_rn(xf, r, c1);
                    y2 = __fmaf_rn(xf, r, c2);
                } else {
                    const float y = __fmul_rn(__fsub_rn(xf, mn), r);
                    y1 = __fadd_rn(y, win);
                    y2 = __fsub_rn(y, win);
                }
                // the magic sums' bits, 0x4B400000 + code; the constant goes below
                const uint32_t t1 = __float_as_uint(__fadd_rn(y1, kRoundMagic));
                const uint32_t t2 = __float_as_uint(__fadd_rn(y2, kRoundMagic));
                const int bit = i * B;
                packed[bit >> 5] += t1 << (bit & 31);
                if ((bit & 31) + B > 32) packed[(bit >> 5) + 1] += t1 >> (32 - (bit & 31));
                if constexpr (B == 3) apart[0] |= (t1 - t2) << i;
                else apart[bit >> 5] += t2 << (bit & 31);  // y2's codes; subtracted below
            }
        };
        if (fma_ok) fast(std::true_type{});
        else fast(std::false_type{});
#pragma unroll
        for (int w = 0; w < (B == 3 ? 0 : B); ++w) apart[w] = packed[w] - apart[w];
#pragma unroll
        for (int w = 0; w < B; ++w) packed[w] -= magic_pack_word<B>(w);
        // element i again from memory: the lane has just read the row through
        // L1 (read-only cached loads), so it is a cache hit, and one load
        // costs the integer pipe less than a select tree over the 16 registers
        auto redo = [&](int i) -> uint32_t {
            const float xf = __uint_as_float((uint32_t)__ldg(src + i) << 16);
            const float a = __fsub_rn(xf, mn);
            // the code the fast path packed (y1's), and the half-integer h
            // that y is near (within W: the brackets straddle it)
            const float y = fma_ok ? __fmaf_rn(xf, r, -mr) : __fmul_rn(a, r);
            const float y1 = fma_ok ? __fmaf_rn(xf, r, c1) : __fadd_rn(y, win);
            const uint32_t c_fast = __float_as_uint(__fadd_rn(y1, kRoundMagic)) - kRoundMagicBits;
            const float ri = __fsub_rn(__fadd_rn(y, kRoundMagic), kRoundMagic);
            // e = a - h*s is exact (|e| < s*2^(B-20) on a grid no finer than
            // ulp(s)/4, i.e. <= B+6 significant bits), so a/s = h + e/s
            // exactly.  RN(a/s) == h iff |e| <= s*ulp(h)/2 (h has few
            // significant bits, so a tie at that distance rounds to h); then
            // the code is h rounded half to even, otherwise the integer on
            // the side of h that e points to.
            const float h = __fadd_rn(ri, (y >= ri) ? 0.5f : -0.5f);
            const float e = __fmaf_rn(-h, s, a);
            const float half_ulp = __uint_as_float((__float_as_uint(h) & 0x7F800000u) - (24u << 23));
            const uint32_t n = __float_as_uint(__fadd_rn(__fsub_rn(h, 0.5f), kRoundMagic)) - kRoundMagicBits;
            uint32_t c;
            if (fabsf(e) <= __fmul_rn(s, half_ulp)) c = n + (n & 1u);
            else c = (e > 0.0f) ? n + 1u : n;
            return c ^ c_fast;  // the field's correction (XOR: no carries across fields)
        };
        if constexpr (B == 3) {
            for (uint32_t near = apart[0]; near != 0u; near &= near - 1u) {
                const int i = __ffs(near) - 1;
                const uint32_t flip = redo(i);
                const int bit = i * B;
#pragma unroll
                for (int k = 0; k < B; ++k) {
                    if ((bit >> 5) == k) packed[k] ^= flip << (bit & 31);
                    if ((bit >> 5) + 1 == k && (bit & 31) + B > 32) packed[k] ^= flip >> (32 - (bit & 31));
                }
            }
        } else {
#pragma unroll
            for (int w = 0; w < B; ++w)
                for (uint32_t near = apart[w]; near != 0u; near &= near - 1u) {
                    const int b = __ffs(near) - 1;  // the low bit of element (32 w + b) / B's field
                    packed[w] ^= redo((32 * w + b) / B) << b;
                }
        }
    }
    s_out = s;
    mn_out = mn;
}

// Dequantize 32 codes (B words, code j at bit j*B) into 16 bf16x2 words.
template <int B>
__device__ __forceinline__ void dequantize_half_group(const uint32_t (&packed)[B], float s, float mn,
                                                      uint32_t (&y)[16]) {
    constexpr uint32_t mask = (1u << B) - 1u;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        uint32_t c[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int bit = (i + k) * B;
            uint32_t v = packed[bit >> 5] >> (bit & 31);
            if ((bit & 31) + B > 32) v |= packed[(bit >> 5) + 1] << (32 - (bit & 31));
            c[k] = v & mask;
        }
        // exact small-integer -> float: 2^23 + c, minus 2^23
        const float c0 = __fsub_rn(__uint_as_float(0x4B000000u | c[0]), 8388608.0f);
        const float c1 = __fsub_rn(__uint_as_float(0x4B000000u | c[1]), 8388608.0f);
        y[i >> 1] = pack_bf16x2(__fmaf_rn(c0, s, mn), __fmaf_rn(c1, s, mn));
    }
}

struct CodecArgs {
    const uint16_t *x;       // bf16 (quantize input / dequantize output)
    int64_t x_head_stride;   // elements
    int64_t x_tok_stride;    // elements
    int64_t n_tokens;
    int32_t n_heads;
    uint8_t *codes;
    float *scalemin;
    int64_t head_cap;        // rows per head in codes/scalemin
};

// Grid: 1-D, a few blocks per SM.  The (head, group) space is swept in one
// global, contiguous order: warp w handles groups [16w, 16w+16) of the flat
// sequence head-major, then jumps by all warps * 16, so concurrent warps touch
// one narrow window of memory (TLB- and DRAM-page friendly) and every warp's
// share is balanced across heads.  The (head, group) cursor advances without
// division.  Each lane pair owns one group.
struct SweepCursor {
    int64_t grp;  // group within the head
    int h;        // head
};

__device__ __forceinline__ void sweep_advance(SweepCursor &c, int64_t step, int64_t n_groups) {
    c.grp += step;
    while (c.grp >= n_groups) {
        c.grp -= n_groups;
        ++c.h;
    }
}

template <int B, int NG>
__global__ void __launch_bounds__(256) quantize_kernel(CodecArgs a) {
    constexpr int RB = 8 * B * NG;  // row bytes
    const int64_t n_groups = a.n_tokens * NG;
    const int lane = threadIdx.x & 31;
    const int half = lane & 1;
    const int64_t warp_global = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t warp_stride = (int64_t)gridDim.x * (blockDim.x >> 5);
    SweepCursor cur{0, 0};
    sweep_advance(cur, warp_global * 16 + (lane >> 1), n_groups);
    for (; cur.h < a.n_heads; sweep_advance(cur, warp_stride * 16, n_groups)) {
        const int64_t t = cur.grp / NG;
        const int g = (int)(cur.grp - t * NG);
        const uint16_t *src = a.x + (int64_t)cur.h * a.x_head_stride + t * a.x_tok_stride + g * kGroup + half * 32;
        // the row is one of the input's and of the outputs' (debug build); a
        // refused row is neither read nor written, and its lanes still take
        // part in the pair's shuffles
        const bool ok = dcheck(t < a.n_tokens && t < a.head_cap && cur.h < a.n_heads, kDbgCodec);
        uint32_t x[16];
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 q = ok ? __ldg(s4 + v) : make_uint4(0, 0, 0, 0);
            x[4 * v + 0] = q.x; x[4 * v + 1] = q.y; x[4 * v + 2] = q.z; x[4 * v + 3] = q.w;
        }
        uint32_t packed[B];
        float s, mn;
        quantize_half_group<B>(x, src, packed, s, mn);
        if (!ok) continue;
        const int64_t row = (int64_t)cur.h * a.head_cap + t;
        uint8_t *dst = a.codes + row * RB + g * 8 * B + half * 4 * B;
        if constexpr (B == 4) {
            *reinterpret_cast<uint4 *>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        } else if constexpr (B == 8) {
            reinterpret_cast<uint4 *>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<uint4 *>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        } else if constexpr (B == 2) {
            *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
        } else {
#pragma unroll
            for (int w = 0; w < B; ++w) reinterpret_cast<uint32_t *>(dst)[w] = packed[w];
        }
        if (half == 0) *reinterpret_cast<float2 *>(a.scalemin + (row * NG + g) * 2) = make_float2(s, mn);
    }
}

// Dequantize: the rows of all heads form one flat sequence (head-major).  A
// warp unit is RPU consecutive rows, 32*CPL chunks of 8 elements; lane l owns
// chunks l, l + 32, ... of its unit, so each warp load of codes and each
// 16-byte store of a warp covers consecutive bytes (one 512-byte store when
// the output rows are contiguous).  kDeqUnroll units per iteration: all their
// loads are issued before the first conversion and store.
constexpr int kDeqUnroll = 4;

template <int NG>
struct DeqShape {
    static constexpr int CPR = 8 * NG;           // 8-element chunks per row
    static constexpr int CPL = NG == 3 ? 3 : 1;  // chunks per lane per unit
    static constexpr int RPU = 32 * CPL / CPR;   // rows per unit: 4, 2, 4, 1
};

// The 8 codes of chunk d8 of a row (B bytes at byte d8*B, code j at bit B*j):
// in .x (and .y for B = 8), read with aligned loads that stay inside the row.
template <int B>
__device__ __forceinline__ uint2 load_chunk_codes(const uint8_t *row, int d8) {
    if constexpr (B == 8) {
        return __ldcs(reinterpret_cast<const uint2 *>(row) + d8);
    } else if constexpr (B == 4) {
        return make_uint2(__ldcs(reinterpret_cast<const uint32_t *>(row) + d8), 0u);
    } else if constexpr (B == 2) {
        return make_uint2(__ldcs(reinterpret_cast<const unsigned short *>(row) + d8), 0u);
    } else {
        // 3 bytes at any byte offset: the aligned word holding the first, and
        // the next one only when the bytes run into it (it then still lies
        // inside the row: rows are 8-byte multiples)
        const int off = 3 * d8, w = off & ~3, sh = 8 * (off & 3);
        const uint32_t x = __ldcs(reinterpret_cast<const uint32_t *>(row + w));
        if ((off & 3) < 2) return make_uint2(x >> sh, 0u);
        const uint32_t y = __ldcs(reinterpret_cast<const uint32_t *>(row + w + 4));
        return make_uint2(__funnelshift_r(x, y, sh), 0u);
    }
}

// 8 codes -> 8 bf16 values bf16_rne(fmaf(c, s, mn)), as one 16-byte vector.
template <int B>
__device__ __forceinline__ uint4 dequant_chunk(uint2 w, float s, float mn) {
    constexpr uint32_t mask = (1u << B) - 1u;
    uint32_t y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float c[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = 2 * j + e;
            const uint32_t code = (B == 8) ? ((i < 4 ? w.x : w.y) >> (8 * (i & 3))) & 255u : (w.x >> (B * i)) & mask;
            // exact small integer -> float: 2^23 + c, minus 2^23
            c[e] = __fsub_rn(__uint_as_float(0x4B000000u | code), 8388608.0f);
        }
        y[j] = pack_bf16x2(__fmaf_rn(c[0], s, mn), __fmaf_rn(c[1], s, mn));
    }
    return make_uint4(y[0], y[1], y[2], y[3]);
}

template <int B, int NG>
__global__ void __launch_bounds__(256) dequantize_kernel(CodecArgs a) {
    using S = DeqShape<NG>;
    constexpr int RB = 8 * B * NG;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    // rows between a lane's consecutive units, split into whole heads and tokens
    const int64_t step = warps * S::RPU;
    const int64_t step_h = step / a.n_tokens, step_t = step - step_h * a.n_tokens;
    // one (head, token) cursor per chunk the lane owns in a unit
    int64_t h[S::CPL], t[S::CPL];
    int d8[S::CPL];
#pragma unroll
    for (int k = 0; k < S::CPL; ++k) {
        const int uc = 32 * k + lane;
        d8[k] = uc % S::CPR;
        const int64_t r = warp * S::RPU + uc / S::CPR;
        h[k] = r / a.n_tokens;
        t[k] = r - h[k] * a.n_tokens;
    }
    uint16_t *yout = const_cast<uint16_t *>(a.x);
    while (h[0] < a.n_heads || (S::CPL > 1 && h[S::CPL - 1] < a.n_heads)) {
        uint2 cw[kDeqUnroll][S::CPL];
        float2 sm[kDeqUnroll][S::CPL];
        int64_t hh[kDeqUnroll][S::CPL], tt[kDeqUnroll][S::CPL];
#pragma unroll
        for (int u = 0; u < kDeqUnroll; ++u) {
#pragma unroll
            for (int k = 0; k < S::CPL; ++k) {
                hh[u][k] = h[k];
                tt[u][k] = t[k];
                if (h[k] < a.n_heads && dcheck(t[k] < a.n_tokens && t[k] < a.head_cap, kDbgCodec)) {
                    const int64_t row = h[k] * a.head_cap + t[k];
                    cw[u][k] = load_chunk_codes<B>(a.codes + row * RB, d8[k]);
                    sm[u][k] = __ldcs(reinterpret_cast<const float2 *>(a.scalemin + (row * NG + d8[k] / 8) * 2));
                } else {
                    hh[u][k] = a.n_heads;  // nothing to store
                }
                t[k] += step_t;
                h[k] += step_h;
                if (t[k] >= a.n_tokens) {
                    t[k] -= a.n_tokens;
                    ++h[k];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kDeqUnroll; ++u) {
#pragma unroll
            for (int k = 0; k < S::CPL; ++k) {
                if (hh[u][k] >= a.n_heads) continue;
                const uint4 v = dequant_chunk<B>(cw[u][k], sm[u][k].x, sm[u][k].y);
                __stcs(reinterpret_cast<uint4 *>(yout + hh[u][k] * a.x_head_stride + tt[u][k] * a.x_tok_stride +
                                                 d8[k] * 8),
                       v);
            }
        }
    }
}

// ------------------------------------------------------------- append ----

// One view's slice of a kvq_append launch, resolved on the host.
struct AppendView {
    uint8_t *codes[2];    // K, V
    float *scalemin[2];
    uint16_t *window[2];  // bf16 ring [H][cap_window][D] (may be null when cap_window == 0)
    int64_t cap_packed;
    int64_t packed_row;   // packed index the flushed token goes to (if flush)
    int32_t cap_window;
    int32_t slot;         // ring slot written by the new token (-1: no window)
    int32_t flush;        // 1: quantize (oldest slot | new token) into packed_row
    int32_t bits;
};

constexpr int kAppendMaxViews = 128;

struct AppendArgs {
    const uint16_t *k_new;  // bf16 [n_views][H][D]
    const uint16_t *v_new;
    int32_t n_views;
    int32_t n_kv_heads;
    int32_t early;          // 1: release the next grid (this step's attention) before waiting
    AppendView views[kAppendMaxViews];
};

// Grid: (n_views, n_kv_heads, 2 = K/V); one warp per block.  Lanes 0..2*NG-1
// each own half a group of the row being flushed (same arithmetic as the
// bulk quantize kernel); all lanes then copy the new token into the ring.
// In a decode step (early) the loads and the quantization run before the
// dependency wait: the rows read (the ring's oldest token, the new token) are
// not written by the grid before, which only reads this layer's cache or
// none of it, so only the stores wait and the append adds little to the
// step.  A plain append waits first.
template <int NG>
__global__ void __launch_bounds__(32) append_kernel(AppendArgs a) {
    constexpr int D = NG * kGroup;
    // The next grid is released before the wait only when it is this step's
    // attention grid, which knows the rows written here and waits before
    // reading them.  Any other grid after a plain append starts when the
    // append has completed.
    if (a.early) pdl_launch_dependents();
    else pdl_wait();  // the rows it reads or overwrites may belong to the preceding grid
    const AppendView &v = a.views[blockIdx.x];
    const int h = blockIdx.y;
    const int kv = blockIdx.z;
    const int lane = threadIdx.x;
    // the view, the packed row and the ring slot exist (debug build; uniform
    // over the warp, so a refused block returns whole)
    if (!dcheck((int)blockIdx.x < a.n_views && h < a.n_kv_heads &&
                    (!v.flush || (v.packed_row >= 0 && v.packed_row < v.cap_packed)) &&
                    (v.slot < 0 || v.slot < v.cap_window) && (v.flush || v.slot >= 0),
                kDbgAppend)) {
        if (a.early) pdl_wait();
        return;
    }
    const uint16_t *newrow = (kv ? a.v_new : a.k_new) + ((int64_t)blockIdx.x * a.n_kv_heads + h) * D;
    uint16_t *ring = v.window[kv];
    uint16_t *slotrow = (v.slot >= 0) ? ring + ((int64_t)h * v.cap_window + v.slot) * D : nullptr;

    // 1) quantize the flushed row: the oldest ring token, or the new token if there is no ring
    const int g = lane >> 1, half = lane & 1;
    const bool active = g < NG;
    uint32_t packed[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    float s = 0.f, mn = 0.f;
    if (v.flush) {
        const uint16_t *src = (v.cap_window > 0) ? slotrow : newrow;
        uint32_t x[16];
        if (active) {
            const uint4 *p = reinterpret_cast<const uint4 *>(src + g * kGroup + half * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint4 q = p[k];
                x[4 * k] = q.x; x[4 * k + 1] = q.y; x[4 * k + 2] = q.z; x[4 * k + 3] = q.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = 0u;
        }
        switch (v.bits) {
#define KVQ_APPEND_Q(BB)                                                          \
    case BB: {                                                                    \
        uint32_t pk[BB];                                                          \
        quantize_half_group<BB>(x, src + g * kGroup + half * 32, pk, s, mn);      \
        _Pragma("unroll") for (int w = 0; w < BB; ++w) packed[w] = pk[w];         \
    } break;
            KVQ_APPEND_Q(2)
            KVQ_APPEND_Q(3)
            KVQ_APPEND_Q(4)
            KVQ_APPEND_Q(8)
#undef KVQ_APPEND_Q
            default: break;
        }
    }
    // 2) the new token, for its ring slot (D/8 <= 32 vectors: one per lane)
    uint4 nv = make_uint4(0, 0, 0, 0);
    if (slotrow && lane < D / 8) nv = reinterpret_cast<const uint4 *>(newrow)[lane];
    __syncwarp();  // every lane has read the ring's oldest token before any lane overwrites it

    if (a.early) pdl_wait();  // the stores: after the preceding grid, which may still read this layer
    if (v.flush && active) {
        uint8_t *codes_row = v.codes[kv] + ((int64_t)h * v.cap_packed + v.packed_row) * (8 * v.bits * NG);
        uint32_t *dst = reinterpret_cast<uint32_t *>(codes_row + g * 8 * v.bits + half * 4 * v.bits);
#pragma unroll
        for (int w = 0; w < 8; ++w)
            if (w < v.bits) dst[w] = packed[w];
        if (half == 0) {
            float *sm_row = v.scalemin[kv] + ((int64_t)h * v.cap_packed + v.packed_row) * NG * 2;
            *reinterpret_cast<float2 *>(sm_row + g * 2) = make_float2(s, mn);
        }
    }
    if (slotrow && lane < D / 8) reinterpret_cast<uint4 *>(slotrow)[lane] = nv;
}

}  // namespace kvq
