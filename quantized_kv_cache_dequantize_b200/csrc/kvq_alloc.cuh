// kvq_alloc.cuh -- per-view width sensitivity from the recent window and the
// query, for the budgeted width allocation done on the host.
//
// "Coordinated Mixed-Precision KV Cache Quantization for Efficient LLM-based
// Multi-agent Systems", Abstract: each (agent, layer) gets a sensitivity from
// a local attention-error bound on recent queries, keys and values, with no
// calibration data and no trial quantization.  The bound used here: a group of
// range R quantized at b bits moves each element by at most R / (2 (2^b - 1)).
// Over the view's window tokens and per KV head, with R_k[g], R_v[g] the
// largest K, V range of group g and V_max the largest value norm,
//   Delta = scale * max over the group's query heads of sum_g |q_h[g]|_1 R_k[g] / 2
//   E_v   = sqrt(sum_g 64 (R_v[g] / 2)^2)
// bound the logit and value shifts times (2^b - 1), and the output moves by at
// most about S / (2^b - 1), S = 2 V_max Delta + E_v (the largest over KV heads).
#pragma once

#include <cstdint>

#include "kvq_debug.cuh"

namespace kvq {

constexpr int kSensMaxViews = 96;  // views per launch
constexpr int kSensWarps = 8;

struct SensView {
    const uint16_t *k_window;  // bf16 [H_kv][cap_window][D]
    const uint16_t *v_window;
    int32_t cap_window;
    int32_t n_window;
    int32_t window_head;
    int32_t row;               // row of q [row][H_q][D] and of sens [row]
};

struct SensArgs {
    const uint16_t *q;
    float *sens;
    int32_t n_rows;            // rows of q and sens (the debug build's checks)
    float scale;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t group;
    SensView views[kSensMaxViews];
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
    return x;
}
__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    return x;
}

// One CTA per view: warps take the window tokens (a token per warp, two
// elements of each group per lane), then the query heads; fp32 throughout.
template <int NG>
__global__ void __launch_bounds__(32 * kSensWarps) sensitivity_kernel(const __grid_constant__ SensArgs a) {
    constexpr int D = 64 * NG;
    __shared__ float s_rk[kSensWarps][NG], s_rv[kSensWarps][NG], s_vm[kSensWarps], s_delta[kSensWarps];
    const SensView &v = a.views[blockIdx.x];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.group;
    // the view's row and its window ring (debug build; uniform over the CTA)
    if (!dcheck(v.row >= 0 && v.row < a.n_rows && v.n_window <= v.cap_window && v.window_head >= 0 &&
                    (v.n_window == 0 || v.window_head < v.cap_window),
                kDbgSens))
        return;
    float S = 0.f;
    for (int hk = 0; hk < a.n_kv_heads; ++hk) {
        float rk[NG], rv[NG], vm2 = 0.f;
#pragma unroll
        for (int g = 0; g < NG; ++g) rk[g] = rv[g] = 0.f;
        for (int i = warp; i < v.n_window; i += kSensWarps) {
            const int slot = (v.window_head + i) % v.cap_window;
            const int64_t off = ((int64_t)hk * v.cap_window + slot) * D;
            float vs = 0.f;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const uint32_t kk = *reinterpret_cast<const uint32_t *>(v.k_window + off + 64 * g + 2 * lane);
                const uint32_t vv = *reinterpret_cast<const uint32_t *>(v.v_window + off + 64 * g + 2 * lane);
                const float k0 = __uint_as_float(kk << 16), k1 = __uint_as_float(kk & 0xFFFF0000u);
                const float v0 = __uint_as_float(vv << 16), v1 = __uint_as_float(vv & 0xFFFF0000u);
                rk[g] = fmaxf(rk[g], warp_max(fmaxf(k0, k1)) - warp_min(fminf(k0, k1)));
                rv[g] = fmaxf(rv[g], warp_max(fmaxf(v0, v1)) - warp_min(fminf(v0, v1)));
                vs = fmaf(v0, v0, fmaf(v1, v1, vs));
            }
            vm2 = fmaxf(vm2, warp_sum(vs));
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                s_rk[warp][g] = rk[g];
                s_rv[warp][g] = rv[g];
            }
            s_vm[warp] = vm2;
        }
        __syncthreads();
        float RK[NG], RV[NG], VM2 = 0.f;
#pragma unroll
        for (int g = 0; g < NG; ++g) RK[g] = RV[g] = 0.f;
        for (int w = 0; w < kSensWarps; ++w) {
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                RK[g] = fmaxf(RK[g], s_rk[w][g]);
                RV[g] = fmaxf(RV[g], s_rv[w][g]);
            }
            VM2 = fmaxf(VM2, s_vm[w]);
        }
        // the query heads of this KV head: a warp per head
        float best = 0.f;
        for (int j = warp; j < G; j += kSensWarps) {
            const uint16_t *qr = a.q + ((int64_t)v.row * a.n_q_heads + (int64_t)hk * G + j) * D;
            float t = 0.f;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const uint32_t qq = *reinterpret_cast<const uint32_t *>(qr + 64 * g + 2 * lane);
                const float l1 = warp_sum(fabsf(__uint_as_float(qq << 16)) + fabsf(__uint_as_float(qq & 0xFFFF0000u)));
                t = fmaf(l1, RK[g] * 0.5f, t);
            }
            best = fmaxf(best, t);
        }
        if (lane == 0) s_delta[warp] = best;
        __syncthreads();
        float delta = 0.f;
        for (int w = 0; w < kSensWarps; ++w) delta = fmaxf(delta, s_delta[w]);
        delta *= a.scale;
        float ev = 0.f;
#pragma unroll
        for (int g = 0; g < NG; ++g) ev = fmaf(64.f * (RV[g] * 0.5f), RV[g] * 0.5f, ev);
        S = fmaxf(S, fmaf(2.f * sqrtf(VM2), delta, sqrtf(ev)));
        __syncthreads();  // the shared arrays are refilled for the next KV head
    }
    if (tid == 0) a.sens[v.row] = S;
}

}  // namespace kvq
