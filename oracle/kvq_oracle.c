/*
 * kvq_oracle.c -- plain, slow, single-threaded CPU oracle for the quantized
 * KV-cache codec and decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (pages and sections):
 *  - "QKVShare: Quantized KV-Cache Handoff for Multi-Agent On-Device LLMs",
 *    Riepilogo Tecnico / Metodologia: KV groups are quantized into a compact
 *    card; the receiver rebuilds the full-precision past_key_values from it
 *    (the "Percorso di Iniezione", i.e. dequantize), widths from {2,4,8,FP16}.
 *  - "Agent Memory Below the Prompt: Persistent Q4 KV Cache for Multi-Agent LLM
 *    Inference on Edge Devices", Abstract: 4-bit quantized KV caches are loaded
 *    straight into attention, and several agents' quantized caches are
 *    attended concurrently (BatchQuantizedKVCache).
 *  - "Coordinated Mixed-Precision KV Cache Quantization for Efficient LLM-based
 *    Multi-agent Systems", Abstract: per-(agent, layer) widths at average 2, 3
 *    or 4 bits; recent states stay in native precision; only newly quantized
 *    blocks get a width, older blocks are never requantized.
 *
 * The pages name the method but print no bit-level format.  This library's
 * format (the reading every function below follows):
 *  - a group is 64 consecutive elements along head_dim of one (head, token)
 *    row;
 *  - mn = min, mx = max of the group (fp32, exact from bf16);
 *    zero results are stored as +0.0f;
 *  - s = (mx - mn) / (2^b - 1) in fp32 round-to-nearest; s = 0 when mx == mn;
 *  - code c = clamp(round_half_even((x - mn) / s), 0, 2^b - 1), with the
 *    subtraction and the division each one fp32 round-to-nearest operation;
 *    every code is 0 when s == 0;
 *  - code j of a group occupies bits [j*b, j*b + b) of the group's
 *    little-endian byte string (least significant bit first), so a group is
 *    8*b bytes; groups follow each other in head_dim order;
 *  - scale and min are stored as a float pair {s, mn} per group;
 *  - dequantize: y = bf16_round_half_even(fmaf((float)c, s, mn));
 *  - attention attends over the exact affine value mn + s*c (evaluated here
 *    in fp64), followed by the bf16 recent-window tokens.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * fp-contract is off so that no multiply-add is fused behind our back: every
 * fp32 operation below is exactly one IEEE-754 round-to-nearest step.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GROUP 64

/* ---------------------------------------------------------------- bf16 --- */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a finite binary32 to bf16, ties to even.  The 16 dropped bits are
 * compared with the halfway point 0x8000; at exactly halfway the kept part is
 * rounded to an even last bit.  (NaN is outside the library's contract.) */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

/* ------------------------------------------------------------ bit packing */

static int row_bytes(int head_dim, int bits) { return head_dim / 8 * bits; }

/* Write code value c (b bits) as code number j of a group, LSB first. */
static void put_code(uint8_t *group_bytes, int j, int bits, unsigned c) {
    for (int k = 0; k < bits; ++k) {
        int bit = j * bits + k;
        if ((c >> k) & 1u) group_bytes[bit / 8] |= (uint8_t)(1u << (bit % 8));
    }
}

/* Read code number j of a group, LSB first. */
static unsigned get_code(const uint8_t *group_bytes, int j, int bits) {
    unsigned c = 0;
    for (int k = 0; k < bits; ++k) {
        int bit = j * bits + k;
        if ((group_bytes[bit / 8] >> (bit % 8)) & 1u) c |= 1u << k;
    }
    return c;
}

static int bits_ok(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }

/* ------------------------------------------------------------- quantize -- */

/* One group of 64 bf16 values -> 8*bits packed bytes and {s, mn}. */
static void quantize_group(const uint16_t *x, int bits, uint8_t *out, float *s_out, float *mn_out) {
    float v[ORACLE_GROUP];
    for (int i = 0; i < ORACLE_GROUP; ++i) v[i] = bf16_to_f32(x[i]);

    float mn = v[0], mx = v[0];
    for (int i = 1; i < ORACLE_GROUP; ++i) {
        if (v[i] < mn) mn = v[i];
        if (v[i] > mx) mx = v[i];
    }
    if (mn == 0.0f) mn = 0.0f; /* -0 -> +0 */
    if (mx == 0.0f) mx = 0.0f;

    const unsigned qmax = (1u << bits) - 1u;
    float s = 0.0f;
    if (mx != mn) {
        float range = mx - mn;      /* one fp32 RN subtraction */
        s = range / (float)qmax;    /* one fp32 RN division */
    }

    memset(out, 0, (size_t)(8 * bits));
    for (int i = 0; i < ORACLE_GROUP; ++i) {
        unsigned c = 0;
        if (s != 0.0f) {
            float a = v[i] - mn;    /* fp32 RN */
            float t = a / s;        /* fp32 RN */
            float r = nearbyintf(t); /* default rounding mode: half to even */
            if (r < 0.0f) r = 0.0f;
            if (r > (float)qmax) r = (float)qmax;
            c = (unsigned)r;
        }
        put_code(out, i, bits, c);
    }
    *s_out = s;
    *mn_out = mn;
}

/* x: bf16 [n_rows][head_dim]; codes: [n_rows][head_dim*bits/8];
 * scalemin: float [n_rows][head_dim/64][2] = {s, mn}. */
int oracle_quantize_rows(const uint16_t *x, int64_t n_rows, int32_t head_dim, int32_t bits,
                         uint8_t *codes, float *scalemin) {
    if (!bits_ok(bits) || head_dim <= 0 || head_dim % ORACLE_GROUP) return 2;
    const int ng = head_dim / ORACLE_GROUP;
    const int rb = row_bytes(head_dim, bits);
    for (int64_t r = 0; r < n_rows; ++r) {
        for (int g = 0; g < ng; ++g) {
            float s, mn;
            quantize_group(x + r * head_dim + g * ORACLE_GROUP, bits,
                           codes + r * rb + g * 8 * bits, &s, &mn);
            scalemin[(r * ng + g) * 2 + 0] = s;
            scalemin[(r * ng + g) * 2 + 1] = mn;
        }
    }
    return 0;
}

/* ----------------------------------------------------------- dequantize -- */

int oracle_dequantize_rows(const uint8_t *codes, const float *scalemin, int64_t n_rows,
                           int32_t head_dim, int32_t bits, uint16_t *y) {
    if (!bits_ok(bits) || head_dim <= 0 || head_dim % ORACLE_GROUP) return 2;
    const int ng = head_dim / ORACLE_GROUP;
    const int rb = row_bytes(head_dim, bits);
    for (int64_t r = 0; r < n_rows; ++r) {
        for (int g = 0; g < ng; ++g) {
            const float s = scalemin[(r * ng + g) * 2 + 0];
            const float mn = scalemin[(r * ng + g) * 2 + 1];
            const uint8_t *grp = codes + r * rb + g * 8 * bits;
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                unsigned c = get_code(grp, i, bits);
                y[r * head_dim + g * ORACLE_GROUP + i] = f32_to_bf16_rne(fmaf((float)c, s, mn));
            }
        }
    }
    return 0;
}

/* Integer codes, one byte each: c_out [n_rows][head_dim]. */
int oracle_unpack_rows(const uint8_t *codes, int64_t n_rows, int32_t head_dim, int32_t bits,
                       uint8_t *c_out) {
    if (!bits_ok(bits) || head_dim <= 0 || head_dim % ORACLE_GROUP) return 2;
    const int ng = head_dim / ORACLE_GROUP;
    const int rb = row_bytes(head_dim, bits);
    for (int64_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < ng; ++g)
            for (int i = 0; i < ORACLE_GROUP; ++i)
                c_out[r * head_dim + g * ORACLE_GROUP + i] =
                    (uint8_t)get_code(codes + r * rb + g * 8 * bits, i, bits);
    return 0;
}

/* Exact affine value mn + s*c in fp64 (the value attention attends over). */
int oracle_affine_rows(const uint8_t *codes, const float *scalemin, int64_t n_rows,
                       int32_t head_dim, int32_t bits, double *out) {
    if (!bits_ok(bits) || head_dim <= 0 || head_dim % ORACLE_GROUP) return 2;
    const int ng = head_dim / ORACLE_GROUP;
    const int rb = row_bytes(head_dim, bits);
    for (int64_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < ng; ++g) {
            const double s = (double)scalemin[(r * ng + g) * 2 + 0];
            const double mn = (double)scalemin[(r * ng + g) * 2 + 1];
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                unsigned c = get_code(codes + r * rb + g * 8 * bits, i, bits);
                out[r * head_dim + g * ORACLE_GROUP + i] = mn + s * (double)c;
            }
        }
    return 0;
}

/* ------------------------------------------------------ decode attention -- */

/*
 * One (agent, layer) view, one decode query per query head.
 *
 * Sequence attended by every query head: the n_packed quantized tokens, in
 * order, followed by the n_window bf16 recent-window tokens in logical
 * (oldest-first) order.  Query head h reads KV head h / (n_q_heads /
 * n_kv_heads) (consecutive query heads share a KV head).
 *
 *   logit_t = softmax_scale * sum_d q[h][d] * k_t[d]
 *   p_t     = exp(logit_t - max_t logit_t) / sum_t exp(logit_t - max logit)
 *   out[h]  = sum_t p_t * v_t
 *
 * with packed k_t, v_t the exact affine values mn + s*c, window values the
 * bf16 numbers, everything in fp64, softmax in two passes (max, then sums).
 *
 * Layouts: k_codes/v_codes [n_kv][n_packed][head_dim*bits/8],
 * k_sm/v_sm [n_kv][n_packed][head_dim/64][2], k_win/v_win bf16
 * [n_kv][n_window][head_dim], q bf16 [n_q][head_dim], out [n_q][head_dim],
 * probs (optional, may be NULL) [n_q][n_packed + n_window].
 */
int oracle_decode_attn(int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t bits,
                       int64_t n_packed, const uint8_t *k_codes, const float *k_sm,
                       const uint8_t *v_codes, const float *v_sm,
                       int64_t n_window, const uint16_t *k_win, const uint16_t *v_win,
                       const uint16_t *q, double softmax_scale, double *out, double *probs) {
    if (n_kv_heads <= 0 || n_q_heads % n_kv_heads) return 1;
    if (head_dim <= 0 || head_dim % ORACLE_GROUP) return 2;
    if (n_packed > 0 && !bits_ok(bits)) return 2;
    const int64_t n = n_packed + n_window;
    if (n <= 0) return 1;
    const int group_q = n_q_heads / n_kv_heads;
    const int D = head_dim;

    double *kh = (double *)malloc(sizeof(double) * (size_t)(n * D));
    double *vh = (double *)malloc(sizeof(double) * (size_t)(n * D));
    double *logit = (double *)malloc(sizeof(double) * (size_t)n);
    double *qd = (double *)malloc(sizeof(double) * (size_t)D);
    if (!kh || !vh || !logit || !qd) {
        free(kh); free(vh); free(logit); free(qd);
        return 4;
    }

    for (int hk = 0; hk < n_kv_heads; ++hk) {
        /* Keys and values of this KV head as fp64 rows: packed, then window. */
        if (n_packed > 0) {
            const int rb = row_bytes(D, bits);
            const int ng = D / ORACLE_GROUP;
            oracle_affine_rows(k_codes + (int64_t)hk * n_packed * rb,
                               k_sm + (int64_t)hk * n_packed * ng * 2, n_packed, D, bits, kh);
            oracle_affine_rows(v_codes + (int64_t)hk * n_packed * rb,
                               v_sm + (int64_t)hk * n_packed * ng * 2, n_packed, D, bits, vh);
        }
        for (int64_t t = 0; t < n_window; ++t)
            for (int d = 0; d < D; ++d) {
                kh[(n_packed + t) * D + d] = bf16_to_f32(k_win[((int64_t)hk * n_window + t) * D + d]);
                vh[(n_packed + t) * D + d] = bf16_to_f32(v_win[((int64_t)hk * n_window + t) * D + d]);
            }

        for (int j = 0; j < group_q; ++j) {
            const int h = hk * group_q + j;
            for (int d = 0; d < D; ++d) qd[d] = bf16_to_f32(q[(int64_t)h * D + d]);

            double mx = -INFINITY;
            for (int64_t t = 0; t < n; ++t) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qd[d] * kh[t * D + d];
                logit[t] = softmax_scale * acc;
                if (logit[t] > mx) mx = logit[t];
            }
            double denom = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                logit[t] = exp(logit[t] - mx); /* now the unnormalised weight */
                denom += logit[t];
            }
            double *o = out + (int64_t)h * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                const double p = logit[t] / denom;
                if (probs) probs[(int64_t)h * n + t] = p;
                for (int d = 0; d < D; ++d) o[d] += p * vh[t * D + d];
            }
        }
    }
    free(kh); free(vh); free(logit); free(qd);
    return 0;
}
