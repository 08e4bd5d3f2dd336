/*
 * kvq.h -- C ABI of the quantized KV-cache library for NVIDIA B200 (sm_100a).
 *
 * What the library computes (pages and sections):
 *  - "QKVShare: Quantized KV-Cache Handoff for Multi-Agent On-Device LLMs",
 *    Riepilogo Tecnico / Metodologia: an agent hands its KV cache to the next
 *    one as quantized groups instead of making it re-prefill, and the
 *    receiver rebuilds full-precision K/V from them before its forward pass
 *    (kvq_quantize, kvq_dequantize).
 *  - "Agent Memory Below the Prompt: Persistent Q4 KV Cache for Multi-Agent
 *    LLM Inference on Edge Devices", Abstract: 4-bit caches are loaded
 *    directly into the attention layer and several agents' quantized caches
 *    are attended concurrently (kvq_decode_attn over an array of views).
 *  - "Coordinated Mixed-Precision KV Cache Quantization for Efficient
 *    LLM-based Multi-agent Systems", Abstract: each (agent, layer) has its own
 *    width, recent states keep native precision, and only newly quantized
 *    blocks take a width while older blocks stay as they are (kvq_view.bits,
 *    the bf16 recent window, kvq_append); the widths come from a sensitivity
 *    bound and a budgeted allocation (kvq_width_sensitivity,
 *    kvq_allocate_widths), and a sequence may span views of several widths
 *    (kvq_decode_attn_seq).
 *  - QKVShare, Metodologia: the CacheCard artifact that carries the quantized
 *    groups and their metadata (kvq_card_*).
 *  - "Reasoning-Aware Error-Bounded KV-Cache Compression and Sparse Attention
 *    for Long-Context LLMs", Metodologia C: top-K sparse decode attention
 *    (kvq_sparse_decode_attn).
 *
 * Quantization format (the pages leave it open; this is the library's
 * definition):
 *  - group = 64 consecutive elements along head_dim of one (head, token) row;
 *  - mn, mx = min and max of the group in fp32 (a zero is stored as +0.0f);
 *    s = (mx - mn) / (2^bits - 1), one fp32 round-to-nearest division, s = 0
 *    when mx == mn;
 *  - code = clamp(round_half_to_even((x - mn) / s), 0, 2^bits - 1) with
 *    x - mn and the division each one fp32 round-to-nearest step; all codes
 *    are 0 when s == 0;
 *  - code j of a group occupies bits [j*bits, (j+1)*bits) of the group's
 *    little-endian byte string, least significant bit first; a group is
 *    8*bits bytes and the groups of a row follow in head_dim order, so a row
 *    is row_bytes = head_dim*bits/8 bytes;
 *  - per group one float pair {s, mn} ("scalemin");
 *  - dequantized value: bf16_round_half_to_even(fmaf((float)code, s, mn));
 *    attention attends over the affine value mn + s*code without the bf16
 *    rounding.
 *  Supported: bits in {2, 3, 4, 8}; head_dim a multiple of 64, at most 256.
 *  Inputs with NaN or Inf, or whose group range mx - mn overflows fp32, are
 *  outside the contract.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; views and
 *    other structs are HOST memory.  The library allocates no device memory,
 *    never synchronizes the host with the device, and enqueues all work on
 *    `stream` (a cudaStream_t; NULL means the legacy default stream) in the
 *    caller's current CUDA device context.
 *  - Arguments are validated on the host before anything is enqueued; on any
 *    error nothing is enqueued and outputs are untouched.
 *  - KVQ_ERR_CUDA reports a failed launch (the CUDA error is left for the
 *    caller to inspect with cudaGetLastError/cudaPeekAtLastError).
 *  - Calls that share output or workspace memory and overlap on the GPU race;
 *    order them on one stream.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_GROUP_SIZE 64
#define KVQ_MAX_HEAD_DIM 256

typedef enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or stride */
    KVQ_ERR_UNSUPPORTED = 2, /* bits not in {2,3,4,8}, head_dim not 64..256 step 64 */
    KVQ_ERR_CAPACITY = 3,    /* a capacity is exceeded: an append past cap_packed, a card
                                into smaller views, a scratch or a byte budget too small */
    KVQ_ERR_CUDA = 4         /* a kernel launch or device query failed */
} kvq_status;

/* Static, NUL-terminated name of a status code ("unknown status" otherwise). */
const char *kvq_status_string(int32_t status);

/* ABI version of this header (incremented on any incompatible change). */
int32_t kvq_abi_version(void);

/*
 * kvq_quantize -- group-wise affine quantization of bf16 K or V rows
 * (QKVShare, Metodologia: the quantized card; Agent Memory, Abstract: 4-bit
 * format; CoMixKV, Abstract: widths per (agent, layer)).
 *
 *  x          bf16 input, element (h, t, d) at x[h*x_head_stride +
 *             t*x_tok_stride + d] (strides in ELEMENTS; d contiguous).
 *             x must be 16-byte aligned and both strides multiples of 8.
 *  n_heads, n_tokens, head_dim, bits   sizes; n_heads*n_tokens may be 0
 *             (nothing is enqueued).
 *  codes      u8 output, row (h, t) at codes + (h*out_head_cap + t)*row_bytes;
 *             16-byte aligned.
 *  scalemin   float output, group g of row (h, t) at
 *             scalemin + ((h*out_head_cap + t)*(head_dim/64) + g)*2, holding
 *             {s, mn}; 8-byte aligned.
 *  out_head_cap  rows per head in codes/scalemin, >= n_tokens.
 * Result: codes and scalemin are bit-exact functions of x (see format).
 */
kvq_status kvq_quantize(const void *x, int64_t x_head_stride, int64_t x_tok_stride,
                        int32_t n_heads, int64_t n_tokens, int32_t head_dim, int32_t bits,
                        void *codes, float *scalemin, int64_t out_head_cap, void *stream);

/*
 * kvq_dequantize -- inverse of kvq_quantize into bf16 (QKVShare, Metodologia,
 * "Percorso di Iniezione": full-precision past_key_values rebuilt from the
 * quantized card before the receiver's forward pass).
 *
 *  codes, scalemin, in_head_cap   as written by kvq_quantize (same alignment).
 *  y          bf16 output, element (h, t, d) at y[h*y_head_stride +
 *             t*y_tok_stride + d]; 16-byte aligned, strides multiples of 8.
 * Result: y = bf16_rne(fmaf(code, s, mn)), bit-exact.
 */
kvq_status kvq_dequantize(const void *codes, const float *scalemin, int64_t in_head_cap,
                          int32_t n_heads, int64_t n_tokens, int32_t head_dim, int32_t bits,
                          void *y, int64_t y_head_stride, int64_t y_tok_stride, void *stream);

/*
 * One (agent, layer) KV cache: n_packed quantized tokens followed by
 * n_window bf16 recent-window tokens (CoMixKV, Abstract: recent states keep
 * native precision).  All pointers are device memory owned by the caller.
 *
 *  bits          width of this view's packed tokens (2, 3, 4 or 8).
 *  n_packed      packed tokens in use, 0 <= n_packed <= cap_packed.
 *  cap_packed    packed rows per KV head; must be even.
 *  n_window      valid window tokens, 0 <= n_window <= cap_window.
 *  cap_window    window ring slots per KV head (W); 0 = no window.
 *  window_head   ring slot of the oldest window token; window token i
 *                (0 = oldest) lives in slot (window_head + i) % cap_window.
 *  k_codes, v_codes        u8 [n_kv_heads][cap_packed][row_bytes], 16-B aligned.
 *  k_scalemin, v_scalemin  float [n_kv_heads][cap_packed][head_dim/64][2], 16-B aligned.
 *  k_window, v_window      bf16 [n_kv_heads][cap_window][head_dim], 16-B aligned
 *                          (may be NULL when cap_window == 0).
 * The sequence a query attends is packed tokens 0..n_packed-1, then window
 * tokens oldest to newest.
 * Every call takes at most KVQ_MAX_VIEWS views (KVQ_ERR_INVALID_ARG beyond).
 */
#define KVQ_MAX_VIEWS (1 << 22)

typedef struct kvq_view {
    int32_t bits;
    int32_t n_window;
    int32_t cap_window;
    int32_t window_head;
    int64_t n_packed;
    int64_t cap_packed;
    void *k_codes;
    void *v_codes;
    float *k_scalemin;
    float *v_scalemin;
    void *k_window;
    void *v_window;
} kvq_view;

/*
 * kvq_append -- add one new token to each of n_views views (one decode step
 * of several agents or layers in a single launch).  CoMixKV, Abstract: the
 * new token enters in native precision; when the window is full its oldest
 * token is quantized at the view's CURRENT bits and appended to the packed
 * part, while earlier packed tokens are never touched.  With cap_window == 0
 * the new token is quantized immediately.
 *
 *  views      HOST array, read and then updated in place (n_packed, n_window,
 *             window_head) to describe the state after the append.  Each view
 *             must have distinct device buffers from every other view.
 *  k_new, v_new  bf16 [n_views][n_kv_heads][head_dim] device arrays, 16-B aligned.
 * Errors: KVQ_ERR_CAPACITY if any view would need to flush while
 * n_packed == cap_packed (nothing is enqueued and no view is changed).
 */
kvq_status kvq_append(kvq_view *views, int32_t n_views, int32_t n_kv_heads, int32_t head_dim,
                      const void *k_new, const void *v_new, void *stream);

/*
 * Bytes of device workspace kvq_decode_attn needs for these views on the
 * current device (0 when the arguments are invalid).  The workspace must be
 * zero-filled once before its first use; every completed call leaves it
 * ready for the next one.  Its first 4 bytes are a device status word: 0
 * normally; 1 if a bounded wait for a copy into shared memory expired, in
 * which case the outputs of that call are not valid.
 */
size_t kvq_decode_attn_workspace_size(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t head_dim);

/*
 * kvq_decode_attn -- batched split-K decode attention straight over several
 * views' packed caches and bf16 windows (Agent Memory, Abstract:
 * BatchQuantizedKVCache, caches loaded directly into attention; QKVShare,
 * Significato: the fused quantized attention kernel the prototype deferred).
 *
 *  views      HOST array of n_views views (any mix of bits and lengths; each
 *             view must have n_packed + n_window >= 1).
 *  n_q_heads, n_kv_heads   n_q_heads % n_kv_heads == 0; query head h reads
 *             KV head h / (n_q_heads / n_kv_heads).
 *  q          bf16 [n_views][n_q_heads][head_dim] device array, 16-B aligned.
 *  softmax_scale   logits are softmax_scale * (q . k), e.g. 1/sqrt(head_dim).
 *  out        float [n_views][n_q_heads][head_dim] device array, 16-B aligned:
 *             out = sum_t softmax_t * v_t over packed-then-window tokens.
 *  workspace  device scratch of at least kvq_decode_attn_workspace_size(...)
 *             bytes, 256-B aligned, zero-filled before first use.
 * The result is deterministic: the same inputs on the same device give the
 * same bits (no floating-point atomics; partial results merge in a fixed
 * order).
 * Stream order: the attention grid is launched with programmatic stream
 * serialization.  It starts copying the views' packed rows and windows into
 * shared memory before it waits for the preceding kernel of the stream, and
 * reads q, writes out and touches the workspace only after that wait; it
 * lets the next kernel start once it has waited.  Every library call that
 * writes packed rows or windows (kvq_append, kvq_quantize, kvq_card_unpack)
 * lets a following kernel start only when it has completed, and so does any
 * kernel launched without programmatic serialization.  A caller's own kernel
 * that writes a view's rows and calls griddepcontrol.launch_dependents
 * before those writes must not be the kernel right before this call.
 */
kvq_status kvq_decode_attn(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                           int32_t n_kv_heads, int32_t head_dim, const void *q,
                           float softmax_scale, float *out, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * Sequences made of several views (segments).  A sequence's cache may be held
 * by more than one view, each with its own width: blocks flushed before and
 * after a change of the layer's width (CoMixKV, Abstract: only newly quantized
 * blocks take the new allocation, old ones are not requantized), or tokens of
 * one sequence kept at different widths by importance (QKVShare, Metodologia:
 * per-token widths {2, 4, 8, FP16}; FP16 tokens are a view with a window only).
 * Softmax attention does not depend on the order of the (key, value) pairs,
 * so the sequence's output is attention over the union of its views' tokens.
 *
 * KVQ_MAX_SEGMENTS: views holding tokens, per sequence.
 */
#define KVQ_MAX_SEGMENTS 64

/*
 * kvq_decode_attn_seq_workspace_size -- scratch bytes kvq_decode_attn_seq
 * needs for these views and sequences; 0 if the arguments are invalid.
 */
size_t kvq_decode_attn_seq_workspace_size(const kvq_view *views, int32_t n_views,
                                          const int32_t *seq_begin, int32_t n_seqs,
                                          int32_t n_q_heads, int32_t n_kv_heads,
                                          int32_t head_dim);

/*
 * kvq_decode_attn_seq -- kvq_decode_attn over sequences of views.
 *
 *  views      HOST array of n_views views; a view may be empty (no tokens).
 *  seq_begin  HOST int32 [n_seqs + 1]: sequence s is views seq_begin[s] ..
 *             seq_begin[s+1]-1.  seq_begin[0] == 0, seq_begin[n_seqs] ==
 *             n_views, strictly increasing; every sequence holds >= 1 token
 *             and at most KVQ_MAX_SEGMENTS non-empty views.  Views of any
 *             widths may share a sequence.
 *  q          bf16 [n_seqs][n_q_heads][head_dim] device array, 16-B aligned.
 *  out        float [n_seqs][n_q_heads][head_dim], 16-B aligned: attention of
 *             q[s] over the tokens of all views of sequence s.
 *  workspace  at least kvq_decode_attn_seq_workspace_size(...) bytes, 256-B
 *             aligned, zero-filled before first use (left ready for the next
 *             call, as with kvq_decode_attn).
 * Deterministic, like kvq_decode_attn: partials merge in view order, then
 * chunk order.  With seq_begin = {0, 1, ..., n_views} the result is bitwise
 * that of kvq_decode_attn.
 * Errors: KVQ_ERR_INVALID_ARG for a malformed seq_begin or an empty sequence,
 * KVQ_ERR_UNSUPPORTED for more than KVQ_MAX_SEGMENTS non-empty views in a
 * sequence; otherwise as kvq_decode_attn.  Nothing is enqueued on error.
 */
kvq_status kvq_decode_attn_seq(const kvq_view *views, int32_t n_views, const int32_t *seq_begin,
                               int32_t n_seqs, int32_t n_q_heads, int32_t n_kv_heads,
                               int32_t head_dim, const void *q, float softmax_scale, float *out,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * kvq_sparse_decode_attn -- top-K sparse decode attention over packed caches
 * ("Reasoning-Aware Error-Bounded KV-Cache Compression and Sparse Attention
 * for Long-Context LLMs", Metodologia C: a query-aware score picks the K
 * entries that attend this step; the others stay in the cache).
 *
 * For every view and KV head hk:
 *   score(t) = max over the query heads h of hk's group of
 *              softmax_scale * (q_h . k_t), k_t = mn + s*c exactly, for each
 *              packed token t;
 *   the top_k packed tokens by score are selected (equal scores: the lower
 *   token index first; all of them when n_packed <= top_k);
 *   out[h] = softmax attention of q_h over the selected packed tokens and
 *   all of the view's bf16 window tokens (the recent window is always active).
 * With top_k >= n_packed the result is that of kvq_decode_attn (within
 * rounding).  When the full attention puts mass delta on the packed tokens
 * left out and every value vector has norm <= V_max, the output moves by at
 * most 2 * V_max * delta (ibid., Metodologia B).
 *
 *  views, n_q_heads, n_kv_heads, head_dim, q, softmax_scale, out
 *             as kvq_decode_attn.
 *  top_k      >= 1, packed tokens selected per (view, KV head).
 *  selected   NULL, or int32 [n_views][n_kv_heads][top_k] device array that
 *             receives the selected packed-token indices, ascending, padded
 *             with -1 when a view has fewer than top_k packed tokens.
 *  workspace  at least kvq_sparse_decode_attn_workspace_size(...) bytes,
 *             256-B aligned, zero-filled before first use; the first bytes
 *             are left ready for the next call with the same views, heads and
 *             top_k, while the sizes of the views change.
 * Scores are fp32; the attention is that of kvq_decode_attn over one view
 * per (view, KV head) whose packed part is the selected rows, read in place
 * through the selection list (in `selected` or the workspace).  The
 * selection of a view with more than 32768 packed tokens (up to 131072) runs
 * on a thread-block cluster of 2 or 4 CTAs.
 * Tuning and tests (environment, read at every call): KVQ_SELECT_CLUSTER = 2
 * or 4 splits every selection over that many CTAs (same selection);
 * KVQ_CHUNK_TOKENS forces the attention's chunk length (only the rounding of
 * the split-K merge changes).
 * Errors: as kvq_decode_attn, KVQ_ERR_INVALID_ARG for top_k < 1, and
 * KVQ_ERR_CUDA when a launch is refused (e.g. no room for a cluster).
 */
size_t kvq_sparse_decode_attn_workspace_size(const kvq_view *views, int32_t n_views,
                                             int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, int32_t top_k);

kvq_status kvq_sparse_decode_attn(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                  int32_t n_kv_heads, int32_t head_dim, const void *q,
                                  float softmax_scale, int32_t top_k, float *out,
                                  int32_t *selected, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * Width allocation across agents and layers under a shared byte budget
 * ("Coordinated Mixed-Precision KV Cache Quantization for Efficient LLM-based
 * Multi-agent Systems", Abstract: sensitivity from a local attention-error
 * bound on recent queries, keys and values; a shared controller minimizing
 * the total estimated error under byte-level storage costs; the widths apply
 * to newly quantized blocks only).  The page prints no formula; the bound
 * below is the first-order one the group-wise affine format gives.
 *
 * kvq_width_sensitivity -- per view, S such that quantizing its blocks at b
 * bits is expected to move the attention output by at most about
 * S / (2^b - 1).  Over the view's window tokens and per KV head: R_k[g],
 * R_v[g] the largest K, V range of 64-element group g, V_max the largest
 * value norm; Delta = softmax_scale * max over the head's query heads h of
 * sum_g |q_h[g]|_1 * R_k[g] / 2; E_v = sqrt(sum_g 64 * (R_v[g] / 2)^2);
 * S = 2 * V_max * Delta + E_v, the largest over KV heads (0 without window
 * tokens).  fp32.
 *  views      HOST array; only the window part is read.
 *  q          bf16 [n_views][n_q_heads][head_dim] device array, 16-B aligned
 *             (the most recent query of each view).
 *  sens       float [n_views] device array (written).
 * Errors: as kvq_decode_attn's argument checks; nothing is enqueued on error.
 */
kvq_status kvq_width_sensitivity(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                 int32_t n_kv_heads, int32_t head_dim, const void *q,
                                 float softmax_scale, float *sens, void *stream);

/*
 * kvq_allocate_widths -- host only.  Chooses bits[i] in {2, 3, 4, 8} for each
 * view to minimize sum_i sens[i] / (2^bits[i] - 1) subject to
 * sum_i cost_i(bits[i]) <= budget_bytes, where cost_i(b) = capacity[i] *
 * 2 * n_kv_heads * (head_dim*b/8 + (head_dim/64)*8) bytes, the storage of the
 * capacity[i] tokens the view has still to quantize.  The budget is cut into
 * `units` units of ceil(budget_bytes / units) bytes and costs are rounded up
 * to whole units, so the result never exceeds the budget; over those
 * allocations the total is minimal (dynamic programming, O(n_views * units)).
 * Equal totals keep the wider width of the earlier view.
 *  sens       HOST float [n_views], >= 0 and finite.
 *  capacity   HOST int64 [n_views], >= 0.
 *  bits       HOST int32 [n_views] (written).
 *  total_error  NULL or HOST double (written): the minimal total.
 * Errors: KVQ_ERR_CAPACITY if even 2 bits everywhere does not fit;
 * KVQ_ERR_INVALID_ARG for bad arguments (units outside [1, 2^20]);
 * KVQ_ERR_UNSUPPORTED when n_views * (units + 1) exceeds 2^30 (the host
 * memory of the back-pointers).
 */
kvq_status kvq_allocate_widths(const float *sens, const int64_t *capacity, int32_t n_views,
                               int32_t n_kv_heads, int32_t head_dim, uint64_t budget_bytes,
                               int32_t units, int32_t *bits, double *total_error);

/*
 * kvq_append_decode_attn -- one decode step over a batch of views: the
 * effect of kvq_append(views, ..., k_new, v_new) followed by
 * kvq_decode_attn(views, ...) on the appended views, in one call (CoMixKV,
 * Abstract: recent states stay native, only flushed blocks are quantized;
 * Agent Memory, Abstract: attention straight over the quantized caches).
 *
 * Arguments as in those two calls; the workspace is sized by
 * kvq_decode_attn_workspace_size on the views as they will be after the
 * append (each view's counters advanced by one token).  The append grid lets
 * the attention grid start before it waits for the preceding kernel itself,
 * and reads k_new, v_new and the windows' oldest tokens and quantizes before
 * that wait (only its stores follow it); so the attention grid's copies of
 * packed rows and windows overlap the previous step's tail (a previous
 * layer's attention, say), and only the copy of the block holding a row the
 * append writes (the flushed packed row, the new window token) waits for the
 * append grid.  The stream contract of kvq_decode_attn extends to k_new and
 * v_new.  Results and cache contents are the same as with the two calls.
 * Errors: those of kvq_append (nothing enqueued, no counter changed) and of
 * kvq_decode_attn's argument checks, all before anything is enqueued;
 * KVQ_ERR_CUDA if a launch fails (the counters are advanced once the append
 * is enqueued).
 */
kvq_status kvq_append_decode_attn(kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                  int32_t n_kv_heads, int32_t head_dim, const void *k_new,
                                  const void *v_new, const void *q, float softmax_scale,
                                  float *out, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * CacheCard -- one contiguous artifact holding several views' caches, for
 * handing them to another agent or process and for persistence
 * (QKVShare, Metodologia: the CacheCard packs the quantized KV groups, their
 * width assignment and metadata -- sequence length, model id, position
 * offset; Agent Memory, Abstract: per-agent 4-bit caches persisted and
 * reloaded straight into attention).
 *
 * Layout (little-endian; version 1):
 *   [0, 64)          header: "KVQCARD1", u32 version, u32 n_views,
 *                    u32 n_kv_heads, u32 head_dim, u64 model_id,
 *                    u64 total_bytes, 24 bytes zero
 *   [64, 64+64*n)    per view: u32 bits, u32 n_window, u64 n_packed,
 *                    i64 position_offset, u64 data_offset, u64 data_bytes,
 *                    u64 seq_len (= n_packed + n_window), 16 bytes zero
 *   per view, at data_offset (256-byte aligned), six 16-byte-aligned
 *   sections: K codes [H][n_packed][row_bytes], V codes, K scale/min
 *   [H][n_packed][head_dim/64][2] fp32, V scale/min, K window
 *   [H][n_window][head_dim] bf16 oldest first, V window.
 * Only the used rows travel: a card is independent of the views' capacities
 * and of where their rings start.
 */

/* Bytes of the card of these views (0 when the arguments are invalid). */
size_t kvq_card_bytes(const kvq_view *views, int32_t n_views, int32_t n_kv_heads,
                      int32_t head_dim);

/*
 * kvq_card_pack -- write the card of n_views views into DEVICE memory `card`
 * (256-byte aligned, at least kvq_card_bytes bytes), on `stream`; copy it to
 * the host with cudaMemcpyAsync for transfer or storage.
 *  model_id           stored in the header as given (the caller's tag).
 *  position_offsets   HOST array of n_views positions of each view's first
 *                     token, or NULL for zeros.
 */
kvq_status kvq_card_pack(const kvq_view *views, int32_t n_views, int32_t n_kv_heads,
                         int32_t head_dim, uint64_t model_id, const int64_t *position_offsets,
                         void *card, size_t card_bytes, void *stream);

/*
 * kvq_card_read_header / kvq_card_view_info -- read a card held in HOST
 * memory (validated: magic, version, sizes, and every offset where the
 * layout puts it).  Any output pointer may be NULL.  Use them to allocate
 * views that can take the card: each view's bits must match the card's and
 * its capacities must hold n_packed and n_window.
 */
kvq_status kvq_card_read_header(const void *card_host, size_t card_bytes, int32_t *n_views,
                                int32_t *n_kv_heads, int32_t *head_dim, uint64_t *model_id);
kvq_status kvq_card_view_info(const void *card_host, size_t card_bytes, int32_t index,
                              int32_t *bits, int64_t *n_packed, int32_t *n_window,
                              int64_t *position_offset);

/*
 * kvq_card_unpack -- restore a card into n_views views.  The card's bytes
 * are given twice: `card_host` (HOST copy, parsed and validated here) and
 * `card` (DEVICE copy of the same bytes, 256-byte aligned, read by the
 * kernel).  The views' buffers receive the used rows; their counters are set
 * from the card (n_packed, n_window; window_head = 0: the window lands in
 * ring slots 0..n_window-1).
 * Errors (nothing enqueued, no view changed): KVQ_ERR_INVALID_ARG for a card
 * that fails validation, counts that differ from the card's, or a view whose
 * bits differ from its record; KVQ_ERR_CAPACITY when a view cannot hold its
 * record's tokens.
 */
kvq_status kvq_card_unpack(const void *card_host, const void *card, size_t card_bytes,
                           kvq_view *views, int32_t n_views, int32_t n_kv_heads,
                           int32_t head_dim, void *stream);

/*
 * kvq_debug_build -- 1 in the debug build of the library (libkvq_debug.so,
 * compiled with -DKVQ_DEBUG), 0 in the normal one.  No counterpart in the
 * pages: a test aid in place of a sanitizer.  In the debug build every kernel
 * checks the global addresses it computes against the extents of the buffers
 * they belong to (a view head's packed rows, its window ring, q, out, the
 * workspace, the card image, the score and selection arrays); a failed check
 * sets a bit in one device word and the access is skipped, so nothing traps.
 */
int32_t kvq_debug_build(void);

/*
 * kvq_debug_flags -- copy the debug build's flags word of the current device
 * into `flags` (4-byte aligned; device memory or host memory the copy engine
 * can reach, pinned for an asynchronous copy), enqueued on `stream`, then
 * clear the word when `clear` is nonzero.  Stream-ordered: the word holds the
 * failed checks of the kernels enqueued before this call (bit 0 packed-row
 * copies, 1 window copies, 2 shared-memory stages, 3 q/out/scores, 4
 * workspace, 5 codec, 6 append, 7 card, 8 scores, 9 selections, 10
 * sensitivity).  Errors: KVQ_ERR_UNSUPPORTED in the normal build,
 * KVQ_ERR_INVALID_ARG for a null or misaligned `flags`, KVQ_ERR_CUDA when
 * the copy cannot be enqueued.
 */
kvq_status kvq_debug_flags(uint32_t *flags, int32_t clear, void *stream);

/* Bytes of the per-device scratch array kvq_decode_attn_noalloc uses. */
#define KVQ_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * kvq_decode_attn_noalloc -- kvq_decode_attn without a caller-supplied
 * workspace, allocating no device memory.  None of the source pages has a
 * counterpart: this is a convenience of the library.
 *
 * For callers that cannot allocate device memory at the moment they attend:
 * a serving loop that has handed all free HBM to its KV-cache pool (any later
 * cudaMalloc would fail), or a plain C host with no device allocator of its
 * own to hold a workspace.  The scratch instead comes from one fixed array of
 * KVQ_NOALLOC_SCRATCH_BYTES per device, compiled into the library.
 *
 * Arguments, layouts and results are those of kvq_decode_attn without
 * workspace / workspace_bytes; the same kernels run on the same plan, so the
 * result is the same.
 * Set-up: every call looks up the array's device address on the current
 * device (a host-side runtime query, no device work), so a device reset or a
 * re-created primary context never leaves a stale address in use.  The first
 * call on a device also loads the library's device code there; make that
 * first call before any stream capture.
 * Each call clears the array's status word and arrival counters on `stream`
 * before its kernels.  The status word (0, or 1 when a bounded copy wait gave
 * up and the outputs of that call are not valid) can be read back with
 * kvq_decode_attn_noalloc_status before the next call clears it.
 * Errors: KVQ_ERR_CAPACITY, with nothing enqueued, when the views need more
 * scratch than KVQ_NOALLOC_SCRATCH_BYTES (kvq_decode_attn_workspace_size
 * gives the need); KVQ_ERR_CUDA if the address lookup fails; otherwise as
 * kvq_decode_attn.
 * Concurrency: every call on a device shares the one array, so calls that can
 * overlap on the GPU (different streams, different host threads) race and
 * corrupt each other's results: keep them in one stream or serialize them.
 */
kvq_status kvq_decode_attn_noalloc(const kvq_view *views, int32_t n_views, int32_t n_q_heads,
                                   int32_t n_kv_heads, int32_t head_dim, const void *q,
                                   float softmax_scale, float *out, void *stream);

/*
 * kvq_decode_attn_noalloc_status -- copy the status word of the current
 * device's scratch array into `status` (4-byte aligned; device memory, or
 * host memory the copy engine can reach: pinned host memory keeps the copy
 * asynchronous), enqueued on `stream`.  Stream-ordered: it reads the word as
 * the kvq_decode_attn_noalloc call enqueued before it on that stream left it,
 * and a later call clears the word again.  0: the outputs are valid; 1: a
 * bounded copy wait gave up, the outputs of that call are not valid.  Like
 * kvq_decode_attn_noalloc it allocates nothing; no counterpart in the pages.
 * Errors: KVQ_ERR_INVALID_ARG for a null or misaligned `status`,
 * KVQ_ERR_CUDA when the address lookup or the copy cannot be enqueued.
 */
kvq_status kvq_decode_attn_noalloc_status(uint32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
