/*
 * lwm_blockattn.h -- C ABI of liblwm_blockattn.so: blockwise packed causal
 * RoPE self-attention (forward and backward) on one NVIDIA B200 (sm_100a).
 *
 * What is computed (for every batch row b, head h and query token i):
 *   q~_i = R(pos_i) q_i,  k~_j = R(pos_j) k_j      RoPE, interleaved pairs
 *   A(i) = { j : seg_j == seg_i and j <= i }         packing + causal mask
 *   s_ij = (q~_i . k~_j) / sqrt(D)                   for j in A(i)
 *   lse_i = log sum_{j in A(i)} exp(s_ij)            natural log
 *   out_i = sum_{j in A(i)} exp(s_ij - lse_i) v_j
 * and, for the backward, the chain rule of the above with respect to the
 * un-rotated q and k and to v.
 *
 * Where the pages define it:
 *   - blockwise attention over query/key chunks (scan_query_chunk_size,
 *     scan_key_chunk_size = block_q, block_k): "LWM：突破 100 万 Token 的
 *     开源大模型", 配置参数 and 脚本运行说明;
 *   - masked sequence packing (a token attends only inside its example):
 *     same page, 概述 contribution (b); "[论文解读] World Model on
 *     Million-Length Video And Language With Blockwise RingAttention",
 *     提出的方法;
 *   - RoPE with a context-scaled theta: same review, 提出的方法;
 *   - the ring sweep of key/value blocks and the FlashAttention-style
 *     online softmax: "开源巨兽LWM：如何用RingAttention撬动百万Token多模态
 *     世界", 3.1 and 3.2; "Inside Large World Model", Stage I.
 * Readings where the pages are silent: scale 1/sqrt(D); pair k of a head
 * vector is (x[2k], x[2k+1]) with frequency theta^(-2k/D); angles in fp64;
 * the causal rule compares token indices (positions drive RoPE only).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates device memory and never frees anything.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call
 *     except lwm_blockattn_check_inputs and lwm_blockattn_last_status is
 *     asynchronous on `stream`.
 *   - Arguments are validated on the host before any launch; on error a
 *     status code is returned and nothing is launched. Nothing aborts.
 *   - Layouts (row-major, contiguous):
 *       q, k, v, out, dout, dq, dk, dv : [B][N][H][D]
 *       segment_ids, positions         : [B][N] int32
 *       lse                            : [B][H][N] float32
 *   - dtype LWM_DTYPE_BF16: q/k/v/out/dout/dq/dk/dv are bfloat16 and the
 *     tensor-core path runs (tcgen05, fp32 accumulate).
 *     dtype LWM_DTYPE_FP32: those tensors are float32 and an fp32 CUDA-core
 *     path runs (accuracy mode; not a performance target).
 *   - qk_precision LWM_QK_BF16: rotated q and k are rounded to bf16 before
 *     Q K^T. LWM_QK_BF16X3: they are split as hi + lo (both bf16) and
 *     Q K^T = hi.hi + hi.lo + lo.hi, for inputs whose scores are large
 *     enough that bf16 rounding of rotated q/k would move the logsumexp by
 *     more than ~1e-3. Ignored for LWM_DTYPE_FP32.
 *   - Preconditions the kernels trust (lwm_blockattn_check_inputs verifies
 *     them): segment_ids non-decreasing along each batch row (packed
 *     examples are contiguous runs); 0 <= positions < max_pos.
 *   - Supported shapes: D == 128; block_q == 128; block_k == 128 or 64
 *     (the forward sweeps key tiles of block_k keys; with 64 the first key
 *     tile a query block visits leaves half of its rows with no visible
 *     key yet, which the online softmax handles; the key-major backward
 *     visits 128-key units either way, an exact reorganisation with the
 *     same gradients); any N >= 0 (a ragged last block is masked);
 *     B, H >= 0 (0 => no work); every tensor pointer 16-byte aligned.
 */
#ifndef LWM_BLOCKATTN_H
#define LWM_BLOCKATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LWM_BLOCKATTN_VERSION 1

#if defined(__GNUC__)
#define LWM_API __attribute__((visibility("default")))
#else
#define LWM_API
#endif

typedef enum {
  LWM_OK = 0,
  LWM_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size ... */
  LWM_ERR_UNSUPPORTED = 2,   /* valid but not implemented (D != 128 ...)    */
  LWM_ERR_WORKSPACE = 3,     /* workspace null or smaller than required     */
  LWM_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed           */
  LWM_ERR_TIMEOUT = 5,       /* a device-side bounded wait gave up          */
  LWM_ERR_PRECONDITION = 6   /* check_inputs: ids decrease / pos range     */
} lwm_status;

typedef enum { LWM_DTYPE_BF16 = 0, LWM_DTYPE_FP32 = 1 } lwm_dtype;
typedef enum { LWM_QK_BF16 = 0, LWM_QK_BF16X3 = 1 } lwm_qk_precision;

/* Which head dims RoPE rotates together with frequency theta^(-2k/D):
 * LWM_ROPE_INTERLEAVED pairs (x[2k], x[2k+1]) (the Jax/EasyLM layout the
 * LWM checkpoints were trained in); LWM_ROPE_HALF pairs (x[k], x[k+D/2]),
 * the rotate-half layout of Hugging Face LlamaForCausalLM, which is how the
 * PyTorch models load ("LWM：突破 100 万 Token 的开源大模型", 脚本运行说明,
 * 运行 PyTorch 模型). The two give the same attention once the head dims of
 * q and k are permuted; gradients come back in the inputs' layout. */
typedef enum { LWM_ROPE_INTERLEAVED = 0, LWM_ROPE_HALF = 1 } lwm_rope_layout;

/* Tile classes written by lwm_blockattn_classify. */
enum { LWM_TILE_EMPTY = 0, LWM_TILE_PARTIAL = 1, LWM_TILE_FULL = 2 };

/* Bytes of device workspace lwm_blockattn_fwd needs for these sizes,
 * dtype and qk_precision: the RoPE cos/sin table (max_pos x D/2 float
 * pairs), per-block and per-row segment metadata, the work order and, for
 * LWM_DTYPE_BF16, the rotated keys R(pos) k (B*N*H*D bf16; twice that for
 * LWM_QK_BF16X3, which keeps the bf16 residual too). Returns 0 for invalid
 * sizes. */
LWM_API size_t lwm_blockattn_fwd_workspace_size(int B, int N, int H, int D,
                                        int block_q, int block_k,
                                        int max_pos, int dtype,
                                        int qk_precision);

/* Same for lwm_blockattn_bwd: additionally an fp32 dQ accumulator of
 * B*N*H*D floats, the per-row dot(dO, O) of B*H*N floats and, for
 * LWM_DTYPE_BF16, the rotated queries as well as keys. */
LWM_API size_t lwm_blockattn_bwd_workspace_size(int B, int N, int H, int D,
                                        int block_q, int block_k,
                                        int max_pos, int dtype,
                                        int qk_precision);

/* Forward. Writes out [B][N][H][D] (dtype) and lse [B][H][N] (fp32,
 * natural log of the softmax denominator of the scaled scores).
 * theta > 0 is the RoPE base; positions must lie in [0, max_pos);
 * rope_layout is an lwm_rope_layout.
 * The workspace is scratch owned by the caller (>= the size above, 256-byte
 * aligned); its content on entry does not matter and is clobbered.
 * Returns LWM_OK or an error status (nothing launched on error). */
LWM_API int lwm_blockattn_fwd(const void* q, const void* k, const void* v,
                      const int32_t* segment_ids, const int32_t* positions,
                      double theta, int block_q, int block_k, int max_pos,
                      int B, int N, int H, int D, int dtype, int qk_precision,
                      int rope_layout, void* out, float* lse,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Backward. Given the forward's inputs, its out and lse, and dout (the
 * gradient of the loss with respect to out), writes dq, dk, dv (dtype,
 * [B][N][H][D]): gradients with respect to the un-rotated q and k and v.
 * P is recomputed from lse; dq is accumulated in fp32 in the workspace
 * (its summation order is not fixed, so dq is not bit-reproducible). */
LWM_API int lwm_blockattn_bwd(const void* q, const void* k, const void* v,
                      const void* out, const void* dout, const float* lse,
                      const int32_t* segment_ids, const int32_t* positions,
                      double theta, int block_q, int block_k, int max_pos,
                      int B, int N, int H, int D, int dtype, int qk_precision,
                      int rope_layout, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------
 * Ring attention building blocks ("开源巨兽LWM：如何用RingAttention撬动百万
 * Token多模态世界", 3.1 RingAttention: each device keeps its query block,
 * key/value blocks pass around a ring of devices, and each step's partial
 * attention is folded into the running result with the log-sum-exp rule).
 *
 * Bytes of workspace lwm_blockattn_fwd_block needs: RoPE table and the
 * per-row / per-block metadata of Nq queries against Nk keys. */
LWM_API size_t lwm_blockattn_fwd_block_workspace_size(int B, int Nq, int Nk,
                                                      int H, int D,
                                                      int max_pos);

/* Partial forward of query rows [q_off, q_off+Nq) of a packed sequence
 * against its key/value rows [k_off, k_off+Nk) (global token indices; the
 * two ranges may be any pieces of the same sequence). Row i sees key j iff
 * j <= i and seg_q[i] == seg_k[j]; rows with no visible key get out = 0,
 * lse = -inf.
 *   q      [B][Nq][H][D] bf16, un-rotated; rotated here by R(pos_q)
 *   k_rot  [B][Nk][H][D] bf16, keys already rotated (lwm_blockattn_rope_apply
 *          with their own positions and the same rope_layout)
 *   v      [B][Nk][H][D] bf16
 *   seg_q  [B][Nq], pos_q [B][Nq], seg_k [B][Nk] int32; segment ids
 *          non-decreasing along the whole sequence
 *   rope_table  the table of lwm_blockattn_rope_table for (theta, max_pos),
 *          reused across the calls of a ring; NULL: built in the workspace
 *   out    [B][Nq][H][D] bf16, lse [B][H][Nq] fp32 (natural log), written
 *          (not accumulated): fold them into a running result with
 *          lwm_blockattn_merge.
 * D == 128, bf16 only. Async on stream; nothing launched on error. */
LWM_API int lwm_blockattn_fwd_block(const void* q, const void* k_rot,
                                    const void* v, const int32_t* seg_q,
                                    const int32_t* pos_q, const int32_t* seg_k,
                                    int q_off, int k_off, double theta,
                                    int max_pos, const float* rope_table,
                                    int B, int Nq, int Nk, int H, int D,
                                    int rope_layout, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream);

/* In place: (out, lse) <- the attention over the union of two disjoint key
 * sets, given (out, lse) over one and (out_part, lse_part) over the other:
 * with w = exp(lse - M), w' = exp(lse_part - M), M = max(lse, lse_part),
 * out = (w out + w' out_part) / (w + w'), lse = M + log(w + w').
 * Rows where both lse are -inf stay (0, -inf). Shapes as in
 * lwm_blockattn_fwd_block (N rows); D == 128, bf16 only. Async on stream. */
LWM_API int lwm_blockattn_merge(void* out, float* lse, const void* out_part,
                                const float* lse_part, int B, int N, int H,
                                int D, int dtype, void* stream);

/* Backward of the ring (same page, 3.1: the gradients of a key/value
 * block travel around the ring with it and come back to its owner).
 *
 * D_i = sum_d dout_i[d] out_i[d] as fp32 [B][H][N] (out, dout [B][N][H][D]
 * bf16): computed once per query chunk from its final out. */
LWM_API int lwm_blockattn_bwd_delta(const void* out, const void* dout, int B,
                                    int N, int H, int D, int dtype,
                                    float* delta, void* stream);

/* Bytes of workspace lwm_blockattn_bwd_block needs (key-side metadata). */
LWM_API size_t lwm_blockattn_bwd_block_workspace_size(int B, int Nq, int Nk,
                                                      int H, int D);

/* Partial backward of query rows [q_off, q_off+Nq) against the key/value
 * rows [k_off, k_off+Nk) of the same packed sequence (visibility as in
 * lwm_blockattn_fwd_block), given the FINAL lse of the queries (over all
 * keys) and their delta. Adds into fp32 accumulators in the rotated frame
 * and without the 1/sqrt(D) factor:
 *   dq_acc [B][Nq][H][D] += dS K~,   dk_acc [B][Nk][H][D] += dS^T Q~,
 *   dv_acc [B][Nk][H][D] += P^T dO,
 * with P = exp(Q~K~^T/sqrt(D) - lse) on visible pairs, dS = P (dO V^T - D).
 *   q_rot [B][Nq][H][D], k_rot [B][Nk][H][D]: bf16, already rotated
 *   v [B][Nk][H][D], dout [B][Nq][H][D]: bf16; lse, delta [B][H][Nq] fp32
 *   seg_q [B][Nq], seg_k [B][Nk] int32
 * The accumulators are the caller's, zeroed before the first call; turn
 * them into gradients with lwm_blockattn_grad_finish. dq_acc receives
 * atomic adds (order not fixed). D == 128. Async on stream. */
LWM_API int lwm_blockattn_bwd_block(const void* q_rot, const void* k_rot,
                                    const void* v, const void* dout,
                                    const float* lse, const float* delta,
                                    const int32_t* seg_q, const int32_t* seg_k,
                                    int q_off, int k_off, int B, int Nq,
                                    int Nk, int H, int D, float* dq_acc,
                                    float* dk_acc, float* dv_acc,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream);

/* grad (bf16 [B][N][H][D]) from an fp32 accumulator of the same shape:
 * with positions (int32 [B][N]) and a table from lwm_blockattn_rope_table,
 * grad = R(-pos) acc / sqrt(D) (dq, dk; pairs as rope_layout says, the
 * layout the accumulator was built in); with positions == NULL, grad = acc
 * (dv). Async on stream. */
LWM_API int lwm_blockattn_grad_finish(const float* acc,
                                      const int32_t* positions,
                                      const float* rope_table, int max_pos,
                                      int B, int N, int H, int D, int dtype,
                                      int rope_layout, void* grad,
                                      void* stream);

/* ---------------------------------------------------------------------
 * Blockwise feed-forward network: the Llama-2 SwiGLU MLP of the blockwise
 * transformer, run over the tokens in chunks so that only one chunk's
 * intermediate activations exist at a time ("LWM：突破 100 万 Token 的开源大
 * 模型", 配置参数: scan_mlp with scan_mlp_chunk_size 8192; the Llama-2-7B
 * backbone, "Inside Large World Model", Core Architecture).
 *
 * Bytes of workspace lwm_blockffn_fwd needs: one chunk's intermediate,
 * chunk x F bf16 (chunk clipped to T by the caller or not: the larger is
 * safe). */
LWM_API size_t lwm_blockffn_workspace_size(int chunk, int F);

/* y = (silu(x Wg^T) * (x Wu^T)) Wd^T over T tokens, `chunk` tokens at a
 * time.
 *   x      [T][Dm] bf16            y [T][Dm] bf16 (written)
 *   w_gate, w_up [F][Dm] bf16, w_down [Dm][F] bf16 (nn.Linear layout:
 *          row = output feature)
 * silu(h) = h / (1 + e^-h); products accumulate in fp32 on the tensor
 * cores; the intermediate is rounded to bf16 once. Dm and F multiples of
 * 64; only LWM_DTYPE_BF16. Async on stream; nothing launched on error. */
LWM_API int lwm_blockffn_fwd(const void* x, const void* w_gate,
                             const void* w_up, const void* w_down, int T,
                             int Dm, int F, int chunk, int dtype, void* y,
                             void* workspace, size_t workspace_bytes,
                             void* stream);

/* Bytes of workspace lwm_blockffn_bwd needs: one chunk's bf16 dact, dh,
 * dg and act, 4 x chunk x F x 2 bytes. */
LWM_API size_t lwm_blockffn_bwd_workspace_size(int chunk, int F);

/* Backward of lwm_blockffn_fwd, chunk by chunk with h and g recomputed:
 *   dact = dy Wd, dh = dact * g * silu'(h), dg = dact * silu(h),
 *   dx = dh Wg + dg Wu (bf16 [T][Dm], written),
 *   dw_gate = sum_chunks dh^T x, dw_up = dg^T x ([F][Dm] fp32),
 *   dw_down = dy^T act ([Dm][F] fp32), all three written (zeroed first).
 * dy [T][Dm] bf16. dact, dh, dg and act are rounded to bf16 once; the
 * products accumulate in fp32. Dm, F multiples of 64; bf16 only. Async on
 * stream; every argument is checked before the first launch, so a rejected
 * call writes nothing (T = 0 only zeroes the three weight gradients). */
LWM_API int lwm_blockffn_bwd(const void* x, const void* w_gate,
                             const void* w_up, const void* w_down,
                             const void* dy, int T, int Dm, int F, int chunk,
                             int dtype, void* dx, float* dw_gate,
                             float* dw_up, float* dw_down, void* workspace,
                             size_t workspace_bytes, void* stream);

/* General tile classifier, for any block sizes: a planning and reporting
 * tool (how many tiles a packing leaves EMPTY / PARTIAL / FULL). The
 * attention kernels themselves classify from the metadata that
 * lwm_blockattn_visibility exports. For each batch row b and query block
 * t (Tq = ceil(N/block_q) blocks), key blocks j (Tk = ceil(N/block_k)):
 *   kv_lo[b][t] = (start of the packed example holding row t*block_q)
 *                 / block_k,
 *   kv_hi[b][t] = (last valid row of block t) / block_k,
 *   tile_class[b][t][j] = EMPTY outside [kv_lo, kv_hi]; inside it FULL if
 *   key block j ends before query block t starts, both blocks lie inside
 *   [0, N) and the first key and last query share one segment id;
 *   PARTIAL otherwise.
 * With non-decreasing ids this equals "EMPTY: no allowed pair, FULL: all
 * pairs allowed (indices >= N never allowed), PARTIAL: some".
 * block_k must divide block_q; both in [16, 1024]. tile_class may be NULL
 * (then only kv_lo/kv_hi are written). Async on stream. */
LWM_API int lwm_blockattn_classify(const int32_t* segment_ids, int B, int N,
                           int block_q, int block_k, int32_t* kv_lo,
                           int32_t* kv_hi, uint8_t* tile_class,
                           void* stream);

/* The visibility metadata the attention kernels actually run on, exported
 * so that their segment/causal tile classification can be checked
 * bit-exactly (the mask: a query sees the keys of its own packed example
 * at or before it, "LWM：突破 100 万 Token 的开源大模型", 概述 (b); tiles:
 * the query/key chunks of 配置参数). Makes exactly the launches that
 * lwm_blockattn_fwd / _fwd_block (query view) and lwm_blockattn_bwd /
 * _bwd_block (key view) make before their attention kernels.
 * Queries are the global token indices [q_off, q_off + Nq) with ids seg_q
 * [B][Nq]; keys [k_off, k_off + Nk) with ids seg_k [B][Nk] (self-attention:
 * the same array, offsets 0, Nq == Nk). block_q == 128; block_k == 128,
 * or 64 for the query view alone (the forward's 64-key tiles; the
 * backward's key view is always in 128-key units).
 * Query view (all six pointers or none):
 *   row_lo, row_hi [B][Nq]: global indices of the first / last key the row
 *     sees (none: row_lo > row_hi);
 *   kv_lo, kv_hi [B][Tq]: the key blocks (counted from k_off) holding any
 *     key the query block sees (none: kv_lo > kv_hi); the kernel visits
 *     exactly these, every other tile is EMPTY;
 *   lo_max, hi_min [B][Tq]: max row_lo and min row_hi over the block's
 *     rows (INT_MAX / -INT_MAX when a row lies past Nq or sees nothing);
 *     key block j (first key k0 = k_off + block_k j) is FULL, and takes
 *     the mask-free path, iff lo_max <= k0 and hi_min >= k0 + block_k - 1;
 *     other visited tiles are PARTIAL.
 * Key view (all six or none), the same with queries and keys swapped:
 *   col_lo, col_hi [B][Nk]: first / last query that sees the key;
 *   q_lo, q_hi [B][Tk]: the query blocks the key block is visited with;
 *   klo_max, khi_min [B][Tk]: the FULL test for query block t (first query
 *     q0 = q_off + 128 t): klo_max <= q0 and khi_min >= q0 + 127.
 * Caller-owned device buffers; async on stream. Returns LWM_ERR_INVALID_ARG
 * for a partly given view or bad sizes, LWM_ERR_UNSUPPORTED for other
 * block sizes; nothing is launched on error. */
LWM_API int lwm_blockattn_visibility(const int32_t* seg_q,
                                     const int32_t* seg_k, int B, int Nq,
                                     int Nk, int q_off, int k_off,
                                     int block_q, int block_k,
                                     int32_t* row_lo, int32_t* row_hi,
                                     int32_t* kv_lo, int32_t* kv_hi,
                                     int32_t* lo_max, int32_t* hi_min,
                                     int32_t* col_lo, int32_t* col_hi,
                                     int32_t* q_lo, int32_t* q_hi,
                                     int32_t* klo_max, int32_t* khi_min,
                                     void* stream);

/* RoPE table the kernels use: table[p][k] = (cos a, sin a) as float32 with
 * a = p * theta^(-2k/D) evaluated in fp64, p in [0, max_pos),
 * k in [0, D/2). table holds max_pos * D floats. Async on stream. */
LWM_API int lwm_blockattn_rope_table(double theta, int D, int max_pos, float* table,
                             void* stream);

/* Synchronous precondition check: returns LWM_OK if segment_ids are
 * non-decreasing along every row and all positions lie in [0, max_pos),
 * LWM_ERR_PRECONDITION otherwise. If max_pos_out is non-NULL it receives
 * 1 + the largest position seen (a valid max_pos for these inputs).
 * Uses a few bytes of the library's own device memory; synchronises
 * `stream`. */
LWM_API int lwm_blockattn_check_inputs(const int32_t* segment_ids,
                               const int32_t* positions, int B, int N,
                               int max_pos, int* max_pos_out, void* stream);

/* Synchronises `stream`, then returns and clears the device status word
 * that the kernels set when a bounded wait gives up (LWM_ERR_TIMEOUT) or
 * LWM_OK. Also reports a sticky CUDA error as LWM_ERR_CUDA. */
LWM_API int lwm_blockattn_last_status(void* stream);

/* Static string naming a status code. */
LWM_API const char* lwm_status_string(int status);

/* LWM_BLOCKATTN_VERSION of the built library. */
LWM_API int lwm_blockattn_version(void);

/* ---------------------------------------------------------------------
 * Decode (inference against a long KV cache).
 *
 * lwm_blockattn_rope_apply: x_rot = R(pos) x for a bf16 [B][N][H][D] tensor
 * (D == 128, pairs as rope_layout says; x_rot keeps that layout), using a
 * table made by
 * lwm_blockattn_rope_table for positions [0, max_pos). Rotating keys once as
 * they enter a cache lets decode read them as they are. Async on stream.
 * Returns LWM_OK or an error status (nothing launched on error). */
LWM_API int lwm_blockattn_rope_apply(const void* x, const int32_t* positions,
                                     const float* rope_table, int max_pos,
                                     int B, int N, int H, int D, int dtype,
                                     int rope_layout, void* x_rot,
                                     void* stream);

/* Bytes of workspace lwm_blockattn_decode needs (per-chunk partial sums). */
LWM_API size_t lwm_blockattn_decode_workspace_size(int B, int H, int D,
                                                   int L);

/* One query token per (b, h) against a cache of L tokens.
 *   q        [B][H][D] bf16, un-rotated; rotated here by R(q_pos[b])
 *   k_rot    [B][L][H][D] bf16, keys already rotated (rope_apply, same
 *            rope_layout)
 *   v        [B][L][H][D] bf16
 *   kv_start, kv_len [B] int32: the query sees cached keys
 *            [kv_start[b], kv_len[b]) (its own packed example: the query is
 *            the example's last token); values outside [0, L] are clamped
 *   q_pos    [B] int32 RoPE position of the query, in [0, max_pos)
 *   rope_table from lwm_blockattn_rope_table (max_pos positions)
 *   out      [B][H][D] bf16;  lse [B][H] fp32 natural log (-inf if the
 *            range is empty, with out = 0)
 * Split over key chunks (partials in the workspace), then merged; reads
 * each visible key and value row once, in 128-key boxes through a TMA
 * shared-memory ring (k_rot and v must be 16-byte aligned, as every pointer
 * here). Only dtype LWM_DTYPE_BF16. Async on stream; a load that never
 * lands ends the kernel after a bounded wait and records LWM_ERR_TIMEOUT
 * for lwm_blockattn_last_status. */
LWM_API int lwm_blockattn_decode(const void* q, const void* k_rot,
                                 const void* v, const int32_t* kv_start,
                                 const int32_t* kv_len, const int32_t* q_pos,
                                 const float* rope_table, int max_pos, int B,
                                 int L, int H, int D, int dtype,
                                 int rope_layout, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Self-test of the failure path: launches one small CTA that waits on an
 * mbarrier nobody arrives on, with the same bounded wait the attention
 * kernels use and a limit of limit_ns nanoseconds (clamped to [1 ms, 2 s]).
 * When the limit passes, the kernel records LWM_ERR_TIMEOUT in the device
 * status word and returns normally (no trap, the context stays usable);
 * lwm_blockattn_last_status then reports and clears it. Test use only. */
LWM_API int lwm_blockattn_selftest_wait_timeout(uint64_t limit_ns,
                                                void* stream);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all streams), counted on the host at each successful launch. */
LWM_API uint64_t lwm_blockattn_kernel_launches(void);

/* Size of the library-owned scratch array used by
 * lwm_blockattn_fwd_noalloc (64 MiB on every device that loads the
 * library, held until the process exits). */
#define LWM_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* The forward pass for callers that cannot allocate device memory while
 * they run (e.g. a latency-critical serving loop where cudaMalloc could
 * synchronise the device, or a plain C host with no device allocator of
 * its own). The pages have no counterpart to this entry point: it exists
 * only for such callers.
 * Arguments and results are those of lwm_blockattn_fwd without the
 * workspace: the scratch lives in a fixed device array inside the library
 * (LWM_NOALLOC_SCRATCH_BYTES). Every argument is first checked as
 * lwm_blockattn_fwd checks it (same status codes); a valid, supported call
 * whose lwm_blockattn_fwd_workspace_size exceeds the array returns
 * LWM_ERR_WORKSPACE. Nothing is launched on error. The call never
 * allocates or frees memory.
 * The first call on each device looks up that device's scratch address
 * (cudaGetSymbolAddress with the device current); make it before any stream
 * capture begins. All calls share the one array: calls that overlap on the
 * GPU (other streams or threads without ordering) race on it, so serialise
 * them. */
LWM_API int lwm_blockattn_fwd_noalloc(const void* q, const void* k,
                                      const void* v,
                                      const int32_t* segment_ids,
                                      const int32_t* positions, double theta,
                                      int block_q, int block_k, int max_pos,
                                      int B, int N, int H, int D, int dtype,
                                      int qk_precision, int rope_layout,
                                      void* out, float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LWM_BLOCKATTN_H */
