// Launchers of the auxiliary kernels (see aux_kernels.cu).
#pragma once

#include "common.cuh"

namespace lwm {

constexpr int kSortMax = 16384;  // units one CTA sorts in shared memory

cudaError_t launch_rope_table(double theta, int D, int max_pos, float* table,
                              cudaStream_t st);
cudaError_t launch_block_meta(const int32_t* seg, int B, int N, int bq, int bk,
                              int32_t* kv_lo, int32_t* kv_hi, cudaStream_t st);
// hi = R(pos) x in bf16, lo = residual (skipped when lo == nullptr); pairs
// (2k, 2k+1), or (k, k+64) when `half` (rotate-half layout, kept on output).
cudaError_t launch_rope_apply(const void* x, const int32_t* pos,
                              const float* table, int B, int N, int H,
                              bool half, void* hi, void* lo, cudaStream_t st);
// Per-row visible key ranges of queries [q_off, q_off+Nq) against keys
// [k_off, k_off+Nk) (global indices), and per query block the key-block
// range plus the shared row range used for the all-visible test.
// kv_lo / kv_hi count key blocks of bk keys (128 or 64); query blocks are
// 128 rows.
cudaError_t launch_cross_meta(const int32_t* seg_q, const int32_t* seg_k,
                              int B, int Nq, int Nk, int q_off, int k_off,
                              int bk, int32_t* row_lo, int32_t* row_hi,
                              int32_t* kv_lo, int32_t* kv_hi,
                              int32_t* lo_max, int32_t* hi_min,
                              cudaStream_t st);
// Key-side metadata of the same pair of ranges for the key-major backward:
// per key the queries that see it (global indices), per key block the query
// block range and the shared query range of the all-visible test.
cudaError_t launch_cross_meta_keys(const int32_t* seg_q, const int32_t* seg_k,
                                   int B, int Nq, int Nk, int q_off,
                                   int k_off, int32_t* col_lo,
                                   int32_t* col_hi, int32_t* q_lo,
                                   int32_t* q_hi, int32_t* klo_max,
                                   int32_t* khi_min, cudaStream_t st);
// Combine a partial (out_p, lse_p) over another key set into (out, lse).
cudaError_t launch_merge(void* out, float* lse, const void* out_p,
                         const float* lse_p, int B, int N, int H,
                         cudaStream_t st);
cudaError_t launch_fill(float* x, float v, int64_t n, cudaStream_t st);
// rs[i]: first row of row i's packed example; re[i] (if re != nullptr):
// its last row.
cudaError_t launch_row_start(const int32_t* seg, int B, int N, int32_t* rs,
                             int32_t* re, cudaStream_t st);
cudaError_t launch_tile_class(const int32_t* seg, int B, int N, int bq, int bk,
                              const int32_t* kv_lo, const int32_t* kv_hi,
                              uint8_t* cls, cudaStream_t st);
cudaError_t launch_kv_meta(int B, int Tq, int Tk, const int32_t* kv_lo,
                           const int32_t* kv_hi, int32_t* q_lo, int32_t* q_hi,
                           cudaStream_t st);
// Orders the units (b, u), u covering `group` consecutive blocks, by the
// size of the union of their [lo, hi] ranges, longest first, and zeroes
// the work counter the following attention launch hands units out with.
// anchor 1 (2): units are first grouped by the start (end) of that union,
// i.e. by packed example, in ascending order; 0: longest first only.
cudaError_t launch_lpt_order(int B, int T, int group, const int32_t* lo,
                             const int32_t* hi, int anchor, int32_t* order,
                             int32_t* counter, cudaStream_t st);
cudaError_t launch_check_inputs(const int32_t* seg, const int32_t* pos, int B,
                                int N, int max_pos, int* res, cudaStream_t st);
template <typename T>
cudaError_t launch_bwd_delta(const T* out, const T* dout, int B, int N, int H,
                             float* delta, cudaStream_t st);
// dq = R(-pos) acc * scale in T (pairs as in launch_rope_apply);
// pos == nullptr: dq = acc * scale.
template <typename T>
cudaError_t launch_dq_convert(const float* acc, const int32_t* pos,
                              const float* table, int B, int N, int H,
                              float scale, bool half, T* dq, cudaStream_t st);

// CUDA-core kernels (fp32 arithmetic), any I/O type.
// `half`: q and k in the rotate-half layout (dk written, and dq_acc
// accumulated, in that layout too).
template <typename T>
cudaError_t launch_fwd_simt(const T* q, const T* k, const T* v,
                            const int32_t* seg, const int32_t* pos,
                            const float* table, const int32_t* kv_lo, int B,
                            int N, int H, bool half, T* out, float* lse,
                            cudaStream_t st);
template <typename T>
cudaError_t launch_bwd_simt(const T* q, const T* k, const T* v, const T* dout,
                            const float* lse, const float* delta,
                            const int32_t* seg, const int32_t* pos,
                            const float* table, int B, int N, int H, bool half,
                            float* dq_acc, T* dk, T* dv, cudaStream_t st);

}  // namespace lwm
