// Tensor-core (tcgen05) kernels of the blockwise attention path.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace lwm {

// A forward CTA owns this many consecutive 128-row query blocks of one
// (batch row, head); a backward CTA this many 128-key blocks.
constexpr int kFwdBlocksPerUnit = 2;
constexpr int kBwdBlocksPerUnit = 1;

// Forward of query rows [q_off, q_off + Nq) (global token indices) against
// rotated keys / values [k_off, k_off + Nk) of the same packed row; self-
// attention is q_off = k_off = 0, Nq = Nk. Visibility comes as per-row key
// ranges (row_lo/row_hi) and per query block key-block ranges (kv_lo/kv_hi)
// plus the all-visible bounds (lo_max/hi_min), all from launch_cross_meta.
struct FwdArgs {
  const void* q;           // [B][Nq][H][D], un-rotated
  const void* k_rot;       // [B][Nk][H][D], R(pos) k
  const void* k_rot_lo;    // bf16 residual of k_rot (split-QK mode)
  const void* v;           // [B][Nk][H][D]
  void* out;               // [B][Nq][H][D]
  float* lse;              // [B][H][Nq]
  const int32_t* pos_q;    // [B][Nq]
  const float* table;
  const int32_t* kv_lo;
  const int32_t* kv_hi;
  const int32_t* row_lo;
  const int32_t* row_hi;
  const int32_t* lo_max;
  const int32_t* hi_min;
  const int32_t* order;
  int32_t* counter;        // zeroed work counter (units handed out in order)
  int B, Nq, Nk, H, k_off;
  int block_k;             // keys per key block: 128 or 64 (kv_lo / kv_hi
                           // count key blocks of this height)
  bool qk_x3;
  bool rope_half;          // q (and k_rot) in the rotate-half layout
  int* status;
};

// Backward of query rows [q_off, q_off + Nq) against keys / values
// [k_off, k_off + Nk) (key-major: one key block per work unit). Visibility
// comes per key as the range of queries that see it (col_lo/col_hi, global
// indices) and per key block as the query-block range (q_lo/q_hi) plus the
// all-visible bounds (klo_max/khi_min), all from launch_cross_meta_keys.
// dQ~ (unscaled, rotated frame) is reduce-added into dq_acc. dK, dV either
// go out as bf16 (dk = R(-pos_k) dK~ / sqrt(D), dv; dk_acc == nullptr) or
// are added, unscaled and in the rotated frame, into fp32 accumulators
// dk_acc / dv_acc that the caller carries across calls.
struct BwdArgs {
  const void* q_rot;       // [B][Nq][H][D], R(pos) q
  const void* k_rot;       // [B][Nk][H][D], R(pos) k
  const void* v;           // [B][Nk][H][D]
  const void* dout;        // [B][Nq][H][D]
  const float* lse;        // [B][H][Nq]
  const float* delta;      // [B][H][Nq]
  const int32_t* pos_k;    // [B][Nk] (bf16 output mode only)
  const float* table;      // (bf16 output mode only)
  const int32_t* q_lo;
  const int32_t* q_hi;
  const int32_t* col_lo;
  const int32_t* col_hi;
  const int32_t* klo_max;
  const int32_t* khi_min;
  const int32_t* order;
  int32_t* counter;
  float* dq_acc;           // [B][Nq][H][D] fp32
  void* dk;                // [B][Nk][H][D] bf16, or
  void* dv;
  float* dk_acc;           // [B][Nk][H][D] fp32 accumulators
  float* dv_acc;
  int B, Nq, Nk, H, q_off;
  bool rope_half;          // rotate-half layout (dk's R(-pos) pairs)
  int* status;
};

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t st);
// 4-D TMA map over a bf16 [B][N][H][128] tensor, box 64 x 1 x rows x 1,
// 128-byte swizzle. False if the driver's encoder is unavailable/refuses.
bool make_bnhd_map(CUtensorMap* m, const void* base, int B, int N, int H,
                   int rows = kBlock);
// 4-D TMA map over an fp32 [B][N][H][128] tensor, box 32 x 1 x 32 x 1,
// 128-byte swizzle (used for the dQ reduce-add).
bool make_bnhd_f32_map(CUtensorMap* m, const void* base, int B, int N,
                       int H);
// Row-major bf16 [rows][cols] matrix as a 2-D map, box 64 x box_rows,
// 128-byte swizzle (cols * 2 must be a multiple of 16 bytes).
bool make_2d_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                 int box_rows);
bool make_2d_map_strided(CUtensorMap* m, const void* base, int64_t rows,
                         int64_t cols, int64_t ld, int box_rows);
int sm_count();
cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t st);

}  // namespace lwm
