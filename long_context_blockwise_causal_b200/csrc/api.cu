// C ABI of liblwm_blockattn.so (declared in include/lwm_blockattn.h):
// host-side validation, workspace carving and the launch sequence of the
// forward and backward passes.
#include <atomic>
#include <cmath>
#include <cstring>

#include "api_checks.cuh"
#include "aux_kernels.cuh"
#include "decode.cuh"
#include "mlp.cuh"
#include "tc_kernels.cuh"

namespace lwm {

// Device status word set by bounded waits that give up; read and cleared
// by lwm_blockattn_last_status.
__device__ int g_status_word;
// Result words of lwm_blockattn_check_inputs: [0] violation bits, [1] max
// position seen.
__device__ int g_check_words[2];

static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// One CTA waits on a barrier that is never arrived on; the bounded wait
// gives up after limit_ns and records LWM_ERR_TIMEOUT in *status.
__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_word;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    abort_word = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(bar, 0, &abort_word, status, limit_ns);
}

namespace {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Carve {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align_up(count * sizeof(T));
    return p;
  }
};

enum class Pass { kFwd, kFwdBlock, kBwd, kBwdBlock };

// Workspace regions (a pass carves only what it uses).
struct Workspace {
  float* table;          // [max_pos][D/2] float2
  // forward: per query block the key-block range and all-visible bounds,
  // per query row its visible keys (launch_cross_meta)
  int32_t* kv_lo;        // [B][Tq]
  int32_t* kv_hi;
  int32_t* lo_max;
  int32_t* hi_min;
  int32_t* row_lo;       // [B][Nq]
  int32_t* row_hi;
  int32_t* order_fwd;    // [B*Uq] units of two query blocks, longest first
  // backward: the key-side view (launch_cross_meta_keys)
  int32_t* q_lo;         // [B][Tk]
  int32_t* q_hi;
  int32_t* klo_max;
  int32_t* khi_min;
  int32_t* col_lo;       // [B][Nk]
  int32_t* col_hi;
  int32_t* order_bwd;    // [B*Tk]
  int32_t* counter;      // work counter of the attention kernel
  float* delta;          // [B][H][N]
  float* dq_acc;         // [B][N][H][D]
  // bf16 path: rotated keys (and queries for the backward), [B][N][H][D]
  void* k_rot;
  void* k_rot_lo;        // split-QK mode only
  void* q_rot;           // backward only
  size_t bytes;
};

Workspace carve(void* base, int B, int Nq, int Nk, int H, int D, int max_pos,
                Pass pass, int dtype, int qkp) {
  Carve c{static_cast<char*>(base)};
  Workspace w{};
  const bool fwd = pass == Pass::kFwd || pass == Pass::kFwdBlock;
  const bool tc = dtype == LWM_DTYPE_BF16 && qkp == LWM_QK_BF16;
  const int Tq = (Nq + kBlock - 1) / kBlock;
  const int Tk = (Nk + kBlock - 1) / kBlock;
  const int Uq = (Tq + kFwdBlocksPerUnit - 1) / kFwdBlocksPerUnit;
  if (pass != Pass::kBwdBlock) w.table = c.take<float>(size_t(max_pos) * D);
  if (fwd) {
    w.kv_lo = c.take<int32_t>(size_t(B) * Tq);
    w.kv_hi = c.take<int32_t>(size_t(B) * Tq);
    w.lo_max = c.take<int32_t>(size_t(B) * Tq);
    w.hi_min = c.take<int32_t>(size_t(B) * Tq);
    w.row_lo = c.take<int32_t>(size_t(B) * Nq);
    w.row_hi = c.take<int32_t>(size_t(B) * Nq);
    w.order_fwd = c.take<int32_t>(size_t(B) * Uq);
  } else {
    w.q_lo = c.take<int32_t>(size_t(B) * Tk);
    w.q_hi = c.take<int32_t>(size_t(B) * Tk);
    w.klo_max = c.take<int32_t>(size_t(B) * Tk);
    w.khi_min = c.take<int32_t>(size_t(B) * Tk);
    w.col_lo = c.take<int32_t>(size_t(B) * Nk);
    w.col_hi = c.take<int32_t>(size_t(B) * Nk);
    w.order_bwd = c.take<int32_t>(size_t(B) * Tk);
  }
  w.counter = c.take<int32_t>(64);
  if (pass == Pass::kBwd) {
    w.delta = c.take<float>(size_t(B) * H * Nq);
    w.dq_acc = c.take<float>(size_t(B) * Nq * H * D);
  }
  if (dtype == LWM_DTYPE_BF16 && pass == Pass::kFwd) {
    w.k_rot = c.take<uint16_t>(size_t(B) * Nk * H * D);
    if (qkp == LWM_QK_BF16X3) w.k_rot_lo = c.take<uint16_t>(size_t(B) * Nk * H * D);
  }
  if (tc && pass == Pass::kBwd) {
    w.k_rot = c.take<uint16_t>(size_t(B) * Nk * H * D);
    w.q_rot = c.take<uint16_t>(size_t(B) * Nq * H * D);
  }
  w.bytes = c.off;
  return w;
}

bool sizes_ok(int B, int N, int H, int D, int block_q, int block_k,
              int max_pos) {
  return B >= 0 && N >= 0 && H >= 0 && D > 0 && block_q > 0 && block_k > 0 &&
         max_pos >= 0 && (int64_t(B) * N) < (int64_t(1) << 31);
}

// Query blocks of 128 rows; key blocks of 128 or 64 keys (the forward
// sweeps key tiles of that height; the key-major backward visits 128-key
// units either way, which gives the same gradients).
int shape_status(int D, int block_q, int block_k) {
  if (D != kHeadDim || block_q != kBlock ||
      (block_k != kBlock && block_k != kBlock / 2))
    return LWM_ERR_UNSUPPORTED;
  return LWM_OK;
}

inline bool layout_ok(int rope_layout) {
  return rope_layout == LWM_ROPE_INTERLEAVED || rope_layout == LWM_ROPE_HALF;
}

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LWM_OK : LWM_ERR_CUDA; }

#define LWM_TRY(expr)                                  \
  do {                                                 \
    cudaError_t e_ = (expr);                           \
    if (e_ != cudaSuccess) return LWM_ERR_CUDA;        \
  } while (0)

int* status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

// Shared tail of lwm_blockattn_bwd and lwm_blockattn_bwd_block: key-side
// metadata of queries [q_off, q_off+Nq) against keys [k_off, k_off+Nk), the
// longest-first order of the key blocks and the attention kernel.
int run_backward(BwdArgs a, const int32_t* seg_q, const int32_t* seg_k,
                 int k_off, const Workspace& w, cudaStream_t st) {
  LWM_TRY(launch_cross_meta_keys(seg_q, seg_k, a.B, a.Nq, a.Nk, a.q_off,
                                 k_off, w.col_lo, w.col_hi, w.q_lo, w.q_hi,
                                 w.klo_max, w.khi_min, st));
  LWM_TRY(launch_lpt_order(a.B, (a.Nk + kBlock - 1) / kBlock,
                           kBwdBlocksPerUnit, w.q_lo, w.q_hi, 2,
                           w.order_bwd, w.counter, st));
  a.q_lo = w.q_lo; a.q_hi = w.q_hi; a.col_lo = w.col_lo; a.col_hi = w.col_hi;
  a.klo_max = w.klo_max; a.khi_min = w.khi_min;
  a.order = w.order_bwd; a.counter = w.counter;
  a.status = status_word();
  if (!a.status) return LWM_ERR_CUDA;
  return cuda_status(launch_bwd_tc(a, st));
}

// Shared tail of lwm_blockattn_fwd and lwm_blockattn_fwd_block: metadata of
// queries [q_off, q_off+Nq) against keys [k_off, k_off+Nk), the
// longest-first order and the attention kernel (table already built).
int run_forward(const void* q, const void* k_rot, const void* k_rot_lo,
                const void* v, const int32_t* seg_q, const int32_t* pos_q,
                const int32_t* seg_k, int q_off, int k_off, int B, int Nq,
                int Nk, int H, int block_k, bool x3, bool half, void* out,
                float* lse, const Workspace& w, cudaStream_t st) {
  LWM_TRY(launch_cross_meta(seg_q, seg_k, B, Nq, Nk, q_off, k_off, block_k,
                            w.row_lo, w.row_hi, w.kv_lo, w.kv_hi, w.lo_max,
                            w.hi_min, st));
  LWM_TRY(launch_lpt_order(B, (Nq + kBlock - 1) / kBlock, kFwdBlocksPerUnit,
                           w.kv_lo, w.kv_hi, 1, w.order_fwd,
                           w.counter, st));
  FwdArgs a{};
  a.q = q; a.k_rot = k_rot; a.k_rot_lo = k_rot_lo; a.v = v;
  a.out = out; a.lse = lse; a.pos_q = pos_q; a.table = w.table;
  a.kv_lo = w.kv_lo; a.kv_hi = w.kv_hi; a.row_lo = w.row_lo;
  a.row_hi = w.row_hi; a.lo_max = w.lo_max; a.hi_min = w.hi_min;
  a.order = w.order_fwd; a.counter = w.counter;
  a.B = B; a.Nq = Nq; a.Nk = Nk; a.H = H; a.k_off = k_off;
  a.block_k = block_k;
  a.qk_x3 = x3;
  a.rope_half = half;
  a.status = status_word();
  if (!a.status) return LWM_ERR_CUDA;
  return cuda_status(launch_fwd_tc(a, st));
}

}  // namespace

int check_fwd_args(const void* q, const void* k, const void* v,
                   const int32_t* segment_ids, const int32_t* positions,
                   double theta, int block_q, int block_k, int max_pos, int B,
                   int N, int H, int D, int dtype, int qk_precision,
                   int rope_layout, const void* out, const float* lse) {
  if (!sizes_ok(B, N, H, D, block_q, block_k, max_pos))
    return LWM_ERR_INVALID_ARG;
  if (!layout_ok(rope_layout)) return LWM_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !std::isfinite(theta)) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32)
    return LWM_ERR_INVALID_ARG;
  if (qk_precision != LWM_QK_BF16 && qk_precision != LWM_QK_BF16X3)
    return LWM_ERR_INVALID_ARG;
  const int s = shape_status(D, block_q, block_k);
  if (s != LWM_OK) return s;
  if (int64_t(B) * N * H == 0) return kFwdNothingToDo;
  if (max_pos < 1) return LWM_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, segment_ids, positions, out, lse};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  return LWM_OK;
}

}  // namespace lwm

using namespace lwm;

extern "C" {

const char* lwm_status_string(int status) {
  switch (status) {
    case LWM_OK: return "ok";
    case LWM_ERR_INVALID_ARG: return "invalid argument";
    case LWM_ERR_UNSUPPORTED: return "unsupported configuration";
    case LWM_ERR_WORKSPACE: return "workspace missing or too small";
    case LWM_ERR_CUDA: return "CUDA error";
    case LWM_ERR_TIMEOUT: return "device-side wait timed out";
    case LWM_ERR_PRECONDITION: return "input precondition violated";
    default: return "unknown status";
  }
}

int lwm_blockattn_version(void) { return LWM_BLOCKATTN_VERSION; }

int lwm_blockattn_rope_apply(const void* x, const int32_t* positions,
                             const float* rope_table, int max_pos, int B,
                             int N, int H, int D, int dtype, int rope_layout,
                             void* x_rot, void* stream) {
  if (B < 0 || N < 0 || H < 0 || max_pos < 0 ||
      (int64_t(B) * N) >= (int64_t(1) << 31))
    return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim) return LWM_ERR_UNSUPPORTED;
  if (dtype != LWM_DTYPE_BF16) return LWM_ERR_UNSUPPORTED;
  if (!layout_ok(rope_layout)) return LWM_ERR_INVALID_ARG;
  if (int64_t(B) * N * H == 0) return LWM_OK;
  const void* ptrs[] = {x, positions, rope_table, x_rot};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  if (max_pos < 1) return LWM_ERR_INVALID_ARG;
  return cuda_status(launch_rope_apply(x, positions, rope_table, B, N, H,
                                       rope_layout == LWM_ROPE_HALF, x_rot,
                                       nullptr,
                                       static_cast<cudaStream_t>(stream)));
}

size_t lwm_blockattn_decode_workspace_size(int B, int H, int D, int L) {
  if (B < 0 || H < 0 || D != kHeadDim || L < 0) return 0;
  const size_t slots = size_t(B) * H * decode_splits(L);
  return align_up(slots * sizeof(float)) * 2 +
         align_up(slots * kHeadDim * sizeof(float));
}

int lwm_blockattn_decode(const void* q, const void* k_rot, const void* v,
                         const int32_t* kv_start, const int32_t* kv_len,
                         const int32_t* q_pos, const float* rope_table,
                         int max_pos, int B, int L, int H, int D, int dtype,
                         int rope_layout, void* out, float* lse,
                         void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (B < 0 || L < 0 || H < 0 || max_pos < 0 ||
      (int64_t(B) * L) >= (int64_t(1) << 31))
    return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim || dtype != LWM_DTYPE_BF16) return LWM_ERR_UNSUPPORTED;
  if (!layout_ok(rope_layout)) return LWM_ERR_INVALID_ARG;
  if (int64_t(B) * H == 0) return LWM_OK;
  const void* ptrs[] = {q, k_rot, v, kv_start, kv_len, q_pos, rope_table,
                        out, lse, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  if (max_pos < 1) return LWM_ERR_INVALID_ARG;
  const size_t need = lwm_blockattn_decode_workspace_size(B, H, D, L);
  if (workspace_bytes < need) return LWM_ERR_WORKSPACE;
  const size_t slots = size_t(B) * H * decode_splits(L);
  char* ws = static_cast<char*>(workspace);
  float* part_m = reinterpret_cast<float*>(ws);
  float* part_l = reinterpret_cast<float*>(ws + align_up(slots * sizeof(float)));
  float* part_acc =
      reinterpret_cast<float*>(ws + 2 * align_up(slots * sizeof(float)));
  int* st = status_word();
  if (!st) return LWM_ERR_CUDA;
  return cuda_status(launch_decode(q, k_rot, v, kv_start, kv_len, q_pos,
                                   rope_table, max_pos, B, L, H,
                                   rope_layout == LWM_ROPE_HALF, out, lse,
                                   part_m, part_l, part_acc, st,
                                   static_cast<cudaStream_t>(stream)));
}

int lwm_blockattn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000000ull) limit_ns = 1000000ull;
  if (limit_ns > 2000000000ull) limit_ns = 2000000000ull;
  int* st = status_word();
  if (!st) return LWM_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      st, limit_ns);
  note_launch();
  return cuda_status(cudaGetLastError());
}

uint64_t lwm_blockattn_kernel_launches(void) {
  return g_launches.load(std::memory_order_relaxed);
}

size_t lwm_blockattn_fwd_workspace_size(int B, int N, int H, int D,
                                        int block_q, int block_k,
                                        int max_pos, int dtype,
                                        int qk_precision) {
  if (!sizes_ok(B, N, H, D, block_q, block_k, max_pos)) return 0;
  return carve(nullptr, B, N, N, H, D, max_pos, Pass::kFwd, dtype,
               qk_precision)
      .bytes;
}

size_t lwm_blockattn_bwd_workspace_size(int B, int N, int H, int D,
                                        int block_q, int block_k,
                                        int max_pos, int dtype,
                                        int qk_precision) {
  if (!sizes_ok(B, N, H, D, block_q, block_k, max_pos)) return 0;
  return carve(nullptr, B, N, N, H, D, max_pos, Pass::kBwd, dtype,
               qk_precision)
      .bytes;
}

int lwm_blockattn_fwd(const void* q, const void* k, const void* v,
                      const int32_t* segment_ids, const int32_t* positions,
                      double theta, int block_q, int block_k, int max_pos,
                      int B, int N, int H, int D, int dtype, int qk_precision,
                      int rope_layout, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream) {
  const int c = check_fwd_args(q, k, v, segment_ids, positions, theta,
                               block_q, block_k, max_pos, B, N, H, D, dtype,
                               qk_precision, rope_layout, out, lse);
  if (c == kFwdNothingToDo) return LWM_OK;
  if (c != LWM_OK) return c;
  if (!workspace || !aligned16(workspace)) return LWM_ERR_INVALID_ARG;
  const bool half = rope_layout == LWM_ROPE_HALF;
  Workspace w = carve(workspace, B, N, N, H, D, max_pos, Pass::kFwd, dtype,
                      qk_precision);
  if (workspace_bytes < w.bytes) return LWM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LWM_TRY(launch_rope_table(theta, D, max_pos, w.table, st));
  if (dtype == LWM_DTYPE_FP32) {
    LWM_TRY(launch_block_meta(segment_ids, B, N, kBlock, kBlock, w.kv_lo,
                              w.kv_hi, st));
    return cuda_status(launch_fwd_simt<float>(
        static_cast<const float*>(q), static_cast<const float*>(k),
        static_cast<const float*>(v), segment_ids, positions, w.table,
        w.kv_lo, B, N, H, half, static_cast<float*>(out), lse, st));
  }
  // keys are reused by every query block that sees them: rotate them once
  LWM_TRY(launch_rope_apply(k, positions, w.table, B, N, H, half, w.k_rot,
                            w.k_rot_lo, st));
  return run_forward(q, w.k_rot, w.k_rot_lo, v, segment_ids, positions,
                     segment_ids, 0, 0, B, N, N, H, block_k,
                     qk_precision == LWM_QK_BF16X3, half, out, lse, w, st);
}

size_t lwm_blockattn_fwd_block_workspace_size(int B, int Nq, int Nk, int H,
                                              int D, int max_pos) {
  if (!sizes_ok(B, Nq, H, D, kBlock, kBlock, max_pos) || Nk < 0) return 0;
  return carve(nullptr, B, Nq, Nk, H, D, max_pos, Pass::kFwdBlock,
               LWM_DTYPE_BF16, LWM_QK_BF16)
      .bytes;
}

int lwm_blockattn_fwd_block(const void* q, const void* k_rot, const void* v,
                            const int32_t* seg_q, const int32_t* pos_q,
                            const int32_t* seg_k, int q_off, int k_off,
                            double theta, int max_pos,
                            const float* rope_table, int B, int Nq, int Nk,
                            int H, int D, int rope_layout, void* out,
                            float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (!sizes_ok(B, Nq, H, D, kBlock, kBlock, max_pos) || Nk < 0 ||
      q_off < 0 || k_off < 0 || (int64_t(B) * Nk) >= (int64_t(1) << 31))
    return LWM_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !std::isfinite(theta)) return LWM_ERR_INVALID_ARG;
  if (!layout_ok(rope_layout)) return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim) return LWM_ERR_UNSUPPORTED;
  if (int64_t(B) * Nq * H == 0) return LWM_OK;
  if (max_pos < 1) return LWM_ERR_INVALID_ARG;
  const void* ptrs[] = {q, pos_q, seg_q, out, lse, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  if (Nk > 0) {
    const void* kp[] = {k_rot, v, seg_k};
    for (const void* p : kp)
      if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  }
  Workspace w = carve(workspace, B, Nq, Nk, H, D, max_pos, Pass::kFwdBlock,
                      LWM_DTYPE_BF16, LWM_QK_BF16);
  if (workspace_bytes < w.bytes) return LWM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (Nk == 0) {  // no key: every row sees nothing
    LWM_TRY(cudaMemsetAsync(out, 0, size_t(B) * Nq * H * D * 2, st));
    LWM_TRY(launch_fill(lse, -INFINITY, size_t(B) * H * Nq, st));
    return LWM_OK;
  }
  if (rope_table) {
    if (!aligned16(rope_table)) return LWM_ERR_INVALID_ARG;
    w.table = const_cast<float*>(rope_table);
  } else {
    LWM_TRY(launch_rope_table(theta, D, max_pos, w.table, st));
  }
  return run_forward(q, k_rot, nullptr, v, seg_q, pos_q, seg_k, q_off, k_off,
                     B, Nq, Nk, H, kBlock, false, rope_layout == LWM_ROPE_HALF,
                     out, lse, w, st);
}

int lwm_blockattn_merge(void* out, float* lse, const void* out_part,
                        const float* lse_part, int B, int N, int H, int D,
                        int dtype, void* stream) {
  if (B < 0 || N < 0 || H < 0) return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim || dtype != LWM_DTYPE_BF16) return LWM_ERR_UNSUPPORTED;
  if (int64_t(B) * N * H == 0) return LWM_OK;
  const void* ptrs[] = {out, lse, out_part, lse_part};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  return cuda_status(launch_merge(out, lse, out_part, lse_part, B, N, H,
                                  static_cast<cudaStream_t>(stream)));
}

int lwm_blockattn_bwd(const void* q, const void* k, const void* v,
                      const void* out, const void* dout, const float* lse,
                      const int32_t* segment_ids, const int32_t* positions,
                      double theta, int block_q, int block_k, int max_pos,
                      int B, int N, int H, int D, int dtype, int qk_precision,
                      int rope_layout, void* dq, void* dk, void* dv,
                      void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (!sizes_ok(B, N, H, D, block_q, block_k, max_pos))
    return LWM_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !std::isfinite(theta)) return LWM_ERR_INVALID_ARG;
  if (!layout_ok(rope_layout)) return LWM_ERR_INVALID_ARG;
  const bool half = rope_layout == LWM_ROPE_HALF;
  if (dtype != LWM_DTYPE_BF16 && dtype != LWM_DTYPE_FP32)
    return LWM_ERR_INVALID_ARG;
  if (qk_precision != LWM_QK_BF16 && qk_precision != LWM_QK_BF16X3)
    return LWM_ERR_INVALID_ARG;
  int s = shape_status(D, block_q, block_k);
  if (s != LWM_OK) return s;
  if (int64_t(B) * N * H == 0) return LWM_OK;
  if (max_pos < 1) return LWM_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, out, dout, lse, segment_ids, positions,
                        dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  Workspace w = carve(workspace, B, N, N, H, D, max_pos, Pass::kBwd, dtype,
                      qk_precision);
  if (workspace_bytes < w.bytes) return LWM_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LWM_TRY(launch_rope_table(theta, D, max_pos, w.table, st));
  const float scale = 1.f / std::sqrt(float(D));
  LWM_TRY(cudaMemsetAsync(w.dq_acc, 0, sizeof(float) * size_t(B) * N * H * D,
                          st));
  if (dtype == LWM_DTYPE_FP32) {
    using T = float;
    LWM_TRY(launch_bwd_delta<T>(static_cast<const T*>(out),
                                static_cast<const T*>(dout), B, N, H, w.delta,
                                st));
    LWM_TRY(launch_bwd_simt<T>(
        static_cast<const T*>(q), static_cast<const T*>(k),
        static_cast<const T*>(v), static_cast<const T*>(dout), lse, w.delta,
        segment_ids, positions, w.table, B, N, H, half, w.dq_acc,
        static_cast<T*>(dk), static_cast<T*>(dv), st));
    return cuda_status(launch_dq_convert<T>(w.dq_acc, positions, w.table, B,
                                            N, H, scale, half,
                                            static_cast<T*>(dq), st));
  }
  using T = __nv_bfloat16;
  LWM_TRY(launch_bwd_delta<T>(static_cast<const T*>(out),
                              static_cast<const T*>(dout), B, N, H, w.delta,
                              st));
  if (qk_precision == LWM_QK_BF16X3) {
    // fp32 CUDA-core backward: at least the precision of the split product
    LWM_TRY(launch_bwd_simt<T>(
        static_cast<const T*>(q), static_cast<const T*>(k),
        static_cast<const T*>(v), static_cast<const T*>(dout), lse, w.delta,
        segment_ids, positions, w.table, B, N, H, half, w.dq_acc,
        static_cast<T*>(dk), static_cast<T*>(dv), st));
  } else {
    // queries and keys are both re-read inside the key-major sweep: rotate
    // them once
    LWM_TRY(launch_rope_apply(q, positions, w.table, B, N, H, half, w.q_rot,
                              nullptr, st));
    LWM_TRY(launch_rope_apply(k, positions, w.table, B, N, H, half, w.k_rot,
                              nullptr, st));
    BwdArgs a{};
    a.q_rot = w.q_rot; a.k_rot = w.k_rot; a.v = v; a.dout = dout;
    a.lse = lse; a.delta = w.delta; a.pos_k = positions; a.table = w.table;
    a.dq_acc = w.dq_acc; a.dk = dk; a.dv = dv;
    a.B = B; a.Nq = N; a.Nk = N; a.H = H; a.q_off = 0; a.rope_half = half;
    s = run_backward(a, segment_ids, segment_ids, 0, w, st);
    if (s != LWM_OK) return s;
  }
  return cuda_status(launch_dq_convert<T>(w.dq_acc, positions, w.table, B, N,
                                          H, scale, half, static_cast<T*>(dq),
                                          st));
}

size_t lwm_blockattn_bwd_block_workspace_size(int B, int Nq, int Nk, int H,
                                              int D) {
  if (!sizes_ok(B, Nq, H, D, kBlock, kBlock, 0) || Nk < 0 ||
      (int64_t(B) * Nk) >= (int64_t(1) << 31))
    return 0;
  return carve(nullptr, B, Nq, Nk, H, D, 0, Pass::kBwdBlock, LWM_DTYPE_BF16,
               LWM_QK_BF16)
      .bytes;
}

int lwm_blockattn_bwd_block(const void* q_rot, const void* k_rot,
                            const void* v, const void* dout, const float* lse,
                            const float* delta, const int32_t* seg_q,
                            const int32_t* seg_k, int q_off, int k_off, int B,
                            int Nq, int Nk, int H, int D, float* dq_acc,
                            float* dk_acc, float* dv_acc, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (!sizes_ok(B, Nq, H, D, kBlock, kBlock, 0) || Nk < 0 || q_off < 0 ||
      k_off < 0 || (int64_t(B) * Nk) >= (int64_t(1) << 31))
    return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim) return LWM_ERR_UNSUPPORTED;
  if (int64_t(B) * Nq * Nk * H == 0) return LWM_OK;
  const void* ptrs[] = {q_rot, k_rot, v, dout, lse, delta, seg_q, seg_k,
                        dq_acc, dk_acc, dv_acc, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  Workspace w = carve(workspace, B, Nq, Nk, H, D, 0, Pass::kBwdBlock,
                      LWM_DTYPE_BF16, LWM_QK_BF16);
  if (workspace_bytes < w.bytes) return LWM_ERR_WORKSPACE;
  BwdArgs a{};
  a.q_rot = q_rot; a.k_rot = k_rot; a.v = v; a.dout = dout;
  a.lse = lse; a.delta = delta;
  a.dq_acc = dq_acc; a.dk_acc = dk_acc; a.dv_acc = dv_acc;
  a.B = B; a.Nq = Nq; a.Nk = Nk; a.H = H; a.q_off = q_off;
  return run_backward(a, seg_q, seg_k, k_off, w,
                      static_cast<cudaStream_t>(stream));
}

int lwm_blockattn_bwd_delta(const void* out, const void* dout, int B, int N,
                            int H, int D, int dtype, float* delta,
                            void* stream) {
  if (B < 0 || N < 0 || H < 0) return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim || dtype != LWM_DTYPE_BF16) return LWM_ERR_UNSUPPORTED;
  if (int64_t(B) * N * H == 0) return LWM_OK;
  const void* ptrs[] = {out, dout, delta};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  using T = __nv_bfloat16;
  return cuda_status(launch_bwd_delta<T>(static_cast<const T*>(out),
                                         static_cast<const T*>(dout), B, N, H,
                                         delta,
                                         static_cast<cudaStream_t>(stream)));
}

int lwm_blockattn_grad_finish(const float* acc, const int32_t* positions,
                              const float* rope_table, int max_pos, int B,
                              int N, int H, int D, int dtype, int rope_layout,
                              void* grad, void* stream) {
  if (B < 0 || N < 0 || H < 0 || max_pos < 0) return LWM_ERR_INVALID_ARG;
  if (D != kHeadDim || dtype != LWM_DTYPE_BF16) return LWM_ERR_UNSUPPORTED;
  if (!layout_ok(rope_layout)) return LWM_ERR_INVALID_ARG;
  if (int64_t(B) * N * H == 0) return LWM_OK;
  if (!acc || !grad || !aligned16(acc) || !aligned16(grad))
    return LWM_ERR_INVALID_ARG;
  if (positions && (!rope_table || max_pos < 1)) return LWM_ERR_INVALID_ARG;
  const float scale = positions ? 1.f / std::sqrt(float(D)) : 1.f;
  return cuda_status(launch_dq_convert<__nv_bfloat16>(
      acc, positions, rope_table, B, N, H, scale,
      rope_layout == LWM_ROPE_HALF, static_cast<__nv_bfloat16*>(grad),
      static_cast<cudaStream_t>(stream)));
}

size_t lwm_blockffn_workspace_size(int chunk, int F) {
  if (chunk < 1 || F < 1) return 0;
  return align_up(size_t(chunk) * F * 2);
}

int lwm_blockffn_fwd(const void* x, const void* w_gate, const void* w_up,
                     const void* w_down, int T, int Dm, int F, int chunk,
                     int dtype, void* y, void* workspace,
                     size_t workspace_bytes, void* stream) {
  if (T < 0 || Dm < 1 || F < 1 || chunk < 1) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 || Dm % 64 != 0 || F % 64 != 0)
    return LWM_ERR_UNSUPPORTED;
  if (T == 0) return LWM_OK;
  if (int64_t(T) * std::max(Dm, F) >= (int64_t(1) << 40))
    return LWM_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_gate, w_up, w_down, y, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  const int c = std::min(chunk, T);
  if (workspace_bytes < lwm_blockffn_workspace_size(c, F))
    return LWM_ERR_WORKSPACE;
  int* status = status_word();
  if (!status) return LWM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const char* xb = static_cast<const char*>(x);
  char* yb = static_cast<char*>(y);
  // one chunk of tokens at a time: only [chunk][F] of intermediate is live
  for (int t0 = 0; t0 < T; t0 += c) {
    const int m = std::min(c, T - t0);
    LWM_TRY(launch_mlp_up(xb + size_t(t0) * Dm * 2, w_gate, w_up, m, Dm, F,
                          workspace, status, st));
    LWM_TRY(launch_mlp_down(workspace, w_down, m, F, Dm,
                            yb + size_t(t0) * Dm * 2, status, st));
  }
  return LWM_OK;
}

size_t lwm_blockffn_bwd_workspace_size(int chunk, int F) {
  if (chunk < 1 || F < 1) return 0;
  // dact [c][F], dh|dg [c][2F], act [c][F], all bf16
  return 3 * align_up(size_t(chunk) * F * 2) + align_up(size_t(chunk) * F * 2);
}

int lwm_blockffn_bwd(const void* x, const void* w_gate, const void* w_up,
                     const void* w_down, const void* dy, int T, int Dm, int F,
                     int chunk, int dtype, void* dx, float* dw_gate,
                     float* dw_up, float* dw_down, void* workspace,
                     size_t workspace_bytes, void* stream) {
  if (T < 0 || Dm < 1 || F < 1 || chunk < 1) return LWM_ERR_INVALID_ARG;
  if (dtype != LWM_DTYPE_BF16 || Dm % 64 != 0 || F % 64 != 0)
    return LWM_ERR_UNSUPPORTED;
  const void* ptrs[] = {w_gate, w_up, w_down, dw_gate, dw_up, dw_down};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
  if (int64_t(T) * std::max(Dm, F) >= (int64_t(1) << 40))
    return LWM_ERR_INVALID_ARG;
  // every check before the first launch: a rejected call writes nothing
  const int c = std::max(1, std::min(chunk, T));
  int* status = nullptr;
  if (T > 0) {
    const void* ptrs2[] = {x, dy, dx, workspace};
    for (const void* p : ptrs2)
      if (!p || !aligned16(p)) return LWM_ERR_INVALID_ARG;
    if (workspace_bytes < lwm_blockffn_bwd_workspace_size(c, F))
      return LWM_ERR_WORKSPACE;
    status = status_word();
    if (!status) return LWM_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the weight gradients are sums over every token: start from zero
  LWM_TRY(cudaMemsetAsync(dw_gate, 0, size_t(F) * Dm * 4, st));
  LWM_TRY(cudaMemsetAsync(dw_up, 0, size_t(F) * Dm * 4, st));
  LWM_TRY(cudaMemsetAsync(dw_down, 0, size_t(F) * Dm * 4, st));
  if (T == 0) return LWM_OK;
  char* ws = static_cast<char*>(workspace);
  const size_t one = align_up(size_t(c) * F * 2);
  void* dact = ws;
  void* dhg = ws + one;
  void* act = ws + 3 * one;
  const char* xb = static_cast<const char*>(x);
  const char* dyb = static_cast<const char*>(dy);
  char* dxb = static_cast<char*>(dx);
  for (int t0 = 0; t0 < T; t0 += c) {
    const int m = std::min(c, T - t0);
    const size_t off = size_t(t0) * Dm * 2;
    LWM_TRY(launch_mlp_bwd_chunk(xb + off, w_gate, w_up, w_down, dyb + off,
                                 m, Dm, F, dact, dhg, act, dxb + off, dw_gate,
                                 dw_up, dw_down, status, st));
  }
  return LWM_OK;
}

int lwm_blockattn_classify(const int32_t* segment_ids, int B, int N,
                           int block_q, int block_k, int32_t* kv_lo,
                           int32_t* kv_hi, uint8_t* tile_class,
                           void* stream) {
  if (B < 0 || N < 0 || (int64_t(B) * N) >= (int64_t(1) << 31))
    return LWM_ERR_INVALID_ARG;
  if (block_q < 16 || block_q > 1024 || block_k < 16 || block_k > 1024 ||
      block_q % block_k != 0)
    return LWM_ERR_UNSUPPORTED;
  if (int64_t(B) * N == 0) return LWM_OK;
  if (!segment_ids || !kv_lo || !kv_hi) return LWM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LWM_TRY(launch_block_meta(segment_ids, B, N, block_q, block_k, kv_lo, kv_hi,
                            st));
  if (tile_class)
    LWM_TRY(launch_tile_class(segment_ids, B, N, block_q, block_k, kv_lo,
                              kv_hi, tile_class, st));
  return LWM_OK;
}

int lwm_blockattn_visibility(const int32_t* seg_q, const int32_t* seg_k,
                             int B, int Nq, int Nk, int q_off, int k_off,
                             int block_q, int block_k, int32_t* row_lo,
                             int32_t* row_hi, int32_t* kv_lo, int32_t* kv_hi,
                             int32_t* lo_max, int32_t* hi_min,
                             int32_t* col_lo, int32_t* col_hi, int32_t* q_lo,
                             int32_t* q_hi, int32_t* klo_max,
                             int32_t* khi_min, void* stream) {
  if (B < 0 || Nq < 0 || Nk < 0 || q_off < 0 || k_off < 0 ||
      (int64_t(B) * Nq) >= (int64_t(1) << 31) ||
      (int64_t(B) * Nk) >= (int64_t(1) << 31))
    return LWM_ERR_INVALID_ARG;
  if (shape_status(kHeadDim, block_q, block_k) != LWM_OK)
    return LWM_ERR_UNSUPPORTED;
  int32_t* qside[] = {row_lo, row_hi, kv_lo, kv_hi, lo_max, hi_min};
  int32_t* kside[] = {col_lo, col_hi, q_lo, q_hi, klo_max, khi_min};
  // each view is written whole or not at all
  auto group = [](int32_t* const (&g)[6]) {
    int n = 0;
    for (int32_t* p : g) n += p != nullptr;
    return n;
  };
  const int nq = group(qside), nk = group(kside);
  if ((nq != 0 && nq != 6) || (nk != 0 && nk != 6)) return LWM_ERR_INVALID_ARG;
  // the backward's key view is in 128-key units whatever the forward's key
  // block height
  if (nk && block_k != kBlock) return LWM_ERR_UNSUPPORTED;
  if (int64_t(B) * Nq * Nk == 0 || (nq == 0 && nk == 0)) return LWM_OK;
  if (!seg_q || !seg_k) return LWM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the very launches lwm_blockattn_fwd / _fwd_block and lwm_blockattn_bwd /
  // _bwd_block make before their attention kernels
  if (nq)
    LWM_TRY(launch_cross_meta(seg_q, seg_k, B, Nq, Nk, q_off, k_off, block_k,
                              row_lo, row_hi, kv_lo, kv_hi, lo_max, hi_min,
                              st));
  if (nk)
    LWM_TRY(launch_cross_meta_keys(seg_q, seg_k, B, Nq, Nk, q_off, k_off,
                                   col_lo, col_hi, q_lo, q_hi, klo_max,
                                   khi_min, st));
  return LWM_OK;
}

int lwm_blockattn_rope_table(double theta, int D, int max_pos, float* table,
                             void* stream) {
  if (!(theta > 0.0) || !std::isfinite(theta) || D <= 0 || D % 2 ||
      max_pos < 0)
    return LWM_ERR_INVALID_ARG;
  if (max_pos == 0) return LWM_OK;
  if (!table) return LWM_ERR_INVALID_ARG;
  return cuda_status(launch_rope_table(theta, D, max_pos, table,
                                       static_cast<cudaStream_t>(stream)));
}

int lwm_blockattn_check_inputs(const int32_t* segment_ids,
                               const int32_t* positions, int B, int N,
                               int max_pos, int* max_pos_out, void* stream) {
  if (B < 0 || N < 0 || max_pos < 0) return LWM_ERR_INVALID_ARG;
  if (int64_t(B) * N == 0) {
    if (max_pos_out) *max_pos_out = 0;
    return LWM_OK;
  }
  if (!segment_ids || !positions) return LWM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* words = nullptr;
  LWM_TRY(cudaGetSymbolAddress(&words, g_check_words));
  int init[2] = {0, -1};
  LWM_TRY(cudaMemcpyAsync(words, init, sizeof(init), cudaMemcpyHostToDevice,
                          st));
  LWM_TRY(launch_check_inputs(segment_ids, positions, B, N, max_pos,
                              static_cast<int*>(words), st));
  int res[2];
  LWM_TRY(cudaMemcpyAsync(res, words, sizeof(res), cudaMemcpyDeviceToHost, st));
  LWM_TRY(cudaStreamSynchronize(st));
  if (max_pos_out) *max_pos_out = res[1] + 1;
  return res[0] ? LWM_ERR_PRECONDITION : LWM_OK;
}

int lwm_blockattn_last_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LWM_ERR_CUDA;
  void* word = nullptr;
  if (cudaGetSymbolAddress(&word, g_status_word) != cudaSuccess)
    return LWM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LWM_ERR_CUDA;
  int zero = 0;
  if (cudaMemcpy(word, &zero, sizeof(int), cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return LWM_ERR_CUDA;
  return v;
}

}  // extern "C"
