// Backward pass entry for the bf16 path. Interim: the CUDA-core backward
// kernel; the tcgen05 key-major backward replaces it.
#include "aux_kernels.cuh"
#include "tc_kernels.cuh"

namespace lwm {
cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t st) {
  using T = __nv_bfloat16;
  return launch_bwd_simt<T>(static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                            static_cast<const T*>(a.v), static_cast<const T*>(a.dout),
                            a.lse, a.delta, a.seg, a.pos, a.table, a.B, a.N, a.H,
                            a.dq_acc, static_cast<T*>(a.dk), static_cast<T*>(a.dv), st);
}
}  // namespace lwm
