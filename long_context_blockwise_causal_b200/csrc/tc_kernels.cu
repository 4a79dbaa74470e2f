// Temporary: bf16 path on the CUDA-core kernels until the tcgen05 kernels land.
#include "aux_kernels.cuh"
#include "tc_kernels.cuh"

namespace lwm {
cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t st) {
  using T = __nv_bfloat16;
  return launch_fwd_simt<T>(static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                            static_cast<const T*>(a.v), a.seg, a.pos, a.table,
                            a.kv_lo, a.B, a.N, a.H, static_cast<T*>(a.out), a.lse, st);
}
cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t st) {
  using T = __nv_bfloat16;
  return launch_bwd_simt<T>(static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                            static_cast<const T*>(a.v), static_cast<const T*>(a.dout),
                            a.lse, a.delta, a.seg, a.pos, a.table, a.B, a.N, a.H,
                            a.dq_acc, static_cast<T*>(a.dk), static_cast<T*>(a.dv), st);
}
}  // namespace lwm
