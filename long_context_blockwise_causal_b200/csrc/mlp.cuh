// Blockwise feed-forward (SwiGLU MLP) kernels (see mlp.cu).
#pragma once

#include "common.cuh"

namespace lwm {

// act [M][F] = silu(x Wg^T) * (x Wu^T): x [M][Dm], Wg, Wu [F][Dm], bf16.
cudaError_t launch_mlp_up(const void* x, const void* w_gate, const void* w_up,
                          int M, int Dm, int F, void* act, int* status,
                          cudaStream_t st);
// y [M][Dm] = act Wd^T: act [M][F], Wd [Dm][F], bf16.
cudaError_t launch_mlp_down(const void* act, const void* w_down, int M,
                            int F, int Dm, void* y, int* status,
                            cudaStream_t st);

}  // namespace lwm
