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

// The backward of one chunk of M tokens: dact [M][F], dhg [M][2F] and act
// [M][F] are bf16 scratch; dx [M][Dm] bf16 is written; the fp32 weight
// gradients dwg, dwu [F][Dm] and dwd [Dm][F] are added to.
cudaError_t launch_mlp_bwd_chunk(const void* x, const void* w_gate,
                                 const void* w_up, const void* w_down,
                                 const void* dy, int M, int Dm, int F,
                                 void* dact, void* dhg, void* act, void* dx,
                                 float* dwg, float* dwu, float* dwd,
                                 int* status, cudaStream_t st);

}  // namespace lwm
