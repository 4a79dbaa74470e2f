// Blockwise feed-forward network on tcgen05 (sm_100a).
//
// The other half of the blockwise transformer: the MLP runs over the
// sequence in chunks of scan_mlp_chunk_size tokens (8192 in the configs of
// "LWM：突破 100 万 Token 的开源大模型", 配置参数 / 脚本运行说明), so only one
// chunk's [chunk x F] intermediate is ever live. The block is Llama-2's
// ("Inside Large World Model", Core Architecture; Stage I):
//   act = silu(x Wg^T) * (x Wu^T),   y = act Wd^T,
// with Wg, Wu [F][Dm] and Wd [Dm][F] stored as nn.Linear weights (row =
// output feature). Per chunk two launches of one persistent GEMM kernel:
//   up:   a 128 x 256 tile of [x Wg^T | x Wu^T] (128 columns of each, one
//         N = 256 MMA over a B tile stacked from both weights), the SwiGLU
//         epilogue writes the 128 x 128 act tile (bf16);
//   down: a 128 x 256 tile of act Wd^T, stored as bf16.
// Both are dense contractions: tensor-bound.
//
// CTA: warps 0-3 epilogue (TMEM lanes 0-127), warp 4 TMA producer, warp 5
// tcgen05 issuer + TMEM owner. Four 48 KB shared-memory stages (A 128 x 64,
// B 256 x 64, 128-byte swizzle); two 256-column TMEM accumulators, so the
// epilogue of one tile overlaps the MMAs of the next.
#include <cuda.h>

#include "aux_kernels.cuh"
#include "mlp.cuh"
#include "tc_kernels.cuh"

namespace lwm {
namespace {

constexpr int kGemmThreads = 6 * 32;
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kATile = kBM * kBK * 2;            // 16 KB
constexpr int kBTile = kBN * kBK * 2;            // 32 KB
constexpr int kStageBytes = kATile + kBTile;
constexpr uint64_t kGemmWaitNs = 4000000000ull;
enum { gFull = 0, gEmpty = kStages, gAccFull = 2 * kStages,
       gAccEmpty = 2 * kStages + 2, gDone = 2 * kStages + 4,
       kGemmBars = 2 * kStages + 5 };
constexpr int kGemmBarOff = kStages * kStageBytes;
constexpr int kGemmMisc = kGemmBarOff + kGemmBars * 8;
constexpr int kGemmSmem = kGemmMisc + 16 + 1024;   // + alignment slack

enum Epilogue { kEpiSwiGLU = 0, kEpiStore = 1 };

struct GemmParams {
  int M, N, K;            // C [M][N] = A [M][K] . B [N][K]^T (N: output cols)
  int Mt, Nt, Kt;         // tiles
  __nv_bfloat16* out;     // [M][N_out] bf16
  int ld_out;             // row stride of out in elements
  int* status;
};

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
mlp_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                const __grid_constant__ CUtensorMap tm_b0,
                const __grid_constant__ CUtensorMap tm_b1,
                const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kGemmBarOff + 8u * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kGemmMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kGemmMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(gFull + s), 1);
      mbar_init(bar(gEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(gAccFull + b), 1);
      mbar_init(bar(gAccEmpty + b), 4);
    }
    mbar_init(bar(gDone), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b0);
    prefetch_tmap(&tm_b1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntiles = p.Mt * p.Nt;

  if (warp < 4) {
    // ------------------------------------------------------- epilogue
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    int tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tc) {
      const int buf = tc & 1;
      ok = mbar_wait(bar(gAccFull + buf), (tc >> 1) & 1, abort_flag, p.status,
                     kGemmWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int m0 = (t % p.Mt) * kBM, nb = t / p.Mt;
      const int row = m0 + warp * 32 + lane;
      const uint32_t tacc = tmem + lane_off + buf * kBN;
      if (EPI == kEpiSwiGLU) {
        // columns [0,128): x Wg^T, [128,256): x Wu^T of act columns
        // nb*128 .. +127
        __nv_bfloat16* dst = p.out + int64_t(row) * p.ld_out + nb * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t hv[32], gv[32];
          tmem_ld32(tacc + c * 32, hv);
          tmem_ld32(tacc + 128 + c * 32, gv);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float a[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float h = __uint_as_float(hv[x + u]);
              const float g = __uint_as_float(gv[x + u]);
              // silu(h) = h / (1 + e^-h)
              a[u] = h * rcp_approx(1.f + ex2(-h * kLog2e)) * g;
            }
            pk[x >> 1] = pack_bf16x2(a[0], a[1]);
          }
          if (row < p.M && nb * 128 + c * 32 < p.N) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2],
                                 pk[4 * e + 3]);
          }
        }
      } else {
        __nv_bfloat16* dst = p.out + int64_t(row) * p.ld_out + nb * kBN;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            pk[x >> 1] = pack_bf16x2(__uint_as_float(v[x]),
                                     __uint_as_float(v[x + 1]));
          if (row < p.M && nb * kBN + c * 32 < p.N) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2],
                                 pk[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(gAccEmpty + buf));
    }
  } else if (warp == 4) {
    // ------------------------------------------------------- producer
    if (lane == 0) {
      int f = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int m0 = (t % p.Mt) * kBM, nb = t / p.Mt;
        // B rows of the two 128-row halves of the tile
        const int r0 = EPI == kEpiSwiGLU ? nb * 128 : nb * kBN;
        const int r1 = EPI == kEpiSwiGLU ? nb * 128 : nb * kBN + 128;
        for (int kb = 0; kb < p.Kt && ok; ++kb, ++f) {
          const int s = f % kStages;
          if (f >= kStages)
            ok = mbar_wait(bar(gEmpty + s), ((f / kStages) - 1) & 1,
                           abort_flag, p.status, kGemmWaitNs);
          if (!ok) break;
          const uint32_t sa = sbase + s * kStageBytes, sb = sa + kATile;
          mbar_arrive_expect_tx(bar(gFull + s), kStageBytes);
          tma_load_2d(sa, &tm_a, bar(gFull + s), kb * kBK, m0);
          tma_load_2d(sb, &tm_b0, bar(gFull + s), kb * kBK, r0);
          tma_load_2d(sb + kBTile / 2, &tm_b1, bar(gFull + s), kb * kBK, r1);
        }
      }
      // drain: the last stages' loads must land before the CTA exits
      for (int g = f - 1; g >= 0 && g >= f - kStages; --g)
        mbar_wait(bar(gFull + g % kStages), (g / kStages) & 1, nullptr,
                  p.status, kGemmWaitNs);
    }
  } else {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, kBN, 0, 0);
      int c = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tc) {
        const int buf = tc & 1;
        if (tc >= 2)
          ok = mbar_wait(bar(gAccEmpty + buf), ((tc >> 1) - 1) & 1,
                         abort_flag, p.status, kGemmWaitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kBN;
        for (int kb = 0; kb < p.Kt && ok; ++kb, ++c) {
          const int s = c % kStages;
          ok = mbar_wait(bar(gFull + s), (c / kStages) & 1, abort_flag,
                         p.status, kGemmWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = sbase + s * kStageBytes, sb = sa + kATile;
          const uint64_t da = sdesc_sw128(sa, 16, 1024);
          const uint64_t db = sdesc_sw128(sb, 16, 1024);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // +32 bytes per K=16 step
            mma_ss(d, da + uint64_t(k * 2), db + uint64_t(k * 2), idesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(bar(gEmpty + s));
        }
        if (!ok) break;
        mma_commit(bar(gAccFull + buf));
      }
      // every issued MMA must be complete before TMEM is released
      mma_commit(bar(gDone));
      mbar_wait(bar(gDone), 0, nullptr, p.status, kGemmWaitNs);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int EPI>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb0,
                        const CUtensorMap& mb1, const GemmParams& p,
                        cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(
      mlp_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      kGemmSmem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), p.Mt * p.Nt);
  mlp_gemm_kernel<EPI><<<grid, kGemmThreads, kGemmSmem, st>>>(ma, mb0, mb1,
                                                              p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mlp_up(const void* x, const void* w_gate, const void* w_up,
                          int M, int Dm, int F, void* act, int* status,
                          cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  CUtensorMap ma, mg, mu;
  if (!make_2d_map(&ma, x, M, Dm, kBM) || !make_2d_map(&mg, w_gate, F, Dm, 128) ||
      !make_2d_map(&mu, w_up, F, Dm, 128))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M;
  p.N = F;
  p.K = Dm;
  p.Mt = (M + kBM - 1) / kBM;
  p.Nt = (F + 127) / 128;
  p.Kt = (Dm + kBK - 1) / kBK;
  p.out = static_cast<__nv_bfloat16*>(act);
  p.ld_out = F;
  p.status = status;
  return launch_gemm<kEpiSwiGLU>(ma, mg, mu, p, st);
}

cudaError_t launch_mlp_down(const void* act, const void* w_down, int M,
                            int F, int Dm, void* y, int* status,
                            cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  CUtensorMap ma, mb;
  if (!make_2d_map(&ma, act, M, F, kBM) || !make_2d_map(&mb, w_down, Dm, F, 128))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M;
  p.N = Dm;
  p.K = F;
  p.Mt = (M + kBM - 1) / kBM;
  p.Nt = (Dm + kBN - 1) / kBN;
  p.Kt = (F + kBK - 1) / kBK;
  p.out = static_cast<__nv_bfloat16*>(y);
  p.ld_out = Dm;
  p.status = status;
  return launch_gemm<kEpiStore>(ma, mb, mb, p, st);
}

}  // namespace lwm
