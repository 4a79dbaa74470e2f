// Blockwise feed-forward network on tcgen05 (sm_100a).
//
// The other half of the blockwise transformer: the MLP runs over the
// sequence in chunks of scan_mlp_chunk_size tokens (8192 in the configs of
// "LWM：突破 100 万 Token 的开源大模型", 配置参数 / 脚本运行说明), so only one
// chunk's [chunk x F] intermediates are ever live. The block is Llama-2's
// ("Inside Large World Model", Core Architecture; Stage I):
//   h = x Wg^T, g = x Wu^T, act = silu(h) * g,   y = act Wd^T,
// with Wg, Wu [F][Dm] and Wd [Dm][F] stored as nn.Linear weights (row =
// output feature). Its chain rule, per chunk (h and g recomputed):
//   dact = dy Wd,  dh = dact * g * silu'(h),  dg = dact * silu(h),
//   dx = dh Wg + dg Wu,  dWd += dy^T act,  dWg += dh^T x,  dWu += dg^T x.
//
// Every product is one persistent GEMM kernel, C [M][N] = A [M][K] B[N][K]^T
// with either operand stored K-major (rows of K contiguous) or MN-major
// (the transposed storage), and one of four epilogues:
//   SwiGLU      a 128 x 256 tile of [x Wg^T | x Wu^T] (one N = 256 MMA over
//               a B tile stacked from both weights) -> act (bf16);
//   SwiGLUBwd   the same tile plus the matching dact tile read from global
//               memory -> dh, dg (bf16, side by side in one [M][2F] buffer)
//               and act (bf16, for dWd);
//   Store       bf16 C;
//   AccF32      C added into an fp32 accumulator (weight gradients summed
//               over the chunks).
// All are dense contractions: tensor-bound.
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
constexpr int kMnChunk = 64 * kBK * 2;           // 8 KB: 64 MN x 64 K
constexpr uint64_t kGemmWaitNs = 4000000000ull;
enum { gFull = 0, gEmpty = kStages, gAccFull = 2 * kStages,
       gAccEmpty = 2 * kStages + 2, gDone = 2 * kStages + 4,
       kGemmBars = 2 * kStages + 5 };
constexpr int kGemmBarOff = kStages * kStageBytes;
constexpr int kGemmMisc = kGemmBarOff + kGemmBars * 8;
constexpr int kGemmSmem = kGemmMisc + 16 + 1024;   // + alignment slack

enum Epilogue { kEpiSwiGLU = 0, kEpiStore = 1, kEpiAccF32 = 2,
                kEpiSwiGLUBwd = 3 };

struct GemmParams {
  int M, N;               // output rows / columns
  int Mt, Nt, Kt;         // tiles
  int k_split;            // MN-major B: K blocks [0, k_split) from map b0,
                          // the rest from b1 (K offset restarting at 0)
  void* out;              // bf16 [M][ld_out] (Store, SwiGLU: act; SwiGLUBwd:
                          // dh, with dg at out + N) or fp32 (AccF32)
  int ld_out;             // row stride of out in elements
  const __nv_bfloat16* aux;  // SwiGLUBwd: dact [M][N]
  __nv_bfloat16* out2;    // SwiGLUBwd: act [M][N]
  int* status;
};

__device__ __forceinline__ float sigmoid_fast(float h) {
  return rcp_approx(1.f + ex2(-h * kLog2e));
}

template <int EPI, bool A_MN, bool B_MN>
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
  constexpr bool kPairedB = EPI == kEpiSwiGLU || EPI == kEpiSwiGLUBwd;

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
      if (kPairedB) {
        // columns [0,128): h = x Wg^T, [128,256): g = x Wu^T of the
        // intermediate columns nb*128 .. +127
        const int64_t base = int64_t(row) * p.N + nb * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t hv[32], gv[32];
          tmem_ld32(tacc + c * 32, hv);
          tmem_ld32(tacc + 128 + c * 32, gv);
          tmem_wait_ld();
          const bool live = row < p.M && nb * 128 + c * 32 < p.N;
          uint32_t da[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) da[e] = 0u;
          if (EPI == kEpiSwiGLUBwd && live) {
            const uint4* s4 =
                reinterpret_cast<const uint4*>(p.aux + base + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint4 w = s4[e];
              da[4 * e] = w.x;
              da[4 * e + 1] = w.y;
              da[4 * e + 2] = w.z;
              da[4 * e + 3] = w.w;
            }
          }
          uint32_t pa[16], pdh[16], pdg[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float a[2], dh[2], dg[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float h = __uint_as_float(hv[x + u]);
              const float g = __uint_as_float(gv[x + u]);
              // silu(h) = h s with s = 1 / (1 + e^-h);
              // silu'(h) = s (1 + h (1 - s))
              const float s = sigmoid_fast(h);
              a[u] = h * s * g;
              if (EPI == kEpiSwiGLUBwd) {
                const float d = u ? bf16hi_to_f32(da[x >> 1])
                                  : bf16lo_to_f32(da[x >> 1]);
                dh[u] = d * g * s * fmaf(h, 1.f - s, 1.f);
                dg[u] = d * h * s;
              }
            }
            pa[x >> 1] = pack_bf16x2(a[0], a[1]);
            if (EPI == kEpiSwiGLUBwd) {
              pdh[x >> 1] = pack_bf16x2(dh[0], dh[1]);
              pdg[x >> 1] = pack_bf16x2(dg[0], dg[1]);
            }
          }
          if (live) {
            if (EPI == kEpiSwiGLU) {
              uint4* d4 = reinterpret_cast<uint4*>(
                  static_cast<__nv_bfloat16*>(p.out) + base + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                d4[e] = make_uint4(pa[4 * e], pa[4 * e + 1], pa[4 * e + 2],
                                   pa[4 * e + 3]);
            } else {
              // dh and dg side by side in [M][2N]; act in [M][N]
              __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                                 int64_t(row) * p.ld_out + nb * 128 + c * 32;
              uint4* dh4 = reinterpret_cast<uint4*>(o);
              uint4* dg4 = reinterpret_cast<uint4*>(o + p.N);
              uint4* a4 = reinterpret_cast<uint4*>(p.out2 + base + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                dh4[e] = make_uint4(pdh[4 * e], pdh[4 * e + 1],
                                    pdh[4 * e + 2], pdh[4 * e + 3]);
                dg4[e] = make_uint4(pdg[4 * e], pdg[4 * e + 1],
                                    pdg[4 * e + 2], pdg[4 * e + 3]);
                a4[e] = make_uint4(pa[4 * e], pa[4 * e + 1], pa[4 * e + 2],
                                   pa[4 * e + 3]);
              }
            }
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
          const int col = nb * kBN + c * 32;
          if (row >= p.M || col >= p.N) continue;
          if (EPI == kEpiStore) {
            uint32_t pk[16];
#pragma unroll
            for (int x = 0; x < 32; x += 2)
              pk[x >> 1] = pack_bf16x2(__uint_as_float(v[x]),
                                       __uint_as_float(v[x + 1]));
            uint4* d4 = reinterpret_cast<uint4*>(
                static_cast<__nv_bfloat16*>(p.out) + int64_t(row) * p.ld_out +
                col);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2],
                                 pk[4 * e + 3]);
          } else {  // AccF32: one CTA owns the tile, launches are ordered
            float4* d4 = reinterpret_cast<float4*>(
                static_cast<float*>(p.out) + int64_t(row) * p.ld_out + col);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 a = d4[e];
              a.x += __uint_as_float(v[4 * e]);
              a.y += __uint_as_float(v[4 * e + 1]);
              a.z += __uint_as_float(v[4 * e + 2]);
              a.w += __uint_as_float(v[4 * e + 3]);
              d4[e] = a;
            }
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
        // K-major B: rows of the two 128-row halves of the tile
        const int r0 = kPairedB ? nb * 128 : nb * kBN;
        const int r1 = kPairedB ? nb * 128 : nb * kBN + 128;
        for (int kb = 0; kb < p.Kt && ok; ++kb, ++f) {
          const int s = f % kStages;
          if (f >= kStages)
            ok = mbar_wait(bar(gEmpty + s), ((f / kStages) - 1) & 1,
                           abort_flag, p.status, kGemmWaitNs);
          if (!ok) break;
          const uint32_t sa = sbase + s * kStageBytes, sb = sa + kATile;
          mbar_arrive_expect_tx(bar(gFull + s), kStageBytes);
          if (A_MN) {  // [K][M] storage: two 64-wide M chunks
            tma_load_2d(sa, &tm_a, bar(gFull + s), m0, kb * kBK);
            tma_load_2d(sa + kMnChunk, &tm_a, bar(gFull + s), m0 + 64,
                        kb * kBK);
          } else {
            tma_load_2d(sa, &tm_a, bar(gFull + s), kb * kBK, m0);
          }
          if (B_MN) {  // [K][N] storage: four 64-wide N chunks
            const bool second = kb >= p.k_split;
            const CUtensorMap* mb = second ? &tm_b1 : &tm_b0;
            const int kk = (second ? kb - p.k_split : kb) * kBK;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_2d(sb + c * kMnChunk, mb, bar(gFull + s),
                          nb * kBN + c * 64, kk);
          } else {
            tma_load_2d(sb, &tm_b0, bar(gFull + s), kb * kBK, r0);
            tma_load_2d(sb + kBTile / 2, &tm_b1, bar(gFull + s), kb * kBK,
                        r1);
          }
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
      const uint32_t idesc = idesc_bf16(kBM, kBN, A_MN ? 1 : 0, B_MN ? 1 : 0);
      // K-major: 128-byte rows of K, +32 bytes per K = 16 step; MN-major:
      // 64-wide MN chunks 8 KB apart, +16 rows (2 KB) per step
      const uint64_t sta = A_MN ? (2048 >> 4) : (32 >> 4);
      const uint64_t stb = B_MN ? (2048 >> 4) : (32 >> 4);
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
          const uint64_t da = A_MN ? sdesc_sw128(sa, kMnChunk, 1024)
                                   : sdesc_sw128(sa, 16, 1024);
          const uint64_t db = B_MN ? sdesc_sw128(sb, kMnChunk, 1024)
                                   : sdesc_sw128(sb, 16, 1024);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_ss(d, da + k * sta, db + k * stb, idesc,
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

template <int EPI, bool A_MN, bool B_MN>
cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb0,
                        const CUtensorMap& mb1, const GemmParams& p,
                        cudaStream_t st) {
  auto kern = mlp_gemm_kernel<EPI, A_MN, B_MN>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), p.Mt * p.Nt);
  kern<<<grid, kGemmThreads, kGemmSmem, st>>>(ma, mb0, mb1, p);
  note_launch();
  return cudaGetLastError();
}

GemmParams tiles(int M, int N, int K, int n_tile, int* status) {
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.Mt = (M + kBM - 1) / kBM;
  p.Nt = (N + n_tile - 1) / n_tile;
  p.Kt = (K + kBK - 1) / kBK;
  p.k_split = p.Kt;
  p.status = status;
  return p;
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
  GemmParams p = tiles(M, F, Dm, 128, status);
  p.out = act;
  p.ld_out = F;
  return launch_gemm<kEpiSwiGLU, false, false>(ma, mg, mu, p, st);
}

cudaError_t launch_mlp_down(const void* act, const void* w_down, int M,
                            int F, int Dm, void* y, int* status,
                            cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  CUtensorMap ma, mb;
  if (!make_2d_map(&ma, act, M, F, kBM) || !make_2d_map(&mb, w_down, Dm, F, 128))
    return cudaErrorInvalidValue;
  GemmParams p = tiles(M, Dm, F, kBN, status);
  p.out = y;
  p.ld_out = Dm;
  return launch_gemm<kEpiStore, false, false>(ma, mb, mb, p, st);
}

cudaError_t launch_mlp_bwd_chunk(const void* x, const void* w_gate,
                                 const void* w_up, const void* w_down,
                                 const void* dy, int M, int Dm, int F,
                                 void* dact, void* dhg, void* act, void* dx,
                                 float* dwg, float* dwu, float* dwd,
                                 int* status, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  cudaError_t e;
  // 1. dact [M][F] = dy [M][Dm] . Wd [Dm][F]   (B stored [K][N])
  {
    CUtensorMap ma, mb;
    if (!make_2d_map(&ma, dy, M, Dm, kBM) ||
        !make_2d_map(&mb, w_down, Dm, F, 64))
      return cudaErrorInvalidValue;
    GemmParams p = tiles(M, F, Dm, kBN, status);
    p.out = dact;
    p.ld_out = F;
    e = launch_gemm<kEpiStore, false, true>(ma, mb, mb, p, st);
    if (e != cudaSuccess) return e;
  }
  // 2. h, g recomputed; dh, dg -> dhg [M][2F], act -> act [M][F]
  {
    CUtensorMap ma, mg, mu;
    if (!make_2d_map(&ma, x, M, Dm, kBM) ||
        !make_2d_map(&mg, w_gate, F, Dm, 128) ||
        !make_2d_map(&mu, w_up, F, Dm, 128))
      return cudaErrorInvalidValue;
    GemmParams p = tiles(M, F, Dm, 128, status);
    p.out = dhg;
    p.ld_out = 2 * F;
    p.aux = static_cast<const __nv_bfloat16*>(dact);
    p.out2 = static_cast<__nv_bfloat16*>(act);
    e = launch_gemm<kEpiSwiGLUBwd, false, false>(ma, mg, mu, p, st);
    if (e != cudaSuccess) return e;
  }
  // 3. dx [M][Dm] = [dh | dg] [M][2F] . [Wg ; Wu] [2F][Dm]  (B stored
  //    [K][N]: the K blocks of Wg, then those of Wu)
  {
    CUtensorMap ma, mg, mu;
    if (!make_2d_map(&ma, dhg, M, 2 * int64_t(F), kBM) ||
        !make_2d_map(&mg, w_gate, F, Dm, 64) ||
        !make_2d_map(&mu, w_up, F, Dm, 64))
      return cudaErrorInvalidValue;
    GemmParams p = tiles(M, Dm, 2 * F, kBN, status);
    p.k_split = F / kBK;
    p.out = dx;
    p.ld_out = Dm;
    e = launch_gemm<kEpiStore, false, true>(ma, mg, mu, p, st);
    if (e != cudaSuccess) return e;
  }
  // 4. dWd [Dm][F] += dy^T . act: A = dy stored [K = M][Dm], B = act
  //    stored [K = M][F]
  {
    CUtensorMap ma, mb;
    if (!make_2d_map(&ma, dy, M, Dm, 64) || !make_2d_map(&mb, act, M, F, 64))
      return cudaErrorInvalidValue;
    GemmParams p = tiles(Dm, F, M, kBN, status);
    p.out = dwd;
    p.ld_out = F;
    e = launch_gemm<kEpiAccF32, true, true>(ma, mb, mb, p, st);
    if (e != cudaSuccess) return e;
  }
  // 5. dWg [F][Dm] += dh^T . x and 6. dWu += dg^T . x: A = the dh (dg)
  //    half of dhg stored [K = M][2F], B = x stored [K = M][Dm]
  {
    CUtensorMap mx;
    if (!make_2d_map(&mx, x, M, Dm, 64)) return cudaErrorInvalidValue;
    for (int half = 0; half < 2; ++half) {
      CUtensorMap ma;
      const char* base = static_cast<const char*>(dhg) + size_t(half) * F * 2;
      if (!make_2d_map_strided(&ma, base, M, F, 2 * int64_t(F), 64))
        return cudaErrorInvalidValue;
      GemmParams p = tiles(F, Dm, M, kBN, status);
      p.out = half ? dwu : dwg;
      p.ld_out = Dm;
      e = launch_gemm<kEpiAccF32, true, true>(ma, mx, mx, p, st);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

}  // namespace lwm
