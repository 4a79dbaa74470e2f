// Decode attention: one new query token per (batch row, head) against a
// long cache of rotated keys and values (the inference side of the 1M-token
// models, "LWM：突破 100 万 Token 的开源大模型", 概述 / 脚本运行说明; the
// single-needle retrieval over 1M tokens in "[论文解读] World Model on
// Million-Length Video And Language With Blockwise RingAttention", 主要发现).
//
// The query of row b is the cache's last token; under masked packing it
// sees the keys [kv_start[b], kv_len[b]) of its own example (causality is
// automatic: no cached key lies after it). Split-KV: the keys of a (b, h)
// are cut into `splits` chunks (work items); a persistent CTA per SM takes
// the items round-robin and streams each chunk with an online softmax into
// a partial (max, sum, 128-wide accumulator); a second kernel merges the
// partials of a (b, h) into out and lse. The pass reads every visible key
// and value row once (2 x 256 bytes per key): it is bound by HBM bandwidth,
// so the rows come in by TMA, 128 keys (32 KB of K and 32 KB of V) per
// step, through a three-stage shared-memory ring that keeps two steps in
// flight while the third is computed. Per step, 16 lanes share a key row
// (16 bytes each, conflict-free reads of the swizzled tile); every warp
// forms the step's max, probabilities and sum from the 128 scores itself,
// so a step needs two block barriers.
#include <cuda.h>

#include "aux_kernels.cuh"
#include "decode.cuh"
#include "tc_kernels.cuh"

namespace lwm {
namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecRows = 128;                       // keys per step
constexpr int kDecStages = 3;
constexpr int kDecTile = kDecRows * kHeadDim * 2;   // K or V of one step
constexpr int kDecHalf = kDecTile / 2;              // one 64-dim half
constexpr int kDecGroups = kDecThreads / 16;        // 16 lanes per row
static_assert(kDecGroups == 32 && kDecRows == 128,
              "a row group's value rows are g + 32 k, k < 4");
// shared memory (bytes from the 1024-aligned base): stage s holds K at
// 2 s kDecTile and V right after it, each as two 64-dim halves of
// 128-byte rows with the 128-byte swizzle
constexpr int kDecQs = kDecStages * 2 * kDecTile;   // float[128]
constexpr int kDecPs = kDecQs + kHeadDim * 4;       // float[128]
constexpr int kDecAcc = kDecPs + kDecRows * 4;      // float[groups][128]
constexpr int kDecBars = kDecAcc + kDecGroups * kHeadDim * 4;
constexpr int kDecSmem = kDecBars + kDecStages * 8 + 1024;
static_assert(kDecSmem <= 232448, "shared memory per CTA");
constexpr uint64_t kDecWaitNs = 4000000000ull;      // 4 s per wait

struct DecItem {
  int b, h, c0, c1;
  int64_t slot;
};

// Work item `item` = (b, h, split): keys [c0, c1) of (b, h). Out-of-range
// inputs are clamped so no read leaves the cache.
__device__ __forceinline__ DecItem dec_item(int item, int H, int splits,
                                            int L,
                                            const int32_t* __restrict__ kv_start,
                                            const int32_t* __restrict__ kv_len) {
  DecItem d;
  const int split = item % splits, bh = item / splits;
  d.h = bh % H;
  d.b = bh / H;
  const int len = max(0, min(__ldg(kv_len + d.b), L));
  const int start = max(0, min(__ldg(kv_start + d.b), len));
  const int chunk = (len - start + splits - 1) / splits;
  d.c0 = start + split * chunk;
  d.c1 = min(d.c0 + chunk, len);
  d.slot = int64_t(bh) * splits + split;
  return d;
}

// One 16-byte unit (8 bf16, dims 8u..8u+7 of a 64-dim half) of row r of a
// swizzled tile half: the unit sits at position u ^ (r mod 8) of its row.
__device__ __forceinline__ uint4 dec_unit(const uint8_t* half_tile, int r,
                                          int u) {
  return *reinterpret_cast<const uint4*>(half_tile + r * 128 +
                                         ((u ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kDecThreads, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __nv_bfloat16* __restrict__ q,
                    const int32_t* __restrict__ kv_start,
                    const int32_t* __restrict__ kv_len,
                    const int32_t* __restrict__ q_pos,
                    const float2* __restrict__ table, int max_pos, int L,
                    int H, int splits, int n_items, bool half,
                    float scale_log2, float* __restrict__ part_m,
                    float* __restrict__ part_l, float* __restrict__ part_acc,
                    int* status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(smem + kDecQs);
  float* ps = reinterpret_cast<float*>(smem + kDecPs);
  float* racc = reinterpret_cast<float*>(smem + kDecAcc);
  const uint32_t bars = smem_u32(smem + kDecBars);
  auto bar = [&](int s) { return bars + 8u * s; };
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // a row is read by 16 lanes, lane l16 taking 16-byte unit l16 % 8 of
  // 64-dim half l16 / 8, i.e. dims 8 l16 .. 8 l16 + 7
  const int l16 = lane & 15, hf = l16 >> 3, u = l16 & 7;

  if (t == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(bar(s), 1);
    fence_mbar_init();
  }
  __syncthreads();

  // producer state (thread 0): the next step to load, which runs
  // kDecStages - 1 steps ahead of the one being computed; it walks the
  // same (item, step) sequence as the consumers, skipping empty items
  const CUtensorMap* mk = &tm_k;
  const CUtensorMap* mv = &tm_v;
  int p_item = blockIdx.x, p_j0 = 0, p_c1 = 0, p_b = 0, p_h = 0, p_n = 0;
  auto p_seek = [&]() {
    while (p_item < n_items && p_j0 >= p_c1) {
      p_item += gridDim.x;
      if (p_item < n_items) {
        const DecItem d = dec_item(p_item, H, splits, L, kv_start, kv_len);
        p_j0 = d.c0;
        p_c1 = d.c1;
        p_b = d.b;
        p_h = d.h;
      }
    }
  };
  auto p_issue = [&]() {
    if (p_item >= n_items) return;
    const int s = p_n % kDecStages;
    const uint32_t dk = smem_u32(smem + s * 2 * kDecTile);
    const uint32_t dv = dk + kDecTile;
    mbar_arrive_expect_tx(bar(s), 2 * kDecTile);
    tma_load_4d(dk, mk, bar(s), 0, p_h, p_j0, p_b);
    tma_load_4d(dk + kDecHalf, mk, bar(s), 64, p_h, p_j0, p_b);
    tma_load_4d(dv, mv, bar(s), 0, p_h, p_j0, p_b);
    tma_load_4d(dv + kDecHalf, mv, bar(s), 64, p_h, p_j0, p_b);
    ++p_n;
    p_j0 += kDecRows;
    p_seek();
  };
  if (t == 0) {
    if (p_item < n_items) {
      const DecItem d = dec_item(p_item, H, splits, L, kv_start, kv_len);
      p_j0 = d.c0;
      p_c1 = d.c1;
      p_b = d.b;
      p_h = d.h;
      p_seek();
    }
    for (int i = 0; i < kDecStages - 1; ++i) p_issue();
  }

  int f = 0;  // steps consumed
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const DecItem d = dec_item(item, H, splits, L, kv_start, kv_len);
    // rotated, scaled query in the layout of the keys: pair k is dims
    // (2k, 2k+1), or (k, k+64) in the rotate-half layout
    __syncthreads();  // the previous item's readers of qs / racc are done
    if (t < kHeadDim / 2) {
      const __nv_bfloat16* qr = q + (int64_t(d.b) * H + d.h) * kHeadDim;
      const int i0 = half ? t : 2 * t;
      const int i1 = half ? t + kHeadDim / 2 : 2 * t + 1;
      const int pq = max(0, min(__ldg(q_pos + d.b), max_pos - 1));
      const float2 cs = table[int64_t(pq) * (kHeadDim / 2) + t];
      const float a = __bfloat162float(qr[i0]), c = __bfloat162float(qr[i1]);
      qs[i0] = (a * cs.x - c * cs.y) * scale_log2;
      qs[i1] = (a * cs.y + c * cs.x) * scale_log2;
    }
    __syncthreads();
    float qreg[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qreg[e] = qs[8 * l16 + e];
    float m = -INFINITY, l = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    for (int j0 = d.c0; j0 < d.c1; j0 += kDecRows, ++f) {
      const int s = f % kDecStages;
      bool ok = mbar_wait(bar(s), (f / kDecStages) & 1, nullptr, status,
                          kDecWaitNs);
      // every thread is past the previous step here: its stage and ps are
      // free, so the refill goes to that stage
      if (!__syncthreads_and(ok)) return;
      if (t == 0) p_issue();
      const uint8_t* kt = smem + s * 2 * kDecTile + hf * kDecHalf;
      const uint8_t* vt = kt + kDecTile;
      const int nk = min(kDecRows, d.c1 - j0);
      // scores: warp w takes rows 8 w .. 8 w + 7, two per pass
#pragma unroll
      for (int it = 0; it < kDecRows / kDecWarps / 2; ++it) {
        const int r = warp * (kDecRows / kDecWarps) + it * 2 + (lane >> 4);
        const uint4 w4 = dec_unit(kt, r, u);
        const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
        float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          d2 = fma2(make_float2(bf16lo_to_f32(ws[k]), bf16hi_to_f32(ws[k])),
                    make_float2(qreg[2 * k], qreg[2 * k + 1]), d2);
        float dd = d2.x + d2.y;
        dd += __shfl_xor_sync(0xffffffffu, dd, 8);
        dd += __shfl_xor_sync(0xffffffffu, dd, 4);
        dd += __shfl_xor_sync(0xffffffffu, dd, 2);
        dd += __shfl_xor_sync(0xffffffffu, dd, 1);
        if (l16 == 0) ps[r] = r < nk ? dd : -INFINITY;
      }
      __syncthreads();
      // every warp forms the step's max, probabilities and sum itself
      // (lane l holds keys l + 32 k), in the same order, so all agree
      float pk[4];
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pk[k] = ps[lane + 32 * k];
        mx = fmaxf(mx, pk[k]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m, mx);      // finite: the step has a key
      const float alpha = exp2f(m - m_new);  // m = -inf -> 0
      float sm = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pk[k] = exp2f(pk[k] - m_new);        // masked key -> 0
        sm += pk[k];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        sm += __shfl_xor_sync(0xffffffffu, sm, o);
      // values: row group g = t / 16 takes rows g + 32 k, whose
      // probabilities sit in lane g of every warp
      const int g = t >> 4;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
      for (int k = 0; k < kDecRows / kDecGroups; ++k) {
        const int r = g + kDecGroups * k;
        const float pr = __shfl_sync(0xffffffffu, pk[k], g & 31);
        if (r < nk) {
          const uint4 w4 = dec_unit(vt, r, u);
          const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a2 = fma2(
                make_float2(pr, pr),
                make_float2(bf16lo_to_f32(ws[e]), bf16hi_to_f32(ws[e])),
                make_float2(acc[2 * e], acc[2 * e + 1]));
            acc[2 * e] = a2.x;
            acc[2 * e + 1] = a2.y;
          }
        }
      }
      l = l * alpha + sm;
      m = m_new;
    }
    // sum the row groups' accumulators: group g, lane l16 holds dims
    // 8 l16 .. 8 l16 + 7
    {
      float4* dst = reinterpret_cast<float4*>(racc + (t >> 4) * kHeadDim +
                                              8 * l16);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    __syncthreads();
    if (t < kHeadDim) {
      float a = 0.f;
#pragma unroll
      for (int gg = 0; gg < kDecGroups; ++gg) a += racc[gg * kHeadDim + t];
      part_acc[d.slot * kHeadDim + t] = a;
    }
    if (t == 0) {
      part_m[d.slot] = m;
      part_l[d.slot] = l;
    }
  }
}

// out[b][h] = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M); lse likewise.
__global__ void __launch_bounds__(kHeadDim)
decode_combine_kernel(const float* __restrict__ part_m,
                      const float* __restrict__ part_l,
                      const float* __restrict__ part_acc, int H, int splits,
                      __nv_bfloat16* __restrict__ out,
                      float* __restrict__ lse) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int64_t base = (int64_t(b) * H + h) * splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part_m[base + s]);
  float L = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float w = exp2f(part_m[base + s] - M);
      L += part_l[base + s] * w;
      acc += part_acc[(base + s) * kHeadDim + t] * w;
    }
  }
  const int64_t o = (int64_t(b) * H + h);
  out[o * kHeadDim + t] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
  if (t == 0) lse[o] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace

int decode_splits(int L) {
  // about 8K keys per CTA, at least one split
  return std::max(1, (L + 8191) / 8192);
}

cudaError_t launch_decode(const void* q, const void* k_rot, const void* v,
                          const int32_t* kv_start, const int32_t* kv_len,
                          const int32_t* q_pos, const float* table,
                          int max_pos, int B, int L, int H, bool half,
                          void* out, float* lse, float* part_m, float* part_l,
                          float* part_acc, int* status, cudaStream_t st) {
  if (B == 0 || H == 0) return cudaSuccess;
  const int splits = decode_splits(L);
  const int n_items = B * H * splits;
  // an empty cache issues no load; the maps then only need valid shapes
  CUtensorMap mk, mv;
  if (!make_bnhd_map(&mk, k_rot, B, std::max(L, 1), H, kDecRows) ||
      !make_bnhd_map(&mv, v, B, std::max(L, 1), H, kDecRows))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(
      decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
      kDecSmem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_items, sm_count());
  {
    const cudaError_t le = launch_dependent(
        decode_split_kernel, dim3(grid), dim3(kDecThreads), kDecSmem, st, mk,
        mv, static_cast<const __nv_bfloat16*>(q), kv_start, kv_len, q_pos,
        reinterpret_cast<const float2*>(table), max_pos, L, H, splits, n_items,
        half, kLog2e / sqrtf(float(kHeadDim)), part_m, part_l, part_acc,
        status);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    const cudaError_t le = launch_dependent(
        decode_combine_kernel, dim3(H, B), dim3(kHeadDim), 0, st, part_m,
        part_l, part_acc, H, splits, static_cast<__nv_bfloat16*>(out), lse);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace lwm
