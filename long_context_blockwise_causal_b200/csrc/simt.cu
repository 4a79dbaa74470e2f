// CUDA-core blockwise attention with fp32 arithmetic (the fp32-I/O mode
// and the higher-precision backward). Same method as the tensor-core path:
// query blocks sweep key blocks from the diagonal down ("开源巨兽LWM：如何用
// RingAttention撬动百万Token多模态世界", 3.1), an online softmax keeps a
// running max / sum / accumulator (same page, 3.2), packing and causality
// mask every pair ("LWM：突破 100 万 Token 的开源大模型", 概述 (b)), and RoPE
// rotates q and k as they are loaded.
//
// Thread layout: 4 threads per row; thread `part` owns the 16 RoPE pairs
// k = 4*i + part (dims 2k, 2k+1; for q and k in the rotate-half layout the
// pair is dims k, k+64), so a pair never straddles threads and the 4
// threads of a row read 4 consecutive float2 of a shared-memory row
// (conflict free). Values, outputs and their gradients keep (2k, 2k+1).
#include "aux_kernels.cuh"

namespace lwm {
namespace {

constexpr int kRows = 64;     // query rows (forward) / key rows (backward)
constexpr int kKeys = 32;     // keys per step (forward)
constexpr int kQrows = 32;    // query rows per step (backward)
constexpr int kThreads = 256;
constexpr int kPairs = kHeadDim / 2;

template <typename T>
__device__ __forceinline__ float2 ld_pair(const T* p);
template <>
__device__ __forceinline__ float2 ld_pair<float>(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
template <>
__device__ __forceinline__ float2 ld_pair<__nv_bfloat16>(const __nv_bfloat16* p) {
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p);
  return __bfloat1622float2(v);
}
template <typename T>
__device__ __forceinline__ void st_pair(T* p, float a, float b);
template <>
__device__ __forceinline__ void st_pair<float>(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
template <>
__device__ __forceinline__ void st_pair<__nv_bfloat16>(__nv_bfloat16* p,
                                                       float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}

// RoPE pair k of a head row: (2k, 2k+1), or (k, k+64) in the rotate-half
// layout.
template <typename T>
__device__ __forceinline__ float2 ld_rpair(const T* row, int k, bool half) {
  if (!half) return ld_pair(row + 2 * k);
  return make_float2(float(row[k]), float(row[k + kHeadDim / 2]));
}
template <typename T>
__device__ __forceinline__ void st_rpair(T* row, int k, bool half, float a,
                                         float b) {
  if (!half) {
    st_pair(row + 2 * k, a, b);
  } else {
    row[k] = T(a);
    row[k + kHeadDim / 2] = T(b);
  }
}

__device__ __forceinline__ float2 rot(float2 x, float2 cs, float sign) {
  float s = sign * cs.y;
  return make_float2(x.x * cs.x - x.y * s, x.x * s + x.y * cs.x);
}

__device__ __forceinline__ float sum4(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                const T* __restrict__ v, const int32_t* __restrict__ seg,
                const int32_t* __restrict__ pos,
                const float2* __restrict__ table,
                const int32_t* __restrict__ kv_lo, int N, int H,
                bool half, float scale_log2, T* __restrict__ out,
                float* __restrict__ lse) {
  __shared__ float2 Ks[kKeys][kPairs];
  __shared__ float2 Vs[kKeys][kPairs];
  __shared__ int segk[kKeys];
  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * kRows;
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int i = q0 + row;
  const bool valid = i < N;
  const int64_t rowbase = int64_t(b) * N;
  const int seg_i = valid ? seg[rowbase + i] : -1;

  float2 qv[16];
  float2 acc[16];
  {
    int p = valid ? pos[rowbase + i] : 0;
    const T* qp = q + ((rowbase + (valid ? i : 0)) * H + h) * kHeadDim;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      int kk = 4 * e + part;
      float2 x = valid ? ld_rpair(qp, kk, half) : make_float2(0.f, 0.f);
      qv[e] = rot(x, table[int64_t(p) * kPairs + kk], 1.f);
      acc[e] = make_float2(0.f, 0.f);
    }
  }
  float m = -INFINITY, l = 0.f;
  const int Tq128 = (N + kBlock - 1) / kBlock;
  const int kbeg = kv_lo[b * Tq128 + q0 / kBlock] * kBlock;
  const int kend = min(q0 + kRows, N) - 1;  // last key any row can see
  const int first_step = kend / kKeys, last_step = kbeg / kKeys;
  for (int st = first_step; st >= last_step; --st) {
    const int k0 = st * kKeys;
    __syncthreads();
    for (int e = threadIdx.x; e < kKeys * kPairs; e += kThreads) {
      int key = e / kPairs, kk = e % kPairs, j = k0 + key;
      float2 kx = make_float2(0.f, 0.f), vx = kx;
      if (j < N) {
        int64_t off = ((rowbase + j) * H + h) * kHeadDim;
        kx = rot(ld_rpair(k + off, kk, half),
                 table[int64_t(pos[rowbase + j]) * kPairs + kk], 1.f);
        vx = ld_pair(v + off + 2 * kk);
      }
      Ks[key][kk] = kx;
      Vs[key][kk] = vx;
      if (kk == 0) segk[key] = j < N ? seg[rowbase + j] : -2;
    }
    __syncthreads();
    float s[kKeys];
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float2 kx = Ks[j][4 * e + part];
        d = fmaf(qv[e].x, kx.x, fmaf(qv[e].y, kx.y, d));
      }
      d = sum4(d) * scale_log2;
      bool ok = valid && segk[j] == seg_i && (k0 + j) <= i;
      s[j] = ok ? d : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    float m_new = fmaxf(m, mt);
    if (m_new == -INFINITY) continue;  // nothing allowed yet in this row
    float alpha = exp2f(m - m_new);    // m == -inf -> 0
    l *= alpha;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      acc[e].x *= alpha;
      acc[e].y *= alpha;
    }
#pragma unroll
    for (int j = 0; j < kKeys; ++j) {
      float p = exp2f(s[j] - m_new);
      l += p;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float2 vx = Vs[j][4 * e + part];
        acc[e].x = fmaf(p, vx.x, acc[e].x);
        acc[e].y = fmaf(p, vx.y, acc[e].y);
      }
    }
    m = m_new;
  }
  if (!valid) return;
  float inv = l > 0.f ? 1.f / l : 0.f;
  T* op = out + ((rowbase + i) * H + h) * kHeadDim;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    int kk = 4 * e + part;
    st_pair(op + 2 * kk, acc[e].x * inv, acc[e].y * inv);
  }
  if (part == 0) lse[(int64_t(b) * H + h) * N + i] = (m + log2f(l)) * kLn2;
}

// Key-major backward: a CTA owns 64 keys of one (b, h) and visits the
// query blocks that can see them (same segment run, not before the key).
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                const T* __restrict__ v, const T* __restrict__ dout,
                const float* __restrict__ lse, const float* __restrict__ delta,
                const int32_t* __restrict__ seg,
                const int32_t* __restrict__ pos,
                const float2* __restrict__ table, int N, int H, bool half,
                float scale_log2, float scale, float* __restrict__ dq_acc,
                T* __restrict__ dk, T* __restrict__ dv) {
  extern __shared__ float4 smem_f4[];
  float2(*Ks)[kPairs] = reinterpret_cast<float2(*)[kPairs]>(smem_f4);
  float2(*Qs)[kPairs] = Ks + kRows;
  float2(*Gs)[kPairs] = Qs + kQrows;  // dO
  float(*dS)[kRows + 1] = reinterpret_cast<float(*)[kRows + 1]>(Gs + kQrows);
  float* lse_s = &dS[kQrows][0];
  float* del_s = lse_s + kQrows;
  int* segq = reinterpret_cast<int*>(del_s + kQrows);

  const int b = blockIdx.z, h = blockIdx.y;
  const int k0 = blockIdx.x * kRows;
  const int key = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int j = k0 + key;
  const bool valid = j < N;
  const int64_t rowbase = int64_t(b) * N;
  const int seg_j = valid ? seg[rowbase + j] : -2;

  float2 kv[16], vv[16], gk[16], gv[16];
  {
    int p = valid ? pos[rowbase + j] : 0;
    int64_t off = ((rowbase + (valid ? j : 0)) * H + h) * kHeadDim;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      int kk = 4 * e + part;
      float2 x = valid ? ld_rpair(k + off, kk, half) : make_float2(0.f, 0.f);
      kv[e] = rot(x, table[int64_t(p) * kPairs + kk], 1.f);
      Ks[key][kk] = kv[e];
      vv[e] = valid ? ld_pair(v + off + 2 * kk) : make_float2(0.f, 0.f);
      gk[e] = make_float2(0.f, 0.f);
      gv[e] = gk[e];
    }
  }
  const int klast = min(k0 + kRows, N) - 1;
  const int seg_last = seg[rowbase + klast];
  const float* lse_bh = lse + (int64_t(b) * H + h) * N;
  const float* del_bh = delta + (int64_t(b) * H + h) * N;
  for (int i0 = (k0 / kQrows) * kQrows; i0 < N; i0 += kQrows) {
    if (seg[rowbase + i0] > seg_last) break;  // later rows see none of these keys
    __syncthreads();
    for (int e = threadIdx.x; e < kQrows * kPairs; e += kThreads) {
      int r = e / kPairs, kk = e % kPairs, i = i0 + r;
      float2 qx = make_float2(0.f, 0.f), gx = qx;
      if (i < N) {
        int64_t off = ((rowbase + i) * H + h) * kHeadDim;
        qx = rot(ld_rpair(q + off, kk, half),
                 table[int64_t(pos[rowbase + i]) * kPairs + kk], 1.f);
        gx = ld_pair(dout + off + 2 * kk);
      }
      Qs[r][kk] = qx;
      Gs[r][kk] = gx;
      if (kk == 0) {
        segq[r] = i < N ? seg[rowbase + i] : -1;
        lse_s[r] = i < N ? lse_bh[i] * kLog2e : 0.f;
        del_s[r] = i < N ? del_bh[i] : 0.f;
      }
    }
    __syncthreads();
    for (int r = 0; r < kQrows; ++r) {
      const int i = i0 + r;
      float sd = 0.f, dpd = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float2 qx = Qs[r][4 * e + part];
        float2 gx = Gs[r][4 * e + part];
        sd = fmaf(kv[e].x, qx.x, fmaf(kv[e].y, qx.y, sd));
        dpd = fmaf(vv[e].x, gx.x, fmaf(vv[e].y, gx.y, dpd));
      }
      sd = sum4(sd);
      dpd = sum4(dpd);
      bool ok = valid && segq[r] == seg_j && j <= i && i < N;
      float p = ok ? exp2f(sd * scale_log2 - lse_s[r]) : 0.f;
      float ds = p * (dpd - del_s[r]);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float2 qx = Qs[r][4 * e + part];
        float2 gx = Gs[r][4 * e + part];
        gv[e].x = fmaf(p, gx.x, gv[e].x);
        gv[e].y = fmaf(p, gx.y, gv[e].y);
        gk[e].x = fmaf(ds, qx.x, gk[e].x);
        gk[e].y = fmaf(ds, qx.y, gk[e].y);
      }
      if (part == 0) dS[r][key] = ds;
    }
    __syncthreads();
    // dq~[i] += sum_j dS[i][j] k~_j (scale applied in the conversion)
    {
      const int r = threadIdx.x >> 3;           // 32 rows
      const int c = (threadIdx.x & 7) * 8;      // 8 pairs each
      const int i = i0 + r;
      if (i < N) {
        float2 a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = make_float2(0.f, 0.f);
        for (int kk = 0; kk < kRows; ++kk) {
          float w = dS[r][kk];
          if (w == 0.f) continue;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float2 kx = Ks[kk][c + e];
            a[e].x = fmaf(w, kx.x, a[e].x);
            a[e].y = fmaf(w, kx.y, a[e].y);
          }
        }
        // dq~ pairs in the layout q came in (converted by dq_convert)
        float* dst = dq_acc + ((rowbase + i) * H + h) * kHeadDim;
        const int second = half ? kHeadDim / 2 : 1;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (a[e].x != 0.f || a[e].y != 0.f) {
            const int first = half ? c + e : 2 * (c + e);
            atomicAdd(dst + first, a[e].x);
            atomicAdd(dst + first + second, a[e].y);
          }
        }
      }
    }
  }
  if (!valid) return;
  int p = pos[rowbase + j];
  int64_t off = ((rowbase + j) * H + h) * kHeadDim;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    int kk = 4 * e + part;
    float2 g = make_float2(gk[e].x * scale, gk[e].y * scale);
    float2 r = rot(g, table[int64_t(p) * kPairs + kk], -1.f);
    st_rpair(dk + off, kk, half, r.x, r.y);
    st_pair(dv + off + 2 * kk, gv[e].x, gv[e].y);
  }
}

constexpr size_t bwd_smem_bytes() {
  return sizeof(float2) * kPairs * (kRows + 2 * kQrows) +
         sizeof(float) * (kQrows * (kRows + 1) + 2 * kQrows) +
         sizeof(int) * kQrows;
}

}  // namespace

template <typename T>
cudaError_t launch_fwd_simt(const T* q, const T* k, const T* v,
                            const int32_t* seg, const int32_t* pos,
                            const float* table, const int32_t* kv_lo, int B,
                            int N, int H, bool half, T* out, float* lse,
                            cudaStream_t st) {
  if (B == 0 || N == 0 || H == 0) return cudaSuccess;
  dim3 grid((N + kRows - 1) / kRows, H, B);
  float scale_log2 = kLog2e / sqrtf(float(kHeadDim));
  fwd_simt_kernel<T><<<grid, kThreads, 0, st>>>(
      q, k, v, seg, pos, reinterpret_cast<const float2*>(table), kv_lo, N, H,
      half, scale_log2, out, lse);
  note_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_simt(const T* q, const T* k, const T* v, const T* dout,
                            const float* lse, const float* delta,
                            const int32_t* seg, const int32_t* pos,
                            const float* table, int B, int N, int H,
                            bool half, float* dq_acc, T* dk, T* dv,
                            cudaStream_t st) {
  if (B == 0 || N == 0 || H == 0) return cudaSuccess;
  size_t smem = bwd_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(
      bwd_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((N + kRows - 1) / kRows, H, B);
  float scale = 1.f / sqrtf(float(kHeadDim));
  bwd_simt_kernel<T><<<grid, kThreads, smem, st>>>(
      q, k, v, dout, lse, delta, seg, pos,
      reinterpret_cast<const float2*>(table), N, H, half, kLog2e * scale,
      scale, dq_acc, dk, dv);
  note_launch();
  return cudaGetLastError();
}

template cudaError_t launch_fwd_simt<float>(const float*, const float*,
                                            const float*, const int32_t*,
                                            const int32_t*, const float*,
                                            const int32_t*, int, int, int,
                                            bool, float*, float*,
                                            cudaStream_t);
template cudaError_t launch_fwd_simt<__nv_bfloat16>(
    const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
    const int32_t*, const int32_t*, const float*, const int32_t*, int, int,
    int, bool, __nv_bfloat16*, float*, cudaStream_t);
template cudaError_t launch_bwd_simt<float>(const float*, const float*,
                                            const float*, const float*,
                                            const float*, const float*,
                                            const int32_t*, const int32_t*,
                                            const float*, int, int, int,
                                            bool, float*, float*, float*,
                                            cudaStream_t);
template cudaError_t launch_bwd_simt<__nv_bfloat16>(
    const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
    const __nv_bfloat16*, const float*, const float*, const int32_t*,
    const int32_t*, const float*, int, int, int, bool, float*,
    __nv_bfloat16*, __nv_bfloat16*, cudaStream_t);

}  // namespace lwm
