// Decode attention: one new query token per (batch row, head) against a
// long cache of rotated keys and values (the inference side of the 1M-token
// models, "LWM：突破 100 万 Token 的开源大模型", 概述 / 脚本运行说明; the
// single-needle retrieval over 1M tokens in "[论文解读] World Model on
// Million-Length Video And Language With Blockwise RingAttention", 主要发现).
//
// The query of row b is the cache's last token; under masked packing it
// sees the keys [kv_start[b], kv_len[b]) of its own example (causality is
// automatic: no cached key lies after it). Split-KV: a CTA of 128 threads
// streams a chunk of keys of one (b, h) with an online softmax and writes a
// partial (max, sum, 128-wide accumulator); a second kernel merges the
// partials of a (b, h) into out and lse. The pass reads every visible key
// and value row once (2 x 256 bytes per key): it is bound by HBM bandwidth.
#include "aux_kernels.cuh"
#include "decode.cuh"

namespace lwm {
namespace {

constexpr int kDecThreads = 128;   // one key per thread per step; one dim
                                   // of the accumulator per thread
constexpr int kDecStep = 128;      // keys per step

__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(const __nv_bfloat16* __restrict__ q,
                    const __nv_bfloat16* __restrict__ k_rot,
                    const __nv_bfloat16* __restrict__ v,
                    const int32_t* __restrict__ kv_start,
                    const int32_t* __restrict__ kv_len,
                    const int32_t* __restrict__ q_pos,
                    const float2* __restrict__ table, int max_pos, int L,
                    int H, int splits, bool half, float scale_log2,
                    float* __restrict__ part_m, float* __restrict__ part_l,
                    float* __restrict__ part_acc) {
  __shared__ float qs[kHeadDim];
  __shared__ float ps[kDecStep];
  __shared__ float red[kDecThreads / 32];
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  // out-of-range inputs are clamped so no read leaves the cache
  const int len = max(0, min(kv_len[b], L));
  const int start = max(0, min(kv_start[b], len));
  const int chunk = (len - start + splits - 1) / splits;
  const int c0 = start + split * chunk;
  const int c1 = min(c0 + chunk, len);
  const int64_t slot = (int64_t(b) * H + h) * splits + split;
  // rotated query, fp32, in shared memory, in the layout of the keys: pair
  // t is dims (2t, 2t+1), or (t, t+64) in the rotate-half layout
  if (t < kHeadDim / 2) {
    const __nv_bfloat16* qr = q + (int64_t(b) * H + h) * kHeadDim;
    const int i0 = half ? t : 2 * t, i1 = half ? t + kHeadDim / 2 : 2 * t + 1;
    const int pq = max(0, min(q_pos[b], max_pos - 1));
    const float2 cs = table[int64_t(pq) * (kHeadDim / 2) + t];
    const float a = __bfloat162float(qr[i0]), c = __bfloat162float(qr[i1]);
    qs[i0] = (a * cs.x - c * cs.y) * scale_log2;
    qs[i1] = (a * cs.y + c * cs.x) * scale_log2;
  }
  __syncthreads();
  float m = -INFINITY, l = 0.f, acc = 0.f;
  const int64_t row_stride = int64_t(H) * kHeadDim;  // elements per token
  const __nv_bfloat16* kb = k_rot + (int64_t(b) * L * H + h) * kHeadDim;
  const __nv_bfloat16* vb = v + (int64_t(b) * L * H + h) * kHeadDim;
  for (int j0 = c0; j0 < c1; j0 += kDecStep) {
    // score of key j0 + t: its 256-byte row as 16 x 16-byte loads
    const int j = j0 + t;
    float s = -INFINITY;
    if (j < c1) {
      const uint4* kr = reinterpret_cast<const uint4*>(kb + j * row_stride);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint4 w = __ldg(kr + e);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          d0 = fmaf(bf16lo_to_f32(ws[u]), qs[8 * e + 2 * u], d0);
          d1 = fmaf(bf16hi_to_f32(ws[u]), qs[8 * e + 2 * u + 1], d1);
        }
      }
      s = d0 + d1;
    }
    // step max across the CTA
    float mx = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(~0u, mx, o));
    if (lane == 0) red[wid] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float m_new = fmaxf(m, mx);
    const float alpha = exp2f(m - m_new);  // m = -inf -> 0
    const float pj = exp2f(s - m_new);     // s = -inf -> 0
    ps[t] = pj;
    __syncthreads();
    // thread t accumulates dim t over the step's keys (coalesced rows)
    float sum = 0.f, a2 = 0.f;
    const int nk = min(kDecStep, c1 - j0);
    const __nv_bfloat16* vr = vb + int64_t(j0) * row_stride + t;
    for (int jj = 0; jj < nk; ++jj) {
      const float p = ps[jj];
      sum += p;
      a2 = fmaf(p, __bfloat162float(vr[jj * row_stride]), a2);
    }
    acc = acc * alpha + a2;
    l = l * alpha + sum;
    m = m_new;
    __syncthreads();
  }
  part_acc[slot * kHeadDim + t] = acc;
  if (t == 0) {
    part_m[slot] = m;
    part_l[slot] = l;
  }
}

// out[b][h] = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M); lse likewise.
__global__ void __launch_bounds__(kHeadDim)
decode_combine_kernel(const float* __restrict__ part_m,
                      const float* __restrict__ part_l,
                      const float* __restrict__ part_acc, int H, int splits,
                      __nv_bfloat16* __restrict__ out,
                      float* __restrict__ lse) {
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
                          float* part_acc, cudaStream_t st) {
  if (B == 0 || H == 0) return cudaSuccess;
  const int splits = decode_splits(L);
  dim3 grid(splits, H, B);
  decode_split_kernel<<<grid, kDecThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k_rot),
      static_cast<const __nv_bfloat16*>(v), kv_start, kv_len, q_pos,
      reinterpret_cast<const float2*>(table), max_pos, L, H, splits, half,
      kLog2e / sqrtf(float(kHeadDim)), part_m, part_l, part_acc);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(H, B), kHeadDim, 0, st>>>(
      part_m, part_l, part_acc, H, splits,
      static_cast<__nv_bfloat16*>(out), lse);
  note_launch();
  return cudaGetLastError();
}

}  // namespace lwm
