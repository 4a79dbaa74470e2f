// Auxiliary kernels of the blockwise attention path: RoPE table, tile
// classification and block metadata, the longest-first work order, the
// precondition check, the backward preprocess and the dQ conversion.
#include "aux_kernels.cuh"

namespace lwm {

// table[p][k] = (cos a, sin a), a = p * theta^(-2k/D) in fp64 ("[论文解读]
// World Model on Million-Length Video And Language With Blockwise
// RingAttention", 提出的方法: RoPE with a context-scaled theta).
__global__ void rope_table_kernel(double theta, int half_d, int max_pos,
                                  float2* __restrict__ table) {
  pdl_wait();
  pdl_trigger();
  int64_t n = int64_t(max_pos) * half_d;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x) {
    int p = int(e / half_d);
    int k = int(e - int64_t(p) * half_d);
    double inv_freq = pow(theta, -2.0 * double(k) / double(2 * half_d));
    double a = double(p) * inv_freq;
    double s, c;
    sincos(a, &s, &c);
    table[e] = make_float2(float(c), float(s));
  }
}

// hi = R(pos) x rounded to bf16 (RNE); lo (when given) = the bf16 rounding
// of what hi misses, so hi + lo carries the rotated value to ~2^-16. One
// thread per 16-byte chunk (4 interleaved pairs) of a [B][N][H][D] tensor.
__global__ void rope_apply_kernel(const __nv_bfloat16* __restrict__ x,
                                  const int32_t* __restrict__ pos,
                                  const float2* __restrict__ table,
                                  int64_t chunks, int H,
                                  __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo) {
  pdl_wait();
  pdl_trigger();
  constexpr int kChunksPerRow = kHeadDim / 8;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
       e < chunks; e += int64_t(gridDim.x) * blockDim.x) {
    const int c = int(e % kChunksPerRow);
    const int64_t bn = (e / kChunksPerRow) / H;
    const int p = pos[bn];
    const float4* t = reinterpret_cast<const float4*>(
        table + int64_t(p) * (kHeadDim / 2) + c * 4);
    const float4 cs01 = __ldg(t), cs23 = __ldg(t + 1);
    const uint4 w = reinterpret_cast<const uint4*>(x)[e];
    const float cc[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
    const float ss[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t h[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = bf16lo_to_f32(ws[k]), b = bf16hi_to_f32(ws[k]);
      const float ra = fmaf(a, cc[k], -b * ss[k]);
      const float rb = fmaf(a, ss[k], b * cc[k]);
      h[k] = pack_bf16x2(ra, rb);
      l[k] = pack_bf16x2(ra - bf16lo_to_f32(h[k]), rb - bf16hi_to_f32(h[k]));
    }
    reinterpret_cast<uint4*>(hi)[e] = make_uint4(h[0], h[1], h[2], h[3]);
    if (lo) reinterpret_cast<uint4*>(lo)[e] = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

// Same for the rotate-half layout: pair k = (x[k], x[k + 64]). Item c of a
// row rotates dims 8c .. 8c+7 with dims 64 + 8c .. 64 + 8c + 7
// (frequencies 8c .. 8c+7) and writes them back in that layout.
__global__ void rope_apply_half_kernel(const __nv_bfloat16* __restrict__ x,
                                       const int32_t* __restrict__ pos,
                                       const float2* __restrict__ table,
                                       int64_t items, int H,
                                       __nv_bfloat16* __restrict__ hi,
                                       __nv_bfloat16* __restrict__ lo) {
  pdl_wait();
  pdl_trigger();
  constexpr int kItemsPerRow = kHeadDim / 16;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
       e < items; e += int64_t(gridDim.x) * blockDim.x) {
    const int c = int(e % kItemsPerRow);
    const int64_t row = e / kItemsPerRow;  // (b, n, h)
    const int p = pos[row / H];
    const float4* t = reinterpret_cast<const float4*>(
        table + int64_t(p) * (kHeadDim / 2) + c * 8);
    const int64_t i0 = row * (kHeadDim / 8) + c;   // uint4 index, first half
    const int64_t i1 = i0 + kHeadDim / 16;         // second half
    const uint4 wa = reinterpret_cast<const uint4*>(x)[i0];
    const uint4 wb = reinterpret_cast<const uint4*>(x)[i1];
    const uint32_t as[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t bs[4] = {wb.x, wb.y, wb.z, wb.w};
    uint32_t ha[4], hb[4], la[4], lb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 cs = __ldg(t + k);  // pairs 8c + 2k, 8c + 2k + 1
      const float a0 = bf16lo_to_f32(as[k]), a1 = bf16hi_to_f32(as[k]);
      const float b0 = bf16lo_to_f32(bs[k]), b1 = bf16hi_to_f32(bs[k]);
      const float ra0 = fmaf(a0, cs.x, -b0 * cs.y);
      const float rb0 = fmaf(a0, cs.y, b0 * cs.x);
      const float ra1 = fmaf(a1, cs.z, -b1 * cs.w);
      const float rb1 = fmaf(a1, cs.w, b1 * cs.z);
      ha[k] = pack_bf16x2(ra0, ra1);
      hb[k] = pack_bf16x2(rb0, rb1);
      la[k] = pack_bf16x2(ra0 - bf16lo_to_f32(ha[k]), ra1 - bf16hi_to_f32(ha[k]));
      lb[k] = pack_bf16x2(rb0 - bf16lo_to_f32(hb[k]), rb1 - bf16hi_to_f32(hb[k]));
    }
    reinterpret_cast<uint4*>(hi)[i0] = make_uint4(ha[0], ha[1], ha[2], ha[3]);
    reinterpret_cast<uint4*>(hi)[i1] = make_uint4(hb[0], hb[1], hb[2], hb[3]);
    if (lo) {
      reinterpret_cast<uint4*>(lo)[i0] = make_uint4(la[0], la[1], la[2], la[3]);
      reinterpret_cast<uint4*>(lo)[i1] = make_uint4(lb[0], lb[1], lb[2], lb[3]);
    }
  }
}

// First index of the contiguous run holding row i (ids non-decreasing).
__device__ __forceinline__ int run_start(const int32_t* __restrict__ seg,
                                         int i) {
  int v = seg[i];
  int lo = 0, hi = i;  // answer in [0, i]
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (seg[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// rs[b][i] = first index of the packed example holding row i. With
// non-decreasing ids, "seg_j == seg_i and j <= i" is "rs[i] <= j <= i".
// re[b][i] = last index of that example, so key k is seen by rows
// k .. re[k].
__global__ void row_start_kernel(const int32_t* __restrict__ seg, int B, int N,
                                 int32_t* __restrict__ rs,
                                 int32_t* __restrict__ re) {
  int64_t total = int64_t(B) * N;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    int b = int(e / N);
    int i = int(e - int64_t(b) * N);
    const int32_t* s = seg + int64_t(b) * N;
    rs[e] = run_start(s, i);
    if (re) {
      int v = s[i], lo = i, hi = N - 1;  // last index with s == v
      while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (s[mid] > v) hi = mid - 1; else lo = mid;
      }
      re[e] = lo;
    }
  }
}

// Visible key range of each query row against a block of keys, in global
// token indices: row i (global q_off + ii) sees the keys of the block whose
// segment id equals its own and whose index is <= i. With non-decreasing
// ids those keys are contiguous: [row_lo, row_hi] (empty when lo > hi).
// Range summary of one 128-row block (query rows or keys): mn / mx: union
// of the non-empty ranges; lmax / hmin: their intersection; all: every
// entry exists and is non-empty.
struct RangeFold {
  int mn, mx, lmax, hmin;
  bool all;
  __device__ __forceinline__ void add(int lo, int hi) {
    if (lo > hi) { all = false; return; }
    mn = min(mn, lo);
    mx = max(mx, hi);
    lmax = max(lmax, lo);
    hmin = min(hmin, hi);
  }
  __device__ __forceinline__ void merge(const RangeFold& o) {
    mn = min(mn, o.mn);
    mx = max(mx, o.mx);
    lmax = max(lmax, o.lmax);
    hmin = min(hmin, o.hmin);
    all = all && o.all;
  }
  __device__ __forceinline__ void warp_reduce() {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
      hmin = min(hmin, __shfl_xor_sync(0xffffffffu, hmin, o));
    }
    all = __all_sync(0xffffffffu, all);
  }
};

// Per query row i (global q_off + ii): the visible keys are those of its
// segment up to the row itself, as a global index range [row_lo, row_hi]
// (empty when lo > hi); and per query block t (one CTA of 128 threads, a
// thread per row): the key blocks [kv_lo, kv_hi] (block-local) holding any
// visible key (empty: lo = 1, hi = 0), and the tightest row range the
// block shares (lo_max, hi_min; lo_max = INT_MAX if some row is past Nq or
// sees nothing) for the all-visible test of a key block.
__global__ void __launch_bounds__(kBlock)
cross_meta_kernel(const int32_t* __restrict__ seg_q,
                  const int32_t* __restrict__ seg_k, int B, int Nq, int Nk,
                  int q_off, int k_off, int bk, int Tq,
                  int32_t* __restrict__ row_lo, int32_t* __restrict__ row_hi,
                  int32_t* __restrict__ kv_lo, int32_t* __restrict__ kv_hi,
                  int32_t* __restrict__ lo_max, int32_t* __restrict__ hi_min) {
  pdl_wait();
  pdl_trigger();
  __shared__ RangeFold part[kBlock / 32];
  const int e = blockIdx.x;
  const int b = e / Tq, t = e - b * Tq;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ii = t * kBlock + threadIdx.x;
  RangeFold f{0x7fffffff, -1, -0x7fffffff, 0x7fffffff, true};
  if (ii < Nq) {
    const int32_t* sk = seg_k + int64_t(b) * Nk;
    const int v = seg_q[int64_t(b) * Nq + ii];
    int a = 0, z = Nk;  // first key with seg >= v
    while (a < z) { int m = (a + z) >> 1; if (sk[m] < v) a = m + 1; else z = m; }
    const int first = a;
    z = Nk;             // first key with seg > v
    while (a < z) { int m = (a + z) >> 1; if (sk[m] <= v) a = m + 1; else z = m; }
    const int lo = k_off + first;
    const int hi = min(k_off + a - 1, q_off + ii);
    row_lo[int64_t(b) * Nq + ii] = lo;
    row_hi[int64_t(b) * Nq + ii] = hi;
    f.add(lo, hi);
  } else {
    f.all = false;
  }
  f.warp_reduce();
  if (lane == 0) part[warp] = f;
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int w = 1; w < kBlock / 32; ++w) f.merge(part[w]);
  if (f.mx < 0 || f.mn > f.mx) {
    kv_lo[e] = 1;
    kv_hi[e] = 0;
  } else {
    kv_lo[e] = (f.mn - k_off) / bk;
    kv_hi[e] = min((f.mx - k_off) / bk, (Nk - 1) / bk);
  }
  lo_max[e] = f.all ? f.lmax : 0x7fffffff;
  hi_min[e] = f.all ? f.hmin : -0x7fffffff;
}

// Key-side view of the same rule, for the key-major backward: key k
// (global k_off + jj) is seen by the queries [col_lo, col_hi] (global
// indices, empty when lo > hi): those of its segment from k on. Per key
// block j (one CTA of 128 threads, a thread per key): the query blocks
// [q_lo, q_hi] (chunk-local) holding a query that sees one of its keys
// (none: lo = 1, hi = 0), and the tightest shared query range (klo_max,
// khi_min; klo_max = INT_MAX if some key is past Nk or seen by nobody) for
// the all-visible test of a query block.
__global__ void __launch_bounds__(kBlock)
cross_keys_kernel(const int32_t* __restrict__ seg_q,
                  const int32_t* __restrict__ seg_k, int B, int Nq, int Nk,
                  int q_off, int k_off, int Tk, int32_t* __restrict__ col_lo,
                  int32_t* __restrict__ col_hi, int32_t* __restrict__ q_lo,
                  int32_t* __restrict__ q_hi, int32_t* __restrict__ klo_max,
                  int32_t* __restrict__ khi_min) {
  pdl_wait();
  pdl_trigger();
  __shared__ RangeFold part[kBlock / 32];
  const int e = blockIdx.x;
  const int b = e / Tk, j = e - b * Tk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int jj = j * kBlock + threadIdx.x;
  RangeFold f{0x7fffffff, -1, -0x7fffffff, 0x7fffffff, true};
  if (jj < Nk) {
    const int32_t* sq = seg_q + int64_t(b) * Nq;
    const int v = seg_k[int64_t(b) * Nk + jj];
    int a = 0, z = Nq;  // first query with seg >= v
    while (a < z) { int m = (a + z) >> 1; if (sq[m] < v) a = m + 1; else z = m; }
    const int first = a;
    z = Nq;             // first query with seg > v
    while (a < z) { int m = (a + z) >> 1; if (sq[m] <= v) a = m + 1; else z = m; }
    const int lo = max(q_off + first, k_off + jj);
    const int hi = q_off + a - 1;
    col_lo[int64_t(b) * Nk + jj] = lo;
    col_hi[int64_t(b) * Nk + jj] = hi;
    f.add(lo, hi);
  } else {
    f.all = false;
  }
  f.warp_reduce();
  if (lane == 0) part[warp] = f;
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int w = 1; w < kBlock / 32; ++w) f.merge(part[w]);
  if (f.mx < 0 || f.mn > f.mx) {
    q_lo[e] = 1;
    q_hi[e] = 0;
  } else {
    q_lo[e] = (f.mn - q_off) / kBlock;
    q_hi[e] = min((f.mx - q_off) / kBlock, (Nq - 1) / kBlock);
  }
  klo_max[e] = f.all ? f.lmax : 0x7fffffff;
  khi_min[e] = f.all ? f.hmin : -0x7fffffff;
}

// out, lse <- the softmax-weighted combination of (out, lse) and
// (out_part, lse_part) over disjoint key sets: with M = max(lse, lse_p),
// w = e^(lse - M), w_p = e^(lse_p - M): out = (w out + w_p out_p)/(w + w_p),
// lse = M + log(w + w_p). Rows where both are -inf stay (0, -inf).
// Sixteen lanes own one (b, n, h) row (16 bytes each); the lse of a row is
// read by all of them before lane 0 of the group overwrites it.
__global__ void merge_kernel(__nv_bfloat16* __restrict__ out,
                             float* __restrict__ lse,
                             const __nv_bfloat16* __restrict__ out_p,
                             const float* __restrict__ lse_p, int B, int N,
                             int H) {
  pdl_wait();
  pdl_trigger();
  constexpr int kLanesPerRow = kHeadDim / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const int64_t rows = int64_t(B) * N * H;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r0 = warp * kRowsPerWarp; r0 < rows; r0 += warps * kRowsPerWarp) {
    const int64_t row = r0 + lane / kLanesPerRow;  // (b, n, h)
    const bool ok = row < rows;
    int64_t li = 0;
    float l1 = -INFINITY, l2 = -INFINITY;
    if (ok) {
      const int h = int(row % H);
      const int64_t bn = row / H;
      const int n = int(bn % N);
      const int b = int(bn / N);
      li = (int64_t(b) * H + h) * N + n;
      l1 = lse[li];
      l2 = lse_p[li];
    }
    __syncwarp();
    if (!ok) continue;
    const float M = fmaxf(l1, l2);
    float w1 = 0.f, w2 = 0.f;
    if (M != -INFINITY) {
      w1 = __expf(l1 - M);
      w2 = __expf(l2 - M);
    }
    const float den = w1 + w2;
    const float a = den > 0.f ? w1 / den : 0.f, c = den > 0.f ? w2 / den : 0.f;
    const int64_t e = row * kLanesPerRow + (lane % kLanesPerRow);
    uint4 x = reinterpret_cast<const uint4*>(out)[e];
    const uint4 y = reinterpret_cast<const uint4*>(out_p)[e];
    uint32_t* xs = reinterpret_cast<uint32_t*>(&x);
    const uint32_t* ys = reinterpret_cast<const uint32_t*>(&y);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      xs[k] = pack_bf16x2(a * bf16lo_to_f32(xs[k]) + c * bf16lo_to_f32(ys[k]),
                          a * bf16hi_to_f32(xs[k]) + c * bf16hi_to_f32(ys[k]));
    reinterpret_cast<uint4*>(out)[e] = x;
    if (lane % kLanesPerRow == 0)
      lse[li] = den > 0.f ? M + __logf(den) : -INFINITY;
  }
}

__global__ void fill_kernel(float* __restrict__ x, float v, int64_t n) {
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x)
    x[e] = v;
}

__global__ void block_meta_kernel(const int32_t* __restrict__ seg, int B,
                                  int N, int bq, int bk, int Tq,
                                  int32_t* __restrict__ kv_lo,
                                  int32_t* __restrict__ kv_hi) {
  int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= B * Tq) return;
  int b = e / Tq, t = e - b * Tq;
  const int32_t* s = seg + int64_t(b) * N;
  int qs = t * bq;
  int qe = min(qs + bq, N) - 1;
  kv_lo[e] = run_start(s, qs) / bk;
  kv_hi[e] = qe / bk;
}

__global__ void tile_class_kernel(const int32_t* __restrict__ seg, int B,
                                  int N, int bq, int bk, int Tq, int Tk,
                                  const int32_t* __restrict__ kv_lo,
                                  const int32_t* __restrict__ kv_hi,
                                  uint8_t* __restrict__ cls) {
  int64_t total = int64_t(B) * Tq * Tk;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
       e < total; e += int64_t(gridDim.x) * blockDim.x) {
    int j = int(e % Tk);
    int64_t bt = e / Tk;
    int t = int(bt % Tq);
    int b = int(bt / Tq);
    uint8_t c = LWM_TILE_EMPTY;
    if (j >= kv_lo[bt] && j <= kv_hi[bt]) {
      const int32_t* s = seg + int64_t(b) * N;
      int qs = t * bq, qe = qs + bq - 1;
      int ks = j * bk, ke = ks + bk - 1;
      bool full = ke < qs && qe < N && s[ks] == s[qe];
      c = full ? LWM_TILE_FULL : LWM_TILE_PARTIAL;
    }
    cls[e] = c;
  }
}

// Key-block view for the backward: query blocks that see key block j form
// the contiguous range [q_lo, q_hi] (kv_lo and kv_hi are non-decreasing).
__global__ void kv_meta_kernel(int B, int Tq, int Tk,
                               const int32_t* __restrict__ kv_lo,
                               const int32_t* __restrict__ kv_hi,
                               int32_t* __restrict__ q_lo,
                               int32_t* __restrict__ q_hi) {
  int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= B * Tk) return;
  int b = e / Tk, j = e - b * Tk;
  const int32_t* lo = kv_lo + int64_t(b) * Tq;
  const int32_t* hi = kv_hi + int64_t(b) * Tq;
  // first t with hi[t] >= j
  int a = 0, z = Tq;
  while (a < z) { int m = (a + z) >> 1; if (hi[m] < j) a = m + 1; else z = m; }
  int first = a;
  // last t with lo[t] <= j
  a = 0; z = Tq;
  while (a < z) { int m = (a + z) >> 1; if (lo[m] <= j) a = m + 1; else z = m; }
  int last = a - 1;
  q_lo[e] = first;
  q_hi[e] = last;
}

// Longest-first order: one CTA forms the sort key of every unit (b, u)
// (units are groups of `group` blocks of the outer dimension whose inner
// ranges [lo, hi] are unioned; key = descending cost, then ascending unit
// id) and bitonic-sorts up to kSortMax keys in shared memory; the sorted
// unit ids are written to order[].
__global__ void __launch_bounds__(1024)
lpt_sort_kernel(int B, int T, int group, const int32_t* __restrict__ lo,
                const int32_t* __restrict__ hi, int U, int anchor,
                int32_t* __restrict__ order, int32_t* __restrict__ counter) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint64_t sk[];
  if (threadIdx.x == 0) *counter = 0;  // work counter of the next launch
  const int n = B * U;
  int p2 = 1;
  while (p2 < n) p2 <<= 1;
  for (int i = threadIdx.x; i < p2; i += blockDim.x) {
    uint64_t key = ~0ull;
    if (i < n) {
      const int b = i / U, u = i - b * U;
      const int t0 = u * group, t1 = min(t0 + group, T) - 1;
      int l = 0x7fffffff, h = -1;
      for (int t = t0; t <= t1; ++t) {
        const int tl = lo[b * T + t], th = hi[b * T + t];
        if (tl > th) continue;  // no visible block
        l = min(l, tl);
        h = max(h, th);
      }
      const int cost = min(h >= l ? h - l + 1 : 0, 16383);
      // packed examples one after another (units of one example share
      // their range's start, or its end for the key-major backward), so
      // the SMs work inside one or two examples at a time and their
      // inputs stay in L2; longest first within an example
      const int a = anchor == 0 ? 0 : (anchor == 1 ? l : h);
      const uint64_t loc =
          h >= l ? uint64_t(b) * uint64_t(T) + uint64_t(max(a, 0)) : 0;
      // key: example (26 bits) | 16383 - cost (14 bits) | unit id (24 bits;
      // n <= kSortMax), so ascending order is example, then longest first
      key = (loc << 38) | (uint64_t(16383 - cost) << 24) | uint32_t(i);
    }
    sk[i] = key;
  }
  __syncthreads();
  for (int size = 2; size <= p2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < p2; i += blockDim.x) {
        int j = i ^ stride;
        if (j > i) {
          bool up = (i & size) == 0;
          uint64_t a = sk[i], c = sk[j];
          if ((a > c) == up) { sk[i] = c; sk[j] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    order[i] = int32_t(sk[i] & 0xFFFFFFu);  // the unit id: the key's low 24 bits
}

// Fallback order for more units than one CTA can sort: per batch row, the
// units from last to first (longest first for a causal row).
__global__ void reverse_order_kernel(int B, int U, int32_t* __restrict__ order,
                                     int32_t* __restrict__ counter) {
  pdl_wait();
  pdl_trigger();
  int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e == 0) *counter = 0;
  if (e >= B * U) return;
  int b = e / U, u = e - b * U;
  order[e] = b * U + (U - 1 - u);
}

__global__ void check_inputs_kernel(const int32_t* __restrict__ seg,
                                    const int32_t* __restrict__ pos, int B,
                                    int N, int max_pos, int* __restrict__ res) {
  int64_t total = int64_t(B) * N;
  int bad = 0, mx = -1;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
       e < total; e += int64_t(gridDim.x) * blockDim.x) {
    int i = int(e % N);
    int p = pos[e];
    if (p < 0 || p >= max_pos) bad |= 2;
    mx = max(mx, p);
    if (i + 1 < N && seg[e + 1] < seg[e]) bad |= 1;
  }
  if (bad) atomicOr(&res[0], bad);
  atomicMax(&res[1], mx);
}

// D_i = sum_d dO_i[d] * O_i[d] (fp32), stored [B][H][N]; one warp per row.
template <typename T>
__global__ void bwd_delta_kernel(const T* __restrict__ out,
                                 const T* __restrict__ dout, int B, int N,
                                 int H, float* __restrict__ delta) {
  pdl_wait();
  pdl_trigger();
  // 16-byte loads: a row of 128 elements is 16 (bf16) or 32 (fp32) lanes,
  // so a warp reads 2 or 1 whole rows of each tensor per step
  constexpr int kEl = 16 / int(sizeof(T));
  constexpr int kLanesPerRow = kHeadDim / kEl;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const int64_t rows = int64_t(B) * N * H;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow, l = lane % kLanesPerRow;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
       w * kRowsPerWarp < rows; w += nwarps) {
    const int64_t row = w * kRowsPerWarp + sub;
    float acc = 0.f;
    if (row < rows) {
      const uint4 a =
          __ldg(reinterpret_cast<const uint4*>(out + row * kHeadDim) + l);
      const uint4 c =
          __ldg(reinterpret_cast<const uint4*>(dout + row * kHeadDim) + l);
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
      const uint32_t wc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (sizeof(T) == 2) {
          acc = fmaf(bf16lo_to_f32(wa[e]), bf16lo_to_f32(wc[e]), acc);
          acc = fmaf(bf16hi_to_f32(wa[e]), bf16hi_to_f32(wc[e]), acc);
        } else {
          acc = fmaf(__uint_as_float(wa[e]), __uint_as_float(wc[e]), acc);
        }
      }
    }
#pragma unroll
    for (int o = kLanesPerRow / 2; o > 0; o >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (l == 0 && row < rows) {
      const int h = int(row % H);
      const int64_t bn = row / H;
      const int n = int(bn % N);
      const int b = int(bn / N);
      delta[(int64_t(b) * H + h) * N + n] = acc;
    }
  }
}

// Four consecutive values of T from floats (one 8- or 16-byte store).
__device__ __forceinline__ void store4(__nv_bfloat16* p, float a, float b,
                                       float c, float d) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(a, b),
                                            pack_bf16x2(c, d));
}
__device__ __forceinline__ void store4(float* p, float a, float b, float c,
                                       float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

// dq = R(-pos) * dq_acc * scale, rounded to T (pos == nullptr: no
// rotation). One thread per four RoPE pairs of a (b, n, h) row: pairs
// 4u .. 4u+3, which are the values 8u .. 8u+7 in the interleaved layout and
// 4u .. 4u+3 with 64+4u .. 64+4u+3 in the rotate-half layout.
template <typename T, bool HALF>
__global__ void dq_convert_kernel(const float* __restrict__ acc,
                                  const int32_t* __restrict__ pos,
                                  const float4* __restrict__ table, int B,
                                  int N, int H, float scale,
                                  T* __restrict__ dq) {
  pdl_wait();
  pdl_trigger();
  constexpr int kQuads = kHeadDim / 8;  // groups of 4 pairs per row
  const int64_t total = int64_t(B) * N * H * kQuads;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
       e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int u = int(e % kQuads);
    const int64_t bnh = e / kQuads;
    const int64_t row = bnh * kHeadDim;
    // a[i], b[i]: the two elements of pair 4u + i
    float a[4], b[4];
    if (HALF) {
      const float4 x = *reinterpret_cast<const float4*>(acc + row + 4 * u);
      const float4 y = *reinterpret_cast<const float4*>(acc + row + 64 + 4 * u);
      a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w;
      b[0] = y.x; b[1] = y.y; b[2] = y.z; b[3] = y.w;
    } else {
      const float4 x = *reinterpret_cast<const float4*>(acc + row + 8 * u);
      const float4 y = *reinterpret_cast<const float4*>(acc + row + 8 * u + 4);
      a[0] = x.x; b[0] = x.y; a[1] = x.z; b[1] = x.w;
      a[2] = y.x; b[2] = y.y; a[3] = y.z; b[3] = y.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] *= scale;
      b[i] *= scale;
    }
    if (pos) {
      // inverse rotation: (a, b) -> (a c + b s, -a s + b c)
      const float4* t = table + int64_t(pos[bnh / H]) * (kHeadDim / 4) + 2 * u;
      const float4 c01 = t[0], c23 = t[1];
      const float cs[4] = {c01.x, c01.z, c23.x, c23.z};
      const float sn[4] = {c01.y, c01.w, c23.y, c23.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float ra = a[i] * cs[i] + b[i] * sn[i];
        const float rb = b[i] * cs[i] - a[i] * sn[i];
        a[i] = ra;
        b[i] = rb;
      }
    }
    if (HALF) {
      store4(dq + row + 4 * u, a[0], a[1], a[2], a[3]);
      store4(dq + row + 64 + 4 * u, b[0], b[1], b[2], b[3]);
    } else {
      store4(dq + row + 8 * u, a[0], b[0], a[1], b[1]);
      store4(dq + row + 8 * u + 4, a[2], b[2], a[3], b[3]);
    }
  }
}

// ------------------------------------------------------------ launchers
static inline int grid_for(int64_t n, int threads, int cap = 148 * 16) {
  int64_t g = (n + threads - 1) / threads;
  return int(g < 1 ? 1 : (g > cap ? cap : g));
}

cudaError_t launch_rope_table(double theta, int D, int max_pos, float* table,
                              cudaStream_t st) {
  if (max_pos <= 0) return cudaSuccess;
  int64_t n = int64_t(max_pos) * (D / 2);
  {
    const cudaError_t le = launch_dependent(
        rope_table_kernel, dim3(grid_for(n, 256, 148 * 32)), dim3(256), 0, st,
        theta, D / 2, max_pos, reinterpret_cast<float2*>(table));
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_block_meta(const int32_t* seg, int B, int N, int bq, int bk,
                              int32_t* kv_lo, int32_t* kv_hi,
                              cudaStream_t st) {
  int Tq = (N + bq - 1) / bq;
  int n = B * Tq;
  if (n == 0) return cudaSuccess;
  block_meta_kernel<<<(n + 255) / 256, 256, 0, st>>>(seg, B, N, bq, bk, Tq,
                                                      kv_lo, kv_hi);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_rope_apply(const void* x, const int32_t* pos,
                              const float* table, int B, int N, int H,
                              bool half, void* hi, void* lo, cudaStream_t st) {
  int64_t chunks = int64_t(B) * N * H * (kHeadDim / 8);
  if (chunks == 0) return cudaSuccess;
  if (half) {
    {
      const cudaError_t le = launch_dependent(
          rope_apply_half_kernel, dim3(grid_for(chunks / 2, 256, 148 * 16)),
          dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x), pos,
          reinterpret_cast<const float2*>(table), chunks / 2, H,
          static_cast<__nv_bfloat16*>(hi), static_cast<__nv_bfloat16*>(lo));
      if (le != cudaSuccess) return le;
    }
  } else {
    {
      const cudaError_t le = launch_dependent(
          rope_apply_kernel, dim3(grid_for(chunks, 256, 148 * 16)), dim3(256),
          0, st, static_cast<const __nv_bfloat16*>(x), pos,
          reinterpret_cast<const float2*>(table), chunks, H,
          static_cast<__nv_bfloat16*>(hi), static_cast<__nv_bfloat16*>(lo));
      if (le != cudaSuccess) return le;
    }
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_cross_meta(const int32_t* seg_q, const int32_t* seg_k,
                              int B, int Nq, int Nk, int q_off, int k_off,
                              int bk, int32_t* row_lo, int32_t* row_hi,
                              int32_t* kv_lo, int32_t* kv_hi,
                              int32_t* lo_max, int32_t* hi_min,
                              cudaStream_t st) {
  const int64_t n = int64_t(B) * Nq;
  if (n == 0) return cudaSuccess;
  const int Tq = (Nq + kBlock - 1) / kBlock;
  {
    const cudaError_t le = launch_dependent(
        cross_meta_kernel, dim3(B * Tq), dim3(kBlock), 0, st, seg_q, seg_k, B,
        Nq, Nk, q_off, k_off, bk, Tq, row_lo, row_hi, kv_lo, kv_hi, lo_max,
        hi_min);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_cross_meta_keys(const int32_t* seg_q, const int32_t* seg_k,
                                   int B, int Nq, int Nk, int q_off,
                                   int k_off, int32_t* col_lo,
                                   int32_t* col_hi, int32_t* q_lo,
                                   int32_t* q_hi, int32_t* klo_max,
                                   int32_t* khi_min, cudaStream_t st) {
  const int64_t n = int64_t(B) * Nk;
  if (n == 0) return cudaSuccess;
  const int Tk = (Nk + kBlock - 1) / kBlock;
  {
    const cudaError_t le = launch_dependent(
        cross_keys_kernel, dim3(B * Tk), dim3(kBlock), 0, st, seg_q, seg_k, B,
        Nq, Nk, q_off, k_off, Tk, col_lo, col_hi, q_lo, q_hi, klo_max, khi_min);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_merge(void* out, float* lse, const void* out_p,
                         const float* lse_p, int B, int N, int H,
                         cudaStream_t st) {
  const int64_t n = int64_t(B) * N * H * (kHeadDim / 8);
  if (n == 0) return cudaSuccess;
  {
    const cudaError_t le = launch_dependent(
        merge_kernel, dim3(grid_for(n, 256, 148 * 16)), dim3(256), 0, st,
        static_cast<__nv_bfloat16*>(out), lse,
        static_cast<const __nv_bfloat16*>(out_p), lse_p, B, N, H);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_fill(float* x, float v, int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  fill_kernel<<<grid_for(n, 256, 148 * 8), 256, 0, st>>>(x, v, n);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_row_start(const int32_t* seg, int B, int N, int32_t* rs,
                             int32_t* re, cudaStream_t st) {
  int64_t n = int64_t(B) * N;
  if (n == 0) return cudaSuccess;
  row_start_kernel<<<grid_for(n, 256, 148 * 16), 256, 0, st>>>(seg, B, N, rs,
                                                                re);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_tile_class(const int32_t* seg, int B, int N, int bq,
                              int bk, const int32_t* kv_lo,
                              const int32_t* kv_hi, uint8_t* cls,
                              cudaStream_t st) {
  int Tq = (N + bq - 1) / bq, Tk = (N + bk - 1) / bk;
  int64_t n = int64_t(B) * Tq * Tk;
  if (n == 0) return cudaSuccess;
  tile_class_kernel<<<grid_for(n, 256, 148 * 32), 256, 0, st>>>(
      seg, B, N, bq, bk, Tq, Tk, kv_lo, kv_hi, cls);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_kv_meta(int B, int Tq, int Tk, const int32_t* kv_lo,
                           const int32_t* kv_hi, int32_t* q_lo, int32_t* q_hi,
                           cudaStream_t st) {
  int n = B * Tk;
  if (n == 0) return cudaSuccess;
  kv_meta_kernel<<<(n + 255) / 256, 256, 0, st>>>(B, Tq, Tk, kv_lo, kv_hi,
                                                   q_lo, q_hi);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_lpt_order(int B, int T, int group, const int32_t* lo,
                             const int32_t* hi, int anchor, int32_t* order,
                             int32_t* counter, cudaStream_t st) {
  int U = (T + group - 1) / group;
  int n = B * U;
  if (n == 0) return cudaSuccess;
  if (n <= kSortMax) {
    int p2 = 1;
    while (p2 < n) p2 <<= 1;
    size_t smem = size_t(p2) * sizeof(uint64_t);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(
          lpt_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
          int(smem));
      if (e != cudaSuccess) return e;
    }
    {
      const cudaError_t le = launch_dependent(
          lpt_sort_kernel, dim3(1), dim3(1024), smem, st, B, T, group, lo, hi,
          U, anchor, order, counter);
      if (le != cudaSuccess) return le;
    }
    note_launch();
  } else {
    {
      const cudaError_t le = launch_dependent(
          reverse_order_kernel, dim3((n + 255) / 256), dim3(256), 0, st, B, U,
          order, counter);
      if (le != cudaSuccess) return le;
    }
    note_launch();
  }
  return cudaGetLastError();
}

cudaError_t launch_check_inputs(const int32_t* seg, const int32_t* pos, int B,
                                int N, int max_pos, int* res,
                                cudaStream_t st) {
  int64_t n = int64_t(B) * N;
  if (n == 0) return cudaSuccess;
  check_inputs_kernel<<<grid_for(n, 256), 256, 0, st>>>(seg, pos, B, N,
                                                         max_pos, res);
  note_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_delta(const T* out, const T* dout, int B, int N, int H,
                             float* delta, cudaStream_t st) {
  int64_t rows = int64_t(B) * N * H;
  if (rows == 0) return cudaSuccess;
  // one warp per 1 (fp32) or 2 (bf16) rows per step, grid-stride
  const int64_t threads = (rows * int64_t(sizeof(T)) + 3) / 4 * 32;
  {
    const cudaError_t le = launch_dependent(
        bwd_delta_kernel<T>, dim3(grid_for(threads, 256, 148 * 16)),
        dim3(256), 0, st, out, dout, B, N, H, delta);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dq_convert(const float* acc, const int32_t* pos,
                              const float* table, int B, int N, int H,
                              float scale, bool half, T* dq, cudaStream_t st) {
  const int64_t n = int64_t(B) * N * H * (kHeadDim / 8);
  if (n == 0) return cudaSuccess;
  const float4* t4 = reinterpret_cast<const float4*>(table);
  if (half)
    {
      const cudaError_t le = launch_dependent(
          dq_convert_kernel<T, true>, dim3(grid_for(n, 256, 148 * 32)),
          dim3(256), 0, st, acc, pos, t4, B, N, H, scale, dq);
      if (le != cudaSuccess) return le;
    }
  else
    {
      const cudaError_t le = launch_dependent(
          dq_convert_kernel<T, false>, dim3(grid_for(n, 256, 148 * 32)),
          dim3(256), 0, st, acc, pos, t4, B, N, H, scale, dq);
      if (le != cudaSuccess) return le;
    }
  note_launch();
  return cudaGetLastError();
}

template cudaError_t launch_bwd_delta<__nv_bfloat16>(const __nv_bfloat16*,
                                                     const __nv_bfloat16*, int,
                                                     int, int, float*,
                                                     cudaStream_t);
template cudaError_t launch_bwd_delta<float>(const float*, const float*, int,
                                             int, int, float*, cudaStream_t);
template cudaError_t launch_dq_convert<__nv_bfloat16>(const float*,
                                                      const int32_t*,
                                                      const float*, int, int,
                                                      int, float, bool,
                                                      __nv_bfloat16*,
                                                      cudaStream_t);
template cudaError_t launch_dq_convert<float>(const float*, const int32_t*,
                                              const float*, int, int, int,
                                              float, bool, float*,
                                              cudaStream_t);

}  // namespace lwm
