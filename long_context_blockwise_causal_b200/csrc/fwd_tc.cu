// Forward blockwise packed causal RoPE attention on tcgen05 (sm_100a).
//
// Method ("开源巨兽LWM：如何用RingAttention撬动百万Token多模态世界", 3.1-3.2;
// "LWM：突破 100 万 Token 的开源大模型", 配置参数 and 概述 (b)): the query
// blocks of one (batch row, head) sweep the key/value blocks from the block
// holding their diagonal down to the start of their packed example, keeping
// a running max, a running sum and an output accumulator (online softmax);
// RoPE ("[论文解读] World Model on Million-Length Video And Language With
// Blockwise RingAttention", 提出的方法) is applied to each Q tile in shared
// memory right after it lands. Keys are rotated once per token by a
// separate pass (each key block is read by every query block that sees it,
// so rotating it in the loader would repeat the work O(N/128) times).
//
// CTA = persistent worker over units of 2 x 128 query rows of one (b, h):
//   warps 0-3   softmax for query sub-tile 0 (TMEM lanes 0-127)
//   warps 4-7   softmax for query sub-tile 1
//   warps 8-11  RoPE: rotate each landed Q tile in place (fp32 math,
//               bf16 round to nearest even; hi/lo split in the x3 mode)
//   warp 12     TMA producer (Q per unit, rotated K and V per key block)
//   warp 13     tcgen05 issuer (one elected lane) + TMEM owner
//   warps 14-15 idle (they complete the fourth warpgroup, which setmaxnreg
//               needs; their registers go to the softmax warps)
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P (bf16)
// is written over the first 64 columns of S and read from there by the
// P.V MMA. O is rescaled in TMEM only when a row max grows by more than
// 2^8 (the result is exact either way: max and sum stay consistent).
#include <cuda.h>

#include "aux_kernels.cuh"
#include "tc_kernels.cuh"

namespace lwm {
namespace {

constexpr int kThreadsFwd = 16 * 32;
// Register budget per warpgroup after setmaxnreg (launch: 128 each). The
// four groups share each SM sub-partition, so the sum must stay 4 x 128.
constexpr int kRegsSoftmax = 184, kRegsRope = 72, kRegsMisc = 72;
static_assert(2 * kRegsSoftmax + kRegsRope + kRegsMisc == 4 * 128,
              "register split must equal the launch allocation");
constexpr int kTileBytes = kBlock * kHeadDim * 2;       // 32 KB bf16 tile
constexpr int kHalfTileBytes = kTileBytes / 2;          // one 64-wide d chunk
constexpr uint64_t kWaitLimitNs = 4000000000ull;        // 4 s per wait
constexpr float kRescaleThreshold = 8.0f;               // log2 units

// BK: keys per key block (the key tile the forward sweeps), 128 or 64.
template <bool X3, int BK>
struct FwdCfg {
  static_assert(BK == 128 || BK == 64, "key blocks of 128 or 64 keys");
  static constexpr int kKVTile = BK * kHeadDim * 2;   // one K or V tile
  static constexpr int kKVHalf = kKVTile / 2;         // one 64-wide d chunk
  static constexpr int KS = BK == 128 ? (X3 ? 1 : 2) : (X3 ? 2 : 4);
  static constexpr int VS = KS;
  static constexpr int kQ = 0;
  static constexpr int kQlo = kQ + 2 * kTileBytes;
  static constexpr int kK = kQlo + (X3 ? 2 * kTileBytes : 0);
  static constexpr int kKlo = kK + KS * kKVTile;
  static constexpr int kV = kKlo + (X3 ? KS * kKVTile : 0);
  static constexpr int kBars = kV + VS * kKVTile;
  // barrier slots
  static constexpr int bQFull = 0, bQReady = 2, bQEmpty = 4, bSFull = 6,
                       bPFull = 8, bOFull = 10, bOEmpty = 12, bEpi = 14,
                       bDone = 16, bItemFull = 17, bItemEmpty = 19,
                       bKFull = 21, bKEmpty = bKFull + KS,
                       bVFull = bKEmpty + KS, bVEmpty = bVFull + VS,
                       kNumBars = bVEmpty + VS;
  static constexpr int kMisc = kBars + kNumBars * 8;
  static constexpr int kSmem = kMisc + 32 + 1024;  // + alignment slack
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

struct FwdParams {
  int32_t* counter;
  const int32_t* pos_q;
  const float2* table;
  const int32_t* kv_lo;
  const int32_t* kv_hi;
  const int32_t* row_lo;
  const int32_t* row_hi;
  const int32_t* lo_max;
  const int32_t* hi_min;
  const int32_t* order;
  float* lse;
  int* status;
  int B, Nq, Nk, H, Tq, U, G, k_off;
  int rope_half;  // Q in the rotate-half layout
  int total_items;
  float scale_log2;
};

struct Item {
  int b, h, t[2];
  int lo[2], hi[2];
  int jlo, jhi;
  bool present[2];
};

__device__ __forceinline__ Item get_item(const FwdParams& p, int it) {
  Item m;
  int per_group = p.G * p.B * p.U;
  int hg = it / per_group;
  int rem = it - hg * per_group;
  int r = rem / p.G;
  int hh = rem - r * p.G;
  m.h = hg * p.G + hh;
  int unit = p.order[r];
  m.b = unit / p.U;
  int u = unit - m.b * p.U;
  m.jlo = 1 << 30;
  m.jhi = -1;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    m.t[s] = 2 * u + s;
    m.present[s] = m.t[s] < p.Tq;
    if (m.present[s]) {
      m.lo[s] = p.kv_lo[m.b * p.Tq + m.t[s]];
      m.hi[s] = p.kv_hi[m.b * p.Tq + m.t[s]];
      if (m.lo[s] <= m.hi[s]) {  // a query block may see no key block
        m.jlo = min(m.jlo, m.lo[s]);
        m.jhi = max(m.jhi, m.hi[s]);
      }
    } else {
      m.lo[s] = 1;
      m.hi[s] = 0;
    }
  }
  return m;
}

// (b, h) of work item `it` and the query block of its sub-tile s: the
// arithmetic of get_item and its one load of the order (the softmax warps
// recompute this after the key sweep instead of keeping it in registers
// through it)
struct Place {
  int b, h, t;
};

__device__ __forceinline__ Place item_place(const FwdParams& p, int it,
                                            int s) {
  Place q;
  const int per_group = p.G * p.B * p.U;
  const int hg = it / per_group;
  const int rem = it - hg * per_group;
  const int r = rem / p.G;
  q.h = hg * p.G + (rem - r * p.G);
  const int unit = p.order[r];
  q.b = unit / p.U;
  q.t = 2 * (unit - q.b * p.U) + s;
  return q;
}

__device__ __forceinline__ bool active(const Item& m, int s, int j) {
  return j >= m.lo[s] && j <= m.hi[s];
}

// RoPE of one row of a landed 128x128 bf16 tile (two SW128 64-wide d
// chunks), in place. Thread r owns row r: its 16 chunks sit at distinct
// swizzled 16-byte slots of its 128-byte rows, so a quarter-warp touches
// 8 different slots (no bank conflicts). The row's 64 (cos, sin) pairs are
// read in quarters of 16 pairs; cs holds the first quarter, loaded by the
// caller ahead of the barrier wait. lo_dst (x3 mode) receives the bf16
// residual of each rotated value.
template <bool X3>
__device__ __forceinline__ void rope_row(uint8_t* tile, uint8_t* lo_dst,
                                         const float4* __restrict__ trow,
                                         float4 (&cs)[8], int r, bool valid) {
  if (!valid) {
    if (X3) {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4*>(lo_dst + (c >> 3) * kHalfTileBytes +
                                  r * 128 + (((c & 7) ^ (r & 7)) << 4)) =
            make_uint4(0, 0, 0, 0);
    }
    return;  // zero-filled by TMA; nothing to rotate
  }
#pragma unroll
  for (int qt = 0; qt < 4; ++qt) {
    if (qt > 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] = __ldg(trow + qt * 8 + e);
    }
#pragma unroll
    for (int cl = 0; cl < 4; ++cl) {
      const int lc = (qt & 1) * 4 + cl;
      const int off =
          (qt >> 1) * kHalfTileBytes + r * 128 + ((lc ^ (r & 7)) << 4);
      uint4 w = *reinterpret_cast<uint4*>(tile + off);
      const float c4[4] = {cs[2 * cl].x, cs[2 * cl].z, cs[2 * cl + 1].x,
                           cs[2 * cl + 1].z};
      const float s4[4] = {cs[2 * cl].y, cs[2 * cl].w, cs[2 * cl + 1].y,
                           cs[2 * cl + 1].w};
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      uint32_t hi_out[4], lo_out[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo_to_f32(ws[e]);
        const float b = bf16hi_to_f32(ws[e]);
        const float ra = fmaf(a, c4[e], -b * s4[e]);
        const float rb = fmaf(a, s4[e], b * c4[e]);
        const uint32_t h = pack_bf16x2(ra, rb);
        hi_out[e] = h;
        if (X3)
          lo_out[e] = pack_bf16x2(ra - bf16lo_to_f32(h), rb - bf16hi_to_f32(h));
      }
      *reinterpret_cast<uint4*>(tile + off) =
          make_uint4(hi_out[0], hi_out[1], hi_out[2], hi_out[3]);
      if (X3)
        *reinterpret_cast<uint4*>(lo_dst + off) =
            make_uint4(lo_out[0], lo_out[1], lo_out[2], lo_out[3]);
    }
  }
}

// The same for the rotate-half layout: pair k is (dim k, dim k + 64), so
// the 16-byte slot lc of d chunk 0 pairs with slot lc of d chunk 1 (same
// swizzled offset, 16 KB apart); slot lc holds pairs 8 lc .. 8 lc + 7. The
// rotated values stay in that layout (the keys were rotated in it too).
template <bool X3>
__device__ __forceinline__ void rope_row_half(uint8_t* tile, uint8_t* lo_dst,
                                              const float4* __restrict__ trow,
                                              float4 (&cs)[8], int r,
                                              bool valid) {
  if (!valid) {
    if (X3) {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4*>(lo_dst + (c >> 3) * kHalfTileBytes +
                                  r * 128 + (((c & 7) ^ (r & 7)) << 4)) =
            make_uint4(0, 0, 0, 0);
    }
    return;
  }
#pragma unroll
  for (int qt = 0; qt < 4; ++qt) {  // cs: pairs 16 qt .. 16 qt + 15
    if (qt > 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] = __ldg(trow + qt * 8 + e);
    }
#pragma unroll
    for (int cl = 0; cl < 2; ++cl) {
      const int lc = 2 * qt + cl;
      const int off0 = r * 128 + ((lc ^ (r & 7)) << 4);
      const int off1 = off0 + kHalfTileBytes;
      const uint4 w0 = *reinterpret_cast<uint4*>(tile + off0);
      const uint4 w1 = *reinterpret_cast<uint4*>(tile + off1);
      const uint32_t a[4] = {w0.x, w0.y, w0.z, w0.w};
      const uint32_t b[4] = {w1.x, w1.y, w1.z, w1.w};
      uint32_t ha[4], hb[4], la[4], lb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 t = cs[4 * cl + e];  // pairs 8 lc + 2e, 8 lc + 2e + 1
        const float a0 = bf16lo_to_f32(a[e]), a1 = bf16hi_to_f32(a[e]);
        const float b0 = bf16lo_to_f32(b[e]), b1 = bf16hi_to_f32(b[e]);
        const float ra0 = fmaf(a0, t.x, -b0 * t.y);
        const float rb0 = fmaf(a0, t.y, b0 * t.x);
        const float ra1 = fmaf(a1, t.z, -b1 * t.w);
        const float rb1 = fmaf(a1, t.w, b1 * t.z);
        ha[e] = pack_bf16x2(ra0, ra1);
        hb[e] = pack_bf16x2(rb0, rb1);
        if (X3) {
          la[e] = pack_bf16x2(ra0 - bf16lo_to_f32(ha[e]),
                              ra1 - bf16hi_to_f32(ha[e]));
          lb[e] = pack_bf16x2(rb0 - bf16lo_to_f32(hb[e]),
                              rb1 - bf16hi_to_f32(hb[e]));
        }
      }
      *reinterpret_cast<uint4*>(tile + off0) =
          make_uint4(ha[0], ha[1], ha[2], ha[3]);
      *reinterpret_cast<uint4*>(tile + off1) =
          make_uint4(hb[0], hb[1], hb[2], hb[3]);
      if (X3) {
        *reinterpret_cast<uint4*>(lo_dst + off0) =
            make_uint4(la[0], la[1], la[2], la[3]);
        *reinterpret_cast<uint4*>(lo_dst + off1) =
            make_uint4(lb[0], lb[1], lb[2], lb[3]);
      }
    }
  }
}

// Loads (position, first quarter of cos/sin) of tile row r before the wait.
__device__ __forceinline__ const float4* rope_prefetch(
    const int32_t* __restrict__ pos, const float2* __restrict__ table,
    int64_t rowbase, int grow, int N, float4 (&cs)[8], bool& valid) {
  valid = grow < N;
  const float4* trow = nullptr;
  if (valid) {
    const int pp = __ldg(pos + rowbase + grow);
    trow = reinterpret_cast<const float4*>(table + int64_t(pp) * (kHeadDim / 2));
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = __ldg(trow + e);
  }
  return trow;
}

template <bool X3, int BK>
__global__ void __launch_bounds__(kThreadsFwd, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_o,
              const __grid_constant__ CUtensorMap tm_klo,
              const FwdParams p) {
  pdl_wait();
  pdl_trigger();
  using C = FwdCfg<X3, BK>;
  constexpr int NC = BK / 32;   // 32-column chunks of an S row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::kBars;
  auto bar = [&](int i) { return bars + 8u * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  // two-slot ring of work units: the producer takes the next unit from the
  // global counter (longest first) and every other role reads it from here
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::kMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::bQFull + s), 1);
      mbar_init(bar(C::bQReady + s), 4);
      mbar_init(bar(C::bQEmpty + s), 1);
      mbar_init(bar(C::bSFull + s), 1);
      mbar_init(bar(C::bPFull + s), 4);
      mbar_init(bar(C::bOFull + s), 1);
      mbar_init(bar(C::bOEmpty + s), 4);
      mbar_init(bar(C::bEpi + s), 128);
    }
    mbar_init(bar(C::bDone), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::bItemFull + i), 1);
      // consumers: 8 softmax warps, 4 RoPE warps, the MMA lane
      mbar_init(bar(C::bItemEmpty + i), 13);
    }
    for (int i = 0; i < C::KS; ++i) {
      mbar_init(bar(C::bKFull + i), 1);
      mbar_init(bar(C::bKEmpty + i), 1);
    }
    for (int i = 0; i < C::VS; ++i) {
      mbar_init(bar(C::bVFull + i), 1);
      mbar_init(bar(C::bVEmpty + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
    if (X3) prefetch_tmap(&tm_klo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int nitems = p.total_items;

  if (warp < 8) {
    // ------------------------------------------------ softmax (warps 0-7)
    regs_inc<kRegsSoftmax>();
    const int s = warp >> 2;                 // query sub-tile
    const int r = (warp & 3) * 32 + lane;    // row in the sub-tile = TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + s * 128;
    const uint32_t tO = tmem + lane_off + 256 + s * 128;
    int sc = 0, oc = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      ok = mbar_wait(bar(C::bItemFull + (n & 1)), (n >> 1) & 1, abort_flag,
                     p.status, kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int it = item_slot[n & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::bItemEmpty + (n & 1)));
      if (it < 0) break;
      const Item m = get_item(p, it);
      // this warp's sub-tile as scalars: s is a run-time value, and an
      // array indexed by it would live in local memory (reloaded after
      // every asm statement of the tile loop)
      const bool my_present = s ? m.present[1] : m.present[0];
      const int my_t = s ? m.t[1] : m.t[0];
      const int my_lo = s ? m.lo[1] : m.lo[0];
      const int my_hi = s ? m.hi[1] : m.hi[0];
      if (!my_present) continue;
      const int64_t rowbase = int64_t(m.b) * p.Nq;
      const int q0 = my_t * kBlock;
      const int i = q0 + r;
      const bool valid = i < p.Nq;
      // allowed keys of this row (global indices): lo_i <= key <= hi_i
      const int lo_i = valid ? __ldg(p.row_lo + rowbase + i) : 1;
      const int hi_i = valid ? __ldg(p.row_hi + rowbase + i) : 0;
      const int lo_max = __ldg(p.lo_max + m.b * p.Tq + my_t);
      const int hi_min = __ldg(p.hi_min + m.b * p.Tq + my_t);
      float m_used = -INFINITY, l = 0.f;
      bool first = true;
      for (int j = my_hi; j >= my_lo && ok; --j) {
        ok = mbar_wait(bar(C::bSFull + s), sc & 1, abort_flag, p.status,
                       kWaitLimitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        sc++;
        tc_fence_after();
        const int k0 = p.k_off + j * BK;  // global index of key 0
        // every pair of the tile allowed: every row of the block sees the
        // whole key block
        const bool full = lo_max <= k0 && hi_min >= k0 + BK - 1;
        // the whole S row of this thread (BK columns) in registers
        uint32_t v[NC][32];
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(tS + c * 32, v[c]);
        tmem_wait_ld();
        if (!full) {  // mask: keep lo_i <= key <= hi_i
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const int lo = lo_i - (k0 + c * 32), hi = hi_i - (k0 + c * 32);
#pragma unroll
            for (int x = 0; x < 32; ++x)
              v[c][x] = (x >= lo && x <= hi) ? v[c][x] : 0xff800000u;
          }
        }
        float mc[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          mc[c] = __uint_as_float(v[c][0]);
#pragma unroll
          for (int x = 1; x < 31; x += 2)
            mc[c] = max3(mc[c], __uint_as_float(v[c][x]),
                         __uint_as_float(v[c][x + 1]));
          mc[c] = fmaxf(mc[c], __uint_as_float(v[c][31]));
        }
        float mx = mc[0];
#pragma unroll
        for (int c = 1; c < NC; ++c) mx = fmaxf(mx, mc[c]);
        const float m_tile = mx * p.scale_log2;
        float m_new = m_used;
        bool rescale = false;
        if (m_tile > m_used + kRescaleThreshold) {
          m_new = m_tile;
          rescale = true;
        }
        const float alpha = rescale ? ex2(m_used - m_new) : 1.f;
        l *= alpha;
        const float sub = m_new == -INFINITY ? 0.f : m_new;
        // P = 2^(S*c - m) (bf16, over S columns [0, BK/2)), row sum in
        // fp32; a row that has seen no key yet keeps m = -inf and gets
        // P = 0 (the subtrahend is 0, its scores are -inf)
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nsub2 = make_float2(-sub, -sub);
        // one row-sum accumulator per 32-column chunk: four short add
        // chains instead of one through the whole row (this is also the
        // form in which the softmax warps fit their registers unspilled)
        float2 lsc[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint32_t pk[16];
          lsc[c] = make_float2(0.f, 0.f);
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const float2 t = fma2(make_float2(__uint_as_float(v[c][x]),
                                              __uint_as_float(v[c][x + 1])),
                                  sc2, nsub2);
            const float p0 = ex2(t.x), p1 = ex2(t.y);
            lsc[c] = add2(lsc[c], make_float2(p0, p1));
            pk[x >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        float2 lsum = lsc[0];
#pragma unroll
        for (int c = 1; c < NC; ++c) lsum = add2(lsum, lsc[c]);
        l += lsum.x + lsum.y;
        // O holds every P.V issued so far for this row (the S MMA this
        // tile waited on was issued after them); rescale it when the max
        // moved past the threshold
        if (!first && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x)
              o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::bPFull + s));
        m_used = m_new;
        first = false;
      }
      if (!ok) break;
      // ---------------------------------------------- epilogue
      // where this sub-tile's rows go, recomputed (its load overlaps the
      // wait for the last P.V)
      const Place pl = item_place(p, it, s);
      ok = mbar_wait(bar(C::bOFull + s), oc & 1, abort_flag, p.status,
                     kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      oc++;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint8_t* stage = smem + C::kQ + s * kTileBytes;  // Q_s is free now
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        // rows that saw no key (l == 0) write 0; O was never written then
        for (int x = 0; x < 32; x += 2)
          pk[x >> 1] = l > 0.f ? pack_bf16x2(__uint_as_float(v[x]) * inv,
                                             __uint_as_float(v[x + 1]) * inv)
                               : 0u;
        // columns c*32 .. c*32+31 = d chunk (c>>1), 16-byte chunks
        // (c&1)*4 .. +3 of that 128-byte row
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int lc = (c & 1) * 4 + e;
          int off = (c >> 1) * kHalfTileBytes + r * 128 + ((lc ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(stage + off) =
              make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::bOEmpty + s));
      fence_proxy_async_smem();
      mbar_arrive(bar(C::bEpi + s));
      if (r == 0 &&
          mbar_wait(bar(C::bEpi + s), (oc - 1) & 1, abort_flag, p.status,
                    kWaitLimitNs)) {
        uint32_t src = sbase + C::kQ + s * kTileBytes;
        tma_store_4d(&tm_o, src, 0, pl.h, pl.t * kBlock, pl.b);
        tma_store_4d(&tm_o, src + kHalfTileBytes, 64, pl.h, pl.t * kBlock,
                     pl.b);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(bar(C::bQEmpty + s));
      }
      if (pl.t * kBlock + r < p.Nq)
        p.lse[(int64_t(pl.b) * p.H + pl.h) * p.Nq + pl.t * kBlock + r] =
            l > 0.f ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
    }
    if (threadIdx.x == 0 || threadIdx.x == 128) bulk_wait0();
  } else if (warp < 12) {
    // ------------------------------------------------ RoPE rotation
    regs_dec<kRegsRope>();
    const int r = threadIdx.x - 8 * 32;  // tile row owned by this thread
    int qcount[2] = {0, 0};
    bool ok = true;
    for (int n = 0; ok; ++n) {
      ok = mbar_wait(bar(C::bItemFull + (n & 1)), (n >> 1) & 1, abort_flag,
                     p.status, kWaitLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int it = item_slot[n & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::bItemEmpty + (n & 1)));
      if (it < 0) break;
      Item m = get_item(p, it);
      const int64_t rowbase = int64_t(m.b) * p.Nq;
            for (int s = 0; s < 2 && ok; ++s) {
        if (!m.present[s]) continue;
        float4 cs0[8];
        bool valid;
        const float4* trow = rope_prefetch(p.pos_q, p.table, rowbase,
                                           m.t[s] * kBlock + r, p.Nq, cs0,
                                           valid);
        ok = mbar_wait(bar(C::bQFull + s), qcount[s] & 1, abort_flag,
                       p.status, kWaitLimitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        qcount[s]++;
        if (p.rope_half)
          rope_row_half<X3>(smem + C::kQ + s * kTileBytes,
                            smem + C::kQlo + s * kTileBytes, trow, cs0, r,
                            valid);
        else
          rope_row<X3>(smem + C::kQ + s * kTileBytes,
                       smem + C::kQlo + s * kTileBytes, trow, cs0, r, valid);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::bQReady + s));
      }
    }
  } else {
    // warps 12-15 share one register budget (one setmaxnreg for the
    // whole warpgroup), then split: 12 producer, 13 MMA, 14-15 idle
    regs_dec<kRegsMisc>();
    if (warp == 12) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int qfill[2] = {0, 0};
      int kfill = 0, vfill = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        if (n >= 2) {
          ok = mbar_wait(bar(C::bItemEmpty + (n & 1)), ((n >> 1) - 1) & 1,
                         abort_flag, p.status, kWaitLimitNs);
          if (!ok) break;
        }
        int it = atomicAdd(p.counter, 1);
        if (it >= nitems) it = -1;
        item_slot[n & 1] = it;
        mbar_arrive(bar(C::bItemFull + (n & 1)));
        if (it < 0) break;
        Item m = get_item(p, it);
        #pragma unroll
        for (int s = 0; s < 2 && ok; ++s) {
          if (!m.present[s]) continue;
          if (qfill[s] > 0)
            ok = mbar_wait(bar(C::bQEmpty + s), (qfill[s] - 1) & 1,
                           abort_flag, p.status, kWaitLimitNs);
          if (!ok) break;
          uint32_t dst = sbase + C::kQ + s * kTileBytes;
          mbar_arrive_expect_tx(bar(C::bQFull + s), kTileBytes);
          tma_load_4d(dst, &tm_q, bar(C::bQFull + s), 0, m.h,
                      m.t[s] * kBlock, m.b);
          tma_load_4d(dst + kHalfTileBytes, &tm_q, bar(C::bQFull + s), 64,
                      m.h, m.t[s] * kBlock, m.b);
          qfill[s]++;
        }
        for (int j = m.jhi; j >= m.jlo && ok; --j) {
          int ks = kfill % C::KS;
          if (kfill >= C::KS)
            ok = mbar_wait(bar(C::bKEmpty + ks), ((kfill / C::KS) - 1) & 1,
                           abort_flag, p.status, kWaitLimitNs);
          if (!ok) break;
          uint32_t kd = sbase + C::kK + ks * C::kKVTile;
          mbar_arrive_expect_tx(bar(C::bKFull + ks),
                                X3 ? 2 * C::kKVTile : C::kKVTile);
          tma_load_4d(kd, &tm_k, bar(C::bKFull + ks), 0, m.h, j * BK, m.b);
          tma_load_4d(kd + C::kKVHalf, &tm_k, bar(C::bKFull + ks), 64, m.h,
                      j * BK, m.b);
          if (X3) {
            uint32_t kl = sbase + C::kKlo + ks * C::kKVTile;
            tma_load_4d(kl, &tm_klo, bar(C::bKFull + ks), 0, m.h, j * BK,
                        m.b);
            tma_load_4d(kl + C::kKVHalf, &tm_klo, bar(C::bKFull + ks), 64,
                        m.h, j * BK, m.b);
          }
          kfill++;
          int vs = vfill % C::VS;
          if (vfill >= C::VS)
            ok = mbar_wait(bar(C::bVEmpty + vs), ((vfill / C::VS) - 1) & 1,
                           abort_flag, p.status, kWaitLimitNs);
          if (!ok) break;
          uint32_t vd = sbase + C::kV + vs * C::kKVTile;
          mbar_arrive_expect_tx(bar(C::bVFull + vs), C::kKVTile);
          tma_load_4d(vd, &tm_v, bar(C::bVFull + vs), 0, m.h, j * BK, m.b);
          tma_load_4d(vd + C::kKVHalf, &tm_v, bar(C::bVFull + vs), 64, m.h,
                      j * BK, m.b);
          vfill++;
        }
      }
      // Drain: every armed load must land before the CTA may exit (on the
      // normal path these phases have completed already).
      for (int s = 0; s < 2; ++s)
        if (qfill[s] > 0)
          mbar_wait(bar(C::bQFull + s), (qfill[s] - 1) & 1, nullptr,
                    p.status, kWaitLimitNs);
      for (int f = kfill - 1; f >= 0 && f >= kfill - C::KS; --f)
        mbar_wait(bar(C::bKFull + f % C::KS), (f / C::KS) & 1, nullptr,
                  p.status, kWaitLimitNs);
      for (int f = vfill - 1; f >= 0 && f >= vfill - C::VS; --f)
        mbar_wait(bar(C::bVFull + f % C::VS), (f / C::VS) & 1, nullptr,
                  p.status, kWaitLimitNs);
    }
    } else if (warp == 13) {
    // ------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, BK, 0, 0);
      const uint32_t idPV = idesc_bf16(128, 128, 0, 1);
      // SW128 descriptors at shared-memory offset 0: K-major (Q, K tiles)
      // and MN-major with the 64-wide d chunks BK * 128 bytes apart (V)
      const uint64_t kdesc0 = sdesc_sw128(sbase, 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(sbase + C::kV, C::kKVHalf, 1024);
      int kc = 0, vc = 0;
      // per sub-tile s, as bits of one word (the issuer's registers are
      // scarce): parity of Q tiles taken (bit s), of P tiles taken (2 + s),
      // of O hand-overs (4 + s), any O handed over yet (6 + s); per unit:
      // Q waited for (8 + s), P.V started (10 + s)
      uint32_t st = 0;
      auto bit = [&](int i) { return (st >> i) & 1u; };
      auto flip = [&](int i) { st ^= 1u << i; };
      bool ok = true;
      for (int n = 0; ok; ++n) {
        ok = mbar_wait(bar(C::bItemFull + (n & 1)), (n >> 1) & 1, abort_flag,
                       p.status, kWaitLimitNs);
        if (!ok) break;
        const int it = item_slot[n & 1];
        mbar_arrive(bar(C::bItemEmpty + (n & 1)));
        if (it < 0) break;
        Item m = get_item(p, it);
        st &= 0xFFu;  // the per-unit bits start clear
        int prev = -1;
        for (int j = m.jhi; j >= m.jlo - 1 && ok; --j) {
          const bool has_j = j >= m.jlo;
          const int ks = kc % C::KS;
          const int vs = vc % C::VS;
          if (has_j) {
            ok = mbar_wait(bar(C::bKFull + ks), (kc / C::KS) & 1, abort_flag,
                           p.status, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
          }
          if (prev >= 0) {
            ok = mbar_wait(bar(C::bVFull + vs), (vc / C::VS) & 1, abort_flag,
                           p.status, kWaitLimitNs);
            if (!ok) break;
            tc_fence_after();
          }
          #pragma unroll
          for (int s = 0; s < 2 && ok; ++s) {
            if (prev >= 0 && active(m, s, prev)) {
              ok = mbar_wait(bar(C::bPFull + s), bit(2 + s), abort_flag,
                             p.status, kWaitLimitNs);
              if (!ok) break;
              flip(2 + s);
              if (!bit(10 + s) && bit(6 + s)) {
                // the previous hand-over of O_s has parity bit(4 + s) ^ 1
                ok = mbar_wait(bar(C::bOEmpty + s), bit(4 + s) ^ 1u,
                               abort_flag, p.status, kWaitLimitNs);
                if (!ok) break;
              }
              tc_fence_after();
              // descriptor start fields are addr >> 4 in the low 14 bits;
              // offsets inside shared memory never carry out of them
              uint64_t vb0;
              asm volatile("mov.b64 %0, %1;" : "=l"(vb0) : "l"(vdesc0));
              const uint64_t vdesc = vb0 + uint64_t((vs * C::kKVTile) >> 4);
              const uint32_t a_tm = tmem + s * 128;        // P over S_s
              const uint32_t d_tm = tmem + 256 + s * 128;  // O_s
#pragma unroll
              for (int k = 0; k < BK / 16; ++k)
                mma_ts(d_tm, a_tm + k * 8, vdesc + uint64_t(k * (2048 >> 4)),
                       idPV, (bit(10 + s) || k > 0) ? 1u : 0u);
              st |= 1u << (10 + s);
            }
            if (has_j && active(m, s, j)) {
              if (!bit(8 + s)) {
                ok = mbar_wait(bar(C::bQReady + s), bit(s), abort_flag,
                               p.status, kWaitLimitNs);
                if (!ok) break;
                flip(s);
                st |= 1u << (8 + s);
                tc_fence_after();
              }
              // the base goes through an opaque move, so the compiler
              // forms each MMA's descriptor here instead of keeping all
              // of them live across the key-block loop
              uint64_t kb0;
              asm volatile("mov.b64 %0, %1;" : "=l"(kb0) : "l"(kdesc0));
              const uint64_t qd = kb0 + uint64_t((C::kQ + s * kTileBytes) >> 4);
              const uint64_t kd = kb0 + uint64_t((C::kK + ks * C::kKVTile) >> 4);
              const uint32_t d_tm = tmem + s * 128;
              const int npass = X3 ? 3 : 1;
#pragma unroll
              for (int pass = 0; pass < npass; ++pass) {
                // pass 0: hi.hi, 1: hi(Q).lo(K), 2: lo(Q).hi(K)
                const uint64_t qa =
                    qd + uint64_t(pass == 2 ? (C::kQlo - C::kQ) >> 4 : 0);
                const uint64_t ka =
                    kd + uint64_t(pass == 1 ? (C::kKlo - C::kK) >> 4 : 0);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  // 16 of d: the 32-byte step inside a 128-byte row, the
                  // 64-wide d chunks a tile apart (Q: 128 rows, K: BK rows)
                  const uint64_t qo =
                      uint64_t(((k >> 2) * kHalfTileBytes + (k & 3) * 32) >> 4);
                  const uint64_t ko =
                      uint64_t(((k >> 2) * C::kKVHalf + (k & 3) * 32) >> 4);
                  mma_ss(d_tm, qa + qo, ka + ko, idS,
                         (pass > 0 || k > 0) ? 1u : 0u);
                }
              }
              mma_commit(bar(C::bSFull + s));
            }
          }
          if (!ok) break;
          if (has_j) {
            mma_commit(bar(C::bKEmpty + ks));
            kc++;
          }
          if (prev >= 0) {
            mma_commit(bar(C::bVEmpty + vs));
            vc++;
          }
          prev = has_j ? j : -1;
        }
        if (!ok) break;
        // a sub-tile that sees no key block issued no MMA: its Q tile is
        // still consumed here, so the rotation is done with it before the
        // epilogue stages the (zero) output in the same buffer
        #pragma unroll
        for (int s = 0; s < 2 && ok; ++s)
          if (m.present[s] && !bit(8 + s)) {
            ok = mbar_wait(bar(C::bQReady + s), bit(s), abort_flag,
                           p.status, kWaitLimitNs);
            flip(s);
          }
        if (!ok) break;
        #pragma unroll
        for (int s = 0; s < 2; ++s)
          if (m.present[s]) {
            mma_commit(bar(C::bOFull + s));
            flip(4 + s);
            st |= 1u << (6 + s);
          }
      }
      // every issued MMA must be complete before TMEM is released
      mma_commit(bar(C::bDone));
      mbar_wait(bar(C::bDone), 0, nullptr, p.status, kWaitLimitNs);
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType,
                                   cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle,
                                   CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

}  // namespace

// [B][N][H][D] bf16 tensor as a 4-D map {D, H, N, B}; box 64 x 1 x rows x 1
// with the 128-byte swizzle (one 64-wide d chunk of `rows` rows per copy).
bool make_bnhd_map(CUtensorMap* m, const void* base, int B, int N, int H,
                   int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {cuuint64_t(kHeadDim), cuuint64_t(H), cuuint64_t(N),
                        cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(kHeadDim) * 2,
                           cuuint64_t(H) * kHeadDim * 2,
                           cuuint64_t(N) * H * kHeadDim * 2};
  cuuint32_t box[4] = {64, 1, cuuint32_t(rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major bf16 [rows][cols] matrix as a 2-D map {cols, rows}; box 64
// columns (128 bytes) x box_rows rows with the 128-byte swizzle.
bool make_2d_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                 int box_rows) {
  return make_2d_map_strided(m, base, rows, cols, cols, box_rows);
}

// The same for a [rows][cols] window of a wider matrix (row stride ld
// elements).
bool make_2d_map_strided(CUtensorMap* m, const void* base, int64_t rows,
                         int64_t cols, int64_t ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 [B][N][H][128] tensor as a 4-D map {D, H, N, B}; box 32 x 1 x 32 x 1
// (one 128-byte column chunk of 32 rows) with the 128-byte swizzle.
bool make_bnhd_f32_map(CUtensorMap* m, const void* base, int B, int N,
                       int H) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {cuuint64_t(kHeadDim), cuuint64_t(H), cuuint64_t(N),
                        cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(kHeadDim) * 4,
                           cuuint64_t(H) * kHeadDim * 4,
                           cuuint64_t(N) * H * kHeadDim * 4};
  cuuint32_t box[4] = {32, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return 148;
  return n;
}

template <bool X3, int BK>
static cudaError_t launch_fwd_impl(const FwdArgs& a, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mo, mklo;
  if (!make_bnhd_map(&mq, a.q, a.B, a.Nq, a.H) ||
      !make_bnhd_map(&mo, a.out, a.B, a.Nq, a.H) ||
      !make_bnhd_map(&mk, a.k_rot, a.B, a.Nk, a.H, BK) ||
      !make_bnhd_map(&mv, a.v, a.B, a.Nk, a.H, BK) ||
      !make_bnhd_map(&mklo, X3 ? a.k_rot_lo : a.k_rot, a.B, a.Nk, a.H, BK))
    return cudaErrorInvalidValue;
  FwdParams p{};
  p.counter = a.counter;
  p.pos_q = a.pos_q;
  p.table = reinterpret_cast<const float2*>(a.table);
  p.kv_lo = a.kv_lo;
  p.kv_hi = a.kv_hi;
  p.row_lo = a.row_lo;
  p.row_hi = a.row_hi;
  p.lo_max = a.lo_max;
  p.hi_min = a.hi_min;
  p.order = a.order;
  p.lse = a.lse;
  p.status = a.status;
  p.B = a.B;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.H = a.H;
  p.k_off = a.k_off;
  p.rope_half = a.rope_half ? 1 : 0;
  p.Tq = (a.Nq + kBlock - 1) / kBlock;
  p.U = (p.Tq + kFwdBlocksPerUnit - 1) / kFwdBlocksPerUnit;
  // heads interleaved per scheduling round: 2 keeps the K/V of the heads
  // in flight L2-resident while still mixing costs across CTAs
  p.G = 1;
  for (int g = 2; g >= 1; --g)
    if (a.H % g == 0) { p.G = g; break; }
  p.total_items = a.B * p.U * a.H;
  p.scale_log2 = kLog2e / sqrtf(float(kHeadDim));
  constexpr int smem = FwdCfg<X3, BK>::kSmem;
  // setmaxnreg hands out exactly the registers the block was launched with;
  // refuse to launch a build whose allocation differs (it could wait
  // forever for registers that do not exist).
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, fwd_tc_kernel<X3, BK>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != 128) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(fwd_tc_kernel<X3, BK>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int grid = std::min(sm_count(), p.total_items);
  {
    const cudaError_t le = launch_dependent(
        fwd_tc_kernel<X3, BK>, dim3(grid), dim3(kThreadsFwd), smem, st, mq, mk,
        mv, mo, mklo, p);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.Nq == 0 || a.Nk == 0 || a.H == 0) return cudaSuccess;
  if (a.block_k == 64)
    return a.qk_x3 ? launch_fwd_impl<true, 64>(a, st)
                   : launch_fwd_impl<false, 64>(a, st);
  if (a.block_k != kBlock) return cudaErrorInvalidValue;
  return a.qk_x3 ? launch_fwd_impl<true, 128>(a, st)
                 : launch_fwd_impl<false, 128>(a, st);
}

}  // namespace lwm
