// Backward blockwise packed causal RoPE attention on tcgen05 (sm_100a).
//
// The chain rule of the forward ("LWM：突破 100 万 Token 的开源大模型",
// 配置参数 / 概述 (b); "开源巨兽LWM：如何用RingAttention撬动百万Token多模态
// 世界", 3.1-3.2), organised key-major: a persistent CTA owns one 128-key
// block of one (batch row, head), keeps its dK and dV accumulators in TMEM,
// and visits every 128-query block that can see it (the queries of the same
// packed example at or after the key). Per query block i, with P recomputed
// from the forward's logsumexp (scores in log2 units):
//   S^T  = K~ Q~_i^T            (tcgen05, TMEM region A, cols   0..127)
//   dP^T = V dO_i^T             (tcgen05, TMEM region B, cols 128..255)
//   P^T  = 2^(S^T c - lse_i log2 e) (masked; computed as soon as S^T lands,
//          while dP^T is still on the tensor pipe), dS^T = P^T (dP^T - D_i)
//          written back as bf16 over the first 64 columns of A and B
//   dV  += P^T dO_i, dK~ += dS^T Q~_i   (A operands read from TMEM)
//   dQ~_i = dS K~               (A = dS, staged in shared memory; result in
//          region B once dK has read dS^T, so region A is free for the next
//          S^T at once; added to an fp32 accumulator in global memory by
//          TMA reduce-add, staged in the block's then-dead Q~/dO buffers)
// Queries and keys arrive pre-rotated (R(pos) q, R(pos) k); dK = R(-pos)
// (dK~ / sqrt(D)) in the epilogue, dQ the same in the conversion kernel.
//
// Warps: 0-7 compute (thread = key row = TMEM lane; warps w and w + 4
// share the lanes and split the 128 columns; they also move each block's
// dQ out of TMEM into shared memory right after its MMA), 8-11 dQ
// reduce-add and per-block (lse, D) staging, 12 TMA producer, 13 tcgen05
// issuer + TMEM owner, 14-15 idle (complete the warpgroup for setmaxnreg).
#include <cuda.h>

#include "aux_kernels.cuh"
#include "tc_kernels.cuh"

namespace lwm {
namespace {

constexpr int kThreadsBwd = 16 * 32;
constexpr int kLaunchRegsBwd = 128;   // 65536 / 512
// two compute warpgroups, the dQ warpgroup, the producer/MMA warpgroup
constexpr int kRegsCompute = 152, kRegsDq = 128, kRegsMiscBwd = 80;
static_assert(2 * kRegsCompute + kRegsDq + kRegsMiscBwd == 4 * kLaunchRegsBwd,
              "register split must equal the launch allocation");
constexpr int kTile = kBlock * kHeadDim * 2;   // 32 KB
constexpr int kHalf = kTile / 2;
constexpr uint64_t kWaitNs = 4000000000ull;

// shared memory map (bytes); tiles 1024-aligned
constexpr int kSK = 0, kSV = kTile, kSQ = 2 * kTile, kSDO = 4 * kTile,
              kSDS = 6 * kTile, kSAux = 7 * kTile,  // lse2[2][128], D[2][128]
              kSBars = kSAux + 4 * 128 * 4;
enum {
  bKVFull = 0, bKVEmpty, bQFull0, bQFull1, bQEmpty0, bQEmpty1, bAux0, bAux1,
  bStFull, bDptFull, bPFull, bDqFull, bDqEmpty, bAccFull, bAccEmpty, bDoneB,
  bItemFull0, bItemFull1, bItemEmpty0, bItemEmpty1, bDqStaged, bDsFull,
  kNumBarsB
};
constexpr int kSMisc = kSBars + kNumBarsB * 8;
constexpr int kSmemBwd = kSMisc + 16;   // tmem addr, abort, 2 work slots

struct BwdParams {
  int32_t* counter;
  const int32_t* col_lo;
  const int32_t* col_hi;
  const int32_t* klo_max;
  const int32_t* khi_min;
  const int32_t* pos_k;
  const float2* table;
  const int32_t* q_lo;
  const int32_t* q_hi;
  const int32_t* order;
  const float* lse;
  const float* delta;
  float* dq_acc;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dk_acc;
  float* dv_acc;
  int* status;
  int B, Nq, Nk, H, Tk, G, q_off, total_items;
  int rope_half;
  float scale_log2, scale;
};

struct BItem {
  int b, h, j, qlo, qhi;
};

__device__ __forceinline__ BItem get_bitem(const BwdParams& p, int it) {
  BItem m;
  const int per_group = p.G * p.B * p.Tk;
  const int hg = it / per_group;
  const int rem = it - hg * per_group;
  const int r = rem / p.G;
  m.h = hg * p.G + (rem - r * p.G);
  const int unit = p.order[r];
  m.b = unit / p.Tk;
  m.j = unit - m.b * p.Tk;
  m.qlo = p.q_lo[unit];
  m.qhi = p.q_hi[unit];
  return m;
}

__global__ void __launch_bounds__(kThreadsBwd, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq,
              const BwdParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + kSBars + 8u * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kSMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSMisc + 4);
  // two-slot ring of work units (producer -> other roles)
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + kSMisc + 8);
  float* aux_lse = reinterpret_cast<float*>(smem + kSAux);        // [2][128]
  float* aux_del = aux_lse + 2 * 128;                             // [2][128]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (sbase & 1023) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicMax(p.status, LWM_ERR_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(bar(bKVFull), 1);
    mbar_init(bar(bKVEmpty), 1);
    mbar_init(bar(bQFull0), 1);
    mbar_init(bar(bQFull1), 1);
    // a Q~/dO stage is free once its MMAs are done (one commit) and the dQ
    // warps have reduced dQ of that block out of it (one arrive per warp)
    mbar_init(bar(bQEmpty0), 5);
    mbar_init(bar(bQEmpty1), 5);
    mbar_init(bar(bAux0), 128);
    mbar_init(bar(bAux1), 128);
    mbar_init(bar(bStFull), 1);
    mbar_init(bar(bDptFull), 1);
    mbar_init(bar(bPFull), 8);
    mbar_init(bar(bDsFull), 8);
    mbar_init(bar(bDqFull), 1);
    // the compute warps drain dQ from TMEM into the stage buffers
    mbar_init(bar(bDqEmpty), 8);
    mbar_init(bar(bDqStaged), 8);
    mbar_init(bar(bAccFull), 1);
    mbar_init(bar(bAccEmpty), 8);
    mbar_init(bar(bDoneB), 1);
    mbar_init(bar(bItemFull0), 1);
    mbar_init(bar(bItemFull1), 1);
    // consumers: 8 compute warps, 4 dQ warps, the MMA lane
    mbar_init(bar(bItemEmpty0), 13);
    mbar_init(bar(bItemEmpty1), 13);
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
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tA = tmem, tB = tmem + 128, tC = tmem + 256, tD = tmem + 384;
  const int nitems = p.total_items;

  if (warp < 8) {
    // ---------------------------------------------------- compute (keys)
    // two warps per TMEM lane quadrant: warp w owns key rows 32 (w % 4) ..
    // +31 and the 64 query columns (or d columns) of half ch = w / 4
    regs_inc<kRegsCompute>();
    const int q4 = warp & 3, ch = warp >> 2;
    const int r = q4 * 32 + lane;  // key row of the block = TMEM lane
    const uint32_t lane_off = uint32_t(q4 * 32) << 16;
    int g = 0, n = 0;
    bool ok = true;
    for (int u = 0; ok; ++u) {
      ok = mbar_wait(bar(bItemFull0 + (u & 1)), (u >> 1) & 1, abort_flag,
                     p.status, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int it = item_slot[u & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bItemEmpty0 + (u & 1)));
      if (it < 0) break;
      const BItem m = get_bitem(p, it);
      const int64_t rowbase = int64_t(m.b) * p.Nk;
      const int k0 = m.j * kBlock;
      const int kj = k0 + r;
      const bool valid_k = kj < p.Nk;
      // key kj is seen by the queries lo_k .. hi_k (global indices; none
      // for a key >= Nk)
      const int lo_k = valid_k ? __ldg(p.col_lo + rowbase + kj) : 1;
      const int hi_k = valid_k ? __ldg(p.col_hi + rowbase + kj) : 0;
      const int klo_max = __ldg(p.klo_max + m.b * p.Tk + m.j);
      const int khi_min = __ldg(p.khi_min + m.b * p.Tk + m.j);
      for (int i = m.qlo; i <= m.qhi && ok; ++i) {
        const int st = g & 1;
        ok = mbar_wait(bar(bStFull), g & 1, abort_flag, p.status, kWaitNs);
        if (ok)
          ok = mbar_wait(bar(bAux0 + st), (g >> 1) & 1, abort_flag, p.status,
                         kWaitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int q0 = p.q_off + i * kBlock;  // global index of query 0
        // every key of the block seen by every query of the block
        const bool full = klo_max <= q0 && khi_min >= q0 + kBlock - 1;
        const float* ls = aux_lse + st * 128 + ch * 64;
        const float* dl = aux_del + st * 128 + ch * 64;
        uint8_t* dsrow = smem + kSDS + ch * kHalf + r * 128;
        // this warp's 64 query columns of S^T / dP^T start at column ch*64;
        // its bf16 P^T and dS^T go to the first 32 of those columns (inside
        // its own range, so the other half's loads are never overwritten)
        const uint32_t colA = tA + lane_off + ch * 64;
        const uint32_t colB = tB + lane_off + ch * 64;
        // phase 1 (while dP^T is still on the tensor pipe; its end lets dV
        // start while phase 2 runs):
        // P^T = 2^(S^T c - lse log2 e), masked; bf16 copy over S^T
        float pf[2][32];
        {
          uint32_t sv[2][32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) tmem_ld32(colA + cc * 32, sv[cc]);
          tmem_wait_ld();
          if (!full) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int qb = q0 + ch * 64 + cc * 32;
              const int lo = lo_k - qb, hi = hi_k - qb;
#pragma unroll
              for (int x = 0; x < 32; ++x)
                sv[cc][x] = (x >= lo && x <= hi) ? sv[cc][x] : 0xff800000u;
            }
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t pp[16];
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
              const float4 l4 = *reinterpret_cast<const float4*>(ls + cc * 32 + x);
              const float2 t0 = fma2(make_float2(__uint_as_float(sv[cc][x]),
                                                 __uint_as_float(sv[cc][x + 1])),
                                     make_float2(p.scale_log2, p.scale_log2),
                                     make_float2(-l4.x, -l4.y));
              const float2 t1 = fma2(make_float2(__uint_as_float(sv[cc][x + 2]),
                                                 __uint_as_float(sv[cc][x + 3])),
                                     make_float2(p.scale_log2, p.scale_log2),
                                     make_float2(-l4.z, -l4.w));
              pf[cc][x] = ex2(t0.x);
              pf[cc][x + 1] = ex2(t0.y);
              pf[cc][x + 2] = ex2(t1.x);
              pf[cc][x + 3] = ex2(t1.y);
              pp[x >> 1] = pack_bf16x2(pf[cc][x], pf[cc][x + 1]);
              pp[(x >> 1) + 1] = pack_bf16x2(pf[cc][x + 2], pf[cc][x + 3]);
            }
            tmem_st16(colA + cc * 16, pp);
          }
        }
        // P^T is in TMEM: dV runs on the tensor pipe while dS is formed
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bPFull));
        // phase 2: dS^T = P^T (dP^T - D) once dP^T has landed
        ok = mbar_wait(bar(bDptFull), g & 1, abort_flag, p.status, kWaitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          tmem_wait_st();
          break;
        }
        tc_fence_after();
        {
          uint32_t dv[2][32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) tmem_ld32(colB + cc * 32, dv[cc]);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t pd[16];
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
              const float4 d4 = *reinterpret_cast<const float4*>(dl + cc * 32 + x);
              const float ds0 = pf[cc][x] * (__uint_as_float(dv[cc][x]) - d4.x);
              const float ds1 = pf[cc][x + 1] * (__uint_as_float(dv[cc][x + 1]) - d4.y);
              const float ds2 = pf[cc][x + 2] * (__uint_as_float(dv[cc][x + 2]) - d4.z);
              const float ds3 = pf[cc][x + 3] * (__uint_as_float(dv[cc][x + 3]) - d4.w);
              pd[x >> 1] = pack_bf16x2(ds0, ds1);
              pd[(x >> 1) + 1] = pack_bf16x2(ds2, ds3);
            }
            tmem_st16(colB + cc * 16, pd);
            // dS row r, queries ch*64 + cc*32 .. +31: the query half ch of
            // the tile, 16-byte chunks cc*4 .. +3 of that 128-byte row
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int lc = cc * 4 + e;
              *reinterpret_cast<uint4*>(dsrow + ((lc ^ (r & 7)) << 4)) =
                  make_uint4(pd[4 * e], pd[4 * e + 1], pd[4 * e + 2],
                             pd[4 * e + 3]);
            }
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bDsFull));
        // dQ~ of this block: once its MMA is done (it follows dV and dK),
        // this warp moves its 64 d columns out of TMEM (then TMEM is free
        // for the next dP^T) into the block's own Q~ / dO stage buffers,
        // which its MMAs no longer read, as two 32-column 4 KB boxes
        // (128-byte swizzle) of its 32 rows; the dQ warps reduce-add them
        ok = mbar_wait(bar(bDqFull), g & 1, abort_flag, p.status, kWaitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t dqv[2][32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
            tmem_ld32(tB + lane_off + ch * 64 + cc * 32, dqv[cc]);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(bDqEmpty));
          const int qoff = kSQ + st * kTile, ooff = kSDO + st * kTile;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * ch + cc;  // 32-column chunk of d
            const int box = (c < 2 ? qoff : ooff) + (q4 * 2 + (c & 1)) * 4096;
            uint8_t* rowp = smem + box + lane * 128;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              *reinterpret_cast<uint4*>(rowp + ((e ^ (lane & 7)) << 4)) =
                  make_uint4(dqv[cc][4 * e], dqv[cc][4 * e + 1],
                             dqv[cc][4 * e + 2], dqv[cc][4 * e + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(bDqStaged));
        }
        ++g;
      }
      if (!ok) break;
      // ------------------------------------------------ item epilogue
      ok = mbar_wait(bar(bAccFull), n & 1, abort_flag, p.status, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int64_t orow = ((rowbase + (valid_k ? kj : 0)) * p.H + m.h) * kHeadDim;
      // a key block no query sees issued no MMA: its accumulators hold
      // nothing of this item (bf16 mode writes zeros, fp32 mode adds none)
      const bool seen = m.qlo <= m.qhi;
      const float4* trow = reinterpret_cast<const float4*>(
          p.table + int64_t(valid_k && p.pos_k ? __ldg(p.pos_k + rowbase + kj)
                                               : 0) *
                        (kHeadDim / 2));
      if (p.dk_acc) {
        // fp32 accumulators carried across calls: add dV and the unscaled,
        // rotated dK~ (this thread owns key row kj, d columns ch*64 .. +63)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = ch * 64 + (c & 1) * 32;
          uint32_t v[32];
          tmem_ld32((c < 2 ? tC : tD) + lane_off + col, v);
          tmem_wait_ld();
          if (valid_k && seen) {
            float4* dst = reinterpret_cast<float4*>(
                (c < 2 ? p.dv_acc : p.dk_acc) + orow + col);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 a = dst[e];
              a.x += __uint_as_float(v[4 * e]);
              a.y += __uint_as_float(v[4 * e + 1]);
              a.z += __uint_as_float(v[4 * e + 2]);
              a.w += __uint_as_float(v[4 * e + 3]);
              dst[e] = a;
            }
          }
        }
      } else {
        // dV: d columns ch*64 .. +63
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = ch * 64 + c * 32;
          uint32_t v[32];
          tmem_ld32(tC + lane_off + col, v);
          tmem_wait_ld();
          if (!seen)
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = 0u;
          if (valid_k) {
            uint4* dst = reinterpret_cast<uint4*>(p.dv + orow + col);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(
                  pack_bf16x2(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                  pack_bf16x2(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                  pack_bf16x2(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                  pack_bf16x2(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
          }
        }
        if (p.rope_half) {
          // pair k = (dim k, dim k + 64): this warp takes columns ch*32 ..
          // +31 with (ch+2)*32 .. +31, i.e. pairs ch*32 .. ch*32 + 31
          uint32_t va[32], vb[32];
          tmem_ld32(tD + lane_off + ch * 32, va);
          tmem_ld32(tD + lane_off + (ch + 2) * 32, vb);
          tmem_wait_ld();
          if (!seen)
#pragma unroll
            for (int x = 0; x < 32; ++x) va[x] = vb[x] = 0u;
          if (valid_k) {
            uint32_t oa[16], ob[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {  // pairs ch*32 + 2e, 2e + 1
              const float4 cs = __ldg(trow + ch * 16 + e);
              const float a0 = __uint_as_float(va[2 * e]) * p.scale;
              const float a1 = __uint_as_float(va[2 * e + 1]) * p.scale;
              const float b0 = __uint_as_float(vb[2 * e]) * p.scale;
              const float b1 = __uint_as_float(vb[2 * e + 1]) * p.scale;
              // R(-pos): (a, b) -> (a c + b s, b c - a s)
              oa[e] = pack_bf16x2(fmaf(a0, cs.x, b0 * cs.y),
                                  fmaf(a1, cs.z, b1 * cs.w));
              ob[e] = pack_bf16x2(fmaf(b0, cs.x, -a0 * cs.y),
                                  fmaf(b1, cs.z, -a1 * cs.w));
            }
            uint4* da = reinterpret_cast<uint4*>(p.dk + orow + ch * 32);
            uint4* db = reinterpret_cast<uint4*>(p.dk + orow + (ch + 2) * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              da[e] = make_uint4(oa[4 * e], oa[4 * e + 1], oa[4 * e + 2],
                                 oa[4 * e + 3]);
              db[e] = make_uint4(ob[4 * e], ob[4 * e + 1], ob[4 * e + 2],
                                 ob[4 * e + 3]);
            }
          }
        } else {
          // interleaved pairs (2k, 2k+1): d columns ch*64 .. +63
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int col = ch * 64 + c * 32;
            uint32_t v[32];
            tmem_ld32(tD + lane_off + col, v);
            tmem_wait_ld();
            if (!seen)
#pragma unroll
              for (int x = 0; x < 32; ++x) v[x] = 0u;
            if (valid_k) {
              uint32_t o[16];
#pragma unroll
              for (int e = 0; e < 8; ++e) {  // pairs col/2 + 2e, 2e+1
                const float4 cs = __ldg(trow + col / 4 + e);
                const float a0 = __uint_as_float(v[4 * e]) * p.scale;
                const float b0 = __uint_as_float(v[4 * e + 1]) * p.scale;
                const float a1 = __uint_as_float(v[4 * e + 2]) * p.scale;
                const float b1 = __uint_as_float(v[4 * e + 3]) * p.scale;
                // R(-pos): (a, b) -> (a c + b s, b c - a s)
                o[2 * e] = pack_bf16x2(fmaf(a0, cs.x, b0 * cs.y),
                                       fmaf(b0, cs.x, -a0 * cs.y));
                o[2 * e + 1] = pack_bf16x2(fmaf(a1, cs.z, b1 * cs.w),
                                           fmaf(b1, cs.z, -a1 * cs.w));
              }
              uint4* dst = reinterpret_cast<uint4*>(p.dk + orow + col);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2],
                                    o[4 * e + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bAccEmpty));
      ++n;
    }
  } else if (warp < 12) {
    // ---------------------------------------------------- dQ + staging
    regs_dec<kRegsDq>();
    const int r = (warp - 8) * 32 + lane;  // query row of the block
    int g = 0;
    bool ok = true;
    int pb = 0, ph = 0, pq0 = 0;  // the block whose dQ is pending
    // dQ of block t, staged by the compute warps in the block's own Q~ and
    // dO stage buffers (this warp's 32 rows as four 32-column 4 KB boxes,
    // 128-byte swizzle): a TMA reduce-add of each box into the fp32
    // accumulator; the stage goes back to the producer after the reduce
    // has read it.
    const int wq = warp - 8;
    int pst = 0;  // stage of the pending block
    auto flush = [&](int t) -> bool {
      // the compute warps have staged dQ of block t in its stage buffers
      bool w = mbar_wait(bar(bDqStaged), t & 1, abort_flag, p.status,
                         kWaitNs);
      w = __all_sync(0xffffffffu, w);
      if (!w) return false;
      const int qoff = kSQ + pst * kTile, ooff = kSDO + pst * kTile;
      if (lane == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int box = (c < 2 ? qoff : ooff) + (wq * 2 + (c & 1)) * 4096;
          tma_reduce_add_4d(&tm_dq, sbase + box, c * 32, ph, pq0 + wq * 32,
                            pb);
        }
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(bar(bQEmpty0 + pst));
      }
      __syncwarp();
      return true;
    };
    for (int u = 0; ok; ++u) {
      ok = mbar_wait(bar(bItemFull0 + (u & 1)), (u >> 1) & 1, abort_flag,
                     p.status, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int it = item_slot[u & 1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bItemEmpty0 + (u & 1)));
      if (it < 0) break;
      const BItem m = get_bitem(p, it);
      const float* lse_bh = p.lse + (int64_t(m.b) * p.H + m.h) * p.Nq;
      const float* del_bh = p.delta + (int64_t(m.b) * p.H + m.h) * p.Nq;
      for (int i = m.qlo; i <= m.qhi && ok; ++i) {
        const int st = g & 1;
        const int q = i * kBlock + r;
        // stage (lse log2 e, D) of this block; the slot's previous user
        // (block g-2) finished with it before its dQ, flushed last round
        aux_lse[st * 128 + r] = q < p.Nq ? __ldg(lse_bh + q) * kLog2e : 0.f;
        aux_del[st * 128 + r] = q < p.Nq ? __ldg(del_bh + q) : 0.f;
        mbar_arrive(bar(bAux0 + st));
        if (g > 0) ok = flush(g - 1);
        pb = m.b;
        ph = m.h;
        pq0 = i * kBlock;
        pst = st;
        ++g;
      }
    }
    if (ok && g > 0) flush(g - 1);
    if (lane == 0) bulk_wait0();
  } else {
    // warps 8-11 share one register budget, then split: 8 producer,
    // 9 MMA, 10-11 idle
    regs_dec<kRegsMiscBwd>();
    if (warp == 12) {
    // ---------------------------------------------------- TMA producer
    if (lane == 0) {
      int g = 0, n = 0;
      bool ok = true;
      for (int u = 0; ok; ++u) {
        if (u >= 2) {
          ok = mbar_wait(bar(bItemEmpty0 + (u & 1)), ((u >> 1) - 1) & 1,
                         abort_flag, p.status, kWaitNs);
          if (!ok) break;
        }
        int it = atomicAdd(p.counter, 1);
        if (it >= nitems) it = -1;
        item_slot[u & 1] = it;
        mbar_arrive(bar(bItemFull0 + (u & 1)));
        if (it < 0) break;
        const BItem m = get_bitem(p, it);
        if (n > 0)
          ok = mbar_wait(bar(bKVEmpty), (n - 1) & 1, abort_flag, p.status,
                         kWaitNs);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(bKVFull), 2 * kTile);
        const int k0 = m.j * kBlock;
        tma_load_4d(sbase + kSK, &tm_k, bar(bKVFull), 0, m.h, k0, m.b);
        tma_load_4d(sbase + kSK + kHalf, &tm_k, bar(bKVFull), 64, m.h, k0,
                    m.b);
        tma_load_4d(sbase + kSV, &tm_v, bar(bKVFull), 0, m.h, k0, m.b);
        tma_load_4d(sbase + kSV + kHalf, &tm_v, bar(bKVFull), 64, m.h, k0,
                    m.b);
        ++n;
        for (int i = m.qlo; i <= m.qhi && ok; ++i) {
          const int st = g & 1;
          if (g >= 2)
            ok = mbar_wait(bar(bQEmpty0 + st), ((g >> 1) - 1) & 1, abort_flag,
                           p.status, kWaitNs);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(bQFull0 + st), 2 * kTile);
          const int q0 = i * kBlock;
          const uint32_t qd = sbase + kSQ + st * kTile;
          const uint32_t od = sbase + kSDO + st * kTile;
          tma_load_4d(qd, &tm_q, bar(bQFull0 + st), 0, m.h, q0, m.b);
          tma_load_4d(qd + kHalf, &tm_q, bar(bQFull0 + st), 64, m.h, q0, m.b);
          tma_load_4d(od, &tm_do, bar(bQFull0 + st), 0, m.h, q0, m.b);
          tma_load_4d(od + kHalf, &tm_do, bar(bQFull0 + st), 64, m.h, q0,
                      m.b);
          ++g;
        }
      }
      // drain loads that may still be in flight
      if (n > 0)
        mbar_wait(bar(bKVFull), (n - 1) & 1, nullptr, p.status, kWaitNs);
      for (int f = g - 1; f >= 0 && f >= g - 2; --f)
        mbar_wait(bar(bQFull0 + (f & 1)), (f >> 1) & 1, nullptr, p.status,
                  kWaitNs);
    }
    } else if (warp == 13) {
    // ---------------------------------------------------- tcgen05 issuer
    if (lane == 0) {
      const uint32_t idKK = idesc_bf16(128, 128, 0, 0);  // A, B K-major
      const uint32_t idKM = idesc_bf16(128, 128, 0, 1);  // B MN-major
      const uint32_t idMM = idesc_bf16(128, 128, 1, 1);  // A, B MN-major
      int g = 0, n = 0;
      bool ok = true;
      for (int u = 0; ok; ++u) {
        ok = mbar_wait(bar(bItemFull0 + (u & 1)), (u >> 1) & 1, abort_flag,
                       p.status, kWaitNs);
        if (!ok) break;
        const int it = item_slot[u & 1];
        mbar_arrive(bar(bItemEmpty0 + (u & 1)));
        if (it < 0) break;
        const BItem m = get_bitem(p, it);
        ok = mbar_wait(bar(bKVFull), n & 1, abort_flag, p.status, kWaitNs);
        if (!ok) break;
        bool first_q = true;
        for (int i = m.qlo; i <= m.qhi && ok; ++i) {
          const int st = g & 1;
          ok = mbar_wait(bar(bQFull0 + st), (g >> 1) & 1, abort_flag,
                         p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qb = sbase + kSQ + st * kTile;
          const uint32_t ob = sbase + kSDO + st * kTile;
          // S^T = K~ Q~^T into A: A's last readers (dV of block g-1, the
          // compute warps' loads) are done by issue order / p_full
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
            mma_ss(tA, sdesc_sw128(sbase + kSK + off, 16, 1024),
                   sdesc_sw128(qb + off, 16, 1024), idKK, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(bStFull));
          // dP^T = V dO^T into B once dQ of block g-1 has left it
          if (g > 0)
            ok = mbar_wait(bar(bDqEmpty), (g - 1) & 1, abort_flag, p.status,
                           kWaitNs);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
            mma_ss(tB, sdesc_sw128(sbase + kSV + off, 16, 1024),
                   sdesc_sw128(ob + off, 16, 1024), idKK, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(bDptFull));
          ok = mbar_wait(bar(bPFull), g & 1, abort_flag, p.status, kWaitNs);
          if (ok && first_q && n > 0)
            ok = mbar_wait(bar(bAccEmpty), (n - 1) & 1, abort_flag, p.status,
                           kWaitNs);
          if (!ok) break;
          tc_fence_after();
          // bf16 P^T / dS^T of queries 64.. sit 32 columns further on
          // (each compute warp packs its half inside its own S^T columns)
#pragma unroll
          for (int k = 0; k < 8; ++k)  // dV += P^T dO
            mma_ts(tC, tA + 8 * k + (k >= 4 ? 32 : 0),
                   sdesc_sw128(ob + 2048 * k, kHalf, 1024), idKM,
                   (!first_q || k > 0) ? 1u : 0u);
          ok = mbar_wait(bar(bDsFull), g & 1, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k)  // dK~ += dS^T Q~
            mma_ts(tD, tB + 8 * k + (k >= 4 ? 32 : 0),
                   sdesc_sw128(qb + 2048 * k, kHalf, 1024), idKM,
                   (!first_q || k > 0) ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < 8; ++k)  // dQ~ = dS K~, into B after dK read it
            mma_ss(tB, sdesc_sw128(sbase + kSDS + 2048 * k, kHalf, 1024),
                   sdesc_sw128(sbase + kSK + 2048 * k, kHalf, 1024), idMM,
                   k > 0 ? 1u : 0u);
          mma_commit(bar(bDqFull));
          mma_commit(bar(bQEmpty0 + st));
          first_q = false;
          ++g;
        }
        if (!ok) break;
        // a key block no query sees issued no MMA and so never waited for
        // the previous item's epilogue: wait here, or bAccFull would
        // complete a second phase before the compute warps saw the first
        if (first_q && n > 0)
          ok = mbar_wait(bar(bAccEmpty), (n - 1) & 1, abort_flag, p.status,
                         kWaitNs);
        if (!ok) break;
        mma_commit(bar(bAccFull));
        mma_commit(bar(bKVEmpty));
        ++n;
      }
      mma_commit(bar(bDoneB));
      mbar_wait(bar(bDoneB), 0, nullptr, p.status, kWaitNs);
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

}  // namespace

cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.Nq == 0 || a.Nk == 0 || a.H == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (!make_bnhd_map(&mq, a.q_rot, a.B, a.Nq, a.H) ||
      !make_bnhd_map(&mk, a.k_rot, a.B, a.Nk, a.H) ||
      !make_bnhd_map(&mv, a.v, a.B, a.Nk, a.H) ||
      !make_bnhd_map(&mdo, a.dout, a.B, a.Nq, a.H) ||
      !make_bnhd_f32_map(&mdq, a.dq_acc, a.B, a.Nq, a.H))
    return cudaErrorInvalidValue;
  if (!a.dk_acc != !a.dv_acc) return cudaErrorInvalidValue;
  BwdParams p{};
  p.counter = a.counter;
  p.col_lo = a.col_lo;
  p.col_hi = a.col_hi;
  p.klo_max = a.klo_max;
  p.khi_min = a.khi_min;
  p.pos_k = a.pos_k;
  p.table = reinterpret_cast<const float2*>(a.table);
  p.q_lo = a.q_lo;
  p.q_hi = a.q_hi;
  p.order = a.order;
  p.lse = a.lse;
  p.delta = a.delta;
  p.dq_acc = a.dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.dk_acc = a.dk_acc;
  p.dv_acc = a.dv_acc;
  p.status = a.status;
  p.B = a.B;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.H = a.H;
  p.q_off = a.q_off;
  p.rope_half = a.rope_half ? 1 : 0;
  p.Tk = (a.Nk + kBlock - 1) / kBlock;
  // one head per scheduling round: the fp32 dQ accumulator, Q~ and dO of
  // a head (16 + 8 + 8 MB at 32K) then stay L2-resident while ~148 key
  // blocks of that head reduce into it (4 heads at once measured 7% slower
  // from DRAM read-modify-write of dQ)
  p.G = 1;
  p.total_items = a.B * p.Tk * a.H;
  p.scale = 1.f / sqrtf(float(kHeadDim));
  p.scale_log2 = kLog2e * p.scale;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, bwd_tc_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegsBwd) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(bwd_tc_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBwd);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), p.total_items);
  {
    const cudaError_t le = launch_dependent(
        bwd_tc_kernel, dim3(grid), dim3(kThreadsBwd), kSmemBwd, st, mq, mk, mv,
        mdo, mdq, p);
    if (le != cudaSuccess) return le;
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace lwm
