// attn_bwd_persist.cuh -- persistent form of the RIB attention backward.
//
// The same arithmetic as attn_bwd_kernel in attn_bwd.cuh (gradients of the
// augmented score of the English summary §2.A: dV = P^T dO, dS = P * (dP - D),
// d[Qc,Qp] = tau dS [Kc,Kp], d[Kc,Kp] = tau dS^T [Qc,Qp]), with the same
// warp roles, TMEM columns and per-query-tile pipeline, but one CTA per SM
// walking work items = (unit, key tile) instead of one CTA per item.  Every
// barrier phase is counted across items, so the next item's key tile and
// query stages load, and its S^T/dP^T MMAs start, while the current item's
// last tiles finish; the key tile is double-buffered by item parity and the
// dV/dK accumulators are handed to the drain warps (acc_full) and back
// (acc_free), which write the item's dV, dKc and dKp partial off the compute
// warps' path.
//
// Small windows carry few query tiles per key tile (2 at M = 16, 8 at
// M = 32), so one CTA per item pays its set-up (barrier init, TMEM
// allocation, the pipeline's ramp and drain) on very little work; walking
// items amortises it.  At 96 x 96 windows (72 query tiles per item) the
// per-item kernel is a little faster, and the host picks between the two
// by window size.
#pragma once

#include "attn_bwd.cuh"

namespace rib {
namespace pbwd {

constexpr int kBwdStages = 3;   // query-tile ring (the second key buffer takes the room of one)

struct __align__(1024) BwdSmem {
  uint8_t kc[2][8192];             // key tile, content, [128 rows][64 B], 64B swizzle
  uint8_t kp[2][8192];             // key tile, positional zero-padded to 32 ch (kc + 16 KB)
  uint8_t v[2][8192];              // ([item parity]: the next item's keys load early)
  uint8_t ds[2][32768];            // dS^T [128 keys x 128 queries] bf16, core matrices
  uint8_t qc[kBwdStages][8192];
  uint8_t qp[kBwdStages][8192];    // positional, zero-padded (qc + kBwdStages * 8 KB)
  uint8_t dO[kBwdStages][8192];
  float dq_stage[48 * 128];        // dQ of one query tile, [channel][row], for the bulk reduce
  float lse2[kBwdStages][128];     // -lse * log2(e), tile row order
  float dd[kBwdStages][128];       // -D = -rowsum(dO * O), tile row order
  uint64_t k_full[2], k_free[2];   // key buffers (item parity)
  uint64_t q_full[kBwdStages], q_empty[kBwdStages];
  // pt_free: P^T (and dS^T) in TMEM and the dS buffer written next are free
  uint64_t s_full, s_free, ds_full, pt_free;
  uint64_t dq_full, dq_free;
  uint64_t acc_full, acc_free;     // dV/dK accumulators: an item's MMAs done / read by its epilogue
  int drain_ok[4];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kPBwdSmemBytes = sizeof(BwdSmem) + 1024;
static_assert(kPBwdSmemBytes <= 227 * 1024, "backward shared memory exceeds the per-CTA limit");

// The CTA's work items, in order: item li is it = blockIdx.x + li * gridDim.x,
// unit it / n_tiles, key tile it % n_tiles.  Every barrier phase is counted
// across items (query tile I = li n + i), so the pipeline runs on from one
// item to the next; the keys of item li sit in buffer li & 1.
__device__ __forceinline__ void bwd_item(const BwdParams& p, int it, UnitCoord& u, int& unit,
                                         int& kt) {
  unit = it / p.n_tiles;
  kt = it % p.n_tiles;
  u = decode_unit(unit, p.heads, p.nW, p.nWx);
}

// Warp 12, lane 0: each item's key tile (once the MMAs of the item two back
// have read that buffer), then its query tiles through the ring.
__device__ __forceinline__ void bwd_producer(BwdSmem& sm, const CUtensorMap* tq,
                                             const CUtensorMap* tdo, const CUtensorMap* tqp,
                                             const CUtensorMap* tkp, const CUtensorMap* tlse2,
                                             const CUtensorMap* tdd, const BwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const bool pos = p.rank > 0;
  const int n = p.n_tiles;
  const uint32_t q_bytes = 2u * 8192u + (pos ? 8192u : 0u) + 2u * 512u;
  int I = 0, li = 0, k_issued = 0;
  bool ok = true;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    UnitCoord u;
    int unit, kt;
    bwd_item(p, it, u, unit, kt);
    const int hh = u.head;
    const int by = u.wy * p.M + p.s, bx = u.wx * p.M + p.s;
    const int kb = li & 1;
    if (li >= 2 &&
        !(ok = mbar_wait(&sm.k_free[kb], ((li >> 1) - 1) & 1, ab, p.wait_limit_ns,
                         SITE_BWD_PRODUCER)))
      break;
    {
      int i0, j0;
      tile_origin(kt, p.tiles_x, i0, j0);
      const int y = wrap_once(by + i0, p.H);
      mbar_arrive_expect_tx(&sm.k_full[kb], 2u * 8192u + (pos ? 8192u : 0u));
      for (int c = 0; c < 2; ++c) {
        const int x = wrap_once(bx + j0 + 8 * c, p.W);
        tma_load_5d(sm.kc[kb] + c * 4096, tq, &sm.k_full[kb], 0, p.heads + hh, x, y, u.b);
        tma_load_5d(sm.v[kb] + c * 4096, tq, &sm.k_full[kb], 0, 2 * p.heads + hh, x, y, u.b);
        if (pos) tma_load_4d(sm.kp[kb] + c * 4096, tkp, &sm.k_full[kb], 0, j0 + 8 * c, i0, hh);
      }
      ++k_issued;
    }
    for (int i = 0; i < n; ++i, ++I) {
      const int st = I % kBwdStages, use = I / kBwdStages;
      if (use > 0 &&
          !(ok = mbar_wait(&sm.q_empty[st], (use - 1) & 1, ab, p.wait_limit_ns,
                           SITE_BWD_PRODUCER)))
        break;
      mbar_arrive_expect_tx(&sm.q_full[st], q_bytes);
      int i0, j0;
      tile_origin(i, p.tiles_x, i0, j0);
      const int y = wrap_once(by + i0, p.H);
      for (int c = 0; c < 2; ++c) {
        const int x = wrap_once(bx + j0 + 8 * c, p.W);
        tma_load_5d(sm.qc[st] + c * 4096, tq, &sm.q_full[st], 0, hh, x, y, u.b);
        tma_load_5d(sm.dO[st] + c * 4096, tdo, &sm.q_full[st], 0, hh, x, y, u.b);
        if (pos) tma_load_4d(sm.qp[st] + c * 4096, tqp, &sm.q_full[st], 0, j0 + 8 * c, i0, hh);
        tma_load_4d(&sm.lse2[st][c * 64], tlse2, &sm.q_full[st], x, y, hh, u.b);
        tma_load_4d(&sm.dd[st][c * 64], tdd, &sm.q_full[st], x, y, hh, u.b);
      }
    }
  }
  if (*ab) {
    // Aborted: let every copy this thread started land before the CTA exits
    // (the latest phase of each key buffer and of each ring stage).
    volatile int no_abort = 0;
    for (int q = k_issued - 1; q >= 0 && q >= k_issued - 2; --q)
      mbar_wait(&sm.k_full[q & 1], (q >> 1) & 1, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
    for (int ii = I - 1; ii >= 0 && ii >= I - kBwdStages; --ii)
      mbar_wait(&sm.q_full[ii % kBwdStages], (ii / kBwdStages) & 1, &no_abort, kBwdDrainNs,
                SITE_BWD_DRAIN);
  }
}

// Warp 13 (all lanes; one elected lane issues): S^T = K_aug Q_aug^T and
// dP^T = V dO^T of every query tile, each
// issued as soon as the compute warps have pulled the previous one into
// registers.
__device__ __forceinline__ void bwd_mma_scores(BwdSmem& sm, uint32_t tmem, const BwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const bool pos = p.rank > 0;
  const int n = p.n_tiles;
  bool ok = true;
  int li = 0;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    const int kb = li & 1;
    const uint32_t kc = smem_u32(sm.kc[kb]), kp = smem_u32(sm.kp[kb]), v = smem_u32(sm.v[kb]);
    if (!(ok = warp_wait(&sm.k_full[kb], (li >> 1) & 1, ab, lim, SITE_BWD_MMA))) break;
    for (int i = 0; ok && i < n; ++i) {
      const int I = li * n + i, st = I % kBwdStages;
      ok = warp_wait(&sm.q_full[st], (I / kBwdStages) & 1, ab, lim, SITE_BWD_MMA) &&
           (I == 0 || warp_wait(&sm.s_free, (I - 1) & 1, ab, lim, SITE_BWD_MMA));
      if (!ok) break;
      tc_fence_after();
      // S^T = K_aug Q_aug^T  (M = keys, N = queries, K = 32 + 16)
      const uint64_t a = make_sdesc(kc, 16, 512, kLayoutSW64);
      const uint64_t b = make_sdesc(smem_u32(sm.qc[st]), 16, 512, kLayoutSW64);
      umma_ss3_elect(tmem + kBColS, a, b, a + 2, b + 2, make_sdesc(kp, 16, 512, kLayoutSW64),
                     make_sdesc(smem_u32(sm.qp[st]), 16, 512, kLayoutSW64), kIdescBS,
                     pos ? 1u : 0u);
      // dP^T = V dO^T  (M = keys, N = queries, K = 32)
      const uint64_t av = make_sdesc(v, 16, 512, kLayoutSW64);
      const uint64_t bo = make_sdesc(smem_u32(sm.dO[st]), 16, 512, kLayoutSW64);
      umma_ss3_elect(tmem + kBColDP, av, bo, av + 2, bo + 2, av, bo, kIdescBS, 0u);
      umma_commit_elect(&sm.s_full);
    }
    if (ok) umma_commit_elect(&sm.k_free[kb]);   // this item's key-buffer reads are issued
  }
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
}

// Warp 14 (all lanes; one elected lane issues): dV += P^T dO (A = P^T from
// TMEM) of every query tile of every item; an item's first step overwrites
// dV once the previous item's epilogue has read it (acc_free).  P^T
// (pt_free) and the query stage (q_empty) are released by this warp and
// warp 15 together (two arrivals); after an item's last step the commit to
// acc_full tells the epilogue that dV is complete.
__device__ __forceinline__ void bwd_mma_grads(BwdSmem& sm, uint32_t tmem, const BwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int n = p.n_tiles;
  bool ok = true;
  int li = 0;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    for (int i = 0; ok && i < n; ++i) {
      const int I = li * n + i, st = I % kBwdStages;
      // ds_full(I) implies the stage's tiles have landed: the compute warps
      // waited for them (q_full) before forming P^T and dS.
      if (!(ok = warp_wait(&sm.ds_full, I & 1, ab, lim, SITE_BWD_MMA))) break;
      if (i == 0 && li > 0 &&
          !(ok = warp_wait(&sm.acc_free, (li - 1) & 1, ab, lim, SITE_BWD_MMA)))
        break;
      tc_fence_after();
      const uint32_t dO = smem_u32(sm.dO[st]);
      // dV += P^T dO   (K = queries, 16 per step; A from TMEM)
      umma_ts8_elect(tmem + kBColDV, tmem + kBColP, make_sdesc(dO, 16, 512, kLayoutSW64),
                     1024 >> 4, kIdescBV, i > 0 ? 1u : 0u);
      umma_commit_elect(&sm.pt_free);
      umma_commit_elect(&sm.q_empty[st]);
    }
    if (ok) umma_commit_elect(&sm.acc_full);   // every dV MMA of the item has completed
  }
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
}

// Warp 15 (all lanes; one elected lane issues): dK_aug += dS^T [Qc|Qp] (A =
// dS^T, the dS core matrices read K-major), then dQ_aug = dS [Kc|Kp] (A = the
// same core matrices read MN-major) of every query tile of every item.  Its
// dK commit releases P^T together with warp 14's dV commit, so the compute
// warps cannot form tile I+1 before this warp has taken tile I: ds_full
// never runs ahead of it.  After an item: acc_full (dK complete) and k_free
// (its dQ MMAs, the last readers of the item's keys, are issued).
__device__ __forceinline__ void bwd_mma_dq(BwdSmem& sm, uint32_t tmem, const BwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int n = p.n_tiles;
  const uint32_t lbo_q = smem_u32(sm.qp[0]) - smem_u32(sm.qc[0]);  // [Qc|Qp] atoms
  bool ok = true;
  int li = 0;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    const int kb = li & 1;
    const uint32_t kc = smem_u32(sm.kc[kb]);
    const uint32_t lbo_k = smem_u32(sm.kp[kb]) - kc;                 // [Kc|Kp] atoms
    for (int i = 0; ok && i < n; ++i) {
      const int I = li * n + i, st = I % kBwdStages;
      if (!(ok = warp_wait(&sm.ds_full, I & 1, ab, lim, SITE_BWD_MMA))) break;
      if (i == 0 && li > 0 &&
          !(ok = warp_wait(&sm.acc_free, (li - 1) & 1, ab, lim, SITE_BWD_MMA)))
        break;
      tc_fence_after();
      if (kBwdDkSmem) {
        // A = dS^T read K-major from the dS core matrices in shared memory
        // (key groups of 8 every 128 B, query groups of 8 every 2048 B)
        umma_ss8_elect(tmem + kBColDK,
                       make_sdesc(smem_u32(sm.ds[I & 1]), 2048, 128, kLayoutNone), 4096 >> 4,
                       make_sdesc(smem_u32(sm.qc[st]), lbo_q, 512, kLayoutSW64), 1024 >> 4,
                       kIdescBK, i > 0 ? 1u : 0u);
      } else {
        umma_ts8_elect(tmem + kBColDK, tmem + kBColDST,
                       make_sdesc(smem_u32(sm.qc[st]), lbo_q, 512, kLayoutSW64), 1024 >> 4,
                       kIdescBK, i > 0 ? 1u : 0u);
      }
      umma_commit_elect(&sm.pt_free);
      umma_commit_elect(&sm.q_empty[st]);
      // the single dQ buffer is free once the drain warps pulled tile I-1
      if (I > 0 && !(ok = warp_wait(&sm.dq_free, (I - 1) & 1, ab, lim, SITE_BWD_MMA))) break;
      tc_fence_after();
      const uint32_t ds = smem_u32(sm.ds[I & 1]);
      // step k: 16 queries further in dS (256 B), 16 keys further in [Kc|Kp] (1 KB)
      umma_ss8_elect(tmem + kBColDQ, make_sdesc(ds, 128, 2048, kLayoutNone), 256 >> 4,
                     make_sdesc(kc, lbo_k, 512, kLayoutSW64), 1024 >> 4, kIdescBQ, 0u);
      umma_commit_elect(&sm.dq_full);
    }
    if (ok) {
      umma_commit_elect(&sm.acc_full);    // every dK MMA of the item has completed
      umma_commit_elect(&sm.k_free[kb]);
    }
  }
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
}

// Warps 8-11: drain dQ of every query tile from TMEM into the staging tile
// (lane quarter wq = warp & 3, all 48 channels), then one thread folds the
// tile into the fp32 accumulator with a bulk reduce-add.  After an item's
// last query tile they also write its dV, dKc and dKp partial (key rows
// 32 wq .. 32 wq + 31, once acc_full says every gradient MMA of the item is
// done) and hand the accumulators back (acc_free), off the compute warps'
// path.  The four warps take every decision together (flags in shared
// memory between two named-barrier syncs), so their barrier counts agree.
__device__ __forceinline__ void bwd_drain(BwdSmem& sm, uint32_t tmem, const BwdParams& p,
                                          int wq) {
  volatile int* ab = &sm.abort_flag;
  const int lane = threadIdx.x & 31;
  const bool pos = p.rank > 0;
  const bool leader = wq == 0 && lane == 0;
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  const int row = wq * 32 + lane;
  const uint32_t tile_bytes = 48u * 128u * 4u;
  volatile int* drain_ok = sm.drain_ok;
  const int n = p.n_tiles;
  bool all_ok = true;
  int li = 0;
  for (int item = blockIdx.x; all_ok && item < p.n_items; item += gridDim.x, ++li) {
    const int unit = item / n, kt = item % n;
    for (int it = 0; it < n; ++it) {
      const int I = li * n + it;
      const bool ok = warp_wait(&sm.dq_full, I & 1, ab, p.wait_limit_ns, SITE_BWD_COMPUTE);
      tc_fence_after();
      uint32_t r32[32], r16[16] = {0};
      if (ok) {
        tmem_ld_x32(tmem + lane_off + kBColDQ, r32);
        if (pos) tmem_ld_x16(tmem + lane_off + kBColDQ + 32, r16);
        tmem_wait_ld();
        reg_fence_x32(r32);
        reg_fence_x16(r16);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.dq_free);
      }
      if (lane == 0) drain_ok[wq] = ok ? 1 : 0;
      // the staging tile is free once the previous bulk reduce has read it
      if (leader) tma_store_wait_read_all();
      named_bar_sync(kDrainBar, 128);
      // every drain thread reads the same four flags: one decision for all
      all_ok = drain_ok[0] && drain_ok[1] && drain_ok[2] && drain_ok[3];
      if (all_ok) {
#pragma unroll
        for (int c = 0; c < 32; ++c) sm.dq_stage[c * 128 + row] = __uint_as_float(r32[c]);
#pragma unroll
        for (int c = 0; c < 16; ++c) sm.dq_stage[(32 + c) * 128 + row] = __uint_as_float(r16[c]);
        fence_proxy_async_smem();
      }
      named_bar_sync(kDrainBar, 128);
      if (!all_ok) break;
      if (leader) {
        if (rib_guard((static_cast<size_t>(unit) * p.n_tiles + it + 1) * 48 * 128 - 1,
                      bwd_units(p) * p.n_tiles * 48 * 128, G_BWD_DQ_ACC))
          bulk_reduce_add_f32(p.dq_acc + (static_cast<size_t>(unit) * p.n_tiles + it) * 48 * 128,
                              sm.dq_stage, tile_bytes);
        tma_store_commit();
      }
    }
    if (!all_ok) break;
    // ---- the item's key gradients
    {
      const bool ok = warp_wait(&sm.acc_full, li & 1, ab, p.wait_limit_ns, SITE_BWD_COMPUTE);
      if (lane == 0) drain_ok[wq] = ok ? 1 : 0;
      named_bar_sync(kDrainBar, 128);
      all_ok = drain_ok[0] && drain_ok[1] && drain_ok[2] && drain_ok[3];
      named_bar_sync(kDrainBar, 128);
      if (!all_ok) break;
      tc_fence_after();
      const UnitCoord u = decode_unit(unit, p.heads, p.nW, p.nWx);
      int i0, j0, ii, jl;
      tile_origin(kt, p.tiles_x, i0, j0);
      tile_row_local(row, i0, j0, ii, jl);
      const int y = wrap_once(u.wy * p.M + ii + p.s, p.H);
      const int x = wrap_once(u.wx * p.M + jl + p.s, p.W);
      const size_t pix = (static_cast<size_t>(u.b) * p.H + y) * p.W + x;
      __nv_bfloat16* base = p.dqkv + pix * 3 * p.heads * 32;
      const float t = p.scale;
      uint32_t r32[32], r16[16];
      // one accumulator at a time (these warps run with few registers)
      for (int a = 0; a < 2; ++a) {   // dV, then dKc (scaled by tau)
        tmem_ld_x32(tmem + lane_off + (a == 0 ? kBColDV : kBColDK), r32);
        tmem_wait_ld();
        reg_fence_x32(r32);
        const float f = a == 0 ? 1.f : t;
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(r32[2 * e]) * f, __uint_as_float(r32[2 * e + 1]) * f);
        if (rib_guard(pix * 3 * p.heads * 32 + ((a == 0 ? 2 : 1) * p.heads + u.head) * 32 + 31,
                      static_cast<size_t>(p.B) * p.H * p.W * 3 * p.heads * 32, G_BWD_DQKV))
          store_row64(base + ((a == 0 ? 2 : 1) * p.heads + u.head) * 32, w, p.dqkv_v8 != 0);
      }
      if (pos) {
        tmem_ld_x16(tmem + lane_off + kBColDK + 32, r16);
        tmem_wait_ld();
        reg_fence_x16(r16);
        const size_t kp0 = ((static_cast<size_t>(unit) * p.n_tiles + kt) * 128 + row) * 16;
        uint32_t w16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w16[e] = __float_as_uint(__uint_as_float(r16[e]) * t);
        // the workspace partials are 256-byte aligned: always whole sectors
        if (rib_guard(kp0 + 15, bwd_units(p) * p.n_tiles * 128 * 16, G_BWD_DKP_PART))
          store_row64(p.dkp_part + kp0, w16, true);
      }
      // every read of the accumulators is complete: the next item may overwrite them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_free);
    }
  }
  // the reductions must be complete before the kernel's work is considered done
  if (leader) tma_store_wait_all();
}

// One work item (the CTA's li-th: unit, key tile kt) of a compute warp;
// false on abort.
template <bool kMask>
__device__ __forceinline__ bool bwd_compute_item(BwdSmem& sm, uint32_t tmem, const BwdParams& p,
                                                 const UnitCoord& u, int unit, int kt, int g,
                                                 int wq, int li) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int lane = threadIdx.x & 31;
  const int n = p.n_tiles;
  const int key = wq * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  const float sl = p.scale_log2;
  const uint64_t sl2 = pk2(sl, sl);
  // region mask: bands of this thread's key token.  A warp's 32 keys are a
  // 4 x 8 block and its 64 query columns an 8 x 8 block, so the mask is one
  // warp-uniform decision per query tile (kv); masked blocks have P = dS = 0.
  const bool mask_on = kMask && (u.wy == p.nW / p.nWx - 1 || u.wx == p.nWx - 1);
  int kbr = 0, kbc = 0;
  if (mask_on) {
    int ki0, kj0, ki, kj;
    tile_origin(kt, p.tiles_x, ki0, kj0);
    tile_row_local(key, ki0, kj0, ki, kj);
    kbr = region_band(u.wy * p.M + ki, p.H, p.M, p.s);
    kbc = region_band(u.wx * p.M + kj, p.W, p.M, p.s);
  }
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    const int I = li * n + i;   // query tile counted across items
    const int st = I % kBwdStages;
    bool kv = true;
    if (mask_on) {
      int qi0, qj0;
      tile_origin(i, p.tiles_x, qi0, qj0);
      kv = region_band(u.wy * p.M + qi0, p.H, p.M, p.s) == kbr &&
           region_band(u.wx * p.M + qj0 + 8 * g, p.W, p.M, p.s) == kbc;
    }
    // S^T/dP^T of tile i, and the stage's lse / D rows (written by TMA)
    if (!(ok = warp_wait2(&sm.s_full, I & 1, &sm.q_full[st], (I / kBwdStages) & 1, ab, lim,
                          SITE_BWD_COMPUTE)))
      break;
    tc_fence_after();
    uint32_t s[2][32], dp[2][32];
    tmem_ld_x32(tmem + lane_off + kBColS + 64 * g, s[0]);
    tmem_ld_x32(tmem + lane_off + kBColS + 64 * g + 32, s[1]);
    tmem_ld_x32(tmem + lane_off + kBColDP + 64 * g, dp[0]);
    tmem_ld_x32(tmem + lane_off + kBColDP + 64 * g + 32, dp[1]);
    tmem_wait_ld();
    reg_fence_x32(s[0]);
    reg_fence_x32(s[1]);
    reg_fence_x32(dp[0]);
    reg_fence_x32(dp[1]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.s_free);
    // lse*log2e and D of this query tile
    const float4* lse4 = reinterpret_cast<const float4*>(sm.lse2[st] + 64 * g);
    const float4* dd4 = reinterpret_cast<const float4*>(sm.dd[st] + 64 * g);
    // the whole 64-column slice in registers: P and dS, packed bf16 pairs
    uint32_t pk[32], dk[32];
#pragma unroll
    for (int v4 = 0; v4 < 16; ++v4) {
      const float4 l = lse4[v4];    // -lse*log2e
      const float4 dv = dd4[v4];    // -D
      const uint32_t* sc = &s[v4 >> 3][(v4 & 7) * 4];
      const uint32_t* dc = &dp[v4 >> 3][(v4 & 7) * 4];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const uint64_t nl = h2 ? pk2(l.z, l.w) : pk2(l.x, l.y);
        const uint64_t nd = h2 ? pk2(dv.z, dv.w) : pk2(dv.x, dv.y);
        const uint64_t x2 = ffma2(pk2(__uint_as_float(sc[2 * h2]), __uint_as_float(sc[2 * h2 + 1])),
                                  sl2, nl);
        uint64_t p2;
        if (((2 * v4 + h2) & 7) < kBwdPolyPairs) {
          p2 = exp2_fma2(x2);
        } else {
          p2 = pk2(ex2_approx(lo2(x2)), ex2_approx(hi2(x2)));
        }
        const uint64_t d2 = fmul2(p2, fadd2(pk2(__uint_as_float(dc[2 * h2]),
                                                __uint_as_float(dc[2 * h2 + 1])), nd));
        pk[2 * v4 + h2] = pack_bf16x2(lo2(p2), hi2(p2));
        dk[2 * v4 + h2] = pack_bf16x2(lo2(d2), hi2(d2));
      }
    }
    // P^T and dS^T (TMEM) are free once dV(i-1) and dK(i-1) completed.  The
    // dS buffer i&1 (shared memory) is free once tile i-2's dK and dQ MMAs
    // completed: warp 15 issued those before dK(i-1), and its pt_free commit
    // after dK(i-1) tracks every MMA it issued before, so pt_free covers both.
    if (I > 0 && !(ok = warp_wait(&sm.pt_free, (I - 1) & 1, ab, lim, SITE_BWD_COMPUTE))) break;
    tc_fence_after();
    uint8_t* ds_row = sm.ds[I & 1];
    if (kv) {
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t p8[8], d8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p8[e] = pk[8 * ch + e];
          d8[e] = dk[8 * ch + e];
        }
        tmem_st_x8(tmem + lane_off + kBColP + 32 * g + 8 * ch, p8);
        if (!kBwdDkSmem) tmem_st_x8(tmem + lane_off + kBColDST + 32 * g + 8 * ch, d8);
        const int q = 64 * g + 16 * ch;
        *reinterpret_cast<uint4*>(ds_row + ds_offset(key, q)) =
            make_uint4(d8[0], d8[1], d8[2], d8[3]);
        *reinterpret_cast<uint4*>(ds_row + ds_offset(key, q + 8)) =
            make_uint4(d8[4], d8[5], d8[6], d8[7]);
      }
    } else {
      // a masked block: P = dS = 0 (a store path of its own, so that the
      // unmasked path carries no per-element selects)
      const uint32_t z8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        tmem_st_x8(tmem + lane_off + kBColP + 32 * g + 8 * ch, z8);
        if (!kBwdDkSmem) tmem_st_x8(tmem + lane_off + kBColDST + 32 * g + 8 * ch, z8);
        const int q = 64 * g + 16 * ch;
        *reinterpret_cast<uint4*>(ds_row + ds_offset(key, q)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(ds_row + ds_offset(key, q + 8)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.ds_full);
  }
  return ok;
}

// Warps 0-7: every work item of the CTA in turn.
template <bool kMask>
__device__ __forceinline__ void bwd_compute(BwdSmem& sm, uint32_t tmem, const BwdParams& p, int g,
                                            int wq) {
  int li = 0;
  for (int it = blockIdx.x; it < p.n_items; it += gridDim.x, ++li) {
    UnitCoord u;
    int unit, kt;
    bwd_item(p, it, u, unit, kt);
    if (!bwd_compute_item<kMask>(sm, tmem, p, u, unit, kt, g, wq, li)) return;
  }
}

// grid min(n_items, SMs) (each CTA walks the work items it, it + gridDim.x,
// ...), block kBwdThreads, dynamic smem kPBwdSmemBytes.
// kMask: the shifted-window region mask (a separate instantiation).
template <bool kMask>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_persistent_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                               const __grid_constant__ CUtensorMap tm_dout,
                               const __grid_constant__ CUtensorMap tm_qp,
                               const __grid_constant__ CUtensorMap tm_kp,
                               const __grid_constant__ CUtensorMap tm_lse2,
                               const __grid_constant__ CUtensorMap tm_dd, const BwdParams p) {
  extern __shared__ uint8_t sm_raw_bwd[];
  BwdSmem& sm = *align1024<BwdSmem>(sm_raw_bwd);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.k_full[b], 1);
      mbar_init(&sm.k_free[b], 2);   // warps 13 and 15, after an item's last key reads
    }
    for (int st = 0; st < kBwdStages; ++st) {
      mbar_init(&sm.q_full[st], 1);
      mbar_init(&sm.q_empty[st], 2);   // warps 14 and 15
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 8);
    mbar_init(&sm.ds_full, 8);
    mbar_init(&sm.pt_free, 2);       // dV (warp 14) and dK (warp 15)
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_free, 4);
    mbar_init(&sm.acc_full, 2);      // warps 14 and 15, after an item's last dV / dK MMA
    mbar_init(&sm.acc_free, 4);      // the four drain warps, accumulators read
    mbar_init(&sm.drain, 3);   // one commit from each MMA-issuing warp
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_dout);
    tma_prefetch_desc(&tm_lse2);
    tma_prefetch_desc(&tm_dd);
  }
  if (warp == 14) {
    tmem_alloc(&sm.tmem_base, kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp < 8) {
    regs_inc<kBwdComputeRegs>();
    bwd_compute<kMask>(sm, tmem, p, warp >> 2, warp & 3);
  } else {
    regs_dec<kBwdServiceRegs>();
    if (warp < 12) {
      bwd_drain(sm, tmem, p, warp & 3);
    } else if (warp == 12) {
      if (lane == 0) bwd_producer(sm, &tm_qkv, &tm_dout, &tm_qp, &tm_kp, &tm_lse2, &tm_dd, p);
    } else if (warp == 13) {
      bwd_mma_scores(sm, tmem, p);
    } else if (warp == 14) {
      bwd_mma_grads(sm, tmem, p);
    } else {
      bwd_mma_dq(sm, tmem, p);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 14) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTmemCols);
  }
}

}  // namespace pbwd
}  // namespace rib
