// attn_bwd.cuh -- RIB window attention backward on tcgen05 tensor cores.
//
// Gradients of the forward in attn_fwd.cuh (the augmented score of the
// English summary §2.A, score equation).  With P = softmax(S),
// S = tau [Qc,Qp][Kc,Kp]^T and D = rowsum(dO * O):
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//   d[Qc,Qp] = tau dS [Kc,Kp],  d[Kc,Kp] = tau dS^T [Qc,Qp].
// The positional parts dQp, dKp are summed over batch entries and windows
// because one Qp/Kp set serves every window of the geometry.
//
// Kernels, in launch order:
//   bwd_preprocess   D and lse*log2(e) per pixel and head; zeroes dQ acc
//   attn_bwd_kernel  one CTA per (key tile, unit): keeps K, V, Kp of its 128
//                    keys in shared memory and streams the unit's query
//                    tiles; dK, dV accumulate in TMEM; dQ partials go to an
//                    fp32 accumulator through one bulk TMA reduce-add per
//                    query tile (the order of the key tiles' adds follows
//                    CTA scheduling, so dQ is not bit-reproducible)
//   dq_finalize      dQ content channels -> bf16 dqkv at the rolled pixels
//   posgrad_reduce   fixed-order sums over (batch, window) of dQp, dKp
//
// attn_bwd_kernel, 512 threads (4 warpgroups):
//   warps 0-7   compute: thread = key row (TMEM lane), warps 0-3 take query
//               columns 0-63 and warps 4-7 columns 64-127 of each tile
//               (168 registers each after setmaxnreg)
//   warps 8-11  dQ drain: TMEM -> shared-memory staging tile -> one bulk
//               TMA reduce-add into the fp32 accumulator per query tile
//   warp  12    TMA producer (K tile once; Q/dO/Qp/lse/D tiles, 4 stages)
//   warp  13    issues the S^T / dP^T MMAs
//   warp  14    TMEM allocator; issues the dV MMAs
//   warp  15    issues the dK_aug, then the dQ_aug MMAs
// Each MMA-issuing warp runs converged and issues through one elected lane
// (a thread issues one tcgen05.mma per ~43 cycles that way, against ~90 from
// a divergent branch), and the three MMA groups have separate issuers so
// that no group's waits hold back another's.  The compute warps neither
// drain dQ (dedicated warps do) nor wait for the previous tile's gradient
// MMAs before their exponentials (they form the whole tile in registers
// first, then wait for the P^T buffer).
// Per query tile i:  S^T = K_aug Q_aug^T and dP^T = V dO^T (MMA, TMEM) ->
// compute warps form P^T (to TMEM) and dS (to shared memory as 8 x 8 core
// matrices, double-buffered) -> MMA: dV += P^T dO (A from TMEM),
// dK_aug += dS^T [Qc|Qp] (A = the dS core matrices read K-major) and
// dQ_aug = dS [Kc|Kp] (A = the same core matrices read MN-major) -> drain
// warps fold dQ into the fp32 accumulator with one bulk reduce-add per tile
// (per-thread vector atomics cost more L2 time than the whole rest of the
// kernel).
// At d = 32 the MMAs are narrow: a tcgen05.mma of M=128, K=16 costs ~40-50
// cycles however small N is, and with both operands in shared memory an
// N <= 64 MMA moves more bytes than its flops cover.  So P^T, the A of the
// dV MMA, comes from TMEM; dS^T is read from the shared dS tile instead (a
// TMEM copy would cost the compute warps a store per element), the positional
// tiles are fetched zero-padded to 32 channels (TMA fills the out-of-bounds
// half with zeros) so that [Qc|Qp] and [Kc|Kp] form one N=48 B operand of two
// 64B-swizzle atoms, and dK_aug, dQ_aug are one MMA chain each (29 MMAs per
// tile).  S/dP of tile i+1 are issued as soon as the compute warps have
// pulled tile i into registers; P^T is released right after the dV/dK MMAs
// and dS is double-buffered, so the compute warps never wait on the
// gradient MMAs of the previous tile (what they do wait on is the latency
// of testing barriers that are already complete).  Exponentials are split between MUFU
// and the FMA pipe (exp2_fma2), with packed f32x2 arithmetic.
#pragma once

#include "geom.cuh"
#include "ptx.cuh"

namespace rib {

constexpr int kBwdStages = 4;
constexpr int kBwdThreads = 512;
constexpr int kBwdLaunchRegs = 128;     // 65536 / 512: what the host checks ptxas gave
constexpr int kBwdComputeRegs = 168;    // warpgroups 0-1
constexpr int kBwdServiceRegs = 80;     // warpgroups 2-3
static_assert(2 * 128 * kBwdComputeRegs + 2 * 128 * kBwdServiceRegs <=
                  kBwdThreads * kBwdLaunchRegs,
              "register split exceeds the launch budget");
constexpr uint32_t kBwdTmemCols = 512;
// TMEM columns (512): S^T, dP^T fp32; P^T bf16; (dS^T bf16, used only when
// RIB_BWD_DK_SMEM is 0); dV; dK = [dKc | dKp]; dQ = [dQc | dQp]
constexpr uint32_t kBColS = 0, kBColDP = 128, kBColP = 256, kBColDST = 320, kBColDV = 384,
                   kBColDK = 416, kBColDQ = 464;
// Of every 8 element pairs, how many exponentials run on the FMA pipe.  The
// backward's exponential phase runs at about the MUFU rate with two compute
// warps per scheduler; moving one pair in eight to the FMA pipe measured
// ~1 % faster on the 96x96 training workload, two or three pairs slower.
#ifndef RIB_BWD_POLY_PAIRS
#define RIB_BWD_POLY_PAIRS 1
#endif
constexpr int kBwdPolyPairs = RIB_BWD_POLY_PAIRS;
#ifndef RIB_BWD_DK_SMEM
#define RIB_BWD_DK_SMEM 1
#endif
constexpr bool kBwdDkSmem = RIB_BWD_DK_SMEM != 0;
constexpr uint64_t kBwdDrainNs = 200ull * 1000ull * 1000ull;

struct BwdParams {
  int B, H, W, heads, M, s, rank, nWx, nW, tiles_x, n_tiles;
  int region_mask;   // shifted-window region mask on (requires s > 0)
  float scale;       // tau
  float scale_log2;  // tau * log2(e)
  __nv_bfloat16* dqkv;
  int dqkv_v8;       // dqkv is 32-byte aligned: rows go out as whole 32-byte sectors
  float* dq_acc;     // [units][n_tiles][48][128]  (channel-major per tile)
  float* dkp_part;   // [units][n_tiles][128][16]
  int n_items;       // persistent form only: work items (unit, key tile), units * n_tiles
  uint64_t wait_limit_ns;
};

// Units (batch entry, window, head) of a call: the extent of the per-unit
// buffers, for the debug build's guards.
__device__ __forceinline__ size_t bwd_units(const BwdParams& p) {
  return static_cast<size_t>(p.B) * p.nW * p.heads;
}

struct __align__(1024) BwdSmem {
  uint8_t kc[8192];                // key tile, content, [128 rows][64 B], 64B swizzle
  uint8_t kp[8192];                // key tile, positional zero-padded to 32 ch (kc + 8 KB)
  uint8_t v[8192];
  uint8_t ds[2][32768];            // dS^T [128 keys x 128 queries] bf16, core matrices
  uint8_t qc[kBwdStages][8192];
  uint8_t qp[kBwdStages][8192];    // positional, zero-padded (qc + kBwdStages * 8 KB)
  uint8_t dO[kBwdStages][8192];
  float dq_stage[48 * 128];        // dQ of one query tile, [channel][row], for the bulk reduce
  float lse2[kBwdStages][128];     // -lse * log2(e), tile row order
  float dd[kBwdStages][128];       // -D = -rowsum(dO * O), tile row order
  uint64_t k_full;
  uint64_t q_full[kBwdStages], q_empty[kBwdStages];
  // pt_free: P^T (and dS^T) in TMEM and the dS buffer written next are free
  uint64_t s_full, s_free, ds_full, pt_free;
  uint64_t dq_full, dq_free, mma_done;
  int drain_ok[4];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kBwdSmemBytes = sizeof(BwdSmem) + 1024;
static_assert(kBwdSmemBytes <= 227 * 1024, "backward shared memory exceeds the per-CTA limit");

constexpr uint32_t kIdescBS = make_idesc_bf16(128, 128, false, false);   // S^T, dP^T
constexpr uint32_t kIdescBV = make_idesc_bf16(128, 32, false, true);     // dV
constexpr uint32_t kIdescBK = make_idesc_bf16(128, 48, false, true);     // dK_aug
constexpr uint32_t kIdescBQ = make_idesc_bf16(128, 48, true, true);      // dQ_aug

// Byte offset of element (key k, query q) of dS^T: 8 x 8 core matrices of
// 128 contiguous bytes; key groups of 8 every 128 B, query groups of 8
// every 2048 B.
__device__ __forceinline__ uint32_t ds_offset(int k, int q) {
  return static_cast<uint32_t>((q >> 3) * 2048 + (k >> 3) * 128 + (k & 7) * 16 + (q & 7) * 2);
}

__device__ __forceinline__ void bwd_producer(BwdSmem& sm, const CUtensorMap* tq,
                                             const CUtensorMap* tdo, const CUtensorMap* tqp,
                                             const CUtensorMap* tkp, const CUtensorMap* tlse2,
                                             const CUtensorMap* tdd, const BwdParams& p,
                                             const UnitCoord& u, int kt) {
  volatile int* ab = &sm.abort_flag;
  const int hh = u.head;
  const int by = u.wy * p.M + p.s, bx = u.wx * p.M + p.s;
  const bool pos = p.rank > 0;
  {
    int i0, j0;
    tile_origin(kt, p.tiles_x, i0, j0);
    const int y = wrap_once(by + i0, p.H);
    mbar_arrive_expect_tx(&sm.k_full, 2u * 8192u + (pos ? 8192u : 0u));
    for (int c = 0; c < 2; ++c) {
      const int x = wrap_once(bx + j0 + 8 * c, p.W);
      tma_load_5d(sm.kc + c * 4096, tq, &sm.k_full, 0, p.heads + hh, x, y, u.b);
      tma_load_5d(sm.v + c * 4096, tq, &sm.k_full, 0, 2 * p.heads + hh, x, y, u.b);
      if (pos) tma_load_4d(sm.kp + c * 4096, tkp, &sm.k_full, 0, j0 + 8 * c, i0, hh);
    }
  }
  const uint32_t q_bytes = 2u * 8192u + (pos ? 8192u : 0u) + 2u * 512u;
  int i = 0;
  for (; i < p.n_tiles; ++i) {
    const int st = i % kBwdStages, use = i / kBwdStages;
    if (use > 0 &&
        !mbar_wait(&sm.q_empty[st], (use - 1) & 1, ab, p.wait_limit_ns, SITE_BWD_PRODUCER))
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
  if (*ab) {
    volatile int no_abort = 0;
    mbar_wait(&sm.k_full, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
    for (int ii = i - 1; ii >= 0 && ii >= i - kBwdStages; --ii)
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
  const uint32_t kc = smem_u32(sm.kc), kp = smem_u32(sm.kp), v = smem_u32(sm.v);
  bool ok = warp_wait(&sm.k_full, 0, ab, lim, SITE_BWD_MMA);
  for (int i = 0; ok && i < n; ++i) {
    const int st = i % kBwdStages;
    ok = warp_wait(&sm.q_full[st], (i / kBwdStages) & 1, ab, lim, SITE_BWD_MMA) &&
         (i == 0 || warp_wait(&sm.s_free, (i - 1) & 1, ab, lim, SITE_BWD_MMA));
    if (!ok) break;
    tc_fence_after();
    // S^T = K_aug Q_aug^T  (M = keys, N = queries, K = 32 + 16)
    const uint64_t a = make_sdesc(kc, 16, 512, kLayoutSW64);
    const uint64_t b = make_sdesc(smem_u32(sm.qc[st]), 16, 512, kLayoutSW64);
    umma_ss3_elect(tmem + kBColS, a, b, a + 2, b + 2, make_sdesc(kp, 16, 512, kLayoutSW64),
                   make_sdesc(smem_u32(sm.qp[st]), 16, 512, kLayoutSW64), kIdescBS, pos ? 1u : 0u);
    // dP^T = V dO^T  (M = keys, N = queries, K = 32)
    const uint64_t av = make_sdesc(v, 16, 512, kLayoutSW64);
    const uint64_t bo = make_sdesc(smem_u32(sm.dO[st]), 16, 512, kLayoutSW64);
    umma_ss3_elect(tmem + kBColDP, av, bo, av + 2, bo + 2, av, bo, kIdescBS, 0u);
    umma_commit_elect(&sm.s_full);
  }
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
}

// Warp 14 (all lanes; one elected lane issues): dV += P^T dO (A = P^T from
// TMEM) of every query tile.  P^T/dS^T (pt_free) and the query stage
// (q_empty) are released by this warp and warp 15 together (two arrivals).
__device__ __forceinline__ void bwd_mma_grads(BwdSmem& sm, uint32_t tmem, const BwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int n = p.n_tiles;
  bool ok = true;
  for (int i = 0; ok && i < n; ++i) {
    const int st = i % kBwdStages;
    // ds_full(i) implies the stage's tiles have landed: the compute warps
    // waited for them (q_full) before forming P^T and dS^T.
    if (!(ok = warp_wait(&sm.ds_full, i & 1, ab, lim, SITE_BWD_MMA))) break;
    tc_fence_after();
    const uint32_t dO = smem_u32(sm.dO[st]);
    // dV += P^T dO   (K = queries, 16 per step; A from TMEM)
    umma_ts8_elect(tmem + kBColDV, tmem + kBColP, make_sdesc(dO, 16, 512, kLayoutSW64),
                   1024 >> 4, kIdescBV, i > 0 ? 1u : 0u);
    umma_commit_elect(&sm.pt_free);
    umma_commit_elect(&sm.q_empty[st]);
  }
  umma_commit_elect(&sm.mma_done);   // every dV MMA of the kernel has completed
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
}

// Warp 15 (all lanes; one elected lane issues): dK_aug += dS^T [Qc|Qp] (A =
// dS^T from TMEM), then dQ_aug = dS [Kc|Kp] (A = dS MN-major core matrices
// in shared memory) of every query tile.  Its dK commit releases P^T/dS^T
// together with warp 14's dV commit, so the compute warps cannot form tile
// i+1 before this warp has taken tile i: ds_full never runs ahead of it.
__device__ __forceinline__ void bwd_mma_dq(BwdSmem& sm, uint32_t tmem, const BwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int n = p.n_tiles;
  const uint32_t kc = smem_u32(sm.kc), kp = smem_u32(sm.kp);
  const uint32_t lbo_k = kp - kc;                                   // [Kc|Kp] atoms
  const uint32_t lbo_q = smem_u32(sm.qp[0]) - smem_u32(sm.qc[0]);  // [Qc|Qp] atoms
  bool ok = true;
  for (int i = 0; ok && i < n; ++i) {
    const int st = i % kBwdStages;
    if (!(ok = warp_wait(&sm.ds_full, i & 1, ab, lim, SITE_BWD_MMA))) break;
    tc_fence_after();
    if (kBwdDkSmem) {
      // A = dS^T read K-major from the dS core matrices in shared memory
      // (key groups of 8 every 128 B, query groups of 8 every 2048 B)
      umma_ss8_elect(tmem + kBColDK, make_sdesc(smem_u32(sm.ds[i & 1]), 2048, 128, kLayoutNone),
                     4096 >> 4, make_sdesc(smem_u32(sm.qc[st]), lbo_q, 512, kLayoutSW64),
                     1024 >> 4, kIdescBK, i > 0 ? 1u : 0u);
    } else {
      umma_ts8_elect(tmem + kBColDK, tmem + kBColDST,
                     make_sdesc(smem_u32(sm.qc[st]), lbo_q, 512, kLayoutSW64), 1024 >> 4,
                     kIdescBK, i > 0 ? 1u : 0u);
    }
    umma_commit_elect(&sm.pt_free);
    umma_commit_elect(&sm.q_empty[st]);
    // the single dQ buffer is free once the drain warps pulled tile i-1
    if (i > 0 && !(ok = warp_wait(&sm.dq_free, (i - 1) & 1, ab, lim, SITE_BWD_MMA))) break;
    tc_fence_after();
    const uint32_t ds = smem_u32(sm.ds[i & 1]);
    // step k: 16 queries further in dS (256 B), 16 keys further in [Kc|Kp] (1 KB)
    umma_ss8_elect(tmem + kBColDQ, make_sdesc(ds, 128, 2048, kLayoutNone), 256 >> 4,
                   make_sdesc(kc, lbo_k, 512, kLayoutSW64), 1024 >> 4, kIdescBQ, 0u);
    umma_commit_elect(&sm.dq_full);
  }
  umma_commit_elect(&sm.mma_done);   // every dK MMA of the kernel has completed
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kBwdDrainNs, SITE_BWD_DRAIN);
}

// Warps 8-11: drain dQ of every query tile from TMEM into the staging tile
// (lane quarter wq = warp & 3, all 48 channels), then one thread folds the
// tile into the fp32 accumulator with a bulk reduce-add.
constexpr int kDrainBar = 1;   // named barrier of the 4 drain warps
__device__ __forceinline__ void bwd_drain(BwdSmem& sm, uint32_t tmem, const BwdParams& p,
                                          int unit, int wq) {
  volatile int* ab = &sm.abort_flag;
  const int lane = threadIdx.x & 31;
  const bool pos = p.rank > 0;
  const bool leader = wq == 0 && lane == 0;
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  const int row = wq * 32 + lane;
  const uint32_t tile_bytes = 48u * 128u * 4u;
  volatile int* drain_ok = sm.drain_ok;
  for (int it = 0; it < p.n_tiles; ++it) {
    const bool ok = warp_wait(&sm.dq_full, it & 1, ab, p.wait_limit_ns, SITE_BWD_COMPUTE);
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
    const bool all_ok = drain_ok[0] && drain_ok[1] && drain_ok[2] && drain_ok[3];
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
      const size_t dq0 = (static_cast<size_t>(unit) * p.n_tiles + it) * 48 * 128;
      if (rib_guard(dq0 + 48 * 128 - 1, bwd_units(p) * p.n_tiles * 48 * 128, G_BWD_DQ_ACC))
        bulk_reduce_add_f32(p.dq_acc + dq0, sm.dq_stage, tile_bytes);
      tma_store_commit();
    }
  }
  // the reductions must be complete before the kernel's work is considered done
  if (leader) tma_store_wait_all();
}

template <bool kMask>
__device__ __forceinline__ void bwd_compute(BwdSmem& sm, uint32_t tmem, const BwdParams& p,
                                            const UnitCoord& u, int unit, int kt, int g,
                                            int wq) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int lane = threadIdx.x & 31;
  const bool pos = p.rank > 0;
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
    const int st = i % kBwdStages;
    bool kv = true;
    if (mask_on) {
      int qi0, qj0;
      tile_origin(i, p.tiles_x, qi0, qj0);
      kv = region_band(u.wy * p.M + qi0, p.H, p.M, p.s) == kbr &&
           region_band(u.wx * p.M + qj0 + 8 * g, p.W, p.M, p.s) == kbc;
    }
    // S^T/dP^T of tile i, and the stage's lse / D rows (written by TMA)
    if (!(ok = warp_wait2(&sm.s_full, i & 1, &sm.q_full[st], (i / kBwdStages) & 1, ab, lim,
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
    if (i > 0 && !(ok = warp_wait(&sm.pt_free, (i - 1) & 1, ab, lim, SITE_BWD_COMPUTE))) break;
    tc_fence_after();
    uint8_t* ds_row = sm.ds[i & 1];
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
  if (!ok) return;
  if (!warp_wait(&sm.mma_done, 0, ab, lim, SITE_BWD_COMPUTE)) return;
  tc_fence_after();
  int i0, j0, ii, jl;
  tile_origin(kt, p.tiles_x, i0, j0);
  tile_row_local(key, i0, j0, ii, jl);
  const int y = wrap_once(u.wy * p.M + ii + p.s, p.H);
  const int x = wrap_once(u.wx * p.M + jl + p.s, p.W);
  const size_t pix = (static_cast<size_t>(u.b) * p.H + y) * p.W + x;
  __nv_bfloat16* base = p.dqkv + pix * 3 * p.heads * 32;
  const size_t n_dqkv = static_cast<size_t>(p.B) * p.H * p.W * 3 * p.heads * 32;
  uint32_t r[32];
  if (g == 0) {  // dV
    tmem_ld_x32(tmem + lane_off + kBColDV, r);
    tmem_wait_ld();
    reg_fence_x32(r);
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      w[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
    if (rib_guard(pix * 3 * p.heads * 32 + (2 * p.heads + u.head) * 32 + 31, n_dqkv, G_BWD_DQKV))
      store_row64(base + (2 * p.heads + u.head) * 32, w, p.dqkv_v8 != 0);
    if (pos) {
      uint32_t r16[16];
      tmem_ld_x16(tmem + lane_off + kBColDK + 32, r16);
      tmem_wait_ld();
      reg_fence_x16(r16);
      const size_t kp0 = ((static_cast<size_t>(unit) * p.n_tiles + kt) * 128 + key) * 16;
      const float t = p.scale;
      uint32_t w16[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) w16[e] = __float_as_uint(__uint_as_float(r16[e]) * t);
      // the workspace partials are 256-byte aligned: always whole sectors
      if (rib_guard(kp0 + 15, bwd_units(p) * p.n_tiles * 128 * 16, G_BWD_DKP_PART))
        store_row64(p.dkp_part + kp0, w16, true);
    }
  } else {  // dKc
    tmem_ld_x32(tmem + lane_off + kBColDK, r);
    tmem_wait_ld();
    reg_fence_x32(r);
    const float t = p.scale;
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * t, __uint_as_float(r[2 * e + 1]) * t);
    if (rib_guard(pix * 3 * p.heads * 32 + (p.heads + u.head) * 32 + 31, n_dqkv, G_BWD_DQKV))
      store_row64(base + (p.heads + u.head) * 32, w, p.dqkv_v8 != 0);
  }
}

// grid (n_tiles, units), block kBwdThreads, dynamic smem kBwdSmemBytes.
// kMask: the shifted-window region mask (a separate instantiation).
template <bool kMask>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                    const __grid_constant__ CUtensorMap tm_dout,
                    const __grid_constant__ CUtensorMap tm_qp,
                    const __grid_constant__ CUtensorMap tm_kp,
                    const __grid_constant__ CUtensorMap tm_lse2,
                    const __grid_constant__ CUtensorMap tm_dd, const BwdParams p) {
  extern __shared__ uint8_t sm_raw_bwd[];
  BwdSmem& sm = *align1024<BwdSmem>(sm_raw_bwd);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const UnitCoord u = decode_unit(unit, p.heads, p.nW, p.nWx);
  const int kt = blockIdx.x;
  if (threadIdx.x == 0) {
    mbar_init(&sm.k_full, 1);
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
    mbar_init(&sm.mma_done, 2);
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
    bwd_compute<kMask>(sm, tmem, p, u, unit, kt, warp >> 2, warp & 3);
  } else {
    regs_dec<kBwdServiceRegs>();
    if (warp < 12) {
      bwd_drain(sm, tmem, p, unit, warp & 3);
    } else if (warp == 12) {
      if (lane == 0) bwd_producer(sm, &tm_qkv, &tm_dout, &tm_qp, &tm_kp, &tm_lse2, &tm_dd, p, u, kt);
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

// ---------------------------------------------------------------- helpers

struct BwdAuxParams {
  int B, H, W, heads, M, s, nWx, nW, tiles_x, n_tiles, rank;
  float scale;
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  const float* lse;
  float* lse2;      // [B][heads][H][W]
  float* dd;        // [B][heads][H][W]
  float* dq_acc;    // [units][n_tiles][48][128]
  const float* dkp_part;
  size_t dq_acc_floats;
  __nv_bfloat16* dqkv;
  int dq_v8;        // dqkv is 32-byte aligned: dq_finalize writes whole 32-byte sectors
  float* dqp;       // [heads][M][M][rank]
  float* dkp;
  int pg_chunks;    // posgrad_reduce: warps sharing one group of outputs (1, 2, 4, 8, 16)
};

// One thread per (b, head, y, x): -D = -sum_c dO*O and -lse*log2(e), stored
// negated for the fused multiply-adds of the main kernel; the grid also
// zeroes the dQ accumulator.
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdAuxParams p) {
  const size_t n = static_cast<size_t>(p.B) * p.heads * p.H * p.W;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += stride) {
    const int x = static_cast<int>(idx % p.W);
    size_t r = idx / p.W;
    const int y = static_cast<int>(r % p.H);
    r /= p.H;
    const int h = static_cast<int>(r % p.heads);
    const int b = static_cast<int>(r / p.heads);
    const size_t row = (((static_cast<size_t>(b) * p.H + y) * p.W + x) * p.heads + h) * 32;
    const uint4* o4 = reinterpret_cast<const uint4*>(p.out + row);
    const uint4* g4 = reinterpret_cast<const uint4*>(p.dout + row);
    float acc = 0.f;
    if (!rib_guard(row + 31, n * 32, G_BWD_PRE_IN)) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 a = o4[q], c = g4[q];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
        const float2 fc = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cv[e]));
        acc = fmaf(fa.x, fc.x, acc);
        acc = fmaf(fa.y, fc.y, acc);
      }
    }
    p.dd[idx] = -acc;
    p.lse2[idx] = -p.lse[idx] * 1.4426950408889634f;
  }
  float4* z = reinterpret_cast<float4*>(p.dq_acc);
  const size_t nz = p.dq_acc_floats / 4;
  for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < nz;
       idx += stride)
    z[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// One thread per (unit, tile row): dQc * tau -> bf16 at the rolled pixel.
__global__ void __launch_bounds__(256) dq_finalize_kernel(const BwdAuxParams p) {
  const size_t n = static_cast<size_t>(p.B) * p.nW * p.heads * p.n_tiles * 128;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  const int row = static_cast<int>(idx & 127);
  const size_t ut = idx >> 7;
  const int tile = static_cast<int>(ut % p.n_tiles);
  const int unit = static_cast<int>(ut / p.n_tiles);
  const UnitCoord u = decode_unit(unit, p.heads, p.nW, p.nWx);
  int i0, j0, i, j;
  tile_origin(tile, p.tiles_x, i0, j0);
  tile_row_local(row, i0, j0, i, j);
  const int y = wrap_once(u.wy * p.M + i + p.s, p.H);
  const int x = wrap_once(u.wx * p.M + j + p.s, p.W);
  const float* src = p.dq_acc + (ut * 48) * 128 + row;     // [tile][channel][row]
  const size_t pix = (static_cast<size_t>(u.b) * p.H + y) * p.W + x;
  uint4* dst = reinterpret_cast<uint4*>(p.dqkv + (pix * 3 * p.heads + u.head) * 32);
  const float t = p.scale;
  if (!rib_guard((ut * 48 + 31) * 128 + row, p.dq_acc_floats, G_DQ_FIN_IN) ||
      !rib_guard((pix * 3 * p.heads + u.head) * 32 + 31,
                 static_cast<size_t>(p.B) * p.H * p.W * 3 * p.heads * 32, G_DQ_FIN_OUT))
    return;
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(src[2 * e * 128] * t, src[(2 * e + 1) * 128] * t);
  if (p.dq_v8) {
    // two 32-byte stores: each a whole sector of the row's 64 bytes (16-byte
    // stores from 32 different rows would half-fill a sector each)
    st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    st_global_v8(dst + 2, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// dQp[h][i][j][r] = tau * sum over the B*nW units of head h of the dQ
// accumulator's positional channels, dKp likewise from the dKp partials
// (one Qp/Kp set serves every window).  grid (heads*N*rank / kPgBlockOut, 2):
// blockIdx.y 0 sums dQp, 1 sums dKp.  Outputs are taken in the layout their
// source is read in (dQp: row fastest, matching the accumulator's
// [unit][tile][channel][row]; dKp: rank fastest, matching the partials'
// [unit][tile][row][rank]), 32 consecutive ones per warp, so each warp's
// loads are 128-byte runs.  p.pg_chunks warps share a group of 32 outputs
// and sum consecutive ranges of the units (eight accumulators taking the
// units in turn, the remainder going to the first); the group's first warp
// adds their sums in warp order.
// The order is fixed: the result is deterministic.  Many units (small
// windows) get 16 warps per group, few (large windows) one.  The grid is
// sized to the SMs and the blocks loop over the passes.
constexpr int kPgWarps = 16;
constexpr int kPgBlockOut = 32 * kPgWarps;   // outputs per block pass with one warp per group
__global__ void __launch_bounds__(32 * kPgWarps, 2) posgrad_reduce_kernel(const BwdAuxParams p) {
  __shared__ float part[kPgWarps][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int chunks = p.pg_chunks, groups = kPgWarps / chunks, grp = w / chunks,
            cw = w % chunks;
  const bool kside = blockIdx.y == 1;
  const int rank = p.rank;
  const size_t n_out = static_cast<size_t>(p.heads) * p.n_tiles * rank * 128;
  const size_t n_pass = (n_out + 32 * groups - 1) / (32 * groups);
  const int total = p.B * p.nW;
  const int per = (total + chunks - 1) / chunks;
  const int b0 = cw * per, b1 = min(total, b0 + per);
  const size_t unit_stride = static_cast<size_t>(p.heads) * p.n_tiles;
  const size_t step = kside ? unit_stride * 128 * 16 : unit_stride * 48 * 128;
  const size_t n_src = kside ? p.dq_acc_floats / 48 * 16 : p.dq_acc_floats;
  // the blocks walk the passes (groups x 32 outputs each) in a grid-stride loop
  for (size_t pass = blockIdx.x; pass < n_pass; pass += gridDim.x) {
    const size_t o = (pass * groups + grp) * 32 + lane;
    int h = 0, tile = 0, r = 0, row = 0;
    if (o < n_out) {
      size_t rem = o;
      if (kside) {          // o = ((h * n_tiles + tile) * 128 + row) * rank + r
        r = static_cast<int>(rem % rank);
        rem /= rank;
        row = static_cast<int>(rem % 128);
        rem /= 128;
      } else {              // o = ((h * n_tiles + tile) * rank + r) * 128 + row
        row = static_cast<int>(rem % 128);
        rem /= 128;
        r = static_cast<int>(rem % rank);
        rem /= rank;
      }
      tile = static_cast<int>(rem % p.n_tiles);
      h = static_cast<int>(rem / p.n_tiles);
    }
    // element of unit (bw, h) that this output sums: base + bw * step
    const size_t first = static_cast<size_t>(h) * p.n_tiles + tile;
    const size_t base = kside ? (first * 128 + row) * 16 + r : (first * 48 + 32 + r) * 128 + row;
    const float* src = (kside ? p.dkp_part : p.dq_acc) + base;
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (o < n_out && (b1 <= b0 || rib_guard(base + (b1 - 1) * step, n_src, G_POSGRAD_IN))) {
      int bw = b0;
      for (; bw + 7 < b1; bw += 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] += src[(bw + e) * step];
      }
      for (; bw < b1; ++bw) a[0] += src[bw * step];
    }
    part[w][lane] = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
    __syncthreads();
    if (cw == 0 && o < n_out) {
      float sum = 0.f;
      for (int c = 0; c < chunks; ++c) sum += part[w + c][lane];
      int i0, j0, i, j;
      tile_origin(tile, p.tiles_x, i0, j0);
      tile_row_local(row, i0, j0, i, j);
      const size_t dst = (static_cast<size_t>(h * p.M + i) * p.M + j) * rank + r;
      if (rib_guard(dst, n_out, G_POSGRAD_OUT)) {
        if (kside)
          p.dkp[dst] = sum;
        else
          p.dqp[dst] = sum * p.scale;
      }
    }
    __syncthreads();   // part is read before the next pass writes it
  }
}

}  // namespace rib
