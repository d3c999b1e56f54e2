// attn_fwd.cuh -- RIB window attention forward on tcgen05 tensor cores.
//
// "Rank-Factorized Implicit Neural Bias" (gist.science English summary,
// Technical Summary §2.A steps 3-4 and the score equation; the paper's
// abstract): the positional tokens are concatenated channel-wise with the
// content tokens, so the biased score is one dot product in the augmented
// space, S = [Qc,Qp][Kc,Kp]^T = Qc Kc^T + Qp Kp^T, and attention runs
// flash-style without an N x N score or bias matrix.
//
// Here the concatenation is never materialised either: the augmented
// contraction (K = 32 + 16) is three K=16 tcgen05.mma steps, two over the
// content tiles and one over the positional tiles, accumulating into the
// same TMEM score tile.
//
// Persistent CTAs, one per SM, each walking work items = one unit (batch,
// window, head) x two 128-query tiles (A, B); every barrier phase is counted
// across items, so the next item's loads and score MMAs overlap the end of
// the current one.  384 threads (3 warpgroups):
//   warps 0-3    softmax group A: warp w owns TMEM lanes 32 w.. (query rows)
//                and all 128 key columns of each score tile, one thread per
//                query row, so the row maximum needs no exchange
//   warps 4-7    softmax group B, the same for the second query tile
//   warp  8      TMA producer: each item's Q tiles (two buffers, by item
//                parity), then its K/V/Kp tiles through a 3-stage
//                shared-memory ring; boxes at rolled map coordinates
//   warp  9      TMEM allocator; issues the score MMAs
//   warp  10     issues the PV MMAs of query tile A
//   warp  11     issues the PV MMAs of query tile B
// Each SM sub-partition runs one softmax warp of each query tile; a thread's
// 128 independent columns keep the exponential pipes fed.  The softmax
// warpgroups take 208 registers (the 128 scores of a row stay in registers)
// and the service warpgroup 56 (setmaxnreg).
//
// One thread issues at most one tcgen05.mma every ~43 cycles (an elected
// lane of a converged warp; ~90 from a divergent branch), while the tensor
// pipe retires an M=128, N=48, K=16 MMA in ~24 cycles; so the MMAs of a key
// tile (3 score MMAs per query tile, 8 PV MMAs per query tile) are spread
// over three issuing threads.
//
// TMEM (512 columns): three score regions R0..R2 of 128 fp32 columns, then
// [O|L]_A and [O|L]_B (48 columns each).  Score tiles are numbered
// k = 2j + X (key tile j, query tile X) and S(k) goes to region k % 3.
// Softmax group X pulls S(k) into registers, writes P(k) as packed bf16 over
// the first 64 columns of the same region, and signals p_full; the PV thread
// of X then issues [O|L]_X += P(k) [V_j | 1] with P read from TMEM as the A
// operand (the second swizzle atom of the B operand is an all-ones tile, so
// the tensor core also accumulates the softmax denominators L from the very
// bf16 P it multiplies with V) and frees the region.  The score MMA of
// k + 3 reuses the region once that PV has completed; an item's first PV
// overwrites [O|L]_X once the previous item's epilogue has read it.  The softmax warps
// therefore never wait for a PV MMA, except before the rare rescale of O:
// the running max is updated lazily, O and L being rescaled only when the
// max grows by more than 2^8.
//
// The exponentials are the bottleneck of this kernel (16K per 128x128 tile
// against 320 tensor-core cycles of MMA at d_qk=48, d_v=32), so a fixed
// share of them (kPolyPairs of every 16 pairs) runs on the FMA pipe
// (exp2_fma2) and the rest on MUFU ex2; scaling uses packed f32x2 FMAs.
#pragma once

#include "geom.cuh"
#include "ptx.cuh"

namespace rib {

constexpr int kFwdStages = 3;
constexpr int kFwdThreads = 384;
constexpr int kFwdLaunchRegs = 168;     // what the host checks ptxas gave (65536 / 384)
constexpr int kFwdSoftmaxRegs = 208;    // warpgroups 0-1
constexpr int kFwdServiceRegs = 56;     // warpgroup 2
static_assert(2 * 128 * kFwdSoftmaxRegs + 128 * kFwdServiceRegs <= kFwdThreads * kFwdLaunchRegs,
              "register split exceeds the launch budget");
constexpr uint32_t kFwdTmemCols = 512;
constexpr int kRegions = 3;
constexpr uint32_t kColO = 384;  // [O|L]_X at kColO + 48 X, L at +32
constexpr int kOCols = 48;
static_assert(kRegions * 128 + 2 * kOCols <= kFwdTmemCols, "forward TMEM layout exceeds 512 columns");
// Of every 16 element pairs, how many exponentials run on the FMA pipe.
#ifndef RIB_FWD_POLY_PAIRS
#define RIB_FWD_POLY_PAIRS 5
#endif
constexpr int kPolyPairs = RIB_FWD_POLY_PAIRS;
constexpr uint64_t kFwdDrainNs = 200ull * 1000ull * 1000ull;
#ifndef RIB_FWD_SLEEP_NS
#define RIB_FWD_SLEEP_NS 20000
#endif
constexpr uint32_t kFwdSleepNs = RIB_FWD_SLEEP_NS;  // per retry of a waiting warp (0: poll)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdParams {
  int B, H, W, heads, M, s, rank, nWx, nW, tiles_x, n_tiles;
  int n_items;       // work items: (unit, pair of query tiles), units * n_tiles / 2
  int region_mask;   // shifted-window region mask on (requires s > 0)
  float scale_log2;  // softmax scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  const __nv_bfloat16* gate;   // CLA gate G [B][H][W][heads*32], or null
  __nv_bfloat16* out_gated;    // O * G, written when gate is set
  int out_v8, gated_v8;        // out / out_gated 32-byte aligned: rows as whole sectors
  uint64_t wait_limit_ns;
};

struct __align__(1024) FwdSmem {
  uint8_t qc[2][2][8192];         // [item parity][tile X] [128 rows][64 B], 64B swizzle
  uint8_t kc[kFwdStages][8192];
  uint8_t v[kFwdStages][8192];
  uint8_t ones[8192];             // bf16 1.0 everywhere: B atom that yields the row sums
  uint8_t qp[2][2][4096];         // [item parity][tile X] [128 rows][32 B], 32B swizzle
  uint8_t kp[kFwdStages][4096];
  uint64_t q_full[2], q_free[2];  // Q buffers (item parity): loaded / read by every score MMA
  uint64_t o_free[2];             // [O|L]_X read by the epilogue of the tile's last item
  uint64_t kv_full[kFwdStages];
  uint64_t kv_empty[kFwdStages];  // both PV threads release a stage
  uint64_t s_full[kRegions], r_free[kRegions];
  uint64_t p_full[2][2];          // [tile X][key tile parity]
  int pv_count[2];                // PV steps of tile X known complete
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kFwdSmemBytes = sizeof(FwdSmem) + 1024;  // + alignment slack
static_assert(kFwdSmemBytes <= 227 * 1024, "forward shared memory exceeds the per-CTA limit");

constexpr uint32_t kIdescS = make_idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = make_idesc_bf16(128, kOCols, false, true);

// The CTA's work items, in order: item li is it = blockIdx.x + li * gridDim.x,
// unit it / (n_tiles / 2), query tiles 2 (it % (n_tiles / 2)) and the next.
// Every barrier phase below is counted across items (key tile J = li n + j,
// score tile K = 2 J + X), so the pipeline runs on from one item to the next.
__device__ __forceinline__ void fwd_item(const FwdParams& p, int it, UnitCoord& u, int& tile0) {
  const int pairs = p.n_tiles / 2;
  u = decode_unit(it / pairs, p.heads, p.nW, p.nWx);
  tile0 = 2 * (it % pairs);
}

// Warp 8, lane 0: Q of each item into the buffer of its parity (once the
// score MMAs of the item two back have read it), then its K/V/Kp tiles
// through the ring.
__device__ __forceinline__ void fwd_producer(FwdSmem& sm, const CUtensorMap* tq,
                                             const CUtensorMap* tqp, const CUtensorMap* tkp,
                                             const FwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const bool pos = p.rank > 0;
  const int n = p.n_tiles;
  const uint32_t kv_bytes = 2u * 8192u + (pos ? 4096u : 0u);
  int J = 0, li = 0, q_issued = 0;
  bool ok = true;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    UnitCoord u;
    int tile0;
    fwd_item(p, it, u, tile0);
    const int hh = u.head;
    const int by = u.wy * p.M + p.s, bx = u.wx * p.M + p.s;
    const int qb = li & 1;
    if (li >= 2 &&
        !(ok = mbar_wait(&sm.q_free[qb], ((li >> 1) - 1) & 1, ab, p.wait_limit_ns,
                         SITE_FWD_PRODUCER)))
      break;
    mbar_arrive_expect_tx(&sm.q_full[qb], 2u * (8192u + (pos ? 4096u : 0u)));
    for (int X = 0; X < 2; ++X) {
      int i0, j0;
      tile_origin(tile0 + X, p.tiles_x, i0, j0);
      const int y = wrap_once(by + i0, p.H);
      for (int c = 0; c < 2; ++c) {
        const int x = wrap_once(bx + j0 + 8 * c, p.W);
        tma_load_5d(sm.qc[qb][X] + c * 4096, tq, &sm.q_full[qb], 0, hh, x, y, u.b);
        if (pos)
          tma_load_4d(sm.qp[qb][X] + c * 2048, tqp, &sm.q_full[qb], 0, j0 + 8 * c, i0, hh);
      }
    }
    ++q_issued;
    for (int j = 0; j < n; ++j, ++J) {
      const int st = J % kFwdStages, use = J / kFwdStages;
      if (use > 0 &&
          !(ok = mbar_wait(&sm.kv_empty[st], (use - 1) & 1, ab, p.wait_limit_ns,
                           SITE_FWD_PRODUCER)))
        break;
      mbar_arrive_expect_tx(&sm.kv_full[st], kv_bytes);
      int i0, j0;
      tile_origin(j, p.tiles_x, i0, j0);
      const int y = wrap_once(by + i0, p.H);
      for (int c = 0; c < 2; ++c) {
        const int x = wrap_once(bx + j0 + 8 * c, p.W);
        tma_load_5d(sm.kc[st] + c * 4096, tq, &sm.kv_full[st], 0, p.heads + hh, x, y, u.b);
        tma_load_5d(sm.v[st] + c * 4096, tq, &sm.kv_full[st], 0, 2 * p.heads + hh, x, y, u.b);
        if (pos) tma_load_4d(sm.kp[st] + c * 2048, tkp, &sm.kv_full[st], 0, j0 + 8 * c, i0, hh);
      }
    }
  }
  if (*ab) {
    // Aborted: let every copy this thread started land before the CTA exits
    // (the latest phase of each Q buffer and of each ring stage).
    volatile int no_abort = 0;
    for (int q = q_issued - 1; q >= 0 && q >= q_issued - 2; --q)
      mbar_wait(&sm.q_full[q & 1], (q >> 1) & 1, &no_abort, kFwdDrainNs, SITE_FWD_DRAIN);
    for (int jj = J - 1; jj >= 0 && jj >= J - kFwdStages; --jj)
      mbar_wait(&sm.kv_full[jj % kFwdStages], (jj / kFwdStages) & 1, &no_abort, kFwdDrainNs,
                SITE_FWD_DRAIN);
  }
}

// Warp 9: S(K) = Q_X K_J^T into region K % 3 for the score tiles
// K = 2 J + X of every item, in order, each once the region has been freed
// by the PV MMA of score tile K - 3.  After an item's last score tile the
// commit to q_free releases its Q buffer.
// Phase arithmetic: a region's barriers complete once per use, and use
// K + 3 cannot start before use K has been consumed, so no barrier is ever
// more than one phase ahead of the parity a waiter asks for.
__device__ __forceinline__ void fwd_mma_scores(FwdSmem& sm, uint32_t tmem, const FwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const bool pos = p.rank > 0;
  const int n = p.n_tiles;
  bool ok = true;
  int li = 0;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    const int qb = li & 1;
    if (!(ok = warp_wait(&sm.q_full[qb], (li >> 1) & 1, ab, lim, SITE_FWD_MMA))) break;
    for (int k = 0; ok && k < 2 * n; ++k) {
      const int X = k & 1, J = li * n + (k >> 1), K = 2 * J + X;
      const int r = K % kRegions, st = J % kFwdStages;
      if (X == 0 &&
          !(ok = warp_wait(&sm.kv_full[st], (J / kFwdStages) & 1, ab, lim, SITE_FWD_MMA)))
        break;
      if (K >= kRegions &&
          !(ok = warp_wait(&sm.r_free[r], (K / kRegions - 1) & 1, ab, lim, SITE_FWD_MMA)))
        break;
      tc_fence_after();
      const uint32_t d = tmem + r * 128;
      const uint64_t a = make_sdesc(smem_u32(sm.qc[qb][X]), 16, 512, kLayoutSW64);
      const uint64_t b = make_sdesc(smem_u32(sm.kc[st]), 16, 512, kLayoutSW64);
      umma_ss_elect(d, a, b, kIdescS, 0u);
      umma_ss_elect(d, a + 2, b + 2, kIdescS, 1u);  // channels 16..31: start address + 32 B
      if (pos)
        umma_ss_elect(d, make_sdesc(smem_u32(sm.qp[qb][X]), 16, 256, kLayoutSW32),
                      make_sdesc(smem_u32(sm.kp[st]), 16, 256, kLayoutSW32), kIdescS, 1u);
      umma_commit_elect(&sm.s_full[r]);
    }
    if (ok) umma_commit_elect(&sm.q_free[qb]);
  }
  // Every MMA issued above must finish before the tensor memory is freed.
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kFwdDrainNs, SITE_FWD_DRAIN);
}

// Warps 10 (X = 0) and 11 (X = 1), all lanes, one elected lane issuing:
// [O|L]_X (+)= P(K) [V_J | 1] for K = 2 J + X once group X has written P(K);
// the first key tile of an item overwrites [O|L]_X, once the epilogue of the
// previous item has read it (o_free).  The commits free the region and
// release K/V stage J (kv_empty counts one arrival per PV thread); the warp
// then waits for its own MMAs (on the region's barrier) and publishes how
// many PV steps of tile X are complete in pv_count[X] (counted across
// items), which the softmax warps read before touching [O|L]_X (the rare
// rescale, and the epilogue).  The accumulation into [O|L]_X is serial
// anyway, and the next P arrives much later, so the wait costs this thread
// nothing.
__device__ __forceinline__ void fwd_mma_pv(FwdSmem& sm, uint32_t tmem, const FwdParams& p,
                                           int X) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int n = p.n_tiles;
  const uint32_t d = tmem + kColO + X * kOCols;
  bool ok = true;
  int li = 0;
  for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++li) {
    for (int j = 0; ok && j < n; ++j) {
      const int J = li * n + j, K = 2 * J + X, r = K % kRegions, st = J % kFwdStages;
      if (j == 0 && li > 0 &&
          !(ok = warp_wait(&sm.o_free[X], (li - 1) & 1, ab, lim, SITE_FWD_MMA)))
        break;
      // p_full(K) implies K/V stage st has landed: S(K) was computed from it
      if (!(ok = warp_wait(&sm.p_full[X][J & 1], (J >> 1) & 1, ab, lim, SITE_FWD_MMA))) break;
      tc_fence_after();
      const uint32_t vaddr = smem_u32(sm.v[st]);
      // B = [V | ones]: two MN-major 64B-swizzle atoms, the second LBO bytes
      // on; step k reads the next 16 keys (1 KB of V further)
      const uint32_t lbo = smem_u32(sm.ones) - vaddr;
      umma_ts8_elect(d, tmem + r * 128, make_sdesc(vaddr, lbo, 512, kLayoutSW64), 1024 >> 4,
                     kIdescPV, j > 0 ? 1u : 0u);
      umma_commit_elect(&sm.r_free[r]);
      umma_commit_elect(&sm.kv_empty[st]);
      // r_free[r] is exact for this thread: its next phase needs S(K + 3),
      // which needs this phase
      if (!(ok = warp_wait(&sm.r_free[r], (K / kRegions) & 1, ab, lim, SITE_FWD_MMA))) break;
      tc_fence_before();
      if ((threadIdx.x & 31) == 0) st_release_shared(&sm.pv_count[X], J + 1);
    }
  }
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kFwdDrainNs, SITE_FWD_DRAIN);
}

// Waits (bounded) until pv_count[X] >= need, i.e. until the first `need`
// PV steps of tile X have completed.  Warp-uniform.
__device__ __forceinline__ bool wait_pv_count(FwdSmem& sm, int X, int need, const FwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  bool ok = true;
  if (ld_acquire_shared(&sm.pv_count[X]) < need) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_shared(&sm.pv_count[X]) < need) {
      if (*ab) { ok = false; break; }
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        record_error(kErrTimeout, SITE_FWD_SOFTMAX);
        *ab = 1;
        ok = false;
        break;
      }
      __nanosleep(64);
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  if (ok) tc_fence_after();
  return ok;
}

// One work item (the CTA's li-th) of a softmax warp: tile X of the item's
// pair, 32 rows (quarter wq), all 128 key columns of each score tile (one
// thread = one query row).  Returns false on abort.
template <bool kMask>
__device__ __forceinline__ bool fwd_softmax_item(FwdSmem& sm, uint32_t tmem, const FwdParams& p,
                                                 const UnitCoord& u, int tile0, int X, int wq,
                                                 int li) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t tO = tl + kColO + X * kOCols;
  const float sl = p.scale_log2;
  const uint64_t sl2 = pk2(sl, sl);
  const int n = p.n_tiles;
  // region mask: bands of this row's query token.  A warp's 32 rows are a
  // 4 x 8 block of the window and each half (64 columns) of a key tile an
  // 8 x 8 block, so the mask is one warp-uniform decision per key-tile half.
  const bool mask_on = kMask && (u.wy == p.nW / p.nWx - 1 || u.wx == p.nWx - 1);
  int qbr = 0, qbc = 0;
  if (mask_on) {
    int qi0, qj0, qi, qj;
    tile_origin(tile0 + X, p.tiles_x, qi0, qj0);
    tile_row_local(row, qi0, qj0, qi, qj);
    qbr = region_band(u.wy * p.M + qi, p.H, p.M, p.s);
    qbc = region_band(u.wx * p.M + qj, p.W, p.M, p.s);
  }
  float m_run = 0.f;
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const int J = li * n + j;   // key tile counted across items
    const int k = 2 * J + X, r = k % kRegions;
    bool kv0 = true, kv1 = true;
    if (mask_on) {
      int ki0, kj0;
      tile_origin(j, p.tiles_x, ki0, kj0);
      const bool rows_ok = region_band(u.wy * p.M + ki0, p.H, p.M, p.s) == qbr;
      kv0 = rows_ok && region_band(u.wx * p.M + kj0, p.W, p.M, p.s) == qbc;
      kv1 = rows_ok && region_band(u.wx * p.M + kj0 + 8, p.W, p.M, p.s) == qbc;
    }
    const uint32_t tS = tl + r * 128;  // the row's 128 score columns
    const uint32_t tP = tl + r * 128;  // its 128 bf16 P values, packed in pairs
    if (!(ok = warp_wait(&sm.s_full[r], (k / kRegions) & 1, ab, lim, SITE_FWD_SOFTMAX,
                         kFwdSleepNs)))
      break;
    tc_fence_after();
    uint32_t s[4][32];
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld_x32(tS + 32 * q, s[q]);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) reg_fence_x32(s[q]);

    // row maximum over the 128 columns: eight independent chains of 16
    float m8[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t* v = &s[q >> 1][(q & 1) * 16];
      float m = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
      for (int e = 3; e + 1 < 16; e += 2)
        m = fmax3(m, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
      m8[q] = fmaxf(m, __uint_as_float(v[15]));
    }
    float mh0 = fmaxf(fmax3(m8[0], m8[1], m8[2]), m8[3]);
    float mh1 = fmaxf(fmax3(m8[4], m8[5], m8[6]), m8[7]);
    if (!kv0) mh0 = -INFINITY;   // a masked key block adds nothing to the row maximum
    if (!kv1) mh1 = -INFINITY;
    const float mx = fmaxf(mh0, mh1);

    // (a key tile masked for the whole row leaves mx = -inf: the running
    // maximum then stays at a finite floor, so no -inf - -inf arises)
    const float m_tile = mask_on ? fmaxf(mx * sl, -1e30f) : mx * sl;
    float m_new = m_run, alpha = 1.f;
    bool resc = false;
    if (j == 0) {
      m_new = m_tile;
    } else if (m_tile > m_run + kRescaleThreshold) {
      m_new = m_tile;
      alpha = ex2_approx(m_run - m_tile);
      resc = true;
    }
    const uint64_t neg2 = pk2(-m_new, -m_new);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint64_t x2 = ffma2(pk2(__uint_as_float(s[c][2 * e]),
                                      __uint_as_float(s[c][2 * e + 1])), sl2, neg2);
        float p0, p1;
        if (e < kPolyPairs) {
          const uint64_t e2 = exp2_fma2(x2);
          p0 = lo2(e2);
          p1 = hi2(e2);
        } else {
          p0 = ex2_approx(lo2(x2));
          p1 = ex2_approx(hi2(x2));
        }
        pk[e] = pack_bf16x2(p0, p1);
      }
      if (c < 2 ? kv0 : kv1) {
        tmem_st_x16(tP + c * 16, pk);
      } else {
        // a masked block: P = 0 exactly (its own store, so that the
        // unmasked path carries no per-element selects)
        const uint32_t z16[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        tmem_st_x16(tP + c * 16, z16);
      }
    }
    // rescale [O|L] of this warp's rows once every PV step accumulated so
    // far has completed
    if (__any_sync(0xffffffffu, resc)) {
      if (!(ok = wait_pv_count(sm, X, J, p))) break;
      uint32_t o[32], l[16];
      tmem_ld_x32(tO, o);
      tmem_ld_x16(tO + 32, l);
      tmem_wait_ld();
      reg_fence_x32(o);
      reg_fence_x16(l);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
#pragma unroll
      for (int e = 0; e < 16; ++e) l[e] = __float_as_uint(__uint_as_float(l[e]) * alpha);
      tmem_st_x32(tO, o);
      tmem_st_x16(tO + 32, l);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.p_full[X][J & 1]);
    m_run = m_new;
  }
  if (!ok) return false;
  if (!wait_pv_count(sm, X, (li + 1) * n, p)) return false;
  uint32_t o[32], l[16];
  tmem_ld_x32(tO, o);
  tmem_ld_x16(tO + 32, l);
  tmem_wait_ld();
  reg_fence_x32(o);
  reg_fence_x16(l);
  // [O|L]_X is read: the next item's first PV MMA may overwrite it
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&sm.o_free[X]);
  const float l_run = __uint_as_float(l[0]);
  const float inv = 1.f / l_run;
  uint32_t pk[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
  int i0, j0, i, jl;
  tile_origin(tile0 + X, p.tiles_x, i0, j0);
  tile_row_local(row, i0, j0, i, jl);
  const int y = wrap_once(u.wy * p.M + i + p.s, p.H);
  const int x = wrap_once(u.wx * p.M + jl + p.s, p.W);
  const size_t pix = (static_cast<size_t>(u.b) * p.H + y) * p.W + x;
  const size_t row0 = (pix * p.heads + u.head) * 32;   // first of the row's 32 channels
  const size_t n_out = static_cast<size_t>(p.B) * p.H * p.W * p.heads * 32;
  if (rib_guard(row0 + 31, n_out, G_FWD_OUT)) store_row64(p.out + row0, pk, p.out_v8 != 0);
  if (p.gate != nullptr && rib_guard(row0 + 31, n_out, G_FWD_GATE)) {
    // convolutional local attention: O' = O * G at the same pixel and
    // channels (German summary, Methodik §B); O itself is kept for the
    // backward.  The product is formed from the fp32 O, then rounded.
    const uint4* g4 = reinterpret_cast<const uint4*>(p.gate + (pix * p.heads + u.head) * 32);
    uint32_t r16[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 gv = g4[q];
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
        const int c = 8 * q + 2 * e;
        r16[4 * q + e] = pack_bf16x2(__uint_as_float(o[c]) * inv * gf.x,
                                     __uint_as_float(o[c + 1]) * inv * gf.y);
      }
    }
    store_row64(p.out_gated + (pix * p.heads + u.head) * 32, r16, p.gated_v8 != 0);
  }
  const size_t li_ = (static_cast<size_t>(u.b * p.heads + u.head) * p.H + y) * p.W + x;
  if (rib_guard(li_, static_cast<size_t>(p.B) * p.heads * p.H * p.W, G_FWD_LSE))
    p.lse[li_] = (m_run + log2f(l_run)) * 0.69314718055994531f;
  return true;
}

// Warps 0-7: the softmax of every work item of the CTA in turn.
template <bool kMask>
__device__ __forceinline__ void fwd_softmax(FwdSmem& sm, uint32_t tmem, const FwdParams& p, int X,
                                            int wq) {
  int li = 0;
  for (int it = blockIdx.x; it < p.n_items; it += gridDim.x, ++li) {
    UnitCoord u;
    int tile0;
    fwd_item(p, it, u, tile0);
    if (!fwd_softmax_item<kMask>(sm, tmem, p, u, tile0, X, wq, li)) return;
  }
}

// grid min(n_items, SMs) (each CTA walks the work items it, it + gridDim.x,
// ...), block kFwdThreads, dynamic smem kFwdSmemBytes.
// kMask: the shifted-window region mask (a separate instantiation, so that
// the unmasked kernel carries none of its code).
template <bool kMask>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                    const __grid_constant__ CUtensorMap tm_qp,
                    const __grid_constant__ CUtensorMap tm_kp, const FwdParams p) {
  extern __shared__ uint8_t sm_raw_fwd[];
  FwdSmem& sm = *align1024<FwdSmem>(sm_raw_fwd);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.q_full[b], 1);
      mbar_init(&sm.q_free[b], 1);  // the score-MMA thread's commit after an item
      mbar_init(&sm.o_free[b], 4);  // the four epilogue warps of tile b
    }
    for (int st = 0; st < kFwdStages; ++st) {
      mbar_init(&sm.kv_full[st], 1);
      mbar_init(&sm.kv_empty[st], 2);  // one commit from each PV thread
    }
    for (int r = 0; r < kRegions; ++r) {
      mbar_init(&sm.s_full[r], 1);
      mbar_init(&sm.r_free[r], 1);
    }
    for (int X = 0; X < 2; ++X) {
      mbar_init(&sm.p_full[X][0], 4);
      mbar_init(&sm.p_full[X][1], 4);
      sm.pv_count[X] = 0;
    }
    mbar_init(&sm.drain, 3);   // one commit from each MMA-issuing thread
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  {
    // all-ones B atom (bf16 1.0 = 0x3F80), read by the tensor core
    uint4* ones = reinterpret_cast<uint4*>(sm.ones);
    for (int i = threadIdx.x; i < 8192 / 16; i += blockDim.x)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    if (p.rank > 0) {
      tma_prefetch_desc(&tm_qp);
      tma_prefetch_desc(&tm_kp);
    }
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp < 8) {
    regs_inc<kFwdSoftmaxRegs>();
    fwd_softmax<kMask>(sm, tmem, p, warp >> 2, warp & 3);
  } else {
    regs_dec<kFwdServiceRegs>();
    if (warp == 8) {
      if (lane == 0) fwd_producer(sm, &tm_qkv, &tm_qp, &tm_kp, p);
    } else if (warp == 9) {
      fwd_mma_scores(sm, tmem, p);
    } else {
      fwd_mma_pv(sm, tmem, p, warp - 10);  // warps 10, 11
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace rib
