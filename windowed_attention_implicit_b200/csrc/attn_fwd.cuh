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
// CTA = one unit (batch, window, head) x two 128-query tiles (A, B), 640
// threads (5 warpgroups):
//   warps 0-7    softmax group A: warp w owns TMEM lanes 32(w%4).. (query
//                rows) and key columns 64((w/4)%2).. of each score tile; the
//                two warps sharing a row exchange partial row maxima
//   warps 8-15   softmax group B, the same for the second query tile
//   warp  16     TMA producer: Q tiles once, then K/V/Kp tiles through a
//                3-stage shared-memory ring; boxes at rolled map coordinates
//   warp  17     TMEM allocator; issues the score MMAs S_X(j) = Q_X K_j^T
//   warp  18     issues the PV MMAs and releases K/V stages
//   warp  19     idle
// Four softmax warps per SM sub-partition hide the latency of the
// exponential chains (with one row per thread there were only two); the
// softmax warpgroups take 104 registers and the service warpgroup 64
// (setmaxnreg).
// A tcgen05.commit blocks its issuing thread until the thread's MMAs have
// completed (~270 cycles), so scores and PV are issued by two threads: one
// thread's commit never leaves the tensor pipe idle.
// TMEM (512 columns): S_A, S_B fp32 [128 x 128]; P_A, P_B bf16 [128 x 128]
// (64 packed columns each); [O|L]_A, [O|L]_B fp32 [128 x 48].
// Per key tile j and group X: S_X(j) = Q_X K_j^T (MMA) -> online softmax in
// registers -> P_X(j) to TMEM -> [O|L]_X += P_X(j) [V_j | 1] (MMA, A from
// TMEM): the second swizzle atom of the B operand is an all-ones tile, so the
// tensor core also accumulates the softmax denominators L from the very bf16
// P it multiplies with V.  S_X(j+1) is issued as soon as group X has pulled
// S_X(j) into registers, so score MMAs overlap the exponentials.  The
// running max is updated lazily: O and L are rescaled only when the max
// grows by more than 2^8.
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
constexpr int kFwdThreads = 640;
constexpr int kFwdLaunchRegs = 96;      // what the host checks ptxas gave (65536 / 640)
constexpr int kFwdSoftmaxRegs = 104;    // warpgroups 0-3
constexpr int kFwdServiceRegs = 64;     // warpgroup 4
static_assert(4 * 128 * kFwdSoftmaxRegs + 128 * kFwdServiceRegs <= kFwdThreads * kFwdLaunchRegs,
              "register split exceeds the launch budget");
constexpr uint32_t kFwdTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;  // O_X at kColO + 48 X, L at +32
constexpr int kOCols = 48;
// Of every 16 element pairs, how many exponentials run on the FMA pipe.
#ifndef RIB_FWD_POLY_PAIRS
#define RIB_FWD_POLY_PAIRS 6
#endif
constexpr int kPolyPairs = RIB_FWD_POLY_PAIRS;
constexpr uint64_t kFwdDrainNs = 200ull * 1000ull * 1000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdParams {
  int B, H, W, heads, M, s, rank, nWx, nW, tiles_x, n_tiles;
  float scale_log2;  // softmax scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  uint64_t wait_limit_ns;
};

struct __align__(1024) FwdSmem {
  uint8_t qc[2][8192];            // [128 rows][64 B], 64B swizzle
  uint8_t kc[kFwdStages][8192];
  uint8_t v[kFwdStages][8192];
  uint8_t ones[8192];             // bf16 1.0 everywhere: B atom that yields the row sums
  uint8_t qp[2][4096];            // [128 rows][32 B], 32B swizzle
  uint8_t kp[kFwdStages][4096];
  uint64_t q_full;
  uint64_t kv_full[kFwdStages];
  uint64_t kv_empty[kFwdStages];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t pair_bar[2][4];        // the two warps sharing 32 rows of a tile
  uint64_t drain;
  float red_max[2][2][2][128];    // [tile parity][group][column half][row] partial maxima
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kFwdSmemBytes = sizeof(FwdSmem) + 1024;  // + alignment slack
static_assert(kFwdSmemBytes <= 227 * 1024, "forward shared memory exceeds the per-CTA limit");

constexpr uint32_t kIdescS = make_idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = make_idesc_bf16(128, kOCols, false, true);

__device__ __forceinline__ void fwd_producer(FwdSmem& sm, const CUtensorMap* tq,
                                             const CUtensorMap* tqp, const CUtensorMap* tkp,
                                             const FwdParams& p, const UnitCoord& u, int tile0) {
  volatile int* ab = &sm.abort_flag;
  const int hh = u.head;
  const int by = u.wy * p.M + p.s, bx = u.wx * p.M + p.s;
  const bool pos = p.rank > 0;
  mbar_arrive_expect_tx(&sm.q_full, 2u * (8192u + (pos ? 4096u : 0u)));
  for (int X = 0; X < 2; ++X) {
    int i0, j0;
    tile_origin(tile0 + X, p.tiles_x, i0, j0);
    const int y = wrap_once(by + i0, p.H);
    for (int c = 0; c < 2; ++c) {
      const int x = wrap_once(bx + j0 + 8 * c, p.W);
      tma_load_5d(sm.qc[X] + c * 4096, tq, &sm.q_full, 0, hh, x, y, u.b);
      if (pos) tma_load_4d(sm.qp[X] + c * 2048, tqp, &sm.q_full, 0, j0 + 8 * c, i0, hh);
    }
  }
  const uint32_t kv_bytes = 2u * 8192u + (pos ? 4096u : 0u);
  int j = 0;
  for (; j < p.n_tiles; ++j) {
    const int st = j % kFwdStages, use = j / kFwdStages;
    if (use > 0 &&
        !mbar_wait(&sm.kv_empty[st], (use - 1) & 1, ab, p.wait_limit_ns, SITE_FWD_PRODUCER))
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
  if (*ab) {
    // Aborted: let every copy this thread started land before the CTA exits.
    volatile int no_abort = 0;
    mbar_wait(&sm.q_full, 0, &no_abort, kFwdDrainNs, SITE_FWD_DRAIN);
    for (int jj = j - 1; jj >= 0 && jj >= j - kFwdStages; --jj)
      mbar_wait(&sm.kv_full[jj % kFwdStages], (jj / kFwdStages) & 1, &no_abort, kFwdDrainNs,
                SITE_FWD_DRAIN);
  }
}

// Warp 9: S_X(j) = Q_X K_j^T for both query tiles of every key tile, each as
// soon as group X has pulled S_X(j-1) into registers.
__device__ __forceinline__ void fwd_mma_scores(FwdSmem& sm, uint32_t tmem, const FwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const bool pos = p.rank > 0;
  const int n = p.n_tiles;
  bool ok = mbar_wait(&sm.q_full, 0, ab, lim, SITE_FWD_MMA);
  for (int j = 0; ok && j < n; ++j) {
    const int st = j % kFwdStages;
    ok = mbar_wait(&sm.kv_full[st], (j / kFwdStages) & 1, ab, lim, SITE_FWD_MMA);
    for (int X = 0; ok && X < 2; ++X) {
      if (j > 0 && !(ok = mbar_wait(&sm.s_free[X], (j - 1) & 1, ab, lim, SITE_FWD_MMA))) break;
      tc_fence_after();
      const uint32_t d = tmem + kColS + X * 128;
      const uint64_t a = make_sdesc(smem_u32(sm.qc[X]), 16, 512, kLayoutSW64);
      const uint64_t b = make_sdesc(smem_u32(sm.kc[st]), 16, 512, kLayoutSW64);
      umma_ss(d, a, b, kIdescS, 0u);
      umma_ss(d, a + 2, b + 2, kIdescS, 1u);  // channels 16..31: start address + 32 B
      if (pos)
        umma_ss(d, make_sdesc(smem_u32(sm.qp[X]), 16, 256, kLayoutSW32),
                make_sdesc(smem_u32(sm.kp[st]), 16, 256, kLayoutSW32), kIdescS, 1u);
      umma_commit(&sm.s_full[X]);
    }
  }
  // Every MMA issued above must finish before the tensor memory is freed.
  umma_commit(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kFwdDrainNs, SITE_FWD_DRAIN);
}

// Warp 10: [O|L]_X += P_X(j) [V_j | 1] once group X has written P_X(j), then
// releases the K/V stage of tile j.
__device__ __forceinline__ void fwd_mma_pv(FwdSmem& sm, uint32_t tmem, const FwdParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int n = p.n_tiles;
  bool ok = true;
  for (int j = 0; ok && j < n; ++j) {
    const int st = j % kFwdStages;
    const uint32_t vaddr = smem_u32(sm.v[st]);
    // B = [V | ones]: two MN-major 64B-swizzle atoms, the second LBO bytes on
    const uint32_t lbo = smem_u32(sm.ones) - vaddr;
    for (int X = 0; ok && X < 2; ++X) {
      // p_full_X(j) implies K/V stage st has landed: S_X(j) was computed from it
      if (!(ok = mbar_wait(&sm.p_full[X], j & 1, ab, lim, SITE_FWD_MMA))) break;
      tc_fence_after();
      const uint32_t d = tmem + kColO + X * kOCols;
      const uint32_t a = tmem + kColP + X * 64;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        umma_ts(d, a + k * 8, make_sdesc(vaddr + k * 1024, lbo, 512, kLayoutSW64), kIdescPV,
                (j > 0 || k > 0) ? 1u : 0u);
      umma_commit(&sm.pv_done[X]);
    }
    if (ok) umma_commit(&sm.kv_empty[st]);
  }
  umma_commit(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kFwdDrainNs, SITE_FWD_DRAIN);
}

__device__ __forceinline__ void fwd_softmax(FwdSmem& sm, uint32_t tmem, const FwdParams& p,
                                            const UnitCoord& u, int tile0, int X, int h, int wq) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t tS = tmem + lane_off + kColS + X * 128 + 64 * h;
  const uint32_t tP = tmem + lane_off + kColP + X * 64 + 32 * h;
  const uint32_t tO = tmem + lane_off + kColO + X * kOCols;
  const float sl = p.scale_log2;
  const uint64_t sl2 = pk2(sl, sl);
  const int n = p.n_tiles;
  float m_run = 0.f;
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    if (!(ok = warp_wait(&sm.s_full[X], j & 1, ab, lim, SITE_FWD_SOFTMAX))) break;
    tc_fence_after();
    uint32_t s[2][32];
    tmem_ld_x32(tS, s[0]);
    tmem_ld_x32(tS + 32, s[1]);
    tmem_wait_ld();
    reg_fence_x32(s[0]);
    reg_fence_x32(s[1]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.s_free[X]);

    // row maximum: this warp's 64 columns, then the partner warp's
    float mx = __uint_as_float(s[0][0]);
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int e = (c == 0 ? 1 : 0); e + 1 < 32; e += 2)
        mx = fmax3(mx, __uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1]));
    mx = fmaxf(mx, __uint_as_float(s[1][31]));
    sm.red_max[j & 1][X][h][row] = mx;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.pair_bar[X][wq]);
    if (!(ok = warp_wait(&sm.pair_bar[X][wq], j & 1, ab, lim, SITE_FWD_SOFTMAX))) break;
    mx = fmaxf(mx, sm.red_max[j & 1][X][h ^ 1][row]);

    const float m_tile = mx * sl;
    float m_new = m_run, alpha = 1.f;
    bool resc = false;
    if (j == 0) {
      m_new = m_tile;
    } else if (m_tile > m_run + kRescaleThreshold) {
      m_new = m_tile;
      alpha = ex2_approx(m_run - m_tile);
      resc = true;
    }
    if (j > 0) {
      // P_X and [O|L]_X are free once PV_X(j-1) has completed.
      if (!(ok = warp_wait(&sm.pv_done[X], (j - 1) & 1, ab, lim, SITE_FWD_SOFTMAX))) break;
      tc_fence_after();
    }
    const uint64_t neg2 = pk2(-m_new, -m_new);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
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
      tmem_st_x16(tP + c * 16, pk);
    }
    // the column-half-0 warp of each row pair rescales [O|L] (both halves
    // took the same decision from the same row maximum)
    if (h == 0 && j > 0 && __any_sync(0xffffffffu, resc)) {
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
    if (lane == 0) mbar_arrive(&sm.p_full[X]);
    m_run = m_new;
  }
  if (!ok || h != 0) return;
  if (!warp_wait(&sm.pv_done[X], (n - 1) & 1, ab, lim, SITE_FWD_SOFTMAX)) return;
  tc_fence_after();
  uint32_t o[32], l[16];
  tmem_ld_x32(tO, o);
  tmem_ld_x16(tO + 32, l);
  tmem_wait_ld();
  reg_fence_x32(o);
  reg_fence_x16(l);
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
  uint4* dst = reinterpret_cast<uint4*>(p.out + (pix * p.heads + u.head) * 32);
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  p.lse[(static_cast<size_t>(u.b * p.heads + u.head) * p.H + y) * p.W + x] =
      (m_run + log2f(l_run)) * 0.69314718055994531f;
}

// grid (n_tiles / 2, units), block kFwdThreads, dynamic smem kFwdSmemBytes.
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                    const __grid_constant__ CUtensorMap tm_qp,
                    const __grid_constant__ CUtensorMap tm_kp, const FwdParams p) {
  extern __shared__ uint8_t sm_raw_fwd[];
  FwdSmem& sm = *align1024<FwdSmem>(sm_raw_fwd);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UnitCoord u = decode_unit(blockIdx.y, p.heads, p.nW, p.nWx);
  const int tile0 = blockIdx.x * 2;
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int st = 0; st < kFwdStages; ++st) {
      mbar_init(&sm.kv_full[st], 1);
      mbar_init(&sm.kv_empty[st], 1);
    }
    for (int X = 0; X < 2; ++X) {
      mbar_init(&sm.s_full[X], 1);
      mbar_init(&sm.s_free[X], 8);
      mbar_init(&sm.p_full[X], 8);
      mbar_init(&sm.pv_done[X], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&sm.pair_bar[X][q], 2);
    }
    mbar_init(&sm.drain, 2);   // one commit from each MMA-issuing thread
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
  if (warp == 16 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    if (p.rank > 0) {
      tma_prefetch_desc(&tm_qp);
      tma_prefetch_desc(&tm_kp);
    }
  }
  if (warp == 17) {
    tmem_alloc(&sm.tmem_base, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp < 16) {
    regs_inc<kFwdSoftmaxRegs>();
    fwd_softmax(sm, tmem, p, u, tile0, warp >> 3, (warp >> 2) & 1, warp & 3);
  } else {
    regs_dec<kFwdServiceRegs>();
    if (warp == 16) {
      if (lane == 0) fwd_producer(sm, &tm_qkv, &tm_qp, &tm_kp, p, u, tile0);
    } else if (warp == 17) {
      if (lane == 0) fwd_mma_scores(sm, tmem, p);
    } else if (warp == 18) {
      if (lane == 0) fwd_mma_pv(sm, tmem, p);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace rib
