// attn_fwd_tf32.cuh -- RIB window attention forward for fp32 inputs on the
// tcgen05 tensor cores in tf32 (kind::tf32).
//
// The same computation as attn_fwd.cuh (the augmented score of the English
// summary, Technical Summary §2.A steps 3-4 and the score equation:
// S = tau [Qc,Qp][Kc,Kp]^T = tau (Qc Kc^T + Qp Kp^T), online softmax over
// the window's keys, O = P V), for callers whose features and position
// tokens are fp32: nothing is rounded to bf16.  The tensor cores read the
// fp32 operands as tf32 (10 explicit mantissa bits against bf16's 7) and
// accumulate in fp32; P is rounded to tf32 by the softmax threads (round to
// nearest) and the softmax denominator is summed from the rounded values, so
// numerator and denominator see the same P.
//
// One CTA per (unit, 128-query tile), 192 threads:
//   warps 0-3  softmax: thread = query row (TMEM lane), all 128 key columns
//   warp  4    TMA producer: the Q tile, then K/V/Kp tiles through a
//              2-stage ring (boxes at rolled map coordinates, as in the bf16
//              kernels: the cyclic shift costs nothing)
//   warp  5    TMEM allocator; issues the MMAs through one elected lane
// V is loaded through its own tensor map with the 128-byte swizzle of
// 32-byte granules: a tf32 operand read MN-major (channels contiguous) must
// be in that layout (4-row swizzle atoms, 512 bytes apart along the keys).
// TMEM (256 columns, so two CTAs share an SM): S of the current key tile in
// columns 0-127, overwritten in place by P; O in columns 128-159.
// Per key tile j: S(j) = Q K_j^T (4 content + 2 positional K=8 steps) ->
// softmax warps: row max, rescale of O and l when the max grows (O is final
// for tile j-1: S(j) is issued only after PV(j-1) completed), P in place ->
// O += P V_j (16 K=8 steps, A = P from TMEM, B = V read MN-major).  The
// steps of one CTA are serial; the other CTA on the SM fills the gaps.  The
// variant exists for precision, not speed: the bf16 kernel is the fast path.
#pragma once

#include "geom.cuh"
#include "ptx.cuh"

namespace rib {

constexpr int kTfThreads = 192;
constexpr int kTfStages = 2;
constexpr uint32_t kTfTmemCols = 256;
constexpr uint32_t kTfColS = 0, kTfColO = 128;
constexpr uint64_t kTfDrainNs = 200ull * 1000ull * 1000ull;

struct TfParams {
  int B, H, W, heads, M, s, rank, nWx, nW, tiles_x, n_tiles;
  float scale_log2;  // softmax scale * log2(e)
  float* out;        // fp32 [B][H][W][heads][32]
  float* lse;        // fp32 [B][heads][H][W]
  uint64_t wait_limit_ns;
};

struct __align__(1024) TfSmem {
  uint8_t qc[16384];              // [128 rows][32 fp32], 128B swizzle
  uint8_t kc[kTfStages][16384];
  uint8_t v[kTfStages][16384];    // read MN-major by the PV MMA (32B-granule swizzle)
  uint8_t qp[8192];               // [128 rows][16 fp32], 64B swizzle
  uint8_t kp[kTfStages][8192];
  uint64_t q_full;
  uint64_t kv_full[kTfStages], kv_empty[kTfStages];
  uint64_t s_full, p_full, pv_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kTfSmemBytes = sizeof(TfSmem) + 1024;  // + alignment slack
static_assert(2 * kTfSmemBytes <= 228 * 1024, "two tf32 forward CTAs must fit one SM");

constexpr uint32_t kIdescTfS = make_idesc_tf32(128, 128, false, false);
constexpr uint32_t kIdescTfPV = make_idesc_tf32(128, 32, false, true);

// Warp 4, lane 0.
__device__ __forceinline__ void tf_producer(TfSmem& sm, const CUtensorMap* tq,
                                            const CUtensorMap* tv, const CUtensorMap* tqp,
                                            const CUtensorMap* tkp, const TfParams& p,
                                            const UnitCoord& u, int qt) {
  volatile int* ab = &sm.abort_flag;
  const bool pos = p.rank > 0;
  const int hh = u.head;
  const int by = u.wy * p.M + p.s, bx = u.wx * p.M + p.s;
  {
    int i0, j0;
    tile_origin(qt, p.tiles_x, i0, j0);
    const int y = wrap_once(by + i0, p.H);
    mbar_arrive_expect_tx(&sm.q_full, 16384u + (pos ? 8192u : 0u));
    for (int c = 0; c < 2; ++c) {
      const int x = wrap_once(bx + j0 + 8 * c, p.W);
      tma_load_5d(sm.qc + c * 8192, tq, &sm.q_full, 0, hh, x, y, u.b);
      if (pos) tma_load_4d(sm.qp + c * 4096, tqp, &sm.q_full, 0, j0 + 8 * c, i0, hh);
    }
  }
  const uint32_t kv_bytes = 2u * 16384u + (pos ? 8192u : 0u);
  int j = 0;
  for (; j < p.n_tiles; ++j) {
    const int st = j % kTfStages, use = j / kTfStages;
    if (use > 0 &&
        !mbar_wait(&sm.kv_empty[st], (use - 1) & 1, ab, p.wait_limit_ns, SITE_FWD_PRODUCER))
      break;
    mbar_arrive_expect_tx(&sm.kv_full[st], kv_bytes);
    int i0, j0;
    tile_origin(j, p.tiles_x, i0, j0);
    const int y = wrap_once(by + i0, p.H);
    for (int c = 0; c < 2; ++c) {
      const int x = wrap_once(bx + j0 + 8 * c, p.W);
      tma_load_5d(sm.kc[st] + c * 8192, tq, &sm.kv_full[st], 0, p.heads + hh, x, y, u.b);
      tma_load_5d(sm.v[st] + c * 8192, tv, &sm.kv_full[st], 0, 2 * p.heads + hh, x, y, u.b);
      if (pos) tma_load_4d(sm.kp[st] + c * 4096, tkp, &sm.kv_full[st], 0, j0 + 8 * c, i0, hh);
    }
  }
  if (*ab) {
    // Aborted: let every copy this thread started land before the CTA exits.
    volatile int no_abort = 0;
    mbar_wait(&sm.q_full, 0, &no_abort, kTfDrainNs, SITE_FWD_DRAIN);
    for (int jj = j - 1; jj >= 0 && jj >= j - kTfStages; --jj)
      mbar_wait(&sm.kv_full[jj % kTfStages], (jj / kTfStages) & 1, &no_abort, kTfDrainNs,
                SITE_FWD_DRAIN);
  }
}

// Warp 5, all lanes (one elected lane issues).
__device__ __forceinline__ void tf_mma(TfSmem& sm, uint32_t tmem, const TfParams& p) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const bool pos = p.rank > 0;
  bool ok = warp_wait(&sm.q_full, 0, ab, lim, SITE_FWD_MMA);
  for (int j = 0; ok && j < p.n_tiles; ++j) {
    const int st = j % kTfStages;
    ok = warp_wait(&sm.kv_full[st], (j / kTfStages) & 1, ab, lim, SITE_FWD_MMA) &&
         (j == 0 || warp_wait(&sm.pv_done, (j - 1) & 1, ab, lim, SITE_FWD_MMA));
    if (!ok) break;
    tc_fence_after();
    // S = Q_aug K_aug^T: K = 8 fp32 (32 bytes) per step inside the swizzle atoms
    const uint64_t a = make_sdesc(smem_u32(sm.qc), 16, 1024, kLayoutSW128);
    const uint64_t b = make_sdesc(smem_u32(sm.kc[st]), 16, 1024, kLayoutSW128);
    for (int k = 0; k < 4; ++k)
      umma_tf32_ss_elect(tmem + kTfColS, a + 2 * k, b + 2 * k, kIdescTfS, k > 0 ? 1u : 0u);
    if (pos) {
      const uint64_t ap = make_sdesc(smem_u32(sm.qp), 16, 512, kLayoutSW64);
      const uint64_t bp = make_sdesc(smem_u32(sm.kp[st]), 16, 512, kLayoutSW64);
      for (int k = 0; k < 2; ++k)
        umma_tf32_ss_elect(tmem + kTfColS, ap + 2 * k, bp + 2 * k, kIdescTfS, 1u);
    }
    umma_commit_elect(&sm.s_full);
    if (!(ok = warp_wait(&sm.p_full, j & 1, ab, lim, SITE_FWD_MMA))) break;
    tc_fence_after();
    // O += P V: B = V, MN-major (channels contiguous, one 128-byte atom
    // wide), two 4-key atoms of 512 bytes per step; A = 8 fp32 columns of P
    const uint64_t bv = make_sdesc(smem_u32(sm.v[st]), 16384, 512, kLayoutSW128B32);
    for (int k = 0; k < 16; ++k)
      umma_tf32_ts_elect(tmem + kTfColO, tmem + kTfColS + 8 * k, bv + 64 * k, kIdescTfPV,
                         (j > 0 || k > 0) ? 1u : 0u);
    umma_commit_elect(&sm.pv_done);
    umma_commit_elect(&sm.kv_empty[st]);
  }
  // Every MMA issued above must finish before the tensor memory is freed.
  umma_commit_elect(&sm.drain);
  volatile int no_abort = 0;
  mbar_wait(&sm.drain, 0, &no_abort, kTfDrainNs, SITE_FWD_DRAIN);
}

// Warps 0-3: thread = query row of the tile.
__device__ __forceinline__ void tf_softmax(TfSmem& sm, uint32_t tmem, const TfParams& p,
                                           const UnitCoord& u, int qt, int wq) {
  volatile int* ab = &sm.abort_flag;
  const uint64_t lim = p.wait_limit_ns;
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const float sl = p.scale_log2;
  float m_run = 0.f, l_run = 0.f;
  for (int j = 0; j < p.n_tiles; ++j) {
    if (!warp_wait(&sm.s_full, j & 1, ab, lim, SITE_FWD_SOFTMAX)) return;
    tc_fence_after();
    uint32_t s[32];
    float mx = -INFINITY;
    for (int c = 0; c < 4; ++c) {
      tmem_ld_x32(tl + kTfColS + 32 * c, s);
      tmem_wait_ld();
      reg_fence_x32(s);
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        mx = fmax3(mx, __uint_as_float(s[e]), __uint_as_float(s[e + 1]));
    }
    const float m_tile = mx * sl;
    float m_new = m_tile;
    if (j > 0) {
      m_new = fmaxf(m_run, m_tile);
      const float alpha = ex2_approx(m_run - m_new);
      l_run *= alpha;
      // O holds PV(0..j-1), complete: S(j) was issued after PV(j-1) finished
      if (__any_sync(0xffffffffu, m_new > m_run)) {
        uint32_t o[32];
        tmem_ld_x32(tl + kTfColO, o);
        tmem_wait_ld();
        reg_fence_x32(o);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st_x32(tl + kTfColO, o);
      }
    }
    for (int c = 0; c < 4; ++c) {
      tmem_ld_x32(tl + kTfColS + 32 * c, s);
      tmem_wait_ld();
      reg_fence_x32(s);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float pe = round_tf32(ex2_approx(fmaf(__uint_as_float(s[e]), sl, -m_new)));
        l_run += pe;
        s[e] = __float_as_uint(pe);
      }
      tmem_st_x32(tl + kTfColS + 32 * c, s);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.p_full);
    m_run = m_new;
  }
  if (!warp_wait(&sm.pv_done, (p.n_tiles - 1) & 1, ab, lim, SITE_FWD_SOFTMAX)) return;
  tc_fence_after();
  uint32_t o[32];
  tmem_ld_x32(tl + kTfColO, o);
  tmem_wait_ld();
  reg_fence_x32(o);
  const float inv = 1.f / l_run;
  int i0, j0, i, jl;
  tile_origin(qt, p.tiles_x, i0, j0);
  tile_row_local(row, i0, j0, i, jl);
  const int y = wrap_once(u.wy * p.M + i + p.s, p.H);
  const int x = wrap_once(u.wx * p.M + jl + p.s, p.W);
  const size_t pix = (static_cast<size_t>(u.b) * p.H + y) * p.W + x;
  const size_t row0 = (pix * p.heads + u.head) * 32;
  float4* dst = reinterpret_cast<float4*>(p.out + row0);
  if (rib_guard(row0 + 31, static_cast<size_t>(p.B) * p.H * p.W * p.heads * 32, G_TF32_OUT)) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      dst[q] = make_float4(__uint_as_float(o[4 * q]) * inv, __uint_as_float(o[4 * q + 1]) * inv,
                           __uint_as_float(o[4 * q + 2]) * inv,
                           __uint_as_float(o[4 * q + 3]) * inv);
  }
  const size_t li_ = (static_cast<size_t>(u.b * p.heads + u.head) * p.H + y) * p.W + x;
  if (rib_guard(li_, static_cast<size_t>(p.B) * p.heads * p.H * p.W, G_TF32_LSE))
    p.lse[li_] = (m_run + log2f(l_run)) * 0.69314718055994531f;
}

// grid (n_tiles, units), block kTfThreads, dynamic smem kTfSmemBytes.
__global__ void __launch_bounds__(kTfThreads, 2)
    attn_fwd_tf32_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_qp,
                         const __grid_constant__ CUtensorMap tm_kp, const TfParams p) {
  extern __shared__ uint8_t sm_raw_tf[];
  TfSmem& sm = *align1024<TfSmem>(sm_raw_tf);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x;
  const UnitCoord u = decode_unit(blockIdx.y, p.heads, p.nW, p.nWx);
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int st = 0; st < kTfStages; ++st) {
      mbar_init(&sm.kv_full[st], 1);
      mbar_init(&sm.kv_empty[st], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, 4);     // the four softmax warps
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_v);
    if (p.rank > 0) {
      tma_prefetch_desc(&tm_qp);
      tma_prefetch_desc(&tm_kp);
    }
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, kTfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp < 4) {
    tf_softmax(sm, tmem, p, u, qt, warp);
  } else if (warp == 4) {
    if (lane == 0) tf_producer(sm, &tm_qkv, &tm_v, &tm_qp, &tm_kp, p, u, qt);
  } else {
    tf_mma(sm, tmem, p);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTfTmemCols);
  }
}

}  // namespace rib
