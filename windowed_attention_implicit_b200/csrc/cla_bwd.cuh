// cla_bwd.cuh -- backward of the convolutional local attention gate (CLA).
//
// Forward (cla.cuh; English summary §2.B, German summary Methodik §B,
// Chinese summary §2.B): y = b_dw + DW3x3(x), z = b_pw + y W_pw^T,
// G = sigmoid(z), O' = O * G.  With dO' the gradient of O':
//   dO    = dO' * G                   (what the attention backward receives)
//   dz    = dO' * O * G * (1 - G)
//   db_pw = sum_pixels dz,            dW_pw = sum_pixels dz^T y
//   dy    = dz W_pw
//   db_dw = sum_pixels dy,            dW_dw[c][u][v] = sum_pixels dy[p][c] x[p + (u-1, v-1)][c]
//   dx[p][c] = sum_{u,v} W_dw[c][u][v] dy[p - (u-1, v-1)][c]   (zero outside the map)
//
// Kernels, in launch order (persistent grids, tiles of
// 8 x 16 pixels; sums over pixels go through per-CTA partials and a
// fixed-order reduction, so the weight gradients are deterministic):
//   cla_bwd_dz_kernel    dO, dz (to the workspace), db_pw partials: a plain
//                        element-wise stream
//   cla_bwd_dy_kernel    dy = dz W_pw on the tensor cores (tcgen05; dz tiles
//                        by TMA through a 2-stage ring, W_pw^T resident in
//                        shared memory, two TMEM accumulators)
//   cla_bwd_dwpw_kernel  dW_pw partials = sum over the CTA's 8 x 8-pixel
//                        tiles of dz^T y, y recomputed from x; dz by TMA,
//                        both operands MN-major with the 128-byte swizzle,
//                        the C x C partial in TMEM
//   cla_bwd_dx_kernel    dx, and dW_dw / db_dw partials (FMA pipe, two CTAs per SM,
//                        x and dy halos staged by TMA)
//   cla_bwd_reduce_kernel fixed-order sums of the partials
#pragma once

#include "cla.cuh"

namespace rib {

constexpr int kDzEwThreads = 512;   // element-wise dz kernel
constexpr int kClaDxThreads = 256;

struct ClaBwdParams {
  const __nv_bfloat16* x;
  const float* w_dw;   // [C][3][3]
  const float* b_dw;   // [C]
  const float* w_pw;   // [C][C] ([out][in])
  const __nv_bfloat16* gate;
  const __nv_bfloat16* out;        // O (ungated)
  const __nv_bfloat16* dout_g;     // dO'
  __nv_bfloat16* dout;             // dO = dO' * G
  __nv_bfloat16* dx;
  float *dw_dw, *db_dw, *dw_pw, *db_pw;
  __nv_bfloat16* dz;               // workspace [P][C]
  __nv_bfloat16* dy;               // workspace [P][C]
  float* part_dbpw;                // [grid][C]
  float* part_dwpw;                // [grid][C][C]
  float* part_dw;                  // [grid_dx][10][C]  (9 taps, then the bias)
  int B, H, W, C, tiles_x, tiles_per_img, n_tiles, grid, grid_dx;
  int tiles_x8, n_tiles8;          // 8 x 8-pixel tiles of the dW_pw kernel
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void cla_tile(const ClaBwdParams& p, int t, int& b, int& i0, int& j0) {
  b = t / p.tiles_per_img;
  const int tt = t % p.tiles_per_img;
  i0 = (tt / p.tiles_x) * 8;
  j0 = (tt % p.tiles_x) * 16;
}

__device__ __forceinline__ size_t cla_pix(const ClaBwdParams& p, int b, int i, int j) {
  return (static_cast<size_t>(b) * p.H + i) * p.W + j;
}

// Elements of one [B][H][W][C] tensor: the extent the debug build's guards use.
__device__ __forceinline__ size_t cla_elems(const ClaBwdParams& p) {
  return static_cast<size_t>(p.B) * p.H * p.W * p.C;
}

// Element-wise dz kernel: thread = (pixel slot, channel octet), kDzBatch
// pixels' loads in flight at once (three 16-byte loads a pixel: 48
// registers at 4).
constexpr int kDzBatch = 4;

__device__ __forceinline__ uint4 ldg_nc_v4(const __nv_bfloat16* ptr) {
  return __ldg(reinterpret_cast<const uint4*>(ptr));
}

// -------------------------------------------------------------- dO, dz
// Element-wise: dO = dO' G, dz = dO' O G (1 - G), and the per-CTA db_pw
// partials.  Thread = (pixel slot sl, channel octet k): the octet stays the
// thread's for the whole grid-stride walk over the pixels (pixel
// (n gridDim + blockIdx) slots + sl), so its eight db_pw sums run in a fixed
// order; consecutive threads read consecutive 16-byte octets of one pixel,
// and kDzBatch pixels' loads are in flight before any is used.  A plain
// stream: no shared-memory tile, no tensor-core step (dy is the next
// kernel's).
// grid p.grid, block kDzEwThreads.
__global__ void __launch_bounds__(kDzEwThreads) cla_bwd_dz_kernel(const ClaBwdParams p) {
  __shared__ float red[8 * kDzEwThreads];   // [slot][C] db_pw partials
  const int C = p.C;
  const int octets = C / 8, slots = kDzEwThreads / octets;
  const int sl = threadIdx.x / octets, k = threadIdx.x % octets;
  const bool act = sl < slots;
  const size_t n_pix = static_cast<size_t>(p.B) * p.H * p.W;
  const size_t step = static_cast<size_t>(gridDim.x) * slots;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // db_pw, channels 8k..8k+7
  for (size_t p0 = static_cast<size_t>(blockIdx.x) * slots + sl; act && p0 < n_pix;
       p0 += kDzBatch * step) {
    uint4 dgv[kDzBatch], ov[kDzBatch], gv[kDzBatch];
#pragma unroll
    for (int e = 0; e < kDzBatch; ++e) {
      const size_t pix = p0 + e * step;
      const size_t off = pix * C + 8 * k;
      if (pix < n_pix && rib_guard(off + 7, cla_elems(p), G_CLA_IN)) {
        dgv[e] = ldg_nc_v4(p.dout_g + off);
        ov[e] = ldg_nc_v4(p.out + off);
        gv[e] = ldg_nc_v4(p.gate + off);
      } else {
        dgv[e] = ov[e] = gv[e] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int e = 0; e < kDzBatch; ++e) {
      const size_t pix = p0 + e * step;
      if (pix >= n_pix) continue;
      const size_t off = pix * C + 8 * k;
      const uint32_t dw[4] = {dgv[e].x, dgv[e].y, dgv[e].z, dgv[e].w};
      const uint32_t ow[4] = {ov[e].x, ov[e].y, ov[e].z, ov[e].w};
      const uint32_t gw[4] = {gv[e].x, gv[e].y, gv[e].z, gv[e].w};
      uint32_t dov[4], zv[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 dg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dw[h]));
        const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[h]));
        const float2 gt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[h]));
        const float z0 = dg.x * o.x * gt.x * (1.f - gt.x), z1 = dg.y * o.y * gt.y * (1.f - gt.y);
        dov[h] = pack_bf16x2(dg.x * gt.x, dg.y * gt.y);
        zv[h] = pack_bf16x2(z0, z1);
        acc[2 * h] += z0;
        acc[2 * h + 1] += z1;
      }
      if (rib_guard(off + 7, cla_elems(p), G_CLA_OUT)) {
        *reinterpret_cast<uint4*>(p.dout + off) = make_uint4(dov[0], dov[1], dov[2], dov[3]);
        *reinterpret_cast<uint4*>(p.dz + off) = make_uint4(zv[0], zv[1], zv[2], zv[3]);
      }
    }
  }
  // db_pw partial of this CTA: the slots' sums, added in slot order
  // (thread (sl, k) holds channels 8k..8k+7 at red[sl * C + 8k + e] = red[8 tid + e])
#pragma unroll
  for (int e = 0; e < 8; ++e) red[8 * threadIdx.x + e] = act ? acc[e] : 0.f;
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < slots; ++w) s += red[w * C + c];
    if (rib_guard(static_cast<size_t>(blockIdx.x) * C + c, static_cast<size_t>(p.grid) * C,
                  G_CLA_PART))
      p.part_dbpw[static_cast<size_t>(blockIdx.x) * C + c] = s;
  }
}

// -------------------------------------------------------------- dy
// dy = dz W_pw on tiles of 8 x 16 pixels (M = 128 pixels, N = C, K = C),
// warp-specialised and pipelined:
//   warp 8 (lane 0)  TMA: the dz tile, one 64-channel x 16 x 8 box per
//                    chunk with the 128-byte swizzle (rows = pixels, the
//                    canonical K-major A layout), into a kDyStages ring
//   warp 9           MMAs through an elected lane: C / 16 K-steps into one
//                    of two TMEM accumulators, B = W_pw^T resident in shared
//                    memory, K-major with the 128-byte swizzle (64-channel
//                    chunks of C rows; with no swizzle the tensor core's
//                    shared-memory reads conflict and the MMAs run far
//                    slower)
//   warps 0-7        epilogue: TMEM lanes (pixels) -> bf16 -> a staging tile
//                    in shared memory (the same swizzled layout) -> one TMA
//                    store per 64-channel chunk, so dy leaves as whole
//                    16-pixel rows (6 KB runs); warp w takes lane quarter
//                    w % 4 and every other 32-column chunk from 32 (w / 4)
//                    and frees the accumulator once its TMEM loads are done
// Tile n's MMAs run while the epilogue drains tile n - 1 and the TMA loads
// tile n + 1 and on.
constexpr int kDyThreads = 320;
constexpr int kDyStages = 2;
constexpr uint32_t kDyChunk = 128u * 128u;   // one 64-channel chunk of a 128-pixel tile
__host__ __device__ __forceinline__ size_t cla_dy_smem_bytes(int C) {
  const size_t chunks = (C + 63) / 64;
  return 128ull * C * chunks + (kDyStages + 1) * chunks * kDyChunk + 256 + 1024;
}

// grid p.grid, block kDyThreads, dynamic smem cla_dy_smem_bytes(C).
// tm_dz: dz [B][H][W][C] (workspace), boxes of 64 channels x 16 x 8, 128-byte
// swizzle; tm_dy: dy (workspace), the same boxes.
constexpr int kDyEpiBar = 1;   // named barrier of the eight epilogue warps
__global__ void __launch_bounds__(kDyThreads, 1)
    cla_bwd_dy_kernel(const __grid_constant__ CUtensorMap tm_dz,
                      const __grid_constant__ CUtensorMap tm_dy, const ClaBwdParams p) {
  extern __shared__ uint8_t dy_raw[];
  uint8_t* base = dy_raw + ((1024u - (smem_u32(dy_raw) & 1023u)) & 1023u);
  const int C = p.C, chunks = (C + 63) / 64;
  const uint32_t stage_bytes = static_cast<uint32_t>(chunks) * kDyChunk;
  uint8_t* sA0 = base;                                              // dz stages (1024-aligned)
  uint8_t* sY = base + kDyStages * stage_bytes;                     // dy staging tile
  uint8_t* sB = sY + stage_bytes;                                   // W_pw^T [N = c][K = o]
  const uint32_t b_chunk = static_cast<uint32_t>(C) * 128u;        // one 64-channel K chunk of B
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + static_cast<size_t>(b_chunk) * chunks);
  uint64_t* empty = full + kDyStages;                               // [kDyStages]
  uint64_t* acc_full = empty + kDyStages;                           // [2]
  uint64_t* acc_free = acc_full + 2;                                // [2]
  uint64_t* drain = acc_free + 2;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);
  volatile int* epi_ok = abort_flag + 1;   // [8]: each epilogue warp's status, per tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int my_tiles = (p.n_tiles - static_cast<int>(blockIdx.x) + G - 1) / G;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDyStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_free[i], 8);   // the eight epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // B(n = c, k = o) = W_pw[o][c]: dy[p][c] = sum_o dz[p][o] W_pw[o][c].
  // Element (c, o) sits in K chunk o / 64, row c, 16-byte granule
  // ((o % 64) / 8) ^ (c % 8) of the row's 128 bytes.
  // Pair i is W_pw[2i], W_pw[2i + 1]; eight pairs' loads are issued before
  // any store, so the fill costs a few memory latencies, not one per pair.
  const int n_pairs = C * C / 2;
  for (int i0 = threadIdx.x; i0 < n_pairs; i0 += 8 * blockDim.x) {
    float2 wv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = i0 + e * static_cast<int>(blockDim.x);
      wv[e] = i < n_pairs ? __ldg(reinterpret_cast<const float2*>(p.w_pw) + i)
                          : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = i0 + e * static_cast<int>(blockDim.x);
      if (i >= n_pairs) break;
      const int o = (2 * i) / C, c = (2 * i) % C;
      const uint32_t ko = static_cast<uint32_t>(o & 63) * 2;   // byte in the unswizzled row
      const uint32_t g = static_cast<uint32_t>(o >> 6) * b_chunk;
      *reinterpret_cast<__nv_bfloat16*>(sB + g + c * 128 + (ko ^ ((c & 7) << 4))) =
          __float2bfloat16_rn(wv[e].x);
      *reinterpret_cast<__nv_bfloat16*>(sB + g + (c + 1) * 128 + (ko ^ (((c + 1) & 7) << 4))) =
          __float2bfloat16_rn(wv[e].y);
    }
  }
  fence_proxy_async_smem();
  if (warp == 9) {
    tmem_alloc(tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint64_t lim = p.wait_limit_ns;
  if (warp == 8) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int n = 0; ok && n < my_tiles; ++n) {
        const int s = n % kDyStages;
        if (n >= kDyStages &&
            !(ok = mbar_wait(&empty[s], ((n - kDyStages) / kDyStages) & 1, abort_flag, lim,
                             SITE_CLA)))
          break;
        int b, i0, j0;
        cla_tile(p, static_cast<int>(blockIdx.x) + n * G, b, i0, j0);
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        for (int g = 0; g < chunks; ++g)
          tma_load_4d(sA0 + s * stage_bytes + g * kDyChunk, &tm_dz, &full[s], 64 * g, j0, i0, b);
        ++issued;
      }
      if (*abort_flag) {
        // the loads still in flight land before the CTA exits
        volatile int no_abort = 0;
        for (int n = max(0, issued - kDyStages); n < issued; ++n)
          mbar_wait(&full[n % kDyStages], (n / kDyStages) & 1, &no_abort, 200000000ull, SITE_CLA);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------ MMA issue
    const uint32_t idesc = make_idesc_bf16(128, C, false, false);
    const uint32_t b0 = smem_u32(sB);
    bool ok = true;
    for (int n = 0; ok && n < my_tiles; ++n) {
      const int s = n % kDyStages, a = n & 1;
      ok = warp_wait(&full[s], (n / kDyStages) & 1, abort_flag, lim, SITE_CLA) &&
           (n < 2 || warp_wait(&acc_free[a], ((n - 2) >> 1) & 1, abort_flag, lim, SITE_CLA));
      if (!ok) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA0 + s * stage_bytes);
      for (int ks = 0; ks < C / 16; ++ks) {
        // K-step ks: channels 16 ks.. = chunk ks / 4, 32 (ks % 4) bytes into
        // its rows, for both operands
        const uint64_t adesc =
            make_sdesc(a0 + (ks >> 2) * kDyChunk, 16, 1024, kLayoutSW128) + (ks & 3) * 2;
        const uint64_t bdesc =
            make_sdesc(b0 + (ks >> 2) * b_chunk, 16, 1024, kLayoutSW128) + (ks & 3) * 2;
        umma_ss_elect(tmem + a * 256, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
      }
      umma_commit_elect(&empty[s]);
      umma_commit_elect(&acc_full[a]);
    }
    // every MMA issued above completes before the tensor memory is freed
    umma_commit_elect(drain);
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort, 200000000ull, SITE_CLA);
  } else {
    // ------------------------------------------------ epilogue (warps 0-7)
    const int q = warp & 3, h = warp >> 2;
    const int r = q * 32 + lane;   // tile row = pixel (i0 + r / 16, j0 + r % 16)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool leader = warp == 0 && lane == 0;
    for (int n = 0; n < my_tiles; ++n) {
      const int a = n & 1;
      const bool got = warp_wait(&acc_full[a], (n >> 1) & 1, abort_flag, lim, SITE_CLA);
      // this warp's chunks: columns 32 h + 64 j, j < 3 (C <= 192)
      uint32_t v[3][32];
      if (got) {
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 3; ++j)
          if (32 * h + 64 * j < C) tmem_ld_x32(tmem + a * 256 + lane_off + 32 * h + 64 * j, v[j]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_free[a]);   // the accumulator is in registers
      }
      // the staging tile is free once the previous tile's stores have read it
      if (lane == 0) epi_ok[warp] = got ? 1 : 0;
      if (leader) tma_store_wait_read_all();
      named_bar_sync(kDyEpiBar, 256);
      // one decision for all eight warps, from flags written before the barrier
      const bool all_ok = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3] && epi_ok[4] &&
                          epi_ok[5] && epi_ok[6] && epi_ok[7];
      if (!all_ok) break;
      {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int c0 = 32 * h + 64 * j;
          if (c0 >= C) continue;
          reg_fence_x32(v[j]);
          // row r of chunk c0 / 64: 16-byte granules (c0 % 64) / 8 + t, XOR r % 8
          uint8_t* row = sY + (c0 >> 6) * kDyChunk + r * 128;
          const int g0 = (c0 & 63) >> 3;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint32_t* w = &v[j][8 * t];
            *reinterpret_cast<uint4*>(row + (((g0 + t) ^ (r & 7)) << 4)) =
                make_uint4(pack_bf16x2(__uint_as_float(w[0]), __uint_as_float(w[1])),
                           pack_bf16x2(__uint_as_float(w[2]), __uint_as_float(w[3])),
                           pack_bf16x2(__uint_as_float(w[4]), __uint_as_float(w[5])),
                           pack_bf16x2(__uint_as_float(w[6]), __uint_as_float(w[7])));
          }
        }
        fence_proxy_async_smem();
      }
      named_bar_sync(kDyEpiBar, 256);
      if (leader) {
        int b, i0, j0;
        cla_tile(p, static_cast<int>(blockIdx.x) + n * G, b, i0, j0);
        for (int g = 0; g < chunks; ++g)
          tma_store_4d(&tm_dy, sY + g * kDyChunk, 64 * g, j0, i0, b);
        tma_store_commit();
      }
    }
    // the stores are complete before the kernel's work is considered done
    if (leader) tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -------------------------------------------------------------- dW_pw
// dW_pw = sum over pixels of dz^T y on tiles of 8 x 8 pixels (K = 64 per
// tile).  A tile stored as 64 rows (pixels) of 128 bytes (64 channels) with
// the 128-byte swizzle is, per 64-channel chunk, exactly one canonical
// MN-major atom column of a K = 64 operand: dz^T (M = output channel) and
// y^T (N = input channel) both take that form, 8 KB per chunk, chunks
// kDwpwAtom bytes apart (LBO), 8-pixel row groups 1024 bytes apart (SBO).
// Warp-specialised, 4 C/64 + 1 warps:
//   y warps (4 per chunk)  recompute y = b_dw + DW3x3(x) from the tile's x
//       halo: a thread keeps the 9 taps of one channel octet in registers
//       and walks 4 vertically adjacent pixels of one column (6 halo rows
//       read once each), writing y into one of two y buffers;
//   the last warp           issues the TMA loads (dz, one 64 x 8 x 8 box per
//       chunk with the 128-byte swizzle, into a 3-buffer ring; the x halo,
//       one 64 x 10 x 10 box per chunk, into one of two slots) and, through
//       an elected lane, the MMAs D_m (+)= dz^T[o in 128 m ..] y over the
//       tile's four K = 16 steps (M blocks m = 0, 1 when C > 128), which
//       accumulate in TMEM over all of the CTA's tiles.
// The MMAs of tile n run while the y warps compute tile n + 1.  M block 1
// of a C = 160 or 192 map reads one atom past dz's chunks (the next buffer
// in shared memory): those are accumulator rows o >= C, never read.
constexpr int kDwpwPix = 64;
constexpr uint32_t kDwpwAtom = kDwpwPix * 128;                      // 8 KB
constexpr uint32_t kDwpwHaloBytes = 10u * 10u * 64u * 2u;           // one chunk's halo
constexpr uint32_t kDwpwHaloSlot = (kDwpwHaloBytes + 1023u) & ~1023u;
constexpr int kDwpwA = 3, kDwpwB = 2, kDwpwH = 2;                   // ring depths (tiles)
constexpr int kDwpwMaxChunks = 3;                                   // C <= 192
constexpr int kDwpwThreads = 32 * (4 * kDwpwMaxChunks + 1);         // 416

struct DwpwLayout {
  uint32_t a, b, halo, bars, total;   // byte offsets from a 1024-aligned base
};
__host__ __device__ __forceinline__ DwpwLayout cla_dwpw_layout(int C) {
  const uint32_t chunks = static_cast<uint32_t>((C + 63) / 64);
  const uint32_t chunk_bytes = chunks * kDwpwAtom;
  DwpwLayout L;
  L.a = 0;                                    // kDwpwA dz tiles
  L.b = L.a + kDwpwA * chunk_bytes;           // kDwpwB y tiles (after dz: the atom past the
  L.halo = L.b + kDwpwB * chunk_bytes;        //   last dz tile stays inside the allocation)
  L.bars = L.halo + kDwpwH * chunks * kDwpwHaloSlot;
  L.total = L.bars + 256u;
  return L;
}
__host__ __device__ __forceinline__ size_t cla_dwpw_smem_bytes(int C) {
  return static_cast<size_t>(cla_dwpw_layout(C).total) + 1024;
}

// grid p.grid, block kDwpwThreads, dynamic smem cla_dwpw_smem_bytes(C); C <= 192.
// tm_x: x [B][H][W][C], boxes of 64 channels x 10 x 10 (no swizzle);
// tm_dz: dz [B][H][W][C], boxes of 64 channels x 8 x 8, 128-byte swizzle.
// p.n_tiles8 tiles of 8 x 8 pixels, p.tiles_x8 per image row.
__global__ void __launch_bounds__(kDwpwThreads, 1)
    cla_bwd_dwpw_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_dz, const ClaBwdParams p) {
  extern __shared__ uint8_t dw_raw[];
  uint8_t* base = dw_raw + ((1024u - (smem_u32(dw_raw) & 1023u)) & 1023u);
  const int C = p.C, octets = C / 8, chunks = (C + 63) / 64;
  const DwpwLayout L = cla_dwpw_layout(C);
  const uint32_t chunk_bytes = static_cast<uint32_t>(chunks) * kDwpwAtom;
  uint64_t* dz_full = reinterpret_cast<uint64_t*>(base + L.bars);   // [kDwpwA]
  uint64_t* a_free = dz_full + kDwpwA;                               // [kDwpwA]
  uint64_t* b_free = a_free + kDwpwA;                                // [kDwpwB]
  uint64_t* y_full = b_free + kDwpwB;                                // [kDwpwB]
  uint64_t* h_full = y_full + kDwpwB;                                // [kDwpwH]
  uint32_t* tbase = reinterpret_cast<uint32_t*>(h_full + kDwpwH);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int y_warps = 4 * chunks, mma_warp = kDwpwThreads / 32 - 1;
  const int G = gridDim.x;
  const int my_tiles = (p.n_tiles8 - static_cast<int>(blockIdx.x) + G - 1) / G;
  const int blocks = C > 128 ? 2 : 1;
  const uint32_t tcols = blocks == 2 ? 512u : 256u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDwpwA; ++i) {
      mbar_init(&dz_full[i], 1);
      mbar_init(&a_free[i], 1);
    }
    for (int i = 0; i < kDwpwB; ++i) {
      mbar_init(&b_free[i], 1);
      mbar_init(&y_full[i], 32 * y_warps);
    }
    for (int i = 0; i < kDwpwH; ++i) mbar_init(&h_full[i], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tbase, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  auto tile_origin8 = [&](int n, int& b, int& i0, int& j0) {
    const int t = static_cast<int>(blockIdx.x) + n * G;
    const int per_img = p.n_tiles8 / p.B;
    b = t / per_img;
    const int tt = t % per_img;
    i0 = (tt / p.tiles_x8) * 8;
    j0 = (tt % p.tiles_x8) * 8;
  };
  bool ok = true;
  if (warp == mma_warp) {
    // ------------------------------------------------ TMA loads and MMAs
    int dz_issued = 0, h_issued = 0, dz_seen = 0, n_mma = 0;
    auto issue_dz = [&](int n) {   // lane 0
      int b, i0, j0;
      tile_origin8(n, b, i0, j0);
      uint64_t* bar = &dz_full[n % kDwpwA];
      mbar_arrive_expect_tx(bar, kDwpwAtom * chunks);
      for (int g = 0; g < chunks; ++g)
        tma_load_4d(base + L.a + (n % kDwpwA) * chunk_bytes + g * kDwpwAtom, &tm_dz, bar, 64 * g,
                    j0, i0, b);
      ++dz_issued;
    };
    auto issue_halo = [&](int n) {   // lane 0
      int b, i0, j0;
      tile_origin8(n, b, i0, j0);
      uint64_t* bar = &h_full[n % kDwpwH];
      mbar_arrive_expect_tx(bar, kDwpwHaloBytes * chunks);
      for (int g = 0; g < chunks; ++g)
        tma_load_4d(base + L.halo + ((n % kDwpwH) * chunks + g) * kDwpwHaloSlot, &tm_x, bar,
                    64 * g, j0 - 1, i0 - 1, b);
      ++h_issued;
    };
    if (lane == 0) {
      for (int n = 0; n < 2 && n < my_tiles; ++n) {
        issue_dz(n);
        issue_halo(n);
      }
    }
    const uint32_t idesc = make_idesc_bf16(128, C, true, true);
    for (int n = 0; ok && n < my_tiles; ++n) {
      ok = mbar_wait(&y_full[n % kDwpwB], (n / kDwpwB) & 1, abort_flag, p.wait_limit_ns,
                     SITE_CLA) &&
           mbar_wait(&dz_full[n % kDwpwA], (n / kDwpwA) & 1, abort_flag, p.wait_limit_ns,
                     SITE_CLA);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++dz_seen;
      tc_fence_after();
      const uint32_t a0 = smem_u32(base + L.a + (n % kDwpwA) * chunk_bytes);
      const uint64_t bdesc =
          make_sdesc(smem_u32(base + L.b + (n % kDwpwB) * chunk_bytes), kDwpwAtom, 1024,
                     kLayoutSW128);
      for (int m = 0; m < blocks; ++m) {
        const uint64_t adesc = make_sdesc(a0 + 2 * m * kDwpwAtom, kDwpwAtom, 1024, kLayoutSW128);
        for (int ks = 0; ks < 4; ++ks)
          umma_ss_elect(tmem + 256 * m, adesc + ks * (2048 >> 4), bdesc + ks * (2048 >> 4), idesc,
                        (n > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit_elect(&a_free[n % kDwpwA]);
      umma_commit_elect(&b_free[n % kDwpwB]);
      ++n_mma;
      // the y warps are done with halo slot n % 2: tile n + 2's halo goes there
      if (lane == 0 && n + kDwpwH < my_tiles) issue_halo(n + kDwpwH);
      // dz of tile n + 2 goes to the buffer the MMAs of tile n - 1 read
      if (n + 2 < my_tiles) {
        if (n >= 1)
          ok = mbar_wait(&a_free[(n + 2) % kDwpwA], ((n - 1) / kDwpwA) & 1, abort_flag,
                         p.wait_limit_ns, SITE_CLA);
        ok = __all_sync(0xffffffffu, ok);
        if (ok && lane == 0) issue_dz(n + 2);
      }
    }
    // The accumulator is read once the last tile's MMAs (and so every
    // earlier one) are done.  After an error, every TMA load and MMA still
    // in flight lands before the CTA exits.
    volatile int no_abort = 0;
    const uint64_t drain = 200ull * 1000ull * 1000ull;
    bool w = true;
    if (n_mma > 0)
      w = mbar_wait(&a_free[(n_mma - 1) % kDwpwA], ((n_mma - 1) / kDwpwA) & 1,
                    ok ? abort_flag : &no_abort, ok ? p.wait_limit_ns : drain, SITE_CLA);
    if (!ok) {
      *abort_flag = 1;
      for (int n = dz_seen; n < dz_issued; ++n)
        mbar_wait(&dz_full[n % kDwpwA], (n / kDwpwA) & 1, &no_abort, drain, SITE_CLA);
      // halo loads are issued for tiles the y warps have consumed, or for the
      // next two: wait for those not yet seen complete
      for (int n = max(0, h_issued - kDwpwH); n < h_issued; ++n)
        mbar_wait(&h_full[n % kDwpwH], (n / kDwpwH) & 1, &no_abort, drain, SITE_CLA);
    }
    w = __all_sync(0xffffffffu, w);
    if (!w && lane == 0) *abort_flag = 1;
  } else if (warp < y_warps) {
    // ------------------------------------------------ y = b_dw + DW3x3(x)
    // thread: chunk g = warp / 4, octet ko of it, column j and rows 4 h ..
    // 4 h + 3 of the tile; a warp covers 4 neighbouring columns x 8 octets,
    // so its halo reads and y stores are 512-byte runs
    const int g = warp >> 2, ko = lane & 7;
    const int pg = ((warp & 3) << 2) | (lane >> 3);   // 0..15
    const int j = pg & 7, h = pg >> 3;
    const int k = 8 * g + ko;                         // channel octet
    const bool act = k < octets;
    uint64_t wp[9][4];                                // taps (u, v) of channels 8k .. 8k+7
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 8 * k + 2 * e;
#pragma unroll
      for (int tp = 0; tp < 9; ++tp)
        wp[tp][e] = act ? pk2(p.w_dw[c * 9 + tp], p.w_dw[(c + 1) * 9 + tp]) : 0ull;
    }
    for (int n = 0; ok && n < my_tiles; ++n) {
      ok = mbar_wait(&h_full[n % kDwpwH], (n / kDwpwH) & 1, abort_flag, p.wait_limit_ns,
                     SITE_CLA);
      if (ok && n >= kDwpwB)   // y buffer n % 2 was last read by the MMAs of tile n - 2
        ok = mbar_wait(&b_free[n % kDwpwB], ((n - kDwpwB) / kDwpwB) & 1, abort_flag,
                       p.wait_limit_ns, SITE_CLA);
      if (!ok) break;
      uint8_t* sB = base + L.b + (n % kDwpwB) * chunk_bytes + g * kDwpwAtom;
      const uint8_t* hs = base + L.halo + ((n % kDwpwH) * chunks + g) * kDwpwHaloSlot + ko * 16;
      uint64_t acc[4][4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {   // b_dw (re-read per tile: fewer live registers)
        const float2 bd = act ? __ldg(reinterpret_cast<const float2*>(p.b_dw + 8 * k + 2 * e))
                              : make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[m][e] = pk2(bd.x, bd.y);
      }
      // halo row ri (map row 4h + ri - 1 of the tile) feeds pixel m with tap
      // row u = ri - m; for each pixel the taps arrive in (u, v) order.  Each
      // halo vector is converted once and used by up to three pixels.
#pragma unroll
      for (int ri = 0; ri < 6; ++ri)
#pragma unroll
        for (int v = 0; v < 3; ++v) {
          const uint4 xv = *reinterpret_cast<const uint4*>(hs + ((4 * h + ri) * 10 + j + v) * 128);
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
          uint64_t xf[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            xf[e] = pk2(__uint_as_float(xw[e] << 16), __uint_as_float(xw[e] & 0xffff0000u));
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int u = ri - m;
            if (u < 0 || u > 2) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][e] = ffma2(wp[u * 3 + v][e], xf[e], acc[m][e]);
          }
        }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = (4 * h + m) * 8 + j;
        const uint4 yv = act ? make_uint4(pack_bf16x2(lo2(acc[m][0]), hi2(acc[m][0])),
                                          pack_bf16x2(lo2(acc[m][1]), hi2(acc[m][1])),
                                          pack_bf16x2(lo2(acc[m][2]), hi2(acc[m][2])),
                                          pack_bf16x2(lo2(acc[m][3]), hi2(acc[m][3])))
                             : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sB + r * 128 + ((ko ^ (r & 7)) << 4)) = yv;
      }
      fence_proxy_async_smem();
      mbar_arrive(&y_full[n % kDwpwB]);
    }
  }
  __syncthreads();
  ok = *abort_flag == 0;
  tc_fence_after();
  // the CTA's partial dW_pw: warp w < 8 reads TMEM lanes 32 (w % 4).. of
  // block w / 4 (rows o), all C columns
  if (warp < 4 * blocks) {
    const int q = warp & 3, blk = warp >> 2;
    const int o = blk * 128 + q * 32 + lane;
    const uint32_t taddr = tmem + blk * 256 + (static_cast<uint32_t>(q * 32) << 16);
    float* dst = p.part_dwpw + (static_cast<size_t>(blockIdx.x) * C + o) * C;
    const bool in = o >= C || rib_guard((static_cast<size_t>(blockIdx.x) * C + o) * C + C - 1,
                                        static_cast<size_t>(p.grid) * C * C, G_CLA_PART);
    for (int c0 = 0; ok && c0 < C; c0 += 32) {   // every lane: the TMEM loads are collective
      uint32_t v[32];
      if (my_tiles > 0) {
        tmem_ld_x32(taddr + c0, v);
        tmem_wait_ld();
        reg_fence_x32(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;   // no tiles: an empty sum
      }
      if (o < C && in) {
        float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                              __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// -------------------------------------------------------------- dx, dW_dw, db_dw
// grid p.grid_dx (two CTAs per SM), block kClaDxThreads, dynamic smem
// cla_dx_smem_bytes().  One 64-channel group at a time over all of the CTA's
// tiles (lanes along channel pairs, so each thread keeps 20 partial sums);
// per tile, the 10 x 18-pixel halos of x and dy come by TMA into one of two
// shared-memory stages (the next tile's load overlaps this tile's work; the
// zero padding is the TMA's out-of-range fill), and a warp walks down a
// tile column with the 3 x 3 neighbourhoods of x and dy in registers,
// reading only the new row of each per pixel.
constexpr uint32_t kClaHaloSlot = (kClaHaloBytes + 1023u) & ~1023u;   // one 10 x 18 halo box
__host__ __device__ __forceinline__ size_t cla_dx_smem_bytes() {
  return 4ull * kClaHaloSlot + 64 + 1024;
}

__device__ __forceinline__ float2 cla_lds2(const uint8_t* ptr) {
  const uint32_t v = *reinterpret_cast<const uint32_t*>(ptr);
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
}

__global__ void __launch_bounds__(kClaDxThreads, 2)
    cla_bwd_dx_kernel(const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_dy, const ClaBwdParams p) {
  extern __shared__ uint8_t dx_raw[];
  uint8_t* base = dx_raw + ((1024u - (smem_u32(dx_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + 4 * kClaHaloSlot);   // [2] stages
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.C;
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const int G = gridDim.x;
  const int my_tiles = (p.n_tiles - static_cast<int>(blockIdx.x) + G - 1) / G;
  // stage s: x halo at base + s * chunk, dy halo at base + (2 + s) * chunk
  auto hx = [&](int st) { return base + st * kClaHaloSlot; };
  auto hdy = [&](int st) { return base + (2 + st) * kClaHaloSlot; };
  int issued = 0, consumed = 0;   // halo loads (thread 0 issues; all threads consume)
  auto issue = [&](int g, int k) {
    int b, i0, j0;
    cla_tile(p, static_cast<int>(blockIdx.x) + k * G, b, i0, j0);
    const int st = issued & 1;
    mbar_arrive_expect_tx(&full[st], 2 * kClaHaloBytes);
    tma_load_4d(hx(st), &tm_x, &full[st], 64 * g, j0 - 1, i0 - 1, b);
    tma_load_4d(hdy(st), &tm_dy, &full[st], 64 * g, j0 - 1, i0 - 1, b);
    ++issued;
  };
  bool ok = true;
  for (int g = 0; ok && g * 64 < C; ++g) {
    const int c = g * 64 + 2 * lane;
    const bool act = c < C;
    float w0[9], w1[9], aw0[9], aw1[9], ab0 = 0.f, ab1 = 0.f;
#pragma unroll
    for (int tp = 0; tp < 9; ++tp) {
      w0[tp] = act ? p.w_dw[c * 9 + tp] : 0.f;
      w1[tp] = act ? p.w_dw[(c + 1) * 9 + tp] : 0.f;
      aw0[tp] = aw1[tp] = 0.f;
    }
    if (threadIdx.x == 0 && my_tiles > 0) issue(g, 0);
    for (int k = 0; k < my_tiles; ++k) {
      // the other stage was released by the barrier at the end of tile k-1
      if (threadIdx.x == 0 && k + 1 < my_tiles) issue(g, k + 1);
      const int st = consumed & 1;
      ok = mbar_wait(&full[st], (consumed >> 1) & 1, abort_flag, p.wait_limit_ns, SITE_CLA);
      if (!__syncthreads_and(ok)) {
        ok = false;
        break;
      }
      ++consumed;
      int b, i0, j0;
      cla_tile(p, static_cast<int>(blockIdx.x) + k * G, b, i0, j0);
      const uint8_t* xs = hx(st) + lane * 4;     // halo [10 rows][18 cols][64 ch]
      const uint8_t* ys = hdy(st) + lane * 4;
      for (int jc = warp; act && jc < 16; jc += kClaDxThreads / 32) {
        // xw[u][v] = x(i + u - 1, jc + v - 1), dw[u][v] = dy(i + u - 1, jc + v - 1):
        // halo row i + u, halo column jc + v
        float2 xw[3][3], dw[3][3];
#pragma unroll
        for (int u = 0; u < 3; ++u)
#pragma unroll
          for (int v = 0; v < 3; ++v) {
            const int o = (u * 18 + jc + v) * 128;
            xw[u][v] = cla_lds2(xs + o);
            dw[u][v] = cla_lds2(ys + o);
          }
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) {
          const float2 d = dw[1][1];
          ab0 += d.x;
          ab1 += d.y;
          float dx0 = 0.f, dx1 = 0.f;
#pragma unroll
          for (int u = 0; u < 3; ++u)
#pragma unroll
            for (int v = 0; v < 3; ++v) {
              const int tp = u * 3 + v;
              // dW_dw: dy here times x at (i + u - 1, j + v - 1)
              aw0[tp] = fmaf(d.x, xw[u][v].x, aw0[tp]);
              aw1[tp] = fmaf(d.y, xw[u][v].y, aw1[tp]);
              // dx: tap (u, v) times dy at (i - u + 1, j - v + 1)
              dx0 = fmaf(w0[tp], dw[2 - u][2 - v].x, dx0);
              dx1 = fmaf(w1[tp], dw[2 - u][2 - v].y, dx1);
            }
          if (rib_guard(cla_pix(p, b, i0 + ii, j0 + jc) * C + c + 1, cla_elems(p), G_CLA_OUT))
            *reinterpret_cast<uint32_t*>(p.dx + cla_pix(p, b, i0 + ii, j0 + jc) * C + c) =
                pack_bf16x2(dx0, dx1);
          if (ii < 7) {
#pragma unroll
            for (int v = 0; v < 3; ++v) {
              xw[0][v] = xw[1][v];
              xw[1][v] = xw[2][v];
              dw[0][v] = dw[1][v];
              dw[1][v] = dw[2][v];
              const int o = ((ii + 3) * 18 + jc + v) * 128;
              xw[2][v] = cla_lds2(xs + o);
              dw[2][v] = cla_lds2(ys + o);
            }
          }
        }
      }
      __syncthreads();   // stage st is read: it may be refilled
    }
    if (!ok) break;
    // this group's partials: the warps' sums, added in warp order, staged in
    // the (now idle) first x halo
    float* red = reinterpret_cast<float*>(hx(0));   // [warp][10][64]
#pragma unroll
    for (int tp = 0; tp < 9; ++tp) {
      red[(warp * 10 + tp) * 64 + 2 * lane] = aw0[tp];
      red[(warp * 10 + tp) * 64 + 2 * lane + 1] = aw1[tp];
    }
    red[(warp * 10 + 9) * 64 + 2 * lane] = ab0;
    red[(warp * 10 + 9) * 64 + 2 * lane + 1] = ab1;
    __syncthreads();
    for (int e = threadIdx.x; e < 10 * 64; e += blockDim.x) {
      const int tp = e / 64, cc = e % 64;
      if (g * 64 + cc >= C) continue;
      float sacc = 0.f;
      for (int w = 0; w < kClaDxThreads / 32; ++w) sacc += red[(w * 10 + tp) * 64 + cc];
      if (rib_guard((static_cast<size_t>(blockIdx.x) * 10 + tp) * C + g * 64 + cc,
                    static_cast<size_t>(p.grid_dx) * 10 * C, G_CLA_PART))
        p.part_dw[(static_cast<size_t>(blockIdx.x) * 10 + tp) * C + g * 64 + cc] = sacc;
    }
    __syncthreads();   // red is read before the next group's first halo lands there
  }
  if (!ok && threadIdx.x == 0) {
    // a halo still in flight lands before the CTA exits
    volatile int no_abort = 0;
    for (int q = consumed; q < issued; ++q)
      mbar_wait(&full[q & 1], (q >> 1) & 1, &no_abort, 200ull * 1000ull * 1000ull, SITE_CLA);
  }
}

// -------------------------------------------------------------- reduction
// Fixed-order sums over the CTAs' partials of the C*C dW_pw, C db_pw and
// 10C dW_dw / db_dw gradient elements.  A block takes 32 consecutive
// elements (lane = element, so every warp's loads are 128-byte runs); warp
// w sums the partials of CTAs [w per, (w + 1) per) with four accumulators
// taking the CTAs in turn, and warp 0 adds the kClaRedWarps warp sums in warp
// order, so the result is the same on every run.
constexpr int kClaRedWarps = 16;
__global__ void __launch_bounds__(32 * kClaRedWarps) cla_bwd_reduce_kernel(const ClaBwdParams p) {
  __shared__ float part[kClaRedWarps][32];
  const int C = p.C, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int n_pw = C * C, n_all = n_pw + 11 * C;
  const int idx = blockIdx.x * 32 + lane;
  // element idx: its partials are src[k * stride], k < count
  const float* src = nullptr;
  size_t stride = 0;
  int count = 0;
  if (idx < n_pw) {
    src = p.part_dwpw + idx;
    stride = static_cast<size_t>(n_pw);
    count = p.grid;
  } else if (idx < n_pw + C) {
    src = p.part_dbpw + (idx - n_pw);
    stride = static_cast<size_t>(C);
    count = p.grid;
  } else if (idx < n_all) {
    src = p.part_dw + (idx - n_pw - C);   // [k][10][C]: element (tap, c) at k * 10C + tap * C + c
    stride = 10ull * C;
    count = p.grid_dx;
  }
  const int per = (count + kClaRedWarps - 1) / kClaRedWarps;
  const int k0 = min(count, w * per), k1 = min(count, k0 + per);
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (src) {
    int k = k0;
    for (; k + 3 < k1; k += 4) {
#pragma unroll
      for (int e = 0; e < 4; ++e) a[e] += src[(k + e) * stride];
    }
    for (; k < k1; ++k) a[0] += src[k * stride];
  }
  part[w][lane] = (a[0] + a[1]) + (a[2] + a[3]);
  __syncthreads();
  if (w != 0 || !src) return;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kClaRedWarps; ++i) s += part[i][lane];
  if (idx < n_pw) {
    p.dw_pw[idx] = s;
  } else if (idx < n_pw + C) {
    p.db_pw[idx - n_pw] = s;
  } else {
    const int e = idx - n_pw - C, tp = e / C, c = e % C;
    if (tp < 9) p.dw_dw[c * 9 + tp] = s;
    else p.db_dw[c] = s;
  }
}

}  // namespace rib
