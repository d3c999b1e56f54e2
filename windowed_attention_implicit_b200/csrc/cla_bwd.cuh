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
//   cla_bwd_dz_kernel    dO, dz (to the workspace), db_pw partials, and
//                        dy = dz W_pw on the tensor cores (tcgen05, dz tile
//                        and W_pw^T in shared memory, accumulator in TMEM)
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

constexpr int kDzThreads = 384;   // dz kernel (12 warps: up to 168 registers a thread)
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

// Element-wise part of the dz kernel: thread = (pixel slot, channel octet),
// kDzBatch pixels' loads in flight at once (three 16-byte loads a pixel:
// 48 registers at 4).
constexpr int kDzBatch = 4;
// W_pw^T (2 C^2 bytes) | two dz tiles (256 C bytes each) | db_pw slots | barriers
__host__ __device__ __forceinline__ size_t cla_dz_smem_bytes(int C) {
  return 2ull * C * C + 2ull * 256 * C + 4ull * 8 * kDzThreads + 64 + 1024;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const __nv_bfloat16* ptr) {
  return __ldg(reinterpret_cast<const uint4*>(ptr));
}

// -------------------------------------------------------------- dz and dy
// grid p.grid, block kDzThreads, dynamic smem cla_dz_smem_bytes(C).
// The dz tile and the dy accumulator are double-buffered: tile n's MMAs run
// while the threads do tile n + 1's element-wise part, and its dy is read
// from TMEM after that.
__global__ void __launch_bounds__(kDzThreads, 1) cla_bwd_dz_kernel(const ClaBwdParams p) {
  extern __shared__ uint8_t dz_raw[];
  uint8_t* base = dz_raw + ((1024u - (smem_u32(dz_raw) & 1023u)) & 1023u);
  const int C = p.C;
  uint8_t* sB = base;                                   // W_pw^T bf16 [N = c][K = o]
  uint8_t* sA0 = base + 2ull * C * C;                   // dz bf16 [M = 128 pixels][K = o], x2
  float* red = reinterpret_cast<float*>(sA0 + 2ull * 256 * C);   // [slot][C] db_pw partials
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 8 * kDzThreads);   // [2]
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 3);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // B(n = c, k = o) = W_pw[o][c]: dy[p][c] = sum_o dz[p][o] W_pw[o][c]
  for (int i = threadIdx.x; i < C * C / 2; i += blockDim.x) {
    const int o = (2 * i) / C, c = (2 * i) % C;
    const float2 w = *reinterpret_cast<const float2*>(p.w_pw + static_cast<size_t>(o) * C + c);
    *reinterpret_cast<__nv_bfloat16*>(sB + cla_kmajor_offset(c, o, C)) = __float2bfloat16_rn(w.x);
    *reinterpret_cast<__nv_bfloat16*>(sB + cla_kmajor_offset(c + 1, o, C)) =
        __float2bfloat16_rn(w.y);
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint32_t idesc = make_idesc_bf16(128, C, false, false);
  const uint64_t bdesc = make_sdesc(smem_u32(sB), 128, 16 * C, kLayoutNone);
  // element-wise part: thread = (pixel slot sl, channel octet k); slots
  // take pixels sl, sl + slots, ...; consecutive threads read consecutive
  // 16-byte octets of one pixel
  const int octets = C / 8, slots = kDzThreads / octets;
  const int sl = threadIdx.x / octets, k = threadIdx.x % octets;
  const bool act = sl < slots;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // db_pw, channels 8k..8k+7
  const int G = gridDim.x;
  const int my_tiles = (p.n_tiles - static_cast<int>(blockIdx.x) + G - 1) / G;
  // dy of tile n (accumulator n % 2) to the workspace: warp w reads TMEM
  // lanes 32 (w % 4).. (pixels), columns 32 (w / 4) + 128 i
  auto drain_dy = [&](int n) -> bool {
    bool ok = mbar_wait(&bar[n & 1], (n >> 1) & 1, abort_flag, p.wait_limit_ns, SITE_CLA);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (!ok) return false;
    int b, i0, j0;
    cla_tile(p, static_cast<int>(blockIdx.x) + n * G, b, i0, j0);
    const int q = warp & 3, slot = warp >> 2;
    const int r = q * 32 + lane;
    const size_t pix = cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15));
    __nv_bfloat16* dst = p.dy + pix * C;
    const uint32_t taddr = tmem + (n & 1) * 256 + (static_cast<uint32_t>(q * 32) << 16);
    for (int c0 = 32 * slot; c0 < C; c0 += 32 * (kDzThreads / 128)) {
      uint32_t v[32];
      tmem_ld_x32(taddr + c0, v);
      tmem_wait_ld();
      reg_fence_x32(v);
      if (!rib_guard(pix * C + c0 + 31, cla_elems(p), G_CLA_OUT)) continue;
      uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        d4[e] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                           pack_bf16x2(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                           pack_bf16x2(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                           pack_bf16x2(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
    }
    return true;
  };
  bool ok = true;
  int n_mma = 0;
  for (int n = 0; n < my_tiles; ++n) {
    int b, i0, j0;
    cla_tile(p, static_cast<int>(blockIdx.x) + n * G, b, i0, j0);
    uint8_t* sA = sA0 + (n & 1) * 256ull * C;   // last read by tile n - 2's MMAs, drained
    for (int r0 = sl; ok && act && r0 < 128; r0 += kDzBatch * slots) {
      uint4 dgv[kDzBatch], ov[kDzBatch], gv[kDzBatch];
#pragma unroll
      for (int e = 0; e < kDzBatch; ++e) {
        const int r = r0 + e * slots;
        if (r < 128) {
          const size_t off = cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15)) * C + 8 * k;
          if (!rib_guard(off + 7, cla_elems(p), G_CLA_IN)) {
            dgv[e] = ov[e] = gv[e] = make_uint4(0, 0, 0, 0);
            continue;
          }
          dgv[e] = ldg_nc_v4(p.dout_g + off);
          ov[e] = ldg_nc_v4(p.out + off);
          gv[e] = ldg_nc_v4(p.gate + off);
        }
      }
#pragma unroll
      for (int e = 0; e < kDzBatch; ++e) {
        const int r = r0 + e * slots;
        if (r >= 128) continue;
        const size_t off = cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15)) * C + 8 * k;
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
        const uint4 z4 = make_uint4(zv[0], zv[1], zv[2], zv[3]);
        if (rib_guard(off + 7, cla_elems(p), G_CLA_OUT)) {
          *reinterpret_cast<uint4*>(p.dout + off) = make_uint4(dov[0], dov[1], dov[2], dov[3]);
          *reinterpret_cast<uint4*>(p.dz + off) = z4;
        }
        *reinterpret_cast<uint4*>(sA + cla_kmajor_offset(r, 8 * k, C)) = z4;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) break;
    // ---- dy = dz W_pw  (M = 128 pixels, N = C, K = C) into accumulator n % 2
    if (warp == 0) {
      const uint64_t adesc = make_sdesc(smem_u32(sA), 128, 16 * C, kLayoutNone);
      for (int ks = 0; ks < C / 16; ++ks)
        umma_ss_elect(tmem + (n & 1) * 256, adesc + ks * 16, bdesc + ks * 16, idesc,
                      ks > 0 ? 1u : 0u);
      umma_commit_elect(&bar[n & 1]);
    }
    ++n_mma;
    // tile n - 1's dy, whose MMAs ran during this tile's element-wise part
    if (n >= 1) ok = drain_dy(n - 1);
    tc_fence_before();
    ok = __syncthreads_and(ok);   // accumulator (n - 1) % 2 and dz tile (n - 1) % 2 are free
    tc_fence_after();
    if (!ok) break;
  }
  if (ok && n_mma > 0) ok = drain_dy(n_mma - 1);
  ok = __syncthreads_and(ok);
  if (!ok && warp == 0 && n_mma > 0) {
    // the last tile's MMAs (and every earlier one) land before the CTA exits
    volatile int no_abort = 0;
    mbar_wait(&bar[(n_mma - 1) & 1], ((n_mma - 1) >> 1) & 1, &no_abort, 200ull * 1000ull * 1000ull,
              SITE_CLA);
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
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
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
