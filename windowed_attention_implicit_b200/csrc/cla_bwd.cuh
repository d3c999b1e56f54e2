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
//   cla_bwd_dwpw_kernel  dW_pw partials = sum over the CTA's tiles of
//                        dz^T y, y recomputed from x; both operands MN-major
//                        in shared memory, the C x C partial in TMEM
//   cla_bwd_dx_kernel    dx, and dW_dw / db_dw partials (FMA pipe, two CTAs per SM,
//                        x and dy halos staged by TMA)
//   cla_bwd_reduce_kernel fixed-order sums of the partials
#pragma once

#include "cla.cuh"

namespace rib {

constexpr int kClaBwdThreads = 512;   // dz and dW_pw kernels
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
// kDzBatch pixels' loads in flight at once.
constexpr int kDzBatch = 2;
__host__ __device__ __forceinline__ size_t cla_dz_smem_bytes(int C) {
  return 2ull * C * C + 256ull * C + 4ull * 8 * kClaBwdThreads + 64 + 1024;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const __nv_bfloat16* ptr) {
  return __ldg(reinterpret_cast<const uint4*>(ptr));
}

// -------------------------------------------------------------- dz and dy
// grid p.grid, block kClaBwdThreads, dynamic smem cla_dz_smem_bytes(C).
__global__ void __launch_bounds__(kClaBwdThreads, 1) cla_bwd_dz_kernel(const ClaBwdParams p) {
  extern __shared__ uint8_t dz_raw[];
  uint8_t* base = dz_raw + ((1024u - (smem_u32(dz_raw) & 1023u)) & 1023u);
  const int C = p.C;
  uint8_t* sB = base;                                   // W_pw^T bf16 [N = c][K = o]
  uint8_t* sA = base + 2ull * C * C;                    // dz bf16 [M = 128 pixels][K = o]
  float* red = reinterpret_cast<float*>(sA + 256ull * C);   // [slot][C] db_pw partials
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 8 * kClaBwdThreads);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
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
    tmem_alloc(tbase, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint32_t idesc = make_idesc_bf16(128, C, false, false);
  const uint64_t adesc = make_sdesc(smem_u32(sA), 128, 16 * C, kLayoutNone);
  const uint64_t bdesc = make_sdesc(smem_u32(sB), 128, 16 * C, kLayoutNone);
  // element-wise part: thread = (pixel slot sl, channel octet k); slots
  // take pixels sl, sl + slots, ...; consecutive threads read consecutive
  // 16-byte octets of one pixel
  const int octets = C / 8, slots = kClaBwdThreads / octets;
  const int sl = threadIdx.x / octets, k = threadIdx.x % octets;
  const bool act = sl < slots;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // db_pw, channels 8k..8k+7
  bool ok = true;
  int phase = 0;
  for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x) {
    int b, i0, j0;
    cla_tile(p, t, b, i0, j0);
    for (int r0 = sl; act && r0 < 128; r0 += kDzBatch * slots) {
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
    __syncthreads();
    tc_fence_after();
    // ---- dy = dz W_pw  (M = 128 pixels, N = C, K = C)
    if (warp == 0) {
      for (int ks = 0; ks < C / 16; ++ks)
        umma_ss_elect(tmem, adesc + ks * 16, bdesc + ks * 16, idesc, ks > 0 ? 1u : 0u);
      umma_commit_elect(bar);
    }
    ok = mbar_wait(bar, phase, abort_flag, p.wait_limit_ns, SITE_CLA);
    phase ^= 1;
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (ok) {
      // warp w reads TMEM lanes 32 (w % 4).. (pixels), columns 32 (w / 4) + 32 k (warps / 4)
      const int q = warp & 3, slot = warp >> 2;
      const int r = q * 32 + lane;
      __nv_bfloat16* dst = p.dy + cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15)) * C;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = 32 * slot; c0 < C; c0 += 32 * (kClaBwdThreads / 128)) {
        uint32_t v[32];
        tmem_ld_x32(taddr + c0, v);
        tmem_wait_ld();
        reg_fence_x32(v);
        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
        if (!rib_guard(cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15)) * C + c0 + 31, cla_elems(p),
                       G_CLA_OUT))
          continue;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                             pack_bf16x2(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                             pack_bf16x2(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                             pack_bf16x2(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
      }
    }
    tc_fence_before();
    __syncthreads();   // accumulator read before the next tile's MMAs
    tc_fence_after();
  }
  if (!ok) {
    volatile int no_abort = 0;
    mbar_wait(bar, phase ^ 1, &no_abort, 200ull * 1000ull * 1000ull, SITE_CLA);
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
    tmem_dealloc(tmem, 256);
  }
}

// -------------------------------------------------------------- dW_pw
// Byte offset of element (k = pixel r, mn = channel) in an MN-major
// no-swizzle operand of K = 128 pixels: core matrices of 8 pixels x 16 bytes
// (8 channels), K-adjacent ones 128 bytes apart (LBO), MN-adjacent ones
// 2048 bytes apart (SBO).
__device__ __forceinline__ uint32_t cla_mnmajor_offset(int r, int mn) {
  return static_cast<uint32_t>((mn >> 3) * 2048 + (r >> 3) * 128 + (r & 7) * 16 + (mn & 7) * 2);
}

// A: dz^T [M = 256 output channels, padded][K = 128 pixels]; B: y^T [N = C][K];
// the tile's x halo (10 x 18 pixels, one TMA box per 64 channels); weights
// of the depth-wise convolution [9][C] and its bias [C].
constexpr uint32_t kDwpwHaloChunk = (kClaHaloBytes + 1023u) & ~1023u;
__host__ __device__ __forceinline__ size_t cla_dwpw_smem_bytes(int C) {
  return 256ull * 256 + 256ull * C + kDwpwHaloChunk * ((C + 63) / 64) + 40ull * C + 64 + 1024;
}

// grid p.grid, block kClaBwdThreads, dynamic smem cla_dwpw_smem_bytes(C).
// tm_x: x [B][H][W][C] as a 4D map with boxes of 64 channels x 18 x 10.
__global__ void __launch_bounds__(kClaBwdThreads, 1)
    cla_bwd_dwpw_kernel(const __grid_constant__ CUtensorMap tm_x, const ClaBwdParams p) {
  extern __shared__ uint8_t dw_raw[];
  uint8_t* base = dw_raw + ((1024u - (smem_u32(dw_raw) & 1023u)) & 1023u);
  const int C = p.C, octets = C / 8;
  uint8_t* sA = base;                          // dz^T, 64 KB
  uint8_t* sB = base + 256 * 256;              // y^T, 256 C bytes
  const int chunks = (C + 63) / 64;
  uint8_t* sH = sB + 256ull * C;               // halo [chunk][10 rows][18 cols][64 ch]
  float* sWdw = reinterpret_cast<float*>(sH + static_cast<size_t>(kDwpwHaloChunk) * chunks);
  float* sBdw = sWdw + 9 * C;                  // ([tap][C] weights before it)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sBdw + C);
  uint64_t* halo_bar = bar + 1;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 3);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init(halo_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // thread 0 loads the halo of each of the CTA's tiles; halos issued / waited for
  int halo_issued = 0, halo_seen = 0;
  auto load_halo = [&](int t) {
    int b, i0, j0;
    cla_tile(p, t, b, i0, j0);
    mbar_arrive_expect_tx(halo_bar, kClaHaloBytes * chunks);
    for (int g = 0; g < chunks; ++g)
      tma_load_4d(sH + g * kDwpwHaloChunk, &tm_x, halo_bar, 64 * g, j0 - 1, i0 - 1, b);
    ++halo_issued;
  };
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    sBdw[i] = p.b_dw[i];
#pragma unroll
    for (int tp = 0; tp < 9; ++tp) sWdw[tp * C + i] = p.w_dw[i * 9 + tp];
  }
  // rows C..255 of dz^T are padding: zero them once (they only feed
  // accumulator rows that are never read, but stay finite)
  for (int i = threadIdx.x * 16; i < 256 * 256; i += blockDim.x * 16)
    *reinterpret_cast<uint4*>(sA + i) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint32_t idesc = make_idesc_bf16(128, C, true, true);
  const uint64_t adesc = make_sdesc(smem_u32(sA), 128, 2048, kLayoutNone);
  const uint64_t bdesc = make_sdesc(smem_u32(sB), 128, 2048, kLayoutNone);
  const bool two = C > 128;
  // (after the barrier initialisation above is visible to the async proxy)
  if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < p.n_tiles) load_halo(blockIdx.x);
  bool ok = true;
  int phase = 0, n_done = 0;
  for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x, ++n_done) {
    int b, i0, j0;
    cla_tile(p, t, b, i0, j0);
    // items: (pixel r, channel octet k = 8 ch + ko); a warp takes 4
    // neighbouring pixels x 8 octets of one 64-channel chunk, so its global
    // reads are 128-byte runs and its halo reads 512 contiguous bytes
    const int n_items = chunks * 1024;
    // dz^T: 8 output channels of pixel r
#pragma unroll 2
    for (int it = threadIdx.x; it < n_items; it += blockDim.x) {
      const int ko = it & 7, q = it >> 5, ch = q % chunks, k = ch * 8 + ko;
      const int r = (q / chunks) * 4 + ((it >> 3) & 3);
      if (k >= octets) continue;
      const size_t zoff = cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15)) * C + 8 * k;
      const uint4 zv = rib_guard(zoff + 7, cla_elems(p), G_CLA_IN) ? ldg_nc_v4(p.dz + zoff)
                                                                   : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sA + cla_mnmajor_offset(r, 8 * k)) = zv;
    }
    ok = mbar_wait(halo_bar, halo_seen & 1, abort_flag, p.wait_limit_ns, SITE_CLA);
    ++halo_seen;
    if (!__syncthreads_and(ok)) {
      ok = false;
      break;
    }
    // y^T: the depth-wise convolution of x from the halo (zero outside the
    // map: the TMA fills out-of-range pixels with zeros)
#pragma unroll 2
    for (int it = threadIdx.x; it < n_items; it += blockDim.x) {
      const int ko = it & 7, q = it >> 5, ch = q % chunks, k = ch * 8 + ko;
      const int r = (q / chunks) * 4 + ((it >> 3) & 3);
      if (k >= octets) continue;
      const int i = r >> 4, j = r & 15;   // tile-local; halo row i + u, column j + v
      const uint8_t* h = sH + ch * kDwpwHaloChunk + ko * 16;
      float a[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = sBdw[8 * k + e];
#pragma unroll
      for (int u = 0; u < 3; ++u)
#pragma unroll
        for (int v = 0; v < 3; ++v) {
          const uint4 xv = *reinterpret_cast<const uint4*>(h + ((i + u) * 18 + (j + v)) * 128);
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
          const float* w = sWdw + (u * 3 + v) * C + 8 * k;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[e]));
            a[2 * e] = fmaf(w[2 * e], xf.x, a[2 * e]);
            a[2 * e + 1] = fmaf(w[2 * e + 1], xf.y, a[2 * e + 1]);
          }
        }
      *reinterpret_cast<uint4*>(sB + cla_mnmajor_offset(r, 8 * k)) =
          make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                     pack_bf16x2(a[6], a[7]));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the halo is read: fetch the next tile's while this one's MMAs run
    if (threadIdx.x == 0 && t + static_cast<int>(gridDim.x) < p.n_tiles)
      load_halo(t + gridDim.x);
    // D0 (+)= dz^T[o 0..127] y, D1 (+)= dz^T[o 128..255] y: 8 K-steps of 16 pixels
    if (warp == 0) {
      const uint32_t acc = n_done > 0 ? 1u : 0u;
      for (int ks = 0; ks < 8; ++ks) {
        umma_ss_elect(tmem, adesc + ks * 16, bdesc + ks * 16, idesc, (acc | ks) ? 1u : 0u);
        if (two)
          umma_ss_elect(tmem + 256, adesc + (16 * 2048 >> 4) + ks * 16, bdesc + ks * 16, idesc,
                        (acc | ks) ? 1u : 0u);
      }
      umma_commit_elect(bar);
    }
    // the operands are rewritten for the next tile once the MMAs are done
    ok = mbar_wait(bar, phase, abort_flag, p.wait_limit_ns, SITE_CLA);
    phase ^= 1;
    ok = __syncthreads_and(ok);
    tc_fence_after();
  }
  if (!ok) {
    volatile int no_abort = 0;
    mbar_wait(bar, phase ^ 1, &no_abort, 200ull * 1000ull * 1000ull, SITE_CLA);
    // a halo still in flight lands before the CTA exits
    if (threadIdx.x == 0 && halo_issued > halo_seen)
      mbar_wait(halo_bar, (halo_issued - 1) & 1, &no_abort, 200ull * 1000ull * 1000ull, SITE_CLA);
  }
  // the CTA's partial dW_pw: rows o from TMEM lanes, C columns each
  if (ok && warp < 8) {
    const int q = warp & 3, half = warp >> 2;
    const int o = half * 128 + q * 32 + lane;
    const uint32_t taddr = tmem + half * 256 + (static_cast<uint32_t>(q * 32) << 16);
    if (half == 0 || two) {
      float* dst = p.part_dwpw + (static_cast<size_t>(blockIdx.x) * C + o) * C;
      const bool in = o >= C || rib_guard((static_cast<size_t>(blockIdx.x) * C + o) * C + C - 1,
                                          static_cast<size_t>(p.grid) * C * C, G_CLA_PART);
      for (int c0 = 0; c0 < C; c0 += 32) {   // every lane: the TMEM loads are collective
        uint32_t v[32];
        tmem_ld_x32(taddr + c0, v);
        tmem_wait_ld();
        reg_fence_x32(v);
        if (o < C && n_done > 0 && in) {
          float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        } else if (o < C && in) {
          for (int e = 0; e < 32; ++e) dst[c0 + e] = 0.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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
__host__ __device__ __forceinline__ size_t cla_dx_smem_bytes() {
  return 4ull * kDwpwHaloChunk + 64 + 1024;
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
  uint64_t* full = reinterpret_cast<uint64_t*>(base + 4 * kDwpwHaloChunk);   // [2] stages
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
  auto hx = [&](int st) { return base + st * kDwpwHaloChunk; };
  auto hdy = [&](int st) { return base + (2 + st) * kDwpwHaloChunk; };
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
// Fixed-order sums over the CTAs' partials; one thread per gradient element
// (C*C of dW_pw, then C of db_pw, 9C of dW_dw, C of db_dw).
__global__ void __launch_bounds__(256) cla_bwd_reduce_kernel(const ClaBwdParams p) {
  const int C = p.C;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int n_pw = C * C;
  if (idx >= n_pw + 11 * C) return;
  float s = 0.f;
  if (idx < n_pw) {
    for (int k = 0; k < p.grid; ++k) s += p.part_dwpw[static_cast<size_t>(k) * n_pw + idx];
    p.dw_pw[idx] = s;
  } else if (idx < n_pw + C) {
    const int o = idx - n_pw;
    for (int k = 0; k < p.grid; ++k) s += p.part_dbpw[static_cast<size_t>(k) * C + o];
    p.db_pw[o] = s;
  } else {
    const int e = idx - n_pw - C;           // 0 .. 10C-1: tap-major [10][C]
    const int tp = e / C, c = e % C;
    for (int k = 0; k < p.grid_dx; ++k) s += p.part_dw[(static_cast<size_t>(k) * 10 + tp) * C + c];
    if (tp < 9) p.dw_dw[c * 9 + tp] = s;
    else p.db_dw[c] = s;
  }
}

}  // namespace rib
