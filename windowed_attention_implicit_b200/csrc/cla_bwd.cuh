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
//   cla_bwd_dx_kernel    dx, and dW_dw / db_dw partials (FMA pipe, two CTAs per SM)
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

__host__ __device__ __forceinline__ size_t cla_dz_smem_bytes(int C) {
  return 2ull * C * C + 256ull * C + 4ull * (kClaBwdThreads / 32) * C + 64 + 1024;
}

// -------------------------------------------------------------- dz and dy
// grid p.grid, block kClaBwdThreads, dynamic smem cla_dz_smem_bytes(C).
__global__ void __launch_bounds__(kClaBwdThreads, 1) cla_bwd_dz_kernel(const ClaBwdParams p) {
  extern __shared__ uint8_t dz_raw[];
  uint8_t* base = dz_raw + ((1024u - (smem_u32(dz_raw) & 1023u)) & 1023u);
  const int C = p.C;
  uint8_t* sB = base;                                   // W_pw^T bf16 [N = c][K = o]
  uint8_t* sA = base + 2ull * C * C;                    // dz bf16 [M = 128 pixels][K = o]
  float* red = reinterpret_cast<float*>(sA + 256ull * C);   // [warps][C]
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + (kClaBwdThreads / 32) * C);
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
  const int groups = (C + 63) / 64;
  float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};  // db_pw, per group
  bool ok = true;
  int phase = 0;
  for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x) {
    int b, i0, j0;
    cla_tile(p, t, b, i0, j0);
    // ---- element-wise: lanes along channel pairs, warps over pixels
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (g >= groups) break;
      const int c = g * 64 + 2 * lane;
      if (c >= C) continue;
      for (int r = warp; r < 128; r += kClaBwdThreads / 32) {
        const size_t off = cla_pix(p, b, i0 + (r >> 4), j0 + (r & 15)) * C + c;
        const float2 dg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p.dout_g + off));
        const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p.out + off));
        const float2 gt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p.gate + off));
        const float z0 = dg.x * o.x * gt.x * (1.f - gt.x), z1 = dg.y * o.y * gt.y * (1.f - gt.y);
        *reinterpret_cast<uint32_t*>(p.dout + off) = pack_bf16x2(dg.x * gt.x, dg.y * gt.y);
        const uint32_t zb = pack_bf16x2(z0, z1);
        *reinterpret_cast<uint32_t*>(p.dz + off) = zb;
        *reinterpret_cast<uint32_t*>(sA + cla_kmajor_offset(r, c, C)) = zb;
        acc[g][0] += z0;
        acc[g][1] += z1;
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
  // db_pw partial of this CTA: the warps' sums, added in warp order
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int c = g * 64 + 2 * lane;
    if (g < groups && c < C) {
      red[warp * C + c] = acc[g][0];
      red[warp * C + c + 1] = acc[g][1];
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < kClaBwdThreads / 32; ++w) s += red[w * C + c];
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
// weights of the depth-wise convolution [9][C] and its bias [C].
__host__ __device__ __forceinline__ size_t cla_dwpw_smem_bytes(int C) {
  return 256ull * 256 + 256ull * C + 40ull * C + 64 + 1024;
}

// grid p.grid, block kClaBwdThreads, dynamic smem cla_dwpw_smem_bytes(C).
__global__ void __launch_bounds__(kClaBwdThreads, 1) cla_bwd_dwpw_kernel(const ClaBwdParams p) {
  extern __shared__ uint8_t dw_raw[];
  uint8_t* base = dw_raw + ((1024u - (smem_u32(dw_raw) & 1023u)) & 1023u);
  const int C = p.C, octets = C / 8;
  uint8_t* sA = base;                          // dz^T, 64 KB
  uint8_t* sB = base + 256 * 256;              // y^T, 256 C bytes
  float* sWdw = reinterpret_cast<float*>(sB + 256ull * C);   // [tap][C]
  float* sBdw = sWdw + 9 * C;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sBdw + C);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
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
  bool ok = true;
  int phase = 0, n_done = 0;
  for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x, ++n_done) {
    int b, i0, j0;
    cla_tile(p, t, b, i0, j0);
    // items: (channel octet k, pixel r), consecutive threads on consecutive
    // pixels, so each 16-byte shared-memory store lands in its own banks
    for (int it = threadIdx.x; it < octets * 128; it += blockDim.x) {
      const int k = it >> 7, r = it & 127;
      const int i = i0 + (r >> 4), j = j0 + (r & 15);
      // dz^T: 8 output channels of pixel r
      const uint4 zv = *reinterpret_cast<const uint4*>(p.dz + cla_pix(p, b, i, j) * C + 8 * k);
      *reinterpret_cast<uint4*>(sA + cla_mnmajor_offset(r, 8 * k)) = zv;
      // y^T: the depth-wise convolution of x, 8 input channels of pixel r
      float a[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = sBdw[8 * k + e];
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int ii = i + u - 1;
        if (ii < 0 || ii >= p.H) continue;
#pragma unroll
        for (int v = 0; v < 3; ++v) {
          const int jj = j + v - 1;
          if (jj < 0 || jj >= p.W) continue;
          const uint4 xv = *reinterpret_cast<const uint4*>(p.x + cla_pix(p, b, ii, jj) * C + 8 * k);
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
          const float* w = sWdw + (u * 3 + v) * C + 8 * k;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[e]));
            a[2 * e] = fmaf(w[2 * e], xf.x, a[2 * e]);
            a[2 * e + 1] = fmaf(w[2 * e + 1], xf.y, a[2 * e + 1]);
          }
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
  }
  // the CTA's partial dW_pw: rows o from TMEM lanes, C columns each
  if (ok && warp < 8) {
    const int q = warp & 3, half = warp >> 2;
    const int o = half * 128 + q * 32 + lane;
    const uint32_t taddr = tmem + half * 256 + (static_cast<uint32_t>(q * 32) << 16);
    if (half == 0 || two) {
      float* dst = p.part_dwpw + (static_cast<size_t>(blockIdx.x) * C + o) * C;
      for (int c0 = 0; c0 < C; c0 += 32) {
        uint32_t v[32];
        tmem_ld_x32(taddr + c0, v);
        tmem_wait_ld();
        reg_fence_x32(v);
        if (o < C && n_done > 0) {
          float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        } else if (o < C) {
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
// grid p.grid_dx, block kClaDxThreads, static smem.  Lanes along channel
// pairs, warps over the tile's pixels; one 64-channel group at a time over
// all of the CTA's tiles, so each thread keeps 20 partial sums.
__global__ void __launch_bounds__(kClaDxThreads) cla_bwd_dx_kernel(const ClaBwdParams p) {
  __shared__ float red[kClaDxThreads / 32][10][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.C;
  for (int g = 0; g * 64 < C; ++g) {
    const int c = g * 64 + 2 * lane;
    const bool act = c < C;
    float w0[9], w1[9], aw0[9], aw1[9], ab0 = 0.f, ab1 = 0.f;
#pragma unroll
    for (int tp = 0; tp < 9; ++tp) {
      w0[tp] = act ? p.w_dw[c * 9 + tp] : 0.f;
      w1[tp] = act ? p.w_dw[(c + 1) * 9 + tp] : 0.f;
      aw0[tp] = aw1[tp] = 0.f;
    }
    for (int t = blockIdx.x; act && t < p.n_tiles; t += gridDim.x) {
      int b, i0, j0;
      cla_tile(p, t, b, i0, j0);
      for (int r = warp; r < 128; r += kClaDxThreads / 32) {
        const int i = i0 + (r >> 4), j = j0 + (r & 15);
        const float2 d = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162*>(p.dy + cla_pix(p, b, i, j) * C + c));
        ab0 += d.x;
        ab1 += d.y;
        float dx0 = 0.f, dx1 = 0.f;
#pragma unroll
        for (int u = 0; u < 3; ++u)
#pragma unroll
          for (int v = 0; v < 3; ++v) {
            const int tp = u * 3 + v;
            // dW_dw: dy here times x at (i + u - 1, j + v - 1)
            const int xi = i + u - 1, xj = j + v - 1;
            if (xi >= 0 && xi < p.H && xj >= 0 && xj < p.W) {
              const float2 xf = __bfloat1622float2(
                  *reinterpret_cast<const __nv_bfloat162*>(p.x + cla_pix(p, b, xi, xj) * C + c));
              aw0[tp] = fmaf(d.x, xf.x, aw0[tp]);
              aw1[tp] = fmaf(d.y, xf.y, aw1[tp]);
            }
            // dx: W_dw tap (u, v) times dy at (i - u + 1, j - v + 1)
            const int yi = i - u + 1, yj = j - v + 1;
            if (yi >= 0 && yi < p.H && yj >= 0 && yj < p.W) {
              const float2 df = __bfloat1622float2(
                  *reinterpret_cast<const __nv_bfloat162*>(p.dy + cla_pix(p, b, yi, yj) * C + c));
              dx0 = fmaf(w0[tp], df.x, dx0);
              dx1 = fmaf(w1[tp], df.y, dx1);
            }
          }
        *reinterpret_cast<uint32_t*>(p.dx + cla_pix(p, b, i, j) * C + c) = pack_bf16x2(dx0, dx1);
      }
    }
    // this group's partials: the warps' sums, added in warp order
#pragma unroll
    for (int tp = 0; tp < 9; ++tp) {
      red[warp][tp][2 * lane] = aw0[tp];
      red[warp][tp][2 * lane + 1] = aw1[tp];
    }
    red[warp][9][2 * lane] = ab0;
    red[warp][9][2 * lane + 1] = ab1;
    __syncthreads();
    for (int e = threadIdx.x; e < 10 * 64; e += blockDim.x) {
      const int tp = e / 64, cc = e % 64;
      if (g * 64 + cc >= C) continue;
      float s = 0.f;
      for (int w = 0; w < kClaDxThreads / 32; ++w) s += red[w][tp][cc];
      p.part_dw[(static_cast<size_t>(blockIdx.x) * 10 + tp) * C + g * 64 + cc] = s;
    }
    __syncthreads();
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
