// cla.cuh -- convolutional local attention gate (CLA) on tcgen05 tensor cores.
//
// "Rank-Factorized Implicit Neural Bias" pages: English summary, Technical
// Summary §2.B (a lightweight path of a depth-wise convolution, a point-wise
// convolution and a sigmoid produces a gating map that modulates the
// self-attention output); German summary, Methodik §B (O' = O * G); Chinese
// summary §2.B (the depth-wise convolution is 3x3, the point-wise one 1x1).
//
//   y = b_dw + DW3x3(x)      (per channel, zero padding 1, cross-correlation)
//   z = b_pw + y W_pw^T      (1x1 convolution = a C x C matrix per pixel)
//   G = 1 / (1 + exp(-z))
//
// x and G are bf16 [B][H][W][C]; the weights are fp32 (W_pw [C_out][C_in]).
// cla_gate_kernel is persistent (one CTA per SM) over tiles of 8 x 16
// pixels: eight warps compute y in fp32 from x (lanes along channels, so
// every tap is one coalesced 128-byte load per warp) and write it as bf16
// into shared memory in the canonical no-swizzle K-major core-matrix layout;
// one elected lane issues the point-wise convolution as C/16 tcgen05.mma
// steps (M = 128 pixels, N = C, K = C) into tensor memory, W_pw having been
// rounded to bf16 into shared memory once per CTA; four warps read the
// accumulator back, add b_pw, apply the sigmoid and store G.
#pragma once

#include "geom.cuh"
#include "ptx.cuh"

namespace rib {

constexpr int kClaThreads = 256;
constexpr int kClaMaxC = 256;           // N of one MMA
constexpr uint32_t kClaTmemCols = 256;

struct ClaParams {
  const __nv_bfloat16* x;
  const float* w_dw;   // [C][3][3]
  const float* b_dw;   // [C]
  const float* w_pw;   // [C][C]
  const float* b_pw;   // [C]
  __nv_bfloat16* gate;
  int B, H, W, C, tiles_x, tiles_per_img, n_tiles;
  uint64_t wait_limit_ns;
};

// Byte offset of element (row r, k) in a K-major no-swizzle operand with
// core matrices of 8 rows x 16 bytes: K-adjacent core matrices 128 bytes
// apart (LBO), row-adjacent ones 16 C bytes apart (SBO).
__device__ __forceinline__ uint32_t cla_kmajor_offset(int r, int k, int C) {
  return static_cast<uint32_t>((k >> 3) * 128 + (r >> 3) * 16 * C + (r & 7) * 16 + (k & 7) * 2);
}

// W_pw (2 C^2 bytes) + the y tile (256 C bytes, padded to 2 C^2 where that
// fits, so that no reading of the operand strides can leave the allocation)
// + barriers + alignment slack.
__host__ __device__ __forceinline__ size_t cla_a_bytes(int C) {
  const size_t a = 128ull * C * 2, pad = 2ull * C * C;
  return (2ull * C * C + pad + 1280 <= 227ull * 1024 && pad > a) ? pad : a;
}
__host__ __device__ __forceinline__ size_t cla_smem_bytes(int C) {
  return static_cast<size_t>(C) * C * 2 + cla_a_bytes(C) + 256 + 1024;
}

// grid min(n_tiles, #SMs), block kClaThreads, dynamic smem cla_smem_bytes(C).
__global__ void __launch_bounds__(kClaThreads, 1) cla_gate_kernel(const ClaParams p) {
  extern __shared__ uint8_t cla_raw[];
  uint8_t* base = cla_raw + ((1024u - (smem_u32(cla_raw) & 1023u)) & 1023u);
  const int C = p.C;
  uint8_t* sB = base;                                  // W_pw bf16, [N=C][K=C]
  uint8_t* sA = base + static_cast<size_t>(C) * C * 2;  // y bf16, [M=128][K=C]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sA + cla_a_bytes(C));
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // W_pw -> bf16 B operand (row n = output channel, k = input channel)
  for (int i = threadIdx.x; i < C * C / 2; i += blockDim.x) {
    const int n = (2 * i) / C, k = (2 * i) % C;
    const float2 w = *reinterpret_cast<const float2*>(p.w_pw + static_cast<size_t>(n) * C + k);
    *reinterpret_cast<uint32_t*>(sB + cla_kmajor_offset(n, k, C)) = pack_bf16x2(w.x, w.y);
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tbase, kClaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint32_t idesc = make_idesc_bf16(128, C, false, false);
  const uint64_t adesc = make_sdesc(smem_u32(sA), 128, 16 * C, kLayoutNone);
  const uint64_t bdesc = make_sdesc(smem_u32(sB), 128, 16 * C, kLayoutNone);
  const int groups = (C + 63) / 64;   // 64-channel groups: 32 lanes x 2 channels
  bool ok = true;
  int phase = 0;
  for (int t = blockIdx.x; ok && t < p.n_tiles; t += gridDim.x, phase ^= 1) {
    const int b = t / p.tiles_per_img, tt = t % p.tiles_per_img;
    const int i0 = (tt / p.tiles_x) * 8, j0 = (tt % p.tiles_x) * 16;
    // ---- depth-wise 3x3: per 64-channel group (lane = channel pair), the
    // warps take every 8th pixel of the tile
    for (int g = 0; g < groups; ++g) {
      const int c = g * 64 + 2 * lane;
      if (c >= C) break;   // last group of C = 96: lanes 0-15
      float w0[9], w1[9];
#pragma unroll
      for (int tp = 0; tp < 9; ++tp) {
        w0[tp] = p.w_dw[c * 9 + tp];
        w1[tp] = p.w_dw[(c + 1) * 9 + tp];
      }
      const float bias0 = p.b_dw[c], bias1 = p.b_dw[c + 1];
      for (int r = warp; r < 128; r += kClaThreads / 32) {
        const int i = i0 + (r >> 4), j = j0 + (r & 15);
        float a0 = bias0, a1 = bias1;
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          const int ii = i + u - 1;
          if (ii < 0 || ii >= p.H) continue;
#pragma unroll
          for (int v = 0; v < 3; ++v) {
            const int jj = j + v - 1;
            if (jj < 0 || jj >= p.W) continue;
            const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                p.x + ((static_cast<size_t>(b) * p.H + ii) * p.W + jj) * C + c));
            a0 = fmaf(w0[u * 3 + v], xf.x, a0);
            a1 = fmaf(w1[u * 3 + v], xf.y, a1);
          }
        }
        *reinterpret_cast<uint32_t*>(sA + cla_kmajor_offset(r, c, C)) = pack_bf16x2(a0, a1);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- point-wise 1x1: D[128 x C] = y W_pw^T, K-steps of 16 channels
    if (warp == 0) {
#pragma unroll 1
      for (int ks = 0; ks < C / 16; ++ks)
        umma_ss_elect(tmem, adesc + ks * 16, bdesc + ks * 16, idesc, ks > 0 ? 1u : 0u);
      umma_commit_elect(bar);
    }
    // every thread waits: the accumulator is read by warps 0-3 and the A
    // tile is rewritten by everyone for the next tile
    ok = mbar_wait(bar, phase, abort_flag, p.wait_limit_ns, SITE_CLA);
    ok = __syncthreads_and(ok);
    tc_fence_after();
    // ---- epilogue: warps w and w+4 share TMEM lanes 32(w%4).. (pixels)
    if (ok) {
      const int q = warp & 3, half = warp >> 2;
      const int r = q * 32 + lane;
      const int i = i0 + (r >> 4), j = j0 + (r & 15);
      __nv_bfloat16* dst = p.gate + ((static_cast<size_t>(b) * p.H + i) * p.W + j) * C;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = half * 32; c0 < C; c0 += 64) {
        uint32_t z[32];
        tmem_ld_x32(taddr + c0, z);
        tmem_wait_ld();
        reg_fence_x32(z);
        uint32_t gk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float z0 = __uint_as_float(z[2 * e]) + p.b_pw[c0 + 2 * e];
          const float z1 = __uint_as_float(z[2 * e + 1]) + p.b_pw[c0 + 2 * e + 1];
          gk[e] = pack_bf16x2(1.f / (1.f + __expf(-z0)), 1.f / (1.f + __expf(-z1)));
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_uint4(gk[4 * e], gk[4 * e + 1], gk[4 * e + 2], gk[4 * e + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();   // accumulator drained before the next tile's MMAs
    tc_fence_after();
  }
  if (!ok) {
    // a wait gave up: let the MMAs issued for this tile finish before the
    // tensor memory is released
    // (the loop's increment already flipped `phase` past the failed wait)
    volatile int no_abort = 0;
    mbar_wait(bar, phase ^ 1, &no_abort, 200ull * 1000ull * 1000ull, SITE_CLA);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kClaTmemCols);
  }
}

}  // namespace rib
