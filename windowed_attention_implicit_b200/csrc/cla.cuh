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
// pixels and warp-specialised, 448 threads:
//   warp 0       TMA: the tile's 10 x 18-pixel halo, 64 channels at a time,
//                into a 2-stage ring; the zero padding of the convolution is
//                the TMA's out-of-bounds fill
//   warp 1       TMEM allocator; issues the point-wise convolution as C/16
//                tcgen05.mma steps (M = 128 pixels, N = C, K = C), W_pw
//                having been rounded to bf16 into shared memory once per CTA
//   warps 2-9    depth-wise 3x3 in fp32 from the halo (lane = channel quad
//                of one of two neighbouring pixels),
//                y written as bf16 into one of two A tiles in the canonical
//                no-swizzle K-major core-matrix layout
//   warps 10-17  epilogue: accumulator (one of two in tensor memory) + b_pw,
//                sigmoid(z) = 0.5 + 0.5 tanh(z / 2), G stored as bf16; two
//                warps per TMEM lane quarter, each taking half the channels
// so the halo copy, the depth-wise pass, the MMAs and the epilogue of
// successive tiles overlap.
#pragma once

#include "geom.cuh"
#include "ptx.cuh"

namespace rib {

constexpr int kClaThreads = 576;
constexpr int kClaEpiWarps = 8;
constexpr int kClaDwWarps = 8;
constexpr int kClaMaxC = 256;           // N of one MMA
constexpr uint32_t kClaTmemCols = 512;  // two accumulators of up to 256 columns
constexpr uint32_t kClaHaloBytes = 10u * 18u * 64u * 2u;  // one 64-channel halo box

struct ClaParams {
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
__host__ __device__ __forceinline__ uint32_t cla_kmajor_offset(int r, int k, int C) {
  return static_cast<uint32_t>((k >> 3) * 128 + (r >> 3) * 16 * C + (r & 7) * 16 + (k & 7) * 2);
}

struct ClaLayout {
  uint32_t w, a0, a1, halo0, halo1, bias, bars, total;
};

// W_pw (2 C^2 bytes) | two y tiles (256 C bytes each) | two halo stages |
// barriers; offsets from a 1024-aligned base.
__host__ __device__ __forceinline__ ClaLayout cla_layout(int C) {
  ClaLayout L;
  L.w = 0;
  L.a0 = 2u * C * C;
  L.a1 = L.a0 + 256u * C;
  L.halo0 = (L.a1 + 256u * C + 1023u) & ~1023u;
  L.halo1 = L.halo0 + ((kClaHaloBytes + 1023u) & ~1023u);
  L.bias = L.halo1 + ((kClaHaloBytes + 1023u) & ~1023u);
  L.bars = L.bias + 4u * C + 40u * C;   // b_pw, then w_dw as [9][C] and b_dw
  L.total = L.bars + 256u;
  return L;
}

__host__ __device__ __forceinline__ size_t cla_smem_bytes(int C) {
  return static_cast<size_t>(cla_layout(C).total) + 1024;
}

struct ClaBars {
  uint64_t halo_full[2], halo_empty[2], a_full[2], a_free[2], d_full[2], d_free[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// grid min(n_tiles, #SMs), block kClaThreads, dynamic smem cla_smem_bytes(C).
__global__ void __launch_bounds__(kClaThreads, 1)
    cla_gate_kernel(const __grid_constant__ CUtensorMap tm_x, const ClaParams p) {
  extern __shared__ uint8_t cla_raw[];
  uint8_t* base = cla_raw + ((1024u - (smem_u32(cla_raw) & 1023u)) & 1023u);
  const int C = p.C;
  const ClaLayout L = cla_layout(C);
  uint8_t* sW = base + L.w;
  // buffer s of the y tiles / halo stages (selects, not arrays: no local memory)
  auto sA = [&](int s) { return base + (s ? L.a1 : L.a0); };
  auto sH = [&](int s) { return base + (s ? L.halo1 : L.halo0); };
  ClaBars& bb = *reinterpret_cast<ClaBars*>(base + L.bars);
  volatile int* ab = &bb.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;
  const int chunks = (C + 63) / 64;
  const int my_tiles = blockIdx.x < p.n_tiles ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bb.halo_full[i], 1);
      mbar_init(&bb.halo_empty[i], kClaDwWarps);
      mbar_init(&bb.a_full[i], kClaDwWarps);
      mbar_init(&bb.a_free[i], 1);
      mbar_init(&bb.d_full[i], 1);
      mbar_init(&bb.d_free[i], kClaEpiWarps);
    }
    mbar_init(&bb.drain, 1);
    bb.abort_flag = 0;
    fence_mbarrier_init();
  }
  // W_pw -> bf16 B operand (row n = output channel, k = input channel).
  // Pair i is W_pw[2i], W_pw[2i + 1]; eight pairs' loads are issued before
  // any store, so the fill costs a few memory latencies, not one per pair.
  const int n_pairs = C * C / 2;
  for (int i0 = threadIdx.x; i0 < n_pairs; i0 += 8 * blockDim.x) {
    float2 w[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = i0 + e * static_cast<int>(blockDim.x);
      w[e] = i < n_pairs ? __ldg(reinterpret_cast<const float2*>(p.w_pw) + i)
                         : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = i0 + e * static_cast<int>(blockDim.x);
      if (i >= n_pairs) break;
      const int n = (2 * i) / C, k = (2 * i) % C;
      *reinterpret_cast<uint32_t*>(sW + cla_kmajor_offset(n, k, C)) = pack_bf16x2(w[e].x, w[e].y);
    }
  }
  float* sBias = reinterpret_cast<float*>(base + L.bias);
  float* sWdw = sBias + C;       // [tap][channel]: a warp reads 64 consecutive channels
  float* sBdw = sWdw + 9 * C;
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    sBias[i] = p.b_pw[i];
    sBdw[i] = p.b_dw[i];
#pragma unroll
    for (int tp = 0; tp < 9; ++tp) sWdw[tp * C + i] = p.w_dw[i * 9 + tp];
  }
  fence_proxy_async_smem();
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm_x);
  if (warp == 1) {
    tmem_alloc(&bb.tmem_base, kClaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bb.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int q = 0;  // running chunk number
      bool ok = true;
      for (int n = 0; ok && n < my_tiles; ++n) {
        const int t = blockIdx.x + n * gridDim.x;
        const int b = t / p.tiles_per_img, tt = t % p.tiles_per_img;
        const int i0 = (tt / p.tiles_x) * 8, j0 = (tt % p.tiles_x) * 16;
        for (int g = 0; ok && g < chunks; ++g, ++q) {
          const int st = q & 1;
          if (q >= 2 && !(ok = mbar_wait(&bb.halo_empty[st], ((q >> 1) - 1) & 1, ab, lim, SITE_CLA)))
            break;
          mbar_arrive_expect_tx(&bb.halo_full[st], kClaHaloBytes);
          tma_load_4d(sH(st), &tm_x, &bb.halo_full[st], 64 * g, j0 - 1, i0 - 1, b);
        }
      }
      if (!ok) {  // let issued copies land before the CTA exits
        volatile int no_abort = 0;
        for (int qq = q - 1; qq >= 0 && qq >= q - 2; --qq)
          mbar_wait(&bb.halo_full[qq & 1], (qq >> 1) & 1, &no_abort, 200000000ull, SITE_CLA);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t idesc = make_idesc_bf16(128, C, false, false);
    const uint64_t bdesc = make_sdesc(smem_u32(sW), 128, 16 * C, kLayoutNone);
    bool ok = true;
    for (int n = 0; ok && n < my_tiles; ++n) {
      const int s = n & 1;
      if (!(ok = warp_wait(&bb.a_full[s], (n >> 1) & 1, ab, lim, SITE_CLA))) break;
      if (n >= 2 && !(ok = warp_wait(&bb.d_free[s], ((n >> 1) - 1) & 1, ab, lim, SITE_CLA))) break;
      tc_fence_after();
      const uint64_t adesc = make_sdesc(smem_u32(sA(s)), 128, 16 * C, kLayoutNone);
      const uint32_t d = tmem + s * 256;
      for (int ks = 0; ks < C / 16; ++ks)
        umma_ss_elect(d, adesc + ks * 16, bdesc + ks * 16, idesc, ks > 0 ? 1u : 0u);
      umma_commit_elect(&bb.a_free[s]);
      umma_commit_elect(&bb.d_full[s]);
    }
    umma_commit_elect(&bb.drain);
    volatile int no_abort = 0;
    mbar_wait(&bb.drain, 0, &no_abort, 200000000ull, SITE_CLA);
  } else if (warp < 2 + kClaDwWarps) {
    // ---------------------------------------------------------- depth-wise
    const int dw = warp - 2;
    int q = 0;
    bool ok = true;
    for (int n = 0; ok && n < my_tiles; ++n) {
      const int s = n & 1;
      // the A tile is free once the MMAs of tile n-2 have read it
      if (n >= 2 && !(ok = warp_wait(&bb.a_free[s], ((n >> 1) - 1) & 1, ab, lim, SITE_CLA))) break;
      for (int g = 0; g < chunks; ++g, ++q) {
        const int st = q & 1;
        if (!(ok = warp_wait(&bb.halo_full[st], (q >> 1) & 1, ab, lim, SITE_CLA))) break;
        // lane = (channel quad cq of the chunk, pixel parity pp): 16 lanes read
        // one pixel's 128 bytes, the warp two neighbouring pixels at a time
        const int cq = lane & 15, pp = lane >> 4;
        const int c = g * 64 + 4 * cq;
        if (c < C) {
          float4 w4[9];
#pragma unroll
          for (int tp = 0; tp < 9; ++tp) w4[tp] = *reinterpret_cast<const float4*>(sWdw + tp * C + c);
          const float4 b4 = *reinterpret_cast<const float4*>(sBdw + c);
          const uint8_t* h = sH(st) + cq * 8;     // halo [10 rows][18 cols][64 ch]
#pragma unroll 2
          for (int m = 0; m < 128 / (2 * kClaDwWarps); ++m) {
            const int r = 2 * (dw + kClaDwWarps * m) + pp;
            const int i = r >> 4, j = r & 15;     // tile-local; halo row i+u, col j+v
            float a0 = b4.x, a1 = b4.y, a2 = b4.z, a3 = b4.w;
#pragma unroll
            for (int u = 0; u < 3; ++u)
#pragma unroll
              for (int v = 0; v < 3; ++v) {
                const uint2 xv =
                    *reinterpret_cast<const uint2*>(h + ((i + u) * 18 + (j + v)) * 128);
                const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv.x));
                const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv.y));
                const float4 w = w4[u * 3 + v];
                a0 = fmaf(w.x, x01.x, a0);
                a1 = fmaf(w.y, x01.y, a1);
                a2 = fmaf(w.z, x23.x, a2);
                a3 = fmaf(w.w, x23.y, a3);
              }
            *reinterpret_cast<uint2*>(sA(s) + cla_kmajor_offset(r, c, C)) =
                make_uint2(pack_bf16x2(a0, a1), pack_bf16x2(a2, a3));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bb.halo_empty[st]);
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bb.a_full[s]);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int qd = warp & 3;   // TMEM lane quarter (warps 10-17 -> 2, 3, 0, 1, 2, 3, 0, 1)
    const int half = (warp - 2 - kClaDwWarps) >> 2;
    bool ok = true;
    for (int n = 0; ok && n < my_tiles; ++n) {
      const int s = n & 1;
      if (!(ok = warp_wait(&bb.d_full[s], (n >> 1) & 1, ab, lim, SITE_CLA))) break;
      tc_fence_after();
      const int t = blockIdx.x + n * gridDim.x;
      const int b = t / p.tiles_per_img, tt = t % p.tiles_per_img;
      const int i0 = (tt / p.tiles_x) * 8, j0 = (tt % p.tiles_x) * 16;
      const int r = qd * 32 + lane;
      __nv_bfloat16* dst =
          p.gate + ((static_cast<size_t>(b) * p.H + i0 + (r >> 4)) * p.W + j0 + (r & 15)) * C;
      const uint32_t taddr = tmem + s * 256 + (static_cast<uint32_t>(qd * 32) << 16);
      for (int c0 = 32 * half; c0 < C; c0 += 64) {
        uint32_t z[32];
        tmem_ld_x32(taddr + c0, z);
        tmem_wait_ld();
        reg_fence_x32(z);
        uint32_t gk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float z0 = __uint_as_float(z[2 * e]) + sBias[c0 + 2 * e];
          const float z1 = __uint_as_float(z[2 * e + 1]) + sBias[c0 + 2 * e + 1];
          gk[e] = pack_bf16x2(fmaf(0.5f, tanh_approx(0.5f * z0), 0.5f),
                              fmaf(0.5f, tanh_approx(0.5f * z1), 0.5f));
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
        const size_t g0 = ((static_cast<size_t>(b) * p.H + i0 + (r >> 4)) * p.W + j0 + (r & 15)) *
                              C + c0;
        if (rib_guard(g0 + 31, static_cast<size_t>(p.B) * p.H * p.W * C, G_CLA_GATE)) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            d4[e] = make_uint4(gk[4 * e], gk[4 * e + 1], gk[4 * e + 2], gk[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bb.d_free[s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kClaTmemCols);
  }
}

}  // namespace rib
