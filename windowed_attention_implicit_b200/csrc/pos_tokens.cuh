// pos_tokens.cuh -- position tokens Qp, Kp of one window geometry and the
// backward of the position MLPs.
//
// "Rank-Factorized Implicit Neural Bias" (gist.science English summary,
// Technical Summary §2.A steps 1-2; German summary §A step 1): each token of
// the window gets a normalised 2D coordinate in [-1, 1], expanded by a
// Fourier feature map and fed to a lightweight MLP that outputs the low-rank
// positional query / key tokens.  Here: coordinates local to the window with
// endpoints included, features [sin(w x), cos(w x), sin(w y), cos(w y)],
// Linear -> GELU(erf) -> Linear, one MLP per side.
//
// This is small FMA-pipe work (about 0.8 GFLOP at M = 96) computed once per
// geometry and cached by the caller, so the kernels favour exactness: the
// Fourier features are evaluated in fp64 and rounded once to fp32, the MLP
// runs in fp32 with fp32 accumulation.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace rib {

struct PosParams {
  int M, N, F, hid, dout, rank;
  const float* freqs;
  const float* w1[2];
  const float* b1[2];
  const float* w2[2];
  const float* b2[2];
  float* out32[2];
  __nv_bfloat16* out16[2];
  // backward
  const float* dtok[2];  // dL/dQp, dL/dKp fp32 [heads][N][rank]
  float* partial;        // [2][n_chunks][n_params]
  int n_chunks;
  int n_params;          // hid*4F + hid + dout*hid + dout
  float* grads[2][4];    // dw1, db1, dw2, db2 per side
};

constexpr int kPosTok = 64;       // tokens per CTA (forward and backward partials)
constexpr int kMlpBwdTok = kPosTok;
constexpr int kPosThreads = 256;  // 4 threads per token

// Shared-memory layouts are token-major with rows padded by one float: a warp
// covers 32 consecutive tokens at a fixed feature (conflict-free) or 32
// consecutive features of one token (conflict-free), and weight rows are read
// with the same address across the warp (broadcast).
__host__ __device__ constexpr int pad1(int n) { return n + 1; }

// Fourier features of tokens [t0, t0 + kPosTok) into g[kPosTok][ld]
// (fp64 math, fp32 store).
__device__ __forceinline__ void fourier_tile(const PosParams& p, int t0, float* g, int ld) {
  const int F = p.F;
  for (int idx = threadIdx.x; idx < kPosTok * F; idx += blockDim.x) {
    const int t = idx % kPosTok, k = idx / kPosTok;
    const int tok = t0 + t;
    float* row = g + t * ld;
    if (tok < p.N) {
      const int i = tok / p.M, j = tok - i * p.M;
      const double den = p.M > 1 ? static_cast<double>(p.M - 1) : 1.0;
      const double y = p.M > 1 ? -1.0 + 2.0 * i / den : 0.0;
      const double x = p.M > 1 ? -1.0 + 2.0 * j / den : 0.0;
      const double w = static_cast<double>(__ldg(p.freqs + k));
      double sx, cx, sy, cy;
      sincos(w * x, &sx, &cx);
      sincos(w * y, &sy, &cy);
      row[k] = static_cast<float>(sx);
      row[F + k] = static_cast<float>(cx);
      row[2 * F + k] = static_cast<float>(sy);
      row[3 * F + k] = static_cast<float>(cy);
    } else {
      row[k] = row[F + k] = row[2 * F + k] = row[3 * F + k] = 0.f;
    }
  }
}

__device__ __forceinline__ float gelu_erf(float a) {
  return 0.5f * a * (1.f + erff(a * 0.70710678118654752f));
}

__device__ __forceinline__ float gelu_erf_grad(float a) {
  const float cdf = 0.5f * (1.f + erff(a * 0.70710678118654752f));
  const float pdf = 0.39894228040143268f * expf(-0.5f * a * a);
  return cdf + a * pdf;
}

// sum_k a[k*sa] * b[k*sb] for k < n with four independent accumulators
// combined in a fixed order (latency of one FMA chain hidden, result
// deterministic).  `ldg` reads `a` through the read-only cache.
template <bool kLdgA>
__device__ __forceinline__ float dot4(const float* a, int sa, const float* b, int sb, int n,
                                      float init) {
  float c0 = init, c1 = 0.f, c2 = 0.f, c3 = 0.f;
  int k = 0;
  for (; k + 3 < n; k += 4) {
    const float a0 = kLdgA ? __ldg(a + (k + 0) * sa) : a[(k + 0) * sa];
    const float a1 = kLdgA ? __ldg(a + (k + 1) * sa) : a[(k + 1) * sa];
    const float a2 = kLdgA ? __ldg(a + (k + 2) * sa) : a[(k + 2) * sa];
    const float a3 = kLdgA ? __ldg(a + (k + 3) * sa) : a[(k + 3) * sa];
    c0 = fmaf(a0, b[(k + 0) * sb], c0);
    c1 = fmaf(a1, b[(k + 1) * sb], c1);
    c2 = fmaf(a2, b[(k + 2) * sb], c2);
    c3 = fmaf(a3, b[(k + 3) * sb], c3);
  }
  for (; k < n; ++k) c0 = fmaf(kLdgA ? __ldg(a + k * sa) : a[k * sa], b[k * sb], c0);
  return (c0 + c1) + (c2 + c3);
}

__host__ __device__ constexpr size_t pos_fwd_smem_floats(int F, int hid) {
  return static_cast<size_t>(kPosTok) * (pad1(4 * F) + pad1(hid));
}

__host__ __device__ constexpr size_t mlp_bwd_smem_floats(int F, int hid, int dout) {
  return static_cast<size_t>(kPosTok) * (pad1(4 * F) + 2 * pad1(hid) + pad1(dout));
}

// grid (ceil(N / kPosTok), 2): blockIdx.y selects the q (0) or k (1) MLP.
__global__ void __launch_bounds__(kPosThreads) pos_tokens_kernel(PosParams p) {
  extern __shared__ float sm_pos[];
  const int side = blockIdx.y;
  const int t0 = blockIdx.x * kPosTok;
  const int din = 4 * p.F, ldg = pad1(din), ldh = pad1(p.hid);
  float* g = sm_pos;                   // [kPosTok][din+1]
  float* h = g + kPosTok * ldg;        // [kPosTok][hid+1]
  fourier_tile(p, t0, g, ldg);
  __syncthreads();
  const int t = threadIdx.x % kPosTok, q = threadIdx.x / kPosTok;  // 4 threads per token
  const int nq = blockDim.x / kPosTok;
  const float* w1 = p.w1[side];
  const float* b1 = p.b1[side];
  const float* gr = g + t * ldg;
  for (int jh = q; jh < p.hid; jh += nq) {
    // (debug build) the weight row's last element lies in W1
    if (!rib_guard(static_cast<size_t>(jh) * din + din - 1, static_cast<size_t>(p.hid) * din,
                   G_POS_W))
      continue;
    const float acc = dot4<true>(w1 + static_cast<size_t>(jh) * din, 1, gr, 1, din, __ldg(b1 + jh));
    h[t * ldh + jh] = gelu_erf(acc);
  }
  __syncthreads();
  const int tok = t0 + t;
  if (tok >= p.N) return;
  const float* w2 = p.w2[side];
  const float* b2 = p.b2[side];
  const float* hr = h + t * ldh;
  for (int o = q; o < p.dout; o += nq) {
    if (!rib_guard(static_cast<size_t>(o) * p.hid + p.hid - 1,
                   static_cast<size_t>(p.dout) * p.hid, G_POS_W))
      continue;
    const float acc = dot4<true>(w2 + static_cast<size_t>(o) * p.hid, 1, hr, 1, p.hid, __ldg(b2 + o));
    const int head = o / p.rank, r = o - head * p.rank;
    const size_t off = (static_cast<size_t>(head) * p.N + tok) * p.rank + r;
    if (!rib_guard(off, static_cast<size_t>(p.dout) * p.N, G_POS_OUT)) continue;
    p.out32[side][off] = acc;
    if (p.out16[side]) p.out16[side][off] = __float2bfloat16_rn(acc);
  }
}

// Partial sums over kPosTok tokens of the position-MLP weight gradients.
// grid (n_chunks, 2).  partial[side][chunk][:] = [dw1 | db1 | dw2 | db2].
__global__ void __launch_bounds__(kPosThreads) mlp_bwd_partial_kernel(PosParams p) {
  extern __shared__ float sm_pos[];
  const int side = blockIdx.y;
  const int chunk = blockIdx.x;
  const int t0 = chunk * kPosTok;
  // (debug build) this chunk's slice of the partials lies in the buffer
  if (!rib_guard((static_cast<size_t>(side) * p.n_chunks + chunk + 1) * p.n_params - 1,
                 2ull * p.n_chunks * p.n_params, G_MLP_PART))
    return;
  const int din = 4 * p.F, hid = p.hid, dout = p.dout;
  const int ldg = pad1(din), ldh = pad1(hid), ldo = pad1(dout);
  constexpr int T = kPosTok;
  float* g = sm_pos;             // [T][din+1]  Fourier features
  float* h = g + T * ldg;        // [T][hid+1]  GELU(a)
  float* da = h + T * ldh;       // [T][hid+1]  dL/da
  float* go = da + T * ldh;      // [T][dout+1] dL/d(out)
  fourier_tile(p, t0, g, ldg);
  for (int idx = threadIdx.x; idx < T * dout; idx += blockDim.x) {
    const int o = idx / T, t = idx - o * T;
    const int tok = t0 + t;
    const int head = o / p.rank, r = o - head * p.rank;
    const size_t gi = (static_cast<size_t>(head) * p.N + tok) * p.rank + r;
    go[t * ldo + o] = tok < p.N && rib_guard(gi, static_cast<size_t>(dout) * p.N, G_MLP_IN)
                          ? p.dtok[side][gi]
                          : 0.f;
  }
  __syncthreads();
  const float* w1 = p.w1[side];
  const float* b1 = p.b1[side];
  const float* w2 = p.w2[side];
  {
    const int t = threadIdx.x % T, q = threadIdx.x / T, nq = blockDim.x / T;
    const float* gr = g + t * ldg;
    const float* gor = go + t * ldo;
    for (int jh = q; jh < hid; jh += nq) {
      if (!rib_guard(static_cast<size_t>(jh) * din + din - 1, static_cast<size_t>(hid) * din,
                     G_POS_W) ||
          !rib_guard(static_cast<size_t>(dout - 1) * hid + jh, static_cast<size_t>(dout) * hid,
                     G_POS_W))
        continue;
      const float acc = dot4<true>(w1 + static_cast<size_t>(jh) * din, 1, gr, 1, din, __ldg(b1 + jh));
      const float dh = dot4<true>(w2 + jh, hid, gor, 1, dout, 0.f);
      h[t * ldh + jh] = gelu_erf(acc);
      da[t * ldh + jh] = dh * gelu_erf_grad(acc);  // tokens past N have go == 0
    }
  }
  __syncthreads();
  float* out = p.partial + (static_cast<size_t>(side) * p.n_chunks + chunk) * p.n_params;
  // dw1[jh][k] = sum_t da[t][jh] g[t][k]  (warp: one jh, consecutive k)
  for (int idx = threadIdx.x; idx < hid * din; idx += blockDim.x) {
    const int jh = idx / din, k = idx - jh * din;
    out[idx] = dot4<false>(da + jh, ldh, g + k, ldg, T, 0.f);
  }
  for (int jh = threadIdx.x; jh < hid; jh += blockDim.x) {
    float acc = 0.f;
    for (int t = 0; t < T; ++t) acc += da[t * ldh + jh];
    out[hid * din + jh] = acc;
  }
  float* o2 = out + hid * din + hid;
  // dw2[o][jh] = sum_t go[t][o] h[t][jh]  (warp: one o, consecutive jh)
  for (int idx = threadIdx.x; idx < dout * hid; idx += blockDim.x) {
    const int o = idx / hid, jh = idx - o * hid;
    o2[idx] = dot4<false>(go + o, ldo, h + jh, ldh, T, 0.f);
  }
  for (int o = threadIdx.x; o < dout; o += blockDim.x) {
    float acc = 0.f;
    for (int t = 0; t < T; ++t) acc += go[t * ldo + o];
    o2[dout * hid + o] = acc;
  }
}

// The same partial sums with register tiles (for hid % 8 == 0, dout % 4 ==
// 0): each contraction runs as outer products of float4 rows, about ten
// FMAs per load instead of one FMA per two loads.  Tile rows are padded by 4
// floats; a thread's four tokens are t, t+16, t+32, t+48, so the 16 token
// groups of a warp read different banks.  Every output is a sum over the
// chunk's tokens in token order (deterministic).
__host__ __device__ constexpr int pad4(int n) { return n + 4; }

__host__ __device__ constexpr size_t mlp_bwd_tiled_smem_floats(int F, int hid, int dout) {
  return static_cast<size_t>(kPosTok) * (pad4(4 * F) + 2 * pad4(hid) + pad4(dout));
}

__device__ __forceinline__ float f4get(const float4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

// grid (n_chunks, 2), block kPosThreads, dynamic smem mlp_bwd_tiled_smem_floats.
__global__ void __launch_bounds__(kPosThreads) mlp_bwd_tiled_kernel(PosParams p) {
  extern __shared__ float4 sm_pos4[];
  float* sm = reinterpret_cast<float*>(sm_pos4);
  const int side = blockIdx.y;
  const int chunk = blockIdx.x;
  const int t0 = chunk * kPosTok;
  // (debug build) this chunk's slice of the partials lies in the buffer
  if (!rib_guard((static_cast<size_t>(side) * p.n_chunks + chunk + 1) * p.n_params - 1,
                 2ull * p.n_chunks * p.n_params, G_MLP_PART))
    return;
  const int din = 4 * p.F, hid = p.hid, dout = p.dout;
  const int ldg = pad4(din), ldh = pad4(hid), ldo = pad4(dout);
  constexpr int T = kPosTok;
  float* g = sm;                 // [T][ldg]  Fourier features
  float* h = g + T * ldg;        // [T][ldh]  GELU(a)
  float* da = h + T * ldh;       // [T][ldh]  dL/da
  float* go = da + T * ldh;      // [T][ldo]  dL/d(out)
  fourier_tile(p, t0, g, ldg);
  for (int idx = threadIdx.x; idx < T * dout; idx += blockDim.x) {
    const int o = idx / T, t = idx - o * T;
    const int tok = t0 + t;
    const int head = o / p.rank, r = o - head * p.rank;
    const size_t gi = (static_cast<size_t>(head) * p.N + tok) * p.rank + r;
    go[t * ldo + o] = tok < p.N && rib_guard(gi, static_cast<size_t>(dout) * p.N, G_MLP_IN)
                          ? p.dtok[side][gi]
                          : 0.f;
  }
  __syncthreads();
  const float* w1 = p.w1[side];
  const float* b1 = p.b1[side];
  const float* w2 = p.w2[side];
  // ---- a = g W1^T + b1 and dh = go W2 for tokens tg + 16 j (j < 4) and
  // hidden units jh0 .. jh0 + 7; then h = GELU(a), da = dh * GELU'(a)
  for (int tile = threadIdx.x; tile < 16 * (hid / 8); tile += blockDim.x) {
    const int tg = tile % 16, jh0 = (tile / 16) * 8;
    // (debug build) the W1 rows and W2 columns this tile reads lie in W1, W2
    if (!rib_guard(static_cast<size_t>(jh0 + 7) * din + din - 1, static_cast<size_t>(hid) * din,
                   G_POS_W) ||
        !rib_guard(static_cast<size_t>(dout - 1) * hid + jh0 + 7, static_cast<size_t>(dout) * hid,
                   G_POS_W))
      continue;
    float acc[4][8], dh[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[j][i] = dh[j][i] = 0.f;
    for (int k = 0; k < din; k += 4) {
      float4 a4[4], b4[8];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        a4[j] = *reinterpret_cast<const float4*>(g + (tg + 16 * j) * ldg + k);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        b4[i] = __ldg(reinterpret_cast<const float4*>(w1 + static_cast<size_t>(jh0 + i) * din + k));
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[j][i] = fmaf(f4get(a4[j], q), f4get(b4[i], q), acc[j][i]);
    }
    for (int o = 0; o < dout; o += 4) {
      float4 a4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        a4[j] = *reinterpret_cast<const float4*>(go + (tg + 16 * j) * ldo + o);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float* wr = w2 + static_cast<size_t>(o + q) * hid + jh0;
        const float4 wa = __ldg(reinterpret_cast<const float4*>(wr));
        const float4 wb = __ldg(reinterpret_cast<const float4*>(wr + 4));
        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 8; ++i) dh[j][i] = fmaf(f4get(a4[j], q), wv[i], dh[j][i]);
      }
    }
    float bias[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) bias[i] = __ldg(b1 + jh0 + i);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float hv[8], dv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = acc[j][i] + bias[i];
        hv[i] = gelu_erf(a);
        dv[i] = dh[j][i] * gelu_erf_grad(a);   // tokens past N have go == 0
      }
      float4* hr = reinterpret_cast<float4*>(h + (tg + 16 * j) * ldh + jh0);
      float4* dr = reinterpret_cast<float4*>(da + (tg + 16 * j) * ldh + jh0);
      hr[0] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      hr[1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
      dr[0] = make_float4(dv[0], dv[1], dv[2], dv[3]);
      dr[1] = make_float4(dv[4], dv[5], dv[6], dv[7]);
    }
  }
  __syncthreads();
  float* out = p.partial + (static_cast<size_t>(side) * p.n_chunks + chunk) * p.n_params;
  // ---- dw1[jh][k] = sum_t da[t][jh] g[t][k]: tiles of 8 jh x 4 k
  for (int tile = threadIdx.x; tile < (hid / 8) * (din / 4); tile += blockDim.x) {
    const int k0 = 4 * (tile % (din / 4)), jh0 = (tile / (din / 4)) * 8;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
    for (int t = 0; t < T; ++t) {
      const float4 d0 = *reinterpret_cast<const float4*>(da + t * ldh + jh0);
      const float4 d1 = *reinterpret_cast<const float4*>(da + t * ldh + jh0 + 4);
      const float4 gv = *reinterpret_cast<const float4*>(g + t * ldg + k0);
      const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[i][0] = fmaf(dv[i], gv.x, acc[i][0]);
        acc[i][1] = fmaf(dv[i], gv.y, acc[i][1]);
        acc[i][2] = fmaf(dv[i], gv.z, acc[i][2]);
        acc[i][3] = fmaf(dv[i], gv.w, acc[i][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<float4*>(out + static_cast<size_t>(jh0 + i) * din + k0) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
  }
  for (int jh = threadIdx.x; jh < hid; jh += blockDim.x) {
    float acc = 0.f;
    for (int t = 0; t < T; ++t) acc += da[t * ldh + jh];
    out[hid * din + jh] = acc;
  }
  float* o2 = out + hid * din + hid;
  // ---- dw2[o][jh] = sum_t go[t][o] h[t][jh]: tiles of 4 o x 8 jh
  for (int tile = threadIdx.x; tile < (dout / 4) * (hid / 8); tile += blockDim.x) {
    const int jh0 = 8 * (tile % (hid / 8)), o0 = (tile / (hid / 8)) * 4;
    float acc[4][8];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q][i] = 0.f;
    for (int t = 0; t < T; ++t) {
      const float4 gv = *reinterpret_cast<const float4*>(go + t * ldo + o0);
      const float4 h0 = *reinterpret_cast<const float4*>(h + t * ldh + jh0);
      const float4 h1 = *reinterpret_cast<const float4*>(h + t * ldh + jh0 + 4);
      const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[0][i] = fmaf(gv.x, hv[i], acc[0][i]);
        acc[1][i] = fmaf(gv.y, hv[i], acc[1][i]);
        acc[2][i] = fmaf(gv.z, hv[i], acc[2][i]);
        acc[3][i] = fmaf(gv.w, hv[i], acc[3][i]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4* dst = reinterpret_cast<float4*>(o2 + static_cast<size_t>(o0 + q) * hid + jh0);
      dst[0] = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
      dst[1] = make_float4(acc[q][4], acc[q][5], acc[q][6], acc[q][7]);
    }
  }
  for (int o = threadIdx.x; o < dout; o += blockDim.x) {
    float acc = 0.f;
    for (int t = 0; t < T; ++t) acc += go[t * ldo + o];
    o2[dout * hid + o] = acc;
  }
}

// Position tokens with register tiles (hid % 8 == 0, rank % 8 == 0): the
// two Linear layers as outer products of float4 rows, tiles of 4 tokens
// (t, t+16, t+32, t+48) x 8 units.
__host__ __device__ constexpr size_t pos_tiled_smem_floats(int F, int hid) {
  return static_cast<size_t>(kPosTok) * (pad4(4 * F) + pad4(hid));
}

// grid (ceil(N / kPosTok), 2), block kPosThreads, dynamic smem pos_tiled_smem_floats.
__global__ void __launch_bounds__(kPosThreads) pos_tokens_tiled_kernel(PosParams p) {
  extern __shared__ float4 sm_pos4[];
  float* sm = reinterpret_cast<float*>(sm_pos4);
  const int side = blockIdx.y;
  const int t0 = blockIdx.x * kPosTok;
  const int din = 4 * p.F, hid = p.hid, dout = p.dout;
  const int ldg = pad4(din), ldh = pad4(hid);
  float* g = sm;                   // [kPosTok][ldg]
  float* h = g + kPosTok * ldg;    // [kPosTok][ldh]
  fourier_tile(p, t0, g, ldg);
  __syncthreads();
  const float* w1 = p.w1[side];
  const float* b1 = p.b1[side];
  const float* w2 = p.w2[side];
  const float* b2 = p.b2[side];
  // h = GELU(g W1^T + b1)
  for (int tile = threadIdx.x; tile < 16 * (hid / 8); tile += blockDim.x) {
    const int tg = tile % 16, jh0 = (tile / 16) * 8;
    if (!rib_guard(static_cast<size_t>(jh0 + 7) * din + din - 1, static_cast<size_t>(hid) * din,
                   G_POS_W))
      continue;
    float acc[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[j][i] = 0.f;
    for (int k = 0; k < din; k += 4) {
      float4 a4[4], b4[8];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        a4[j] = *reinterpret_cast<const float4*>(g + (tg + 16 * j) * ldg + k);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        b4[i] = __ldg(reinterpret_cast<const float4*>(w1 + static_cast<size_t>(jh0 + i) * din + k));
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[j][i] = fmaf(f4get(a4[j], q), f4get(b4[i], q), acc[j][i]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float hv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[i] = gelu_erf(acc[j][i] + __ldg(b1 + jh0 + i));
      float4* hr = reinterpret_cast<float4*>(h + (tg + 16 * j) * ldh + jh0);
      hr[0] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      hr[1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
    }
  }
  __syncthreads();
  // out = h W2^T + b2; 8 consecutive outputs lie in one head (rank % 8 == 0)
  for (int tile = threadIdx.x; tile < 16 * (dout / 8); tile += blockDim.x) {
    const int tg = tile % 16, o0 = (tile / 16) * 8;
    if (!rib_guard(static_cast<size_t>(o0 + 7) * hid + hid - 1, static_cast<size_t>(dout) * hid,
                   G_POS_W))
      continue;
    float acc[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[j][i] = 0.f;
    for (int k = 0; k < hid; k += 4) {
      float4 a4[4], b4[8];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        a4[j] = *reinterpret_cast<const float4*>(h + (tg + 16 * j) * ldh + k);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        b4[i] = __ldg(reinterpret_cast<const float4*>(w2 + static_cast<size_t>(o0 + i) * hid + k));
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[j][i] = fmaf(f4get(a4[j], q), f4get(b4[i], q), acc[j][i]);
    }
    const int head = o0 / p.rank, r0 = o0 - head * p.rank;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tok = t0 + tg + 16 * j;
      if (tok >= p.N) continue;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = acc[j][i] + __ldg(b2 + o0 + i);
      const size_t off = (static_cast<size_t>(head) * p.N + tok) * p.rank + r0;
      if (!rib_guard(off + 7, static_cast<size_t>(dout) * p.N, G_POS_OUT)) continue;
      float4* d32 = reinterpret_cast<float4*>(p.out32[side] + off);
      d32[0] = make_float4(v[0], v[1], v[2], v[3]);
      d32[1] = make_float4(v[4], v[5], v[6], v[7]);
      if (p.out16[side]) {
        uint32_t u[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2v = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
          u[e] = *reinterpret_cast<const uint32_t*>(&b2v);
        }
        *reinterpret_cast<uint4*>(p.out16[side] + off) = make_uint4(u[0], u[1], u[2], u[3]);
      }
    }
  }
}

// Fixed-order sum of the chunk partials: grid (ceil(n_params / 256), 2).
__global__ void __launch_bounds__(256) mlp_bwd_reduce_kernel(PosParams p) {
  const int side = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.n_params) return;
  const float* src = p.partial + static_cast<size_t>(side) * p.n_chunks * p.n_params + idx;
  if (!rib_guard((static_cast<size_t>(side) * p.n_chunks + p.n_chunks - 1) * p.n_params + idx,
                 2ull * p.n_chunks * p.n_params, G_MLP_PART))
    return;
  float acc = 0.f;
  for (int c = 0; c < p.n_chunks; ++c) acc += src[static_cast<size_t>(c) * p.n_params];
  const int din = 4 * p.F;
  const int n_w1 = p.hid * din, n_b1 = p.hid, n_w2 = p.dout * p.hid;
  if (idx < n_w1) p.grads[side][0][idx] = acc;
  else if (idx < n_w1 + n_b1) p.grads[side][1][idx - n_w1] = acc;
  else if (idx < n_w1 + n_b1 + n_w2) p.grads[side][2][idx - n_w1 - n_b1] = acc;
  else p.grads[side][3][idx - n_w1 - n_b1 - n_w2] = acc;
}

}  // namespace rib
