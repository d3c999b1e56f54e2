// rib.cu -- librib.so: the C ABI of include/rib.h.
//
// Host side of every entry point: argument validation (before anything is
// launched), TMA tensor-map encoding for the rolled window addressing,
// workspace carving and kernel launches on the caller's stream.  All device
// code lives in the .cuh files included below, in one translation unit so
// that every kernel shares the per-device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "rib.h"
#include "ptx.cuh"
#include "geom.cuh"
#include "pos_tokens.cuh"
#include "window_copy.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_tf32.cuh"
#include "attn_bwd.cuh"
#include "attn_bwd_persist.cuh"
#include "cla.cuh"
#include "cla_bwd.cuh"

namespace rib {
namespace {

// ---------------------------------------------------------------- helpers

unsigned long long g_wait_limit_ns = 1000000000ull;  // 1 s
// Backward kernel form: RIB_BWD_AUTO picks by window size (rib_bwd_kernel_for)
std::atomic<int> g_bwd_kernel{RIB_BWD_AUTO};
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tiled tensor map; dims/box innermost first, strides in bytes for dims 1..rank-1.
int make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
             const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
             CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return RIB_ERR_CUDA;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides[i];
  }
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s, b, e,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RIB_OK : RIB_ERR_CUDA;
}

// qkv-like tensor [B][H][W][slots][32] bf16 as a 5D map with 8x8-pixel boxes.
int map_tokens(CUtensorMap* m, const void* base, int B, int H, int W, int slots) {
  const uint64_t dims[5] = {32, (uint64_t)slots, (uint64_t)W, (uint64_t)H, (uint64_t)B};
  const uint64_t row = 64;
  const uint64_t strides[4] = {row, row * slots, row * slots * W, row * slots * W * H};
  const uint32_t box[5] = {32, 1, 8, 8, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_64B);
}

// positional tokens [heads][M][M][16] bf16, 8x8-token boxes.
int map_pos(CUtensorMap* m, const void* base, int heads, int M) {
  const uint64_t dims[4] = {16, (uint64_t)M, (uint64_t)M, (uint64_t)heads};
  const uint64_t strides[3] = {32, 32ull * M, 32ull * M * M};
  const uint32_t box[4] = {16, 8, 8, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_32B);
}

// The same tensor fetched as 64-byte rows: the box is 32 channels wide, so
// TMA zero-fills channels 16..31 (out of bounds), giving a 64B-swizzle tile
// that sits beside a content tile as a second atom of one MMA operand.
int map_pos_padded(CUtensorMap* m, const void* base, int heads, int M) {
  const uint64_t dims[4] = {16, (uint64_t)M, (uint64_t)M, (uint64_t)heads};
  const uint64_t strides[3] = {32, 32ull * M, 32ull * M * M};
  const uint32_t box[4] = {32, 8, 8, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_64B);
}

// fp32 qkv-like tensor [B][H][W][slots][32]: 128-byte rows, 128B swizzle
// (the tf32 forward's K-major and MN-major operand tiles).
// sw: CU_TENSOR_MAP_SWIZZLE_128B for K-major operand tiles,
// CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B for the MN-major V tile.
int map_tokens_f32(CUtensorMap* m, const void* base, int B, int H, int W, int slots,
                   CUtensorMapSwizzle sw) {
  const uint64_t dims[5] = {32, (uint64_t)slots, (uint64_t)W, (uint64_t)H, (uint64_t)B};
  const uint64_t row = 128;
  const uint64_t strides[4] = {row, row * slots, row * slots * W, row * slots * W * H};
  const uint32_t box[5] = {32, 1, 8, 8, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, base, dims, strides, box, sw);
}

// fp32 positional tokens [heads][M][M][16]: 64-byte rows, 64B swizzle.
int map_pos_f32(CUtensorMap* m, const void* base, int heads, int M) {
  const uint64_t dims[4] = {16, (uint64_t)M, (uint64_t)M, (uint64_t)heads};
  const uint64_t strides[3] = {64, 64ull * M, 64ull * M * M};
  const uint32_t box[4] = {16, 8, 8, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_64B);
}

// per-pixel fp32 [B][heads][H][W], 8x8-pixel boxes.
int map_pixel_f32(CUtensorMap* m, const void* base, int B, int heads, int H, int W) {
  const uint64_t dims[4] = {(uint64_t)W, (uint64_t)H, (uint64_t)heads, (uint64_t)B};
  const uint64_t strides[3] = {4ull * W, 4ull * W * H, 4ull * W * H * heads};
  const uint32_t box[4] = {8, 8, 1, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ---------------------------------------------------------------- tracing
enum KernelId {
  K_POS, K_FWD, K_BWD_PRE, K_BWD, K_DQ_FIN, K_POSGRAD, K_MLP_PART, K_MLP_RED, K_COPY, K_DEBUG,
  K_CLA, K_CLA_DZ, K_CLA_DWPW, K_CLA_DX, K_CLA_RED, K_BWD_PERSIST, K_FWD_TF32, K_CLA_DY, K_COUNT
};
const char* const kKernelNames[K_COUNT] = {
    "pos_tokens_kernel",   "attn_fwd_kernel",        "bwd_preprocess_kernel",
    "attn_bwd_kernel",     "dq_finalize_kernel",     "posgrad_reduce_kernel",
    "mlp_bwd_partial_kernel", "mlp_bwd_reduce_kernel", "window_copy_kernel",
    "debug_wait_kernel",   "cla_gate_kernel",        "cla_bwd_dz_kernel",
    "cla_bwd_dwpw_kernel", "cla_bwd_dx_kernel",      "cla_bwd_reduce_kernel",
    "attn_bwd_persistent_kernel", "attn_fwd_tf32_kernel", "cla_bwd_dy_kernel"};

struct TraceRec {
  int id;
  cudaEvent_t a, b;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t pooled_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Records CUDA events around one kernel launch when tracing is on.
struct TraceScope {
  int id;
  cudaStream_t st;
  bool on;
  cudaEvent_t a = nullptr, b = nullptr;
  TraceScope(int kid, cudaStream_t s) : id(kid), st(s) {
    std::lock_guard<std::mutex> g(g_trace_mu);
    on = g_trace_on;
    if (on) {
      a = pooled_event();
      b = pooled_event();
      cudaEventRecord(a, st);
    }
  }
  ~TraceScope() {
    if (!on) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> g(g_trace_mu);
    g_trace.push_back({id, a, b});
  }
};

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? RIB_OK : RIB_ERR_CUDA;
}

template <typename K>
int set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes)) == cudaSuccess
             ? RIB_OK
             : RIB_ERR_CUDA;
}

struct AttnGeom {
  int nWx, nW, N, tiles_x, n_tiles, units;
};

// Shape checks shared by forward and backward.
int check_attn(int B, int H, int W, int heads, int head_dim, int M, int shift, int rank,
               AttnGeom* g) {
  if (B < 0 || H <= 0 || W <= 0 || heads <= 0 || M <= 0) return RIB_ERR_ARG;
  if (H % M != 0 || W % M != 0 || shift < 0 || shift >= M) return RIB_ERR_SHAPE;
  if (head_dim != 32 || (rank != 0 && rank != 16)) return RIB_ERR_UNSUPPORTED;
  if (M % 16 != 0 || M > 256 || shift % 8 != 0) return RIB_ERR_UNSUPPORTED;
  if ((long long)B * H > (1ll << 30) || (long long)W * heads * 3 > (1ll << 30))
    return RIB_ERR_UNSUPPORTED;
  g->nWx = W / M;
  g->nW = (H / M) * (W / M);
  g->N = M * M;
  g->tiles_x = M / 16;
  g->n_tiles = g->N / 128;
  const long long units = (long long)B * g->nW * heads;
  if (units > 65535) return RIB_ERR_UNSUPPORTED;
  g->units = static_cast<int>(units);
  return RIB_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct BwdWs {
  size_t lse2, dd, dq_acc, dkp_part, mlp_part, total;
  int n_chunks, n_params;
};

BwdWs bwd_ws_layout(int B, int H, int W, int heads, int M, int rank, const rib_mlp_t* mlp) {
  BwdWs w{};
  const size_t pix = (size_t)B * heads * H * W;
  const size_t tokens = (size_t)B * H * W * heads;  // = units * N
  size_t off = 0;
  w.lse2 = off;
  off = align256(off + pix * 4);
  w.dd = off;
  off = align256(off + pix * 4);
  w.dq_acc = off;
  off = align256(off + tokens * 48 * 4);
  w.dkp_part = off;
  off = align256(off + (rank > 0 ? tokens * 16 * 4 : 0));
  w.mlp_part = off;
  if (mlp && rank > 0) {
    const int N = M * M;
    w.n_chunks = (N + kMlpBwdTok - 1) / kMlpBwdTok;
    w.n_params = mlp->d_hidden * 4 * mlp->n_freq + mlp->d_hidden +
                 mlp->heads * mlp->rank * mlp->d_hidden + mlp->heads * mlp->rank;
    off = align256(off + 2ull * w.n_chunks * w.n_params * 4);
  }
  w.total = off;
  return w;
}

int check_mlp(const rib_mlp_t* m) {
  if (!m || !m->freqs || !m->q_w1 || !m->q_b1 || !m->q_w2 || !m->q_b2 || !m->k_w1 ||
      !m->k_b1 || !m->k_w2 || !m->k_b2)
    return RIB_ERR_ARG;
  if (m->n_freq <= 0 || m->d_hidden <= 0 || m->heads <= 0 || m->rank <= 0) return RIB_ERR_ARG;
  if (m->n_freq > 64 || m->d_hidden > 512 || m->heads * m->rank > 1024) return RIB_ERR_UNSUPPORTED;
  return RIB_OK;
}

PosParams pos_params(const rib_mlp_t* m, int M) {
  PosParams p{};
  p.M = M;
  p.N = M * M;
  p.F = m->n_freq;
  p.hid = m->d_hidden;
  p.dout = m->heads * m->rank;
  p.rank = m->rank;
  p.freqs = m->freqs;
  p.w1[0] = m->q_w1; p.b1[0] = m->q_b1; p.w2[0] = m->q_w2; p.b2[0] = m->q_b2;
  p.w1[1] = m->k_w1; p.b1[1] = m->k_b1; p.w2[1] = m->k_w2; p.b2[1] = m->k_b2;
  return p;
}

// Position-MLP backward: per-chunk partial sums, then a fixed-order chunk sum.
int launch_mlp_bwd(const rib_mlp_t* mlp, int window, const float* dqp, const float* dkp,
                   const rib_mlp_grad_t* dmlp, void* partial, int n_chunks, int n_params,
                   cudaStream_t st) {
  PosParams pp = pos_params(mlp, window);
  pp.dtok[0] = dqp;
  pp.dtok[1] = dkp;
  pp.partial = static_cast<float*>(partial);
  pp.n_chunks = n_chunks;
  pp.n_params = n_params;
  pp.grads[0][0] = dmlp->q_dw1; pp.grads[0][1] = dmlp->q_db1;
  pp.grads[0][2] = dmlp->q_dw2; pp.grads[0][3] = dmlp->q_db2;
  pp.grads[1][0] = dmlp->k_dw1; pp.grads[1][1] = dmlp->k_db1;
  pp.grads[1][2] = dmlp->k_dw2; pp.grads[1][3] = dmlp->k_db2;
  // register-tiled partial sums where the shapes and the weights' alignment
  // allow float4 rows, else the general kernel
  const size_t smem_t = mlp_bwd_tiled_smem_floats(pp.F, pp.hid, pp.dout) * sizeof(float);
  const bool tiled = pp.hid % 8 == 0 && pp.dout % 4 == 0 && smem_t <= 200 * 1024 &&
                     aligned16(pp.w1[0]) && aligned16(pp.w1[1]) && aligned16(pp.w2[0]) &&
                     aligned16(pp.w2[1]);
  const size_t smem = tiled ? smem_t : mlp_bwd_smem_floats(pp.F, pp.hid, pp.dout) * sizeof(float);
  if (smem > 200 * 1024) return RIB_ERR_UNSUPPORTED;
  int rc;
  if ((rc = set_smem(tiled ? mlp_bwd_tiled_kernel : mlp_bwd_partial_kernel, smem))) return rc;
  {
    TraceScope ts(K_MLP_PART, st);
    if (tiled)
      mlp_bwd_tiled_kernel<<<dim3(n_chunks, 2), kPosThreads, smem, st>>>(pp);
    else
      mlp_bwd_partial_kernel<<<dim3(n_chunks, 2), kPosThreads, smem, st>>>(pp);
  }
  if ((rc = launch_status())) return rc;
  {
    TraceScope ts(K_MLP_RED, st);
    mlp_bwd_reduce_kernel<<<dim3((n_params + 255) / 256, 2), 256, 0, st>>>(pp);
  }
  return launch_status();
}

bool mlp_grad_complete(const rib_mlp_grad_t* d) {
  return d && d->q_dw1 && d->q_db1 && d->q_dw2 && d->q_db2 && d->k_dw1 && d->k_db1 &&
         d->k_dw2 && d->k_db2;
}

// Scratch of rib_pos_tokens_bwd_noalloc: part of the library image, one copy
// per device.  Host code cannot take its address directly (the name is a
// host-side stand-in), so each device's address is looked up once with
// cudaGetSymbolAddress and cached here.
__device__ __align__(256) unsigned char g_noalloc_scratch[RIB_NOALLOC_SCRATCH_BYTES];
constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (set up on first use).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RIB_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RIB_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RIB_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return RIB_OK;
}

__global__ void debug_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must run out and record a timeout.
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns, SITE_DEBUG);
}

#ifdef RIB_DEBUG
// Test of the debug build's guards: element `idx` of a shared array of
// `n` floats (n <= 32) is written only if the guard lets it through; an
// index beyond the array is refused and recorded, and nothing is written.
__global__ void debug_guard_kernel(int idx, int n, int* seen) {
  __shared__ float buf[32];
  if (threadIdx.x == 0) buf[0] = 0.f;
  __syncthreads();
  if (threadIdx.x == 0 && rib_guard(static_cast<unsigned long long>(idx),
                                    static_cast<unsigned long long>(n), G_SELFTEST))
    buf[idx & 31] = 1.f;
  __syncthreads();
  if (threadIdx.x == 0 && seen) *seen = buf[0] != 0.f ? 1 : 0;
}
#endif

__global__ void debug_exp2_kernel(const float* x, float* y, int n_pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  const uint64_t r = exp2_fma2(pk2(x[2 * i], x[2 * i + 1]));
  y[2 * i] = lo2(r);
  y[2 * i + 1] = hi2(r);
}

struct ClaBwdLayout {
  size_t dz, dy, part_dbpw, part_dwpw, part_dw, total;
  int grid, grid_dx, n_tiles;
};

int cla_check(int B, int H, int W, int C) {
  if (B < 0 || H <= 0 || W <= 0 || C <= 0) return RIB_ERR_ARG;
  if (C % 32 != 0 || cla_smem_bytes(C) > 227u * 1024u || cla_dy_smem_bytes(C) > 227u * 1024u ||
      cla_dwpw_smem_bytes(C) > 227u * 1024u)
    return RIB_ERR_UNSUPPORTED;
  if (H % 8 != 0 || W % 16 != 0) return RIB_ERR_SHAPE;
  if ((long long)B * H * W * C > (1ll << 40) || B > (1 << 20)) return RIB_ERR_UNSUPPORTED;
  if ((long long)B * (H / 8) * (W / 16) > (1ll << 30)) return RIB_ERR_UNSUPPORTED;
  return RIB_OK;
}

// The partial sums are sized for the launch grids: one CTA per SM for the
// two tensor-core kernels, two per SM for the dx kernel (its registers allow
// two or three; more CTAs would only lengthen the reduction's sums).
ClaBwdLayout cla_bwd_layout(int B, int H, int W, int C, int sms) {
  ClaBwdLayout L;
  L.n_tiles = B * (H / 8) * (W / 16);
  L.grid = std::min(std::min(L.n_tiles, sms), 1024);
  L.grid_dx = std::min(std::min(L.n_tiles, 2 * sms), 2048);
  const size_t P = (size_t)B * H * W;
  size_t off = 0;
  L.dz = off; off = align256(off + P * C * 2);
  L.dy = off; off = align256(off + P * C * 2);
  L.part_dbpw = off; off = align256(off + (size_t)L.grid * C * 4);
  L.part_dwpw = off; off = align256(off + (size_t)L.grid * C * C * 4);
  L.part_dw = off; off = align256(off + (size_t)L.grid_dx * 10 * C * 4);
  L.total = off;
  return L;
}

int device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return RIB_ERR_CUDA;
  return RIB_OK;
}

}  // namespace
}  // namespace rib

using namespace rib;

extern "C" {

const char* rib_version(void) { return "rib-b200 0.1 sm_100a"; }

const char* rib_status_string(int s) {
  switch (s) {
    case RIB_OK: return "RIB_OK";
    case RIB_ERR_ARG: return "RIB_ERR_ARG";
    case RIB_ERR_SHAPE: return "RIB_ERR_SHAPE";
    case RIB_ERR_UNSUPPORTED: return "RIB_ERR_UNSUPPORTED";
    case RIB_ERR_WORKSPACE: return "RIB_ERR_WORKSPACE";
    case RIB_ERR_CUDA: return "RIB_ERR_CUDA";
    case RIB_ERR_TIMEOUT: return "RIB_ERR_TIMEOUT";
    case RIB_ERR_ALIGN: return "RIB_ERR_ALIGN";
    case RIB_ERR_BOUNDS: return "RIB_ERR_BOUNDS";
    default: return "RIB_ERR_UNKNOWN";
  }
}

int rib_last_status(int* site) {
  if (cudaDeviceSynchronize() != cudaSuccess) return RIB_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpyFromSymbol(h, g_status, sizeof(h)) != cudaSuccess) return RIB_ERR_CUDA;
  const int zero[2] = {0, 0};
  if (cudaMemcpyToSymbol(g_status, zero, sizeof(zero)) != cudaSuccess) return RIB_ERR_CUDA;
  if (site) *site = h[1];
  return h[0];
}

int rib_set_bwd_kernel(int which) {
  if (which != RIB_BWD_AUTO && which != RIB_BWD_PER_ITEM && which != RIB_BWD_PERSISTENT)
    return RIB_ERR_ARG;
  g_bwd_kernel.store(which);
  return RIB_OK;
}

int rib_bwd_kernel_for(int window) {
  const int which = g_bwd_kernel.load();
  if (which != RIB_BWD_AUTO) return which;
  // Up to 64 x 64 windows (32 query tiles per key tile) the per-CTA set-up
  // and the pipeline's ramp and drain weigh on few tiles, and the persistent
  // form, which overlaps them with the neighbouring item, is faster; at
  // 96 x 96 windows the per-item kernel is.
  return window <= 64 ? RIB_BWD_PERSISTENT : RIB_BWD_PER_ITEM;
}

int rib_set_wait_limit_ns(unsigned long long limit_ns) {
  g_wait_limit_ns = limit_ns ? limit_ns : kDefaultWaitLimitNs;
  return RIB_OK;
}

int rib_trace_enable(int on) {
  std::lock_guard<std::mutex> g(g_trace_mu);
  if (on) {
    for (auto& r : g_trace) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
    g_trace.clear();
  }
  g_trace_on = on != 0;
  return RIB_OK;
}

int rib_trace_collect(rib_trace_entry_t* entries, int max_entries, int* n_entries) {
  std::lock_guard<std::mutex> g(g_trace_mu);
  int launches[K_COUNT] = {0};
  double ms[K_COUNT] = {0};
  int rc = RIB_OK;
  for (auto& r : g_trace) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      rc = RIB_ERR_CUDA;
    launches[r.id] += 1;
    ms[r.id] += t;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_trace.clear();
  int n = 0;
  for (int k = 0; k < K_COUNT; ++k) {
    if (!launches[k]) continue;
    if (entries && n < max_entries) entries[n] = {kKernelNames[k], launches[k], ms[k]};
    ++n;
  }
  if (n_entries) *n_entries = n < max_entries ? n : max_entries;
  return rc;
}

int rib_debug_exp2(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n < 0 || (n & 1)) return RIB_ERR_ARG;
  if (n == 0) return RIB_OK;
  const int pairs = n / 2;
  debug_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, pairs);
  return launch_status();
}

int rib_debug_build(void) {
#ifdef RIB_DEBUG
  return 1;
#else
  return 0;
#endif
}

int rib_debug_guard_info(unsigned long long* index_extent) {
  if (!index_extent) return RIB_ERR_ARG;
  index_extent[0] = index_extent[1] = 0;
#ifdef RIB_DEBUG
  if (cudaDeviceSynchronize() != cudaSuccess) return RIB_ERR_CUDA;
  if (cudaMemcpyFromSymbol(index_extent, g_guard_info, 2 * sizeof(unsigned long long)) !=
      cudaSuccess)
    return RIB_ERR_CUDA;
  const unsigned long long zero[2] = {0, 0};
  if (cudaMemcpyToSymbol(g_guard_info, zero, sizeof(zero)) != cudaSuccess) return RIB_ERR_CUDA;
#endif
  return RIB_OK;
}

int rib_debug_guard_selftest(int index, int extent, void* stream) {
#ifdef RIB_DEBUG
  if (extent < 0 || extent > 32 || index < 0) return RIB_ERR_ARG;
  debug_guard_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(index, extent, nullptr);
  return launch_status();
#else
  (void)index;
  (void)extent;
  (void)stream;
  return RIB_ERR_UNSUPPORTED;
#endif
}

int rib_debug_wait_timeout(unsigned long long limit_ns, void* stream) {
  debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return launch_status();
}

int rib_pos_tokens(const rib_mlp_t* mlp, int window, float* qp, float* kp, void* qp_bf16,
                   void* kp_bf16, void* stream) {
  int rc = check_mlp(mlp);
  if (rc) return rc;
  if (!qp || !kp) return RIB_ERR_ARG;
  if (window <= 0) return RIB_ERR_ARG;
  if (window > 256) return RIB_ERR_UNSUPPORTED;
  PosParams p = pos_params(mlp, window);
  p.out32[0] = qp;
  p.out32[1] = kp;
  p.out16[0] = static_cast<__nv_bfloat16*>(qp_bf16);
  p.out16[1] = static_cast<__nv_bfloat16*>(kp_bf16);
  // register-tiled MLP where the shapes and alignments allow float4 rows
  const size_t smem_t = pos_tiled_smem_floats(p.F, p.hid) * sizeof(float);
  const bool tiled = p.hid % 8 == 0 && p.rank % 8 == 0 && smem_t <= 200 * 1024 &&
                     aligned16(p.w1[0]) && aligned16(p.w1[1]) && aligned16(p.w2[0]) &&
                     aligned16(p.w2[1]) && aligned16(qp) && aligned16(kp) &&
                     (!qp_bf16 || aligned16(qp_bf16)) && (!kp_bf16 || aligned16(kp_bf16));
  const size_t smem = tiled ? smem_t : pos_fwd_smem_floats(p.F, p.hid) * sizeof(float);
  if (smem > 200 * 1024) return RIB_ERR_UNSUPPORTED;
  if ((rc = set_smem(tiled ? pos_tokens_tiled_kernel : pos_tokens_kernel, smem))) return rc;
  dim3 grid((p.N + kPosTok - 1) / kPosTok, 2);
  TraceScope ts(K_POS, static_cast<cudaStream_t>(stream));
  if (tiled)
    pos_tokens_tiled_kernel<<<grid, kPosThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
  else
    pos_tokens_kernel<<<grid, kPosThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}

size_t rib_pos_tokens_bwd_workspace(const rib_mlp_t* mlp, int window) {
  if (check_mlp(mlp) != RIB_OK || window <= 0 || window > 256) return 0;
  const int N = window * window;
  const size_t n_chunks = (N + kMlpBwdTok - 1) / kMlpBwdTok;
  const size_t n_params = (size_t)mlp->d_hidden * 4 * mlp->n_freq + mlp->d_hidden +
                          (size_t)mlp->heads * mlp->rank * mlp->d_hidden +
                          (size_t)mlp->heads * mlp->rank;
  return align256(2 * n_chunks * n_params * sizeof(float));
}

int rib_pos_tokens_bwd(const rib_mlp_t* mlp, int window, const float* dqp, const float* dkp,
                       const rib_mlp_grad_t* dmlp, void* workspace, size_t workspace_bytes,
                       void* stream) {
  int rc = check_mlp(mlp);
  if (rc) return rc;
  if (window <= 0 || !dqp || !dkp || !mlp_grad_complete(dmlp)) return RIB_ERR_ARG;
  if (window > 256) return RIB_ERR_UNSUPPORTED;
  const size_t need = rib_pos_tokens_bwd_workspace(mlp, window);
  if (!workspace || workspace_bytes < need) return RIB_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RIB_ERR_ALIGN;
  const int N = window * window;
  const int n_chunks = (N + kMlpBwdTok - 1) / kMlpBwdTok;
  const int n_params = mlp->d_hidden * 4 * mlp->n_freq + mlp->d_hidden +
                       mlp->heads * mlp->rank * mlp->d_hidden + mlp->heads * mlp->rank;
  return launch_mlp_bwd(mlp, window, dqp, dkp, dmlp, workspace, n_chunks, n_params,
                        static_cast<cudaStream_t>(stream));
}

int rib_pos_tokens_bwd_noalloc(const rib_mlp_t* mlp, int window, const float* dqp,
                               const float* dkp, const rib_mlp_grad_t* dmlp, void* stream) {
  int rc = check_mlp(mlp);
  if (rc) return rc;
  if (window <= 0 || !dqp || !dkp || !mlp_grad_complete(dmlp)) return RIB_ERR_ARG;
  if (window > 256) return RIB_ERR_UNSUPPORTED;
  if (rib_pos_tokens_bwd_workspace(mlp, window) > RIB_NOALLOC_SCRATCH_BYTES)
    return RIB_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  const int N = window * window;
  const int n_chunks = (N + kMlpBwdTok - 1) / kMlpBwdTok;
  const int n_params = mlp->d_hidden * 4 * mlp->n_freq + mlp->d_hidden +
                       mlp->heads * mlp->rank * mlp->d_hidden + mlp->heads * mlp->rank;
  return launch_mlp_bwd(mlp, window, dqp, dkp, dmlp, scratch, n_chunks, n_params,
                        static_cast<cudaStream_t>(stream));
}

// Kernels that move registers between warpgroups with setmaxnreg are only
// safe when compiled to the per-thread launch budget their split assumes.
// The count is a property of the library's one sm_100a image, so it is read
// once per kernel variant and cached (atomically: calls may come from any
// thread, for any device).
static int check_launch_regs(const void* kern, std::atomic<int>& cache, int expected) {
  int regs = cache.load(std::memory_order_acquire);
  if (regs < 0) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return RIB_ERR_CUDA;
    regs = fa.numRegs;
    cache.store(regs, std::memory_order_release);
  }
  return regs == expected ? RIB_OK : RIB_ERR_UNSUPPORTED;
}

static int attn_fwd_launch(const void* qkv, int B, int H, int W, int heads, int head_dim,
                           int window, int shift, const void* qp_bf16, const void* kp_bf16,
                           int rank, float scale, void* out, float* lse, const void* gate,
                           void* out_gated, int region_mask, void* stream) {
  AttnGeom g;
  int rc = check_attn(B, H, W, heads, head_dim, window, shift, rank, &g);
  if (rc) return rc;
  if (!std::isfinite(scale)) return RIB_ERR_ARG;
  if (B == 0) return RIB_OK;   // an empty batch: nothing to compute or write
  if (!qkv || !out || !lse) return RIB_ERR_ARG;
  if ((gate == nullptr) != (out_gated == nullptr)) return RIB_ERR_ARG;
  if (gate && (!aligned16(gate) || !aligned16(out_gated))) return RIB_ERR_ALIGN;
  if (rank > 0 && (!qp_bf16 || !kp_bf16)) return RIB_ERR_ARG;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(lse) ||
      (rank > 0 && (!aligned16(qp_bf16) || !aligned16(kp_bf16))))
    return RIB_ERR_ALIGN;
  if (!std::isfinite(scale)) return RIB_ERR_ARG;
  const float tau = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(head_dim + rank));
  CUtensorMap tq, tqp, tkp;
  if ((rc = map_tokens(&tq, qkv, B, H, W, 3 * heads))) return rc;
  if (rank > 0) {
    if ((rc = map_pos(&tqp, qp_bf16, heads, window))) return rc;
    if ((rc = map_pos(&tkp, kp_bf16, heads, window))) return rc;
  } else {
    tqp = tq;
    tkp = tq;
  }
  FwdParams p{};
  p.B = B; p.H = H; p.W = W; p.heads = heads; p.M = window; p.s = shift; p.rank = rank;
  p.nWx = g.nWx; p.nW = g.nW; p.tiles_x = g.tiles_x; p.n_tiles = g.n_tiles;
  p.region_mask = region_mask != 0 && shift > 0;
  p.scale_log2 = tau * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.out_gated = static_cast<__nv_bfloat16*>(out_gated);
  p.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 ? 1 : 0;
  p.gated_v8 = (reinterpret_cast<uintptr_t>(out_gated) & 31u) == 0 ? 1 : 0;
  p.wait_limit_ns = g_wait_limit_ns;
  auto* kern = p.region_mask ? attn_fwd_kernel<true> : attn_fwd_kernel<false>;
  if ((rc = set_smem(kern, kFwdSmemBytes))) return rc;
  {
    // setmaxnreg split: only safe with the launch budget it was sized for
    static std::atomic<int> launch_regs[2] = {{-1}, {-1}};
    if ((rc = check_launch_regs(reinterpret_cast<const void*>(kern), launch_regs[p.region_mask ? 1 : 0], kFwdLaunchRegs)))
      return rc;
  }
  // one CTA per SM walks the work items (unit, pair of query tiles)
  int sms = 0;
  if ((rc = device_sms(&sms))) return rc;
  p.n_items = g.units * (g.n_tiles / 2);
  dim3 grid(std::min(p.n_items, sms));
  TraceScope ts(K_FWD, static_cast<cudaStream_t>(stream));
  kern<<<grid, kFwdThreads, kFwdSmemBytes, static_cast<cudaStream_t>(stream)>>>(tq, tqp, tkp, p);
  return launch_status();
}

int rib_window_attn_fwd(const void* qkv, int B, int H, int W, int heads, int head_dim,
                        int window, int shift, const void* qp_bf16, const void* kp_bf16,
                        int rank, float scale, void* out, float* lse, void* stream) {
  return attn_fwd_launch(qkv, B, H, W, heads, head_dim, window, shift, qp_bf16, kp_bf16, rank,
                         scale, out, lse, nullptr, nullptr, 0, stream);
}

int rib_window_attn_fwd_masked(const void* qkv, int B, int H, int W, int heads, int head_dim,
                               int window, int shift, const void* qp_bf16, const void* kp_bf16,
                               int rank, float scale, void* out, float* lse, void* stream) {
  return attn_fwd_launch(qkv, B, H, W, heads, head_dim, window, shift, qp_bf16, kp_bf16, rank,
                         scale, out, lse, nullptr, nullptr, 1, stream);
}

int rib_window_attn_fwd_cla(const void* qkv, int B, int H, int W, int heads, int head_dim,
                            int window, int shift, const void* qp_bf16, const void* kp_bf16,
                            int rank, float scale, const void* gate, void* out, void* out_gated,
                            float* lse, void* stream) {
  if (!gate || !out_gated) return RIB_ERR_ARG;
  return attn_fwd_launch(qkv, B, H, W, heads, head_dim, window, shift, qp_bf16, kp_bf16, rank,
                         scale, out, lse, gate, out_gated, 0, stream);
}

int rib_window_attn_fwd_tf32(const float* qkv, int B, int H, int W, int heads, int head_dim,
                             int window, int shift, const float* qp, const float* kp, int rank,
                             float scale, float* out, float* lse, void* stream) {
  AttnGeom g;
  int rc = check_attn(B, H, W, heads, head_dim, window, shift, rank, &g);
  if (rc) return rc;
  if (B == 0) return RIB_OK;
  if (!qkv || !out || !lse || (rank > 0 && (!qp || !kp))) return RIB_ERR_ARG;
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(lse) ||
      (rank > 0 && (!aligned16(qp) || !aligned16(kp))))
    return RIB_ERR_ALIGN;
  if (!std::isfinite(scale)) return RIB_ERR_ARG;
  const float tau = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(head_dim + rank));
  CUtensorMap tq, tv, tqp, tkp;
  if ((rc = map_tokens_f32(&tq, qkv, B, H, W, 3 * heads, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  if ((rc = map_tokens_f32(&tv, qkv, B, H, W, 3 * heads, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)))
    return rc;
  if (rank > 0) {
    if ((rc = map_pos_f32(&tqp, qp, heads, window))) return rc;
    if ((rc = map_pos_f32(&tkp, kp, heads, window))) return rc;
  } else {
    tqp = tq;
    tkp = tq;
  }
  TfParams p{};
  p.B = B; p.H = H; p.W = W; p.heads = heads; p.M = window; p.s = shift; p.rank = rank;
  p.nWx = g.nWx; p.nW = g.nW; p.tiles_x = g.tiles_x; p.n_tiles = g.n_tiles;
  p.scale_log2 = tau * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.wait_limit_ns = g_wait_limit_ns;
  if ((rc = set_smem(attn_fwd_tf32_kernel, kTfSmemBytes))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  TraceScope ts(K_FWD_TF32, st);
  attn_fwd_tf32_kernel<<<dim3(g.n_tiles, g.units), kTfThreads, kTfSmemBytes, st>>>(tq, tv, tqp,
                                                                                   tkp, p);
  return launch_status();
}

int rib_cla_gate(const void* x, int B, int H, int W, int C, const float* w_dw, const float* b_dw,
                 const float* w_pw, const float* b_pw, void* gate, void* stream) {
  int rc = cla_check(B, H, W, C);
  if (rc) return rc;
  if (B == 0) return RIB_OK;   // an empty batch: nothing to compute or write
  if (!x || !w_dw || !b_dw || !w_pw || !b_pw || !gate) return RIB_ERR_ARG;
  if (!aligned16(x) || !aligned16(gate) || (reinterpret_cast<uintptr_t>(w_pw) & 7u) ||
      (reinterpret_cast<uintptr_t>(w_dw) & 3u) || (reinterpret_cast<uintptr_t>(b_dw) & 3u) ||
      (reinterpret_cast<uintptr_t>(b_pw) & 3u))
    return RIB_ERR_ALIGN;
  // x [B][H][W][C] bf16 as a 4D map; box = one tile's 10 x 18 halo, 64 channels
  CUtensorMap tm;
  const uint64_t dims[4] = {(uint64_t)C, (uint64_t)W, (uint64_t)H, (uint64_t)B};
  const uint64_t strides[3] = {2ull * C, 2ull * C * W, 2ull * C * W * H};
  const uint32_t box[4] = {64, 18, 10, 1};
  rc = make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x, dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  ClaParams p{};
  p.w_dw = w_dw; p.b_dw = b_dw; p.w_pw = w_pw; p.b_pw = b_pw;
  p.gate = static_cast<__nv_bfloat16*>(gate);
  p.B = B; p.H = H; p.W = W; p.C = C;
  p.tiles_x = W / 16;
  p.tiles_per_img = (H / 8) * (W / 16);
  const long long n_tiles = (long long)B * p.tiles_per_img;
  if (n_tiles > (1ll << 30)) return RIB_ERR_UNSUPPORTED;
  p.n_tiles = static_cast<int>(n_tiles);
  p.wait_limit_ns = g_wait_limit_ns;
  const size_t smem = cla_smem_bytes(C);
  if ((rc = set_smem(cla_gate_kernel, smem))) return rc;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return RIB_ERR_CUDA;
  const int grid = static_cast<int>(n_tiles < sms ? n_tiles : sms);
  TraceScope ts(K_CLA, static_cast<cudaStream_t>(stream));
  cla_gate_kernel<<<grid, kClaThreads, smem, static_cast<cudaStream_t>(stream)>>>(tm, p);
  return launch_status();
}

size_t rib_cla_bwd_workspace(int B, int H, int W, int C) {
  int sms = 0;
  if (cla_check(B, H, W, C) != RIB_OK || device_sms(&sms) != RIB_OK) return 0;
  return cla_bwd_layout(B, H, W, C, sms).total;
}

int rib_cla_bwd(const void* x, int B, int H, int W, int C, const float* w_dw, const float* b_dw,
                const float* w_pw, const void* gate, const void* out, const void* dout_gated,
                void* dout, void* dx, float* dw_dw, float* db_dw, float* dw_pw, float* db_pw,
                void* workspace, size_t workspace_bytes, void* stream) {
  int rc = cla_check(B, H, W, C);
  if (rc) return rc;
  if (!dw_dw || !db_dw || !dw_pw || !db_pw) return RIB_ERR_ARG;
  if (B == 0) {
    // an empty batch: the weight gradients are empty sums, zero
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(dw_dw, 0, 9ull * C * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(db_dw, 0, (size_t)C * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(dw_pw, 0, (size_t)C * C * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(db_pw, 0, (size_t)C * sizeof(float), st) != cudaSuccess)
      return RIB_ERR_CUDA;
    return RIB_OK;
  }
  if (!x || !w_dw || !b_dw || !w_pw || !gate || !out || !dout_gated || !dout || !dx)
    return RIB_ERR_ARG;
  const void* a16[] = {x, gate, out, dout_gated, dout, dx, dw_pw};
  for (const void* q : a16)
    if (!aligned16(q)) return RIB_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(w_pw) & 7u) || (reinterpret_cast<uintptr_t>(w_dw) & 3u) ||
      (reinterpret_cast<uintptr_t>(b_dw) & 3u) || (reinterpret_cast<uintptr_t>(dw_dw) & 3u) ||
      (reinterpret_cast<uintptr_t>(db_dw) & 3u) || (reinterpret_cast<uintptr_t>(db_pw) & 3u))
    return RIB_ERR_ALIGN;
  int sms = 0;
  if ((rc = device_sms(&sms))) return rc;
  const ClaBwdLayout L = cla_bwd_layout(B, H, W, C, sms);
  if (!workspace || workspace_bytes < L.total) return RIB_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RIB_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  ClaBwdParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.w_dw = w_dw; p.b_dw = b_dw; p.w_pw = w_pw;
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.out = static_cast<const __nv_bfloat16*>(out);
  p.dout_g = static_cast<const __nv_bfloat16*>(dout_gated);
  p.dout = static_cast<__nv_bfloat16*>(dout);
  p.dx = static_cast<__nv_bfloat16*>(dx);
  p.dw_dw = dw_dw; p.db_dw = db_dw; p.dw_pw = dw_pw; p.db_pw = db_pw;
  p.dz = reinterpret_cast<__nv_bfloat16*>(ws + L.dz);
  p.dy = reinterpret_cast<__nv_bfloat16*>(ws + L.dy);
  p.part_dbpw = reinterpret_cast<float*>(ws + L.part_dbpw);
  p.part_dwpw = reinterpret_cast<float*>(ws + L.part_dwpw);
  p.part_dw = reinterpret_cast<float*>(ws + L.part_dw);
  p.B = B; p.H = H; p.W = W; p.C = C;
  p.tiles_x = W / 16;
  p.tiles_per_img = (H / 8) * (W / 16);
  p.n_tiles = L.n_tiles;
  p.tiles_x8 = W / 8;
  p.n_tiles8 = B * (H / 8) * (W / 8);
  p.grid = L.grid;
  p.grid_dx = L.grid_dx;
  p.wait_limit_ns = g_wait_limit_ns;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // x [B][H][W][C] bf16 as a 4D map; box = one tile's 10 x 18 halo, 64 channels
  CUtensorMap tm_x;
  {
    const uint64_t dims[4] = {(uint64_t)C, (uint64_t)W, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {2ull * C, 2ull * C * W, 2ull * C * W * H};
    const uint32_t box[4] = {64, 18, 10, 1};
    rc = make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  // dy (workspace, [B][H][W][C] bf16) as the same kind of map, for the dx kernel
  CUtensorMap tm_dy;
  {
    const uint64_t dims[4] = {(uint64_t)C, (uint64_t)W, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {2ull * C, 2ull * C * W, 2ull * C * W * H};
    const uint32_t box[4] = {64, 18, 10, 1};
    rc = make_map(&tm_dy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.dy, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  // x again with 10 x 10 boxes (the halo of an 8 x 8 tile), and dz
  // (workspace) with 8 x 8 boxes in the 128-byte swizzle, for the dW_pw
  // kernel; dz and dy with 16 x 8 boxes (a 128-pixel tile), for the dy kernel
  CUtensorMap tm_x10, tm_dz, tm_dz16, tm_dy16;
  {
    const uint64_t dims[4] = {(uint64_t)C, (uint64_t)W, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {2ull * C, 2ull * C * W, 2ull * C * W * H};
    const uint32_t box10[4] = {64, 10, 10, 1};
    rc = make_map(&tm_x10, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, x, dims, strides, box10,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    const uint32_t box8[4] = {64, 8, 8, 1};
    rc = make_map(&tm_dz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.dz, dims, strides, box8,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    const uint32_t box16[4] = {64, 16, 8, 1};
    rc = make_map(&tm_dz16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.dz, dims, strides, box16,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    rc = make_map(&tm_dy16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.dy, dims, strides, box16,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  const size_t smem_dy = cla_dy_smem_bytes(C), smem_dw = cla_dwpw_smem_bytes(C);
  const size_t smem_dx = cla_dx_smem_bytes();
  if ((rc = set_smem(cla_bwd_dy_kernel, smem_dy))) return rc;
  if ((rc = set_smem(cla_bwd_dwpw_kernel, smem_dw))) return rc;
  if ((rc = set_smem(cla_bwd_dx_kernel, smem_dx))) return rc;
  {
    TraceScope ts(K_CLA_DZ, st);
    cla_bwd_dz_kernel<<<L.grid, kDzEwThreads, 0, st>>>(p);
    if ((rc = launch_status())) return rc;
  }
  {
    TraceScope ts(K_CLA_DY, st);
    cla_bwd_dy_kernel<<<L.grid, kDyThreads, smem_dy, st>>>(tm_dz16, tm_dy16, p);
    if ((rc = launch_status())) return rc;
  }
  {
    TraceScope ts(K_CLA_DWPW, st);
    cla_bwd_dwpw_kernel<<<L.grid, kDwpwThreads, smem_dw, st>>>(tm_x10, tm_dz, p);
    if ((rc = launch_status())) return rc;
  }
  {
    TraceScope ts(K_CLA_DX, st);
    cla_bwd_dx_kernel<<<L.grid_dx, kClaDxThreads, smem_dx, st>>>(tm_x, tm_dy, p);
    if ((rc = launch_status())) return rc;
  }
  TraceScope ts(K_CLA_RED, st);
  cla_bwd_reduce_kernel<<<(C * C + 11 * C + 31) / 32, 32 * kClaRedWarps, 0, st>>>(p);
  return launch_status();
}

size_t rib_window_attn_bwd_workspace(int B, int H, int W, int heads, int head_dim, int window,
                                     int rank, const rib_mlp_t* mlp) {
  AttnGeom g;
  if (check_attn(B, H, W, heads, head_dim, window, 0, rank, &g) != RIB_OK) return 0;
  if (mlp && check_mlp(mlp) != RIB_OK) return 0;
  return bwd_ws_layout(B, H, W, heads, window, rank, mlp).total;
}

static int attn_bwd_launch(const void* qkv, const void* out, const void* dout,
                           const float* lse, int B, int H, int W, int heads, int head_dim,
                           int window, int shift, const void* qp_bf16, const void* kp_bf16,
                           int rank, float scale, void* dqkv, float* dqp, float* dkp,
                           const rib_mlp_t* mlp, const rib_mlp_grad_t* dmlp, void* workspace,
                           size_t workspace_bytes, int region_mask, void* stream) {
  AttnGeom g;
  int rc = check_attn(B, H, W, heads, head_dim, window, shift, rank, &g);
  if (rc) return rc;
  const bool do_mlp = mlp != nullptr && dmlp != nullptr && rank > 0;
  if (B == 0) {
    // an empty batch: the position-token gradients are empty sums, zero
    if (rank > 0 && (!dqp || !dkp)) return RIB_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t pbytes = sizeof(float) * heads * g.N * rank;
    if (rank > 0 && (cudaMemsetAsync(dqp, 0, pbytes, st) != cudaSuccess ||
                     cudaMemsetAsync(dkp, 0, pbytes, st) != cudaSuccess))
      return RIB_ERR_CUDA;
    if (do_mlp) {
      if ((rc = check_mlp(mlp))) return rc;
      if (!mlp_grad_complete(dmlp)) return RIB_ERR_ARG;
      const size_t din = 4ull * mlp->n_freq, hid = mlp->d_hidden,
                   dout_n = (size_t)mlp->heads * mlp->rank;
      float* const gp[8] = {dmlp->q_dw1, dmlp->q_db1, dmlp->q_dw2, dmlp->q_db2,
                            dmlp->k_dw1, dmlp->k_db1, dmlp->k_dw2, dmlp->k_db2};
      const size_t gn[4] = {hid * din, hid, dout_n * hid, dout_n};
      for (int i = 0; i < 8; ++i)
        if (cudaMemsetAsync(gp[i], 0, gn[i % 4] * sizeof(float), st) != cudaSuccess)
          return RIB_ERR_CUDA;
    }
    return RIB_OK;
  }
  if (!qkv || !out || !dout || !lse || !dqkv) return RIB_ERR_ARG;
  if (rank > 0 && (!qp_bf16 || !kp_bf16 || !dqp || !dkp)) return RIB_ERR_ARG;
  if (do_mlp) {
    if ((rc = check_mlp(mlp))) return rc;
    if (mlp->heads != heads || mlp->rank != rank) return RIB_ERR_ARG;
    if (!mlp_grad_complete(dmlp)) return RIB_ERR_ARG;
  }
  if (!aligned16(qkv) || !aligned16(out) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dqkv) ||
      (rank > 0 && (!aligned16(qp_bf16) || !aligned16(kp_bf16) || !aligned16(dqp) ||
                    !aligned16(dkp))))
    return RIB_ERR_ALIGN;
  const BwdWs ws = bwd_ws_layout(B, H, W, heads, window, rank, do_mlp ? mlp : nullptr);
  if (!workspace || workspace_bytes < ws.total) return RIB_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RIB_ERR_ALIGN;
  if (!std::isfinite(scale)) return RIB_ERR_ARG;
  const float tau = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(head_dim + rank));
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  BwdAuxParams a{};
  a.B = B; a.H = H; a.W = W; a.heads = heads; a.M = window; a.s = shift;
  a.nWx = g.nWx; a.nW = g.nW; a.tiles_x = g.tiles_x; a.n_tiles = g.n_tiles; a.rank = rank;
  a.scale = tau;
  a.out = static_cast<const __nv_bfloat16*>(out);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.lse = lse;
  a.lse2 = reinterpret_cast<float*>(wsb + ws.lse2);
  a.dd = reinterpret_cast<float*>(wsb + ws.dd);
  a.dq_acc = reinterpret_cast<float*>(wsb + ws.dq_acc);
  a.dkp_part = reinterpret_cast<const float*>(wsb + ws.dkp_part);
  a.dq_acc_floats = (size_t)B * H * W * heads * 48;
  a.dqkv = static_cast<__nv_bfloat16*>(dqkv);
  a.dq_v8 = (reinterpret_cast<uintptr_t>(dqkv) & 31u) == 0 ? 1 : 0;
  a.dqp = dqp;
  a.dkp = dkp;

  CUtensorMap tq, tdo, tqp, tkp, tl, td;
  if ((rc = map_tokens(&tq, qkv, B, H, W, 3 * heads))) return rc;
  if ((rc = map_tokens(&tdo, dout, B, H, W, heads))) return rc;
  if ((rc = map_pixel_f32(&tl, a.lse2, B, heads, H, W))) return rc;
  if ((rc = map_pixel_f32(&td, a.dd, B, heads, H, W))) return rc;
  if (rank > 0) {
    if ((rc = map_pos_padded(&tqp, qp_bf16, heads, window))) return rc;
    if ((rc = map_pos_padded(&tkp, kp_bf16, heads, window))) return rc;
  } else {
    tqp = tq;
    tkp = tq;
  }

  {
    const size_t n = (size_t)B * heads * H * W;
    int blocks = static_cast<int>((n + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    TraceScope ts(K_BWD_PRE, st);
    bwd_preprocess_kernel<<<blocks, 256, 0, st>>>(a);
    if ((rc = launch_status())) return rc;
  }
  BwdParams p{};
  p.region_mask = region_mask != 0 && shift > 0;
  p.B = B; p.H = H; p.W = W; p.heads = heads; p.M = window; p.s = shift; p.rank = rank;
  p.nWx = g.nWx; p.nW = g.nW; p.tiles_x = g.tiles_x; p.n_tiles = g.n_tiles;
  p.scale = tau;
  p.scale_log2 = tau * 1.4426950408889634f;
  p.dqkv = a.dqkv;
  p.dqkv_v8 = a.dq_v8;
  p.dq_acc = a.dq_acc;
  p.dkp_part = reinterpret_cast<float*>(wsb + ws.dkp_part);
  p.n_items = g.units * g.n_tiles;
  p.wait_limit_ns = g_wait_limit_ns;
  // Both forms move registers between warpgroups with setmaxnreg, which is
  // only safe if the compiled launch budget is the one the split assumes.
  static std::atomic<int> launch_regs[4] = {{-1}, {-1}, {-1}, {-1}};
  if (rib_bwd_kernel_for(window) == RIB_BWD_PERSISTENT) {
    auto* kern = p.region_mask ? pbwd::attn_bwd_persistent_kernel<true>
                               : pbwd::attn_bwd_persistent_kernel<false>;
    if ((rc = set_smem(kern, pbwd::kPBwdSmemBytes))) return rc;
    if ((rc = check_launch_regs(reinterpret_cast<const void*>(kern),
                                launch_regs[2 + (p.region_mask ? 1 : 0)], kBwdLaunchRegs)))
      return rc;
    // one CTA per SM walks the work items (unit, key tile)
    int sms = 0;
    if ((rc = device_sms(&sms))) return rc;
    TraceScope ts(K_BWD_PERSIST, st);
    kern<<<std::min(p.n_items, sms), kBwdThreads, pbwd::kPBwdSmemBytes, st>>>(tq, tdo, tqp, tkp,
                                                                             tl, td, p);
  } else {
    auto* kern = p.region_mask ? attn_bwd_kernel<true> : attn_bwd_kernel<false>;
    if ((rc = set_smem(kern, kBwdSmemBytes))) return rc;
    if ((rc = check_launch_regs(reinterpret_cast<const void*>(kern),
                                launch_regs[p.region_mask ? 1 : 0], kBwdLaunchRegs)))
      return rc;
    TraceScope ts(K_BWD, st);
    kern<<<dim3(g.n_tiles, g.units), kBwdThreads, kBwdSmemBytes, st>>>(tq, tdo, tqp, tkp, tl,
                                                                       td, p);
  }
  if ((rc = launch_status())) return rc;
  {
    const size_t n = (size_t)g.units * g.N;
    TraceScope ts(K_DQ_FIN, st);
    dq_finalize_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(a);
    if ((rc = launch_status())) return rc;
  }
  if (rank > 0) {
    const size_t n = (size_t)heads * g.N * rank;
    // about 48 units or fewer per warp: 16 warps per output group for the
    // 1152 units of 16 x 16 windows on a batch-8 192 x 192 map, one for 16
    const int units_bw = B * g.nW;
    a.pg_chunks = 1;
    while (a.pg_chunks < kPgWarps && units_bw > 48 * a.pg_chunks) a.pg_chunks *= 2;
    const size_t per_block = static_cast<size_t>(kPgBlockOut / a.pg_chunks);
    int sms = 0;
    if ((rc = device_sms(&sms))) return rc;
    const size_t passes = (n + per_block - 1) / per_block;
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>(passes, 4ull * sms));
    TraceScope ts(K_POSGRAD, st);
    posgrad_reduce_kernel<<<dim3(blocks, 2), 32 * kPgWarps, 0, st>>>(a);
    if ((rc = launch_status())) return rc;
  }
  if (do_mlp) {
    if ((rc = launch_mlp_bwd(mlp, window, dqp, dkp, dmlp, wsb + ws.mlp_part, ws.n_chunks,
                             ws.n_params, st)))
      return rc;
  }
  return RIB_OK;
}

int rib_window_attn_bwd(const void* qkv, const void* out, const void* dout, const float* lse,
                        int B, int H, int W, int heads, int head_dim, int window, int shift,
                        const void* qp_bf16, const void* kp_bf16, int rank, float scale,
                        void* dqkv, float* dqp, float* dkp, const rib_mlp_t* mlp,
                        const rib_mlp_grad_t* dmlp, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return attn_bwd_launch(qkv, out, dout, lse, B, H, W, heads, head_dim, window, shift, qp_bf16,
                         kp_bf16, rank, scale, dqkv, dqp, dkp, mlp, dmlp, workspace,
                         workspace_bytes, 0, stream);
}

int rib_window_attn_bwd_masked(const void* qkv, const void* out, const void* dout,
                               const float* lse, int B, int H, int W, int heads, int head_dim,
                               int window, int shift, const void* qp_bf16, const void* kp_bf16,
                               int rank, float scale, void* dqkv, float* dqp, float* dkp,
                               const rib_mlp_t* mlp, const rib_mlp_grad_t* dmlp,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return attn_bwd_launch(qkv, out, dout, lse, B, H, W, heads, head_dim, window, shift, qp_bf16,
                         kp_bf16, rank, scale, dqkv, dqp, dkp, mlp, dmlp, workspace,
                         workspace_bytes, 1, stream);
}

static int window_copy(const void* src, void* dst, int B, int H, int W, int C, int eb, int M,
                       int s, int gather, void* stream) {
  if (B < 0 || H <= 0 || W <= 0 || C <= 0 || M <= 0) return RIB_ERR_ARG;
  if (eb != 1 && eb != 2 && eb != 4) return RIB_ERR_ARG;
  if (H % M != 0 || W % M != 0 || s < 0 || s >= M) return RIB_ERR_SHAPE;
  if (M % 8 != 0 || s % 8 != 0 || ((long long)C * eb) % 16 != 0) return RIB_ERR_UNSUPPORTED;
  if (B == 0) return RIB_OK;   // an empty batch: nothing to copy
  if (!src || !dst) return RIB_ERR_ARG;
  if (!aligned16(src) || !aligned16(dst)) return RIB_ERR_ALIGN;
  const int nW = (H / M) * (W / M);
  if (nW > 65535 || B > 65535) return RIB_ERR_UNSUPPORTED;
  int cc = 0;
  for (int c = 1; c <= C && c <= 256; ++c)
    if (C % c == 0 && (c * eb) % 16 == 0 && c * eb <= 512) cc = c;
  if (cc == 0) return RIB_ERR_UNSUPPORTED;
  const CUtensorMapDataType dt = eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                           : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  const void* xmap_base = gather ? src : dst;
  const void* wmap_base = gather ? dst : src;
  CUtensorMap mx, mw;
  const uint64_t ce = (uint64_t)C * eb;
  const uint64_t dx[4] = {(uint64_t)C, (uint64_t)W, (uint64_t)H, (uint64_t)B};
  const uint64_t sx[3] = {ce, ce * W, ce * W * H};
  const uint64_t dw[4] = {(uint64_t)C, (uint64_t)M, (uint64_t)M, (uint64_t)B * nW};
  const uint64_t sw[3] = {ce, ce * M, ce * M * M};
  const uint32_t box[4] = {(uint32_t)cc, 8, 8, 1};
  int rc;
  if ((rc = make_map(&mx, dt, 4, xmap_base, dx, sx, box, CU_TENSOR_MAP_SWIZZLE_NONE))) return rc;
  if ((rc = make_map(&mw, dt, 4, wmap_base, dw, sw, box, CU_TENSOR_MAP_SWIZZLE_NONE))) return rc;
  CopyParams p{};
  p.B = B; p.H = H; p.W = W; p.M = M; p.s = s; p.nWx = W / M; p.nW = nW; p.boxes_x = M / 8;
  p.cc = cc;
  p.n_chunks = C / cc;
  p.box_bytes = static_cast<uint32_t>(cc * eb * 64);
  p.gather = gather;
  p.wait_limit_ns = g_wait_limit_ns;
  const size_t smem = 2ull * p.box_bytes + 1024;
  if ((rc = set_smem(window_copy_kernel, smem))) return rc;
  dim3 grid((M / 8) * (M / 8), nW, B);
  TraceScope ts(K_COPY, static_cast<cudaStream_t>(stream));
  window_copy_kernel<<<grid, 32, smem, static_cast<cudaStream_t>(stream)>>>(mx, mw, p);
  return launch_status();
}

int rib_window_gather(const void* x, int B, int H, int W, int C, int elem_bytes, int window,
                      int shift, void* xw, void* stream) {
  return window_copy(x, xw, B, H, W, C, elem_bytes, window, shift, 1, stream);
}

int rib_window_scatter(const void* xw, int B, int H, int W, int C, int elem_bytes, int window,
                       int shift, void* x, void* stream) {
  return window_copy(xw, x, B, H, W, C, elem_bytes, window, shift, 0, stream);
}

}  // extern "C"
