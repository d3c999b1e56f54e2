// window_copy.cuh -- window partition with cyclic shift as a pure TMA copy.
//
// The shifted-window partition (roll the map by -s, cut M x M windows) done
// with the same rolled box addressing the attention kernels use: every
// 8 x 8-pixel box of a window is loaded by TMA from its rolled map position
// and stored by TMA to the window-contiguous tensor (gather), or the other
// way round (scatter).  No arithmetic touches the data: bit-exact.
//
// Tensor maps (built on the host):
//   map_x : [B][H][W][C]      dims {C, W, H, B}, box {cc, 8, 8, 1}
//   map_w : [B*nW][M][M][C]   dims {C, M, M, B*nW}, box {cc, 8, 8, 1}
// cc divides C, cc <= 256, cc * elem_bytes % 16 == 0.
#pragma once

#include "geom.cuh"
#include "ptx.cuh"

namespace rib {

struct CopyParams {
  int B, H, W, M, s, nWx, nW, boxes_x;  // boxes_x = M / 8
  int cc;                               // channels per TMA box
  int n_chunks;                         // C / cc
  uint32_t box_bytes;                   // cc * 64 * elem_bytes
  int gather;                           // 1: map -> windows, 0: windows -> map
  uint64_t wait_limit_ns;
};

constexpr uint64_t kDrainLimitNs = 200ull * 1000ull * 1000ull;  // 200 ms

// grid ((M/8)^2, nW, B); one warp, lane 0 streams the channel chunks of one
// 8 x 8 box through two shared-memory slots (load k+1 overlaps store k).
__global__ void __launch_bounds__(32) window_copy_kernel(const __grid_constant__ CUtensorMap map_x,
                                                         const __grid_constant__ CUtensorMap map_w,
                                                         const CopyParams p) {
  extern __shared__ uint8_t sm_copy_raw[];
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar[0], 1);
  mbar_init(&bar[1], 1);
  fence_mbarrier_init();
  const int box = blockIdx.x, w = blockIdx.y, b = blockIdx.z;
  const int bi = box / p.boxes_x, bj = box - bi * p.boxes_x;
  const int wy = w / p.nWx, wx = w - wy * p.nWx;
  const int i0 = bi * 8, j0 = bj * 8;
  const int y = wrap_once(wy * p.M + i0 + p.s, p.H);
  const int x = wrap_once(wx * p.M + j0 + p.s, p.W);
  const int uw = b * p.nW + w;
  // TMA boxes start on 1024-byte boundaries (box_bytes is a multiple of 1024)
  uint8_t* sm_copy = align1024<uint8_t>(sm_copy_raw);
  uint8_t* buf[2] = {sm_copy, sm_copy + p.box_bytes};
  auto load = [&](int k) {
    const int slot = k & 1;
    mbar_arrive_expect_tx(&bar[slot], p.box_bytes);
    if (p.gather) tma_load_4d(buf[slot], &map_x, &bar[slot], k * p.cc, x, y, b);
    else          tma_load_4d(buf[slot], &map_w, &bar[slot], k * p.cc, j0, i0, uw);
  };
  load(0);
  int waited = 0;  // loads whose completion has been observed
  for (int k = 0; k < p.n_chunks; ++k) {
    const int slot = k & 1;
    if (!mbar_wait(&bar[slot], (k >> 1) & 1, &abort_flag, p.wait_limit_ns, SITE_COPY)) break;
    waited = k + 1;
    if (k + 1 < p.n_chunks) {
      // slot (k+1)&1 was last read by the store of chunk k-1
      tma_store_wait_read_all();
      load(k + 1);
    }
    if (p.gather) tma_store_4d(&map_w, buf[slot], k * p.cc, j0, i0, uw);
    else          tma_store_4d(&map_x, buf[slot], k * p.cc, x, y, b);
    tma_store_commit();
  }
  // after a timeout: let the loads still in flight land before the CTA exits
  const int issued = waited + 1 < p.n_chunks ? waited + 1 : p.n_chunks;
  for (int k = waited; k < issued; ++k) {
    volatile int no_abort = 0;
    mbar_wait(&bar[k & 1], (k >> 1) & 1, &no_abort, kDrainLimitNs, SITE_COPY);
  }
  tma_store_wait_all();
}

}  // namespace rib
