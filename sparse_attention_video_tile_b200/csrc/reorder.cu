// reorder.cu - raster <-> tiled token reorder (HBM-bound gather).
//
// Tiled order makes the tokens of each non-overlapping (tt, th, tw) tile
// contiguous ("Fast Video Generation with Sliding Tile Attention", summary
// page, "Method details").  The copy is organised in runs: the tw tokens of
// one tile row (fixed batch*head, tile, t and h inside the tile) are
// contiguous in both orders, so each run is one contiguous block of tw*d*2
// bytes on both sides.  A warp copies a run with 16-byte vector loads and
// stores; index arithmetic happens once per run, not per element.
#include <cuda_runtime.h>

#include "internal.h"

namespace sta {
namespace {

struct RunGeo {
  int64_t n_runs;          // batch_heads * L / tw
  int32_t runs_per_bh;     // L / tw
  int32_t runs_per_tile;   // tt * th
  int32_t th, tw, tt;
  int32_t nH, nW;
  int32_t H, W;
  int32_t ntile;
  int64_t L;
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <int CPR>  // 16-byte chunks per token row (d * 2 / 16)
__global__ void __launch_bounds__(256) reorder_kernel(const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, RunGeo g,
                                                      int to_tiled) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int chunks = g.tw * CPR;
  for (int64_t r = warp0; r < g.n_runs; r += nwarps) {
    const int64_t bh = r / g.runs_per_bh;
    const int32_t rr = static_cast<int32_t>(r - bh * g.runs_per_bh);
    const int32_t tile_id = rr / g.runs_per_tile;
    const int32_t rem = rr - tile_id * g.runs_per_tile;
    const int32_t lt = rem / g.th;
    const int32_t lh = rem - lt * g.th;
    const int32_t at = tile_id / (g.nH * g.nW);
    const int32_t ah = (tile_id / g.nW) % g.nH;
    const int32_t aw = tile_id % g.nW;
    const int64_t tiled_row = bh * g.L + static_cast<int64_t>(tile_id) * g.ntile + (lt * g.th + lh) * g.tw;
    const int64_t raster_row =
        bh * g.L + (static_cast<int64_t>(at * g.tt + lt) * g.H + (ah * g.th + lh)) * g.W + aw * g.tw;
    const uint4* s = src + (to_tiled ? raster_row : tiled_row) * CPR;
    uint4* d = dst + (to_tiled ? tiled_row : raster_row) * CPR;
    for (int base = 0; base < chunks; base += 4 * 32) {
      uint4 buf[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 32 + lane;
        if (i < chunks) buf[u] = ld_stream(s + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 32 + lane;
        if (i < chunks) d[i] = buf[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_reorder(const void* src, void* dst, int64_t batch_heads, int32_t d,
                           const Geometry& geo, bool to_tiled, cudaStream_t stream) {
  RunGeo g;
  g.runs_per_bh = static_cast<int32_t>(geo.L / geo.tw);
  g.n_runs = batch_heads * g.runs_per_bh;
  g.runs_per_tile = geo.tt * geo.th;
  g.th = geo.th; g.tw = geo.tw; g.tt = geo.tt;
  g.nH = geo.nH; g.nW = geo.nW;
  g.H = geo.H; g.W = geo.W;
  g.ntile = geo.ntile;
  g.L = geo.L;
  if (g.n_runs == 0) return cudaSuccess;

  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int threads = 256;
  const int64_t warps_needed = g.n_runs;
  int64_t blocks = (warps_needed + 7) / 8;
  const int64_t max_blocks = static_cast<int64_t>(sms) * 8;  // 8 x 256 threads fill an SM
  if (blocks > max_blocks) blocks = max_blocks;
  const uint4* s = static_cast<const uint4*>(src);
  uint4* dd = static_cast<uint4*>(dst);
  if (d == 128)
    reorder_kernel<16><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(s, dd, g, to_tiled ? 1 : 0);
  else
    reorder_kernel<8><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(s, dd, g, to_tiled ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace sta
