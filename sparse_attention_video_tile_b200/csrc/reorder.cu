// reorder.cu - raster <-> tiled token reorder (HBM-bound gather).
//
// Tiled order makes the tokens of each non-overlapping (tt, th, tw) tile
// contiguous ("Fast Video Generation with Sliding Tile Attention", summary
// page, "Method details").  The copy is organised in runs: the tw tokens of
// one tile row (fixed batch*head, tile, t and h inside the tile) are
// contiguous in both orders, so each run is one contiguous block of tw*d*2
// bytes on both sides.  A warp copies a run with 16-byte vector loads and
// stores; index arithmetic happens once per run, not per element.
//
// Padded variant (raster -> tiled only): for a latent that is not a tile
// multiple, the tiled side has the rows of the padded latent (the tile grid
// rounded up), and the rows of pad tokens are written as zeros.
//
// Token-major variant: the raster side is [B, L, heads, d], the layout of a
// [B, L, heads * d] projection in a video transformer, and the tiled side is
// [B, heads, L, d].  A run is then tw token rows heads * d elements apart on
// the raster side, still one contiguous block on the tiled side; runs of the
// same tile row and neighbouring heads go to neighbouring warps, so together
// they read or write the raster rows whole.
#include <cuda_runtime.h>

#include "internal.h"

namespace sta {
namespace {

struct RunGeo {
  int64_t n_runs;          // batch_heads * L / tw (padded: batch_heads * Lpad / tw)
  int32_t runs_per_bh;     // L / tw
  int32_t runs_per_tile;   // tt * th
  int32_t th, tw, tt;
  int32_t nH, nW;
  int32_t H, W;
  int32_t ntile;
  int64_t L;
  int32_t heads;           // token-major only
  int32_t T;               // padded only: grid
  int64_t Lpad;            // padded only: rows of the tiled side per batch*head
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// CPR: 16-byte chunks per token row (d * 2 / 16).  kTokenMajor: the raster
// side is [B, L, heads, d] instead of [B, heads, L, d].
template <int CPR, bool kTokenMajor>
__global__ void __launch_bounds__(256, 6) reorder_kernel(const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, RunGeo g,
                                                      int to_tiled) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int chunks = g.tw * CPR;
  for (int64_t r = warp0; r < g.n_runs; r += nwarps) {
    int64_t bh, b = 0;
    int32_t rr, head = 0;
    if (kTokenMajor) {  // run index = (b * runs_per_bh + rr) * heads + head
      const int64_t br = r / g.heads;
      head = static_cast<int32_t>(r - br * g.heads);
      b = br / g.runs_per_bh;
      rr = static_cast<int32_t>(br - b * g.runs_per_bh);
      bh = b * g.heads + head;
    } else {            // run index = bh * runs_per_bh + rr
      bh = r / g.runs_per_bh;
      rr = static_cast<int32_t>(r - bh * g.runs_per_bh);
    }
    const int32_t tile_id = rr / g.runs_per_tile;
    const int32_t rem = rr - tile_id * g.runs_per_tile;
    const int32_t lt = rem / g.th;
    const int32_t lh = rem - lt * g.th;
    const int32_t at = tile_id / (g.nH * g.nW);
    const int32_t ah = (tile_id / g.nW) % g.nH;
    const int32_t aw = tile_id % g.nW;
    const int64_t tiled_row = bh * g.L + static_cast<int64_t>(tile_id) * g.ntile + (lt * g.th + lh) * g.tw;
    const int64_t n0 = (static_cast<int64_t>(at * g.tt + lt) * g.H + (ah * g.th + lh)) * g.W + aw * g.tw;
    // raster side: token row j of the run starts at (raster_row + j * rstride) * CPR
    const int64_t raster_row = kTokenMajor ? (b * g.L + n0) * g.heads + head : bh * g.L + n0;
    const int64_t rstride = kTokenMajor ? g.heads : 1;
    const uint4* s = src + (to_tiled ? raster_row : tiled_row) * CPR;
    uint4* d = dst + (to_tiled ? tiled_row : raster_row) * CPR;
    for (int base = 0; base < chunks; base += 4 * 32) {
      uint4 buf[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 32 + lane;
        const int64_t ri = (i / CPR) * rstride * CPR + (i % CPR);
        if (i < chunks) buf[u] = ld_stream(s + (to_tiled ? ri : i));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 32 + lane;
        const int64_t ri = (i / CPR) * rstride * CPR + (i % CPR);
        if (i < chunks) d[to_tiled ? i : ri] = buf[u];
      }
    }
  }
}

// Raster [BH, T*H*W, d] -> padded tiled [BH, Lpad, d], pad rows zero.  Same
// runs as reorder_kernel over the padded tile grid; a run (tw tokens of one tile
// row) reads only the tokens inside the grid.
template <int CPR>
__global__ void __launch_bounds__(256, 6) reorder_padded_kernel(const uint4* __restrict__ src,
                                                             uint4* __restrict__ dst, RunGeo g) {
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
    const int64_t tiled_row = bh * g.Lpad + static_cast<int64_t>(tile_id) * g.ntile + (lt * g.th + lh) * g.tw;
    const int32_t t = at * g.tt + lt, h = ah * g.th + lh, w0 = aw * g.tw;
    // real tokens of the run: w0 .. w0 + real - 1
    const int32_t real = (t < g.T && h < g.H) ? min(g.tw, max(g.W - w0, 0)) : 0;
    const int64_t n0 = (static_cast<int64_t>(t) * g.H + h) * g.W + w0;
    const uint4* sp = src + (bh * g.L + n0) * CPR;
    uint4* dp = dst + tiled_row * CPR;
    for (int base = 0; base < chunks; base += 4 * 32) {
      uint4 buf[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 32 + lane;
        buf[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < chunks && i / CPR < real) buf[u] = ld_stream(sp + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 32 + lane;
        if (i < chunks) dp[i] = buf[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_reorder_padded(const void* src, void* dst, int64_t batch_heads, int32_t d, const Geometry& geo,
                                  cudaStream_t stream) {
  RunGeo g;
  g.heads = 0;
  g.runs_per_bh = static_cast<int32_t>(geo.Lpad / geo.tw);
  g.n_runs = batch_heads * g.runs_per_bh;
  g.runs_per_tile = geo.tt * geo.th;
  g.th = geo.th; g.tw = geo.tw; g.tt = geo.tt;
  g.nH = geo.nH; g.nW = geo.nW;
  g.H = geo.H; g.W = geo.W; g.T = geo.T;
  g.ntile = geo.ntile;
  g.L = geo.L;
  g.Lpad = geo.Lpad;
  if (g.n_runs == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  int64_t blocks = (g.n_runs + 7) / 8;
  const int64_t max_blocks = static_cast<int64_t>(sms) * 8;
  if (blocks > max_blocks) blocks = max_blocks;
  const uint4* s = static_cast<const uint4*>(src);
  uint4* dd = static_cast<uint4*>(dst);
  if (d == 128) reorder_padded_kernel<16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(s, dd, g);
  else reorder_padded_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(s, dd, g);
  return cudaGetLastError();
}

cudaError_t launch_reorder(const void* src, void* dst, int64_t batch_heads, int32_t d,
                           const Geometry& geo, bool to_tiled, cudaStream_t stream, int32_t token_major_heads) {
  RunGeo g;
  g.heads = token_major_heads;
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
  const unsigned nb = static_cast<unsigned>(blocks);
  const int tt = to_tiled ? 1 : 0;
  if (token_major_heads > 0) {
    if (d == 128) reorder_kernel<16, true><<<nb, threads, 0, stream>>>(s, dd, g, tt);
    else reorder_kernel<8, true><<<nb, threads, 0, stream>>>(s, dd, g, tt);
  } else {
    if (d == 128) reorder_kernel<16, false><<<nb, threads, 0, stream>>>(s, dd, g, tt);
    else reorder_kernel<8, false><<<nb, threads, 0, stream>>>(s, dd, g, tt);
  }
  return cudaGetLastError();
}

}  // namespace sta
