// internal.h - declarations shared by the library's translation units.
#pragma once

#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/sta.h"

namespace sta {

// Tile geometry derived from (grid, tile).
struct Geometry {
  int32_t T, H, W;        // grid in tokens
  int32_t tt, th, tw;     // tile in tokens
  int32_t nT, nH, nW;     // tile grid (of the padded latent when padded)
  int32_t ntile;          // tokens per tile
  int64_t L;              // real tokens T * H * W
  int64_t Lpad;           // rows of the tiled order: nT * nH * nW * ntile (= L unless padded)
  bool padded;            // grid is not a tile multiple
};

// Validates and fills a Geometry; the grid must be a tile multiple.
// STA_OK or STA_ERR_SHAPE.
sta_status make_geometry(sta_dim3 grid, sta_dim3 tile, Geometry* g);

// Same, but a grid that is not a tile multiple is padded up to the next multiple
// ("padding with masking").
sta_status make_geometry_padded(sta_dim3 grid, sta_dim3 tile, Geometry* g);

// One unit of work of the attention kernel: a block of 128 query rows of one
// (batch, head), with the list of 128-key blocks it attends.
struct WorkItem {
  int32_t bh;       // batch * heads + head
  int32_t q_row0;   // first query row (tiled order)
  int32_t kv_off;   // offset of its key-block list in the schedule's kv_rows
  int32_t kv_len;   // number of key blocks
};

// Host schedule produced by the window enumerator.
struct HostSchedule {
  bool masked = false;                 // Ntile is not a multiple of 128: tile-granular masking in-kernel
  std::vector<WorkItem> items;         // sorted by decreasing cost (kv_len), stable
  std::vector<int32_t> kv_rows;        // first row (tiled order) of each 128-key block
  std::vector<int16_t> head_win;       // [heads][4]: effective window (t, h, w), 0
  // Padded latents only: per entry of kv_rows, -1 if every key of the block is a real
  // token, else the index of a 128-bit validity mask (4 words, bit i = key i is real).
  std::vector<int32_t> kv_mask_id;
  std::vector<uint32_t> kv_masks;
  int64_t attended_pairs = 0;
};

constexpr int kBlockRows = 128;   // query rows per work item and keys per key block

// Window enumerator: per head, per block of 128 query rows, the key blocks of
// the window (see schedule.cpp).
void build_schedule(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                    HostSchedule* out);

// Window enumerator of the raster-order kernel: Ntile must be a multiple of 128 and
// the grid may be padded.  Key blocks without real tokens are left out, partly
// padded ones get a validity mask, and query blocks without real rows get no item.
void build_schedule_raster(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                           HostSchedule* out);

// The same windows seen from the key side, for the backward pass: one item per
// (batch, head, block of 128 key rows) with the list of 128-row query blocks that
// attend it (stored in kv_rows).  Ntile must be a multiple of 128.
void build_schedule_transposed(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                               HostSchedule* out);

// Whether a tile splits into 128-row slabs of whole frames (th * tw divides 128 and
// tt is a multiple of 128 / (th * tw)): the raster-order kernel loads each slab as
// one TMA box.
inline bool raster_tile_ok(int32_t tt, int32_t th, int32_t tw) {
  const int32_t plane = th * tw;
  return plane > 0 && plane <= kBlockRows && kBlockRows % plane == 0 && tt % (kBlockRows / plane) == 0;
}

// Effective window start (first tile) in one dimension.
inline int32_t window_start_1d(int32_t a, int32_t weff, int32_t n) {
  int32_t s = a - weff / 2;
  if (s < 0) s = 0;
  if (s > n - weff) s = n - weff;
  return s;
}

// Kernel launchers (reorder.cu, attention.cu).
// token_major_heads > 0: the raster side is [B, L, heads, d] with that many
// heads (batch_heads must then be B * heads); 0: it is [B * heads, L, d].
cudaError_t launch_reorder(const void* src, void* dst, int64_t batch_heads, int32_t d,
                           const Geometry& g, bool to_tiled, cudaStream_t stream,
                           int32_t token_major_heads = 0);

// Raster [BH, T*H*W, d] -> tiled order of the padded latent [BH, Lpad, d], the
// rows of pad tokens written as zeros (reorder.cu).
cudaError_t launch_reorder_padded(const void* src, void* dst, int64_t batch_heads, int32_t d, const Geometry& g,
                                  cudaStream_t stream);

struct DeviceSchedule {
  const WorkItem* items;
  const int32_t* kv_rows;
  const int16_t* head_win;
  int32_t n_items;
  bool masked;
  const int32_t* kv_mask_id = nullptr;   // padded latents only
  const uint32_t* kv_masks = nullptr;
  int32_t n_kv_rows = 0;                 // entries of kv_rows (for the device checks)
  int32_t n_masks = 0;                   // 128-bit masks in kv_masks
};

// Attention on tiled-order tensors ([BH, L, d]); lse, when not null, receives
// each row's log-sum-exp ([BH, L] fp32, tiled order).
cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out,
                             int32_t batch, int32_t heads, int32_t d, const Geometry& g,
                             const DeviceSchedule& s, float scale, int32_t* err_flag,
                             uint64_t limit_ns, cudaStream_t stream, float* lse = nullptr);

// Attention on raster-order tensors ([BH, T, H, W, d]): the tile reorder is done by
// the TMA loads and the epilogue's addressing; pad tokens read as zeros.
cudaError_t launch_attention_raster(const void* q, const void* k, const void* v, void* out,
                                    int32_t batch, int32_t heads, int32_t d, const Geometry& g,
                                    const DeviceSchedule& s, float scale, int32_t* err_flag,
                                    uint64_t limit_ns, cudaStream_t stream);

// Attention with raster-order q and out ([BH, T, H, W, d], as the raster launcher)
// and k, v in the tiled order of the padded latent ([BH, Lpad, d], pad rows zero,
// as launch_reorder_padded writes them).
cudaError_t launch_attention_mixed(const void* q, const void* k_tiled, const void* v_tiled, void* out,
                                   int32_t batch, int32_t heads, int32_t d, const Geometry& g,
                                   const DeviceSchedule& s, float scale, int32_t* err_flag,
                                   uint64_t limit_ns, cudaStream_t stream);

// Backward pass on tiled-order tensors: D = rowsum(dout * out) into dvec ([BH, L]
// fp32 scratch), then dq over the forward schedule and dk, dv over the transposed
// one (backward.cu).  Ntile must be a multiple of 128.
cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                            const float* lse, float* dvec, void* dq, void* dk, void* dv, int32_t batch,
                            int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& fwd,
                            const DeviceSchedule& tr, float scale, int32_t* err_flag, uint64_t limit_ns,
                            cudaStream_t stream);

cudaError_t launch_selftest_wait(int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream);

// Records the text of a failed CUDA call for sta_last_cuda_error and returns
// STA_ERR_CUDA (api.cu).
sta_status cuda_fail(cudaError_t e);

// The no-alloc entry point's status word on device `dev` (a device address inside
// its static scratch array), or null while that entry point has not been set up on
// the device (noalloc.cu).
int32_t* noalloc_status_word(int dev);

// Forgets every device's no-alloc set-up (scratch address and uploaded schedule),
// so that the next call on a device looks the address up and uploads again
// (noalloc.cu).  Called by sta_shutdown.
void noalloc_reset();

}  // namespace sta
