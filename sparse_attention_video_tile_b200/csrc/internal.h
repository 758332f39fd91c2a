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
  int32_t nT, nH, nW;     // tile grid
  int32_t ntile;          // tokens per tile
  int64_t L;              // tokens
};

// Validates and fills a Geometry; STA_OK or STA_ERR_SHAPE.
sta_status make_geometry(sta_dim3 grid, sta_dim3 tile, Geometry* g);

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
  int64_t attended_pairs = 0;
};

constexpr int kBlockRows = 128;   // query rows per work item and keys per key block

// Window enumerator: per head, per block of 128 query rows, the key blocks of
// the window (see schedule.cpp).
void build_schedule(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                    HostSchedule* out);

// Effective window start (first tile) in one dimension.
inline int32_t window_start_1d(int32_t a, int32_t weff, int32_t n) {
  int32_t s = a - weff / 2;
  if (s < 0) s = 0;
  if (s > n - weff) s = n - weff;
  return s;
}

// Kernel launchers (reorder.cu, attention.cu).
cudaError_t launch_reorder(const void* src, void* dst, int64_t batch_heads, int32_t d,
                           const Geometry& g, bool to_tiled, cudaStream_t stream);

struct DeviceSchedule {
  const WorkItem* items;
  const int32_t* kv_rows;
  const int16_t* head_win;
  int32_t n_items;
  bool masked;
};

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out,
                             int32_t batch, int32_t heads, int32_t d, const Geometry& g,
                             const DeviceSchedule& s, float scale, int32_t* err_flag,
                             uint64_t limit_ns, cudaStream_t stream);

cudaError_t launch_selftest_wait(int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream);

}  // namespace sta
