// api.cu - the C ABI declared in include/sta.h: argument validation, the
// schedule cache, the device status word, and the kernel launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <list>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "internal.h"

namespace sta {
namespace {

thread_local std::string g_last_cuda_error;

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per bounded wait

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, const void* b, int64_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + static_cast<uintptr_t>(bytes) && y < x + static_cast<uintptr_t>(bytes);
}

// Device check: compute capability 10.0 (B200, sm_100a code).
sta_status check_device(int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return cuda_fail(e);
  if (major != 10 || minor != 0) return STA_ERR_ARCH;
  if (dev_out) *dev_out = dev;
  return STA_OK;
}

// ---------------------------------------------------------------- per-device state

struct CachedSchedule {
  HostSchedule host;
  WorkItem* d_items = nullptr;
  int32_t* d_kv_rows = nullptr;
  int16_t* d_head_win = nullptr;
  int32_t* d_kv_mask_id = nullptr;   // padded raster schedules only
  uint32_t* d_kv_masks = nullptr;
};

// (kind, batch, heads, T, H, W, tt, th, tw, windows); kind 0 = tiled order, 1 = raster
// order (padded), 2 = transposed (key blocks with their query blocks, for the backward)
using ScheduleKey = std::tuple<int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t,
                               std::vector<int32_t>>;

// Streams, events and chunk buffers of sta_forward_host (two slots of chunk buffers:
// q, k, v and out in raster order, k and v in the padded tiled order).
struct HostPipe {
  cudaStream_t s_in = nullptr, s_run = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, copied[2] = {nullptr, nullptr}, computed[2] = {nullptr, nullptr},
              drained[2] = {nullptr, nullptr};
  uint8_t* buf = nullptr;
  size_t bytes = 0;
};

struct DeviceState {
  HostPipe pipe;
  int32_t* d_err = nullptr;  // bounded-wait status word
  float* d_dvec = nullptr;   // backward scratch: one float per query row
  size_t dvec_rows = 0;
  std::list<std::pair<ScheduleKey, std::unique_ptr<CachedSchedule>>> schedules;  // most recent first
};

std::mutex g_mu;
std::map<int, DeviceState> g_devices;
constexpr size_t kMaxCachedSchedules = 16;

void free_schedule(CachedSchedule* s) {
  if (s->d_items) cudaFree(s->d_items);
  if (s->d_kv_rows) cudaFree(s->d_kv_rows);
  if (s->d_head_win) cudaFree(s->d_head_win);
  if (s->d_kv_mask_id) cudaFree(s->d_kv_mask_id);
  if (s->d_kv_masks) cudaFree(s->d_kv_masks);
  s->d_items = nullptr;
  s->d_kv_rows = nullptr;
  s->d_head_win = nullptr;
  s->d_kv_mask_id = nullptr;
  s->d_kv_masks = nullptr;
}

// Caller holds g_mu.
sta_status device_state(int dev, DeviceState** out) {
  DeviceState& st = g_devices[dev];
  if (!st.d_err) {
    cudaError_t e = cudaMalloc(&st.d_err, 256);
    if (e != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemset(st.d_err, 0, 256)) != cudaSuccess) return cuda_fail(e);
  }
  *out = &st;
  return STA_OK;
}

template <typename T>
cudaError_t upload(T** dst, const std::vector<T>& v) {
  const size_t bytes = std::max<size_t>(v.size() * sizeof(T), 16);
  cudaError_t e = cudaMalloc(dst, bytes);
  if (e != cudaSuccess) return e;
  if (!v.empty()) e = cudaMemcpy(*dst, v.data(), v.size() * sizeof(T), cudaMemcpyHostToDevice);
  return e;
}

// Caller holds g_mu.
sta_status get_schedule(DeviceState* st, const Geometry& g, int32_t batch, int32_t heads,
                        const sta_dim3* windows, int kind, CachedSchedule** out) {
  std::vector<int32_t> wv(static_cast<size_t>(heads) * 3);
  for (int32_t h = 0; h < heads; ++h) {
    wv[h * 3 + 0] = windows[h].t;
    wv[h * 3 + 1] = windows[h].h;
    wv[h * 3 + 2] = windows[h].w;
  }
  ScheduleKey key{kind, batch, heads, g.T, g.H, g.W, g.tt, g.th, g.tw, std::move(wv)};
  for (auto it = st->schedules.begin(); it != st->schedules.end(); ++it) {
    if (it->first == key) {
      st->schedules.splice(st->schedules.begin(), st->schedules, it);
      *out = st->schedules.front().second.get();
      return STA_OK;
    }
  }
  auto cs = std::make_unique<CachedSchedule>();
  if (kind == 1)
    build_schedule_raster(g, batch, heads, windows, &cs->host);
  else if (kind == 2)
    build_schedule_transposed(g, batch, heads, windows, &cs->host);
  else
    build_schedule(g, batch, heads, windows, &cs->host);
  for (const WorkItem& w : cs->host.items)
    if (w.kv_len < 1) return STA_ERR_ARG;  // cannot happen: a tile always sees itself
#if STA_DEVICE_CHECKS
  // Checked builds only: STA_CHECKS_PLANT_BAD_ROW=1 plants a key-block row far past
  // the tensor in the schedule, so that a test can see the device check catch it.
  // (A tensor-map load at such a row would read zeros, not fault.)
  if (const char* plant = std::getenv("STA_CHECKS_PLANT_BAD_ROW"))
    if (plant[0] == '1' && !cs->host.kv_rows.empty()) cs->host.kv_rows[0] = static_cast<int32_t>(g.Lpad) + 64 * kBlockRows;
#endif
  cudaError_t e;
  if ((e = upload(&cs->d_items, cs->host.items)) != cudaSuccess ||
      (e = upload(&cs->d_kv_rows, cs->host.kv_rows)) != cudaSuccess ||
      (e = upload(&cs->d_head_win, cs->host.head_win)) != cudaSuccess ||
      (!cs->host.kv_masks.empty() && ((e = upload(&cs->d_kv_mask_id, cs->host.kv_mask_id)) != cudaSuccess ||
                                      (e = upload(&cs->d_kv_masks, cs->host.kv_masks)) != cudaSuccess))) {
    free_schedule(cs.get());
    return cuda_fail(e);
  }
  st->schedules.emplace_front(std::move(key), std::move(cs));
  if (st->schedules.size() > kMaxCachedSchedules) {
    // a kernel queued earlier on any stream may still read the evicted schedule's arrays
    cudaError_t es = cudaDeviceSynchronize();
    if (es != cudaSuccess) return cuda_fail(es);
  }
  while (st->schedules.size() > kMaxCachedSchedules) {
    free_schedule(st->schedules.back().second.get());
    st->schedules.pop_back();
  }
  *out = st->schedules.front().second.get();
  return STA_OK;
}

sta_status validate_tensor_args(const void* src, const void* dst, int64_t batch_heads, int32_t d,
                                sta_dim3 grid, sta_dim3 tile, Geometry* g) {
  if (!src || !dst) return STA_ERR_NULL;
  if (!aligned16(src) || !aligned16(dst)) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  sta_status s = make_geometry(grid, tile, g);
  if (s != STA_OK) return s;
  if (batch_heads < 0 || batch_heads > (int64_t(1) << 31)) return STA_ERR_ARG;
  const int64_t bytes = batch_heads * g->L * d * 2;
  if (batch_heads > 0 && overlaps(src, dst, bytes)) return STA_ERR_ALIAS;
  return STA_OK;
}

}  // namespace

sta_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = cudaGetErrorString(e);
  return STA_ERR_CUDA;
}

}  // namespace sta

using namespace sta;

extern "C" {

const char* sta_status_str(sta_status s) {
  switch (s) {
    case STA_OK: return "STA_OK";
    case STA_ERR_NULL: return "STA_ERR_NULL";
    case STA_ERR_ALIGN: return "STA_ERR_ALIGN";
    case STA_ERR_ALIAS: return "STA_ERR_ALIAS";
    case STA_ERR_SHAPE: return "STA_ERR_SHAPE";
    case STA_ERR_WINDOW: return "STA_ERR_WINDOW";
    case STA_ERR_HEADDIM: return "STA_ERR_HEADDIM";
    case STA_ERR_ARCH: return "STA_ERR_ARCH";
    case STA_ERR_CUDA: return "STA_ERR_CUDA";
    case STA_ERR_TIMEOUT: return "STA_ERR_TIMEOUT";
    case STA_ERR_ARG: return "STA_ERR_ARG";
    case STA_ERR_SCRATCH: return "STA_ERR_SCRATCH";
    case STA_ERR_BOUNDS: return "STA_ERR_BOUNDS";
  }
  return "STA_ERR_UNKNOWN";
}

const char* sta_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

sta_status sta_tile_index_map(sta_dim3 grid, sta_dim3 tile, int32_t* tiled_of_raster) {
  Geometry g;
  sta_status s = make_geometry(grid, tile, &g);
  if (s != STA_OK) return s;
  if (!tiled_of_raster) return STA_ERR_NULL;
  // Walk tiles in raster order over the tile grid and tokens in raster order
  // inside each tile; the running counter is the tiled row.
  int32_t m = 0;
  for (int32_t at = 0; at < g.nT; ++at)
    for (int32_t ah = 0; ah < g.nH; ++ah)
      for (int32_t aw = 0; aw < g.nW; ++aw)
        for (int32_t lt = 0; lt < g.tt; ++lt)
          for (int32_t lh = 0; lh < g.th; ++lh)
            for (int32_t lw = 0; lw < g.tw; ++lw) {
              const int64_t n = (static_cast<int64_t>(at * g.tt + lt) * g.H + (ah * g.th + lh)) * g.W + aw * g.tw + lw;
              tiled_of_raster[n] = m++;
            }
  return STA_OK;
}

int64_t sta_attended_pairs(int32_t batch, int32_t heads, sta_dim3 grid, sta_dim3 tile, const sta_dim3* windows) {
  Geometry g;
  if (make_geometry(grid, tile, &g) != STA_OK || batch < 0 || heads < 0 || (heads > 0 && !windows)) return -1;
  int64_t total = 0;
  for (int32_t h = 0; h < heads; ++h) {
    if (windows[h].t < 1 || windows[h].h < 1 || windows[h].w < 1) return -1;
    const int64_t wt = std::min(windows[h].t, g.nT), wh = std::min(windows[h].h, g.nH), ww = std::min(windows[h].w, g.nW);
    total += g.L * g.ntile * wt * wh * ww;
  }
  return total * batch;
}

int64_t sta_schedule_block_pairs(int32_t batch, int32_t heads, sta_dim3 grid, sta_dim3 tile,
                                 const sta_dim3* windows, int32_t transposed, int32_t* out, int64_t capacity) {
  Geometry g;
  if (make_geometry(grid, tile, &g) != STA_OK || batch < 1 || heads < 1 || !windows || capacity < 0) return -1;
  if (g.ntile % kBlockRows != 0) return -1;
  for (int32_t h = 0; h < heads; ++h)
    if (windows[h].t < 1 || windows[h].h < 1 || windows[h].w < 1) return -1;
  HostSchedule hs;
  if (transposed)
    build_schedule_transposed(g, batch, heads, windows, &hs);
  else
    build_schedule(g, batch, heads, windows, &hs);
  int64_t n = 0;
  for (const WorkItem& it : hs.items)
    for (int32_t j = 0; j < it.kv_len; ++j, ++n) {
      if (!out || n >= capacity) continue;
      const int32_t listed = hs.kv_rows[it.kv_off + j];
      out[3 * n + 0] = it.bh;
      out[3 * n + 1] = transposed ? listed : it.q_row0;   // query block
      out[3 * n + 2] = transposed ? it.q_row0 : listed;   // key block
    }
  return n;
}

sta_status sta_tile_reorder(const void* src, void* dst, int64_t batch_heads, int32_t d, sta_dim3 grid,
                            sta_dim3 tile, void* stream) {
  Geometry g;
  sta_status s = validate_tensor_args(src, dst, batch_heads, d, grid, tile, &g);
  if (s != STA_OK) return s;
  if ((s = check_device(nullptr)) != STA_OK) return s;
  cudaError_t e = launch_reorder(src, dst, batch_heads, d, g, true, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}

sta_status sta_tile_unorder(const void* src, void* dst, int64_t batch_heads, int32_t d, sta_dim3 grid,
                            sta_dim3 tile, void* stream) {
  Geometry g;
  sta_status s = validate_tensor_args(src, dst, batch_heads, d, grid, tile, &g);
  if (s != STA_OK) return s;
  if ((s = check_device(nullptr)) != STA_OK) return s;
  cudaError_t e = launch_reorder(src, dst, batch_heads, d, g, false, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}

namespace {
// sta_tile_reorder_tokens and sta_tile_unorder_tokens: validation, launch.
sta_status reorder_tokens_impl(const void* src, void* dst, int32_t batch, int32_t heads, int32_t d,
                               sta_dim3 grid, sta_dim3 tile, bool to_tiled, void* stream) {
  if (batch < 0 || heads < 0) return STA_ERR_ARG;
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  Geometry g;
  sta_status s = validate_tensor_args(src, dst, bh, d, grid, tile, &g);
  if (s != STA_OK) return s;
  if ((s = check_device(nullptr)) != STA_OK) return s;
  if (bh == 0) return STA_OK;
  cudaError_t e = launch_reorder(src, dst, bh, d, g, to_tiled, static_cast<cudaStream_t>(stream), heads);
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}
}  // namespace

sta_status sta_tile_reorder_tokens(const void* src, void* dst, int32_t batch, int32_t heads, int32_t d,
                                   sta_dim3 grid, sta_dim3 tile, void* stream) {
  return reorder_tokens_impl(src, dst, batch, heads, d, grid, tile, true, stream);
}

sta_status sta_tile_unorder_tokens(const void* src, void* dst, int32_t batch, int32_t heads, int32_t d,
                                   sta_dim3 grid, sta_dim3 tile, void* stream) {
  return reorder_tokens_impl(src, dst, batch, heads, d, grid, tile, false, stream);
}

namespace {
// sta_attention_fwd and sta_attention_fwd_lse: validation, schedule, launch.
sta_status attention_fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int32_t batch,
                              int32_t heads, int32_t d, sta_dim3 grid, sta_dim3 tile,
                              const sta_dim3* window_per_head, float scale, void* stream) {
  if (!q || !k || !v || !out || !window_per_head) return STA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return STA_ERR_ALIGN;
  if (lse && reinterpret_cast<uintptr_t>(lse) % 4 != 0) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry(grid, tile, &g);
  if (s != STA_OK) return s;
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > (int64_t(1) << 24)) return STA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return STA_ERR_ARG;
  for (int32_t h = 0; h < heads; ++h)
    if (window_per_head[h].t < 1 || window_per_head[h].h < 1 || window_per_head[h].w < 1) return STA_ERR_WINDOW;
  const int64_t bytes = static_cast<int64_t>(batch) * heads * g.L * d * 2;
  if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes)) return STA_ERR_ALIAS;
  if (lse) {
    const int64_t lbytes = static_cast<int64_t>(batch) * heads * g.L * 4;
    auto hit = [&](const void* t) {
      const char* a = static_cast<const char*>(t);
      const char* b = reinterpret_cast<const char*>(lse);
      return a < b + lbytes && b < a + bytes;
    };
    if (hit(q) || hit(k) || hit(v) || hit(out)) return STA_ERR_ALIAS;
  }
  int dev = 0;
  if ((s = check_device(&dev)) != STA_OK) return s;

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((s = device_state(dev, &st)) != STA_OK) return s;
  CachedSchedule* cs = nullptr;
  if ((s = get_schedule(st, g, batch, heads, window_per_head, 0, &cs)) != STA_OK) return s;
  DeviceSchedule ds{cs->d_items, cs->d_kv_rows, cs->d_head_win, static_cast<int32_t>(cs->host.items.size()),
                    cs->host.masked};
  ds.n_kv_rows = static_cast<int32_t>(cs->host.kv_rows.size());
  cudaError_t e = launch_attention(q, k, v, out, batch, heads, d, g, ds, scale, st->d_err, kWaitLimitNs,
                                   static_cast<cudaStream_t>(stream), lse);
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}
}  // namespace

sta_status sta_attention_fwd(const void* q, const void* k, const void* v, void* out, int32_t batch,
                             int32_t heads, int32_t d, sta_dim3 grid, sta_dim3 tile,
                             const sta_dim3* window_per_head, float scale, void* stream) {
  return attention_fwd_impl(q, k, v, out, nullptr, batch, heads, d, grid, tile, window_per_head, scale, stream);
}

sta_status sta_attention_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                                 int32_t batch, int32_t heads, int32_t d, sta_dim3 grid, sta_dim3 tile,
                                 const sta_dim3* window_per_head, float scale, void* stream) {
  if (!lse) return STA_ERR_NULL;
  return attention_fwd_impl(q, k, v, out, lse, batch, heads, d, grid, tile, window_per_head, scale, stream);
}

sta_status sta_attention_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, int32_t batch, int32_t heads,
                             int32_t d, sta_dim3 grid, sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                             void* stream) {
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !window_per_head) return STA_ERR_NULL;
  const void* bf[8] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* t : bf)
    if (!aligned16(t)) return STA_ERR_ALIGN;
  if (!aligned16(lse)) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry(grid, tile, &g);
  if (s != STA_OK) return s;
  if (g.ntile % kBlockRows != 0) return STA_ERR_SHAPE;
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > (int64_t(1) << 24)) return STA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return STA_ERR_ARG;
  for (int32_t h = 0; h < heads; ++h)
    if (window_per_head[h].t < 1 || window_per_head[h].h < 1 || window_per_head[h].w < 1) return STA_ERR_WINDOW;
  const int64_t rows = static_cast<int64_t>(batch) * heads * g.L;
  const int64_t bytes = rows * d * 2;
  // each output overlaps no other tensor
  const void* outs[3] = {dq, dk, dv};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 5; ++j)
      if (overlaps(outs[i], bf[j], bytes)) return STA_ERR_ALIAS;
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], outs[j], bytes)) return STA_ERR_ALIAS;
    const char* a = static_cast<const char*>(outs[i]);
    const char* l = reinterpret_cast<const char*>(lse);
    if (a < l + rows * 4 && l < a + bytes) return STA_ERR_ALIAS;
  }
  int dev = 0;
  if ((s = check_device(&dev)) != STA_OK) return s;

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((s = device_state(dev, &st)) != STA_OK) return s;
  if (st->dvec_rows < static_cast<size_t>(rows)) {
    // grows only; kept for later calls (stream-ordered use, so the old buffer is
    // freed after synchronising)
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    if (st->d_dvec) cudaFree(st->d_dvec);
    st->d_dvec = nullptr;
    st->dvec_rows = 0;
    if ((e = cudaMalloc(&st->d_dvec, static_cast<size_t>(rows) * sizeof(float))) != cudaSuccess) return cuda_fail(e);
    st->dvec_rows = static_cast<size_t>(rows);
  }
  CachedSchedule* fw = nullptr;
  if ((s = get_schedule(st, g, batch, heads, window_per_head, 0, &fw)) != STA_OK) return s;
  CachedSchedule* tr = nullptr;
  if ((s = get_schedule(st, g, batch, heads, window_per_head, 2, &tr)) != STA_OK) return s;
  // a new schedule may have evicted the other from the cache: look the forward one up again
  if ((s = get_schedule(st, g, batch, heads, window_per_head, 0, &fw)) != STA_OK) return s;
  DeviceSchedule dfw{fw->d_items, fw->d_kv_rows, fw->d_head_win, static_cast<int32_t>(fw->host.items.size()), false};
  DeviceSchedule dtr{tr->d_items, tr->d_kv_rows, tr->d_head_win, static_cast<int32_t>(tr->host.items.size()), false};
  dfw.n_kv_rows = static_cast<int32_t>(fw->host.kv_rows.size());
  dtr.n_kv_rows = static_cast<int32_t>(tr->host.kv_rows.size());
  cudaError_t e = launch_backward(q, k, v, out, dout, lse, st->d_dvec, dq, dk, dv, batch, heads, d, g, dfw, dtr,
                                  scale, st->d_err, kWaitLimitNs, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}

sta_status sta_attention_fwd_raster(const void* q, const void* k, const void* v, void* out, int32_t batch,
                                    int32_t heads, int32_t d, sta_dim3 grid, sta_dim3 tile,
                                    const sta_dim3* window_per_head, float scale, void* stream) {
  if (!q || !k || !v || !out || !window_per_head) return STA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry_padded(grid, tile, &g);
  if (s != STA_OK) return s;
  if (!raster_tile_ok(g.tt, g.th, g.tw) || g.ntile % kBlockRows != 0) return STA_ERR_SHAPE;
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > (int64_t(1) << 24)) return STA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return STA_ERR_ARG;
  for (int32_t h = 0; h < heads; ++h)
    if (window_per_head[h].t < 1 || window_per_head[h].h < 1 || window_per_head[h].w < 1) return STA_ERR_WINDOW;
  const int64_t bytes = static_cast<int64_t>(batch) * heads * g.L * d * 2;
  if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes)) return STA_ERR_ALIAS;
  int dev = 0;
  if ((s = check_device(&dev)) != STA_OK) return s;

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((s = device_state(dev, &st)) != STA_OK) return s;
  CachedSchedule* cs = nullptr;
  if ((s = get_schedule(st, g, batch, heads, window_per_head, 1, &cs)) != STA_OK) return s;
  DeviceSchedule ds{cs->d_items, cs->d_kv_rows, cs->d_head_win, static_cast<int32_t>(cs->host.items.size()), false,
                    cs->d_kv_mask_id, cs->d_kv_masks, static_cast<int32_t>(cs->host.kv_rows.size()),
                    static_cast<int32_t>(cs->host.kv_masks.size() / 4)};
  cudaError_t e = launch_attention_raster(q, k, v, out, batch, heads, d, g, ds, scale, st->d_err, kWaitLimitNs,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}

namespace {
// Reads a device status word into *flag; if it is set, clears it.  A flag is
// 0x100 | site for an expired wait and 0x200 | code for a failed device check.
sta_status read_and_clear(int32_t* word, int32_t* flag) {
  cudaError_t e = cudaMemcpy(flag, word, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (*flag != 0 && (e = cudaMemset(word, 0, sizeof(int32_t))) != cudaSuccess) return cuda_fail(e);
  return STA_OK;
}

// The status words of the current device: the allocating entry points' word (if
// allocated) and the no-alloc entry point's word (if set up).  Caller holds no lock.
int status_words(int dev, int32_t* words[2]) {
  int n = 0;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_devices.find(dev);
    if (it != g_devices.end() && it->second.d_err) words[n++] = it->second.d_err;
  }
  if (int32_t* w = noalloc_status_word(dev)) words[n++] = w;
  return n;
}
}  // namespace

sta_status sta_tile_reorder_padded(const void* src, void* dst, int64_t batch_heads, int32_t d, sta_dim3 grid,
                                   sta_dim3 tile, void* stream) {
  if (!src || !dst) return STA_ERR_NULL;
  if (!aligned16(src) || !aligned16(dst)) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry_padded(grid, tile, &g);
  if (s != STA_OK) return s;
  if (batch_heads < 0 || batch_heads > (int64_t(1) << 31)) return STA_ERR_ARG;
  const char* a = static_cast<const char*>(src);
  const char* b = static_cast<const char*>(dst);
  if (batch_heads > 0 && a < b + batch_heads * g.Lpad * d * 2 && b < a + batch_heads * g.L * d * 2) return STA_ERR_ALIAS;
  if ((s = check_device(nullptr)) != STA_OK) return s;
  cudaError_t e = launch_reorder_padded(src, dst, batch_heads, d, g, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}

sta_status sta_attention_fwd_mixed(const void* q, const void* k_tiled, const void* v_tiled, void* out, int32_t batch,
                                   int32_t heads, int32_t d, sta_dim3 grid, sta_dim3 tile,
                                   const sta_dim3* window_per_head, float scale, void* stream) {
  if (!q || !k_tiled || !v_tiled || !out || !window_per_head) return STA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_tiled) || !aligned16(v_tiled) || !aligned16(out)) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry_padded(grid, tile, &g);
  if (s != STA_OK) return s;
  if (!raster_tile_ok(g.tt, g.th, g.tw) || g.ntile % kBlockRows != 0) return STA_ERR_SHAPE;
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > (int64_t(1) << 24)) return STA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return STA_ERR_ARG;
  for (int32_t h = 0; h < heads; ++h)
    if (window_per_head[h].t < 1 || window_per_head[h].h < 1 || window_per_head[h].w < 1) return STA_ERR_WINDOW;
  const int64_t rows = static_cast<int64_t>(batch) * heads;
  const int64_t raster_bytes = rows * g.L * d * 2, tiled_bytes = rows * g.Lpad * d * 2;
  auto hit = [](const void* x, int64_t nx, const void* y, int64_t ny) {
    const char* a = static_cast<const char*>(x);
    const char* b = static_cast<const char*>(y);
    return a < b + ny && b < a + nx;
  };
  if (hit(out, raster_bytes, q, raster_bytes) || hit(out, raster_bytes, k_tiled, tiled_bytes) ||
      hit(out, raster_bytes, v_tiled, tiled_bytes))
    return STA_ERR_ALIAS;
  int dev = 0;
  if ((s = check_device(&dev)) != STA_OK) return s;

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((s = device_state(dev, &st)) != STA_OK) return s;
  CachedSchedule* cs = nullptr;
  if ((s = get_schedule(st, g, batch, heads, window_per_head, 1, &cs)) != STA_OK) return s;
  DeviceSchedule ds{cs->d_items, cs->d_kv_rows, cs->d_head_win, static_cast<int32_t>(cs->host.items.size()), false,
                    cs->d_kv_mask_id, cs->d_kv_masks, static_cast<int32_t>(cs->host.kv_rows.size()),
                    static_cast<int32_t>(cs->host.kv_masks.size() / 4)};
  cudaError_t e = launch_attention_mixed(q, k_tiled, v_tiled, out, batch, heads, d, g, ds, scale, st->d_err,
                                         kWaitLimitNs, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}

namespace {
cudaError_t pipe_init(HostPipe* pp) {
  if (pp->s_in) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  for (cudaStream_t* s : {&pp->s_in, &pp->s_run, &pp->s_out})
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
  for (cudaEvent_t* ev : {&pp->start, &pp->copied[0], &pp->copied[1], &pp->computed[0], &pp->computed[1],
                          &pp->drained[0], &pp->drained[1]})
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  return e;
}

void pipe_free(HostPipe* pp) {
  for (cudaStream_t s : {pp->s_in, pp->s_run, pp->s_out})
    if (s) cudaStreamDestroy(s);
  for (cudaEvent_t ev : {pp->start, pp->copied[0], pp->copied[1], pp->computed[0], pp->computed[1], pp->drained[0],
                         pp->drained[1]})
    if (ev) cudaEventDestroy(ev);
  if (pp->buf) cudaFree(pp->buf);
  *pp = HostPipe{};
}
}  // namespace

sta_status sta_forward_host(const void* q, const void* k, const void* v, void* out, int32_t batch, int32_t heads,
                            int32_t d, sta_dim3 grid, sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                            int32_t heads_per_chunk, void* stream) {
  if (!q || !k || !v || !out || !window_per_head) return STA_ERR_NULL;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry_padded(grid, tile, &g);
  if (s != STA_OK) return s;
  if (!raster_tile_ok(g.tt, g.th, g.tw) || g.ntile % kBlockRows != 0) return STA_ERR_SHAPE;
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > (int64_t(1) << 24)) return STA_ERR_ARG;
  if (heads_per_chunk < 1) return STA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return STA_ERR_ARG;
  for (int32_t h = 0; h < heads; ++h)
    if (window_per_head[h].t < 1 || window_per_head[h].h < 1 || window_per_head[h].w < 1) return STA_ERR_WINDOW;
  const int64_t head_bytes = g.L * d * 2;   // one (batch, head) slice, raster order
  const int64_t bytes = static_cast<int64_t>(batch) * heads * head_bytes;
  if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes)) return STA_ERR_ALIAS;
  int dev = 0;
  if ((s = check_device(&dev)) != STA_OK) return s;

  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((s = device_state(dev, &st)) != STA_OK) return s;
  HostPipe& pp = st->pipe;
  cudaError_t e = pipe_init(&pp);
  if (e != cudaSuccess) return cuda_fail(e);
  const int32_t hc = std::min(heads_per_chunk, heads);
  const int64_t raster = hc * head_bytes, tiled = hc * g.Lpad * d * 2;
  const size_t slot_bytes = static_cast<size_t>(4 * raster + 2 * tiled);   // q, k, v, out; k, v tiled
  if (pp.bytes < 2 * slot_bytes) {
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e);
    if (pp.buf) cudaFree(pp.buf);
    pp.buf = nullptr;
    pp.bytes = 0;
    if ((e = cudaMalloc(&pp.buf, 2 * slot_bytes)) != cudaSuccess) return cuda_fail(e);
    pp.bytes = 2 * slot_bytes;
  }
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  const uint8_t* hv = static_cast<const uint8_t*>(v);
  uint8_t* hout = static_cast<uint8_t*>(out);
  // the work starts after what is queued on the caller's stream
  if ((e = cudaEventRecord(pp.start, static_cast<cudaStream_t>(stream))) != cudaSuccess) return cuda_fail(e);
  for (cudaStream_t sx : {pp.s_in, pp.s_run, pp.s_out})
    if ((e = cudaStreamWaitEvent(sx, pp.start, 0)) != cudaSuccess) return cuda_fail(e);
  bool used[2] = {false, false};
  int64_t i = 0;
  for (int32_t b = 0; b < batch && e == cudaSuccess; ++b) {
    for (int32_t h0 = 0; h0 < heads && e == cudaSuccess; h0 += hc, ++i) {
      const int slot = static_cast<int>(i & 1);
      const int32_t n = std::min(hc, heads - h0);
      const int64_t off = (static_cast<int64_t>(b) * heads + h0) * head_bytes, len = n * head_bytes;
      uint8_t* dq = pp.buf + slot * slot_bytes;
      uint8_t *dk = dq + raster, *dv = dk + raster, *dout = dv + raster, *dkt = dout + raster, *dvt = dkt + tiled;
      CachedSchedule* cs = nullptr;
      if ((s = get_schedule(st, g, 1, n, window_per_head + h0, 1, &cs)) != STA_OK) break;
      DeviceSchedule ds{cs->d_items, cs->d_kv_rows, cs->d_head_win, static_cast<int32_t>(cs->host.items.size()),
                        false, cs->d_kv_mask_id, cs->d_kv_masks, static_cast<int32_t>(cs->host.kv_rows.size()),
                        static_cast<int32_t>(cs->host.kv_masks.size() / 4)};
      // copy in: the slot's inputs are free once its previous chunk was computed
      if (used[slot] && (e = cudaStreamWaitEvent(pp.s_in, pp.computed[slot], 0)) != cudaSuccess) break;
      if ((e = cudaMemcpyAsync(dq, hq + off, len, cudaMemcpyHostToDevice, pp.s_in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(dk, hk + off, len, cudaMemcpyHostToDevice, pp.s_in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(dv, hv + off, len, cudaMemcpyHostToDevice, pp.s_in)) != cudaSuccess ||
          (e = cudaEventRecord(pp.copied[slot], pp.s_in)) != cudaSuccess)
        break;
      // compute: after the copy in, and once the slot's previous output was copied out
      if ((e = cudaStreamWaitEvent(pp.s_run, pp.copied[slot], 0)) != cudaSuccess) break;
      if (used[slot] && (e = cudaStreamWaitEvent(pp.s_run, pp.drained[slot], 0)) != cudaSuccess) break;
      if ((e = launch_reorder_padded(dk, dkt, n, d, g, pp.s_run)) != cudaSuccess ||
          (e = launch_reorder_padded(dv, dvt, n, d, g, pp.s_run)) != cudaSuccess ||
          (e = launch_attention_mixed(dq, dkt, dvt, dout, 1, n, d, g, ds, scale, st->d_err, kWaitLimitNs,
                                      pp.s_run)) != cudaSuccess ||
          (e = cudaEventRecord(pp.computed[slot], pp.s_run)) != cudaSuccess)
        break;
      // copy out
      if ((e = cudaStreamWaitEvent(pp.s_out, pp.computed[slot], 0)) != cudaSuccess ||
          (e = cudaMemcpyAsync(hout + off, dout, len, cudaMemcpyDeviceToHost, pp.s_out)) != cudaSuccess ||
          (e = cudaEventRecord(pp.drained[slot], pp.s_out)) != cudaSuccess)
        break;
      used[slot] = true;
    }
  }
  // every queued copy and kernel completes before the call returns, also after an error
  const cudaError_t e_in = cudaStreamSynchronize(pp.s_in), e_run = cudaStreamSynchronize(pp.s_run),
                    e_out = cudaStreamSynchronize(pp.s_out);
  if (s != STA_OK) return s;
  if (e != cudaSuccess) return cuda_fail(e);
  for (cudaError_t ex : {e_in, e_run, e_out})
    if (ex != cudaSuccess) return cuda_fail(ex);
  return STA_OK;
}

sta_status sta_check_device_status(void* stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess) return cuda_fail(e);
  int32_t* words[2];
  const int n = status_words(dev, words);
  sta_status result = STA_OK;
  for (int i = 0; i < n; ++i) {
    int32_t flag = 0;
    sta_status s = read_and_clear(words[i], &flag);
    if (s != STA_OK) return s;
    if ((flag & 0x200) != 0) result = STA_ERR_BOUNDS;
    else if (flag != 0 && result == STA_OK) result = STA_ERR_TIMEOUT;
  }
  return result;
}

sta_status sta_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns < 100000ull) limit_ns = 100000ull;
  if (limit_ns > 5000000000ull) limit_ns = 5000000000ull;
  sta_status s;
  int dev = 0;
  if ((s = check_device(&dev)) != STA_OK) return s;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* st = nullptr;
    if ((s = device_state(dev, &st)) != STA_OK) return s;
  }
  // One run-out wait per status word of the device; each word must report it.
  int32_t* words[2];
  const int n = status_words(dev, words);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  for (int i = 0; i < n; ++i)
    if ((e = launch_selftest_wait(words[i], limit_ns, cs)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamSynchronize(cs)) != cudaSuccess) return cuda_fail(e);
  bool all = n > 0;
  for (int i = 0; i < n; ++i) {
    int32_t flag = 0;
    if ((s = read_and_clear(words[i], &flag)) != STA_OK) return s;
    all = all && (flag & 0x100) != 0;
  }
  return all ? STA_ERR_TIMEOUT : STA_OK;
}

void sta_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_devices) {
    if (cudaSetDevice(kv.first) != cudaSuccess) continue;
    for (auto& s : kv.second.schedules) free_schedule(s.second.get());
    kv.second.schedules.clear();
    if (kv.second.d_err) cudaFree(kv.second.d_err);
    kv.second.d_err = nullptr;
    if (kv.second.d_dvec) cudaFree(kv.second.d_dvec);
    kv.second.d_dvec = nullptr;
    kv.second.dvec_rows = 0;
    pipe_free(&kv.second.pipe);
  }
  g_devices.clear();
  noalloc_reset();
  cudaSetDevice(cur);
}

}  // extern "C"
