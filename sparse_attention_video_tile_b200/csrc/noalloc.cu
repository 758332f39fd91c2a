// noalloc.cu - sta_attention_fwd_noalloc: the attention forward without any
// device allocation by the library.
//
// sta_attention_fwd keeps its work schedule and a status word in device memory
// that the library allocates with cudaMalloc on first use.  Some callers cannot
// allow that: code that runs inside a memory pool or arena it must not bypass,
// a host process that pre-reserves all device memory before the library is
// first called, or a runtime whose allocator must see every device allocation
// for accounting.  This variant instead keeps the same scratch (status word,
// work items, key-block lists, per-head windows) in one file-scope device array
// of fixed size, kScratchBytes, which every GPU that loads the library holds
// until the process exits.  The caller still owns q, k, v and out.
//
// Host code cannot use the array's name as a device address (it is a host-side
// stand-in), so the device address is obtained once per device with
// cudaGetSymbolAddress while that device is current; the first call on a
// device performs this set-up, so make that first call before any stream
// capture.
//
// All calls share the array and it keeps the last call's contents: the status
// word is cleared at the start of every call, and the schedule is uploaded
// again whenever the configuration differs from the last one uploaded on the
// device.  Calls that overlap on the GPU (for instance on two streams) race on
// the array and must be ordered by the caller.
//
// A kernel that gives up on a bounded wait records it in the status word, which
// sta_check_device_status reads (and clears) beside the allocating entry points'
// word.  sta_shutdown forgets the set-up, so after it (or after a device reset,
// which re-initialises the array) the next call looks the address up again and
// uploads its schedule anew.
#include <cuda_runtime.h>

#include <array>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace sta {
namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;   // 4 MiB per device
constexpr size_t kStatusBytes = 256;                // status word (+ padding)
constexpr uint64_t kNoAllocWaitLimitNs = 2000000000ull;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct NoAllocDevice {
  bool ready = false;
  unsigned char* base = nullptr;          // device address of g_noalloc_scratch
  bool has_schedule = false;
  std::vector<int32_t> key;               // configuration of the uploaded schedule
  HostSchedule sched;                     // host copy of the uploaded schedule
  size_t off_items = 0, off_kv = 0, off_win = 0;
};

std::mutex g_noalloc_mu;
std::array<NoAllocDevice, kMaxDevices> g_noalloc;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

int32_t* noalloc_status_word(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const NoAllocDevice& nd = g_noalloc[dev];
  return nd.ready ? reinterpret_cast<int32_t*>(nd.base) : nullptr;
}

void noalloc_reset() {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (NoAllocDevice& nd : g_noalloc) nd = NoAllocDevice();
}

}  // namespace sta

using namespace sta;

extern "C" sta_status sta_attention_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                                int32_t batch, int32_t heads, int32_t d, sta_dim3 grid,
                                                sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                                                void* stream) {
  // Argument checks (same rules as sta_attention_fwd).
  if (!q || !k || !v || !out || !window_per_head) return STA_ERR_NULL;
  auto a16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; };
  if (!a16(q) || !a16(k) || !a16(v) || !a16(out)) return STA_ERR_ALIGN;
  if (d != 64 && d != 128) return STA_ERR_HEADDIM;
  Geometry g;
  sta_status s = make_geometry(grid, tile, &g);
  if (s != STA_OK) return s;
  if (batch < 1 || heads < 1 || static_cast<int64_t>(batch) * heads > (int64_t(1) << 24)) return STA_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return STA_ERR_ARG;
  for (int32_t h = 0; h < heads; ++h)
    if (window_per_head[h].t < 1 || window_per_head[h].h < 1 || window_per_head[h].w < 1) return STA_ERR_WINDOW;
  const int64_t bytes = static_cast<int64_t>(batch) * heads * g.L * d * 2;
  auto overlap = [bytes](const void* x, const void* y) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
    return a < b + static_cast<uintptr_t>(bytes) && b < a + static_cast<uintptr_t>(bytes);
  };
  if (overlap(out, q) || overlap(out, k) || overlap(out, v)) return STA_ERR_ALIAS;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e);
  if (major != 10 || minor != 0) return STA_ERR_ARCH;
  if (dev < 0 || dev >= kMaxDevices) return STA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& nd = g_noalloc[dev];
  if (!nd.ready) {
    // Once per device, with the device current: the scratch array's device address.
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    if (ptr == nullptr) return cuda_fail(cudaErrorInvalidSymbol);
    nd.base = static_cast<unsigned char*>(ptr);
    nd.ready = true;
  }

  std::vector<int32_t> key = {batch, heads, g.T, g.H, g.W, g.tt, g.th, g.tw};
  for (int32_t h = 0; h < heads; ++h) {
    key.push_back(window_per_head[h].t);
    key.push_back(window_per_head[h].h);
    key.push_back(window_per_head[h].w);
  }
  if (!nd.has_schedule || nd.key != key) {
    HostSchedule hs;
    build_schedule(g, batch, heads, window_per_head, &hs);
    for (const WorkItem& w : hs.items)
      if (w.kv_len < 1) return STA_ERR_ARG;
    const size_t off_items = kStatusBytes;
    const size_t off_kv = align256(off_items + hs.items.size() * sizeof(WorkItem));
    const size_t off_win = align256(off_kv + hs.kv_rows.size() * sizeof(int32_t));
    const size_t end = off_win + hs.head_win.size() * sizeof(int16_t);
    if (end > kScratchBytes) return STA_ERR_SCRATCH;  // schedule larger than the fixed scratch
    // Upload.  From pageable host memory the copy first waits for the stream's
    // earlier work (so a previous call on this stream is done with the array)
    // and returns once the source has been staged.
    nd.has_schedule = false;
    if ((e = cudaMemcpyAsync(nd.base + off_items, hs.items.data(), hs.items.size() * sizeof(WorkItem),
                             cudaMemcpyHostToDevice, st)) != cudaSuccess ||
        (e = cudaMemcpyAsync(nd.base + off_kv, hs.kv_rows.data(), hs.kv_rows.size() * sizeof(int32_t),
                             cudaMemcpyHostToDevice, st)) != cudaSuccess ||
        (e = cudaMemcpyAsync(nd.base + off_win, hs.head_win.data(), hs.head_win.size() * sizeof(int16_t),
                             cudaMemcpyHostToDevice, st)) != cudaSuccess)
      return cuda_fail(e);
    nd.sched = std::move(hs);
    nd.key = std::move(key);
    nd.off_items = off_items;
    nd.off_kv = off_kv;
    nd.off_win = off_win;
    nd.has_schedule = true;
  }
  // The status word must start at zero for every call.
  if ((e = cudaMemsetAsync(nd.base, 0, kStatusBytes, st)) != cudaSuccess) return cuda_fail(e);

  DeviceSchedule ds{reinterpret_cast<const WorkItem*>(nd.base + nd.off_items),
                    reinterpret_cast<const int32_t*>(nd.base + nd.off_kv),
                    reinterpret_cast<const int16_t*>(nd.base + nd.off_win),
                    static_cast<int32_t>(nd.sched.items.size()), nd.sched.masked};
  ds.n_kv_rows = static_cast<int32_t>(nd.sched.kv_rows.size());
  e = launch_attention(q, k, v, out, batch, heads, d, g, ds, scale, reinterpret_cast<int32_t*>(nd.base),
                       kNoAllocWaitLimitNs, st);
  return e == cudaSuccess ? STA_OK : cuda_fail(e);
}
