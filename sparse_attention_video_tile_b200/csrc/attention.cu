// attention.cu - Sliding Tile Attention forward for sm_100a.
//
// "Fast Video Generation with Sliding Tile Attention": each query tile attends
// densely to the key tiles of its window (abstract; summary page, "Method
// details"), blocks are either fully attended or skipped (summary page, "Core
// innovation"), and the kernel is built around asynchronous loads and block
// management (summary page, "AI overview").  On B200 that becomes:
//
//   * one CTA works on a block of 128 query rows at a time (persistent grid,
//     two CTAs per SM, work items from the host window enumerator);
//   * warp 4, the producer, streams Q once per item and then only the key and
//     value blocks of the window into a two-stage shared-memory ring with TMA
//     (128-byte swizzle, completion on mbarriers);
//   * warp 5 issues tcgen05 MMAs from one thread: S = Q K^T (both operands in
//     shared memory, fp32 accumulator in TMEM columns [0, 128)) and O += P V
//     (P read from TMEM where it overwrote S, V from shared memory, O in TMEM
//     columns [128, 128 + d));
//   * warps 0-3 (128 threads, one query row each, TMEM lane = row) run the
//     online softmax in fp32: row max, p = 2^(s*scale*log2e - m), row sum,
//     P rounded to bf16 and written back to TMEM; O is rescaled only when the
//     running max grows by more than 2^8 (the result is unchanged: O and the
//     row sum always carry the same factor), then the epilogue divides by the
//     row sum and writes bf16 rows.
// With Ntile a multiple of 128 no element mask exists at all.  Otherwise
// (small tiles, ragged tails) the softmax masks whole key tiles outside the
// row's window and keys past L.
//
// The two CTAs on an SM interleave: while one runs its softmax the other's
// MMAs keep the tensor core busy.  Every wait is bounded (see ptx.cuh): a
// stuck pipeline records an error code and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace sta {
namespace {

using namespace ptx;

constexpr int kThreads = 256;       // warps 0-3 softmax, 4 producer, 5 MMA, 6-7 idle
constexpr int kStages = 2;          // key/value ring stages (K and V alternate)
constexpr int kTmemCols = 256;      // S: [0,128), O: [128, 128 + d)
constexpr int kSCol = 0;
constexpr int kOCol = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Register split: launched at 128 per thread (256 threads, two CTAs per SM);
// the softmax warpgroup takes 208, the other warpgroup keeps 48:
// 128 * 208 + 128 * 48 = 256 * 128.
constexpr int kLaunchRegs = 128;
constexpr int kDefaultPoly16 = 0;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsOther = 48;
static_assert(128 * kRegsSoftmax + 128 * kRegsOther == kThreads * kLaunchRegs, "register split must match the launch");

struct FwdParams {
  const WorkItem* items;
  const int32_t* kv_rows;
  const int16_t* head_win;   // [heads][4]
  __nv_bfloat16* out;        // [BH, L, d] tiled order
  int32_t n_items;
  int32_t heads;
  int32_t L;
  int32_t nT, nH, nW;
  int32_t ntile;
  float scale_log2;          // scale * log2(e)
  int32_t* err;
  uint64_t limit_ns;
};

template <int D>
struct Smem {
  static constexpr int kBlockBytes = kBlockRows * D * 2;  // one 128-row block of Q, K or V
  static constexpr int kQ = 0;
  static constexpr int kStage0 = kBlockBytes;
  static constexpr int kBar = kStage0 + kStages * kBlockBytes;
  // barriers (8 bytes each)
  static constexpr int kQFull = kBar + 0;
  static constexpr int kQEmpty = kBar + 8;
  static constexpr int kKvFull = kBar + 16;                 // kStages
  static constexpr int kKvEmpty = kKvFull + 8 * kStages;    // kStages
  static constexpr int kSFull = kKvEmpty + 8 * kStages;
  static constexpr int kPFull = kSFull + 8;
  static constexpr int kOFull = kPFull + 8;
  static constexpr int kDrain = kOFull + 8;
  static constexpr int kTmemSlot = kDrain + 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kEnd = kAbort + 4;
  // + slack to align the base to 1024; never below 96 KB so that at most two CTAs
  // (2 x 256 TMEM columns) share an SM, whatever d is.
  static constexpr int kDynBytes = (kEnd + 1024) > 98304 ? (kEnd + 1024) : 98304;
};

// Descriptor of a K-major bf16 operand stored as [rows][64] boxes of 128 bytes per
// row (128-byte swizzle); k16 selects the 16-element slice along K.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int k16) {
  const uint32_t addr = base + static_cast<uint32_t>((k16 >> 2) * (kBlockRows * 128) + (k16 & 3) * 32);
  return sdesc_sw128(addr, 16, 1024);
}

// Descriptor of V as the MN-major B operand of P*V: rows are keys (K dim),
// 64-wide boxes of d (N dim) at 16 KB apart; k16 selects 16 keys.
__device__ __forceinline__ uint64_t vmn_desc(uint32_t base, int k16) {
  const uint32_t addr = base + static_cast<uint32_t>(k16 * 16 * 128);
  return sdesc_sw128(addr, kBlockRows * 128, 1024);
}

template <int D, bool MASKED, int POLY16>
__global__ void __launch_bounds__(kThreads, 2)
    sta_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using S = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kTmemSlot);

  if (threadIdx.x == 0) {
    mbar_init(sb + S::kQFull, 1);
    mbar_init(sb + S::kQEmpty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sb + S::kKvFull + 8 * s, 1);
      mbar_init(sb + S::kKvEmpty + 8 * s, 1);
    }
    mbar_init(sb + S::kSFull, 1);
    mbar_init(sb + S::kPFull, 128);
    mbar_init(sb + S::kOFull, 1);
    mbar_init(sb + S::kDrain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 5) {
    tmem_alloc(sb + S::kTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  WaitCtx wc{abort_flag, p.err, p.limit_ns};
  constexpr uint32_t kBoxBytes = kBlockRows * 128;       // one 128 x 64 bf16 box
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kBlockBytes = S::kBlockBytes;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec<kRegsOther>();
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t kv_seq = 0, it = 0, q_loads = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++it) {
        const WorkItem item = p.items[w];
        ok = mbar_wait(sb + S::kQEmpty, (it & 1) ^ 1, wc, 1);
        if (!ok) break;
        ++q_loads;
        mbar_arrive_expect_tx(sb + S::kQFull, kBlockBytes);
        for (int b = 0; b < kBoxes; ++b)
          tma_load_3d(sb + S::kQ + b * kBoxBytes, &tm_q, sb + S::kQFull, b * 64, item.q_row0, item.bh);
        for (int j = 0; j < item.kv_len && ok; ++j) {
          const int32_t kv_row = p.kv_rows[item.kv_off + j];
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t st = kv_seq % kStages;
            const uint32_t par = ((kv_seq / kStages) & 1) ^ 1;
            ok = mbar_wait(sb + S::kKvEmpty + 8 * st, par, wc, 2);
            if (!ok) break;
            const uint32_t dst = sb + S::kStage0 + st * kBlockBytes;
            const uint32_t full = sb + S::kKvFull + 8 * st;
            mbar_arrive_expect_tx(full, kBlockBytes);
            const CUtensorMap* m = kv == 0 ? &tm_k : &tm_v;
            for (int b = 0; b < kBoxes; ++b) tma_load_3d(dst + b * kBoxBytes, m, full, b * 64, kv_row, item.bh);
            ++kv_seq;
          }
        }
      }
      // Drain: every load issued has landed before the CTA may exit.  Waiting on a
      // phase that already completed returns at once.
      if (q_loads > 0) mbar_wait_drain(sb + S::kQFull, (q_loads - 1) & 1, p.limit_ns);
      for (uint32_t s = 0; s < kStages && s < kv_seq; ++s) {
        const uint32_t last = kv_seq - 1 - ((kv_seq - 1 - s) % kStages);  // last sequence number on stage s
        mbar_wait_drain(sb + S::kKvFull + 8 * s, (last / kStages) & 1, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    setmaxnreg_dec<kRegsOther>();
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      uint32_t kv_seq = 0, it = 0, sp = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++it) {
        const WorkItem item = p.items[w];
        ok = mbar_wait(sb + S::kQFull, it & 1, wc, 3);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < item.kv_len && ok; ++j) {
          // S = Q K^T
          uint32_t st = kv_seq % kStages;
          ok = mbar_wait(sb + S::kKvFull + 8 * st, (kv_seq / kStages) & 1, wc, 4);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kbase = sb + S::kStage0 + st * kBlockBytes;
#pragma unroll
          for (int k16 = 0; k16 < D / 16; ++k16)
            umma_ss(tmem + kSCol, kmajor_desc(sb + S::kQ, k16), kmajor_desc(kbase, k16), idesc_qk,
                    k16 > 0 ? 1u : 0u);
          umma_commit(sb + S::kKvEmpty + 8 * st);
          if (j == item.kv_len - 1) umma_commit(sb + S::kQEmpty);
          umma_commit(sb + S::kSFull);
          ++kv_seq;
          // O += P V once the softmax has written P
          ok = mbar_wait(sb + S::kPFull, sp & 1, wc, 5);
          ++sp;
          if (!ok) break;
          tc_fence_after();
          st = kv_seq % kStages;
          ok = mbar_wait(sb + S::kKvFull + 8 * st, (kv_seq / kStages) & 1, wc, 6);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vbase = sb + S::kStage0 + st * kBlockBytes;
#pragma unroll
          for (int k16 = 0; k16 < kBlockRows / 16; ++k16)
            umma_ts(tmem + kOCol, tmem + kSCol + k16 * 8, vmn_desc(vbase, k16), idesc_pv,
                    (j > 0 || k16 > 0) ? 1u : 0u);
          umma_commit(sb + S::kKvEmpty + 8 * st);
          ++kv_seq;
        }
        if (ok) umma_commit(sb + S::kOFull);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      umma_commit(sb + S::kDrain);
      mbar_wait_drain(sb + S::kDrain, 0, p.limit_ns);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax + epilogue
    setmaxnreg_inc<kRegsSoftmax>();
    const int row = threadIdx.x;                          // 0..127 = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t sphase = 0, it = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++it) {
      const WorkItem item = p.items[w];
      float m_run = -INFINITY;
      float l_run = 0.f;
      // masked path: this row's window box in tile coordinates
      int32_t ws_t = 0, ws_h = 0, ws_w = 0, we_t = 0, we_h = 0, we_w = 0;
      if (MASKED) {
        const int head = item.bh % p.heads;
        const int32_t et = p.head_win[head * 4 + 0], eh = p.head_win[head * 4 + 1], ew = p.head_win[head * 4 + 2];
        const int32_t qrow = item.q_row0 + row;
        const int32_t qt = (qrow < p.L ? qrow : p.L - 1) / p.ntile;
        const int32_t at = qt / (p.nH * p.nW), ah = (qt / p.nW) % p.nH, aw = qt % p.nW;
        ws_t = min(max(at - et / 2, 0), p.nT - et); we_t = ws_t + et;
        ws_h = min(max(ah - eh / 2, 0), p.nH - eh); we_h = ws_h + eh;
        ws_w = min(max(aw - ew / 2, 0), p.nW - ew); we_w = ws_w + ew;
      }
      for (int j = 0; j < item.kv_len; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kSFull, sphase & 1, wc, 7));
        ++sphase;
        if (!ok) break;
        tc_fence_after();
        // The whole score row (128 fp32) in one round trip.
        uint32_t r[128];
        tmem_ld32_at<0>(trow + kSCol, r);
        tmem_ld32_at<32>(trow + kSCol + 32, r);
        tmem_ld32_at<64>(trow + kSCol + 64, r);
        tmem_ld32_at<96>(trow + kSCol + 96, r);
        tmem_wait_ld();
        if (MASKED) {
          const int32_t kv_row = p.kv_rows[item.kv_off + j];
#pragma unroll
          for (int i = 0; i < 128; ++i) {
            const int32_t key = kv_row + i;
            bool in = key < p.L;
            if (in) {
              const int32_t kt = key / p.ntile;
              const int32_t bt = kt / (p.nH * p.nW), bh_ = (kt / p.nW) % p.nH, bw = kt % p.nW;
              in = bt >= ws_t && bt < we_t && bh_ >= ws_h && bh_ < we_h && bw >= ws_w && bw < we_w;
            }
            if (!in) r[i] = __float_as_uint(-INFINITY);
          }
        }
#define SV(i) __uint_as_float(r[i])
        // Row max: eight independent chains of three-input maxima.
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float a = max3f(SV(k), SV(k + 8), SV(k + 16));
#pragma unroll
          for (int t = 24; t < 120; t += 16) a = max3f(a, SV(k + t), SV(k + t + 8));
          mx8[k] = fmaxf(a, SV(k + 120));
        }
        const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_blk = mx * sl2;
        // The running max moves only when it grows by more than 2^8: p stays <= 256
        // and O and the row sum always carry the same factor, so O / l is exact.
        const bool need = (m_run != -INFINITY) && (m_blk > m_run + kRescaleThreshold);
        float f = 1.0f;
        if (m_run == -INFINITY) {
          m_run = m_blk;  // first contribution to this row: nothing accumulated yet
        } else if (need) {
          f = ex2_approx(m_run - m_blk);
          l_run *= f;
          m_run = m_blk;
        }
        // O (complete up to the previous block: its P*V finished before this S was
        // committed) is rescaled by the whole warp when any of its rows needs it;
        // tcgen05.ld/st are warp-collective.
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(trow + kOCol + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(trow + kOCol + c * 32, o);
          }
        }
        const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
        // p = 2^(s * scale * log2e - m): POLY16 of every 16 columns on the FMA pipe,
        // the rest on MUFU; eight partial row sums; P packed to bf16 pairs.
        float ls[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) ls[k] = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 128; i += 2) {
          const float x0 = fmaf(SV(i), sl2, nm);
          const float x1 = fmaf(SV(i + 1), sl2, nm);
          const float p0 = (!MASKED && (i & 15) >= 16 - POLY16) ? exp2_poly3(x0) : ex2_approx(x0);
          const float p1 = (!MASKED && ((i + 1) & 15) >= 16 - POLY16) ? exp2_poly3(x1) : ex2_approx(x1);
          ls[i & 7] += p0;
          ls[(i + 1) & 7] += p1;
          pk[i >> 1] = pack_bf16x2(p0, p1);
        }
#undef SV
        tmem_st32_at<0>(trow + kSCol, pk);
        tmem_st32_at<32>(trow + kSCol + 32, pk);
        l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(sb + S::kPFull);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 rows (tiled order)
      ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kOFull, it & 1, wc, 8));
      if (!ok) break;
      tc_fence_after();
      uint32_t o[D];
      tmem_ld32_at<0>(trow + kOCol, o);
      tmem_ld32_at<32>(trow + kOCol + 32, o);
      if constexpr (D == 128) {
        tmem_ld32_at<64>(trow + kOCol + 64, o);
        tmem_ld32_at<96>(trow + kOCol + 96, o);
      }
      tmem_wait_ld();
      tc_fence_before();
      const float inv_l = 1.0f / l_run;
      const int32_t qrow = item.q_row0 + row;
      if (qrow < p.L) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<int64_t>(item.bh) * p.L + qrow) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 v4;
          v4.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv_l, __uint_as_float(o[8 * c + 1]) * inv_l);
          v4.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv_l, __uint_as_float(o[8 * c + 3]) * inv_l);
          v4.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv_l, __uint_as_float(o[8 * c + 5]) * inv_l);
          v4.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv_l, __uint_as_float(o[8 * c + 7]) * inv_l);
          dst[c] = v4;
        }
      }
    }
  } else {
    setmaxnreg_dec<kRegsOther>();  // warps 6-7: no role
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

// Self-test kernel for the bounded wait: waits on a barrier nobody arrives on.
__global__ void selftest_wait_kernel(int32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  WaitCtx wc{&abort_flag, err, limit_ns};
  mbar_wait(b, 0, wc, 0x7F);
  __syncthreads();
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Tensor map of a [BH, L, d] bf16 tensor with a 128-row x 64-column box, 128-byte
// swizzle; rows past L read as zero.
bool make_tmap(CUtensorMap* m, const void* base, int64_t bh, int64_t L, int d) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kBlockRows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool MASKED, int POLY16>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                     cudaStream_t stream) {
  auto kern = sta_fwd_kernel<D, MASKED, POLY16>;
  const int smem = Smem<D>::kDynBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // setmaxnreg redistributes the registers a CTA is launched with; the split in
  // the kernel adds up only if the kernel was compiled to exactly kLaunchRegs.
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // Two CTAs per SM by design (registers, shared memory and TMEM - 2 x 256 of 512
  // columns - all allow exactly two).  CTAs share nothing, so a grid larger than
  // what is resident only queues.
  int grid = sms * 2;
  if (grid > p.n_items) grid = p.n_items;
  if (grid < 1) return cudaSuccess;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

// Share of exponentials computed on the FMA pipe, in sixteenths (the rest use
// MUFU ex2).  STA_EXP_POLY16 in the environment overrides the default; only the
// instantiated values are accepted.
int exp_poly16() {
  static int v = [] {
    const char* e = std::getenv("STA_EXP_POLY16");
    int x = e ? std::atoi(e) : kDefaultPoly16;
    if (x != 0 && x != 4 && x != 6 && x != 8) x = kDefaultPoly16;
    return x;
  }();
  return v;
}

template <int D, bool MASKED>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                     cudaStream_t stream) {
  if (MASKED) return launch_t<D, MASKED, 0>(tq, tk, tv, p, stream);
  switch (exp_poly16()) {
    case 0: return launch_t<D, MASKED, 0>(tq, tk, tv, p, stream);
    case 4: return launch_t<D, MASKED, 4>(tq, tk, tv, p, stream);
    case 8: return launch_t<D, MASKED, 8>(tq, tk, tv, p, stream);
    case 6: return launch_t<D, MASKED, 6>(tq, tk, tv, p, stream);
    default: return launch_t<D, MASKED, 0>(tq, tk, tv, p, stream);
  }
}

}  // namespace

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, int32_t batch,
                             int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& s, float scale,
                             int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, bh, g.L, d) || !make_tmap(&tk, k, bh, g.L, d) || !make_tmap(&tv, v, bh, g.L, d))
    return cudaErrorInvalidValue;
  FwdParams p;
  p.items = s.items;
  p.kv_rows = s.kv_rows;
  p.head_win = s.head_win;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.n_items = s.n_items;
  p.heads = heads;
  p.L = static_cast<int32_t>(g.L);
  p.nT = g.nT; p.nH = g.nH; p.nW = g.nW;
  p.ntile = g.ntile;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err_flag;
  p.limit_ns = limit_ns;
  if (d == 128) {
    return s.masked ? launch_d<128, true>(tq, tk, tv, p, stream) : launch_d<128, false>(tq, tk, tv, p, stream);
  }
  return s.masked ? launch_d<64, true>(tq, tk, tv, p, stream) : launch_d<64, false>(tq, tk, tv, p, stream);
}

cudaError_t launch_selftest_wait(int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(err_flag, limit_ns);
  return cudaGetLastError();
}

}  // namespace sta
