// attention.cu - Sliding Tile Attention forward for sm_100a.
//
// "Fast Video Generation with Sliding Tile Attention": each query tile attends
// densely to the key tiles of its window (abstract; summary page, "Method
// details"), blocks are either fully attended or skipped (summary page, "Core
// innovation"), and the kernel is built around asynchronous loads and block
// management (summary page, "AI overview").  On B200 that becomes:
//
//   * a persistent grid of one CTA per SM; each CTA runs two lanes, each lane a
//     block of 128 query rows (one work item of the host window enumerator) at a
//     time;
//   * warp 8, the producer, streams each lane's Q once per item and then only
//     the key and value blocks of the lane's window into a four-stage shared
//     memory ring with TMA (128-byte swizzle, completion on mbarriers);
//   * warp 9 issues every tcgen05 MMA from one thread: S = Q K^T (both operands
//     in shared memory, fp32 accumulator in TMEM) and O += P V (P read from TMEM
//     where it overwrote S, V from shared memory, O in TMEM);
//   * warps 0-3 (lane 0) and 4-7 (lane 1), one query row per thread, TMEM lane
//     = row, run the online softmax in fp32: row max, p = 2^(s*scale*log2e - m),
//     row sum, P rounded to bf16 and written back to TMEM; O is rescaled only
//     when the running max grows by more than 2^8 (the result is unchanged: O
//     and the row sum always carry the same factor); the epilogue divides by the
//     row sum and writes bf16 rows.
//
// The producer and the MMA issuer walk the same fixed sequence of turns,
// alternating lanes: a turn issues a lane's P*V for block j and its Q*K^T for
// block j+1.  The tensor core therefore always has the other lane's work queued
// while one lane's softmax runs (ping-pong), and the load order equals the
// consumption order, so one ring serves both lanes.
//
// With Ntile a multiple of 128 no element mask exists at all.  Otherwise
// (small tiles, ragged tails) the softmax masks whole key tiles outside the
// row's window and keys past L.  Every wait is bounded (see ptx.cuh): a stuck
// pipeline records an error code and the CTA drains and exits.
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

constexpr int kLanes = 2;
constexpr int kThreads = 384;       // warps 0-3 / 4-7 softmax of lane 0 / 1, 8-9 producers, 10-11 MMA issuers
constexpr int kProducerWarp0 = 8;   // + lane
constexpr int kMmaWarp0 = 10;       // + lane; warp 10 also owns the TMEM allocation
constexpr int kStages = 2;          // per-lane key/value ring stages (K_j, V_j, K_j+1, ... in order)
constexpr int kTmemCols = 512;      // lane l: S at 256 l, O at 256 l + 128
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Register split: launched at 168 per thread (384 threads, one CTA per SM);
// the two softmax warpgroups take 208 each, the producer/MMA warpgroup keeps 88:
// 2 * 128 * 208 + 128 * 88 = 384 * 168.
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsOther = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == kThreads * kLaunchRegs,
              "register split must match the launch");
constexpr int kDefaultPoly8 = 0;

struct FwdParams {
  const WorkItem* items;
  const int32_t* kv_rows;
  const int32_t* kv_mask_id; // per kv_rows entry: -1 or a key-validity mask (padded latents), or null
  const uint32_t* kv_masks;  // 4 words per mask
  const int16_t* head_win;   // [heads][4]
  __nv_bfloat16* out;        // [BH, L, d] tiled order
  int32_t n_items;
  int32_t heads;
  int32_t L;
  int32_t nT, nH, nW;
  int32_t ntile;
  // raster-order tensors: grid, tile, frames per 128-row slab
  int32_t T, H, W, tt, th, tw, bt;
  float scale_log2;          // scale * log2(e)
  int32_t* err;
  uint64_t limit_ns;
};

template <int D>
struct Smem {
  static constexpr int kBlockBytes = kBlockRows * D * 2;  // one 128-row block of Q, K or V
  static constexpr int kQ0 = 0;                            // lane l's Q at kQ0 + l * kBlockBytes
  static constexpr int kStage0 = kLanes * kBlockBytes;     // lane l's stage s at kStage0 + (l * kStages + s) * kBlockBytes
  static constexpr int kBar = kStage0 + kLanes * kStages * kBlockBytes;
  // per-lane barriers (8 bytes each), lane l's copy at + l * kBarStride
  static constexpr int kQFull = 0;
  static constexpr int kQEmpty = 8;
  static constexpr int kKvFull = 16;                       // [stage]
  static constexpr int kKvEmpty = kKvFull + 8 * kStages;   // [stage]
  static constexpr int kSFull = kKvEmpty + 8 * kStages;
  static constexpr int kPLo = kSFull + 8;                  // P of keys 0-63 written
  static constexpr int kPHi = kPLo + 8;                    // P of keys 64-127 written
  static constexpr int kOFull = kPHi + 8;
  static constexpr int kDrain = kOFull + 8;
  static constexpr int kTurn = kDrain + 8;                 // this lane may run its exponentials
  static constexpr int kBarStride = kTurn + 8;
  static constexpr int kTmemSlot = kBar + kLanes * kBarStride;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kEnd = kAbort + 4;
  static constexpr int kDynBytes = kEnd + 1024;  // + slack to align the base to 1024
  static_assert(kDynBytes <= 227 * 1024, "shared memory budget");
};

// TMA coordinates (x, w, h, t) of the 128-row slab that starts at tiled row
// `row` of the (padded) latent, for raster-order tensors [BH, T, H, W, d].
struct SlabCoord {
  int32_t w, h, t;
};
__device__ __forceinline__ SlabCoord slab_coord(const FwdParams& p, int32_t row) {
  const int32_t tile = row / p.ntile;
  const int32_t b = (row - tile * p.ntile) / kBlockRows;
  const int32_t at = tile / (p.nH * p.nW), ah = (tile / p.nW) % p.nH, aw = tile % p.nW;
  return SlabCoord{aw * p.tw, ah * p.th, at * p.tt + b * p.bt};
}

// Item k of lane l of CTA c is (k * gridDim.x + c) * 2 + l: at any time the CTAs
// work on adjacent items (neighbouring query blocks, overlapping windows).
__device__ __forceinline__ int32_t lane_item(int32_t k, int lane) {
  return (k * static_cast<int32_t>(gridDim.x) + static_cast<int32_t>(blockIdx.x)) * kLanes + lane;
}

template <int D, bool MASKED, int POLY8, bool RASTER>
__global__ void __launch_bounds__(kThreads, 1)
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
    for (int l = 0; l < kLanes; ++l) {
      const uint32_t b = sb + S::kBar + l * S::kBarStride;
      mbar_init(b + S::kQFull, 1);
      mbar_init(b + S::kQEmpty, 1);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(b + S::kKvFull + 8 * s, 1);
        mbar_init(b + S::kKvEmpty + 8 * s, 1);
      }
      mbar_init(b + S::kSFull, 1);
      mbar_init(b + S::kPLo, 4);   // one arrival per softmax warp
      mbar_init(b + S::kPHi, 4);
      mbar_init(b + S::kOFull, 1);
      mbar_init(b + S::kDrain, 1);
      mbar_init(b + S::kTurn, 4);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp0) {
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

  if (warp == kProducerWarp0 || warp == kProducerWarp0 + 1) {
    // ------------------------------------------------------------ producer of one lane
    setmaxnreg_dec<kRegsOther>();
    const int ln = warp - kProducerWarp0;
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint32_t bars = sb + S::kBar + ln * S::kBarStride;
      const uint32_t qdst = sb + S::kQ0 + ln * kBlockBytes;
      const uint32_t ring = sb + S::kStage0 + ln * kStages * kBlockBytes;
      uint32_t kv_seq = 0, q_loads = 0;
      bool ok = true;
      // one key or value block into the lane's next ring stage
      auto load_block = [&](const CUtensorMap* m, int32_t row, int32_t bh) -> bool {
        const uint32_t st = kv_seq % kStages;
        if (!mbar_wait(bars + S::kKvEmpty + 8 * st, ((kv_seq / kStages) & 1) ^ 1, wc, 2)) return false;
        const uint32_t dst = ring + st * kBlockBytes;
        const uint32_t full = bars + S::kKvFull + 8 * st;
        mbar_arrive_expect_tx(full, kBlockBytes);
        if constexpr (RASTER) {
          const SlabCoord c = slab_coord(p, row);
          for (int b = 0; b < kBoxes; ++b) tma_load_5d(dst + b * kBoxBytes, m, full, b * 64, c.w, c.h, c.t, bh);
        } else {
          for (int b = 0; b < kBoxes; ++b) tma_load_3d(dst + b * kBoxBytes, m, full, b * 64, row, bh);
        }
        ++kv_seq;
        return true;
      };
      for (int32_t k = 0; ok; ++k) {
        const int32_t idx = lane_item(k, ln);
        if (idx >= p.n_items) break;
        const WorkItem item = p.items[idx];
        ok = mbar_wait(bars + S::kQEmpty, (q_loads & 1) ^ 1, wc, 1);
        if (!ok) break;
        ++q_loads;
        mbar_arrive_expect_tx(bars + S::kQFull, kBlockBytes);
        if constexpr (RASTER) {
          const SlabCoord c = slab_coord(p, item.q_row0);
          for (int b = 0; b < kBoxes; ++b)
            tma_load_5d(qdst + b * kBoxBytes, &tm_q, bars + S::kQFull, b * 64, c.w, c.h, c.t, item.bh);
        } else {
          for (int b = 0; b < kBoxes; ++b)
            tma_load_3d(qdst + b * kBoxBytes, &tm_q, bars + S::kQFull, b * 64, item.q_row0, item.bh);
        }
        for (int32_t j = 0; j < item.kv_len && ok; ++j) {
          const int32_t row = p.kv_rows[item.kv_off + j];
          ok = load_block(&tm_k, row, item.bh) && load_block(&tm_v, row, item.bh);
        }
      }
      // Drain: every load issued has landed before the CTA may exit.  Waiting on a
      // phase that already completed returns at once.
      if (q_loads > 0) mbar_wait_drain(bars + S::kQFull, (q_loads - 1) & 1, p.limit_ns);
      for (uint32_t s = 0; s < kStages && s < kv_seq; ++s) {
        const uint32_t last = kv_seq - 1 - ((kv_seq - 1 - s) % kStages);  // last sequence number on stage s
        mbar_wait_drain(bars + S::kKvFull + 8 * s, (last / kStages) & 1, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp0 || warp == kMmaWarp0 + 1) {
    // ------------------------------------------------------------ MMA issuer of one lane
    setmaxnreg_dec<kRegsOther>();
    const int ln = warp - kMmaWarp0;
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t bars = sb + S::kBar + ln * S::kBarStride;
      const uint32_t tS = tmem + 256 * ln, tO = tS + 128;
      // Shared-memory descriptors differ only in the start-address field (bits 0-13,
      // address >> 4; every address here is below 256 KB, so adding an offset never
      // carries out of the field): one base descriptor per role plus offsets.
      const uint64_t dq = sdesc_sw128(sb + S::kQ0 + ln * kBlockBytes, 16, 1024);        // K-major (Q)
      const uint32_t ring = sb + S::kStage0 + ln * kStages * kBlockBytes;
      const uint64_t dk0 = sdesc_sw128(ring, 16, 1024);                                   // K-major (K)
      const uint64_t dv0 = sdesc_sw128(ring, kBlockRows * 128, 1024);                     // MN-major (V)
      constexpr uint32_t kStageStep = kBlockBytes >> 4;
      // slice k16 of a K-major block: 64-column boxes of 16 KB, 32 bytes per 16 columns
      auto koff = [](int k16) -> uint64_t { return static_cast<uint64_t>(((k16 >> 2) * 16384 + (k16 & 3) * 32) >> 4); };
      auto wait_stage = [&](uint32_t seq, int site) -> bool {
        return mbar_wait(bars + S::kKvFull + 8 * (seq % kStages), (seq / kStages) & 1, wc, site);
      };
      // S = Q K^T from ring stage st
      auto issue_qk = [&](uint32_t st) {
        const uint64_t dk = dk0 + st * kStageStep;
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16)
          umma_ss(tS, dq + koff(k16), dk + koff(k16), idesc_qk, k16 > 0 ? 1u : 0u);
        umma_commit(bars + S::kKvEmpty + 8 * st);
      };
      // O += P V for keys [64 h, 64 h + 64) of ring stage st (16 keys = 2 KB per slice)
      auto issue_pv_half = [&](uint32_t st, int h, bool accumulate) {
        const uint64_t dv = dv0 + st * kStageStep;
#pragma unroll
        for (int k16 = 4 * h; k16 < 4 * h + 4; ++k16)
          umma_ts(tO, tS + k16 * 8, dv + static_cast<uint64_t>(k16 * (2048 >> 4)), idesc_pv,
                  (accumulate || k16 > 0) ? 1u : 0u);
      };
      uint32_t kv_seq = 0, p_waits = 0;
      bool ok = true;
      for (int32_t k = 0; ok; ++k) {
        const int32_t idx = lane_item(k, ln);
        if (idx >= p.n_items) break;
        const int32_t n = p.items[idx].kv_len;
        ok = mbar_wait(bars + S::kQFull, k & 1, wc, 3) && wait_stage(kv_seq, 4);
        if (!ok) break;
        tc_fence_after();
        issue_qk(kv_seq % kStages);  // S_0
        ++kv_seq;
        if (n == 1) umma_commit(bars + S::kQEmpty);
        umma_commit(bars + S::kSFull);
        for (int32_t j = 0; j < n && ok; ++j) {
          // V_j and K_j+1 were loaded ahead: wait for them first, so that only the
          // softmax hand-off (P_j) stands between S_j and these MMAs.
          const bool has_k = j + 1 < n;
          ok = wait_stage(kv_seq, 6) && (!has_k || wait_stage(kv_seq + 1, 4)) &&
               mbar_wait(bars + S::kPLo, p_waits & 1, wc, 5);
          if (!ok) break;
          tc_fence_after();
          // O += P_j V_j, the first 64 keys as soon as their P is written
          issue_pv_half(kv_seq % kStages, 0, j > 0);
          ok = mbar_wait(bars + S::kPHi, p_waits & 1, wc, 10);
          ++p_waits;
          if (!ok) break;
          tc_fence_after();
          issue_pv_half(kv_seq % kStages, 1, true);
          umma_commit(bars + S::kKvEmpty + 8 * (kv_seq % kStages));
          ++kv_seq;
          if (has_k) {
            issue_qk(kv_seq % kStages);  // S_j+1 (overwrites P_j after P_j V_j, in issue order)
            ++kv_seq;
            if (j + 2 == n) umma_commit(bars + S::kQEmpty);
            umma_commit(bars + S::kSFull);
          }
        }
        if (ok) umma_commit(bars + S::kOFull);
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      umma_commit(bars + S::kDrain);
      mbar_wait_drain(bars + S::kDrain, 0, p.limit_ns);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax + epilogue
    setmaxnreg_inc<kRegsSoftmax>();
    const int ln = warp >> 2;                             // this warpgroup's lane
    const int row = threadIdx.x & 127;                    // TMEM lane = query row in the block
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + 256 * ln;
    const uint32_t tS = trow, tO = trow + 128;
    const uint32_t bars = sb + S::kBar + ln * S::kBarStride;
    const uint32_t bar_s = bars + S::kSFull, bar_plo = bars + S::kPLo, bar_phi = bars + S::kPHi,
                   bar_o = bars + S::kOFull;
    const float sl2 = p.scale_log2;
    uint32_t sphase = 0, it = 0;
    bool ok = true;
    // Turn token: the two lanes' exponential loops alternate (lane 0 block b after
    // lane 1 block b-1, lane 1 block b after lane 0 block b) while both have blocks,
    // so that each has the SM's MUFU units to itself and the other lane's MMAs run
    // meanwhile.  A lane never gets more than one phase ahead, so parity waits are
    // exact.
    int32_t other_total = 0;
    for (int32_t kk = 0;; ++kk) {
      const int32_t oi = lane_item(kk, ln ^ 1);
      if (oi >= p.n_items) break;
      other_total += p.items[oi].kv_len;
    }
    const uint32_t my_turn = bars + S::kTurn;
    const uint32_t their_turn = sb + S::kBar + (ln ^ 1) * S::kBarStride + S::kTurn;
    for (int32_t k = 0; ok; ++k, ++it) {
      const int32_t idx = lane_item(k, ln);
      if (idx >= p.n_items) break;
      const WorkItem item = p.items[idx];
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
        ok = __all_sync(0xffffffffu, mbar_wait(bar_s, sphase & 1, wc, 7));
        const int32_t blk = static_cast<int32_t>(sphase);  // blocks of this lane before this one
        ++sphase;
        if (!ok) break;
        tc_fence_after();
        // The whole score row (128 fp32) in one round trip.
        uint32_t r[128];
        tmem_ld32_at<0>(tS, r);
        tmem_ld32_at<32>(tS + 32, r);
        tmem_ld32_at<64>(tS + 64, r);
        tmem_ld32_at<96>(tS + 96, r);
        tmem_wait_ld();
        if (!MASKED && p.kv_mask_id != nullptr) {
          // padded latent: keys of pad tokens in this block do not exist
          const int32_t mid = p.kv_mask_id[item.kv_off + j];
          if (mid >= 0) {
            const uint4 mw = *reinterpret_cast<const uint4*>(p.kv_masks + 4 * mid);
            const uint32_t words[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (!((words[i >> 5] >> (i & 31)) & 1u)) r[i] = __float_as_uint(-INFINITY);
          }
        }
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
        for (int q = 0; q < 8; ++q) {
          float a = max3f(SV(q), SV(q + 8), SV(q + 16));
#pragma unroll
          for (int t = 24; t < 120; t += 16) a = max3f(a, SV(q + t), SV(q + t + 8));
          mx8[q] = fmaxf(a, SV(q + 120));
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
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tO + c * 32, o);
          }
        }
        const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
        {
          const int32_t need = ln == 0 ? blk - 1 : blk;  // the other lane's block to wait for
          if (need >= 0 && need < other_total) {
            ok = __all_sync(0xffffffffu, mbar_wait(my_turn, static_cast<uint32_t>(need & 1), wc, 9));
            if (!ok) break;
          }
        }
        // p = 2^(s * scale * log2e - m): POLY8 of every 8 column pairs on the FMA pipe,
        // the rest on MUFU; partial row sums; P packed to bf16 pairs.  Each half
        // of the row (64 keys) is stored and handed to the MMA issuer on its own, so
        // P V of the first half overlaps the exponentials of the second.
        // x = s * scale * log2e - m and the row sums use packed fp32 pairs (one
        // instruction per two columns); four pair-accumulators break the add chain.
        const uint64_t sl2x2 = f32x2(sl2, sl2), nmx2 = f32x2(nm, nm);
        uint64_t ls2[4] = {0, 0, 0, 0};
        uint32_t pk[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 64 * h; i < 64 * h + 64; i += 2) {
            const uint64_t x2 = fma_f32x2(f32x2(SV(i), SV(i + 1)), sl2x2, nmx2);
            float p0, p1;
            if (!MASKED && ((i >> 1) & 7) >= 8 - POLY8) {
              // x >= -125 is kept by the clamp below; x <= 8 by the rescale threshold
              float x0, x1;
              f32x2_split(x2, x0, x1);
              exp2_poly3_pair(f32x2(fmaxf(x0, -125.f), fmaxf(x1, -125.f)), p0, p1);
            } else {
              float x0, x1;
              f32x2_split(x2, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            ls2[(i >> 1) & 3] = add_f32x2(ls2[(i >> 1) & 3], f32x2(p0, p1));
            pk[i >> 1] = pack_bf16x2(p0, p1);
          }
          // Each warp publishes its P with one elected arrival once all its lanes'
          // TMEM stores are complete (wait::st, fence before the warp sync).
          if (h == 0) {
            tmem_st32_at<0>(tS, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_plo);
          } else {
            if (lane == 0) mbar_arrive(their_turn);  // the other lane may start its exponentials
            tmem_st32_at<32>(tS + 32, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_phi);
          }
        }
#undef SV
        {
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f32x2_split(ls2[0], a0, a1);
          f32x2_split(ls2[1], b0, b1);
          f32x2_split(ls2[2], c0, c1);
          f32x2_split(ls2[3], d0, d1);
          l_run += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        }
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 rows (tiled order)
      ok = __all_sync(0xffffffffu, mbar_wait(bar_o, it & 1, wc, 8));
      if (!ok) break;
      tc_fence_after();
      uint32_t o[D];
      tmem_ld32_at<0>(tO, o);
      tmem_ld32_at<32>(tO + 32, o);
      if constexpr (D == 128) {
        tmem_ld32_at<64>(tO + 64, o);
        tmem_ld32_at<96>(tO + 96, o);
      }
      tmem_wait_ld();
      tc_fence_before();
      const float inv_l = 1.0f / l_run;
      const int32_t qrow = item.q_row0 + row;
      int64_t out_row = -1;  // destination row, or -1 for no real token
      if constexpr (RASTER) {
        const int32_t tile = qrow / p.ntile, local = qrow - tile * p.ntile;
        const int32_t at = tile / (p.nH * p.nW), ah = (tile / p.nW) % p.nH, aw = tile % p.nW;
        const int32_t t = at * p.tt + local / (p.th * p.tw);
        const int32_t hh = ah * p.th + (local / p.tw) % p.th;
        const int32_t w = aw * p.tw + local % p.tw;
        if (t < p.T && hh < p.H && w < p.W)
          out_row = ((static_cast<int64_t>(item.bh) * p.T + t) * p.H + hh) * p.W + w;
      } else if (qrow < p.L) {
        out_row = static_cast<int64_t>(item.bh) * p.L + qrow;
      }
      if (out_row >= 0) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + out_row * D);
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
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp0) tmem_dealloc(tmem, kTmemCols);
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

// Tensor map of a raster-order [BH, T, H, W, d] bf16 tensor whose box is one
// 128-row slab of a tile (bt frames x th x tw tokens) x 64 columns, 128-byte
// swizzle: the box's rows come out in tile-local raster order, the tiled order.
// Coordinates past the grid (pad tokens of a padded latent) read as zero.
bool make_tmap_raster(CUtensorMap* m, const void* base, int64_t bh, const Geometry& g, int d, int bt) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(g.W), static_cast<cuuint64_t>(g.H),
                        static_cast<cuuint64_t>(g.T), static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, row * g.W * g.H * g.T};
  cuuint32_t box[5] = {64, static_cast<cuuint32_t>(g.tw), static_cast<cuuint32_t>(g.th), static_cast<cuuint32_t>(bt), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool MASKED, int POLY8, bool RASTER>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                     cudaStream_t stream) {
  auto kern = sta_fwd_kernel<D, MASKED, POLY8, RASTER>;
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
  // One CTA per SM (two lanes of 128 query rows each; 512 TMEM columns).
  int grid = sms;
  const int pairs = (p.n_items + kLanes - 1) / kLanes;
  if (grid > pairs) grid = pairs;
  if (grid < 1) return cudaSuccess;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

// Share of exponentials computed on the FMA pipe, in column pairs out of every 8
// (the rest use MUFU ex2).  STA_EXP_POLY8 in the environment overrides the
// default; only the instantiated values (0, 1) are accepted.
int exp_poly8() {
  static int v = [] {
    const char* e = std::getenv("STA_EXP_POLY8");
    int x = e ? std::atoi(e) : kDefaultPoly8;
    if (x < 0 || x > 1) x = kDefaultPoly8;
    return x;
  }();
  return v;
}

template <int D, bool MASKED, bool RASTER>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                     cudaStream_t stream) {
  if (MASKED) return launch_t<D, MASKED, 0, RASTER>(tq, tk, tv, p, stream);
  if (exp_poly8() == 1) return launch_t<D, MASKED, 1, RASTER>(tq, tk, tv, p, stream);
  return launch_t<D, MASKED, 0, RASTER>(tq, tk, tv, p, stream);
}

FwdParams make_params(void* out, int32_t heads, const Geometry& g, const DeviceSchedule& s, float scale,
                      int32_t* err_flag, uint64_t limit_ns) {
  FwdParams p;
  p.items = s.items;
  p.kv_rows = s.kv_rows;
  p.kv_mask_id = s.kv_mask_id;
  p.kv_masks = s.kv_masks;
  p.head_win = s.head_win;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.n_items = s.n_items;
  p.heads = heads;
  p.L = static_cast<int32_t>(g.L);
  p.nT = g.nT; p.nH = g.nH; p.nW = g.nW;
  p.ntile = g.ntile;
  p.T = g.T; p.H = g.H; p.W = g.W;
  p.tt = g.tt; p.th = g.th; p.tw = g.tw;
  p.bt = (g.th * g.tw) > 0 ? kBlockRows / (g.th * g.tw) : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err_flag;
  p.limit_ns = limit_ns;
  return p;
}

}  // namespace

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, int32_t batch,
                             int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& s, float scale,
                             int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, bh, g.L, d) || !make_tmap(&tk, k, bh, g.L, d) || !make_tmap(&tv, v, bh, g.L, d))
    return cudaErrorInvalidValue;
  const FwdParams p = make_params(out, heads, g, s, scale, err_flag, limit_ns);
  if (d == 128)
    return s.masked ? launch_d<128, true, false>(tq, tk, tv, p, stream) : launch_d<128, false, false>(tq, tk, tv, p, stream);
  return s.masked ? launch_d<64, true, false>(tq, tk, tv, p, stream) : launch_d<64, false, false>(tq, tk, tv, p, stream);
}

cudaError_t launch_attention_raster(const void* q, const void* k, const void* v, void* out, int32_t batch,
                                    int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& s,
                                    float scale, int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  if (s.masked || !raster_tile_ok(g.tt, g.th, g.tw) || g.ntile % kBlockRows != 0) return cudaErrorInvalidValue;
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  const int bt = kBlockRows / (g.th * g.tw);
  CUtensorMap tq, tk, tv;
  if (!make_tmap_raster(&tq, q, bh, g, d, bt) || !make_tmap_raster(&tk, k, bh, g, d, bt) ||
      !make_tmap_raster(&tv, v, bh, g, d, bt))
    return cudaErrorInvalidValue;
  const FwdParams p = make_params(out, heads, g, s, scale, err_flag, limit_ns);
  if (d == 128) return launch_d<128, false, true>(tq, tk, tv, p, stream);
  return launch_d<64, false, true>(tq, tk, tv, p, stream);
}

cudaError_t launch_selftest_wait(int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(err_flag, limit_ns);
  return cudaGetLastError();
}

}  // namespace sta
