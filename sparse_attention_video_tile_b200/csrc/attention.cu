// attention.cu - Sliding Tile Attention forward for sm_100a.
//
// "Fast Video Generation with Sliding Tile Attention": each query tile attends
// densely to the key tiles of its window (abstract; summary page, "Method
// details"), blocks are either fully attended or skipped (summary page, "Core
// innovation"), and the kernel is built around asynchronous loads and block
// management (summary page, "AI overview").  On B200 that becomes:
//
//   * a persistent grid of one CTA per SM; a CTA works on one block of 128 query
//     rows (one work item of the host window enumerator) at a time, and walks
//     the key blocks of all its items as one stream;
//   * warp 8, the producer, loads each item's Q (two buffers, so the next item's
//     Q arrives early) and the key and value blocks of the windows into a shared
//     memory ring with TMA (128-byte swizzle, completion on mbarriers), in the
//     order the MMA issuers consume them;
//   * warp 10 issues S = Q K^T (both operands in shared memory, fp32
//     accumulator in TMEM) and warp 9 O += P V (P read from TMEM where it
//     overwrote S, V from shared memory, O in TMEM), one thread each: an MMA
//     issue returns at the tensor core's execution rate, so one issuer's
//     barrier waits and commits are covered by the other's MMAs.  S has three
//     TMEM buffers: S of block g+3 is issued as soon as P V of block g has
//     read P from its buffer, so the scores of the next two blocks are ready
//     while the softmax works on block g;
//   * warps 0-7 run the online softmax in fp32: TMEM lane = query row, and the
//     two warps w and w+4 of TMEM lane quadrant w take the blocks of the CTA's
//     stream alternately, each handling whole rows (all 128 keys) of its blocks,
//     so one warp's exponentials overlap the other's loads and hand-offs on the
//     sub-partition's MUFU unit.  A warp computes p = 2^(s*scale*log2e - m),
//     keeps its part of the row sum, and writes P (bf16) over the first columns
//     of each half of S.  The running max m is only a reference point against
//     overflow: it is the exact row max of the item's first block, and a later
//     block that exceeds it is still exact as long as p stays finite.  Each
//     block publishes which rows' reference it set or raised (block row sums
//     above 2^64 redo the block with their exact max, with O and the row sums
//     rescaled together, so O / l is unchanged); the other warp reads that
//     before publishing its next block and redoes rows it computed against the
//     old reference.  The epilogue adds the two warps' sums, divides and writes
//     bf16 rows, each warp half of the head dimension;
//   * warpgroup 2 (warps 8-11: the producer, the two issuers and one idle warp)
//     lowers its register count with setmaxnreg and the two softmax warpgroups
//     raise theirs to 224 (200 in the mixed-layout kernel), so that a softmax
//     thread holds half a row of S, the row's P and its state without spilling.
//
// Every barrier that is waited on with a parity can never run two phases ahead
// of its waiter (the per-buffer S, P and P*V barriers, the Q pair, the ring).
// The issuers wait for the loads that have almost always landed (K and Q for the
// S issuer, V for the P*V issuer where that is safe) before the wait on the
// S -> P -> P*V -> S chain, so that those checks are not on the chain.
// With Ntile a multiple of 128 no element mask exists at all.  Otherwise (small
// tiles, ragged tails) the softmax masks whole key tiles outside the row's
// window and keys past L; padded latents mask the pad keys of boundary blocks.
// Every wait is bounded (see ptx.cuh): a stuck pipeline records an error code
// and the CTA drains and exits.
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

// Builds with STA_DEVICE_CHECKS=1 (the checked library) test every index the
// kernel takes from the schedule or computes from it (work items, key-block rows,
// mask ids, output rows) before using it.  A failed check records 0x200 | code in
// the status word, sets the CTA's abort flag and skips the access; the pipeline
// then drains as after an expired wait.
#ifndef STA_DEVICE_CHECKS
#define STA_DEVICE_CHECKS 0
#endif

namespace sta {
namespace {

using namespace ptx;

constexpr bool kChecks = STA_DEVICE_CHECKS != 0;

constexpr int kThreads = 384;       // warps 0-7 softmax + epilogue, 8 producer, 9-10 MMA issuers, 11 idle
constexpr int kRegsSoftmax = 224;   // setmaxnreg: warpgroups 0-1 (softmax) raise, warpgroup 2 lowers
constexpr int kRegsOther = 56;      // (per layout in the kernel: 200 and 96 for the mixed layout)
constexpr int kRegsAtLaunch = 168;  // 65536 / 384 rounded down to a multiple of 8
constexpr int kProducerWarp = 8;
constexpr int kPvWarp = 9;          // issues O += P V; also owns the TMEM allocation
constexpr int kSWarp = 10;          // issues S = Q K^T
constexpr int kSBufs = 3;           // score buffers in TMEM
constexpr int kTmemCols = 512;      // S buffer b at 128 b, O at kOCol
constexpr int kOCol = 128 * kSBufs;
constexpr float kOverflowSum = 0x1p64f;     // block row sums above this redo the block with its exact max
constexpr int kDefaultPoly8 = 0;

struct FwdParams {
  const WorkItem* items;
  const int32_t* kv_rows;
  const int32_t* kv_mask_id; // per kv_rows entry: -1 or a key-validity mask (padded latents), or null
  const uint32_t* kv_masks;  // 4 words per mask
  const int16_t* head_win;   // [heads][4]
  __nv_bfloat16* out;        // [BH, L, d] tiled order, or raster order
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
  float* lse;                // per-row log-sum-exp (natural log), same row indexing as out, or null
  // sizes for the device checks
  int32_t n_kv_rows;         // entries of kv_rows (and kv_mask_id)
  int32_t n_masks;           // 128-bit masks in kv_masks
  int32_t n_bh;              // batch * heads
  int32_t rows;              // rows per (batch, head) of the tiled order the schedule indexes
};

template <int D>
struct Smem {
  static constexpr int kQBufs = 2;                         // Q buffers (item k in buffer k mod kQBufs)
  static constexpr int kStages = D == 64 ? 8 : 4;          // key/value ring stages
  static constexpr int kBlockBytes = kBlockRows * D * 2;  // one 128-row block of Q, K or V
  static constexpr int kQ = 0;                             // Q buffer b at kQ + b * kBlockBytes
  static constexpr int kStage0 = kQBufs * kBlockBytes;     // stage s at kStage0 + s * kBlockBytes
  static constexpr int kLx = kStage0 + kStages * kBlockBytes;  // float [item parity][half][row]
  static constexpr int kOw = kLx + 2 * 2 * kBlockRows * 4;    // uint32 [block parity][quadrant]
  static constexpr int kOm = kOw + 2 * 4 * 4;                  // float [block parity][row]
  static constexpr int kBar = kOm + 2 * kBlockRows * 4;
  static constexpr int kQFull = kBar;                      // [Q buffer]
  static constexpr int kQEmpty = kQFull + 16;              // [Q buffer]
  static constexpr int kKvFull = kQEmpty + 16;             // [stage]
  static constexpr int kKvEmpty = kKvFull + 8 * kStages;   // [stage]
  static constexpr int kSFull = kKvEmpty + 8 * kStages;    // [S buffer]: S written
  static constexpr int kPFull = kSFull + 8 * kSBufs;       // [S buffer]: P written (8 warps)
  static constexpr int kPvDone = kPFull + 8 * kSBufs;      // [S buffer]: P V of that block completed
  static constexpr int kOut = kPvDone + 8 * kSBufs;        // [lane quadrant]: outcome of each block published
  static constexpr int kLxBar = kOut + 8 * 4;              // [lane quadrant]: half row sums written
  static constexpr int kOFull = kLxBar + 8 * 4;
  static constexpr int kOFree = kOFull + 8;                // every softmax warp done reading an item's O
  static constexpr int kDrain = kOFree + 8;
  static constexpr int kDrainS = kDrain + 8;
  static constexpr int kTmemSlot = kDrainS + 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kEnd = kAbort + 4;
  static constexpr int kDynBytes = kEnd + 1024;  // + slack to align the base to 1024
  static_assert(kDynBytes <= 227 * 1024, "shared memory budget");
  static_assert(kBlockBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
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

// Position in the stream of key blocks of this CTA: item ordinal k (item index
// k * gridDim.x + blockIdx.x; neighbouring CTAs work on neighbouring items, whose
// windows overlap in L2), block j of that item, and g, the block's ordinal over
// all the CTA's items.
struct BlockCursor {
  int32_t k, j, g;
  WorkItem it;
  bool done;
  __device__ __forceinline__ void load(const FwdParams& p) {
    const int32_t idx = k * static_cast<int32_t>(gridDim.x) + static_cast<int32_t>(blockIdx.x);
    done = idx >= p.n_items;
    if (!done) it = p.items[idx];
  }
  __device__ __forceinline__ void start(const FwdParams& p) {
    k = 0;
    j = 0;
    g = 0;
    load(p);
  }
  __device__ __forceinline__ void next(const FwdParams& p) {
    ++g;
    if (++j == it.kv_len) {
      j = 0;
      ++k;
      load(p);
    }
  }
};

// Layout of the tensors the kernel reads and writes (LAYOUT template argument).
constexpr int kTiled = 0;    // q, k, v, out in tiled order
constexpr int kRaster = 1;   // q, k, v, out in raster order: 5-D boxes, raster output rows
constexpr int kMixed = 2;    // q and out in raster order, k and v in the padded latent's tiled order

template <int D, bool MASKED, int POLY8, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 1)
    sta_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using S = Smem<D>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kTmemSlot);

  if (threadIdx.x == 0) {
    for (int b = 0; b < S::kQBufs; ++b) {
      mbar_init(sb + S::kQFull + 8 * b, 1);
      mbar_init(sb + S::kQEmpty + 8 * b, 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sb + S::kKvFull + 8 * s, 1);
      mbar_init(sb + S::kKvEmpty + 8 * s, 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(sb + S::kSFull + 8 * b, 1);
      mbar_init(sb + S::kPFull + 8 * b, 4);    // one arrival per lane quadrant
      mbar_init(sb + S::kPvDone + 8 * b, 1);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(sb + S::kOut + 8 * q, 32);     // every lane of the publishing warp
      mbar_init(sb + S::kLxBar + 8 * q, 64);   // every thread of the pair
    }
    mbar_init(sb + S::kOFull, 1);
    mbar_init(sb + S::kOFree, 256); // one arrival per softmax thread
    mbar_init(sb + S::kDrain, 1);
    mbar_init(sb + S::kDrainS, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kPvWarp) {
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

  // Register split per layout, timed on B200 like the branch placement below: the
  // mixed-layout instantiation runs about 3 % faster with 200 / 96 than with 224 / 56
  // (216 / 64: 2 %; 208 / 80 and 232 / 40 slower).  The split must fit the registers
  // the block was launched with.
  constexpr int kRegsSm = LAYOUT == kMixed ? 200 : kRegsSoftmax;
  constexpr int kRegsOt = LAYOUT == kMixed ? 96 : kRegsOther;
  static_assert(256 * kRegsSm + 128 * kRegsOt <= kThreads * kRegsAtLaunch, "register split above the launch allocation");
  // The two role branches, softmax warps and the rest, as lambdas, so that the order in
  // which they are placed in the code can be chosen per layout (end of the kernel).
  auto other_roles = [&]() {
    setmaxnreg_dec<kRegsOt>();
    if (warp == kProducerWarp) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        uint32_t kv_seq = 0, q_loads[2] = {0, 0};
        bool ok = true;
        // one 128-row block (Q into buffer `dst`, or K/V into the next ring stage);
        // `raster`: the tensor is in raster order, read as 5-D boxes
        auto tma_block = [&](uint32_t dst, const CUtensorMap* m, uint32_t full, int32_t row, int32_t bh, bool raster) {
          if (raster) {
            const SlabCoord c = slab_coord(p, row);
            for (int b = 0; b < kBoxes; ++b) tma_load_5d(dst + b * kBoxBytes, m, full, b * 64, c.w, c.h, c.t, bh);
          } else {
            for (int b = 0; b < kBoxes; ++b) tma_load_3d(dst + b * kBoxBytes, m, full, b * 64, row, bh);
          }
        };
        auto load_ring = [&](const CUtensorMap* m, int32_t row, int32_t bh) -> bool {
          const uint32_t st = kv_seq % kStages;
          if (!mbar_wait(sb + S::kKvEmpty + 8 * st, ((kv_seq / kStages) & 1) ^ 1, wc, 2)) return false;
          const uint32_t full = sb + S::kKvFull + 8 * st;
          mbar_arrive_expect_tx(full, kBlockBytes);
          tma_block(sb + S::kStage0 + st * kBlockBytes, m, full, row, bh, LAYOUT == kRaster);
          ++kv_seq;
          return true;
        };
        // failed device check: record it and stop; the CTA drains as after an expired wait
        auto fail = [&](int code) {
          atomicCAS(p.err, 0, 0x200 | code);
          *abort_flag = 1;
        };
        // row of key block j of the cursor's item, or -1 after a failed check
        auto kv_row = [&](const BlockCursor& c, int code) -> int32_t {
          const int32_t idx = c.it.kv_off + c.j;
          if (kChecks && !(idx >= 0 && idx < p.n_kv_rows)) {
            fail(code);
            return -1;
          }
          const int32_t row = p.kv_rows[idx];
          if (kChecks && !(row >= 0 && row < p.rows && row % kBlockRows == 0)) {
            fail(code + 1);
            return -1;
          }
          return row;
        };
        // K of block (k, j), preceded by the item's Q when j = 0
        auto load_k = [&](const BlockCursor& c) -> bool {
          if (kChecks && !(c.it.bh >= 0 && c.it.bh < p.n_bh && c.it.q_row0 >= 0 && c.it.q_row0 < p.rows &&
                           c.it.q_row0 % kBlockRows == 0 && c.it.kv_len >= 1)) {
            fail(1);
            return false;
          }
          if (c.j == 0) {
            const int qb = c.k % S::kQBufs;
            if (!mbar_wait(sb + S::kQEmpty + 8 * qb, ((c.k / S::kQBufs) & 1) ^ 1, wc, 1)) return false;
            mbar_arrive_expect_tx(sb + S::kQFull + 8 * qb, kBlockBytes);
            tma_block(sb + S::kQ + qb * kBlockBytes, &tm_q, sb + S::kQFull + 8 * qb, c.it.q_row0, c.it.bh,
                      LAYOUT != kTiled);
            ++q_loads[qb];
          }
          const int32_t row = kv_row(c, 2);
          return row >= 0 && load_ring(&tm_k, row, c.it.bh);
        };
        // Order of the loads: K_0, K_1, K_2, then V_g, K_g+3 for g = 0, 1, ... (the S
        // issuer needs K three blocks ahead of the P V issuer's V).
        BlockCursor kc, vc;
        kc.start(p);
        vc.start(p);
        for (int i = 0; i < kSBufs && ok && !kc.done; ++i) {
          ok = load_k(kc);
          kc.next(p);
        }
        while (ok && !vc.done) {
          const int32_t row = kv_row(vc, 4);
          ok = row >= 0 && load_ring(&tm_v, row, vc.it.bh);
          vc.next(p);
          if (ok && !kc.done) {
            ok = load_k(kc);
            kc.next(p);
          }
        }
        // Drain: every load issued has landed before the CTA may exit.  Waiting on a
        // phase that already completed returns at once.
        for (int b = 0; b < S::kQBufs; ++b)
          if (q_loads[b] > 0) mbar_wait_drain(sb + S::kQFull + 8 * b, (q_loads[b] - 1) & 1, p.limit_ns);
        for (uint32_t s = 0; s < kStages && s < kv_seq; ++s) {
          const uint32_t last = kv_seq - 1 - ((kv_seq - 1 - s) % kStages);  // last sequence number on stage s
          mbar_wait_drain(sb + S::kKvFull + 8 * s, (last / kStages) & 1, p.limit_ns);
        }
      }
      __syncwarp();
    } else if (warp == kPvWarp || warp == kSWarp) {
      // ------------------------------------------------------------ MMA issuers
      // A tcgen05.mma issue returns at about the rate the tensor core executes, so
      // whatever else an issuing thread does (barrier waits, commits, bookkeeping)
      // leaves the tensor core idle unless another thread is issuing meanwhile: S
      // and P*V have one issuer each.
      if (lane == 0) {
        // Shared-memory descriptors differ only in the start-address field (bits 0-13,
        // address >> 4; every address here is below 256 KB, so adding an offset never
        // carries out of the field): one base descriptor per role plus offsets.
        constexpr uint32_t kBlockStep = kBlockBytes >> 4;
        // Ring sequence numbers of the loads, in the producer's order K_0, K_1, K_2,
        // V_0, K_3, V_1, ...: K_g is load g + max(0, g - 2) and V_g is load
        // min(G + g, 2 g + 3), G being the number of blocks of this CTA.
        int32_t G = 0;
        for (int32_t k = 0;; ++k) {
          const int32_t idx = k * static_cast<int32_t>(gridDim.x) + static_cast<int32_t>(blockIdx.x);
          if (idx >= p.n_items) break;
          G += p.items[idx].kv_len;
        }
        auto wait_load = [&](uint32_t seq, int site) -> bool {
          return mbar_wait(sb + S::kKvFull + 8 * (seq % kStages), (seq / kStages) & 1, wc, site);
        };
        BlockCursor c;
        c.start(p);
        bool ok = true;
        if (warp == kSWarp) {
          // S_g = Q K_g^T into S buffer g mod 3, once P_g-3 V_g-3 (which reads P_g-3
          // from that buffer) has completed.
          constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
          const uint64_t dq0 = sdesc_sw128(sb + S::kQ, 16, 1024);                         // K-major (Q)
          const uint64_t dk0 = sdesc_sw128(sb + S::kStage0, 16, 1024);                    // K-major (K)
          // slice k16 of a K-major block: 64-column boxes of 16 KB, 32 bytes per 16 columns
          auto koff = [](int k16) -> uint64_t {
            return static_cast<uint64_t>(((k16 >> 2) * 16384 + (k16 & 3) * 32) >> 4);
          };
          for (; ok && !c.done; c.next(p)) {
            const int32_t g = c.g;
            const int b = g % kSBufs;
            const int qb = c.k % S::kQBufs;
            const uint32_t seq = static_cast<uint32_t>(g + (g > 2 ? g - 2 : 0));
            // K_g and Q first: they have almost always landed, and waiting for them while
            // P V of block g-3 still runs keeps them off the S -> P -> P V -> S chain.  (The
            // load before K_g on its stage is K_g-2, which this thread waited for itself.)
            ok = wait_load(seq, 4) && (c.j != 0 || mbar_wait(sb + S::kQFull + 8 * qb, (c.k / S::kQBufs) & 1, wc, 3)) &&
                 (g < kSBufs || mbar_wait(sb + S::kPvDone + 8 * b, ((g / kSBufs) & 1) ^ 1, wc, 14));
            if (!ok) break;
            tc_fence_after();
            const uint32_t st = seq % kStages;
            const uint64_t dq = dq0 + qb * kBlockStep, dk = dk0 + st * kBlockStep;
  #pragma unroll
            for (int k16 = 0; k16 < D / 16; ++k16)
              umma_ss(tmem + 128 * b, dq + koff(k16), dk + koff(k16), idesc_qk, k16 > 0 ? 1u : 0u);
            umma_commit(sb + S::kKvEmpty + 8 * st);
            if (c.j + 1 == c.it.kv_len) umma_commit(sb + S::kQEmpty + 8 * qb);
            umma_commit(sb + S::kSFull + 8 * b);
          }
        } else {
          // O += P_g V_g: keys 0-63 with P in S columns 0-31, keys 64-127 with P in
          // S columns 64-95 (16 keys = 8 columns of P, 2 KB of V per slice)
          constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
          const uint32_t tO = tmem + kOCol;
          const uint64_t dv0 = sdesc_sw128(sb + S::kStage0, kBlockRows * 128, 1024);      // MN-major (V)
          for (; ok && !c.done; c.next(p)) {
            const int32_t g = c.g;
            const int b = g % kSBufs;
            const uint32_t seq = static_cast<uint32_t>(min(G + g, 2 * g + 3));
            // P_g first: it implies S_g ran, so K_g (the load before V_g on a ring stage
            // when g = 1) has landed and the parity wait for V_g cannot pass early.  An
            // item's first product (accumulate = 0) also waits until every softmax warp
            // has read the previous item's O.
            // V_g before P_g only where the load before V_g on its stage is V_g-2, which this
            // thread waited for itself (g >= 2 with V_g at ring load 2g + 3); elsewhere P_g
            // first, which implies S_g ran and so every earlier load on the stage landed.
            if (g >= 2 && seq == static_cast<uint32_t>(2 * g + 3))
              ok = wait_load(seq, 6) && mbar_wait(sb + S::kPFull + 8 * b, (g / kSBufs) & 1, wc, 5);
            else
              ok = mbar_wait(sb + S::kPFull + 8 * b, (g / kSBufs) & 1, wc, 5) && wait_load(seq, 6);
            ok = ok && (c.j != 0 || c.k == 0 || mbar_wait(sb + S::kOFree, static_cast<uint32_t>(c.k - 1) & 1, wc, 15));
            if (!ok) break;
            tc_fence_after();
            const uint32_t st = seq % kStages;
            const uint64_t dv = dv0 + st * kBlockStep;
            const uint32_t tP = tmem + 128 * b;
  #pragma unroll
            for (int k16 = 0; k16 < 8; ++k16)
              umma_ts(tO, tP + (k16 >> 2) * 64 + (k16 & 3) * 8, dv + static_cast<uint64_t>(k16 * (2048 >> 4)), idesc_pv,
                      (c.j > 0 || k16 > 0) ? 1u : 0u);
            umma_commit(sb + S::kKvEmpty + 8 * st);
            umma_commit(sb + S::kPvDone + 8 * b);
            if (c.j + 1 == c.it.kv_len) umma_commit(sb + S::kOFull);
          }
        }
        // Drain: all MMAs issued by this thread complete before TMEM is freed.
        const uint32_t drain = sb + (warp == kSWarp ? S::kDrainS : S::kDrain);
        umma_commit(drain);
        mbar_wait_drain(drain, 0, p.limit_ns);
      }
      __syncwarp();
    }
  };
  auto softmax_role = [&]() {
    setmaxnreg_inc<kRegsSm>();
    // ------------------------------------------------------------ softmax + epilogue
    // Warps w and w+4 share the rows of TMEM lane quadrant w and take the blocks of
    // the CTA's stream alternately (block g by the warp with h = g mod 2), each
    // handling whole rows (all 128 keys) of its blocks: while one runs its
    // exponentials, the other loads, checks and hands over, so the sub-partition's
    // MUFU unit stays busy.
    const int h = warp >> 2;
    const int quad = warp & 3;                            // TMEM lane quadrant
    const int row = quad * 32 + lane;                     // TMEM lane = query row in the block
    const uint32_t tlane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t tOrow = tlane + kOCol;                 // the row's O
    const uint32_t tO = tOrow + h * (D / 2);              // this warp's half of O in the epilogue
    const uint32_t bar_out = sb + S::kOut + 8 * quad, bar_lx = sb + S::kLxBar + 8 * quad;
    uint32_t* oword = reinterpret_cast<uint32_t*>(smem + S::kOw);   // [block parity][quadrant]
    float* omax = reinterpret_cast<float*>(smem + S::kOm);          // [block parity][row]
    float* lx = reinterpret_cast<float*>(smem + S::kLx);
    const float sl2 = p.scale_log2;
    const bool pad_masks = !MASKED && p.kv_mask_id != nullptr;
    bool ok = true;
    float m_run = -INFINITY;   // reference max of the row (log2 units), shared by the pair
    float l_run = 0.f;         // this warp's part of the row sum
    bool have_m = false;       // this warp holds the reference max of the current item
    int32_t consumed = -1;     // last block whose outcome (published by the other warp) was read
    int32_t ws_t = 0, ws_h = 0, ws_w = 0, we_t = 0, we_h = 0, we_w = 0;
    // Outcome of block gg, published by the other warp: the rows whose reference
    // max it set or raised, with the new value; l follows the same factor as O.
    auto read_outcome = [&](int32_t gg) -> bool {
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar_out, static_cast<uint32_t>(gg) & 1, wc, 12));
      if (!got) return false;
      const uint32_t word = oword[(gg & 1) * 4 + quad];
      if ((word >> lane) & 1u) {
        const float m_new = omax[(gg & 1) * kBlockRows + row];
        if (m_run != -INFINITY) l_run *= ex2_approx(m_run - m_new);
        m_run = m_new;
      }
      consumed = gg;
      return true;
    };
    auto publish = [&](int32_t gg, uint32_t word) {
      if (lane == 0) oword[(gg & 1) * 4 + quad] = word;
      omax[(gg & 1) * kBlockRows + row] = m_run;
      mbar_arrive(bar_out);   // every lane: its own omax entry
    };
    BlockCursor cur;
    cur.start(p);
    while (ok && !cur.done) {
      const int32_t g = cur.g, j = cur.j;
      const WorkItem& item = cur.it;
      if (j == 0) {
        m_run = -INFINITY;
        l_run = 0.f;
        have_m = false;
        if (kChecks && !(item.bh >= 0 && item.bh < p.n_bh)) {
          atomicCAS(p.err, 0, 0x200 | 7);
          *abort_flag = 1;
          break;
        }
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
      }
      if ((g & 1) == h) {
        const int b = g % kSBufs;
        const uint32_t tS = tlane + 128 * b;
        ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kSFull + 8 * b, (g / kSBufs) & 1, wc, 7));
        if (!ok) break;
        tc_fence_after();
        // Keys [32 c, 32 c + 32) of the block that this row attends, as a bit mask.
        auto mask_word = [&](int c) -> uint32_t {
          uint32_t m = 0xffffffffu;
          if (pad_masks) {
            // padded latent: keys of pad tokens in this block do not exist
            int32_t mid = p.kv_mask_id[item.kv_off + j];
            if (kChecks && mid >= p.n_masks) {
              atomicCAS(p.err, 0, 0x200 | 6);
              *abort_flag = 1;
              mid = -1;
            }
            if (mid >= 0) m = p.kv_masks[4 * mid + c];
          }
          if (MASKED) {
            const int32_t kv_row = p.kv_rows[item.kv_off + j];
            m = 0;
            for (int i = 0; i < 32; ++i) {
              const int32_t key = kv_row + 32 * c + i;
              bool in = key < p.L;
              if (in) {
                const int32_t kt = key / p.ntile;
                const int32_t bt = kt / (p.nH * p.nW), bh_ = (kt / p.nW) % p.nH, bw = kt % p.nW;
                in = bt >= ws_t && bt < we_t && bh_ >= ws_h && bh_ < we_h && bw >= ws_w && bw < we_w;
              }
              if (in) m |= 1u << i;
            }
          }
          return m;
        };
        // Exact row max of S_g, 32 columns at a time (masked keys left out).
        auto exact_max = [&]() -> float {
          float mx = -INFINITY;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(tS + 32 * c, v);
            tmem_wait_ld();
            const uint32_t m = (MASKED || pad_masks) ? mask_word(c) : 0xffffffffu;
            float a[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float x[8];
#pragma unroll
              for (int t = 0; t < 8; ++t)
                x[t] = ((m >> (q + 4 * t)) & 1u) ? __uint_as_float(v[q + 4 * t]) : -INFINITY;
              a[q] = max3f(max3f(x[0], x[1], x[2]), max3f(x[3], x[4], x[5]), fmaxf(x[6], x[7]));
            }
            mx = max3f(mx, fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
          }
          return mx;
        };
        // p = 2^(s * scale * log2e - m) for the whole row, 64 keys at a time: POLY8
        // of every 8 column pairs on the FMA pipe, the rest on MUFU; x and the row
        // sums use packed fp32 pairs; P packed to bf16 pairs into pk[32 half + i].
        // Returns the block's row sum.
        uint32_t pk[64];
        auto exps = [&]() -> float {
          const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
          const uint64_t sl2x2 = f32x2(sl2, sl2), nmx2 = f32x2(nm, nm);
          uint64_t ls2[4] = {0, 0, 0, 0};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t r[64];
            tmem_ld32_at<0>(tS + 64 * hh, r);
            tmem_ld32_at<32>(tS + 64 * hh + 32, r);
            tmem_wait_ld();
            if (MASKED || pad_masks) {
              const uint32_t m0 = mask_word(2 * hh), m1 = mask_word(2 * hh + 1);
#pragma unroll
              for (int i = 0; i < 64; ++i)
                if (!((((i < 32) ? m0 : m1) >> (i & 31)) & 1u)) r[i] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              const uint64_t x2 = fma_f32x2(f32x2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), sl2x2, nmx2);
              float p0, p1;
              float x0, x1;
              f32x2_split(x2, x0, x1);
              if (!MASKED && ((i >> 1) & 7) >= 8 - POLY8) {
                // inside [-125, 126] for the cubic; larger x overflow the row sum anyway
                exp2_poly3_pair(f32x2(fminf(fmaxf(x0, -125.f), 126.f), fminf(fmaxf(x1, -125.f), 126.f)), p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              ls2[(i >> 1) & 3] = add_f32x2(ls2[(i >> 1) & 3], f32x2(p0, p1));
              pk[32 * hh + (i >> 1)] = pack_bf16x2(p0, p1);
            }
          }
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f32x2_split(ls2[0], a0, a1);
          f32x2_split(ls2[1], b0, b1);
          f32x2_split(ls2[2], c0, c1);
          f32x2_split(ls2[3], d0, d1);
          return ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        };
        uint32_t my_word = 0;
        if (j == 0) {
          // first block of the item: the exact row max is the reference
          const float mx = exact_max();
          m_run = mx * sl2;
          have_m = true;
          my_word = 0xffffffffu;
        } else if (!have_m) {
          // the other warp took the item's first block: its max is the reference
          ok = read_outcome(g - 1);
          if (!ok) break;
          have_m = true;
        }
        float ps = exps();
        // The reference max is only a guard against overflow: a block that exceeds
        // it is still exact as long as p stays finite.  Rows whose block sum exceeds
        // 2^64 (or is not finite), and rows whose reference the other warp raised
        // in block g-1 (read now, before this block is published), redo the block.
        uint32_t stale = 0;
        if (consumed != g - 1 && g > 0) {
          const float m_before = m_run;
          ok = read_outcome(g - 1);
          if (!ok) break;
          stale = __ballot_sync(0xffffffffu, m_run != m_before);
        }
        const uint32_t ovf = (j == 0) ? 0u : __ballot_sync(0xffffffffu, !(ps <= kOverflowSum));
        if ((ovf | stale) != 0) {
          float f = 1.0f;
          if (ovf != 0) {
            const float mx = exact_max();
            if ((ovf >> lane) & 1u) {
              const float m_new = fmaxf(m_run, mx * sl2);
              f = ex2_approx(m_run - m_new);
              l_run *= f;
              m_run = m_new;
            }
            // O holds P V up to block g-1, whose product may still be running
            const int pb = (g + kSBufs - 1) % kSBufs;
            ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kPvDone + 8 * pb, ((g - 1) / kSBufs) & 1, wc, 11));
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tOrow + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
              tmem_st32(tOrow + c * 32, o);
            }
            my_word = ovf;
          }
          ps = exps();
        }
        publish(g, my_word);
        // P over the first 32 columns of each half of S_g
        tmem_st32_at<0>(tS, pk);
        tmem_st32_at<32>(tS + 64, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sb + S::kPFull + 8 * b);
        l_run += ps;
      }
      if (j + 1 == item.kv_len) {
        // epilogue: O / l -> bf16, this warp's half of the head dimension.  The
        // warp that did not take the last block applies its outcome first.
        const int32_t k = cur.k;
        if (consumed != g && (g & 1) != h) {
          ok = read_outcome(g);
          if (!ok) break;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kOFull, static_cast<uint32_t>(k) & 1, wc, 8));
        if (!ok) break;
        tc_fence_after();
        float* lxk = lx + (k & 1) * 2 * kBlockRows;
        lxk[h * kBlockRows + row] = l_run;
        mbar_arrive(bar_lx);
        ok = __all_sync(0xffffffffu, mbar_wait(bar_lx, static_cast<uint32_t>(k) & 1, wc, 13));
        if (!ok) break;
        const float l_tot = l_run + lxk[(h ^ 1) * kBlockRows + row];
        const float inv_l = 1.0f / l_tot;
        const int32_t qrow = item.q_row0 + row;
        int64_t out_row = -1;  // destination row, or -1 for no real token
        if constexpr (LAYOUT != kTiled) {
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
        if (kChecks && out_row >= static_cast<int64_t>(p.n_bh) * (LAYOUT != kTiled ? p.T * p.H * p.W : p.L)) {
          atomicCAS(p.err, 0, 0x200 | 8);
          *abort_flag = 1;
          out_row = -1;
        }
        // log of the row's sum of exp(scale * s): reference max plus log of the sum
        // taken against it, from log2 units to natural log
        if (p.lse != nullptr && h == 0 && out_row >= 0) p.lse[out_row] = (m_run + log2f(l_tot)) * 0.6931471805599453f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (out_row >= 0 ? out_row : 0) * D + h * (D / 2));
#pragma unroll 1
        for (int c32 = 0; c32 < D / 64; ++c32) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c32, o);
          tmem_wait_ld();
          if (out_row >= 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 v4;
              v4.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv_l, __uint_as_float(o[8 * c + 1]) * inv_l);
              v4.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv_l, __uint_as_float(o[8 * c + 3]) * inv_l);
              v4.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv_l, __uint_as_float(o[8 * c + 5]) * inv_l);
              v4.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv_l, __uint_as_float(o[8 * c + 7]) * inv_l);
              dst[4 * c32 + c] = v4;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(sb + S::kOFree);   // this thread's reads of O are complete
      }
      cur.next(p);
    }
  };
  // Same work either way; the placement changes only how the compiler lays out and
  // schedules the softmax loop.  Timed on B200 (launches alternating in one process,
  // identical outputs): the tiled instantiation runs fastest with the softmax branch
  // last; the mixed-layout one 2-3 % faster with it first, and the one-launch raster
  // one faster with it first than last.
  if constexpr (LAYOUT == kTiled) {
    if (warp >= 8) other_roles(); else softmax_role();
  } else {
    if (warp < 8) softmax_role(); else other_roles();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPvWarp) tmem_dealloc(tmem, kTmemCols);
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

template <int D, bool MASKED, int POLY8, int LAYOUT>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                     cudaStream_t stream) {
  auto kern = sta_fwd_kernel<D, MASKED, POLY8, LAYOUT>;
  const int smem = Smem<D>::kDynBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // One CTA per SM (512 TMEM columns), items strided over the grid.
  int grid = sms;
  if (grid > p.n_items) grid = p.n_items;
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

template <int D, bool MASKED, int LAYOUT>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                     cudaStream_t stream) {
  if (MASKED) return launch_t<D, MASKED, 0, LAYOUT>(tq, tk, tv, p, stream);
  if (exp_poly8() == 1) return launch_t<D, MASKED, 1, LAYOUT>(tq, tk, tv, p, stream);
  return launch_t<D, MASKED, 0, LAYOUT>(tq, tk, tv, p, stream);
}

FwdParams make_params(void* out, int32_t batch_heads, int32_t heads, const Geometry& g, const DeviceSchedule& s,
                      float scale, int32_t* err_flag, uint64_t limit_ns) {
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
  p.lse = nullptr;
  p.n_kv_rows = s.n_kv_rows;
  p.n_masks = s.n_masks;
  p.n_bh = batch_heads;
  p.rows = static_cast<int32_t>(g.Lpad);
  return p;
}

}  // namespace

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, int32_t batch,
                             int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& s, float scale,
                             int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream, float* lse) {
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, bh, g.L, d) || !make_tmap(&tk, k, bh, g.L, d) || !make_tmap(&tv, v, bh, g.L, d))
    return cudaErrorInvalidValue;
  FwdParams p = make_params(out, static_cast<int32_t>(bh), heads, g, s, scale, err_flag, limit_ns);
  p.lse = lse;
  if (d == 128)
    return s.masked ? launch_d<128, true, kTiled>(tq, tk, tv, p, stream) : launch_d<128, false, kTiled>(tq, tk, tv, p, stream);
  return s.masked ? launch_d<64, true, kTiled>(tq, tk, tv, p, stream) : launch_d<64, false, kTiled>(tq, tk, tv, p, stream);
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
  const FwdParams p = make_params(out, static_cast<int32_t>(bh), heads, g, s, scale, err_flag, limit_ns);
  if (d == 128) return launch_d<128, false, kRaster>(tq, tk, tv, p, stream);
  return launch_d<64, false, kRaster>(tq, tk, tv, p, stream);
}

cudaError_t launch_attention_mixed(const void* q, const void* k_tiled, const void* v_tiled, void* out, int32_t batch,
                                   int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& s, float scale,
                                   int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  if (s.masked || !raster_tile_ok(g.tt, g.th, g.tw) || g.ntile % kBlockRows != 0) return cudaErrorInvalidValue;
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  const int bt = kBlockRows / (g.th * g.tw);
  CUtensorMap tq, tk, tv;
  if (!make_tmap_raster(&tq, q, bh, g, d, bt) || !make_tmap(&tk, k_tiled, bh, g.Lpad, d) ||
      !make_tmap(&tv, v_tiled, bh, g.Lpad, d))
    return cudaErrorInvalidValue;
  const FwdParams p = make_params(out, static_cast<int32_t>(bh), heads, g, s, scale, err_flag, limit_ns);
  if (d == 128) return launch_d<128, false, kMixed>(tq, tk, tv, p, stream);
  return launch_d<64, false, kMixed>(tq, tk, tv, p, stream);
}

cudaError_t launch_selftest_wait(int32_t* err_flag, uint64_t limit_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(err_flag, limit_ns);
  return cudaGetLastError();
}

}  // namespace sta
