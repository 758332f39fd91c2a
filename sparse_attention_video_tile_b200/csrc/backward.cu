// backward.cu - Sliding Tile Attention backward pass for sm_100a.
//
// The gradients of O = softmax(scale Q K^T) V restricted to each query tile's
// window of key tiles ("Fast Video Generation with Sliding Tile Attention":
// attention between a query tile and the key tiles of its window is dense,
// summary page "Method details" and "Core innovation"; the backward pass serves
// the fine-tuning the paper describes):
//
//   P = exp(scale S - lse),  dV = P^T dO,  dP = dO V^T,
//   dS = P (dP - D) with D_i = dO_i . O_i,  dQ = scale dS K,  dK = scale dS^T Q,
//
// where lse is the forward's per-row log-sum-exp, so P is rebuilt exactly without
// a row maximum.  Three launches: D per query row (an HBM-bound row dot product),
// dQ over the forward's work items (a 128-row query block and the key blocks of
// its window), and dK, dV over the transposed items (a 128-row key block and the
// query blocks whose windows contain it).  Each attention kernel is one CTA per SM:
//
//   * warp 8 loads the item's fixed operands (Q and dO, or K and V) and streams
//     the per-block operands (K and V, or Q and dO, plus lse and D of the query
//     block) through a two-stage shared-memory ring with TMA;
//   * warp 9 issues the tcgen05 MMAs from one thread: S and dP (both operands in
//     shared memory, fp32 in TMEM, S in columns 0-127 and dP in 128-255), and the
//     accumulations with the bf16 P and dS read from TMEM (dQ += dS K, or
//     dV += P^T dO and dK += dS^T Q; accumulators in columns 256-511);
//   * warps 0-7 do the elementwise step in two phases: TMEM lane = row, warps w
//     and w+4 take columns 0-63 and 64-127 of the rows of lane quadrant w.  Phase
//     A loads S, releases the S columns at once and turns S into P (fp32, in
//     registers); phase B turns dP into dS and stores bf16 over the dP columns: dS
//     over the first 32 of the warp's 64 columns (dQ), or P^T and dS^T interleaved
//     over all 64 (dK, dV: per 32 columns, 16 of P^T then 16 of dS^T, each written
//     after those 32 columns were read).  A warp never writes columns the other
//     warp reads.  At the end of an item each warp scales and stores its half of
//     the accumulators' columns.
//
// The two phases let the tensor core run beside the elementwise step: the issuer
// starts the next block's S as soon as phase A has loaded S, and the accumulations
// and the next block's dP as soon as phase B has stored dS (and P^T), so the next
// block's exponentials overlap this block's accumulations.  Two MMAs that touch the
// same TMEM columns (the next dP over dS and P^T) come from the same thread and
// execute in issue order.  The issuer's waits that have usually completed by the
// time it reaches them (the next block's loads, the S of a block loaded, dS
// stored) are tested without waiting in the middle of the MMA group before them,
// so that their latency overlaps queued MMAs; a test that fails is followed by the
// bounded wait at the point of use.
//
// Tiles must be multiples of 128 rows, so every block pair in a schedule is fully
// attended and no mask exists.  Every wait is bounded (see ptx.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

// Checked builds (STA_DEVICE_CHECKS=1) test every index taken from the work
// schedule (items, streamed block rows) before it addresses memory, as in the
// forward kernel: a failure records 0x200 | code, sets the abort flag and skips
// the access.
#ifndef STA_DEVICE_CHECKS
#define STA_DEVICE_CHECKS 0
#endif

namespace sta {
namespace {

using namespace ptx;

constexpr bool kBwdChecks = STA_DEVICE_CHECKS != 0;

// True if the phase with parity `parity` of `bar` has completed; never waits.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

constexpr int kBwdThreads = 320;   // warps 0-7 elementwise + epilogue, 8 producer, 9 MMA issuer
constexpr int kBwdProducer = 8;
constexpr int kBwdMma = 9;
constexpr int kBwdTmemCols = 512;  // S at 0, dP at 128, accumulators at 256 (and 384)

enum BwdKind { kDq = 0, kDkDv = 1 };

struct BwdParams {
  const WorkItem* items;
  const int32_t* rows;       // per item: first rows of the streamed blocks
  int32_t n_items;
  int32_t L;
  const float* lse;          // [BH, L] natural log
  const float* dvec;         // [BH, L] D_i = dO_i . O_i
  __nv_bfloat16* out0;       // dq, or dk
  __nv_bfloat16* out1;       // unused, or dv
  float scale;
  float scale_log2;          // scale * log2(e)
  int32_t* err;
  uint64_t limit_ns;
  int32_t n_rows;            // entries of rows (device checks)
  int32_t n_bh;              // batch * heads (device checks)
};

template <int D>
struct BwdSmem {
  static constexpr int kBlockBytes = kBlockRows * D * 2;
  static constexpr int kFix0 = 0;                          // Q (dQ) or K (dK, dV)
  static constexpr int kFix1 = kBlockBytes;                // dO (dQ) or V (dK, dV)
  static constexpr int kStageBytes = 2 * kBlockBytes + 1024;  // two blocks + lse and D of a query block
  static constexpr int kStage0 = 2 * kBlockBytes;
  static constexpr int kBar = kStage0 + 2 * kStageBytes;
  static constexpr int kFixFull = kBar;
  static constexpr int kFixEmpty = kFixFull + 8;
  static constexpr int kKvFull = kFixEmpty + 8;    // [2]
  static constexpr int kKvEmpty = kKvFull + 16;    // [2]
  static constexpr int kSFull = kKvEmpty + 16;    // S (S^T) of a block in TMEM
  static constexpr int kDFull = kSFull + 8;       // dP (dP^T) of a block in TMEM
  static constexpr int kSFree = kDFull + 8;       // phase A has loaded S (S^T)
  static constexpr int kPFull = kSFree + 8;       // phase B done: dS (P^T and dS^T) stored over dP
  static constexpr int kOFull = kPFull + 8;
  static constexpr int kDrain = kOFull + 8;
  static constexpr int kTmemSlot = kDrain + 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kEnd = kAbort + 4;
  static constexpr int kDynBytes = kEnd + 1024;
  static_assert(kDynBytes <= 227 * 1024, "shared memory budget");
};

// D_i = dO_i . O_i for every row (one warp per row, fp32 sums of bf16 products).
__global__ void bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
                                  float* __restrict__ dvec, int64_t rows, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(dout + r * d);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(out + r * d);
    float acc = 0.f;
    for (int i = lane; i < d / 2; i += 32) {
      const float2 x = __bfloat1622float2(a[i]), y = __bfloat1622float2(b[i]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dvec[r] = acc;
  }
}

// tm[0..3] = q, k, v, dO (tiled order [BH, L, d], 128 x 64 boxes).
template <int D, int KIND>
__global__ void __launch_bounds__(kBwdThreads, 1)
    sta_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const BwdParams p) {
  using S = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kTmemSlot);

  if (threadIdx.x == 0) {
    mbar_init(sb + S::kFixFull, 1);
    mbar_init(sb + S::kFixEmpty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(sb + S::kKvFull + 8 * s, 1);
      mbar_init(sb + S::kKvEmpty + 8 * s, 1);
    }
    mbar_init(sb + S::kSFull, 1);
    mbar_init(sb + S::kDFull, 1);
    mbar_init(sb + S::kSFree, 8);   // one arrival per elementwise warp
    mbar_init(sb + S::kPFull, 8);
    mbar_init(sb + S::kOFull, 1);
    mbar_init(sb + S::kDrain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kBwdMma) {
    tmem_alloc(sb + S::kTmemSlot, kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{abort_flag, p.err, p.limit_ns};
  constexpr uint32_t kBoxBytes = kBlockRows * 128;
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kBlockBytes = S::kBlockBytes;
  // Fixed operands (per item) and streamed operands (per block) of each kind.
  const CUtensorMap* fix0 = KIND == kDq ? &tm_q : &tm_k;
  const CUtensorMap* fix1 = KIND == kDq ? &tm_do : &tm_v;
  const CUtensorMap* str0 = KIND == kDq ? &tm_k : &tm_q;
  const CUtensorMap* str1 = KIND == kDq ? &tm_v : &tm_do;

  if (warp == kBwdProducer) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      uint32_t seq = 0, nfix = 0;
      bool ok = true;
      auto tma_block = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int32_t row, int32_t bh) {
        for (int b = 0; b < kBoxes; ++b) tma_load_3d(dst + b * kBoxBytes, m, bar, b * 64, row, bh);
      };
      for (int32_t k = 0; ok; ++k) {
        const int32_t idx = k * static_cast<int32_t>(gridDim.x) + static_cast<int32_t>(blockIdx.x);
        if (idx >= p.n_items) break;
        const WorkItem it = p.items[idx];
        if (kBwdChecks && !(it.bh >= 0 && it.bh < p.n_bh && it.q_row0 >= 0 && it.q_row0 < p.L &&
                            it.q_row0 % kBlockRows == 0 && it.kv_off >= 0 && it.kv_len >= 1 &&
                            it.kv_off + it.kv_len <= p.n_rows)) {
          atomicCAS(p.err, 0, 0x200 | 21);
          *abort_flag = 1;
          break;
        }
        ok = mbar_wait(sb + S::kFixEmpty, (nfix & 1) ^ 1, wc, 1);
        if (!ok) break;
        ++nfix;
        mbar_arrive_expect_tx(sb + S::kFixFull, 2 * kBlockBytes);
        tma_block(sb + S::kFix0, fix0, sb + S::kFixFull, it.q_row0, it.bh);
        tma_block(sb + S::kFix1, fix1, sb + S::kFixFull, it.q_row0, it.bh);
        for (int32_t j = 0; j < it.kv_len && ok; ++j) {
          const uint32_t st = seq & 1;
          ok = mbar_wait(sb + S::kKvEmpty + 8 * st, ((seq >> 1) & 1) ^ 1, wc, 2);
          if (!ok) break;
          const int32_t row = p.rows[it.kv_off + j];
          if (kBwdChecks && !(row >= 0 && row < p.L && row % kBlockRows == 0)) {
            atomicCAS(p.err, 0, 0x200 | 22);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t base = sb + S::kStage0 + st * S::kStageBytes;
          const uint32_t full = sb + S::kKvFull + 8 * st;
          mbar_arrive_expect_tx(full, 2 * kBlockBytes + (KIND == kDkDv ? 1024u : 0u));
          tma_block(base, str0, full, row, it.bh);
          tma_block(base + kBlockBytes, str1, full, row, it.bh);
          if (KIND == kDkDv) {
            const int64_t r0 = static_cast<int64_t>(it.bh) * p.L + row;
            bulk_load(base + 2 * kBlockBytes, p.lse + r0, 512, full);
            bulk_load(base + 2 * kBlockBytes + 512, p.dvec + r0, 512, full);
          }
          ++seq;
        }
      }
      if (nfix > 0) mbar_wait_drain(sb + S::kFixFull, (nfix - 1) & 1, p.limit_ns);
      for (uint32_t s = 0; s < 2 && s < seq; ++s) {
        const uint32_t last = seq - 1 - ((seq - 1 - s) & 1);
        mbar_wait_drain(sb + S::kKvFull + 8 * s, (last >> 1) & 1, p.limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == kBwdMma) {
    if (lane == 0) {
      // Issue order per block b of the CTA's stream (stage b & 1):
      //   wait S of b loaded -> S of b+1 (within an item) -> wait phase B of b
      //   -> dQ += dS K (or dV += P^T dO, dK += dS^T Q) -> release the stage
      //   -> [item boundary: wait the next fixed operands, S of b+1] -> dP of b+1.
      // One thread issues everything, so a later MMA that overwrites an operand an
      // earlier one reads (dP over dS and P^T) executes after it.
      constexpr uint32_t idesc_ss = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_ts = idesc_bf16_f32(128, D, false, true);
      const uint64_t dfix0 = sdesc_sw128(sb + S::kFix0, 16, 1024);
      const uint64_t dfix1 = sdesc_sw128(sb + S::kFix1, 16, 1024);
      auto koff = [](int k16) -> uint64_t { return static_cast<uint64_t>(((k16 >> 2) * 16384 + (k16 & 3) * 32) >> 4); };
      const uint32_t tS = tmem, tP = tmem + 128, tA0 = tmem + 256, tA1 = tmem + 384;
      auto stage_base = [&](uint32_t b) { return sb + S::kStage0 + (b & 1) * S::kStageBytes; };
      // `mid` runs after the first half of a group's MMAs (the early tests)
      auto issue_s = [&](uint32_t b, auto&& mid) {   // S (S^T) = fix0 str0^T, K-major operands
        const uint64_t ds0 = sdesc_sw128(stage_base(b), 16, 1024);
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16) {
          if (k16 == D / 32) mid();
          umma_ss(tS, dfix0 + koff(k16), ds0 + koff(k16), idesc_ss, k16 > 0);
        }
        umma_commit(sb + S::kSFull);
      };
      auto issue_dp = [&](uint32_t b, auto&& mid) {  // dP (dP^T) = fix1 str1^T
        const uint64_t ds1 = sdesc_sw128(stage_base(b) + kBlockBytes, 16, 1024);
#pragma unroll
        for (int k16 = 0; k16 < D / 16; ++k16) {
          if (k16 == D / 32) mid();
          umma_ss(tP, dfix1 + koff(k16), ds1 + koff(k16), idesc_ss, k16 > 0);
        }
        umma_commit(sb + S::kDFull);
      };
      auto item_len = [&](int32_t kk) -> int32_t {
        const int32_t idx = kk * static_cast<int32_t>(gridDim.x) + static_cast<int32_t>(blockIdx.x);
        return idx < p.n_items ? p.items[idx].kv_len : 0;
      };
      auto kv_full = [&](uint32_t b) { return mbar_wait(sb + S::kKvFull + 8 * (b & 1), (b >> 1) & 1, wc, 4); };
      auto kv_test = [&](uint32_t b) { return mbar_test(sb + S::kKvFull + 8 * (b & 1), (b >> 1) & 1); };
      int32_t k = 0, j = 0, n = item_len(0);
      uint32_t seq = 0, nfix = 0;
      // early test results for the current block: its S loaded, the next block's loads
      bool s_free_ok = false, kv_ok = false;
      bool ok = n > 0;
      if (ok) {
        ok = mbar_wait(sb + S::kFixFull, 0, wc, 3) && kv_full(0);
        nfix = 1;
        if (ok) {
          tc_fence_after();
          issue_s(0, [] {});
          issue_dp(0, [&] {
            s_free_ok = mbar_test(sb + S::kSFree, 0);
            kv_ok = n > 1 && kv_test(1);
          });
          if (n == 1) umma_commit(sb + S::kFixEmpty);
        }
      }
      while (ok) {
        const bool new_item = j + 1 == n;               // the next block starts item k + 1
        const int32_t n_next = new_item ? item_len(k + 1) : n;
        const bool has_next = n_next > 0;
        const bool next_is_last = new_item ? n_next == 1 : j + 2 == n;
        const uint32_t base = stage_base(seq);
        // accumulations: B operands are the stage's blocks read MN-major (16 rows = 2 KB
        // per K16 slice); A is bf16 in TMEM over the dP columns
        const uint64_t dm0 = sdesc_sw128(base, kBlockRows * 128, 1024);
        const uint64_t dm1 = sdesc_sw128(base + kBlockBytes, kBlockRows * 128, 1024);
        if (!s_free_ok) ok = mbar_wait(sb + S::kSFree, seq & 1, wc, 5);
        if (!ok) break;
        bool p_ok = false;
        if (has_next && !new_item) {   // next block's S while the elementwise warps finish this one
          if (!kv_ok) ok = kv_full(seq + 1);
          if (!ok) break;
          tc_fence_after();
          issue_s(seq + 1, [&] { p_ok = mbar_test(sb + S::kPFull, seq & 1); });
        }
        if (!p_ok) ok = mbar_wait(sb + S::kPFull, seq & 1, wc, 7);
        if (!ok) break;
        tc_fence_after();
        if (KIND == kDq) {
          // dQ += dS K; dS over the first 32 of each warp's 64 dP columns
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            umma_ts(tA0, tP + (k16 >> 2) * 64 + (k16 & 3) * 8, dm0 + static_cast<uint64_t>(k16 * (2048 >> 4)),
                    idesc_ts, (j > 0 || k16 > 0));
        } else {
          // dV += P^T dO and dK += dS^T Q; K16 slice k16 (16 queries) of P^T at column
          // 64 (k16 / 4) + 32 ((k16 / 2) mod 2) + 8 (k16 mod 2) of the dP region, dS^T 16 further
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            umma_ts(tA0, tP + (k16 >> 2) * 64 + ((k16 >> 1) & 1) * 32 + (k16 & 1) * 8,
                    dm1 + static_cast<uint64_t>(k16 * (2048 >> 4)), idesc_ts, (j > 0 || k16 > 0));
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16)
            umma_ts(tA1, tP + (k16 >> 2) * 64 + ((k16 >> 1) & 1) * 32 + 16 + (k16 & 1) * 8,
                    dm0 + static_cast<uint64_t>(k16 * (2048 >> 4)), idesc_ts, (j > 0 || k16 > 0));
        }
        umma_commit(sb + S::kKvEmpty + 8 * (seq & 1));
        if (new_item) umma_commit(sb + S::kOFull);
        if (!has_next) break;
        if (new_item) {                 // the next item's fixed operands load after this item's last dP
          ok = mbar_wait(sb + S::kFixFull, nfix & 1, wc, 3) && kv_full(seq + 1);
          ++nfix;
          if (!ok) break;
          tc_fence_after();
          issue_s(seq + 1, [] {});
        }
        // early tests for block seq + 1: its S loaded, and block seq + 2's loads when
        // it belongs to the same item (its S is then issued in the next iteration)
        issue_dp(seq + 1, [&] {
          s_free_ok = mbar_test(sb + S::kSFree, (seq + 1) & 1);
          kv_ok = !next_is_last && kv_test(seq + 2);
        });
        if (next_is_last) umma_commit(sb + S::kFixEmpty);
        ++seq;
        if (new_item) {
          ++k;
          j = 0;
          n = n_next;
        } else {
          ++j;
        }
      }
      umma_commit(sb + S::kDrain);
      mbar_wait_drain(sb + S::kDrain, 0, p.limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise + epilogue
    const int quad = warp & 3, hh = warp >> 2;   // lane quadrant; columns [64 hh, 64 hh + 64)
    const int row = quad * 32 + lane;             // TMEM lane = row of the item's block
    const uint32_t tl = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t tS = tl + 64 * hh, tP = tl + 128 + 64 * hh, tA0 = tl + 256, tA1 = tl + 384;
    const float sl2 = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    uint32_t seq = 0;
    bool ok = true;
    for (int32_t k = 0; ok; ++k) {
      const int32_t idx = k * static_cast<int32_t>(gridDim.x) + static_cast<int32_t>(blockIdx.x);
      if (idx >= p.n_items) break;
      const WorkItem it = p.items[idx];
      if (kBwdChecks && !(it.bh >= 0 && it.bh < p.n_bh && it.q_row0 >= 0 && it.q_row0 < p.L)) {
        atomicCAS(p.err, 0, 0x200 | 23);
        *abort_flag = 1;
        break;
      }
      const int64_t grow = static_cast<int64_t>(it.bh) * p.L + it.q_row0 + row;   // this thread's row
      float lse2_row = 0.f, d_row = 0.f;
      if (KIND == kDq) {
        lse2_row = p.lse[grow] * kLog2e;
        d_row = p.dvec[grow];
      }
      for (int32_t j = 0; j < it.kv_len; ++j, ++seq) {
        const uint32_t st = seq & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kSFull, seq & 1, wc, 8));
        if (!ok) break;
        if (KIND == kDkDv) {
          // lse and D of the streamed query block, in the stage's shared memory
          ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kKvFull + 8 * st, (seq >> 1) & 1, wc, 9));
          if (!ok) break;
        }
        tc_fence_after();
        const float4* col_lse4 = reinterpret_cast<const float4*>(smem + S::kStage0 + st * S::kStageBytes +
                                                                 2 * kBlockBytes) + 16 * hh;
        const float4* col_d4 = col_lse4 + 32;
        // phase A: P (P^T) of this thread's row over this warp's 64 columns, kept in fp32
        float pf[64];
        {
          uint32_t s_lo[32], s_hi[32];
          tmem_ld32(tS, s_lo);
          tmem_ld32(tS + 32, s_hi);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sb + S::kSFree);   // S may be overwritten by the next block's
          if (KIND == kDq) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              pf[i] = ex2_approx(fmaf(__uint_as_float(s_lo[i]), sl2, -lse2_row));
              pf[32 + i] = ex2_approx(fmaf(__uint_as_float(s_hi[i]), sl2, -lse2_row));
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 lv = col_lse4[i / 4], hv = col_lse4[8 + i / 4];
              const float l2[4] = {lv.x * kLog2e, lv.y * kLog2e, lv.z * kLog2e, lv.w * kLog2e};
              const float h2[4] = {hv.x * kLog2e, hv.y * kLog2e, hv.z * kLog2e, hv.w * kLog2e};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                pf[i + u] = ex2_approx(fmaf(__uint_as_float(s_lo[i + u]), sl2, -l2[u]));
                pf[32 + i + u] = ex2_approx(fmaf(__uint_as_float(s_hi[i + u]), sl2, -h2[u]));
              }
            }
          }
        }
        // phase B: dS = P (dP - D), bf16 over this warp's dP columns (and P^T for dK, dV)
        ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kDFull, seq & 1, wc, 10));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t d32[32], dk[16];
          tmem_ld32(tP + 32 * c, d32);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float dd[4];
            if (KIND == kDq) {
              dd[0] = dd[1] = dd[2] = dd[3] = d_row;
            } else {
              const float4 dv4 = col_d4[8 * c + i / 4];
              dd[0] = dv4.x; dd[1] = dv4.y; dd[2] = dv4.z; dd[3] = dv4.w;
            }
            float dsv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) dsv[u] = pf[32 * c + i + u] * (__uint_as_float(d32[i + u]) - dd[u]);
            dk[i >> 1] = pack_bf16x2(dsv[0], dsv[1]);
            dk[(i >> 1) + 1] = pack_bf16x2(dsv[2], dsv[3]);
          }
          if (KIND == kDq) {
            tmem_st16(tP + 16 * c, dk);
          } else {
            // columns 32c .. 32c + 31 were read above: P^T over the first 16, dS^T over the next 16
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) pk[i >> 1] = pack_bf16x2(pf[32 * c + i], pf[32 * c + i + 1]);
            tmem_st16(tP + 32 * c, pk);
            tmem_st16(tP + 32 * c + 16, dk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sb + S::kPFull);
      }
      if (!ok) break;
      // epilogue: the item's accumulators, scaled, as bf16 rows
      ok = __all_sync(0xffffffffu, mbar_wait(sb + S::kOFull, static_cast<uint32_t>(k) & 1, wc, 11));
      if (!ok) break;
      tc_fence_after();
      for (int a = 0; a < (KIND == kDq ? 1 : 2); ++a) {
        // this warp's half of the accumulator's columns
        const uint32_t tacc = (a == 0 ? tA0 : tA1) + hh * (D / 2);
        // dQ (a = 0) and dK (a = 1 of dK, dV) carry the softmax scale; dV does not
        const float mul = (KIND == kDq || a == 1) ? p.scale : 1.0f;
        __nv_bfloat16* dst_t = KIND == kDq ? p.out0 : (a == 0 ? p.out1 : p.out0);
        uint4* dst = reinterpret_cast<uint4*>(dst_t + grow * D + hh * (D / 2));
#pragma unroll 1
        for (int c32 = 0; c32 < D / 64; ++c32) {
          uint32_t o[32];
          tmem_ld32(tacc + 32 * c32, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 v4;
            v4.x = pack_bf16x2(__uint_as_float(o[8 * c + 0]) * mul, __uint_as_float(o[8 * c + 1]) * mul);
            v4.y = pack_bf16x2(__uint_as_float(o[8 * c + 2]) * mul, __uint_as_float(o[8 * c + 3]) * mul);
            v4.z = pack_bf16x2(__uint_as_float(o[8 * c + 4]) * mul, __uint_as_float(o[8 * c + 5]) * mul);
            v4.w = pack_bf16x2(__uint_as_float(o[8 * c + 6]) * mul, __uint_as_float(o[8 * c + 7]) * mul);
            dst[4 * c32 + c] = v4;
          }
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwdMma) tmem_dealloc(tmem, kBwdTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 bwd_encode_fn() {
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

// [BH, L, d] bf16, 128-row x 64-column box, 128-byte swizzle; rows past L read as zero.
bool bwd_tmap(CUtensorMap* m, const void* base, int64_t bh, int64_t L, int d) {
  auto fn = bwd_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kBlockRows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KIND>
cudaError_t launch_bwd_t(const CUtensorMap* tm, const BwdParams& p, cudaStream_t stream) {
  auto kern = sta_bwd_kernel<D, KIND>;
  const int smem = BwdSmem<D>::kDynBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  int grid = sms < p.n_items ? sms : p.n_items;
  if (grid < 1) return cudaSuccess;
  kern<<<grid, kBwdThreads, smem, stream>>>(tm[0], tm[1], tm[2], tm[3], p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                            const float* lse, float* dvec, void* dq, void* dk, void* dv, int32_t batch,
                            int32_t heads, int32_t d, const Geometry& g, const DeviceSchedule& fwd,
                            const DeviceSchedule& tr, float scale, int32_t* err_flag, uint64_t limit_ns,
                            cudaStream_t stream) {
  const int64_t bh = static_cast<int64_t>(batch) * heads;
  const int64_t rows = bh * g.L;
  if (rows > 0) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    bwd_rowdot_kernel<<<sms * 8, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(dout),
                                                   static_cast<const __nv_bfloat16*>(out), dvec, rows, d);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  CUtensorMap tm[4];
  if (!bwd_tmap(&tm[0], q, bh, g.L, d) || !bwd_tmap(&tm[1], k, bh, g.L, d) || !bwd_tmap(&tm[2], v, bh, g.L, d) ||
      !bwd_tmap(&tm[3], dout, bh, g.L, d))
    return cudaErrorInvalidValue;
  BwdParams p{};
  p.L = static_cast<int32_t>(g.L);
  p.lse = lse;
  p.dvec = dvec;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err_flag;
  p.limit_ns = limit_ns;
  p.n_bh = static_cast<int32_t>(bh);
  // dQ over the forward's items
  p.items = fwd.items;
  p.rows = fwd.kv_rows;
  p.n_rows = fwd.n_kv_rows;
  p.n_items = fwd.n_items;
  p.out0 = static_cast<__nv_bfloat16*>(dq);
  p.out1 = nullptr;
  cudaError_t e = d == 128 ? launch_bwd_t<128, kDq>(tm, p, stream) : launch_bwd_t<64, kDq>(tm, p, stream);
  if (e != cudaSuccess) return e;
  // dK, dV over the transposed items
  p.items = tr.items;
  p.rows = tr.kv_rows;
  p.n_rows = tr.n_kv_rows;
  p.n_items = tr.n_items;
  p.out0 = static_cast<__nv_bfloat16*>(dk);
  p.out1 = static_cast<__nv_bfloat16*>(dv);
  return d == 128 ? launch_bwd_t<128, kDkDv>(tm, p, stream) : launch_bwd_t<64, kDkDv>(tm, p, stream);
}

}  // namespace sta
