/*
 * sta.h - C ABI of the B200 (sm_100a) Sliding Tile Attention library: tile
 * reorders, the forward pass (with or without its log-sum-exp) and the backward
 * pass.
 *
 * Method: "Fast Video Generation with Sliding Tile Attention" (arXiv 2502.04507).
 *   - abstract: attention restricted to a local 3D window that moves tile by
 *     tile rather than token by token;
 *   - summary page, "Method details": the latent video (T, H, W) is cut into
 *     non-overlapping (tt, th, tw) tiles whose tokens are made contiguous, so
 *     attention between a query tile and a key tile is a dense block;
 *   - summary page, "Core innovation": blocks are fully attended or skipped;
 *     "Technical contribution": the window is set per attention head;
 *   - review reply on input resolution: tile (6, 8, 8); latent dimensions must
 *     be multiples of the tile.
 * Window rule: query tile a attends key tile k iff, in every dimension x,
 *   s_x <= k_x < s_x + w'_x  with  w'_x = min(w_x, n_x)  and
 *   s_x = clamp(a_x - floor(w'_x / 2), 0, n_x - w'_x),
 * n_x being the number of tiles in dimension x and w_x the head's window, in
 * tiles.  A window wider than the grid therefore covers the grid.
 *
 * Layout conventions (all entry points):
 *   - every q/k/v/out tensor is a contiguous bf16 array [batch, heads, L, d]
 *     (row-major, d fastest), L = T * H * W tokens, d in {64, 128}; the one
 *     exception is the raster side of the token-major reorders,
 *     [batch, L, heads, d];
 *   - raster order: token n = (t * H + h) * W + w;
 *   - tiled order: tiles in raster order over the tile grid, tokens in raster
 *     order inside a tile; tile i occupies rows [i * Ntile, (i + 1) * Ntile).
 *
 * Ownership and execution: the caller owns every device buffer.  Calls are
 * asynchronous on the given stream (a cudaStream_t passed as void*, NULL = the
 * legacy default stream), out of place, and never synchronise unless stated.
 * The attention calls build a work schedule per configuration on first use
 * (a blocking upload) and keep the 16 most recently used; evicting an older one
 * synchronises the device first, since a queued kernel may still read it.
 * On an invalid argument a call returns an error before touching any buffer or
 * the device.  Nothing is printed.
 */
#ifndef STA_H_
#define STA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t t, h, w;
} sta_dim3;

typedef enum {
  STA_OK = 0,
  STA_ERR_NULL = 1,      /* a required pointer is NULL */
  STA_ERR_ALIGN = 2,     /* a device pointer is not 16-byte aligned */
  STA_ERR_ALIAS = 3,     /* an output overlaps an input */
  STA_ERR_SHAPE = 4,     /* grid/tile not positive, grid not a multiple of the tile, sizes too large */
  STA_ERR_WINDOW = 5,    /* a window dimension is < 1 */
  STA_ERR_HEADDIM = 6,   /* d is not 64 or 128 */
  STA_ERR_ARCH = 7,      /* the current device is not compute capability 10.0 (B200) */
  STA_ERR_CUDA = 8,      /* a CUDA runtime/driver call failed (message via sta_last_cuda_error) */
  STA_ERR_TIMEOUT = 9,   /* a kernel's bounded wait expired; the kernel gave up */
  STA_ERR_ARG = 10,      /* another argument is out of range (batch, heads, scale not finite ...) */
  STA_ERR_SCRATCH = 11,  /* the work schedule does not fit the fixed scratch of sta_attention_fwd_noalloc */
  STA_ERR_BOUNDS = 12    /* a device-side bounds check failed (libsta_checked.so only); the kernel skipped the access */
} sta_status;

/* Human-readable name of a status code.  Static storage; never NULL. */
const char* sta_status_str(sta_status s);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* sta_last_cuda_error(void);

/*
 * Index map raster -> tiled (host only, no device use).
 *   tiled_of_raster: host array of L = T*H*W int32 written by the call;
 *   tiled_of_raster[n] is the tiled row of raster token n.
 * Errors: STA_ERR_NULL, STA_ERR_SHAPE.
 */
sta_status sta_tile_index_map(sta_dim3 grid, sta_dim3 tile, int32_t* tiled_of_raster);

/*
 * Attended (query, key) token pairs summed over batch and heads (host only):
 *   batch * sum_h L * Ntile * prod_x min(w_h,x, n_x).
 * FLOPs of the forward pass are 4 * d * pairs.  windows: host array of `heads`
 * entries.  Returns -1 on an invalid argument.
 */
int64_t sta_attended_pairs(int32_t batch, int32_t heads, sta_dim3 grid, sta_dim3 tile,
                           const sta_dim3* windows);

/*
 * The (query block, key block) pairs of the work schedules (host only), so that
 * they can be checked against the window rule without a GPU: the forward's
 * schedule (transposed = 0: each 128-row query block with the 128-row key blocks
 * of its window) or the backward's key-side schedule (transposed = 1: each key
 * block with the query blocks whose windows contain it).  Up to `capacity`
 * triples (batch * heads + head, first tiled row of the query block, first tiled
 * row of the key block) are written to `out` (host int32[3 * capacity], may be
 * NULL); returns the number of pairs, or -1 on an invalid argument or a tile
 * that does not hold a multiple of 128 tokens.  No device is touched.
 */
int64_t sta_schedule_block_pairs(int32_t batch, int32_t heads, sta_dim3 grid, sta_dim3 tile,
                                 const sta_dim3* windows, int32_t transposed, int32_t* out,
                                 int64_t capacity);

/*
 * Reorder raster -> tiled (summary page, "Method details": tokens of a tile made
 * contiguous).  src, dst: device bf16 [batch_heads, L, d], 16-byte aligned, not
 * overlapping.  dst[bh, tiled(n), :] = src[bh, n, :], bit-exact.
 * HBM-bound gather of d*2-byte rows with 16-byte vector accesses.
 * Errors: NULL, ALIGN, ALIAS, SHAPE, HEADDIM, ARG, ARCH, CUDA.
 */
sta_status sta_tile_reorder(const void* src, void* dst, int64_t batch_heads, int32_t d,
                            sta_dim3 grid, sta_dim3 tile, void* stream);

/* Inverse of sta_tile_reorder: dst[bh, n, :] = src[bh, tiled(n), :]. */
sta_status sta_tile_unorder(const void* src, void* dst, int64_t batch_heads, int32_t d,
                            sta_dim3 grid, sta_dim3 tile, void* stream);

/*
 * Reorder with a token-major raster side (summary page, "Method details": the
 * same tile order): src is device bf16 [batch, L, heads, d] in raster order,
 * the layout of a [batch, L, heads * d] projection; dst is device bf16
 * [batch, heads, L, d] in tiled order, as sta_attention_fwd takes it.
 *   dst[b, h, tiled(n), :] = src[b, n, h, :], bit-exact.
 * Both 16-byte aligned, not overlapping.  batch = 0 or heads = 0 is a no-op.
 * Errors: NULL, ALIGN, ALIAS, SHAPE, HEADDIM, ARG (negative batch or heads),
 * ARCH, CUDA.
 */
sta_status sta_tile_reorder_tokens(const void* src, void* dst, int32_t batch, int32_t heads, int32_t d,
                                   sta_dim3 grid, sta_dim3 tile, void* stream);

/* Inverse of sta_tile_reorder_tokens: src tiled [batch, heads, L, d], dst
 * token-major raster [batch, L, heads, d]; dst[b, n, h, :] = src[b, h, tiled(n), :]. */
sta_status sta_tile_unorder_tokens(const void* src, void* dst, int32_t batch, int32_t heads, int32_t d,
                                   sta_dim3 grid, sta_dim3 tile, void* stream);

/*
 * STA forward on tiled-order tensors (abstract; "Method details"; "Core
 * innovation"): for every head h and query token i,
 *   out[i] = sum_j softmax_j(scale * q_i . k_j) v_j
 * over the key tokens j whose tile lies in the window of i's tile (rule above,
 * window_per_head[h]).  q, k, v, out: device bf16 [batch, heads, L, d] in tiled
 * order, 16-byte aligned; out must not overlap q, k or v.  window_per_head:
 * host array of `heads` windows in tiles, read during the call only.
 * Arithmetic: bf16 inputs, fp32 tensor-core accumulation, fp32 online softmax,
 * probabilities rounded to bf16 for the P*V product, output rounded to bf16.
 * The first call with a new (batch, heads, grid, tile, windows) builds and
 * uploads a work schedule synchronously (do it before any stream capture);
 * later calls reuse it.  Kernel timeouts are reported by
 * sta_check_device_status.
 * Errors: NULL, ALIGN, ALIAS, SHAPE, WINDOW, HEADDIM, ARG, ARCH, CUDA.
 */
sta_status sta_attention_fwd(const void* q, const void* k, const void* v, void* out,
                             int32_t batch, int32_t heads, int32_t d, sta_dim3 grid,
                             sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                             void* stream);

/*
 * sta_attention_fwd that also returns each query row's log-sum-exp: the
 * normaliser of the row's softmax, lse[i] = log(sum_j exp(scale * q_i . k_j)) over
 * the keys j of the row's window (natural log), which a backward pass uses to
 * rebuild the probabilities without a second row maximum.
 *   lse: device fp32 [batch, heads, L], tiled order like q (row n of the tiled
 *   tensors), 4-byte aligned, not overlapping q, k, v or out.
 * Everything else as sta_attention_fwd.
 * Errors: those of sta_attention_fwd; NULL also for a null lse, ALIGN for an
 * unaligned lse, ALIAS for an lse overlapping another tensor.
 */
sta_status sta_attention_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                                 int32_t batch, int32_t heads, int32_t d, sta_dim3 grid,
                                 sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                                 void* stream);

/*
 * STA backward pass ("Fast Video Generation with Sliding Tile Attention": the
 * gradients of the tile-windowed attention of sta_attention_fwd, for the
 * fine-tuning the paper describes).  With P = softmax(scale q k^T) over each row's
 * window, rebuilt from lse:
 *   dv = P^T dout,  ds = P (dout v^T - D) with D_i = dout_i . out_i,
 *   dq = scale ds k,  dk = scale ds^T q.
 *   q, k, v, out, dout: device bf16 [batch, heads, L, d], tiled order, as passed to
 *   and returned by sta_attention_fwd_lse; lse: its fp32 [batch, heads, L] output.
 *   dq, dk, dv: device bf16 [batch, heads, L, d], tiled order, written.
 *   All 16-byte aligned; the outputs overlap no input and no other output.
 * Arithmetic: bf16 operands, fp32 tensor-core accumulation, P and ds rounded to
 * bf16 for the products that take them, bf16 results.
 * The tile must hold a multiple of 128 tokens (for example (6,8,8) or (1,8,16)).
 * The library keeps one fp32 per query row of scratch (the row terms D; grown on
 * demand, freed by sta_shutdown), so the first call of a larger size synchronises
 * the device.  All backward calls on a device share it: calls that overlap on the
 * GPU (different streams) race on it; order them.
 * Errors: NULL, ALIGN, ALIAS, SHAPE (also: tile not a multiple of 128 tokens),
 * WINDOW, HEADDIM, ARG, ARCH, CUDA.
 */
sta_status sta_attention_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, int32_t batch, int32_t heads,
                             int32_t d, sta_dim3 grid, sta_dim3 tile, const sta_dim3* window_per_head,
                             float scale, void* stream);

/*
 * STA forward on raster-order tensors, with the tile reorder fused into the
 * kernel's loads and stores, and padding with masking ("Fast Video Generation with
 * Sliding Tile Attention", review reply on input resolution): the grid need not be
 * a multiple of the tile.  The latent is treated as padded up to the next tile
 * multiple; windows live on that padded tile grid; pad tokens are never keys and
 * produce no output.
 *   q, k, v, out: device bf16 [batch, heads, T*H*W, d] in raster order (token
 *   n = (t*H + h)*W + w), 16-byte aligned; out must not overlap q, k or v.
 *   The tile must split into 128-row slabs of whole frames: th*tw divides 128 and
 *   tt is a multiple of 128/(th*tw) (for example (6,8,8) or (1,8,16)); other tiles
 *   use sta_tile_reorder + sta_attention_fwd + sta_tile_unorder.
 * Results equal those of that three-call path (up to fp32 summation order) on
 * tile-multiple grids.  Same arithmetic, schedule caching and status reporting as
 * sta_attention_fwd.
 * Errors: NULL, ALIGN, ALIAS, SHAPE (tile cannot be split as above, sizes too
 * large), WINDOW, HEADDIM, ARG, ARCH, CUDA.
 */
sta_status sta_attention_fwd_raster(const void* q, const void* k, const void* v, void* out,
                                    int32_t batch, int32_t heads, int32_t d, sta_dim3 grid,
                                    sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                                    void* stream);

/*
 * Tile reorder into the padded latent (raster -> tiled), for grids that need not
 * be tile multiples ("padding with masking", review reply on input resolution).
 * The latent is treated as padded up to the next tile multiple in every dimension:
 * Lpad = ceil(T/tt)*tt * ceil(H/th)*th * ceil(W/tw)*tw rows per (batch, head).
 *   src: device bf16 [batch_heads, T*H*W, d], raster order; 16-byte aligned.
 *   dst: device bf16 [batch_heads, Lpad, d], tiled order of the padded latent;
 *        the rows of pad tokens are written as zeros.  Must not overlap src.
 * On tile-multiple grids the result equals sta_tile_reorder's.  Asynchronous on
 * `stream`.
 * Errors: NULL, ALIGN, ALIAS, SHAPE (nonpositive sizes, too large), HEADDIM, ARG,
 * ARCH, CUDA.
 */
sta_status sta_tile_reorder_padded(const void* src, void* dst, int64_t batch_heads, int32_t d, sta_dim3 grid,
                                   sta_dim3 tile, void* stream);

/*
 * STA forward with raster-order queries and output and tiled-order keys and
 * values: the query blocks are read from raster order by the kernel's loads (one
 * load per block of 128 queries, the same 5-D boxes as sta_attention_fwd_raster)
 * and the output rows are written to raster order, while the key and value blocks,
 * read once for every query block whose window holds them, come from tiled copies
 * (sta_tile_reorder_padded), 128 contiguous rows each.  The grid need not be a
 * tile multiple (padding with masking, as sta_attention_fwd_raster).
 *   q, out: device bf16 [batch, heads, T*H*W, d], raster order, 16-byte aligned;
 *   k_tiled, v_tiled: device bf16 [batch, heads, Lpad, d], tiled order of the
 *   padded latent with zero pad rows, as written by sta_tile_reorder_padded;
 *   out must not overlap q, k_tiled or v_tiled.
 *   The tile must split into 128-row slabs of whole frames, as for
 *   sta_attention_fwd_raster.
 * Results equal sta_attention_fwd_raster's bit for bit (same schedule and
 * arithmetic).  Same schedule caching and status reporting as sta_attention_fwd.
 * Errors: NULL, ALIGN, ALIAS, SHAPE, WINDOW, HEADDIM, ARG, ARCH, CUDA.
 */
sta_status sta_attention_fwd_mixed(const void* q, const void* k_tiled, const void* v_tiled, void* out,
                                   int32_t batch, int32_t heads, int32_t d, sta_dim3 grid, sta_dim3 tile,
                                   const sta_dim3* window_per_head, float scale, void* stream);

/*
 * STA forward from host memory to host memory.  The paper has no counterpart: it
 * is the whole-job call for data that lives on the host.
 *   q, k, v, out: host bf16 [batch, heads, T*H*W, d], raster order.  Pinned memory
 *   (cudaHostAlloc, cudaHostRegister) lets the copies overlap the computation;
 *   pageable memory works, with copies that do not.  out must not overlap q, k, v.
 * The heads go through the current device in chunks of heads_per_chunk heads of one
 * batch entry: while one chunk is computed (sta_tile_reorder_padded of k and v,
 * then sta_attention_fwd_mixed), the next is copied in and the one before copied
 * out, on three CUDA streams the library owns.  The work starts after what is
 * already queued on `stream`, and the call returns once out holds the result.
 * Per head the result equals sta_attention_fwd_mixed's on device tensors bit for
 * bit (heads are independent).  The tile must split into 128-row slabs of whole
 * frames, as for sta_attention_fwd_mixed; the grid may be padded.  The library
 * keeps two sets of chunk buffers on the device (grown as needed, freed by
 * sta_shutdown), and the call holds the library's lock throughout, so concurrent
 * calls of the library from other threads wait for it.  A bounded wait that ran
 * out is reported by sta_check_device_status.
 * Errors: NULL, SHAPE, WINDOW, HEADDIM, ARG (batch, heads, scale or heads_per_chunk
 * out of range), ALIAS, ARCH, CUDA.
 */
sta_status sta_forward_host(const void* q, const void* k, const void* v, void* out, int32_t batch, int32_t heads,
                            int32_t d, sta_dim3 grid, sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                            int32_t heads_per_chunk, void* stream);

/*
 * sta_attention_fwd without any device allocation by the library.  The paper has
 * no counterpart: this entry point exists for callers that cannot let a library
 * call cudaMalloc - code running inside a memory pool or arena it must not
 * bypass, processes that reserve all device memory up front, or runtimes whose
 * allocator must account for every device allocation.
 * Same arguments, layout, semantics and errors as sta_attention_fwd, plus
 * STA_ERR_SCRATCH when the work schedule exceeds the fixed scratch.
 * Scratch: one static device array of 4 MiB per GPU that loads the library,
 * held until the process exits (enough for every workload here; the largest,
 * 24 heads at 48x48x80 with per-head windows, needs about 3 MB).  The array
 * keeps the last call's contents: its status word is cleared on every call and
 * the schedule is uploaded again when the configuration changes.  Calls that
 * overlap on the GPU (different streams) race on the array; order them.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * Bounded-wait timeouts of this variant are recorded in the array's status word,
 * which sta_check_device_status reports and clears like the other entry points'
 * (synchronise the stream the call ran on through it).  After sta_shutdown, or a
 * device reset, the next call sets the device up again.
 */
sta_status sta_attention_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                     int32_t batch, int32_t heads, int32_t d, sta_dim3 grid,
                                     sta_dim3 tile, const sta_dim3* window_per_head, float scale,
                                     void* stream);

/*
 * Synchronises `stream` and reports whether any kernel of this library on the
 * current device gave up on a bounded wait since the last check
 * (STA_ERR_TIMEOUT) or, in the checked build (libsta_checked.so, compiled with
 * STA_DEVICE_CHECKS=1), failed a bounds check on an index taken from its work
 * schedule (STA_ERR_BOUNDS, which takes precedence), then clears the flag.  The flags read are the allocating
 * entry points' status word and, once sta_attention_fwd_noalloc has run on the
 * device, that entry point's own.  Returns STA_ERR_CUDA if the stream has a
 * pending CUDA error.
 */
sta_status sta_check_device_status(void* stream);

/*
 * Self-test of the bounded-wait path: for each status word of the current
 * device (see sta_check_device_status) launches one block whose threads wait on
 * a shared-memory barrier that nothing completes, with a limit of `limit_ns`
 * nanoseconds (clamped to [1e5, 5e9]) and the expiry recorded in that word, then
 * synchronises `stream`.  Returns STA_ERR_TIMEOUT if every word recorded its
 * expiry (a correct library), and leaves the words cleared and the context
 * usable.  No schedule or tensor is touched.
 */
sta_status sta_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* Releases the library's cached schedules and device workspaces (all devices). */
void sta_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* STA_H_ */
