/* The C ABI used from plain C99: every entry point of sta.h is bound to a
 * function pointer of the type spelled out below, so a change of a signature in
 * the header fails to compile here, and a symbol missing from the library fails
 * to link.  Only host entry points are called (no device is touched): the index
 * map, the attended-pair count and the status strings are printed for the test
 * to compare with the oracle. */
#include <stdio.h>
#include <string.h>

#include "sta.h"

typedef sta_status (*reorder_fn)(const void*, void*, int64_t, int32_t, sta_dim3, sta_dim3, void*);
typedef sta_status (*reorder_tokens_fn)(const void*, void*, int32_t, int32_t, int32_t, sta_dim3, sta_dim3, void*);
typedef sta_status (*fwd_fn)(const void*, const void*, const void*, void*, int32_t, int32_t, int32_t, sta_dim3,
                             sta_dim3, const sta_dim3*, float, void*);
typedef sta_status (*fwd_lse_fn)(const void*, const void*, const void*, void*, float*, int32_t, int32_t, int32_t,
                                 sta_dim3, sta_dim3, const sta_dim3*, float, void*);
typedef sta_status (*bwd_fn)(const void*, const void*, const void*, const void*, const void*, const float*, void*,
                             void*, void*, int32_t, int32_t, int32_t, sta_dim3, sta_dim3, const sta_dim3*, float,
                             void*);

int main(void) {
  const reorder_fn reorders[2] = {sta_tile_reorder, sta_tile_unorder};
  const reorder_tokens_fn reorders_tokens[2] = {sta_tile_reorder_tokens, sta_tile_unorder_tokens};
  const fwd_fn forwards[3] = {sta_attention_fwd, sta_attention_fwd_raster, sta_attention_fwd_noalloc};
  const fwd_lse_fn fwd_lse = sta_attention_fwd_lse;
  const bwd_fn bwd = sta_attention_bwd;
  sta_status (*index_map)(sta_dim3, sta_dim3, int32_t*) = sta_tile_index_map;
  int64_t (*pairs_fn)(int32_t, int32_t, sta_dim3, sta_dim3, const sta_dim3*) = sta_attended_pairs;
  int64_t (*block_pairs)(int32_t, int32_t, sta_dim3, sta_dim3, const sta_dim3*, int32_t, int32_t*, int64_t) =
      sta_schedule_block_pairs;
  sta_status (*check)(void*) = sta_check_device_status;
  sta_status (*selftest)(uint64_t, void*) = sta_selftest_bounded_wait;
  const char* (*status_str)(sta_status) = sta_status_str;
  const char* (*last_error)(void) = sta_last_cuda_error;
  void (*shutdown)(void) = sta_shutdown;
  if (!reorders[0] || !reorders[1] || !reorders_tokens[0] || !reorders_tokens[1] || !forwards[0] || !forwards[1] ||
      !forwards[2] || !fwd_lse || !bwd || !check || !selftest || !last_error || !shutdown || !block_pairs)
    return 2;

  const sta_dim3 grid = {4, 8, 8}, tile = {2, 4, 4};
  const sta_dim3 windows[2] = {{1, 1, 1}, {3, 3, 3}};
  static int32_t map[4 * 8 * 8];
  if (index_map(grid, tile, map) != STA_OK) return 3;
  printf("map");
  for (int i = 0; i < 4 * 8 * 8; ++i) printf(" %d", (int)map[i]);
  printf("\npairs %lld\n", (long long)pairs_fn(1, 2, grid, tile, windows));
  printf("status %s %s\n", status_str(STA_OK), status_str(STA_ERR_SHAPE));
  /* validation runs before any device call: a null pointer is rejected on any machine */
  printf("null %s\n", status_str(reorders[0](NULL, map, 1, 64, grid, tile, NULL)));
  return 0;
}
