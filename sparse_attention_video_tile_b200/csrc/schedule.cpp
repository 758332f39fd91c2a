// schedule.cpp - host window enumerator and work scheduler.
//
// For every head the effective window w' = min(w, n) and, for every query tile
// a, the window start s = clamp(a - floor(w'/2), 0, n - w') per dimension give
// the key tiles the tile attends (sliding tile attention: the window moves
// tile by tile, "Fast Video Generation with Sliding Tile Attention", abstract;
// per-head windows, summary page, "Technical contribution").
//
// The attention kernel works on blocks of 128 query rows and 128 key rows in
// tiled order.  When Ntile is a multiple of 128 every block lies inside one
// tile, so a query block attends whole key blocks and needs no mask: its list
// is the window's tiles, each expanded to Ntile/128 key blocks, shared by the
// Ntile/128 query blocks of the tile.  Otherwise a block may straddle tiles;
// its list is the union of the key blocks touched by the windows of the tiles
// it covers, and the kernel masks at tile granularity.
//
// Work items are ordered by decreasing cost (number of key blocks), ties kept
// in (batch*head, query block) order, so that a strided assignment of items to
// a persistent grid balances per-head windows of different sizes, and CTAs that
// run at the same time share key/value tiles in L2.
#include <algorithm>
#include <array>
#include <map>
#include <set>
#include <tuple>

#include "internal.h"

namespace sta {

sta_status make_geometry(sta_dim3 grid, sta_dim3 tile, Geometry* g) {
  if (grid.t <= 0 || grid.h <= 0 || grid.w <= 0 || tile.t <= 0 || tile.h <= 0 || tile.w <= 0)
    return STA_ERR_SHAPE;
  if (grid.t % tile.t || grid.h % tile.h || grid.w % tile.w) return STA_ERR_SHAPE;
  const int64_t L = static_cast<int64_t>(grid.t) * grid.h * grid.w;
  if (L >= (int64_t(1) << 31) - kBlockRows) return STA_ERR_SHAPE;
  g->T = grid.t; g->H = grid.h; g->W = grid.w;
  g->tt = tile.t; g->th = tile.h; g->tw = tile.w;
  g->nT = grid.t / tile.t; g->nH = grid.h / tile.h; g->nW = grid.w / tile.w;
  g->ntile = tile.t * tile.h * tile.w;
  g->L = L;
  g->Lpad = L;
  g->padded = false;
  return STA_OK;
}

sta_status make_geometry_padded(sta_dim3 grid, sta_dim3 tile, Geometry* g) {
  if (grid.t <= 0 || grid.h <= 0 || grid.w <= 0 || tile.t <= 0 || tile.h <= 0 || tile.w <= 0)
    return STA_ERR_SHAPE;
  const int64_t nT = (grid.t + tile.t - 1) / tile.t, nH = (grid.h + tile.h - 1) / tile.h,
                nW = (grid.w + tile.w - 1) / tile.w;
  const int64_t ntile = static_cast<int64_t>(tile.t) * tile.h * tile.w;
  const int64_t Lpad = nT * nH * nW * ntile;
  if (Lpad >= (int64_t(1) << 31) - kBlockRows || ntile >= (int64_t(1) << 31)) return STA_ERR_SHAPE;
  g->T = grid.t; g->H = grid.h; g->W = grid.w;
  g->tt = tile.t; g->th = tile.h; g->tw = tile.w;
  g->nT = static_cast<int32_t>(nT); g->nH = static_cast<int32_t>(nH); g->nW = static_cast<int32_t>(nW);
  g->ntile = static_cast<int32_t>(ntile);
  g->L = static_cast<int64_t>(grid.t) * grid.h * grid.w;
  g->Lpad = Lpad;
  g->padded = Lpad != g->L;
  return STA_OK;
}

namespace {

struct Eff {
  int32_t t, h, w;
  bool operator<(const Eff& o) const { return std::tie(t, h, w) < std::tie(o.t, o.h, o.w); }
};

// Key tile ids of the window of query tile `qt` (raster order over the tile grid).
void window_tiles(const Geometry& g, const Eff& e, int32_t qt, std::vector<int32_t>* out) {
  const int32_t at = qt / (g.nH * g.nW);
  const int32_t ah = (qt / g.nW) % g.nH;
  const int32_t aw = qt % g.nW;
  const int32_t st = window_start_1d(at, e.t, g.nT);
  const int32_t sh = window_start_1d(ah, e.h, g.nH);
  const int32_t sw = window_start_1d(aw, e.w, g.nW);
  out->clear();
  for (int32_t kt = st; kt < st + e.t; ++kt)
    for (int32_t kh = sh; kh < sh + e.h; ++kh)
      for (int32_t kw = sw; kw < sw + e.w; ++kw) out->push_back((kt * g.nH + kh) * g.nW + kw);
}

}  // namespace

void build_schedule(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                    HostSchedule* s) {
  s->masked = (g.ntile % kBlockRows) != 0;
  s->items.clear();
  s->kv_rows.clear();
  s->head_win.assign(static_cast<size_t>(heads) * 4, 0);
  s->attended_pairs = 0;

  const int32_t n_tiles = g.nT * g.nH * g.nW;
  const int32_t n_qblocks = static_cast<int32_t>((g.L + kBlockRows - 1) / kBlockRows);

  // One list set per distinct effective window.
  std::map<Eff, std::vector<std::pair<int32_t, int32_t>>> lists;  // per query block: (off, len)
  std::vector<int32_t> tiles;
  std::vector<Eff> eff(heads);
  for (int32_t h = 0; h < heads; ++h) {
    Eff e{std::min(windows[h].t, g.nT), std::min(windows[h].h, g.nH), std::min(windows[h].w, g.nW)};
    eff[h] = e;
    s->head_win[h * 4 + 0] = static_cast<int16_t>(e.t);
    s->head_win[h * 4 + 1] = static_cast<int16_t>(e.h);
    s->head_win[h * 4 + 2] = static_cast<int16_t>(e.w);
    s->attended_pairs += static_cast<int64_t>(batch) * g.L * g.ntile * e.t * e.h * e.w;
    if (lists.count(e)) continue;
    std::vector<std::pair<int32_t, int32_t>>& per_qb = lists[e];
    per_qb.resize(n_qblocks);
    if (!s->masked) {
      const int32_t bpt = g.ntile / kBlockRows;  // key/query blocks per tile
      for (int32_t qt = 0; qt < n_tiles; ++qt) {
        window_tiles(g, e, qt, &tiles);
        const int32_t off = static_cast<int32_t>(s->kv_rows.size());
        for (int32_t kt : tiles)
          for (int32_t b = 0; b < bpt; ++b) s->kv_rows.push_back(kt * g.ntile + b * kBlockRows);
        const int32_t len = static_cast<int32_t>(s->kv_rows.size()) - off;
        for (int32_t b = 0; b < bpt; ++b) per_qb[qt * bpt + b] = {off, len};
      }
    } else {
      for (int32_t qb = 0; qb < n_qblocks; ++qb) {
        const int64_t r0 = static_cast<int64_t>(qb) * kBlockRows;
        const int64_t r1 = std::min<int64_t>(g.L, r0 + kBlockRows);
        std::set<int32_t> blocks;
        for (int32_t qt = static_cast<int32_t>(r0 / g.ntile); qt <= static_cast<int32_t>((r1 - 1) / g.ntile); ++qt) {
          window_tiles(g, e, qt, &tiles);
          for (int32_t kt : tiles) {
            const int64_t k0 = static_cast<int64_t>(kt) * g.ntile;
            const int64_t k1 = k0 + g.ntile - 1;
            for (int64_t b = k0 / kBlockRows; b <= k1 / kBlockRows; ++b) blocks.insert(static_cast<int32_t>(b));
          }
        }
        const int32_t off = static_cast<int32_t>(s->kv_rows.size());
        for (int32_t b : blocks) s->kv_rows.push_back(b * kBlockRows);
        per_qb[qb] = {off, static_cast<int32_t>(blocks.size())};
      }
    }
  }

  s->items.reserve(static_cast<size_t>(batch) * heads * n_qblocks);
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t h = 0; h < heads; ++h) {
      const auto& per_qb = lists[eff[h]];
      for (int32_t qb = 0; qb < n_qblocks; ++qb)
        s->items.push_back(WorkItem{b * heads + h, qb * kBlockRows, per_qb[qb].first, per_qb[qb].second});
    }
  std::stable_sort(s->items.begin(), s->items.end(),
                   [](const WorkItem& x, const WorkItem& y) { return x.kv_len > y.kv_len; });
}

void build_schedule_transposed(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                               HostSchedule* s) {
  // Same windows as build_schedule, seen from the key side: key tile c is attended
  // by the query tiles a whose window contains c.  Only Ntile multiples of 128.
  s->masked = false;
  s->items.clear();
  s->kv_rows.clear();
  s->head_win.assign(static_cast<size_t>(heads) * 4, 0);
  s->attended_pairs = 0;
  const int32_t n_tiles = g.nT * g.nH * g.nW;
  const int32_t bpt = g.ntile / kBlockRows;
  const int32_t n_kblocks = n_tiles * bpt;
  std::map<Eff, std::vector<std::pair<int32_t, int32_t>>> lists;  // per key block: (off, len)
  std::vector<int32_t> tiles;
  std::vector<Eff> eff(heads);
  for (int32_t h = 0; h < heads; ++h) {
    Eff e{std::min(windows[h].t, g.nT), std::min(windows[h].h, g.nH), std::min(windows[h].w, g.nW)};
    eff[h] = e;
    s->head_win[h * 4 + 0] = static_cast<int16_t>(e.t);
    s->head_win[h * 4 + 1] = static_cast<int16_t>(e.h);
    s->head_win[h * 4 + 2] = static_cast<int16_t>(e.w);
    s->attended_pairs += static_cast<int64_t>(batch) * g.L * g.ntile * e.t * e.h * e.w;
    if (lists.count(e)) continue;
    std::vector<std::vector<int32_t>> by_key(n_tiles);   // query tiles attending each key tile
    for (int32_t qt = 0; qt < n_tiles; ++qt) {
      window_tiles(g, e, qt, &tiles);
      for (int32_t kt : tiles) by_key[kt].push_back(qt);
    }
    std::vector<std::pair<int32_t, int32_t>>& per_kb = lists[e];
    per_kb.resize(n_kblocks);
    for (int32_t kt = 0; kt < n_tiles; ++kt) {
      const int32_t off = static_cast<int32_t>(s->kv_rows.size());
      for (int32_t qt : by_key[kt])
        for (int32_t b = 0; b < bpt; ++b) s->kv_rows.push_back(qt * g.ntile + b * kBlockRows);
      const int32_t len = static_cast<int32_t>(s->kv_rows.size()) - off;
      for (int32_t b = 0; b < bpt; ++b) per_kb[kt * bpt + b] = {off, len};
    }
  }
  s->items.reserve(static_cast<size_t>(batch) * heads * n_kblocks);
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t h = 0; h < heads; ++h) {
      const auto& per_kb = lists[eff[h]];
      for (int32_t kb = 0; kb < n_kblocks; ++kb)
        s->items.push_back(WorkItem{b * heads + h, kb * kBlockRows, per_kb[kb].first, per_kb[kb].second});
    }
  std::stable_sort(s->items.begin(), s->items.end(),
                   [](const WorkItem& x, const WorkItem& y) { return x.kv_len > y.kv_len; });
}

namespace {

// Whether tiled row m (of the padded latent) is a real token.
bool row_is_real(const Geometry& g, int64_t m) {
  const int64_t tile = m / g.ntile;
  const int32_t local = static_cast<int32_t>(m - tile * g.ntile);
  const int32_t at = static_cast<int32_t>(tile / (static_cast<int64_t>(g.nH) * g.nW));
  const int32_t ah = static_cast<int32_t>((tile / g.nW) % g.nH);
  const int32_t aw = static_cast<int32_t>(tile % g.nW);
  const int32_t lt = local / (g.th * g.tw), lh = (local / g.tw) % g.th, lw = local % g.tw;
  return at * g.tt + lt < g.T && ah * g.th + lh < g.H && aw * g.tw + lw < g.W;
}

}  // namespace

void build_schedule_raster(const Geometry& g, int32_t batch, int32_t heads, const sta_dim3* windows,
                           HostSchedule* s) {
  s->masked = false;
  s->items.clear();
  s->kv_rows.clear();
  s->kv_mask_id.clear();
  s->kv_masks.clear();
  s->head_win.assign(static_cast<size_t>(heads) * 4, 0);
  s->attended_pairs = 0;

  const int32_t n_tiles = g.nT * g.nH * g.nW;
  const int32_t bpt = g.ntile / kBlockRows;  // 128-row blocks per tile
  // Per block of the padded tiled order: real rows and, when partial, a mask id.
  std::vector<int32_t> real_rows(static_cast<size_t>(n_tiles) * bpt, kBlockRows);
  std::vector<int32_t> block_mask(static_cast<size_t>(n_tiles) * bpt, -1);
  if (g.padded) {
    std::map<std::array<uint32_t, 4>, int32_t> dedup;
    for (int64_t blk = 0; blk < static_cast<int64_t>(n_tiles) * bpt; ++blk) {
      std::array<uint32_t, 4> bits{0, 0, 0, 0};
      int32_t n = 0;
      for (int32_t i = 0; i < kBlockRows; ++i)
        if (row_is_real(g, blk * kBlockRows + i)) {
          bits[i >> 5] |= 1u << (i & 31);
          ++n;
        }
      real_rows[blk] = n;
      if (n > 0 && n < kBlockRows) {
        auto it = dedup.find(bits);
        if (it == dedup.end()) {
          const int32_t id = static_cast<int32_t>(s->kv_masks.size() / 4);
          for (uint32_t w : bits) s->kv_masks.push_back(w);
          it = dedup.emplace(bits, id).first;
        }
        block_mask[blk] = it->second;
      }
    }
  }

  std::map<Eff, std::vector<std::pair<int32_t, int32_t>>> lists;  // per query tile: (off, len)
  std::vector<int32_t> tiles;
  std::vector<Eff> eff(heads);
  for (int32_t h = 0; h < heads; ++h) {
    Eff e{std::min(windows[h].t, g.nT), std::min(windows[h].h, g.nH), std::min(windows[h].w, g.nW)};
    eff[h] = e;
    s->head_win[h * 4 + 0] = static_cast<int16_t>(e.t);
    s->head_win[h * 4 + 1] = static_cast<int16_t>(e.h);
    s->head_win[h * 4 + 2] = static_cast<int16_t>(e.w);
    if (lists.count(e)) continue;
    std::vector<std::pair<int32_t, int32_t>>& per_tile = lists[e];
    per_tile.resize(n_tiles);
    for (int32_t qt = 0; qt < n_tiles; ++qt) {
      window_tiles(g, e, qt, &tiles);
      const int32_t off = static_cast<int32_t>(s->kv_rows.size());
      for (int32_t kt : tiles)
        for (int32_t b = 0; b < bpt; ++b) {
          const int64_t blk = static_cast<int64_t>(kt) * bpt + b;
          if (real_rows[blk] == 0) continue;  // nothing but pad keys
          s->kv_rows.push_back(static_cast<int32_t>(blk * kBlockRows));
          s->kv_mask_id.push_back(block_mask[blk]);
        }
      per_tile[qt] = {off, static_cast<int32_t>(s->kv_rows.size()) - off};
    }
  }
  // Attended pairs: real query rows times real keys of their window.
  for (int32_t h = 0; h < heads; ++h) {
    const auto& per_tile = lists[eff[h]];
    for (int32_t qt = 0; qt < n_tiles; ++qt) {
      int64_t keys = 0;
      for (int32_t i = per_tile[qt].first; i < per_tile[qt].first + per_tile[qt].second; ++i)
        keys += real_rows[s->kv_rows[i] / kBlockRows];
      int64_t qrows = 0;
      for (int32_t b = 0; b < bpt; ++b) qrows += real_rows[static_cast<int64_t>(qt) * bpt + b];
      s->attended_pairs += static_cast<int64_t>(batch) * qrows * keys;
    }
  }

  s->items.reserve(static_cast<size_t>(batch) * heads * n_tiles * bpt);
  for (int32_t b = 0; b < batch; ++b)
    for (int32_t h = 0; h < heads; ++h) {
      const auto& per_tile = lists[eff[h]];
      for (int32_t qt = 0; qt < n_tiles; ++qt)
        for (int32_t qb = 0; qb < bpt; ++qb) {
          if (real_rows[static_cast<int64_t>(qt) * bpt + qb] == 0) continue;  // only pad rows
          s->items.push_back(WorkItem{b * heads + h, (qt * bpt + qb) * kBlockRows, per_tile[qt].first,
                                      per_tile[qt].second});
        }
    }
  std::stable_sort(s->items.begin(), s->items.end(),
                   [](const WorkItem& x, const WorkItem& y) { return x.kv_len > y.kv_len; });
}

}  // namespace sta
