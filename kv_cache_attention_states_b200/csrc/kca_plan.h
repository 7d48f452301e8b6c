// kca_plan.h -- integer bookkeeping of the attention calls, shared verbatim by
// the host (validation, workspace sizes, plan queries) and the device (each
// CTA recomputes its own work item from the same formulas, so no plan ever
// has to be copied to the GPU).
//
// Visible keys of a query at position pos: J(pos) = [lo(pos), pos] with
// lo(pos) = window > 0 ? max(0, pos - window + 1) : 0 (the sliding window of
// the local layers; without a window every cached row before the query and
// the query's own row, as chunked prefill requires -- Karume v0.8.0 release
// notes, "Features", conversation-window item).
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define KCA_HD __host__ __device__ __forceinline__
#else
#define KCA_HD inline
#endif

namespace kca {

constexpr int kHeads = 8;        // query heads per KV head
constexpr int kDim = 256;        // head_dim
constexpr int kRowTile = 16;     // query positions per tensor-core row tile (16 x 8 heads = 128 M rows)
constexpr int kKeyTile = 128;    // keys per tensor-core KV tile
constexpr int kPartFloats = 2 + kDim;  // per (slot, row): m, l, acc[256]

KCA_HD int64_t lo_of(int64_t pos, int32_t window) {
  if (window > 0) {
    const int64_t lo = pos - window + 1;
    return lo > 0 ? lo : 0;
  }
  return 0;
}
KCA_HD int64_t n_visible(int64_t pos, int32_t window) {
  const int64_t lo = lo_of(pos, window);
  return pos >= lo ? pos - lo + 1 : 0;
}
KCA_HD int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
// Visible keys of the query at pos that a context shard holding positions
// [key_begin, key_end) sees: [*lo, *lo + n), n returned (key_end <= 0: no
// upper end, i.e. the whole context from key_begin on).
KCA_HD int64_t shard_visible(int64_t pos, int32_t window, int64_t key_begin, int64_t key_end, int64_t* lo) {
  int64_t l = lo_of(pos, window), h = pos + 1;
  if (l < key_begin) l = key_begin;
  if (key_end > 0 && h > key_end) h = key_end;
  *lo = l;
  return h > l ? h - l : 0;
}

// ------------------------------------------------------------ rows path
// One unit = one query row (prefill) or one sequence (decode).  Its visible
// keys are cut into splits of split_len keys; a unit with no visible key has
// one empty split that writes zeros.
struct RowsPlan {
  int32_t n_units;
  int32_t split_len;
  int32_t max_splits;
};

KCA_HD int32_t rows_n_splits(int64_t nkeys, int32_t split_len) {
  return nkeys <= 0 ? 1 : (int32_t)cdiv(nkeys, split_len);
}

// Rows path tuning: resident CTAs per SM the plan aims to fill (the rows
// kernel runs one CTA per SM), the smallest split, and the split quantum
// (the kernel's keys per shared-memory stage).
constexpr int kRowsCtasPerSm = 1;
constexpr int kRowsMinSplit = 64;
constexpr int kRowsSplitQuantum = 16;

// nkeys[u]: visible keys of unit u.  split_len is the smallest multiple of
// the quantum (>= min_split) whose split count fits one wave; when even one
// split per unit does not fit, every unit gets a single split.  Multi-row
// units, whose CTAs cost more to start (a unit's queries, tensor memory, a
// merge of more rows), take longer splits at least.
constexpr int kMultiRowMinSplit = 256;
inline RowsPlan make_rows_plan(int32_t n_units, const int64_t* nkeys, int32_t num_sms,
                               int32_t min_split = kRowsMinSplit) {
  RowsPlan p;
  p.n_units = n_units;
  int64_t max_keys = 0;
  for (int32_t u = 0; u < n_units; ++u) max_keys = nkeys[u] > max_keys ? nkeys[u] : max_keys;
  const int64_t target = (int64_t)(num_sms > 0 ? num_sms : 1) * kRowsCtasPerSm;
  auto count = [&](int64_t len) {
    int64_t c = 0;
    for (int32_t u = 0; u < n_units; ++u) c += rows_n_splits(nkeys[u], (int32_t)len);
    return c;
  };
  int64_t hi = cdiv(max_keys > min_split ? max_keys : min_split, kRowsSplitQuantum);
  int64_t lo = cdiv(min_split, kRowsSplitQuantum);
  if (count(lo * kRowsSplitQuantum) <= target) {
    hi = lo;
  } else {
    // smallest quantum multiple in (lo, hi] whose count fits (count(hi) == n_units)
    while (lo + 1 < hi) {
      const int64_t mid = (lo + hi) / 2;
      if (count(mid * kRowsSplitQuantum) <= target) hi = mid; else lo = mid;
    }
  }
  p.split_len = (int32_t)(hi * kRowsSplitQuantum);
  p.max_splits = rows_n_splits(max_keys, p.split_len);
  return p;
}

// Tensor-core rows kernel: the splits of a unit run as clusters of `cluster`
// CTAs (one CTA per SM), so a unit with n splits takes ceil(n / cluster)
// clusters.  split_len is the smallest multiple of the kernel's stage
// (kRowsMmaStage keys) whose clusters all fit the `slots` clusters that can be
// resident at once; when one split per unit does not fit, every unit gets one.
constexpr int kRowsMmaStage = 64;
constexpr int kRowsMmaMaxClusterParts = 256;   // the kernel merges at most this many cluster partials

inline RowsPlan make_cluster_rows_plan(int32_t n_units, const int64_t* nkeys, int32_t cluster,
                                       int32_t slots) {
  RowsPlan p;
  p.n_units = n_units;
  int64_t max_keys = 0;
  for (int32_t u = 0; u < n_units; ++u) max_keys = nkeys[u] > max_keys ? nkeys[u] : max_keys;
  const int64_t c = cluster > 0 ? cluster : 1;
  const int64_t target = slots > 0 ? slots : 1;
  auto count = [&](int64_t len) {
    int64_t n = 0;
    for (int32_t u = 0; u < n_units; ++u) n += cdiv(rows_n_splits(nkeys[u], (int32_t)len), c);
    return n;
  };
  int64_t hi = cdiv(max_keys > kRowsMmaStage ? max_keys : kRowsMmaStage, kRowsMmaStage);
  int64_t lo = 1;
  if (count(lo * kRowsMmaStage) <= target) {
    hi = lo;
  } else {
    while (lo + 1 < hi) {
      const int64_t mid = (lo + hi) / 2;
      if (count(mid * kRowsMmaStage) <= target) hi = mid; else lo = mid;
    }
  }
  p.split_len = (int32_t)(hi * kRowsMmaStage);
  p.max_splits = rows_n_splits(max_keys, p.split_len);
  return p;
}

// ------------------------------------------------------ tensor-core path
// A chunk of `rows` query rows at chunk_start is cut into row tiles of 16
// positions (x 8 heads = 128 M rows).  Keys are addressed relative to
// kv_lo = lo(chunk_start), the first key any row of the chunk sees, in tiles
// of 128.  Row tiles go in pairs (2q, 2q+1) to the two SMs of a CTA pair,
// which share every K/V tile (each SM loads half of it); a pair covers the
// union of its tiles' key ranges [kb(2q), ke(2q+1)), each row masking the
// keys it does not see.  A pair's range is split into ceil(n/c) items of
// near-equal length, c chosen as the smallest value that keeps the pair
// items within one wave of CTA pairs.
struct TcPlan {
  int64_t chunk_start;
  int64_t kv_lo;
  int64_t ctx_len;      // chunk_start + rows: keys at or beyond it are outside the map
  int32_t rows;
  int32_t window;
  int32_t n_tiles;
  int32_t n_pairs;
  int32_t per_item;     // c: most key tiles one item covers
  int32_t n_items;      // pair items (each runs on a CTA pair)
  int32_t n_slots;      // partial slots: one per (tile, item) of split pairs
  int32_t max_split;    // most items of one pair
};

constexpr int kTcMinItemTiles = 2;

KCA_HD void tc_tile_keys(const TcPlan& p, int32_t t, int32_t* kb, int32_t* ke) {
  const int64_t first = p.chunk_start + (int64_t)t * kRowTile;
  int64_t last = p.chunk_start + (int64_t)(t + 1) * kRowTile - 1;
  const int64_t end = p.chunk_start + p.rows - 1;
  if (last > end) last = end;
  *kb = (int32_t)((lo_of(first, p.window) - p.kv_lo) / kKeyTile);
  *ke = (int32_t)((last - p.kv_lo) / kKeyTile + 1);
}
KCA_HD int32_t tc_pair_tiles(const TcPlan& p, int32_t q) { return 2 * q + 1 < p.n_tiles ? 2 : 1; }
// Key tiles [kb, ke) of pair q: the union of its tiles' ranges (lo and the
// last position both grow with the tile index).
KCA_HD void tc_pair_keys(const TcPlan& p, int32_t q, int32_t* kb, int32_t* ke) {
  int32_t kb1, ke1;
  tc_tile_keys(p, 2 * q, kb, ke);
  if (tc_pair_tiles(p, q) == 2) {
    tc_tile_keys(p, 2 * q + 1, &kb1, &ke1);
    *ke = ke1;
  }
}
KCA_HD int32_t tc_pair_items(const TcPlan& p, int32_t q) {
  int32_t kb, ke;
  tc_pair_keys(p, q, &kb, &ke);
  return (int32_t)cdiv(ke - kb, p.per_item);
}

// Start of split k of a pair's n key tiles cut into s items: ceil(k n / s),
// so the items differ by at most one tile and any longer ones come first.
// The last item holds the causal diagonal (its last tile is partly masked
// and its K / V rows were not read by the previous chunk), so a spare tile
// is better placed on an earlier one.
KCA_HD int32_t tc_split_at(int32_t n, int32_t s, int32_t k) {
  return (int32_t)(((int64_t)k * n + s - 1) / s);
}

struct TcItem {
  int32_t pair;
  int32_t kt_begin;   // key tiles, relative to kv_lo
  int32_t kt_end;
  int32_t slot0;      // partial slot of tile 2 pair, -1 when the pair is not split
  int32_t slot1;      // partial slot of tile 2 pair + 1 (-1 also when that tile does not exist)
  int32_t split;      // index within the pair
  int32_t n_split;
};

// Item `idx` of the plan (items ordered by pair, then by split).
KCA_HD TcItem tc_item(const TcPlan& p, int32_t idx) {
  TcItem it{};
  int32_t base = 0, slot_base = 0;
  for (int32_t q = 0; q < p.n_pairs; ++q) {
    int32_t kb, ke;
    tc_pair_keys(p, q, &kb, &ke);
    const int32_t n = ke - kb;
    const int32_t s = (int32_t)cdiv(n, p.per_item);
    const int32_t nt = tc_pair_tiles(p, q);
    if (idx < base + s) {
      const int32_t k = idx - base;
      it.pair = q;
      it.kt_begin = kb + tc_split_at(n, s, k);
      it.kt_end = kb + tc_split_at(n, s, k + 1);
      it.split = k;
      it.n_split = s;
      it.slot0 = s > 1 ? slot_base + k : -1;
      it.slot1 = (s > 1 && nt == 2) ? slot_base + s + k : -1;
      return it;
    }
    base += s;
    if (s > 1) slot_base += s * nt;
  }
  it.pair = -1;
  return it;
}

// pair_budget: CTA pairs that run at once (one wave).
inline TcPlan make_tc_plan(int64_t chunk_start, int32_t rows, int32_t window, int32_t pair_budget) {
  TcPlan p{};
  p.chunk_start = chunk_start;
  p.rows = rows;
  p.window = window;
  p.kv_lo = lo_of(chunk_start, window);
  p.ctx_len = chunk_start + rows;
  p.n_tiles = (int32_t)cdiv(rows, kRowTile);
  p.n_pairs = (int32_t)cdiv(p.n_tiles, 2);
  int64_t total = 0;
  int32_t longest = 1;
  for (int32_t q = 0; q < p.n_pairs; ++q) {
    int32_t kb, ke;
    tc_pair_keys(p, q, &kb, &ke);
    total += ke - kb;
    if (ke - kb > longest) longest = ke - kb;
  }
  // one wave of CTA pairs, capped by the launch's item table (80 entries)
  const int32_t budget = pair_budget < 1 ? 1 : (pair_budget > 80 ? 80 : pair_budget);
  int32_t c = (int32_t)cdiv(total, budget);
  if (c < kTcMinItemTiles) c = kTcMinItemTiles;
  for (;; ++c) {
    p.per_item = c;
    int64_t items = 0;
    for (int32_t q = 0; q < p.n_pairs; ++q) items += tc_pair_items(p, q);
    if (items <= budget || c >= longest) break;
  }
  int32_t items = 0, slots = 0, most = 1;
  for (int32_t q = 0; q < p.n_pairs; ++q) {
    const int32_t s = tc_pair_items(p, q);
    items += s;
    if (s > 1) slots += s * tc_pair_tiles(p, q);
    if (s > most) most = s;
  }
  p.n_items = items;
  p.n_slots = slots;
  p.max_split = most;
  return p;
}

}  // namespace kca
