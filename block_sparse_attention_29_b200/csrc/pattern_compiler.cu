// pattern_compiler.cu -- host compiler from a static pattern descriptor to
// per-(head, query tile) lists of key blocks.
//
// A row's visible keys are the union, by logical OR ("SAS: Sparse Attention
// Synthesizer", Step 5, component 2), of the primitives of the glossary's
// "Sparse Attention Patterns" table (sliding window with the Mistral rule,
// global tokens, blockwise, BigBird random blocks), capped by the causal
// constraint G_i in {0..i} ("Sparse Attention Weights Assumption").  Each
// primitive contributes one index range per row (random blocks n_random
// ranges), so a tile's per-block pair counts come from range arithmetic: a
// difference array adds tile_k to every block a range covers completely and
// the two edge blocks get their partial lengths.  A block is listed when it
// holds at least one visible pair and is "full" when it holds tile_q*tile_k
// (every pair of the tile, which also rules out ragged tiles and blocks).
//
// A dilated window (dilation k > 1: taps k apart, glossary "Sparse Attention
// Patterns", dilated/strided row) only joins i and j of one residue class
// i mod k, and inside a class, numbered m = i / k, it is the contiguous window
// over N/k positions.  The compiler therefore lists the contiguous window over
// N/k positions once; the kernels run it for every class through a strided
// view of Q, K, V and O.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <vector>

#include "common.h"

namespace sa {

namespace {
struct Range {
  int64_t lo, hi;  // [lo, hi)
};

bool random_on(const sa_pattern_t* p) {
  return p->n_random > 0 && p->random_table != nullptr && p->random_block > 0;
}

// Visible key ranges of row i (unsorted, may overlap), before the causal cap.
int row_ranges(const sa_pattern_t* p, int N, int h, int i, Range* r) {
  int n = 0;
  bool any = false;
  if (p->window > 0) {
    any = true;
    if (p->causal) r[n++] = {int64_t(i) - p->window + 1, int64_t(i) + 1};
    else r[n++] = {int64_t(i) - p->window / 2, int64_t(i) + p->window / 2 + 1};
  }
  if (p->n_global > 0) {
    any = true;
    r[n++] = {0, i < p->n_global ? int64_t(N) : int64_t(p->n_global)};
  }
  if (p->block_local > 0) {
    any = true;
    int64_t lo = int64_t(i / p->block_local) * p->block_local;
    r[n++] = {lo, lo + p->block_local};
  }
  if (random_on(p)) {
    any = true;
    int nrb = (N + p->random_block - 1) / p->random_block;
    const int32_t* row =
        p->random_table + (int64_t(h) * nrb + i / p->random_block) * p->n_random;
    for (int k = 0; k < p->n_random; ++k) {
      int64_t lo = int64_t(row[k]) * p->random_block;
      r[n++] = {lo, lo + p->random_block};
    }
  }
  if (!any) r[n++] = {0, N};
  return n;
}
}  // namespace

int validate_pattern(const sa_pattern_t* p, int H, int N) {
  if (!p) return set_error(SA_ERR_INVALID_ARG, "pattern descriptor is NULL");
  if (H <= 0 || N <= 0) return set_error(SA_ERR_INVALID_ARG, "H and N must be positive");
  if (p->window < 0 || p->n_global < 0 || p->block_local < 0 || p->n_random < 0)
    return set_error(SA_ERR_INVALID_ARG, "negative pattern field");
  if (p->block_q <= 0 || p->block_k <= 0)
    return set_error(SA_ERR_INVALID_ARG, "block_q and block_k must be positive");
  if (p->dilation < 0) return set_error(SA_ERR_INVALID_ARG, "negative dilation");
  if (p->dilation > 1) {
    if (p->window <= 0)
      return set_error(SA_ERR_INVALID_ARG, "dilation %d needs a window", p->dilation);
    if (p->n_global > 0 || p->block_local > 0 || (p->n_random > 0 && p->random_table))
      return set_error(SA_ERR_UNSUPPORTED,
                       "a dilated window cannot be combined with other primitives");
    if (N % p->dilation != 0)
      return set_error(SA_ERR_UNSUPPORTED, "dilation %d does not divide N = %d", p->dilation,
                       N);
  }
  if (p->n_random > 0 && p->random_table != nullptr) {
    if (p->random_block <= 0)
      return set_error(SA_ERR_INVALID_ARG, "random_block must be positive");
    int nrb = (N + p->random_block - 1) / p->random_block;
    int64_t n = int64_t(H) * nrb * p->n_random;
    for (int64_t k = 0; k < n; ++k) {
      int32_t v = p->random_table[k];
      if (v < 0 || v >= nrb)
        return set_error(SA_ERR_INVALID_ARG, "random_table[%lld] = %d outside [0, %d)",
                         (long long)k, v, nrb);
    }
  }
  return SA_OK;
}

int compile_pattern(const sa_pattern_t* p, int H, int N, int tile_q, int tile_k,
                    CompiledPattern* out) {
  int rc = validate_pattern(p, H, N);
  if (rc) return rc;
  if (p->dilation > 1) {   // one residue class: the contiguous window over N/k positions
    sa_pattern_t c = *p;
    c.dilation = 1;
    return compile_pattern(&c, H, N / p->dilation, tile_q, tile_k, out);
  }
  if (tile_q <= 0 || tile_k <= 0) return set_error(SA_ERR_INVALID_ARG, "bad tile size");
  const int H_pat = random_on(p) ? H : 1;
  const int T = (N + tile_q - 1) / tile_q;
  const int n_kb = (N + tile_k - 1) / tile_k;
  out->H_pat = H_pat;
  out->T = T;
  out->n_kb = n_kb;
  out->row_ptr.assign(size_t(H_pat) * T + 1, 0);
  out->kb.clear();
  out->full.clear();
  out->cnt.clear();

  std::vector<Range> ranges(4 + (random_on(p) ? p->n_random : 0));
  std::vector<int64_t> direct(n_kb), diff(n_kb + 1);
  const int64_t full_pairs = int64_t(tile_q) * tile_k;
  for (int hp = 0; hp < H_pat; ++hp) {
    for (int t = 0; t < T; ++t) {
      std::fill(direct.begin(), direct.end(), 0);
      std::fill(diff.begin(), diff.end(), 0);
      const int i0 = t * tile_q, i1 = std::min(N, i0 + tile_q);
      for (int i = i0; i < i1; ++i) {
        int nr = row_ranges(p, N, hp, i, ranges.data());
        std::sort(ranges.begin(), ranges.begin() + nr,
                  [](const Range& a, const Range& b) { return a.lo < b.lo; });
        const int64_t cap = p->causal ? std::min<int64_t>(int64_t(i) + 1, N) : int64_t(N);
        int64_t next = 0;  // keys below `next` are already counted for this row
        for (int k = 0; k < nr; ++k) {
          int64_t lo = std::max<int64_t>(std::max<int64_t>(ranges[k].lo, next), 0);
          int64_t hi = std::min<int64_t>(ranges[k].hi, cap);
          if (hi > lo) {
            int64_t b0 = lo / tile_k, b1 = (hi - 1) / tile_k;
            if (b0 == b1) {
              direct[b0] += hi - lo;
            } else {
              direct[b0] += (b0 + 1) * tile_k - lo;
              direct[b1] += hi - b1 * tile_k;
              diff[b0 + 1] += tile_k;
              diff[b1] -= tile_k;
            }
          }
          next = std::max(next, hi);
        }
      }
      int64_t run = 0;
      for (int b = 0; b < n_kb; ++b) {
        run += diff[b];
        int64_t c = direct[b] + run;
        if (c > 0) {
          out->kb.push_back(b);
          out->full.push_back(c == full_pairs ? 1 : 0);
          out->cnt.push_back(c);
        }
      }
      size_t row = size_t(hp) * T + t;
      if (out->kb.size() > size_t(INT32_MAX))
        return set_error(SA_ERR_NO_MEMORY, "block list longer than 2^31 entries");
      out->row_ptr[row + 1] = int32_t(out->kb.size());
    }
  }
  return SA_OK;
}

void order_units(const CompiledPattern& cp, int B, int H, int H_kv, int64_t kv_bytes, int ctas,
                 int max_unit_blocks, int64_t slot_bytes, UnitOrder* out) {
  const int T = cp.T;
  const int64_t n = int64_t(B) * H * T;
  auto cost_of = [&](int32_t u) {
    const int t = u % T, h = (u / T) % H;
    const int row = (cp.H_pat > 1 ? h : 0) * T + t;
    return cp.row_ptr[row + 1] - cp.row_ptr[row];
  };
  int64_t total = 0;
  std::vector<int32_t> costs;
  costs.reserve(size_t(n));
  for (int64_t u = 0; u < n; ++u) {
    costs.push_back(cost_of(int32_t(u)));
    total += costs.back();
  }
  // Units longer than half of one CTA's share of the work would set the tail
  // if they started late.
  const int64_t heavy = std::max<int64_t>(1, total / (2 * std::max(ctas, 1)) / 2);
  const int64_t share = total / std::max(ctas, 1);   // one CTA's share of the work

  // Split tiles.  A tile whose list is far longer than the others (the rows
  // of global tokens see every key) is cut into pieces of consecutive blocks,
  // each a work unit of its own that writes an unnormalised partial result
  // (O, row maximum, row sum) to a workspace slot; the CTA that finishes a
  // tile's last piece combines them.  The pieces run beside the other units
  // of their head, while that head's K and V are in L2, and spread the tile
  // over many CTAs.  Automatic (max_unit_blocks = 0): pieces of
  // P = max(32, 2 x median list) blocks for tiles longer than one CTA's share
  // of the whole work (unsplit, such a tile alone would set the launch time)
  // and than 2 P, within a 256 MiB workspace; max_unit_blocks > 0 cuts every
  // list longer than that; < 0 never splits.
  int64_t piece_len = 0;
  if (max_unit_blocks > 0) {
    piece_len = max_unit_blocks;
  } else if (max_unit_blocks == 0 && n > 0) {
    std::vector<int32_t> sorted(costs);
    std::nth_element(sorted.begin(), sorted.begin() + sorted.size() / 2, sorted.end());
    piece_len = std::max<int64_t>(32, 2 * int64_t(sorted[sorted.size() / 2]));
  }
  // piece: index into out->pieces, or -1; cost: the list length the order
  // uses (for the pieces of a tile, the longest piece's, so that they stay
  // together in list order)
  struct Item { int32_t id, k0, n, piece, cost; };
  std::vector<Item> items;
  items.reserve(size_t(n));
  out->pieces.clear();
  out->split.clear();
  int64_t slots = 0;
  for (int64_t u = 0; u < n; ++u) {
    const int32_t c = costs[size_t(u)];
    bool split = false;
    if (max_unit_blocks > 0) split = c > piece_len;
    else if (max_unit_blocks == 0) split = c > share && c > 2 * piece_len;
    const int64_t np = split ? (c + piece_len - 1) / piece_len : 1;
    if (split && max_unit_blocks == 0 && (slots + np) * slot_bytes > (int64_t(256) << 20))
      split = false;
    if (!split) {
      items.push_back({int32_t(u), 0, c, -1, c});
      continue;
    }
    // np pieces of near-equal length
    SplitTile st;
    st.id = int32_t(u);
    st.first_slot = int32_t(slots);
    st.n_pieces = int32_t(np);
    st.pad = 0;
    out->split.push_back(st);
    for (int64_t j = 0; j < np; ++j) {
      const int32_t k0 = int32_t(j * c / np), k1 = int32_t((j + 1) * c / np);
      Piece pc;
      pc.id = int32_t(u);
      pc.k0 = k0;
      pc.n = k1 - k0;
      pc.slot = int32_t(slots + j);
      pc.split = int32_t(out->split.size() - 1);
      pc.first_slot = int32_t(slots);
      pc.n_pieces = int32_t(np);
      pc.pad = 0;
      items.push_back({int32_t(u), k0, k1 - k0, int32_t(out->pieces.size()),
                       int32_t((c + np - 1) / np)});
      out->pieces.push_back(pc);
    }
    slots += np;
  }
  out->n_slots = slots;

  // Order: heavy units first, longest first.  When all of K and V fit in half
  // of L2 the rest are ordered tile-major (later tiles first, the larger ones
  // under a causal mask); otherwise K/V-group-major -- all tiles of the query
  // heads that share one K/V head run together, so that head's K and V stay in
  // L2 while they are reused -- longest first inside a group.  The query heads
  // of a group are adjacent either way; the pieces of a split tile run in
  // descending key order, like the tiles of their head.
  const bool group_major = kv_bytes > (int64_t(64) << 20);
  const int group = std::max(H / H_kv, 1);
  const int groups = std::max(H / group, 1);
  // Group-major position of an item: its (b, K/V group) in queue order; the
  // pieces of a split tile move one group earlier, so that they (and the merge
  // their last one triggers) finish while their own group's tiles still run --
  // also for the last group -- with their head's K and V read shortly before.
  auto slot_of = [&](const Item& x) {
    const int bh = x.id / T;
    const int lg = (bh / H) * groups + (bh % H) / group;
    return x.piece >= 0 ? std::max(lg - 1, 0) : lg;
  };
  std::stable_sort(items.begin(), items.end(), [&](const Item& x, const Item& y) {
    const int ca = x.cost, cb = y.cost;
    const bool ha_ = ca > heavy, hb_ = cb > heavy;
    if (ha_ != hb_) return ha_;
    if (ha_ && ca != cb) return ca > cb;
    const int bha = x.id / T, bhb = y.id / T;
    const int ba = bha / H, bb = bhb / H, ha = bha % H, hb = bhb % H;
    if (!ha_ && group_major) {
      const int ga = slot_of(x), gb = slot_of(y);
      if (ga != gb) return ga < gb;
      if (ca != cb) return ca > cb;
      if (ha / group != hb / group) return ha / group < hb / group;
    }
    const int ta = x.id % T, tb = y.id % T;
    if (ta != tb) return ta > tb;
    if (ba != bb) return ba < bb;
    if (ha != hb) return ha < hb;
    return x.k0 > y.k0;
  });
  out->units.resize(items.size());
  for (size_t k = 0; k < items.size(); ++k)
    out->units[k] = items[k].piece < 0 ? items[k].id : ~items[k].piece;
}

}  // namespace sa
