// Host-side plan builder (see plan.h).
//
// The plan is the host half of the pages' plan/run split (M* page
// "mstar.engine.resources.attn.cross", FlashInferCrossManager.plan): it is computed once per
// step and plan label and then read by every layer's run.  It turns the query packing
// (QueryPacking.qo_indptr) and the context page table into
//   * work units: (request, KV head, chunk of query tokens) whose rows are the g = Hq/Hkv
//     query heads of each token, so one KV head's keys are read once for its whole group;
//   * a split-KV schedule that gives every CTA of a persistent grid the same number of key
//     blocks (a unit that straddles two CTAs becomes two or more splits);
//   * the merge map of the split units.
#include "plan.h"

#include <algorithm>
#include <cstring>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

namespace rae {
namespace {

int fail(std::string* err, int code, const std::string& msg) {
  if (err) *err = msg;
  return code;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
// The same for non-negative values that fit in 32 bits (a 32-bit division is several times
// cheaper than a 64-bit one in the plan's per-unit loops).
int32_t ceil_div32(int32_t a, int32_t b) {
  return int32_t((uint32_t(a) + uint32_t(b) - 1u) / uint32_t(b));
}
int64_t align4(int64_t w) { return (w + 3) & ~int64_t(3); }

struct Unit {
  int32_t req, kvh, nkvh, q0, qn, nkeys, rows;
  int32_t w;       // cost of one key block (the scheduler's unit; see tc_block_cost)
  int64_t group;   // units of one group read the same K/V (one request or span, one KV head)
};

// Cost of one 128-key block of a tensor-core unit, in 1/16 of a block step.  The kernel is
// bound by the hand-off between its MMA and softmax warps, not by tensor throughput: a block
// takes about as long with one 128-row query tile as with two (measured 1.05x for two full
// tiles against one), so a unit's cost follows its key blocks, not its rows.
constexpr int32_t kTcStep = 16;
constexpr int32_t kTcLptSlackPct = 15;
int32_t tc_block_cost(int32_t tiles) { return tiles > 1 ? kTcStep + 1 : kTcStep; }

struct Piece {
  int32_t unit, blk0, nblk, cta;
};

// Grid capacity (CTAs resident at once) of a kernel family: the decode kernel fits two CTAs
// per SM; a tcgen05 CTA takes most of an SM's shared memory, so one.
int32_t grid_for(const rae_config& cfg, int32_t kind) {
  if (kind == kKindDecodeSimt) return cfg.num_sms * 2;
  return cfg.num_sms;
}

// Upper bound of the image size for cfg (words): header, CTA pointers, tiles, merge rows
// and the request arrays, each 16-byte aligned.
int64_t max_merge_rows(const rae_config& cfg) {
  return std::min<int64_t>(cfg.max_partial_rows, int64_t(cfg.max_q_tokens) * cfg.num_qo_heads);
}

int64_t image_bound(const rae_config& cfg) {
  int64_t w = kHdrWords;
  w = align4(w + max_ctas_for(cfg) + 1);
  w = align4(w + int64_t(cfg.max_tiles) * 12);
  w = align4(w + cfg.max_batch + 1) + align4(cfg.max_batch + 1) + align4(cfg.max_batch + 1);
  w = align4(w + cfg.max_kv_pages);
  return w;
}

// The schedule of one plan, before it is packed into an image.
struct Schedule {
  int32_t kind = kKindNone;
  std::vector<int32_t> cta_ptr;
  std::vector<Tile> tiles;
  int64_t merge_rows = 0;    // output rows merged from split partials
  int64_t split_units = 0;   // units whose keys were split
};

// Packs a schedule and the request arrays into `image` (compact, offsets in the header).
int emit_image(const Schedule& sc, const int32_t* a, int64_t na, const int32_t* b, int64_t nb,
               const int32_t* c, int64_t nc, const int32_t* d, int64_t nd, int32_t* image,
               int64_t image_words, rae_plan* out, std::string* err) {
  int64_t w = kHdrWords;
  const int64_t o_cta = w;
  w = align4(w + int64_t(sc.cta_ptr.size()));
  const int64_t o_tiles = w;
  w = align4(w + int64_t(sc.tiles.size()) * 12);
  const int64_t o_a = w;
  w = align4(w + na);
  const int64_t o_b = w;
  w = align4(w + nb);
  const int64_t o_c = w;
  w = align4(w + nc);
  const int64_t o_d = w;
  w = align4(w + nd);
  if (w > image_words) return fail(err, RAE_ERR_CAPACITY, "plan image exceeds its slot");
  std::memset(image, 0, size_t(w) * sizeof(int32_t));
  if (!sc.cta_ptr.empty()) std::memcpy(image + o_cta, sc.cta_ptr.data(), sc.cta_ptr.size() * 4);
  if (!sc.tiles.empty()) std::memcpy(image + o_tiles, sc.tiles.data(), sc.tiles.size() * sizeof(Tile));
  if (na) std::memcpy(image + o_a, a, size_t(na) * 4);
  if (nb) std::memcpy(image + o_b, b, size_t(nb) * 4);
  if (nc) std::memcpy(image + o_c, c, size_t(nc) * 4);
  if (nd) std::memcpy(image + o_d, d, size_t(nd) * 4);
  image[kHdrMagic] = kPlanMagic;
  image[kHdrKind] = sc.kind;
  image[kHdrNumTiles] = int32_t(sc.tiles.size());
  image[kHdrNumCtas] = int32_t(sc.cta_ptr.empty() ? 0 : sc.cta_ptr.size() - 1);
  image[kHdrNumMerge] = int32_t(sc.merge_rows);
  image[kHdrSplitUnits] = int32_t(sc.split_units);
  image[kHdrOffCtaPtr] = int32_t(o_cta);
  image[kHdrOffTiles] = int32_t(o_tiles);
  image[kHdrOffA] = int32_t(o_a);
  image[kHdrOffB] = int32_t(o_b);
  image[kHdrOffC] = int32_t(o_c);
  image[kHdrOffD] = int32_t(o_d);
  out->kind = sc.kind;
  out->num_tiles = image[kHdrNumTiles];
  out->num_ctas = image[kHdrNumCtas];
  out->num_merge_rows = image[kHdrNumMerge];
  out->image_words = int32_t(w);
  out->off_cta_ptr = int32_t(o_cta);
  out->off_tiles = int32_t(o_tiles);
  out->off_merge = 0;
  out->off_a = int32_t(o_a);
  out->off_b = int32_t(o_b);
  out->off_c = int32_t(o_c);
  out->off_d = int32_t(o_d);
  return RAE_OK;
}

// Schedules units over the grid: tiles, CTA pointers and merge rows.
//   blk: keys per block; ovh: per-tile overhead in the units of Unit::w; g: query heads per
//   KV head.
//   lpt_factor: whole units are scheduled longest-first when every CTA's share is at least
//   lpt_factor times the largest unit; otherwise the balanced contiguous partition is used,
//   unless whole units (longest-first) leave the busiest CTA within lpt_slack_pct per cent of
//   the partition's (0: never).
int schedule(const rae_config& cfg, int32_t kind, const std::vector<Unit>& units, int32_t blk,
             int32_t ovh, int32_t g, int32_t lpt_factor, int32_t lpt_slack_pct, Schedule* sc,
             std::string* err) {
  const int32_t grid = grid_for(cfg, kind);
  const int64_t nu = int64_t(units.size());
  std::vector<int64_t> nb(nu), cost(nu);
  int64_t total = 0, maxc = 0;
  for (int64_t u = 0; u < nu; ++u) {
    nb[u] = ceil_div32(units[u].nkeys, blk);
    cost[u] = nb[u] * units[u].w + ovh;
    total += cost[u];
    maxc = std::max(maxc, cost[u]);
  }

  std::vector<Piece> pieces;
  std::vector<int32_t> npieces(nu, 0);
  int32_t num_ctas = 0;

  auto lpt = [&]() {
    // Whole units, each to the least-loaded CTA, in an order that keeps the units sharing
    // K/V together in time and still starts the big work first: groups by descending largest
    // unit, units within a group by descending cost.  Consecutive units go to different CTAs
    // that are free at about the same time, so the units of a group (its query chunks) run
    // side by side and read their common K/V blocks through L2 once.
    pieces.clear();
    std::fill(npieces.begin(), npieces.end(), 0);
    std::vector<int64_t> gmax(nu);
    {
      std::vector<std::pair<int64_t, int64_t>> gm;   // (group, largest unit cost)
      for (int64_t u = 0; u < nu; ++u) {
        if (gm.empty() || gm.back().first != units[u].group) gm.push_back({units[u].group, 0});
        gm.back().second = std::max(gm.back().second, cost[u]);
      }
      size_t gi = 0;
      for (int64_t u = 0; u < nu; ++u) {
        while (gm[gi].first != units[u].group) ++gi;
        gmax[u] = gm[gi].second;
      }
    }
    // (descending largest unit of the group, group, descending cost, index): the index makes
    // the order total, so a plain sort gives the stable order
    struct Key {
      int64_t gm, grp, c, u;
    };
    std::vector<Key> keys(nu);
    for (int64_t u = 0; u < nu; ++u) keys[u] = {-gmax[u], units[u].group, -cost[u], u};
    std::sort(keys.begin(), keys.end(), [](const Key& a, const Key& b) {
      if (a.gm != b.gm) return a.gm < b.gm;
      if (a.grp != b.grp) return a.grp < b.grp;
      if (a.c != b.c) return a.c < b.c;
      return a.u < b.u;
    });
    const int32_t ctas = int32_t(std::min<int64_t>(grid, nu));
    // Min-heap of (load, cta): each unit goes to the least-loaded CTA (lowest index on ties),
    // whose load then grows -- one sift-down per unit instead of a pop and a push.
    using Load = std::pair<int64_t, int32_t>;
    std::vector<Load> heap;
    heap.resize(static_cast<size_t>(ctas));
    for (int32_t c = 0; c < ctas; ++c) heap[size_t(c)] = {0, c};   // already a heap
    pieces.reserve(size_t(nu));
    for (const Key& k : keys) {
      const int64_t u = k.u;
      Load& top = heap[0];
      pieces.push_back({int32_t(u), 0, int32_t(nb[u]), top.second});
      npieces[u] = 1;
      top.first += cost[u];
      const Load moved = top;
      size_t i = 0;
      while (true) {
        const size_t l = 2 * i + 1, r = l + 1;
        size_t m = i;
        const Load* best = &moved;
        if (l < heap.size() && heap[l] < *best) { m = l; best = &heap[l]; }
        if (r < heap.size() && heap[r] < *best) { m = r; best = &heap[r]; }
        if (m == i) break;
        heap[i] = heap[m];
        i = m;
      }
      heap[i] = moved;
    }
    // group by CTA, keeping each CTA's pieces in assignment order (a stable counting sort)
    {
      std::vector<int64_t> start(size_t(ctas) + 1, 0);
      for (const Piece& pc : pieces) ++start[size_t(pc.cta) + 1];
      for (int32_t c = 0; c < ctas; ++c) start[size_t(c) + 1] += start[size_t(c)];
      std::vector<Piece> sorted(pieces.size());
      for (const Piece& pc : pieces) sorted[size_t(start[size_t(pc.cta)]++)] = pc;
      pieces.swap(sorted);
    }
    num_ctas = ctas;
  };

  // The largest CTA load of the current pieces (block costs plus the per-piece overhead).
  auto max_load = [&]() -> int64_t {
    std::vector<int64_t> load(size_t(std::max(num_ctas, 0)), 0);
    for (const Piece& pc : pieces) load[size_t(pc.cta)] += int64_t(pc.nblk) * units[size_t(pc.unit)].w + ovh;
    int64_t mx = 0;
    for (int64_t l : load) mx = std::max(mx, l);
    return mx;
  };

  // Greedy fill of CTAs with capacity q (block costs + overhead per piece), in unit order;
  // returns the CTAs used, and the pieces when `emit` is set.
  auto greedy = [&](int64_t q, bool emit) -> int64_t {
    int64_t c = 0, cap = q;
    bool used = false;
    for (int64_t u = 0; u < nu; ++u) {
      int64_t rb = nb[u], s = 0;
      do {
        if (used && cap <= ovh) {
          ++c;
          cap = q;
          used = false;
        }
        const int64_t w = units[u].w;
        // room >= 1; a 32-bit division where it fits (the binary search runs this innermost
        // loop a dozen times per plan)
        auto blocks_that_fit = [&]() -> int64_t {
          const int64_t room = cap - ovh;
          return w == 1 ? room
                 : room < (int64_t(1) << 32) ? int64_t(uint32_t(room) / uint32_t(w))
                                             : room / w;
        };
        int64_t fit = blocks_that_fit();
        if (fit == 0 && used) {
          // Not one block fits in what is left: start the next CTA rather than overfill
          // this one (a block can cost more than the per-piece overhead).
          ++c;
          cap = q;
          used = false;
          fit = blocks_that_fit();
        }
        // An empty CTA takes at least one block even when q is too small for it; the search
        // then finds that q needs too many CTAs.
        const int64_t take = std::min<int64_t>(rb, std::max<int64_t>(fit, 1));
        if (emit) {
          pieces.push_back({int32_t(u), int32_t(s), int32_t(take), int32_t(c)});
          npieces[u] += 1;
        }
        used = true;
        cap -= take * w + ovh;
        s += take;
        rb -= take;
      } while (rb > 0);
    }
    return c + 1;
  };

  auto contiguous = [&]() {
    // Every CTA takes an equal share of the blocks of all units laid end to end; a unit cut
    // by a CTA boundary becomes several splits, merged afterwards in split order.  The share
    // is the smallest capacity whose greedy fill needs no more CTAs than the grid holds.
    pieces.clear();
    std::fill(npieces.begin(), npieces.end(), 0);
    int64_t lo = std::max<int64_t>(ceil_div(total, grid), ovh + 1);
    // Bracket: a CTA's fill falls short of its capacity by less than one unit's cost, so the
    // even share plus the largest unit (and an overhead) almost always fits; double if not.
    int64_t hi = lo + maxc + ovh;
    while (greedy(hi, false) > grid) hi *= 2;
    while (lo < hi) {
      const int64_t mid = lo + (hi - lo) / 2;
      if (greedy(mid, false) <= grid) hi = mid; else lo = mid + 1;
    }
    num_ctas = int32_t(greedy(lo, true));
  };

  if (nu == 0) {
    num_ctas = 0;
  } else if (maxc * lpt_factor <= total / grid) {
    lpt();   // many small units: whole units balance well, no merge needed
  } else {
    contiguous();
    int64_t prow = 0;
    for (int64_t u = 0; u < nu; ++u)
      if (npieces[u] > 1) prow += int64_t(npieces[u]) * units[u].rows;
    if (prow > cfg.max_partial_rows || prow > max_merge_rows(cfg)) {
      lpt();
    } else if (lpt_slack_pct > 0) {
      // Whole units win whenever their busiest CTA is within lpt_slack_pct of the split
      // schedule's: they need no partials or merges, and the units of a group run side by
      // side instead of one after another on one CTA (their K/V read once, through L2).
      const int64_t split_max = max_load();
      std::vector<Piece> split_pieces = pieces;
      std::vector<int32_t> split_np = npieces;
      const int32_t split_ctas = num_ctas;
      lpt();
      if (max_load() * 100 > split_max * (100 + lpt_slack_pct)) {
        pieces.swap(split_pieces);
        npieces.swap(split_np);
        num_ctas = split_ctas;
      }
    }
  }

  if (int64_t(pieces.size()) > cfg.max_tiles)
    return fail(err, RAE_ERR_CAPACITY,
                "plan needs " + std::to_string(pieces.size()) + " tiles > max_tiles " +
                    std::to_string(cfg.max_tiles));

  // Partial rows and arrival counters of the split units.
  std::vector<int64_t> part_base(nu, -1), munit(nu, -1);
  int64_t prow = 0, nmerge = 0, nsu = 0;
  for (int64_t u = 0; u < nu; ++u) {
    if (npieces[u] > 1) {
      part_base[u] = prow;
      munit[u] = nsu++;
      prow += int64_t(npieces[u]) * units[u].rows;
      nmerge += units[u].rows;
    }
  }
  if (prow > cfg.max_partial_rows || nmerge > max_merge_rows(cfg))
    return fail(err, RAE_ERR_CAPACITY, "split-KV partials exceed max_partial_rows");
  if (nsu > cfg.max_tiles) return fail(err, RAE_ERR_CAPACITY, "too many split units");

  sc->kind = kind;
  sc->cta_ptr.assign(size_t(num_ctas) + 1, 0);
  sc->tiles.resize(pieces.size());
  std::vector<int32_t> seen(nu, 0);
  int32_t cur = -1;
  for (size_t i = 0; i < pieces.size(); ++i) {
    const Piece& p = pieces[i];
    while (cur < p.cta) sc->cta_ptr[size_t(++cur)] = int32_t(i);
    const Unit& un = units[size_t(p.unit)];
    Tile t;
    t.req = un.req;
    t.kv_head = un.kvh;
    t.q0 = un.q0;
    t.qn = un.qn;
    t.kv0 = int32_t(std::min<int64_t>(int64_t(p.blk0) * blk, un.nkeys));
    t.kv1 = int32_t(std::min<int64_t>(int64_t(p.blk0 + p.nblk) * blk, un.nkeys));
    t.split = seen[size_t(p.unit)]++;
    t.part = part_base[size_t(p.unit)] < 0
                 ? -1
                 : int32_t(part_base[size_t(p.unit)] + int64_t(t.split) * un.rows);
    t.munit = int32_t(munit[size_t(p.unit)]);
    t.nsplit = npieces[size_t(p.unit)];
    t.nkvh = un.nkvh;
    t.pad1 = 0;
    sc->tiles[i] = t;
  }
  while (cur < num_ctas) sc->cta_ptr[size_t(++cur)] = int32_t(pieces.size());
  sc->merge_rows = nmerge;
  sc->split_units = nsu;
  return RAE_OK;
}

int check_indptr(const int32_t* a, int32_t n, const char* name, std::string* err) {
  if (!a) return fail(err, RAE_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (a[0] != 0) return fail(err, RAE_ERR_INVALID_ARG, std::string(name) + "[0] must be 0");
  for (int32_t i = 0; i < n; ++i)
    if (a[i + 1] < a[i])
      return fail(err, RAE_ERR_INVALID_ARG,
                  std::string(name) + " decreases at " + std::to_string(i));
  return RAE_OK;
}

}  // namespace

int check_config(const rae_config& cfg, std::string* err) {
  if (cfg.head_dim != 64 && cfg.head_dim != 128)
    return fail(err, RAE_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (cfg.page_size != 16 && cfg.page_size != 32 && cfg.page_size != 64)
    return fail(err, RAE_ERR_UNSUPPORTED, "page_size must be 16, 32 or 64");
  if (cfg.num_qo_heads <= 0 || cfg.num_kv_heads <= 0)
    return fail(err, RAE_ERR_INVALID_ARG, "head counts must be positive");
  if (cfg.num_qo_heads % cfg.num_kv_heads != 0)
    return fail(err, RAE_ERR_UNSUPPORTED, "num_qo_heads must be a multiple of num_kv_heads");
  if (cfg.num_qo_heads / cfg.num_kv_heads > kTcRows)
    return fail(err, RAE_ERR_UNSUPPORTED, "more than 128 query heads per KV head");
  if (cfg.max_batch < 1 || cfg.max_q_tokens < 1 || cfg.max_kv_pages < 1 || cfg.max_tiles < 1 ||
      cfg.max_partial_rows < 0)
    return fail(err, RAE_ERR_INVALID_ARG, "capacities must be positive");
  if (cfg.num_sms <= 0) return fail(err, RAE_ERR_INVALID_ARG, "num_sms must be positive");
  if (int64_t(cfg.max_q_tokens) * cfg.num_qo_heads >= (int64_t(1) << 31))
    return fail(err, RAE_ERR_CAPACITY, "max_q_tokens * num_qo_heads overflows int32");
  if (image_bound(cfg) >= (int64_t(1) << 31))
    return fail(err, RAE_ERR_CAPACITY, "plan image too large");
  return RAE_OK;
}

int32_t max_ctas_for(const rae_config& cfg) { return cfg.num_sms * 2; }

int64_t image_words_for(const rae_config& cfg) { return image_bound(cfg); }

int build_paged_plan(const rae_config& cfg, const int32_t* qo_indptr,
                     const int32_t* kv_page_indptr, const int32_t* kv_page_indices,
                     const int32_t* kv_len, int32_t batch, int32_t num_pages, int32_t* image,
                     int64_t image_words, rae_plan* out, std::string* err, bool causal) {
  int rc = check_config(cfg, err);
  if (rc) return rc;
  if (!image) return fail(err, RAE_ERR_INVALID_ARG, "image is NULL");
  if (!out) return fail(err, RAE_ERR_INVALID_ARG, "out is NULL");
  if (batch < 0) return fail(err, RAE_ERR_INVALID_ARG, "batch < 0");
  if (batch > cfg.max_batch) return fail(err, RAE_ERR_CAPACITY, "batch > max_batch");
  if ((rc = check_indptr(qo_indptr, batch, "qo_indptr", err))) return rc;
  if ((rc = check_indptr(kv_page_indptr, batch, "kv_page_indptr", err))) return rc;
  if (batch > 0 && !kv_len) return fail(err, RAE_ERR_INVALID_ARG, "kv_len is NULL");
  const int32_t total_q = qo_indptr[batch];
  const int32_t nnz = kv_page_indptr[batch];
  if (total_q > cfg.max_q_tokens) return fail(err, RAE_ERR_CAPACITY, "total queries > max_q_tokens");
  if (nnz > cfg.max_kv_pages) return fail(err, RAE_ERR_CAPACITY, "page entries > max_kv_pages");
  if (nnz > 0 && !kv_page_indices) return fail(err, RAE_ERR_INVALID_ARG, "kv_page_indices is NULL");
  if (num_pages < 0) return fail(err, RAE_ERR_INVALID_ARG, "num_pages < 0");
  if (int64_t(num_pages) * cfg.num_kv_heads * cfg.page_size >= (int64_t(1) << 31))
    return fail(err, RAE_ERR_CAPACITY, "pool rows overflow int32");
  int32_t page_extent = 0;   // 1 + the largest page id listed: the pool a run must hold
  for (int32_t i = 0; i < nnz; ++i) {
    if (kv_page_indices[i] < 0 || kv_page_indices[i] >= num_pages)
      return fail(err, RAE_ERR_INVALID_ARG,
                  "page id " + std::to_string(kv_page_indices[i]) + " at " + std::to_string(i) +
                      " outside [0, num_pages)");
    page_extent = std::max(page_extent, kv_page_indices[i] + 1);
  }
  for (int32_t b = 0; b < batch; ++b) {
    if (kv_len[b] < 0) return fail(err, RAE_ERR_INVALID_ARG, "kv_len < 0");
    int64_t need = ceil_div(kv_len[b], cfg.page_size);
    if (kv_page_indptr[b + 1] - kv_page_indptr[b] < need)
      return fail(err, RAE_ERR_INVALID_ARG,
                  "request " + std::to_string(b) + " has fewer pages than kv_len needs");
    if (causal && qo_indptr[b + 1] - qo_indptr[b] > kv_len[b])
      return fail(err, RAE_ERR_INVALID_ARG,
                  "request " + std::to_string(b) + " has more queries than sequence tokens");
  }

  const int32_t g = cfg.num_qo_heads / cfg.num_kv_heads;
  int32_t max_qlen = 0;
  for (int32_t b = 0; b < batch; ++b) max_qlen = std::max(max_qlen, qo_indptr[b + 1] - qo_indptr[b]);
  // Kernel family by query rows per (request, KV head): a few rows on CUDA cores (HBM bound),
  // up to 64 rows (d = 128) with keys on the MMA's M side, otherwise 128-row query tiles.
  const int64_t max_rows = int64_t(max_qlen) * g;
  const bool simt = max_rows <= kSimtMaxRows;
  const int32_t swap_n = max_rows <= 32 ? 32 : 64;
  // (causal plans use the two families that apply a per-row key limit)
  const bool swap = !causal && !simt && cfg.head_dim == 128 && max_rows <= 64 && swap_n % g == 0;
  const int32_t kind = simt ? kKindDecodeSimt : (swap ? kKindTcPagedSwap : kKindTcPaged);
  // tcgen05 units hold up to two 128-row query tiles that share every K/V block.
  const int32_t tile_tok = kTcRows / g;
  const int32_t tok_per_unit =
      simt ? std::max(max_qlen, 1) : (swap ? swap_n / g : 2 * tile_tok);

  // A decode unit holds up to kSimtMaxHeads adjacent KV heads (one per consumer warp), so
  // that each 16-key chunk of a page is read as one run over those heads; the other kernels
  // take one KV head per unit.
  const int32_t hpu = simt ? kSimtMaxHeads : 1;
  std::vector<Unit> units;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t qlen = qo_indptr[b + 1] - qo_indptr[b];
    for (int32_t h = 0; h < cfg.num_kv_heads; h += hpu)
      for (int32_t t = 0; t < qlen; t += tok_per_unit) {
        Unit u;
        u.req = b;
        u.kvh = h;
        u.nkvh = std::min(hpu, cfg.num_kv_heads - h);
        u.q0 = qo_indptr[b] + t;
        u.qn = std::min(tok_per_unit, qlen - t);
        // causal: the unit's last query (local index t + qn - 1) sees kv_len - qlen + t + qn
        // keys; no row of the unit sees more
        u.nkeys = causal ? kv_len[b] - qlen + t + u.qn : kv_len[b];
        u.rows = u.qn * g * u.nkvh;
        // decode: a block's bytes grow with the unit's heads
        u.w = simt ? u.nkvh : swap ? 1 : tc_block_cost(ceil_div32(u.qn, tile_tok));
        u.group = int64_t(b) * cfg.num_kv_heads + h;
        units.push_back(u);
      }
  }

  out->batch = batch;
  out->total_q = total_q;
  out->block_size = causal ? 1 : 0;
  out->kv_extent = page_extent;
  // rows per unit and KV head: what the kernel is instantiated for
  int32_t rows_max = 0;
  for (const Unit& u : units) rows_max = std::max(rows_max, u.rows / u.nkvh);
  if (swap) rows_max = swap_n;   // the row count the swapped kernel is instantiated for
  out->rows_max = rows_max;
  Schedule sc;
  // The decode kernel is HBM bound and short: an even split of the bytes over the grid
  // matters more than the small merge it costs.
  // The tensor-core kernel prefers whole units within 15 % of the split schedule's balance
  // (measured on the packed multi-token and causal chunked-prefill workloads: 20 % faster
  // calls with busiest CTAs 6 % and 2 % above the split schedule's).
  rc = simt ? schedule(cfg, kind, units, kSimtChunkKeys, 2, g, 64, 0, &sc, err)
       : swap ? schedule(cfg, kind, units, kTcBlockKeys, 1, g, 4, 0, &sc, err)
              : schedule(cfg, kind, units, kTcBlockKeys, kTcStep, g, 4, kTcLptSlackPct, &sc, err);
  if (rc) return rc;
  rc = emit_image(sc, qo_indptr, batch + 1, kv_len, batch, kv_page_indptr, batch + 1,
                  kv_page_indices, nnz, image, image_words, out, err);
  if (rc) return rc;
  image[kHdrBatch] = batch;
  image[kHdrTotalQ] = total_q;
  image[kHdrBlockSize] = causal ? 1 : 0;   // paged: 1 = causal, queries at the sequence end
  image[kHdrRowsMax] = rows_max;
  return RAE_OK;
}

int build_ragged_plan(const rae_config& cfg, const int32_t* cu_q, const int32_t* cu_kv,
                      int32_t num_spans, int32_t block_size, int32_t* image, int64_t image_words,
                      rae_plan* out, std::string* err) {
  int rc = check_config(cfg, err);
  if (rc) return rc;
  if (!image) return fail(err, RAE_ERR_INVALID_ARG, "image is NULL");
  if (!out) return fail(err, RAE_ERR_INVALID_ARG, "out is NULL");
  if (num_spans < 0) return fail(err, RAE_ERR_INVALID_ARG, "num_spans < 0");
  if (num_spans > cfg.max_batch) return fail(err, RAE_ERR_CAPACITY, "num_spans > max_batch");
  if (block_size < 0) return fail(err, RAE_ERR_INVALID_ARG, "block_size < 0");
  if ((rc = check_indptr(cu_q, num_spans, "cu_seqlens_q", err))) return rc;
  const int32_t* kv = cu_kv ? cu_kv : cu_q;
  if (cu_kv && (rc = check_indptr(cu_kv, num_spans, "cu_seqlens_kv", err))) return rc;
  const int32_t total_q = cu_q[num_spans];
  if (total_q > cfg.max_q_tokens) return fail(err, RAE_ERR_CAPACITY, "total queries > max_q_tokens");

  const int32_t g = cfg.num_qo_heads / cfg.num_kv_heads;
  const int32_t tile_tok = kTcRows / g;
  const int32_t tok_per_unit = 2 * tile_tok;   // two 128-row query tiles per unit
  std::vector<Unit> units;
  units.reserve(size_t(num_spans) * size_t(cfg.num_kv_heads) * 4);
  for (int32_t s = 0; s < num_spans; ++s) {
    const int32_t lq = cu_q[s + 1] - cu_q[s];
    const int32_t lk = kv[s + 1] - kv[s];
    for (int32_t h = 0; h < cfg.num_kv_heads; ++h)
      for (int32_t t = 0; t < lq; t += tok_per_unit) {
        Unit u;
        u.req = s;
        u.kvh = h;
        u.nkvh = 1;
        u.q0 = cu_q[s] + t;
        u.qn = std::min(tok_per_unit, lq - t);
        int64_t lim = lk;
        if (block_size > 0) {
          const int32_t last = t + u.qn - 1;  // local position of the chunk's last token
          lim = std::min<int64_t>(lk, int64_t(uint32_t(last) / uint32_t(block_size) + 1u) * block_size);
        }
        u.nkeys = int32_t(lim);
        u.rows = u.qn * g;
        u.w = tc_block_cost(ceil_div32(u.qn, tile_tok));
        u.group = int64_t(s) * cfg.num_kv_heads + h;
        units.push_back(u);
      }
  }
  out->batch = num_spans;
  out->total_q = total_q;
  out->block_size = block_size;
  out->kv_extent = kv[num_spans];
  out->rows_max = 0;
  for (const Unit& u : units) out->rows_max = std::max(out->rows_max, u.rows);
  Schedule sc;
  rc = schedule(cfg, kKindTcRagged, units, kTcBlockKeys, kTcStep, g, 4, kTcLptSlackPct, &sc, err);
  if (rc) return rc;
  rc = emit_image(sc, cu_q, num_spans + 1, kv, num_spans + 1, nullptr, 0, nullptr, 0, image,
                  image_words, out, err);
  if (rc) return rc;
  image[kHdrBatch] = num_spans;
  image[kHdrTotalQ] = total_q;
  image[kHdrBlockSize] = block_size;
  image[kHdrRowsMax] = out->rows_max;
  return RAE_OK;
}

int build_write_items(const rae_config& cfg, const int32_t* cu_enc, const int32_t* page_indptr,
                      const int32_t* page_indices, const int32_t* start, int32_t batch,
                      int32_t num_pages, WriteItem* items, int64_t max_items, int64_t* num_items,
                      std::string* err) {
  int rc = check_config(cfg, err);
  if (rc) return rc;
  if (batch < 0) return fail(err, RAE_ERR_INVALID_ARG, "batch < 0");
  if (batch > cfg.max_batch) return fail(err, RAE_ERR_CAPACITY, "batch > max_batch");
  if ((rc = check_indptr(cu_enc, batch, "cu_enc", err))) return rc;
  if ((rc = check_indptr(page_indptr, batch, "page_indptr", err))) return rc;
  const int32_t nnz = page_indptr[batch];
  if (nnz > 0 && !page_indices) return fail(err, RAE_ERR_INVALID_ARG, "page_indices is NULL");
  if (num_pages < 0) return fail(err, RAE_ERR_INVALID_ARG, "num_pages < 0");
  if (int64_t(num_pages) * cfg.num_kv_heads * cfg.page_size >= (int64_t(1) << 31))
    return fail(err, RAE_ERR_CAPACITY, "pool rows overflow int32");
  std::vector<uint8_t> used(size_t(num_pages), 0);
  int64_t n = 0;
  const int32_t P = cfg.page_size;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t len = cu_enc[b + 1] - cu_enc[b];
    const int32_t pos0 = start ? start[b] : 0;
    if (pos0 < 0) return fail(err, RAE_ERR_INVALID_ARG, "first position < 0");
    if (len == 0) continue;
    const int64_t end = int64_t(pos0) + len;
    if (page_indptr[b + 1] - page_indptr[b] < ceil_div(end, P))
      return fail(err, RAE_ERR_INVALID_ARG,
                  "request " + std::to_string(b) + " has fewer pages than its tokens need");
    for (int64_t pos = pos0; pos < end;) {
      const int64_t lp = pos / P;
      const int32_t page = page_indices[page_indptr[b] + lp];
      if (page < 0 || page >= num_pages)
        return fail(err, RAE_ERR_INVALID_ARG, "page id " + std::to_string(page) + " out of range");
      if (used[size_t(page)])
        return fail(err, RAE_ERR_INVALID_ARG,
                    "page id " + std::to_string(page) + " written twice in one call");
      used[size_t(page)] = 1;
      if (n >= max_items) return fail(err, RAE_ERR_CAPACITY, "write needs more pages than max_kv_pages");
      WriteItem& it = items[n++];
      it.slot0 = int32_t(pos - lp * P);
      it.ntok = int32_t(std::min<int64_t>(P - it.slot0, end - pos));
      it.src_row = cu_enc[b] + int32_t(pos - pos0);
      it.page = page;
      pos += it.ntok;
    }
  }
  *num_items = n;
  return RAE_OK;
}

}  // namespace rae
