// Host planner: validation, work items with realized cost, LPT / static
// placement, and the work lists the kernels read.
//
// Sources: "Split-KV: Breaking the Context Parallelism Bottleneck in
// Diffusion Drafter Training", section "LPT Scheduling: Load Balancing with
// Real Attention Costs" (cost of each KV block = attention it actually incurs;
// longest first onto the least-loaded rank; the token-count split it
// replaces) and "Split-KV: Efficient Context Parallelism for Training
// Diffusion Drafters", Abstract (LPT over context K/V chunks by realized
// attention cost, planned every step).
//
// Cost of an item (b, c, g, s) with relative key range [lo, hi):
//   G * block_q * sum_j |[lo, hi) ∩ [0, a_j)|
// computed from the sample's sorted anchors and their prefix sums in
// O(log A) per item.
#include <algorithm>
#include <cstring>
#include <iterator>
#include <functional>
#include <numeric>
#include <queue>
#include <vector>

#include "plan_layout.h"

namespace skv {
namespace {

struct Prob {
  int B, Hq, Hkv, d, S, C, sub, P, G, TT;
  int64_t Nq, Ltot;
  const int64_t* ctx;
  const int32_t* aoff;
  const int64_t* anchors;
  const uint8_t* mask;  // block-sparse mask [A][mask_stride], or nullptr
  int mask_stride;
  int mask_words;       // words per (tile, block): ceil(TT / 32)
};

int validate(const skv_problem* p, Prob& q) {
  if (!p || p->num_samples < 1 || !p->ctx_offsets || !p->anchor_offsets) return SKV_EINVAL;
  q.B = p->num_samples;
  q.Hq = p->num_q_heads;
  q.Hkv = p->num_kv_heads;
  q.d = p->head_dim;
  q.S = p->block_q;
  q.C = p->chunk_kv;
  q.sub = p->sub_chunks;
  q.P = p->num_partitions;
  q.ctx = p->ctx_offsets;
  q.aoff = p->anchor_offsets;
  q.anchors = p->anchors;
  if (q.S < 1 || q.C < 1 || q.sub < 1 || q.P < 1 || q.Hq < 1 || q.Hkv < 1) return SKV_EINVAL;
  if (q.C % q.sub != 0 || q.Hq % q.Hkv != 0) return SKV_EINVAL;
  if (q.ctx[0] != 0 || q.aoff[0] != 0) return SKV_EINVAL;
  for (int b = 0; b < q.B; ++b) {
    if (q.ctx[b + 1] <= q.ctx[b]) return SKV_EINVAL;
    if (q.aoff[b + 1] < q.aoff[b]) return SKV_EINVAL;
  }
  const int64_t A = q.aoff[q.B];
  if (A > 0 && !q.anchors) return SKV_EINVAL;
  for (int b = 0; b < q.B; ++b) {
    const int64_t L = q.ctx[b + 1] - q.ctx[b];
    for (int32_t j = q.aoff[b]; j < q.aoff[b + 1]; ++j)
      if (q.anchors[j] < 1 || q.anchors[j] > L) return SKV_EINVAL;
  }
  q.mask = p->key_block_mask;
  q.mask_stride = p->mask_stride;
  if (q.mask) {
    if (q.mask_stride < 1) return SKV_EINVAL;
    for (int b = 0; b < q.B; ++b)
      if ((q.ctx[b + 1] - q.ctx[b] + kTileN - 1) / kTileN > q.mask_stride) return SKV_EINVAL;
  }
  q.G = q.Hq / q.Hkv;
  if (q.d != 64 && q.d != 128) return SKV_EUNSUPPORTED;
  if (q.G > kTileM || kTileM % q.G != 0) return SKV_EUNSUPPORTED;
  q.TT = kTileM / q.G;
  q.mask_words = (q.TT + 31) / 32;
  q.Nq = A * q.S;
  q.Ltot = q.ctx[q.B];
  // 32-bit indices on the device: keys and query tokens (with tile slack).
  if (q.Ltot > (int64_t(1) << 31) - 4 * kTileN) return SKV_EUNSUPPORTED;
  if (q.Nq > (int64_t(1) << 31) - 4 * kTileM) return SKV_EUNSUPPORTED;
  if (q.P > (1 << 20)) return SKV_EUNSUPPORTED;
  return SKV_OK;
}

struct SampleAnchors {
  std::vector<int64_t> a;       // sorted
  std::vector<int64_t> prefix;  // prefix[i] = a[0] + ... + a[i-1]
  int64_t max_a = 0;
  // block-sparse mask: allowed (token-of-anchor, key) pairs per anchor summed over the sample's 128-key
  // blocks before block kb (block_prefix[kb]); a key of block kb counts for anchor j when the mask allows
  // the block and the key lies before a_j
  std::vector<int64_t> block_prefix;
  // executed-tile cost (SKV_PLAN_LPT_TILES): the largest anchor of every query tile of the sample, sorted;
  // under a block mask, per 128-key block the number of query tiles with a token that attends it
  std::vector<int64_t> tile_kmax_sorted;
  std::vector<int32_t> live_tiles_of_block;
};

// sum_j max(0, min(hi, a_j) - lo), relative coordinates, lo < hi.
int64_t pair_sum(const SampleAnchors& s, int64_t lo, int64_t hi) {
  const auto& a = s.a;
  const size_t i0 = std::upper_bound(a.begin(), a.end(), lo) - a.begin();  // first a > lo
  const size_t i1 = std::lower_bound(a.begin(), a.end(), hi) - a.begin();  // first a >= hi
  int64_t mid = 0;
  if (i1 > i0) mid = (s.prefix[i1] - s.prefix[i0]) - static_cast<int64_t>(i1 - i0) * lo;
  const int64_t top = static_cast<int64_t>(a.size() - i1) * (hi - lo);
  return mid + top;
}

struct Built {
  std::vector<skv_item> items;
  std::vector<int64_t> load;
  std::vector<int32_t> placement;  // item ids in placement order
  std::vector<MTile> mtiles;
  std::vector<int32_t> sample_mt;  // [B+1]
  std::vector<int32_t> tok_kend;
  std::vector<FwdUnit> fwd;
  std::vector<int32_t> fwd_part_off;
  std::vector<FwdPair> pairs;
  std::vector<int32_t> pair_off;
  std::vector<int32_t> merge_off, merge_list;
  std::vector<BwdUnit> bwd;
  std::vector<int32_t> bwd_part_off;
  std::vector<int32_t> bwd_item, bwd_part;  // host-side: item and partition of every backward unit
  std::vector<uint32_t> tile_mask;           // block-sparse mask: per (tile, block) words of token bits
  std::vector<int32_t> pair_tile_off, unit_tile_off, live_tiles;
  std::vector<std::vector<int32_t>> unit_live;  // live key tiles of every forward unit (mask only)
  std::vector<int32_t> unit_tiles;              // scratch
  bool mask_aligned = true;                     // items line up with the mask's blocks (kernels can run)
  std::vector<int32_t> bwd_rank, bwd_det_order;
  std::vector<int64_t> dead;  // [2 n_dead]
  int shard = -1, n_queues = 1, kv_heads = 1;
  int64_t kv_rows = 0;
  int64_t total_cost = 0;
  double imbalance = 0.0;
};

void make_items(const Prob& q, int policy, const std::vector<SampleAnchors>& sa, Built& out) {
  // allowed (anchor, key) pairs of the keys [x, y) inside one 128-key block, counted anchor by anchor
  auto block_part = [&](int b, int64_t x, int64_t y) -> int64_t {
    if (y <= x) return 0;
    const int64_t kb = x / kTileN;
    int64_t n = 0;
    for (int32_t j = q.aoff[b]; j < q.aoff[b + 1]; ++j)
      if (q.mask[static_cast<size_t>(j) * q.mask_stride + kb]) n += std::max<int64_t>(0, std::min(y, q.anchors[j]) - x);
    return n;
  };
  auto cost = [&](int b, int64_t lo_abs, int64_t hi_abs) {
    if (policy == SKV_PLAN_LPT_TILES) {
      // 128 x 128 per (query tile, key tile) block in which some token attends some key
      int64_t blocks = 0;
      for (int64_t kb = lo_abs - q.ctx[b]; kb < hi_abs - q.ctx[b]; kb += kTileN) {
        if (q.mask) {
          blocks += sa[b].live_tiles_of_block[kb / kTileN];
        } else {
          const auto& km = sa[b].tile_kmax_sorted;
          blocks += km.end() - std::upper_bound(km.begin(), km.end(), kb);  // tiles whose largest anchor > kb
        }
      }
      return blocks * kTileM * kTileN;
    }
    if (q.mask) {
      // whole blocks from the per-block prefix sums, the partial blocks at either end anchor by anchor
      const int64_t lo = lo_abs - q.ctx[b], hi = hi_abs - q.ctx[b];
      const int64_t f0 = (lo + kTileN - 1) / kTileN, f1 = hi / kTileN;
      int64_t n;
      if (f0 <= f1)
        n = sa[b].block_prefix[f1] - sa[b].block_prefix[f0] + block_part(b, lo, f0 * kTileN) + block_part(b, f1 * kTileN, hi);
      else
        n = block_part(b, lo, hi);  // inside one block
      return static_cast<int64_t>(q.G) * q.S * n;
    }
    return static_cast<int64_t>(q.G) * q.S * pair_sum(sa[b], lo_abs - q.ctx[b], hi_abs - q.ctx[b]);
  };
  out.items.clear();
  if (policy == SKV_PLAN_LPT || policy == SKV_PLAN_LPT_TILES) {
    const int64_t cs = q.C / q.sub;
    for (int b = 0; b < q.B; ++b) {
      const int64_t k0 = q.ctx[b], L = q.ctx[b + 1] - k0;
      const int64_t nc = (L + q.C - 1) / q.C;
      for (int64_t c = 0; c < nc; ++c) {
        const int64_t c_end = std::min<int64_t>((c + 1) * q.C, L);
        for (int g = 0; g < q.Hkv; ++g)
          for (int s = 0; s < q.sub; ++s) {
            const int64_t lo = c * q.C + s * cs, hi = std::min<int64_t>(c * q.C + (s + 1) * cs, c_end);
            if (hi <= lo) continue;
            skv_item it{};
            it.b = b;
            it.c = static_cast<int32_t>(c);
            it.g = g;
            it.sub = s;
            it.key_begin = k0 + lo;
            it.key_end = k0 + hi;
            it.cost = cost(b, k0 + lo, k0 + hi);
            it.partition = -1;
            it.order = -1;
            out.items.push_back(it);
          }
      }
    }
  } else {
    // Pieces of the equal-token split cut at chunk boundaries, in stream order.
    struct Piece { int b; int64_t c, lo, hi; int p, s; };
    std::vector<Piece> pieces;
    const int64_t T = q.Ltot;
    int b = 0;
    for (int p = 0; p < q.P; ++p) {
      const int64_t t0 = (static_cast<int64_t>(p) * T) / q.P, t1 = (static_cast<int64_t>(p + 1) * T) / q.P;
      if (t1 <= t0) continue;
      while (b < q.B && q.ctx[b + 1] <= t0) ++b;
      for (int bb = b; bb < q.B && q.ctx[bb] < t1; ++bb) {
        const int64_t k0 = q.ctx[bb], k1 = q.ctx[bb + 1];
        const int64_t lo_rel = std::max(t0, k0) - k0, hi_rel = std::min(t1, k1) - k0;
        for (int64_t c = lo_rel / q.C; c * q.C < hi_rel; ++c) {
          const int64_t lo = std::max(t0, k0 + c * q.C), hi = std::min({t1, k0 + (c + 1) * q.C, k1});
          if (hi > lo) pieces.push_back({bb, c, lo, hi, p, 0});
        }
      }
    }
    for (size_t i = 0; i < pieces.size(); ++i)
      if (i > 0 && pieces[i - 1].b == pieces[i].b && pieces[i - 1].c == pieces[i].c)
        pieces[i].s = pieces[i - 1].s + 1;
    size_t i = 0;
    while (i < pieces.size()) {
      size_t e = i;
      while (e < pieces.size() && pieces[e].b == pieces[i].b && pieces[e].c == pieces[i].c) ++e;
      for (int g = 0; g < q.Hkv; ++g)
        for (size_t k = i; k < e; ++k) {
          const Piece& pc = pieces[k];
          skv_item it{};
          it.b = pc.b;
          it.c = static_cast<int32_t>(pc.c);
          it.g = g;
          it.sub = pc.s;
          it.key_begin = pc.lo;
          it.key_end = pc.hi;
          it.cost = cost(pc.b, pc.lo, pc.hi);
          it.partition = pc.p;
          it.order = -1;
          out.items.push_back(it);
        }
      i = e;
    }
  }
}

void place(const Prob& q, int policy, Built& out) {
  const size_t n = out.items.size();
  out.placement.resize(n);
  std::iota(out.placement.begin(), out.placement.end(), 0);
  out.load.assign(q.P, 0);
  if (policy == SKV_PLAN_LPT || policy == SKV_PLAN_LPT_TILES) {
    // Items are generated in (b, c, g, s) order, so the index breaks ties.
    std::sort(out.placement.begin(), out.placement.end(), [&](int32_t x, int32_t y) {
      if (out.items[x].cost != out.items[y].cost) return out.items[x].cost > out.items[y].cost;
      return x < y;
    });
    using Slot = std::pair<int64_t, int32_t>;  // (load, partition): smallest first
    std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
    for (int32_t p = 0; p < q.P; ++p) heap.push({0, p});
    for (size_t r = 0; r < n; ++r) {
      skv_item& it = out.items[out.placement[r]];
      Slot s = heap.top();
      heap.pop();
      it.partition = s.second;
      it.order = static_cast<int32_t>(r);
      s.first += it.cost;
      heap.push(s);
    }
  } else {
    for (size_t r = 0; r < n; ++r) out.items[r].order = static_cast<int32_t>(r);
  }
  out.total_cost = 0;
  for (const auto& it : out.items) {
    out.load[it.partition] += it.cost;
    out.total_cost += it.cost;
  }
  const int64_t mx = *std::max_element(out.load.begin(), out.load.end());
  out.imbalance = out.total_cost > 0 ? static_cast<double>(mx) * q.P / static_cast<double>(out.total_cost) - 1.0 : 0.0;
}

// shard < 0: the full plan: one work queue holding every item in placement
// order (`one_queue`), or every partition's items on its own queue; the
// K/V buffers are the packed context, all kv heads per row. shard = p: the
// items of partition p only, on one work queue; the K/V buffers hold those
// items' keys, one kv head per row, items in (b, c, g, s) order (the layout a
// context-parallel rank keeps of its own chunks).
void make_lists(const Prob& q, const std::vector<SampleAnchors>& sa, int shard, bool one_queue, Built& out) {
  // query tiles
  out.mtiles.clear();
  out.sample_mt.assign(q.B + 1, 0);
  out.tok_kend.assign(static_cast<size_t>(q.Nq), 0);
  for (int b = 0; b < q.B; ++b) {
    out.sample_mt[b] = static_cast<int32_t>(out.mtiles.size());
    const int64_t t_begin = static_cast<int64_t>(q.aoff[b]) * q.S, t_end = static_cast<int64_t>(q.aoff[b + 1]) * q.S;
    for (int64_t t = t_begin; t < t_end; ++t)
      out.tok_kend[t] = static_cast<int32_t>(q.ctx[b] + q.anchors[t / q.S]);
    for (int64_t t0 = t_begin; t0 < t_end; t0 += q.TT) {
      const int64_t nt = std::min<int64_t>(q.TT, t_end - t0);
      int64_t amax = 0;
      for (int64_t j = t0 / q.S; j <= (t0 + nt - 1) / q.S; ++j) amax = std::max(amax, q.anchors[j]);
      MTile M{};
      M.b = b;
      M.tok0 = static_cast<int32_t>(t0);
      M.ntok = static_cast<int32_t>(nt);
      M.kmax = static_cast<int32_t>(q.ctx[b] + amax);
      M.kbase = static_cast<int32_t>(q.ctx[b]);
      out.mtiles.push_back(M);
    }
  }
  out.sample_mt[q.B] = static_cast<int32_t>(out.mtiles.size());

  // block-sparse mask: per (tile, block) the tile's tokens that attend keys of the block
  out.tile_mask.clear();
  if (q.mask) {
    int64_t entries = 0;
    for (auto& M : out.mtiles) {
      M.mbase = static_cast<int32_t>(entries);
      entries += (q.ctx[M.b + 1] - q.ctx[M.b] + kTileN - 1) / kTileN;
    }
    out.tile_mask.assign(static_cast<size_t>(entries) * q.mask_words, 0u);
    for (const auto& M : out.mtiles) {
      const int64_t nkb = (q.ctx[M.b + 1] - q.ctx[M.b] + kTileN - 1) / kTileN;
      for (int t = 0; t < M.ntok; ++t) {
        const int64_t j = (M.tok0 + t) / q.S;
        const uint8_t* row = q.mask + static_cast<size_t>(j) * q.mask_stride;
        const int64_t a = q.anchors[j];
        for (int64_t kb = 0; kb < nkb && kb * kTileN < a; ++kb)
          if (row[kb]) out.tile_mask[static_cast<size_t>(M.mbase + kb) * q.mask_words + t / 32] |= 1u << (t % 32);
      }
    }
  }
  // live blocks of tile mt among the sample-relative blocks [kb0, kb1)
  auto block_live = [&](int32_t mt, int64_t kb) -> bool {
    const uint32_t* w = out.tile_mask.data() + static_cast<size_t>(out.mtiles[mt].mbase + kb) * q.mask_words;
    for (int i = 0; i < q.mask_words; ++i)
      if (w[i]) return true;
    return false;
  };

  // K/V rows of every item, and the items each work queue runs in placement order
  const bool per_partition = shard < 0 && !one_queue;
  out.shard = shard;
  out.n_queues = per_partition ? q.P : 1;
  out.kv_heads = shard < 0 ? q.Hkv : 1;
  std::vector<char> in_plan(out.items.size(), shard < 0 ? 1 : 0);
  if (shard < 0) {
    for (auto& it : out.items) it.kv_row = it.key_begin;
    out.kv_rows = q.Ltot;
  } else {
    int64_t row = 0;
    for (size_t id = 0; id < out.items.size(); ++id) {
      skv_item& it = out.items[id];
      if (it.partition == shard) {
        in_plan[id] = 1;
        it.kv_row = row;
        row += it.key_end - it.key_begin;
      } else {
        it.kv_row = -1;
      }
    }
    out.kv_rows = row;
  }
  std::vector<std::vector<int32_t>> by_queue(out.n_queues);
  for (int32_t id : out.placement)
    if (in_plan[id]) by_queue[per_partition ? out.items[id].partition : 0].push_back(id);
  if (!per_partition && q.B > 1) {
    // One queue: samples in the order of their costliest item, each sample's items in placement order.
    // The CTAs then work on one or two samples at a time, so those samples' queries, output gradients and
    // dQ accumulator stay in L2 instead of every sample's at once.
    std::vector<int32_t> rank(q.B, -1);
    int32_t next = 0;
    for (int32_t id : by_queue[0])
      if (rank[out.items[id].b] < 0) rank[out.items[id].b] = next++;
    std::stable_sort(by_queue[0].begin(), by_queue[0].end(),
                     [&](int32_t x, int32_t y) { return rank[out.items[x].b] < rank[out.items[y].b]; });
  }

  out.fwd.clear();
  out.unit_live.clear();
  out.fwd_part_off.assign(out.n_queues + 1, 0);
  out.pairs.clear();
  out.pair_off.assign(out.n_queues + 1, 0);
  out.bwd.clear();
  out.bwd_item.clear();
  out.bwd_part.clear();
  out.bwd_part_off.assign(out.n_queues + 1, 0);
  std::vector<std::pair<int64_t, int32_t>> tiles;
  std::vector<std::pair<int32_t, int32_t>> item_fwd(out.items.size(), {0, 0});  // [first forward unit, count]
  std::vector<int64_t> item_cov_end(out.items.size(), 0);  // end of the keys the item's backward units cover
  for (int p = 0; p < out.n_queues; ++p) {
    out.fwd_part_off[p] = static_cast<int32_t>(out.fwd.size());
    out.pair_off[p] = static_cast<int32_t>(out.pairs.size());
    out.bwd_part_off[p] = static_cast<int32_t>(out.bwd.size());
    for (int32_t id : by_queue[p]) {
      const skv_item& it = out.items[id];
      const int32_t kshift = static_cast<int32_t>(it.key_begin - it.kv_row);
      const int32_t kvh = shard < 0 ? it.g : 0;
      // forward: live query tiles, longest key range first (ties by tile index). Tiles reaching past
      // the item's end all have its full range and come first in index order; only the others,
      // few per item, need sorting. With a block mask a tile is live when one of its tokens attends
      // a key of one of the item's blocks, and its extent is its count of live blocks.
      tiles.clear();
      size_t n_full = 0;
      const int64_t kb_lo = (it.key_begin - q.ctx[it.b]) / kTileN;
      const int64_t kb_hi = (it.key_end - q.ctx[it.b] + kTileN - 1) / kTileN;
      for (int32_t mt = out.sample_mt[it.b]; mt < out.sample_mt[it.b + 1]; ++mt) {
        const int64_t kmax = out.mtiles[mt].kmax;
        if (q.mask) {
          int64_t n_live = 0;
          for (int64_t kb = kb_lo; kb < kb_hi; ++kb) n_live += block_live(mt, kb);
          if (n_live > 0) tiles.push_back({-n_live, mt});
        } else if (kmax >= it.key_end) {
          tiles.insert(tiles.begin() + static_cast<std::ptrdiff_t>(n_full++), {-(it.key_end - it.key_begin), mt});
        } else if (kmax > it.key_begin) {
          tiles.push_back({-(kmax - it.key_begin), mt});
        }
      }
      std::sort(tiles.begin() + static_cast<std::ptrdiff_t>(n_full), tiles.end());
      item_fwd[id] = {static_cast<int32_t>(out.fwd.size()), static_cast<int32_t>(tiles.size())};
      for (size_t ti = 0; ti < tiles.size(); ++ti) {
        const auto& t = tiles[ti];
        FwdUnit u{};
        u.mt = t.second;
        u.g = it.g;
        u.kbeg = static_cast<int32_t>(it.key_begin);
        u.kend = static_cast<int32_t>(it.key_begin - t.first);
        u.item = id;
        u.part = it.partition;
        u.kshift = kshift;
        u.kvh = kvh;
        if (q.mask) {
          // the unit's live key tiles: from its first to its last live block
          out.unit_tiles.clear();
          for (int64_t kb = kb_lo; kb < kb_hi; ++kb)
            if (block_live(u.mt, kb)) out.unit_tiles.push_back(static_cast<int32_t>(q.ctx[it.b] + kb * kTileN));
          u.kbeg = out.unit_tiles.front();
          u.kend = static_cast<int32_t>(std::min<int64_t>(out.unit_tiles.back() + kTileN, it.key_end));
          out.unit_live.push_back(out.unit_tiles);
        }
        // consecutive tiles (similar key extents) share a pair; the first is the longer
        if (ti % 2 == 0) {
          FwdPair pr{};
          pr.slot[0] = static_cast<int32_t>(out.fwd.size());
          pr.slot[1] = -1;
          pr.kbeg = u.kbeg;
          pr.kend = u.kend;
          pr.part = it.partition;
          out.pairs.push_back(pr);
        } else {
          FwdPair& pr = out.pairs.back();
          pr.slot[1] = static_cast<int32_t>(out.fwd.size());
          pr.kbeg = std::min(pr.kbeg, u.kbeg);  // with a block mask the second tile may reach further
          pr.kend = std::max(pr.kend, u.kend);
        }
        out.fwd.push_back(u);
      }
      // backward: key tiles below the sample's largest anchor
      const int64_t kmax_b = q.ctx[it.b] + sa[it.b].max_a;
      // first query tile whose largest anchor reaches past the key tile start (later dead tiles,
      // possible with unsorted anchors, are skipped by the kernel); a tile dead for one key tile is
      // dead for every later one, so the index only moves forward
      int32_t first = out.sample_mt[it.b];
      item_cov_end[id] = it.key_begin;
      for (int64_t kb = it.key_begin; kb < it.key_end && kb < kmax_b; kb += kTileN) {
        BwdUnit u{};
        u.b = it.b;
        u.g = it.g;
        u.kbeg = static_cast<int32_t>(kb);
        u.kend = static_cast<int32_t>(std::min<int64_t>(kb + kTileN, it.key_end));
        while (first < out.sample_mt[it.b + 1] && out.mtiles[first].kmax <= kb) ++first;
        u.mt_begin = first;
        u.mt_end = out.sample_mt[it.b + 1];
        u.kshift = kshift;
        u.kvh = kvh;
        item_cov_end[id] = u.kend;
        out.bwd.push_back(u);
        out.bwd_item.push_back(id);
        out.bwd_part.push_back(it.partition);
      }
    }
  }
  out.fwd_part_off[out.n_queues] = static_cast<int32_t>(out.fwd.size());
  out.pair_off[out.n_queues] = static_cast<int32_t>(out.pairs.size());
  out.bwd_part_off[out.n_queues] = static_cast<int32_t>(out.bwd.size());

  // block-sparse mask: the live key tiles of every forward pair (union of its two units', ascending)
  // and of every forward unit, as first keys; pairs' lists first, then units'
  out.pair_tile_off.clear();
  out.unit_tile_off.clear();
  out.live_tiles.clear();
  if (q.mask) {
    out.pair_tile_off.push_back(0);
    for (const auto& pr : out.pairs) {
      const auto& a = out.unit_live[pr.slot[0]];
      if (pr.slot[1] < 0) {
        out.live_tiles.insert(out.live_tiles.end(), a.begin(), a.end());
      } else {
        const auto& c = out.unit_live[pr.slot[1]];
        std::set_union(a.begin(), a.end(), c.begin(), c.end(), std::back_inserter(out.live_tiles));
      }
      out.pair_tile_off.push_back(static_cast<int32_t>(out.live_tiles.size()));
    }
    const int32_t base = static_cast<int32_t>(out.live_tiles.size());
    out.unit_tile_off.push_back(base);
    for (size_t u = 0; u < out.fwd.size(); ++u) {
      out.live_tiles.insert(out.live_tiles.end(), out.unit_live[u].begin(), out.unit_live[u].end());
      out.unit_tile_off.push_back(static_cast<int32_t>(out.live_tiles.size()));
    }
  }

  // Deterministic backward: the rank of every unit's key tile among the plan's key tiles of its (sample,
  // kv head) in ascending key order, and the dispatch order (sample, rank, kv head). Items of one (sample,
  // kv head) are numbered in ascending key order, so ranks run on from item to item. In a full plan every
  // kv head has the same key tiles, so (sample, rank, kv head) numbers the units densely; a shard's heads
  // differ, so its order is sorted.
  {
    std::vector<int32_t> first_rank(out.items.size(), 0);
    std::vector<int32_t> running(static_cast<size_t>(q.Hkv), 0);
    std::vector<int32_t> tiles_of_sample(q.B, 0);
    int b_prev = -1;
    for (size_t id = 0; id < out.items.size(); ++id) {
      const skv_item& it = out.items[id];
      if (it.b != b_prev) {
        std::fill(running.begin(), running.end(), 0);
        b_prev = it.b;
      }
      if (!in_plan[id]) continue;
      first_rank[id] = running[it.g];
      const int64_t kmax_b = q.ctx[it.b] + sa[it.b].max_a;
      const int64_t hi = std::min<int64_t>(it.key_end, kmax_b);
      const int32_t nt = hi > it.key_begin ? static_cast<int32_t>((hi - it.key_begin + kTileN - 1) / kTileN) : 0;
      running[it.g] += nt;
      tiles_of_sample[it.b] = std::max(tiles_of_sample[it.b], running[it.g]);
    }
    out.bwd_rank.assign(out.bwd.size(), 0);
    for (size_t u = 0; u < out.bwd.size(); ++u) {
      const skv_item& it = out.items[out.bwd_item[u]];
      out.bwd_rank[u] = first_rank[out.bwd_item[u]] + static_cast<int32_t>((out.bwd[u].kbeg - it.key_begin) / kTileN);
    }
    out.bwd_det_order.assign(out.bwd.size(), -1);
    if (shard < 0) {
      std::vector<int64_t> base(q.B + 1, 0);
      for (int b = 0; b < q.B; ++b) base[b + 1] = base[b] + static_cast<int64_t>(tiles_of_sample[b]) * q.Hkv;
      for (size_t u = 0; u < out.bwd.size(); ++u) {
        const int64_t pos = base[out.bwd[u].b] + static_cast<int64_t>(out.bwd_rank[u]) * q.Hkv + out.bwd[u].g;
        if (pos >= 0 && pos < static_cast<int64_t>(out.bwd.size())) out.bwd_det_order[pos] = static_cast<int32_t>(u);
      }
    } else {
      std::iota(out.bwd_det_order.begin(), out.bwd_det_order.end(), 0);
      std::sort(out.bwd_det_order.begin(), out.bwd_det_order.end(), [&](int32_t x, int32_t y) {
        const BwdUnit &a = out.bwd[x], &c = out.bwd[y];
        if (a.b != c.b) return a.b < c.b;
        if (out.bwd_rank[x] != out.bwd_rank[y]) return out.bwd_rank[x] < out.bwd_rank[y];
        return a.g < c.g;
      });
    }
  }

  // merge lists: per (query tile, kv head), forward units in ascending key order
  const size_t nslots = out.mtiles.size() * static_cast<size_t>(q.Hkv);
  out.merge_off.assign(nslots + 1, 0);
  for (const auto& u : out.fwd) out.merge_off[static_cast<size_t>(u.mt) * q.Hkv + u.g + 1]++;
  for (size_t i = 0; i < nslots; ++i) out.merge_off[i + 1] += out.merge_off[i];
  out.merge_list.assign(out.fwd.size(), 0);
  std::vector<int32_t> fill(out.merge_off.begin(), out.merge_off.end() - 1);
  // Items are in (b, c, g, s) order: walking them fills every (tile, kv head) slot in ascending key
  // order (an item has at most one unit per tile, and its key range starts after the previous item's).
  for (size_t id = 0; id < out.items.size(); ++id)
    for (int32_t i = item_fwd[id].first; i < item_fwd[id].first + item_fwd[id].second; ++i) {
      const auto& u = out.fwd[i];
      out.merge_list[fill[static_cast<size_t>(u.mt) * q.Hkv + u.g]++] = i;
    }

  // K/V rows whose gradients are zero (no query attends to them): in a full plan the keys of every
  // sample past its last backward tile; in a shard, the rows of each item past its last backward tile
  out.dead.clear();
  if (shard < 0) {
    std::vector<int64_t> live_end(q.B);
    for (int b = 0; b < q.B; ++b) live_end[b] = q.ctx[b];
    for (const auto& u : out.bwd) live_end[u.b] = std::max<int64_t>(live_end[u.b], u.kend);
    for (int b = 0; b < q.B; ++b) {
      out.dead.push_back(live_end[b]);
      out.dead.push_back(q.ctx[b + 1]);
    }
  } else {
    for (size_t id = 0; id < out.items.size(); ++id) {
      if (!in_plan[id]) continue;
      const skv_item& it = out.items[id];
      if (item_cov_end[id] >= it.key_end) continue;
      const int64_t lo = item_cov_end[id] - (it.key_begin - it.kv_row), hi = it.kv_row + (it.key_end - it.key_begin);
      if (!out.dead.empty() && out.dead.back() == lo)
        out.dead.back() = hi;  // adjacent rows: one range
      else {
        out.dead.push_back(lo);
        out.dead.push_back(hi);
      }
    }
  }
}

int build(const skv_problem* prob, int policy, Built& out, Prob& q, int shard = -1) {
  const bool one_queue = (policy & SKV_PLAN_PARTITION_QUEUES) == 0;
  policy &= ~(SKV_PLAN_PARTIALS_BF16 | SKV_PLAN_PARTITION_QUEUES);
  if (policy != SKV_PLAN_LPT && policy != SKV_PLAN_STATIC && policy != SKV_PLAN_LPT_TILES) return SKV_EINVAL;
  int rc = validate(prob, q);
  if (rc != SKV_OK) return rc;
  std::vector<SampleAnchors> sa(q.B);
  for (int b = 0; b < q.B; ++b) {
    sa[b].a.assign(q.anchors + q.aoff[b], q.anchors + q.aoff[b + 1]);
    std::sort(sa[b].a.begin(), sa[b].a.end());
    sa[b].prefix.assign(sa[b].a.size() + 1, 0);
    for (size_t i = 0; i < sa[b].a.size(); ++i) sa[b].prefix[i + 1] = sa[b].prefix[i] + sa[b].a[i];
    sa[b].max_a = sa[b].a.empty() ? 0 : sa[b].a.back();
  }
  if (shard >= q.P) return SKV_EINVAL;
  if (q.mask) {
    for (int b = 0; b < q.B; ++b) {
      const int64_t nkb = (q.ctx[b + 1] - q.ctx[b] + kTileN - 1) / kTileN;
      std::vector<int64_t>& bp = sa[b].block_prefix;
      bp.assign(nkb + 1, 0);
      for (int32_t j = q.aoff[b]; j < q.aoff[b + 1]; ++j) {
        const uint8_t* row = q.mask + static_cast<size_t>(j) * q.mask_stride;
        const int64_t a = q.anchors[j];
        for (int64_t kb = 0; kb < nkb && kb * kTileN < a; ++kb)
          if (row[kb]) bp[kb + 1] += std::min<int64_t>(a, (kb + 1) * kTileN) - kb * kTileN;
      }
      for (int64_t kb = 0; kb < nkb; ++kb) bp[kb + 1] += bp[kb];
    }
  }
  if (policy == SKV_PLAN_LPT_TILES) {
    if (q.mask && (q.C % kTileN != 0 || (q.C / q.sub) % kTileN != 0)) return SKV_EUNSUPPORTED;
    for (int b = 0; b < q.B; ++b) {
      const int64_t t_begin = static_cast<int64_t>(q.aoff[b]) * q.S, t_end = static_cast<int64_t>(q.aoff[b + 1]) * q.S;
      const int64_t nkb = (q.ctx[b + 1] - q.ctx[b] + kTileN - 1) / kTileN;
      auto& km = sa[b].tile_kmax_sorted;
      km.clear();
      sa[b].live_tiles_of_block.assign(q.mask ? nkb : 0, 0);
      for (int64_t t0 = t_begin; t0 < t_end; t0 += q.TT) {
        const int64_t t1 = std::min<int64_t>(t0 + q.TT, t_end);
        int64_t amax = 0;
        for (int64_t j = t0 / q.S; j <= (t1 - 1) / q.S; ++j) amax = std::max(amax, q.anchors[j]);
        km.push_back(amax);
        if (q.mask) {
          for (int64_t kb = 0; kb < nkb; ++kb) {
            bool live = false;
            for (int64_t j = t0 / q.S; j <= (t1 - 1) / q.S && !live; ++j)
              live = q.mask[static_cast<size_t>(j) * q.mask_stride + kb] && q.anchors[j] > kb * kTileN;
            sa[b].live_tiles_of_block[kb] += live;
          }
        }
      }
      std::sort(km.begin(), km.end());
    }
  }
  make_items(q, policy, sa, out);
  place(q, policy, out);
  // the kernels need every item's key tiles to line up with the mask's 128-key blocks
  out.mask_aligned = true;
  if (q.mask)
    for (const auto& it : out.items)
      if ((it.key_begin - q.ctx[it.b]) % kTileN != 0) out.mask_aligned = false;
  if (q.mask && !out.mask_aligned) {
    // plan (costs, loads, imbalance) only: no work lists, the kernel calls refuse such a plan
    for (auto& it : out.items) it.kv_row = shard < 0 ? it.key_begin : -1;
    out.shard = shard;
    out.n_queues = shard < 0 && !one_queue ? q.P : 1;
    out.kv_heads = shard < 0 ? q.Hkv : 1;
    out.kv_rows = 0;
    out.mtiles.clear();
    out.sample_mt.assign(q.B + 1, 0);
    out.tok_kend.clear();
    out.tile_mask.clear();
    out.fwd.clear();
    out.pairs.clear();
    out.bwd.clear();
    out.bwd_item.clear();
    out.bwd_part.clear();
    out.bwd_rank.clear();
    out.bwd_det_order.clear();
    out.fwd_part_off.assign(out.n_queues + 1, 0);
    out.pair_off.assign(out.n_queues + 1, 0);
    out.bwd_part_off.assign(out.n_queues + 1, 0);
    out.merge_off.assign(1, 0);
    out.merge_list.clear();
    out.pair_tile_off.clear();
    out.unit_tile_off.clear();
    out.live_tiles.clear();
    out.dead.clear();
    return SKV_OK;
  }
  make_lists(q, sa, shard, one_queue, out);
  return SKV_OK;
}

// FNV-1a over the bytes of each value in turn.
struct Fnv {
  uint64_t h = 0xcbf29ce484222325ull;
  template <class T>
  void add(const T& v) {
    const auto* c = reinterpret_cast<const uint8_t*>(&v);
    for (size_t i = 0; i < sizeof(T); ++i) h = (h ^ c[i]) * 0x100000001b3ull;
  }
};

PlanHeader layout_of(const Prob& q, int policy, const Built& b) {
  PlanHeader h{};
  h.magic = kPlanMagic;
  h.version = kPlanVersion;
  h.policy = policy;
  h.B = q.B; h.Hq = q.Hq; h.Hkv = q.Hkv; h.d = q.d; h.block_q = q.S; h.chunk_kv = q.C;
  h.sub_chunks = q.sub; h.P = q.P; h.G = q.G; h.tile_tokens = q.TT;
  h.Nq = q.Nq; h.Ltot = q.Ltot;
  h.total_cost = b.total_cost;
  h.n_items = static_cast<int64_t>(b.items.size());
  h.n_mtiles = static_cast<int64_t>(b.mtiles.size());
  h.n_fwd = static_cast<int64_t>(b.fwd.size());
  h.n_bwd = static_cast<int64_t>(b.bwd.size());
  h.n_fwd_pairs = static_cast<int64_t>(b.pairs.size());
  h.imbalance = b.imbalance;
  h.fingerprint = 0;  // set by skv_plan from the caller's problem
  h.shard = b.shard;
  h.n_queues = b.n_queues;
  h.kv_heads = b.kv_heads;
  h.kv_rows = b.kv_rows;
  h.n_dead = static_cast<int32_t>(b.dead.size() / 2);
  h.empty_slots = 0;
  h.masked = q.mask ? (b.mask_aligned ? 1 : 2) : 0;
  h.mask_words = q.mask_words;
  for (size_t i = 0; i + 1 < b.merge_off.size(); ++i) h.empty_slots += b.merge_off[i + 1] == b.merge_off[i];
  uint64_t off = align_up(sizeof(PlanHeader), 256);
  h.items_off = off;
  off = align_up(off + b.items.size() * sizeof(skv_item), 64);
  h.load_off = off;
  off = align_up(off + static_cast<uint64_t>(q.P) * sizeof(int64_t), 64);
  h.dead_off = off;
  off = align_up(off + b.dead.size() * sizeof(int64_t), 64);
  h.bwd_part_host_off = off;
  off = align_up(off + b.bwd_part.size() * sizeof(int32_t), 256);
  h.dev_off = off;
  uint64_t d = 0;
  auto put = [&](uint64_t bytes) { uint64_t at = d; d = align_up(d + bytes, 256); return at; };
  h.dev.mtiles = put(b.mtiles.size() * sizeof(MTile));
  h.dev.tok_kend = put(b.tok_kend.size() * sizeof(int32_t));
  h.dev.fwd_units = put(b.fwd.size() * sizeof(FwdUnit));
  h.dev.fwd_part_off = put(b.fwd_part_off.size() * sizeof(int32_t));
  h.dev.fwd_pairs = put(b.pairs.size() * sizeof(FwdPair));
  h.dev.fwd_pair_off = put(b.pair_off.size() * sizeof(int32_t));
  h.dev.merge_off = put(b.merge_off.size() * sizeof(int32_t));
  h.dev.merge_list = put(b.merge_list.size() * sizeof(int32_t));
  h.dev.bwd_units = put(b.bwd.size() * sizeof(BwdUnit));
  h.dev.bwd_part_off = put(b.bwd_part_off.size() * sizeof(int32_t));
  h.dev.dead = put(b.dead.size() * sizeof(int64_t));
  h.dev.tile_mask = put(b.tile_mask.size() * sizeof(uint32_t));
  h.dev.pair_tile_off = put(b.pair_tile_off.size() * sizeof(int32_t));
  h.dev.unit_tile_off = put(b.unit_tile_off.size() * sizeof(int32_t));
  h.dev.live_tiles = put(b.live_tiles.size() * sizeof(int32_t));
  h.dev.base_bytes = d;
  h.dev.bwd_rank = put(b.bwd_rank.size() * sizeof(int32_t));
  h.dev.bwd_det_order = put(b.bwd_det_order.size() * sizeof(int32_t));
  h.dev.bytes = d;
  h.total_bytes = h.dev_off + d;
  return h;
}

// Writes a plan front to back: each array at its offset, zeros in the gaps before it. Offsets must come
// in ascending order (layout_of places the arrays in the order write_plan puts them).
struct PlanWriter {
  uint8_t* base;
  uint64_t cur;
  void zero_to(uint64_t off) {
    if (off > cur) std::memset(base + cur, 0, off - cur);
    cur = std::max(cur, off);
  }
  void put(uint64_t off, const void* src, size_t bytes) {
    zero_to(off);
    if (bytes) std::memcpy(base + off, src, bytes);
    cur = std::max(cur, off + bytes);
  }
  template <class T>
  void put(uint64_t off, const std::vector<T>& v) {
    put(off, v.data(), v.size() * sizeof(T));
  }
};

}  // namespace

uint64_t problem_fingerprint(const skv_problem* p) {
  Fnv f;
  f.add(p->num_samples);
  f.add(p->block_q);
  f.add(p->chunk_kv);
  f.add(p->sub_chunks);
  f.add(p->num_partitions);
  f.add(p->num_q_heads);
  f.add(p->num_kv_heads);
  f.add(p->head_dim);
  for (int b = 0; b <= p->num_samples; ++b) {
    f.add(p->ctx_offsets[b]);
    f.add(p->anchor_offsets[b]);
  }
  const int32_t A = p->anchor_offsets[p->num_samples];
  for (int32_t j = 0; j < A; ++j) f.add(p->anchors[j]);
  const int32_t has_mask = p->key_block_mask ? 1 : 0;
  f.add(has_mask);
  if (p->key_block_mask) {
    f.add(p->mask_stride);
    for (size_t i = 0; i < static_cast<size_t>(A) * p->mask_stride; ++i) f.add(p->key_block_mask[i]);
  }
  return f.h;
}

const PlanHeader* checked_plan(const void* plan, const skv_problem* prob, int* rc) {
  *rc = SKV_EINVAL;
  if (!plan || !prob || prob->num_samples < 1 || !prob->ctx_offsets || !prob->anchor_offsets) return nullptr;
  const PlanHeader* h = static_cast<const PlanHeader*>(plan);
  *rc = SKV_EPLAN;
  if (h->magic != kPlanMagic || h->version != kPlanVersion) return nullptr;
  // scalars first: a wrong sample count must not drive the reads of the problem's arrays
  if (h->B != prob->num_samples || h->Hq != prob->num_q_heads || h->Hkv != prob->num_kv_heads ||
      h->d != prob->head_dim || h->block_q != prob->block_q || h->chunk_kv != prob->chunk_kv ||
      h->sub_chunks != prob->sub_chunks || h->P != prob->num_partitions)
    return nullptr;
  if (prob->anchor_offsets[prob->num_samples] > 0 && !prob->anchors) return nullptr;
  if (h->Ltot != prob->ctx_offsets[prob->num_samples] ||
      h->Nq != static_cast<int64_t>(prob->anchor_offsets[prob->num_samples]) * prob->block_q)
    return nullptr;
  if (h->fingerprint != problem_fingerprint(prob)) return nullptr;
  *rc = SKV_OK;
  return h;
}

}  // namespace skv

using namespace skv;

// Planner working set of the calling thread: its vectors keep their capacity from call to call,
// so replanning every step (new anchors) does not reallocate and re-fault megabytes of lists.
Built& scratch() {
  thread_local Built b;
  return b;
}

namespace {

int plan_size(const skv_problem* prob, int policy, int shard, size_t* n_items, size_t* plan_bytes,
              size_t* ws_fwd_bytes, size_t* ws_bwd_bytes) {
  Built& b = scratch();
  Prob q;
  int rc = build(prob, policy, b, q, shard);
  if (rc != SKV_OK) return rc;
  PlanHeader h = layout_of(q, policy, b);
  WsLayout w = ws_layout(h);
  if (n_items) *n_items = b.items.size();
  if (plan_bytes) *plan_bytes = h.total_bytes;
  if (ws_fwd_bytes) *ws_fwd_bytes = w.fwd_end;
  if (ws_bwd_bytes) *ws_bwd_bytes = w.bwd_end;
  return SKV_OK;
}

int write_plan(const skv_problem* prob, int policy, int shard, void* plan, size_t plan_bytes,
               int64_t* partition_load) {
  if (!plan) return SKV_EINVAL;
  Built& b = scratch();
  Prob q;
  int rc = build(prob, policy, b, q, shard);
  if (rc != SKV_OK) return rc;
  PlanHeader h = layout_of(q, policy, b);
  if (plan_bytes < h.total_bytes) return SKV_EWORKSPACE;
  h.fingerprint = problem_fingerprint(prob);
  // The arrays in layout order; only the alignment gaps between them are zeroed, so every byte of the
  // plan is written once and the same problem always gives the same bytes.
  PlanWriter w{static_cast<uint8_t*>(plan), 0};
  w.put(0, &h, sizeof(h));
  w.put(h.items_off, b.items);
  w.put(h.load_off, b.load);
  w.put(h.dead_off, b.dead);
  w.put(h.bwd_part_host_off, b.bwd_part);
  const uint64_t dev = h.dev_off;
  w.put(dev + h.dev.mtiles, b.mtiles);
  w.put(dev + h.dev.tok_kend, b.tok_kend);
  w.put(dev + h.dev.fwd_units, b.fwd);
  w.put(dev + h.dev.fwd_part_off, b.fwd_part_off);
  w.put(dev + h.dev.fwd_pairs, b.pairs);
  w.put(dev + h.dev.fwd_pair_off, b.pair_off);
  w.put(dev + h.dev.merge_off, b.merge_off);
  w.put(dev + h.dev.merge_list, b.merge_list);
  w.put(dev + h.dev.bwd_units, b.bwd);
  w.put(dev + h.dev.bwd_part_off, b.bwd_part_off);
  w.put(dev + h.dev.dead, b.dead);
  w.put(dev + h.dev.tile_mask, b.tile_mask);
  w.put(dev + h.dev.pair_tile_off, b.pair_tile_off);
  w.put(dev + h.dev.unit_tile_off, b.unit_tile_off);
  w.put(dev + h.dev.live_tiles, b.live_tiles);
  w.put(dev + h.dev.bwd_rank, b.bwd_rank);
  w.put(dev + h.dev.bwd_det_order, b.bwd_det_order);
  w.zero_to(h.total_bytes);
  if (partition_load) std::memcpy(partition_load, b.load.data(), b.load.size() * sizeof(int64_t));
  return SKV_OK;
}

}  // namespace

extern "C" int skv_plan_size(const skv_problem* prob, int policy, size_t* n_items, size_t* plan_bytes,
                             size_t* ws_fwd_bytes, size_t* ws_bwd_bytes) {
  return plan_size(prob, policy, -1, n_items, plan_bytes, ws_fwd_bytes, ws_bwd_bytes);
}

extern "C" int skv_plan(const skv_problem* prob, int policy, void* plan, size_t plan_bytes,
                        int64_t* partition_load) {
  return write_plan(prob, policy, -1, plan, plan_bytes, partition_load);
}

extern "C" int skv_plan_shard_size(const skv_problem* prob, int policy, int partition, size_t* n_items,
                                   size_t* plan_bytes, size_t* ws_fwd_bytes, size_t* ws_bwd_bytes) {
  if (partition < 0) return SKV_EINVAL;
  return plan_size(prob, policy, partition, n_items, plan_bytes, ws_fwd_bytes, ws_bwd_bytes);
}

extern "C" int skv_plan_shard(const skv_problem* prob, int policy, int partition, void* plan, size_t plan_bytes,
                              int64_t* partition_load) {
  if (partition < 0) return SKV_EINVAL;
  return write_plan(prob, policy, partition, plan, plan_bytes, partition_load);
}

extern "C" int skv_plan_kv_layout(const void* plan, int64_t* kv_rows, int32_t* kv_heads, int32_t* shard) {
  if (!plan) return SKV_EINVAL;
  const PlanHeader* h = static_cast<const PlanHeader*>(plan);
  if (h->magic != kPlanMagic || h->version != kPlanVersion) return SKV_EPLAN;
  if (kv_rows) *kv_rows = h->kv_rows;
  if (kv_heads) *kv_heads = h->kv_heads;
  if (shard) *shard = h->shard;
  return SKV_OK;
}

extern "C" int skv_plan_items(const void* plan, const skv_item** items, size_t* n_items) {
  if (!plan) return SKV_EINVAL;
  const PlanHeader* h = static_cast<const PlanHeader*>(plan);
  if (h->magic != kPlanMagic || h->version != kPlanVersion) return SKV_EPLAN;
  if (items) *items = reinterpret_cast<const skv_item*>(static_cast<const uint8_t*>(plan) + h->items_off);
  if (n_items) *n_items = static_cast<size_t>(h->n_items);
  return SKV_OK;
}

extern "C" int skv_plan_unit_partitions(const void* plan, int32_t* fwd_part, int32_t* bwd_part) {
  if (!plan) return SKV_EINVAL;
  const PlanHeader* h = static_cast<const PlanHeader*>(plan);
  if (h->magic != kPlanMagic || h->version != kPlanVersion) return SKV_EPLAN;
  const uint8_t* dev = static_cast<const uint8_t*>(plan) + h->dev_off;
  if (fwd_part) {
    const FwdUnit* u = reinterpret_cast<const FwdUnit*>(dev + h->dev.fwd_units);
    for (int64_t i = 0; i < h->n_fwd; ++i) fwd_part[i] = u[i].part;
  }
  if (bwd_part && h->n_bwd > 0)
    std::memcpy(bwd_part, static_cast<const uint8_t*>(plan) + h->bwd_part_host_off, h->n_bwd * sizeof(int32_t));
  return SKV_OK;
}

extern "C" int skv_plan_stats(const void* plan, int64_t* total_cost, int64_t* n_fwd_units, int64_t* n_bwd_units,
                              double* imbalance) {
  if (!plan) return SKV_EINVAL;
  const PlanHeader* h = static_cast<const PlanHeader*>(plan);
  if (h->magic != kPlanMagic || h->version != kPlanVersion) return SKV_EPLAN;
  if (total_cost) *total_cost = h->total_cost;
  if (n_fwd_units) *n_fwd_units = h->n_fwd;
  if (n_bwd_units) *n_bwd_units = h->n_bwd;
  if (imbalance) *imbalance = h->imbalance;
  return SKV_OK;
}
