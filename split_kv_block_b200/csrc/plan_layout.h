// Internal layout of the host plan buffer written by skv_plan and of the
// device workspace. Shared by the planner (plan.cpp), the API layer (api.cu)
// and the kernels; not part of the public ABI.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/skv.h"

namespace skv {

constexpr uint64_t kPlanMagic = 0x31764b5374696c53ull;  // "SlitSKv1"
constexpr uint32_t kPlanVersion = 3;
constexpr int kTileM = 128;  // query rows per tile (TMEM lanes)
constexpr int kTileN = 128;  // keys per tile

// One 128-row query tile of one sample. Rows are ordered (token, head within
// the kv group): row r is token tok0 + r / G, q-head g * G + r % G.
struct MTile {
  int32_t b;
  int32_t tok0;   // first query token (packed index)
  int32_t ntok;   // tokens in the tile, <= 128 / G
  int32_t kmax;   // absolute key end: ctx_offsets[b] + max anchor over its tokens
  int32_t kbase;  // first key of the sample (ctx_offsets[b])
  int32_t mbase;  // block-sparse mask: entry of (this tile, block 0) in the tile-block words
  int32_t pad0, pad1;
};

// Forward unit: one item's key range restricted to one query tile.
// K/V buffer coordinates: key k of the unit is row k - kshift, head kvh of
// the K/V tensors the kernels read (kshift = 0 and kvh = g for a full plan;
// the row in the rank's shard buffer and head 0 for a shard plan).
struct FwdUnit {
  int32_t mt;    // query tile
  int32_t g;     // kv head (selects the query rows' heads)
  int32_t kbeg;  // absolute keys [kbeg, kend)
  int32_t kend;
  int32_t item;  // index into the plan's items
  int32_t part;  // partition
  int32_t kshift;
  int32_t kvh;
};

// Forward pair: two forward units (slots) of one item, processed together by
// one CTA that shares every K/V tile between the two query tiles. slot[1] is
// -1 when the item has an odd number of live query tiles.
struct FwdPair {
  int32_t slot[2];
  int32_t kbeg;  // key range covering both slots
  int32_t kend;
  int32_t part;
  int32_t pad;
};

// Block-sparse mask, per (query tile, key block of 128 keys of the sample):
// mask_words words whose bit t says that token t of the tile attends keys of
// the block (its anchor's mask bit is set and its anchor lies past the
// block's first key). Word group of (tile mt, block kb) starts at
// (mtiles[mt].mbase + kb) * mask_words.

// Backward unit: one tile of <= 128 keys of one item, against every query
// tile of the sample whose kmax exceeds kbeg. K/V, dK and dV coordinates as
// for FwdUnit.
struct BwdUnit {
  int32_t b;
  int32_t g;
  int32_t kbeg;
  int32_t kend;
  int32_t mt_begin;  // query tiles of sample b: [mt_begin, mt_end)
  int32_t mt_end;
  int32_t kshift;
  int32_t kvh;
};

// Offsets (bytes) of the arrays of the device section, relative to its start.
struct DevSection {
  uint64_t mtiles;        // MTile[n_mtiles]
  uint64_t tok_kend;      // int32[Nq]: absolute key end of every query token
  uint64_t fwd_units;     // FwdUnit[n_fwd]
  uint64_t fwd_part_off;  // int32[n_queues + 1]: units of work queue q are [off[q], off[q+1])
  uint64_t fwd_pairs;     // FwdPair[n_fwd_pairs]
  uint64_t fwd_pair_off;  // int32[n_queues + 1]: pairs of work queue q are [off[q], off[q+1])
  uint64_t merge_off;     // int32[n_mtiles * Hkv + 1]
  uint64_t merge_list;    // int32[n_fwd]: fwd unit ids per (tile, kv head), ascending kbeg
  uint64_t bwd_units;     // BwdUnit[n_bwd]
  uint64_t bwd_part_off;  // int32[n_queues + 1]
  uint64_t dead;          // int64[2 n_dead]: [begin, end) K/V rows whose dK/dV are zero
  uint64_t tile_mask;     // uint32[n_tile_blocks * mask_words] (block-sparse mask only)
  uint64_t pair_tile_off; // int32[n_fwd_pairs + 1]: live key tiles of every forward pair (mask only)
  uint64_t unit_tile_off; // int32[n_fwd + 1]: live key tiles of every forward unit (mask only)
  uint64_t live_tiles;    // int32[...]: first keys of those live key tiles, pairs' then units'
  uint64_t base_bytes;    // end of the arrays every call uploads; the ones below only the deterministic backward
  uint64_t bwd_rank;      // int32[n_bwd]: position of the unit's key tile among its (sample, kv head)'s, ascending
  uint64_t bwd_det_order; // int32[n_bwd]: units by (sample, rank, kv head), the deterministic dispatch order
  uint64_t bytes;         // total
};

struct PlanHeader {
  uint64_t magic;
  uint32_t version;
  int32_t policy;
  // problem scalars
  int32_t B, Hq, Hkv, d, block_q, chunk_kv, sub_chunks, P;
  int32_t G, tile_tokens;  // G = Hq / Hkv, tile_tokens = 128 / G
  int32_t shard;           // -1: full plan; p: the items of partition p only (skv_plan_shard)
  int32_t n_queues;        // work queues of the kernels: 1, or P for a full plan with partition queues
  int32_t kv_heads;        // heads per row of the K/V (dK/dV) buffers: Hkv, or 1 for a shard
  int32_t n_dead;          // [begin, end) row ranges whose dK/dV are zero
  int32_t empty_slots;     // (query tile, kv head) slots without a forward unit (possible in a shard)
  int32_t masked;          // block-sparse mask: 0 none; 1 the kernels can run; 2 items do not line up with
                           // the mask's 128-key blocks (plan for costs and loads only, kernel calls refused)
  int32_t mask_words;      // words per (tile, block): ceil(tile_tokens / 32)
  int64_t kv_rows;         // rows of the K/V (dK/dV) buffers: Ltot, or the shard's key count
  int64_t Nq, Ltot;
  int64_t total_cost;
  int64_t n_items, n_mtiles, n_fwd, n_bwd;
  int64_t n_fwd_pairs;
  double imbalance;
  uint64_t fingerprint;  // hash of the problem (shapes, offsets, anchors)
  // host-side arrays, offsets from the start of the plan buffer
  uint64_t items_off;      // skv_item[n_items]
  uint64_t load_off;       // int64[P]
  uint64_t dead_off;       // int64[2 * n_dead]: [begin, end) K/V rows whose dK/dV are zero
  uint64_t bwd_part_host_off;  // int32[n_bwd]: partition of every backward unit
  uint64_t dev_off;        // start of the device section (256-aligned)
  DevSection dev;
  uint64_t total_bytes;
};

// Workspace layout: control block (status word and queue counters, cleared by
// the same host-to-device copy that uploads the plan's device section behind
// it, once per call), device plan section, then the pass-specific scratch.
struct WsLayout {
  uint64_t status;    // int32 status word at offset 0
  uint64_t counters;  // int32[2 * P] queue heads (forward, backward), right after it
  uint64_t merge_ctr; // int32[2]: slots completed, merge tickets taken (forward with the merge in its tail)
  uint64_t arrive;    // int32[n_mtiles * Hkv]: warps that have written their unit's partial, per slot
  uint64_t ready;     // int32[n_mtiles * Hkv]: slot + 1 of the i-th completed slot
  uint64_t control;   // bytes of the control block
  uint64_t dev;       // device section copy
  uint64_t fwd_o;     // fp32 [n_fwd][128][d] partial outputs
  uint64_t fwd_lse;   // fp32 [n_fwd][128] partial LSE
  uint64_t fwd_end;
  uint64_t bwd_delta; // fp32 [Nq][Hq]: D = rowsum(dO * O)
  uint64_t bwd_dq;    // fp32 [Nq][Hq][d]: dQ accumulator
  uint64_t bwd_turn;  // int32 [n_mtiles * Hkv][8]: deterministic dQ, next rank to add per (slot, warp)
  uint64_t bwd_end;
};

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// 64-bit FNV-1a hash of a problem: its scalars, context offsets, anchor
// offsets and anchors (plan.cpp). Stored in every plan by skv_plan.
uint64_t problem_fingerprint(const skv_problem* p);

// The plan's header when `plan` is a plan of this library version written
// for `prob` (same scalars and the same fingerprint); otherwise nullptr with
// *rc = SKV_EINVAL (NULL pointers) or SKV_EPLAN. Host only: it reads the
// problem's arrays and touches no device state (plan.cpp).
const struct PlanHeader* checked_plan(const void* plan, const skv_problem* prob, int* rc);

inline WsLayout ws_layout(const PlanHeader& h) {
  WsLayout w{};
  w.status = 0;
  w.counters = 16;
  const uint64_t n_slots = static_cast<uint64_t>(h.n_mtiles) * h.Hkv;
  w.merge_ctr = w.counters + 2 * sizeof(int32_t) * static_cast<uint64_t>(h.P);
  w.arrive = w.merge_ctr + 2 * sizeof(int32_t);
  w.ready = w.arrive + sizeof(int32_t) * n_slots;
  w.control = w.ready + sizeof(int32_t) * n_slots;
  w.dev = align_up(w.control, 256);
  uint64_t scratch = align_up(w.dev + h.dev.bytes, 256);
  w.fwd_o = scratch;
  const uint64_t part_elem = (h.policy & SKV_PLAN_PARTIALS_BF16) ? 2 : 4;
  w.fwd_lse = align_up(w.fwd_o + static_cast<uint64_t>(h.n_fwd) * kTileM * h.d * part_elem, 256);
  w.fwd_end = align_up(w.fwd_lse + static_cast<uint64_t>(h.n_fwd) * kTileM * 4, 256);
  w.bwd_delta = scratch;
  w.bwd_dq = align_up(w.bwd_delta + static_cast<uint64_t>(h.Nq) * h.Hq * 4, 256);
  w.bwd_turn = align_up(w.bwd_dq + static_cast<uint64_t>(h.Nq) * h.Hq * h.d * 4, 256);
  w.bwd_end = align_up(w.bwd_turn + n_slots * 8 * sizeof(int32_t), 256);
  return w;
}

}  // namespace skv
