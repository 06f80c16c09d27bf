// Split-KV backward on sm_100a, head_dim 128: pipelined version.
//
// Same mathematics as bwd.cu (gradients through the split with P recomputed
// from the merged LSE; "Split-KV: Breaking the Context Parallelism Bottleneck
// in Diffusion Drafter Training", section "Split-KV's Core Mechanism"), laid
// out so that the tensor core is rarely idle:
//   * Two softmax-gradient warpgroups, each owning 64 of the tile's 128 query
//     rows, run two independent half-tile pipelines through the tensor core.
//     Half h has its own TMEM regions: A_h (64 columns) holds S^T of its rows
//     and then P^T (bf16, packed), B_h (64 columns) holds dP^T and then dQ^T;
//     dV and dK accumulate in the last 256 columns for the whole unit. As soon
//     as half h's gradient MMAs of tile i have consumed A_h and its dQ^T has
//     been read out of B_h, S^T and dP^T of half h of tile i+1 are computed,
//     so one half's softmax runs while the other half's MMAs execute.
//   * P^T stays in TMEM and feeds dV += P^T dO as the A operand; dS^T goes to
//     shared memory once and serves as the A operand of dK += dS^T Q and the
//     B operand of dQ^T = K^T dS^T. A half's gradient MMAs run dQ^T first,
//     then dV and dK, so its dQ^T is read out and reduced while the tensor
//     core still works on the half's dV and dK.
//   * dQ is produced transposed (TMEM lane = head-dim index), so the fp32
//     reduction into the shared dQ accumulator writes 128 consecutive floats
//     of a row per warpgroup instruction.
//   * Q and dO tiles are double-buffered.
// Warp roles: 0 scheduler + TMA producer, 1 MMA issuer, 2 TMEM allocator,
// 4..7 warpgroup 0 (rows 0..63), 8..11 warpgroup 1 (rows 64..127).
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace skv {
namespace {

constexpr int kD = 128;
constexpr int kTileBytes = 128 * kD * 2;  // 128 rows x 128 bf16

struct Ctl {
  float lse2[2][128];    // [tile parity][row]: log2-domain LSE (+inf for absent rows)
  float delta[2][128];   // D of the row
  uint8_t kend[2][128];  // keys of this unit the row attends: t < kend (0..128)
  int32_t kmin[2][2][2]; // [warpgroup][tile parity][warp]: min of kend over 32 rows
  uint64_t sched_full[2], sched_empty[2];
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2], do_full[2], do_empty[2];
  uint64_t sdp_full[2];   // per half: S^T and dP^T in TMEM
  uint64_t pds_full[2];   // per half: P^T in TMEM, dS^T in shared memory
  uint64_t dv_done[2];    // per half: dV MMA done (A_h free)
  uint64_t dq_full[2], dq_free[2];
  uint64_t acc_full, acc_free;
  uint64_t meta_full[2][2];  // [warpgroup][tile parity]
  uint64_t final_mma;
  int32_t sched[2];
  uint32_t tmem_base;
};

constexpr int kK = 0;
constexpr int kV = kK + kTileBytes;
constexpr int kQ0 = kV + kTileBytes;          // two stages
constexpr int kDO0 = kQ0 + 2 * kTileBytes;    // two stages
constexpr int kDS = kDO0 + 2 * kTileBytes;    // dS^T [128 keys][128 rows] bf16
constexpr int kCtl = kDS + 128 * 128 * 2;
constexpr int kSmemBytes = kCtl + static_cast<int>(sizeof(Ctl));
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint32_t col_a(int h) { return 64u * h; }         // S^T, then P^T, of half h
__device__ __forceinline__ uint32_t col_b(int h) { return 128u + 64u * h; }  // dP^T, then dQ^T, of half h
constexpr uint32_t kColDV = 256, kColDK = 384;

// kG: compile-time q-heads per kv-head (0 = runtime value p.G). kDet: dQ added
// in ascending key order under turn counters (deterministic backward) instead
// of fp32 atomics in any order. kMask: a block-sparse mask (rows whose block is
// off attend no key of the unit).
template <int kG, bool kDet, bool kMask>
__global__ void __launch_bounds__(384, 1)
    bwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kCtl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* status = p.status;
  const uint64_t lim = p.timeout_ns;
  // The query tiles a unit walks skip the tiles the block mask turns off, except in the deterministic
  // backward: there every unit below a tile's largest anchor takes its turn on that tile's dQ (adding
  // zeros when the mask leaves it nothing), so the turn sequence is the same as without a mask.
  constexpr bool kWalkMask = kMask && !kDet;

  // The 128-byte swizzle needs 1024-byte aligned tiles.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) atomicCAS(status, 0, kStatusBadPlan);
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.sched_full[i], 1);
      mbar_init(&c.sched_empty[i], 1 + 8);
      mbar_init(&c.q_full[i], 1);
      mbar_init(&c.q_empty[i], 1);
      mbar_init(&c.do_full[i], 1);
      mbar_init(&c.do_empty[i], 1);
      mbar_init(&c.pds_full[i], 128);
      mbar_init(&c.sdp_full[i], 1);
      mbar_init(&c.dv_done[i], 1);
      mbar_init(&c.dq_full[i], 1);
      mbar_init(&c.dq_free[i], 128);
      mbar_init(&c.meta_full[i][0], 128);
      mbar_init(&c.meta_full[i][1], 128);
    }
    mbar_init(&c.kv_full, 1);
    mbar_init(&c.kv_empty, 1);
    mbar_init(&c.acc_full, 1);
    mbar_init(&c.acc_free, 256);
    mbar_init(&c.final_mma, 1);
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&c.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ scheduler + producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      int part = static_cast<int>((static_cast<long long>(blockIdx.x) * p.P) / gridDim.x);
      int visited = 0;
      uint32_t n_units = 0, qc = 0, kv_issued = 0;
      bool ok = true;
      auto load_tile = [&](const MTile& M, int g) -> bool {
        const int s = qc & 1;
        const uint32_t use = qc >> 1;
        if (use >= 1 && !mbar_wait(&c.q_empty[s], (use - 1) & 1, status, lim)) return false;
        mbar_arrive_expect_tx(&c.q_full[s], kTileBytes);
        for (int db = 0; db < 2; ++db)
          tma_load_3d(smem + kQ0 + s * kTileBytes + db * 16384, &tmQ, &c.q_full[s], db * 64, g * p.G, M.tok0);
        if (use >= 1 && !mbar_wait(&c.do_empty[s], (use - 1) & 1, status, lim)) return false;
        mbar_arrive_expect_tx(&c.do_full[s], kTileBytes);
        for (int db = 0; db < 2; ++db)
          tma_load_3d(smem + kDO0 + s * kTileBytes + db * 16384, &tmDO, &c.do_full[s], db * 64, g * p.G, M.tok0);
        ++qc;
        return true;
      };
      while (ok) {
        int u = -1;
        if constexpr (kDet) {
          // one queue in (sample, rank, kv head) order: a unit only ever waits for units taken before it
          const int idx = atomicAdd(&p.counters[0], 1);
          if (idx < p.n_bwd) u = p.det_order[idx];
        } else {
          while (visited < p.P) {
            const int cnt = p.part_off[part + 1] - p.part_off[part];
            const int idx = atomicAdd(&p.counters[part], 1);
            if (idx < cnt) {
              u = p.part_off[part] + idx;
              break;
            }
            part = (part + 1 == p.P) ? 0 : part + 1;
            ++visited;
          }
        }
        const int slot = n_units & 1;
        if (n_units >= 2 && !mbar_wait(&c.sched_empty[slot], ((n_units >> 1) - 1) & 1, status, lim)) break;
        c.sched[slot] = u;
        mbar_arrive(&c.sched_full[slot]);
        if (u < 0) break;
        const BwdUnit U = p.units[u];
        bool kv_loaded = false;
        for (int mt = U.mt_begin; mt < U.mt_end && ok; ++mt) {
          const MTile M = p.mtiles[mt];
          if (!tile_live<kWalkMask>(p, M, U.kbeg)) continue;
          if (!load_tile(M, U.g)) { ok = false; break; }
          if (!kv_loaded) {  // after the first Q/dO tile: K/V wait for the previous unit's last MMA
            if (kv_issued >= 1 && !mbar_wait(&c.kv_empty, (kv_issued - 1) & 1, status, lim)) { ok = false; break; }
            mbar_arrive_expect_tx(&c.kv_full, 2 * kTileBytes);
            for (int db = 0; db < 2; ++db) {
              tma_load_3d(smem + kK + db * 16384, &tmK, &c.kv_full, db * 64, U.kvh, U.kbeg - U.kshift);
              tma_load_3d(smem + kV + db * 16384, &tmV, &c.kv_full, db * 64, U.kvh, U.kbeg - U.kshift);
            }
            ++kv_issued;
            kv_loaded = true;
          }
        }
        ++n_units;
      }
      // let every issued load land before the CTA may exit
      if (kv_issued > 0) mbar_wait(&c.kv_full, (kv_issued - 1) & 1, nullptr, lim);
      for (int s = 0; s < 2; ++s) {
        const uint32_t uses = (qc + 1 - s) >> 1;
        if (uses > 0) {
          mbar_wait(&c.q_full[s], (uses - 1) & 1, nullptr, lim);
          mbar_wait(&c.do_full[s], (uses - 1) & 1, nullptr, lim);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // All 32 lanes run the loop (stage indices and descriptors stay warp-uniform); one elected lane issues
    // the MMAs and their commits.
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16(128, 64, false, false);   // S^T_h = K Q_h^T, dP^T_h = V dO_h^T
    constexpr uint32_t idKV = idesc_bf16(128, kD, false, true);   // dV += P^T dO, dK += dS^T Q (half's rows)
    constexpr uint32_t idQ = idesc_bf16(128, 64, true, true);     // dQ^T_h = K^T dS^T_h
    // operand descriptors at their buffers' starts; K steps, row blocks and stages are byte offsets
    const uint64_t dK_k = sdesc_sw128(smem_u32(smem + kK), 16, 1024);          // K as A of S^T (K-major)
    const uint64_t dV_k = sdesc_sw128(smem_u32(smem + kV), 16, 1024);          // V as A of dP^T
    const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + kK), 16384, 1024);      // K^T as A of dQ^T (MN-major)
    const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + kQ0), 16, 1024);         // Q_h as B of S^T
    const uint64_t dDO_k = sdesc_sw128(smem_u32(smem + kDO0), 16, 1024);       // dO_h as B of dP^T
    const uint64_t dQ_mn = sdesc_sw128(smem_u32(smem + kQ0), 16384, 1024);     // Q as B of dK
    const uint64_t dDO_mn = sdesc_sw128(smem_u32(smem + kDO0), 16384, 1024);   // dO as B of dV
    const uint64_t dS_k = sdesc_sw128(smem_u32(smem + kDS), 16, 1024);         // dS^T as A of dK
    const uint64_t dS_mn = sdesc_sw128(smem_u32(smem + kDS), 16384, 1024);     // dS^T as B of dQ^T
    uint32_t n_units = 0, qc = 0, kv_waits = 0;
    bool ok = true;
    // S^T and dP^T of half h of tile number i: rows 64h..64h+63 of its Q / dO tile, into A_h / B_h once
    // half h of tile i - 1 has consumed A_h (its dV) and its dQ^T has been read out of B_h
    auto issue_sdp = [&](uint32_t i, int h) -> bool {
      const int s = i & 1;
      const uint32_t use = i >> 1;
      if (!mbar_wait_warp(&c.q_full[s], use & 1, status, lim)) return false;
      if (!mbar_wait_warp(&c.do_full[s], use & 1, status, lim)) return false;
      if (i >= 1 && (!mbar_wait_warp(&c.dv_done[h], (i - 1) & 1, status, lim) ||
                     !mbar_wait_warp(&c.dq_free[h], (i - 1) & 1, status, lim)))
        return false;
      tc_fence_after();
      const uint32_t rows = s * kTileBytes + h * 8192;
      if (leader) {
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          umma_bf16(tmem + col_a(h), sdesc_add(dK_k, off), sdesc_add(dQ_k, rows + off), idS, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          umma_bf16(tmem + col_b(h), sdesc_add(dV_k, off), sdesc_add(dDO_k, rows + off), idS, ks > 0);
        }
        umma_commit(&c.sdp_full[h]);
      }
      __syncwarp();
      return true;
    };
    while (ok) {
      const int slot = n_units & 1;
      if (!mbar_wait_warp(&c.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
      const int u = c.sched[slot];
      __syncwarp();
      if (leader) mbar_arrive(&c.sched_empty[slot]);
      if (u < 0) break;
      const BwdUnit U = p.units[u];
      bool first = true;
      // live query tiles in order (mt, then nxt); the liveness of the tile after nxt is loaded at the top of
      // a tile and read at its end, so no load stalls the issue of a tile's MMAs
      auto live_from = [&](int i) -> int {
        while (i < U.mt_end && !tile_live<kWalkMask>(p, p.mtiles[i], U.kbeg)) ++i;
        return i;
      };
      int mt = live_from(U.mt_begin);
      int nxt = mt < U.mt_end ? live_from(mt + 1) : U.mt_end;
      while (mt < U.mt_end) {
        const bool live_c = nxt < U.mt_end && nxt + 1 < U.mt_end && tile_live<kWalkMask>(p, p.mtiles[nxt + 1], U.kbeg);
        const int s = qc & 1;
        if (first) {  // a unit's first tile waits for the unit's K/V
          if (!mbar_wait_warp(&c.kv_full, (kv_waits++) & 1, status, lim)) { ok = false; break; }
          if (!issue_sdp(qc, 0) || !issue_sdp(qc, 1)) { ok = false; break; }
        }
        for (int h = 0; h < 2 && ok; ++h) {
          if (!mbar_wait_warp(&c.pds_full[h], qc & 1, status, lim)) { ok = false; break; }
          if (first && h == 0 && n_units >= 1 && !mbar_wait_warp(&c.acc_free, (n_units - 1) & 1, status, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
            // dQ^T of the half's rows = K^T dS^T -> B_h, first: the gradient warps read it out and reduce it
            // while the tensor core runs the half's dV and dK
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks)
              umma_bf16(tmem + col_b(h), sdesc_add(dK_mn, ks * 2048), sdesc_add(dS_mn, h * 16384 + ks * 2048), idQ,
                        ks > 0);
            umma_commit(&c.dq_full[h]);
            // dV += P^T dO over the half's 64 rows (A = P^T_h from TMEM)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint32_t acc = (first && h == 0 && k4 == 0) ? 0u : 1u;
              umma_bf16_ts(tmem + kColDV, tmem + col_a(h) + 8 * k4,
                           sdesc_add(dDO_mn, s * kTileBytes + (64 * h + 16 * k4) * 128), idKV, acc);
            }
            umma_commit(&c.dv_done[h]);
            if (h == 1) umma_commit(&c.do_empty[s]);
            // dK += dS^T Q over the half's rows (the next tile's dS^T is written only after its S^T/dP^T, whose
            // commit covers this MMA)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const uint32_t acc = (first && h == 0 && k4 == 0) ? 0u : 1u;
              umma_bf16(tmem + kColDK, sdesc_add(dS_k, h * 16384 + k4 * 32),
                        sdesc_add(dQ_mn, s * kTileBytes + (64 * h + 16 * k4) * 128), idKV, acc);
            }
            if (h == 1) umma_commit(&c.q_empty[s]);
          }
          __syncwarp();
          // this half of the unit's next tile, as soon as A_h and B_h are free
          if (nxt < U.mt_end && !issue_sdp(qc + 1, h)) { ok = false; break; }
        }
        if (!ok) break;
        first = false;
        ++qc;
        int nn = U.mt_end;
        if (nxt < U.mt_end) {
          nn = nxt + 1;
          if (nn < U.mt_end && !live_c) nn = live_from(nn + 1);
        }
        mt = nxt;
        nxt = nn;
      }
      if (!ok) break;
      // A unit without live query tiles (possible under a block mask) issues no MMA; it still waits for the
      // previous unit's dK/dV read-out before signalling its own, so that acc_full never runs two phases ahead
      // of the gradient warps (its parity would then name the wrong phase).
      if (first && n_units >= 1 && !mbar_wait_warp(&c.acc_free, (n_units - 1) & 1, status, lim)) break;
      if (leader) {
        if (!first) umma_commit(&c.kv_empty);  // K/V were loaded for this unit
        umma_commit(&c.acc_full);
      }
      __syncwarp();
      ++n_units;
    }
    if (leader) umma_commit(&c.final_mma);
    __syncwarp();
    mbar_wait_warp(&c.final_mma, 0, nullptr, lim);
  } else if (warp >= 4) {
    // ------------------------- softmax gradient, dQ drain, dK/dV epilogue
    const int wg = (warp - 4) >> 2;          // warpgroup: rows [64 wg, 64 wg + 64) of the tile
    const int t = (warp & 3) * 32 + lane;    // TMEM lane: key (S^T, dP^T, dV, dK) or d index (dQ^T)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    constexpr float kLog2e = 1.4426950408889634f;
    const int G = kG > 0 ? kG : p.G;
    const int lgG = kG > 0 ? (31 - __clz(kG)) : p.lgG;
    const size_t tok_stride = static_cast<size_t>(p.Hq) * kD;
    uint32_t n_units = 0, qc = 0;
    bool ok = true;
    // Row metadata (LSE, D, key end) of the next live query tile, loaded one tile ahead by threads t < 64
    // (row 64 wg + t) and used only when staged for that tile: the loads never stall the current tile.
    // Rows past the tile's tokens read token tok0 (a valid address) and are masked when staged.
    float rw_lse = 0.f, rw_del = 0.f;
    int rw_ke = 0;
    bool rw_valid = false;
    auto fetch = [&](const MTile& Mx, int g, int kb) {
      if (t < 64) {
        const int r = 64 * wg + t;
        const int tl = r >> lgG;
        rw_valid = tl < Mx.ntok;
        const int token = Mx.tok0 + (rw_valid ? tl : 0), head = g * G + (r & (G - 1));
        rw_lse = p.lse[static_cast<size_t>(token) * p.Hq + head];
        rw_del = p.delta[static_cast<size_t>(token) * p.Hq + head];
        rw_ke = p.tok_kend[token];
        // a row whose block is off attends none of the unit's keys
        if (kMask && rw_valid && !((mask_word(p.tile_mask, p.mask_words, Mx, kb, tl) >> (tl & 31)) & 1u)) rw_ke = 0;
      }
    };
    // the next live query tile of unit U at or after index i (the scan loads only at unit starts and when
    // a prefetched candidate is dead)
    auto live_from = [&](const BwdUnit& U, int i) -> int {
      while (i < U.mt_end && !tile_live<kWalkMask>(p, p.mtiles[i], U.kbeg)) ++i;
      return i;
    };
    while (ok) {
      const int slot = n_units & 1;
      if (!mbar_wait_warp(&c.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
      const int u = c.sched[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.sched_empty[slot]);
      if (u < 0) break;
      const BwdUnit U = p.units[u];
      if (p.stamps && tid == 128) p.stamps[2 * u] = static_cast<long long>(globaltimer_ns());
      const int nkeys = U.kend - U.kbeg;
      // live tiles in order: mt (M), then nxt (Mn); cand is the tile after nxt, loaded one tile ahead (Mc)
      int mt = live_from(U, U.mt_begin);
      MTile M{}, Mn{}, Mc{};
      int nxt = U.mt_end, cand = U.mt_end;
      if (mt < U.mt_end) {
        M = p.mtiles[mt];
        fetch(M, U.g, U.kbeg);
        nxt = live_from(U, mt + 1);
        if (nxt < U.mt_end) {
          Mn = p.mtiles[nxt];
          cand = nxt + 1;
          if (cand < U.mt_end) Mc = p.mtiles[cand];
        }
      }
      bool had_tiles = false;
      while (mt < U.mt_end) {
        had_tiles = true;
        const int par = qc & 1;
        const uint32_t tA = tmem + lane_off + col_a(wg), tB = tmem + lane_off + col_b(wg);
        // stage this tile's metadata, then fetch the next live tile's
        if (t < 64) {
          const int r = 64 * wg + t;
          const int ke = rw_valid ? max(0, min(min(rw_ke, U.kend) - U.kbeg, nkeys)) : 0;
          c.lse2[par][r] = rw_valid ? rw_lse * kLog2e : INFINITY;
          c.delta[par][r] = rw_valid ? rw_del : 0.f;
          c.kend[par][r] = static_cast<uint8_t>(ke);
          const int wmin = __reduce_min_sync(0xffffffffu, ke);
          if (lane == 0) c.kmin[wg][par][warp & 1] = wmin;
        }
        // prefetch: the next tile's row metadata (from Mn, already in registers), then the tile after it from
        // the candidate loaded one tile ago, and the candidate after that
        int nn = U.mt_end;
        MTile Mnn = Mn;
        if (nxt < U.mt_end) {
          fetch(Mn, U.g, U.kbeg);
          nn = cand;
          if (nn < U.mt_end) {
            if (tile_live<kWalkMask>(p, Mc, U.kbeg)) {
              Mnn = Mc;
            } else {
              nn = live_from(U, nn + 1);
              if (nn < U.mt_end) Mnn = p.mtiles[nn];
            }
          }
          if (nn < U.mt_end && nn + 1 < U.mt_end) Mc = p.mtiles[nn + 1];
        }
        mbar_arrive(&c.meta_full[wg][par]);
        if (!mbar_wait_warp(&c.meta_full[wg][par], (qc >> 1) & 1, status, lim)) { ok = false; break; }
        // every row of this half attends key t of every lane of the warp: no per-element mask
        const bool unmasked = __all_sync(0xffffffffu, t < min(c.kmin[wg][par][0], c.kmin[wg][par][1]));
        if (!mbar_wait_warp(&c.sdp_full[wg], qc & 1, status, lim)) { ok = false; break; }
        tc_fence_after();
        uint8_t* dsrow = smem + kDS + wg * 16384;
        const float sl2 = p.scale_log2;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          const int col = 64 * wg + 32 * ch;  // first tile row of this chunk
          uint32_t vs[32], vd[32];
          tmem_ld32(tA + 32 * ch, vs);
          tmem_ld32(tB + 32 * ch, vd);
          tmem_wait_ld();
          uint32_t pk[16];
          uint32_t dk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 L4 = *reinterpret_cast<const float4*>(&c.lse2[par][col + i]);
            const float4 D4 = *reinterpret_cast<const float4*>(&c.delta[par][col + i]);
            float x0 = ex2(fmaf(__uint_as_float(vs[i + 0]), sl2, -L4.x));
            float x1 = ex2(fmaf(__uint_as_float(vs[i + 1]), sl2, -L4.y));
            float x2 = ex2(fmaf(__uint_as_float(vs[i + 2]), sl2, -L4.z));
            float x3 = ex2(fmaf(__uint_as_float(vs[i + 3]), sl2, -L4.w));
            if (!unmasked) {
              const uint32_t k4 = *reinterpret_cast<const uint32_t*>(&c.kend[par][col + i]);
              x0 = t < static_cast<int>(k4 & 0xffu) ? x0 : 0.f;
              x1 = t < static_cast<int>((k4 >> 8) & 0xffu) ? x1 : 0.f;
              x2 = t < static_cast<int>((k4 >> 16) & 0xffu) ? x2 : 0.f;
              x3 = t < static_cast<int>(k4 >> 24) ? x3 : 0.f;
            }
            pk[(i >> 1) + 0] = pack_bf16(x0, x1);
            pk[(i >> 1) + 1] = pack_bf16(x2, x3);
            dk[(i >> 1) + 0] = pack_bf16(x0 * (__uint_as_float(vd[i + 0]) - D4.x), x1 * (__uint_as_float(vd[i + 1]) - D4.y));
            dk[(i >> 1) + 1] = pack_bf16(x2 * (__uint_as_float(vd[i + 2]) - D4.z), x3 * (__uint_as_float(vd[i + 3]) - D4.w));
          }
          // P^T (bf16 pairs) over the S^T columns of this half already read
          tmem_st16(tA + 16 * ch, pk);
          // dS^T row t of this warpgroup's 64-row block: 16-byte chunks 4 ch .. 4 ch + 3
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(dsrow + sw128_off(t, 4 * ch + q)) =
                make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&c.pds_full[wg]);
        // dQ^T of this warpgroup's rows: lane t = head-dim index t
        if (!mbar_wait_warp(&c.dq_full[wg], qc & 1, status, lim)) { ok = false; break; }
        tc_fence_after();
        uint32_t q0[32], q1[32];
        tmem_ld32(tB, q0);
        tmem_ld32(tB + 32, q1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&c.dq_free[wg]);
        // fp32 reduction: row r -> dq_acc[(tok0 + r / G) * Hq + g * G + r % G][t]
        float* base = p.dq_acc + (static_cast<size_t>(M.tok0) * p.Hq + static_cast<size_t>(U.g) * G) * kD + t;
        if constexpr (kDet) {
          // in ascending key order: this warp's 32 head-dim columns of the half's rows, after every
          // lower-ranked unit of the sample and kv head has added its own. Within the turn the adds are
          // fp32 reductions: the turn fixes the order in which they reach each address, and the fence
          // of turn_pass waits for them before the next rank may start.
          int32_t* turn = p.turn + (static_cast<size_t>(mt) * p.Hkv + U.g) * 8 + wg * 4 + (warp & 3);
          const int my = p.rank[u];
          if (turn_wait(turn, my, status, lim, lane)) {
            const int nrows = M.ntok << lgG;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int r = 64 * wg + j;
              if (r < nrows) atomicAdd(base + (r >> lgG) * tok_stride + (r & (G - 1)) * kD, __uint_as_float(q0[j]));
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int r = 64 * wg + 32 + j;
              if (r < nrows) atomicAdd(base + (r >> lgG) * tok_stride + (r & (G - 1)) * kD, __uint_as_float(q1[j]));
            }
            turn_pass(turn, my + 1, lane);
          }
        } else if constexpr (kG > 0) {
          static_assert(64 % (kG > 0 ? kG : 1) == 0, "group size must divide 64");
          constexpr int kTok = 64 / (kG > 0 ? kG : 1);  // tokens per half tile
          const int tl0 = (64 * wg) / (kG > 0 ? kG : 1);
          float* row0 = base + static_cast<size_t>(tl0) * tok_stride;
          const int ntok_here = min(M.ntok - tl0, kTok);  // tokens of this half that exist
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j / kG < ntok_here)
              atomicAdd(row0 + static_cast<size_t>(j / kG) * tok_stride + (j % kG) * kD, __uint_as_float(q0[j]));
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if ((32 + j) / kG < ntok_here)
              atomicAdd(row0 + static_cast<size_t>((32 + j) / kG) * tok_stride + ((32 + j) % kG) * kD,
                        __uint_as_float(q1[j]));
        } else {
          const int nrows = M.ntok << lgG;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int r = 64 * wg + j;
            if (r < nrows) atomicAdd(base + (r >> lgG) * tok_stride + (r & (G - 1)) * kD, __uint_as_float(q0[j]));
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int r = 64 * wg + 32 + j;
            if (r < nrows) atomicAdd(base + (r >> lgG) * tok_stride + (r & (G - 1)) * kD, __uint_as_float(q1[j]));
          }
        }
        ++qc;
        M = Mn;
        mt = nxt;
        Mn = Mnn;
        nxt = nn;
        cand = nn + 1;
      }
      if (!ok) break;
      // dV (warpgroup 0) / dK (warpgroup 1) of the unit's keys
      if (!mbar_wait_warp(&c.acc_full, n_units & 1, status, lim)) break;
      tc_fence_after();
      const uint32_t acc_col = wg == 0 ? kColDV : kColDK;
      const float mul = wg == 0 ? 1.f : p.scale;
      __nv_bfloat16* dst =
          (wg == 0 ? p.dv : p.dk) + (static_cast<size_t>(U.kbeg - U.kshift + t) * p.kv_heads + U.kvh) * kD;
#pragma unroll 1
      for (int cc = 0; cc < kD; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + acc_col + cc, v);
        tmem_wait_ld();
        if (t < nkeys) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (had_tiles) {  // a unit without live query tiles (none are planned) owns zero gradients
              w.x = pack_bf16(__uint_as_float(v[i]) * mul, __uint_as_float(v[i + 1]) * mul);
              w.y = pack_bf16(__uint_as_float(v[i + 2]) * mul, __uint_as_float(v[i + 3]) * mul);
              w.z = pack_bf16(__uint_as_float(v[i + 4]) * mul, __uint_as_float(v[i + 5]) * mul);
              w.w = pack_bf16(__uint_as_float(v[i + 6]) * mul, __uint_as_float(v[i + 7]) * mul);
            }
            *reinterpret_cast<uint4*>(dst + cc + i) = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&c.acc_free);
      if (p.stamps && tid == 128) p.stamps[2 * u + 1] = static_cast<long long>(globaltimer_ns());
      ++n_units;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_bwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                        const BwdParams& p, int grid, cudaStream_t stream) {
  const bool m = p.tile_mask != nullptr;
  auto kern = p.det ? (p.G == 4 ? (m ? bwd2_kernel<4, true, true> : bwd2_kernel<4, true, false>)
                                : (m ? bwd2_kernel<0, true, true> : bwd2_kernel<0, true, false>))
                    : (p.G == 4 ? (m ? bwd2_kernel<4, false, true> : bwd2_kernel<4, false, false>)
                                : (m ? bwd2_kernel<0, false, true> : bwd2_kernel<0, false, false>));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, 384, kSmemBytes, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

}  // namespace skv
