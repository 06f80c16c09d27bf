// Split-KV forward on sm_100a, head_dim 128: two query tiles per CTA.
//
// Same mathematics as fwd.cu (per forward unit: partial softmax attention of
// one 128-row query tile over one item's key range, normalized partial output
// and log-sum-exp; "Split-KV: Breaking the Context Parallelism Bottleneck in
// Diffusion Drafter Training", section "Split-KV's Core Mechanism"), arranged
// for the tensor core:
//   * a work unit is a pair of forward units of the same item (same kv head,
//     same key range up to the longer one's end): every K/V tile loaded by TMA
//     serves both query tiles;
//   * TMEM holds S and O for both tiles (4 x 128 columns); P overwrites the
//     first 64 columns of its S (bf16 pairs) and feeds O += P V as the A
//     operand straight from TMEM;
//   * two softmax warpgroups, one per query tile, alternate with the tensor
//     core: while one computes its P, the MMA warp runs the other tile's PV
//     and next S;
//   * lazy rescaling: a row's reference maximum moves only when the tile
//     maximum exceeds it by more than 8 (log2 units), so O is rarely touched;
//     the final normalization uses the same reference, so the result is exact.
// Warp roles: 0 scheduler + TMA producer, 1 MMA issuer, 2 TMEM allocator,
// 4..7 softmax of tile 0, 8..11 softmax of tile 1.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"
#include "tail_merge.cuh"

namespace skv {
namespace {

constexpr int kD = 128;
constexpr int kTileBytes = 128 * kD * 2;  // a 128 x 128 bf16 tile
constexpr int kQ0 = 0;                    // Q of tile 0 and tile 1
constexpr int kK0 = kQ0 + 2 * kTileBytes; // two K stages
constexpr int kV0 = kK0 + 2 * kTileBytes; // two V stages
constexpr int kCtl = kV0 + 2 * kTileBytes;

struct Ctl {
  uint64_t sched_full[2], sched_empty[2];
  uint64_t q_full[2], q_empty[2];       // per query tile
  uint64_t k_full[2], k_empty[2];       // per K stage
  uint64_t v_full[2], v_empty[2];       // per V stage
  uint64_t s_full[2];                   // per query tile: S in TMEM
  uint64_t p_full[2];                   // per query tile: P in TMEM (128 arrivals)
  uint64_t pv_done[2];                  // per query tile: O += P V completed
  uint64_t o_free[2];                   // per query tile: epilogue has read O (128 arrivals)
  uint64_t final_mma;
  int32_t sched[2];
  uint32_t tmem_base;
  int32_t merge_slot;  // tail merge: slot being merged (broadcast)
};
constexpr int kSmemBytes = kCtl + static_cast<int>(sizeof(Ctl));
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint32_t col_s(int t) { return 128u * t; }        // S of tile t
__device__ __forceinline__ uint32_t col_o(int t) { return 256u + 128u * t; } // O of tile t

// descriptor offset (16-byte units) of K-step ks inside a K-major SW128 tile of 128 rows
__device__ __forceinline__ uint64_t kmaj(int ks) {
  return static_cast<uint64_t>(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
}

// Maximum of a 128-column score row: eight independent three-input chains.
__device__ __forceinline__ float row_max(const uint32_t (&sv)[128]) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 128; i += 2) mx[(i >> 1) & 7] = fmax3(mx[(i >> 1) & 7], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
  return fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7]));
}

// P = 2^(s sl2 - m_use) over one score row (masked entries are -inf -> 0), stored as bf16
// pairs into the first 64 TMEM columns at tS; returns the row sum (four independent sums).
// With kMax it also returns, in raw_max, the maximum of the raw scores: the three-input
// maxima go to the ALU pipe, idle while the exponentials hold the special-function pipe
// (one warp instruction per 8 cycles per SM quarter, the bound of this loop).
template <bool kMax>
__device__ __forceinline__ float exp_row(const uint32_t (&sv)[128], float sl2, float m_use, uint32_t tS,
                                         float& raw_max) {
  float rs[4] = {0.f, 0.f, 0.f, 0.f};
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int cc = 0; cc < 128; cc += 32) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float s0 = __uint_as_float(sv[cc + i]), s1 = __uint_as_float(sv[cc + i + 1]);
      const float s2 = __uint_as_float(sv[cc + i + 2]), s3 = __uint_as_float(sv[cc + i + 3]);
      if (kMax) {
        mx[(i >> 2) & 1] = fmax3(mx[(i >> 2) & 1], s0, s1);
        mx[2 + ((i >> 2) & 1)] = fmax3(mx[2 + ((i >> 2) & 1)], s2, s3);
      }
      const float x0 = ex2(fmaf(s0, sl2, -m_use));
      const float x1 = ex2(fmaf(s1, sl2, -m_use));
      const float x2 = ex2(fmaf(s2, sl2, -m_use));
      const float x3 = ex2(fmaf(s3, sl2, -m_use));
      rs[0] += x0;
      rs[1] += x1;
      rs[2] += x2;
      rs[3] += x3;
      pk[(i >> 1) + 0] = pack_bf16(x0, x1);
      pk[(i >> 1) + 1] = pack_bf16(x2, x3);
    }
    tmem_st16(tS + (cc >> 1), pk);
  }
  if (kMax) raw_max = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
  return (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

// kMerge: the LSE merge runs in the kernel's tail (skv_attn_fwd_merged); the
// plain forward is compiled without that code. kMask: a block-sparse mask;
// every role walks the pair's list of live key tiles (the same list, so they
// agree on the sequence) and the softmax masks the rows whose block is off.
template <bool kMerge, bool kMask>
__global__ void __launch_bounds__(384, 1)
    fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctl& c = *reinterpret_cast<Ctl*>(smem + kCtl);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* status = p.status;
  const uint64_t lim = p.timeout_ns;
  if ((smem_u32(smem) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (tid == 0) atomicCAS(status, 0, kStatusBadPlan);
    return;
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.sched_full[i], 1);
      mbar_init(&c.sched_empty[i], 1 + 8);
      mbar_init(&c.q_full[i], 1);
      mbar_init(&c.q_empty[i], 1);
      mbar_init(&c.k_full[i], 1);
      mbar_init(&c.k_empty[i], 1);
      mbar_init(&c.v_full[i], 1);
      mbar_init(&c.v_empty[i], 1);
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.p_full[i], 128);
      mbar_init(&c.pv_done[i], 1);
      mbar_init(&c.o_free[i], 128);
    }
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
      int part = static_cast<int>((static_cast<long long>(blockIdx.x) * p.P) / gridDim.x);
      int visited = 0;
      uint32_t n_units = 0, kv = 0, k_iss = 0, v_iss = 0, q_iss[2] = {0, 0};
      bool ok = true;
      while (ok) {
        int u = -1;
        while (visited < p.P) {
          const int cnt = p.pair_off[part + 1] - p.pair_off[part];
          const int idx = atomicAdd(&p.counters[part], 1);
          if (idx < cnt) {
            u = p.pair_off[part] + idx;
            break;
          }
          part = (part + 1 == p.P) ? 0 : part + 1;
          ++visited;
        }
        const int slot = n_units & 1;
        if (n_units >= 2 && !mbar_wait(&c.sched_empty[slot], ((n_units >> 1) - 1) & 1, status, lim)) break;
        c.sched[slot] = u;
        mbar_arrive(&c.sched_full[slot]);
        if (u < 0) break;
        const FwdPair pr = p.pairs[u];
        for (int t = 0; t < 2 && ok; ++t) {
          if (pr.slot[t] < 0) continue;
          const FwdUnit U = p.units[pr.slot[t]];
          const MTile M = p.mtiles[U.mt];
          if (q_iss[t] >= 1 && !mbar_wait(&c.q_empty[t], (q_iss[t] - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&c.q_full[t], kTileBytes);
          for (int db = 0; db < 2; ++db)
            tma_load_3d(smem + kQ0 + t * kTileBytes + db * 16384, &tmQ, &c.q_full[t], db * 64, U.g * p.G, M.tok0);
          ++q_iss[t];
        }
        // K/V buffer coordinates of the pair's item: head kvh, key kb at row kb - kshift
        const int kvh = p.units[pr.slot[0]].kvh, kshift = p.units[pr.slot[0]].kshift;
        const int nt_p = kMask ? p.pair_tile_off[u + 1] - p.pair_tile_off[u] : (pr.kend - pr.kbeg + kTileN - 1) / kTileN;
        for (int jt = 0; jt < nt_p && ok; ++jt, ++kv) {
          const int kb = kMask ? p.live_tiles[p.pair_tile_off[u] + jt] : pr.kbeg + jt * kTileN;
          const int st = kv & 1;
          const uint32_t use = kv >> 1;
          if (use >= 1 && !mbar_wait(&c.k_empty[st], (use - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&c.k_full[st], kTileBytes);
          for (int db = 0; db < 2; ++db)
            tma_load_3d(smem + kK0 + st * kTileBytes + db * 16384, &tmK, &c.k_full[st], db * 64, kvh, kb - kshift);
          ++k_iss;
          if (use >= 1 && !mbar_wait(&c.v_empty[st], (use - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&c.v_full[st], kTileBytes);
          for (int db = 0; db < 2; ++db)
            tma_load_3d(smem + kV0 + st * kTileBytes + db * 16384, &tmV, &c.v_full[st], db * 64, kvh, kb - kshift);
          ++v_iss;
        }
        ++n_units;
      }
      // every load this thread issued lands before the CTA can exit
      for (int st = 0; st < 2; ++st) {
        const uint32_t ku = (k_iss + 1 - st) >> 1, vu = (v_iss + 1 - st) >> 1;
        if (ku > 0) mbar_wait(&c.k_full[st], (ku - 1) & 1, nullptr, lim);
        if (vu > 0) mbar_wait(&c.v_full[st], (vu - 1) & 1, nullptr, lim);
      }
      for (int t = 0; t < 2; ++t)
        if (q_iss[t] > 0) mbar_wait(&c.q_full[t], (q_iss[t] - 1) & 1, nullptr, lim);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    {
      // All 32 lanes run the loop (stage indices and counters stay warp-uniform); one elected lane issues
      // the MMAs and their commits.
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);  // S = Q K^T
      constexpr uint32_t idO = idesc_bf16(128, kD, false, true);    // O += P V (P from TMEM)
      const uint64_t dQ0 = sdesc_sw128(smem_u32(smem + kQ0), 16, 1024);
      const uint64_t dK0 = sdesc_sw128(smem_u32(smem + kK0), 16, 1024);
      const uint64_t dV0 = sdesc_sw128(smem_u32(smem + kV0), 16384, 1024);
      constexpr uint64_t kTileDesc = kTileBytes >> 4;
      uint32_t n_units = 0, kv = 0, q_use[2] = {0, 0}, s_cnt[2] = {0, 0}, p_cnt[2] = {0, 0}, pv_cnt[2] = {0, 0},
               unit_cnt[2] = {0, 0};
      bool ok = true;
      // S of tile t for key step with K stage st
      auto issue_s = [&](int t, int st) {
        const uint64_t dq = dQ0 + t * kTileDesc, dk = dK0 + st * kTileDesc;
        if (leader) {
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) umma_bf16(tmem + col_s(t), dq + kmaj(ks), dk + kmaj(ks), idS, ks > 0);
          umma_commit(&c.s_full[t]);
        }
        __syncwarp();
        ++s_cnt[t];
      };
      // O of tile t += P V with V stage st
      auto issue_pv = [&](int t, int st, bool accumulate) {
        const uint64_t dv = dV0 + st * kTileDesc;
        if (leader) {
#pragma unroll
          for (int ks = 0; ks < 128 / 16; ++ks)
            umma_bf16_ts(tmem + col_o(t), tmem + col_s(t) + 8 * ks, dv + ((ks * 2048) >> 4), idO,
                         (accumulate || ks > 0) ? 1u : 0u);
          umma_commit(&c.pv_done[t]);
        }
        __syncwarp();
        ++pv_cnt[t];
      };
      // S of tile t overwrites the P that the tile's last PV read: wait for that PV
      auto wait_pv = [&](int t) -> bool {
        return pv_cnt[t] == 0 || mbar_wait_warp(&c.pv_done[t], (pv_cnt[t] - 1) & 1, status, lim);
      };
      while (ok) {
        const int slot = n_units & 1;
        if (!mbar_wait_warp(&c.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
        const int u = c.sched[slot];
        __syncwarp();
        if (leader) mbar_arrive(&c.sched_empty[slot]);
        if (u < 0) break;
        const FwdPair pr = p.pairs[u];
        const bool has[2] = {pr.slot[0] >= 0, pr.slot[1] >= 0};
        const int nt = kMask ? p.pair_tile_off[u + 1] - p.pair_tile_off[u] : (pr.kend - pr.kbeg + kTileN - 1) / kTileN;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!has[t]) continue;
          if (!mbar_wait_warp(&c.q_full[t], q_use[t] & 1, status, lim)) { ok = false; break; }
        }
        if (!ok) break;
        // key step 0: S of both tiles
        {
          const int st = kv & 1;
          if (!mbar_wait_warp(&c.k_full[st], (kv >> 1) & 1, status, lim)) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (!has[t]) continue;
            if (!wait_pv(t)) { ok = false; break; }
            tc_fence_after();
            issue_s(t, st);
          }
          if (!ok) break;
          if (leader) {
            umma_commit(&c.k_empty[st]);
            if (nt == 1)
              for (int t = 0; t < 2; ++t)
                if (has[t]) umma_commit(&c.q_empty[t]);
          }
          __syncwarp();
        }
        for (int j = 0; j < nt && ok; ++j) {
          const int st = (kv + j) & 1, st1 = (kv + j + 1) & 1;
          const uint32_t use = (kv + j) >> 1, use1 = (kv + j + 1) >> 1;
          if (!mbar_wait_warp(&c.v_full[st], use & 1, status, lim)) { ok = false; break; }
          if (j + 1 < nt && !mbar_wait_warp(&c.k_full[st1], use1 & 1, status, lim)) { ok = false; break; }
          for (int t = 0; t < 2 && ok; ++t) {
            if (!has[t]) continue;
            // O_t += P_t V: P from the tile's softmax warpgroup
            if (!mbar_wait_warp(&c.p_full[t], p_cnt[t] & 1, status, lim)) { ok = false; break; }
            ++p_cnt[t];
            if (j == 0 && unit_cnt[t] >= 1 && !mbar_wait_warp(&c.o_free[t], (unit_cnt[t] - 1) & 1, status, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(t, st, j > 0);
            // next S of this tile once its PV has read P
            if (j + 1 < nt) {
              if (!wait_pv(t)) { ok = false; break; }
              tc_fence_after();
              issue_s(t, st1);
              if (leader && j + 2 == nt) umma_commit(&c.q_empty[t]);
              __syncwarp();
            }
          }
          if (!ok) break;
          if (leader) {
            umma_commit(&c.v_empty[st]);
            if (j + 1 < nt) umma_commit(&c.k_empty[st1]);
          }
          __syncwarp();
        }
        if (!ok) break;
        for (int t = 0; t < 2; ++t)
          if (has[t]) {
            ++q_use[t];
            ++unit_cnt[t];
          }
        kv += nt;
        ++n_units;
      }
      if (leader) umma_commit(&c.final_mma);
      __syncwarp();
      mbar_wait_warp(&c.final_mma, 0, nullptr, lim);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------- softmax + epilogue of tile t
    const int t = (warp - 4) >> 2;                  // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;           // row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + col_s(t), tO = tmem + lane_off + col_o(t);
    const float sl2 = p.scale_log2;
    uint32_t n_units = 0, s_cnt = 0, pv_cnt = 0;
    while (true) {
      const int slot = n_units & 1;
      if (!mbar_wait_warp(&c.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
      const int u = c.sched[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.sched_empty[slot]);
      if (u < 0) break;
      ++n_units;
      const FwdPair pr = p.pairs[u];
      const int nt = kMask ? p.pair_tile_off[u + 1] - p.pair_tile_off[u] : (pr.kend - pr.kbeg + kTileN - 1) / kTileN;
      if (pr.slot[t] < 0) continue;  // odd tile count: this warpgroup sits the pair out
      const int sl = pr.slot[t];
      const FwdUnit U = p.units[sl];
      const MTile M = p.mtiles[U.mt];
      if (p.stamps && r == 0) p.stamps[2 * sl] = static_cast<long long>(globaltimer_ns());
      const int tl = r / p.G;
      const bool valid = tl < M.ntok;
      const int row_end = valid ? min(p.tok_kend[M.tok0 + tl], U.kend) : pr.kbeg;
      float m_ref = -INFINITY, l = 0.f;  // reference maximum (log2 units) and running sum
      bool ok = true;
      for (int j = 0; j < nt; ++j) {
        if (!mbar_wait_warp(&c.s_full[t], s_cnt & 1, status, lim)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        const int kb = kMask ? p.live_tiles[p.pair_tile_off[u] + j] : pr.kbeg + j * kTileN;
        int lim_c = row_end - kb;  // valid columns of this row in the tile
        if (kMask && valid && !((mask_word(p.tile_mask, p.mask_words, M, kb, tl) >> (tl & 31)) & 1u))
          lim_c = 0;  // the row's block is off
        // the whole row of S in registers: four loads in flight, one wait
        uint32_t sv[128];
#pragma unroll
        for (int cc = 0; cc < 128; cc += 32)
          tmem_ld32(tS + cc, *reinterpret_cast<uint32_t(*)[32]>(&sv[cc]));
        tmem_wait_ld();
        if (lim_c < 128) {  // masked keys of this row: -inf
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= lim_c) sv[i] = __float_as_uint(-INFINITY);
        }
        // Lazy reference maximum m_ref (log2 units): it moves only when a tile maximum exceeds it by
        // more than 8, so every P is at most 2^8 and O is rarely rescaled. sl2 > 0, so scaling
        // commutes with the maximum.
        float raw;
        if (j == 0) {
          // first tile of the unit: the reference is this tile's maximum (-inf for a row without keys)
          m_ref = row_max(sv) * sl2;
          l = exp_row<false>(sv, sl2, m_ref == -INFINITY ? 0.f : m_ref, tS, raw);
        } else {
          // later tiles: exponentials against the current reference, the tile maximum alongside;
          // the pass is redone only for a tile whose maximum moves the reference
          const float add = exp_row<true>(sv, sl2, m_ref == -INFINITY ? 0.f : m_ref, tS, raw);
          const float tmax = raw * sl2;
          const bool move = tmax > m_ref + 8.f;
          if (__any_sync(0xffffffffu, move)) {
            const float m_new = move ? tmax : m_ref;
            const float alpha = move ? ex2(m_ref - m_new) : 1.f;  // m_ref = -inf -> 0
            // PV of step j-1 completed before this step's S was issued
#pragma unroll 1
            for (int cc = 0; cc < kD; cc += 32) {
              uint32_t v[32];
              tmem_ld32(tO + cc, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
              tmem_st32(tO + cc, v);
            }
            tmem_wait_st();  // also orders the first pass's P stores before the rewrite
            m_ref = m_new;
            l = l * alpha + exp_row<false>(sv, sl2, m_ref == -INFINITY ? 0.f : m_ref, tS, raw);
          } else {
            l += add;
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&c.p_full[t]);
      }
      if (!ok) break;
      // epilogue: O / l and the natural-log LSE of the partial
      pv_cnt += nt;
      if (!mbar_wait_warp(&c.pv_done[t], (pv_cnt - 1) & 1, status, lim)) break;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      float* orow = p.part_o + (static_cast<size_t>(sl) * kTileM + r) * kD;
      const uint64_t pol = l2_policy_evict_last();
      __nv_bfloat16* orow16 = reinterpret_cast<__nv_bfloat16*>(p.part_o) + (static_cast<size_t>(sl) * kTileM + r) * kD;
#pragma unroll 1
      for (int cc = 0; cc < kD; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tO + cc, v);
        tmem_wait_ld();
        if (p.partial_bf16) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const uint4 w = make_uint4(pack_bf16(__uint_as_float(v[i]) * inv_l, __uint_as_float(v[i + 1]) * inv_l),
                                       pack_bf16(__uint_as_float(v[i + 2]) * inv_l, __uint_as_float(v[i + 3]) * inv_l),
                                       pack_bf16(__uint_as_float(v[i + 4]) * inv_l, __uint_as_float(v[i + 5]) * inv_l),
                                       pack_bf16(__uint_as_float(v[i + 6]) * inv_l, __uint_as_float(v[i + 7]) * inv_l));
            if (p.partials_l2_last)
              st_global_v4u_hint(orow16 + cc + i, w, pol);
            else
              *reinterpret_cast<uint4*>(orow16 + cc + i) = w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 o4 = make_float4(__uint_as_float(v[i]) * inv_l, __uint_as_float(v[i + 1]) * inv_l,
                                          __uint_as_float(v[i + 2]) * inv_l, __uint_as_float(v[i + 3]) * inv_l);
            if (p.partials_l2_last)
              st_global_v4_hint(orow + cc + i, o4, pol);
            else
              *reinterpret_cast<float4*>(orow + cc + i) = o4;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&c.o_free[t]);
      p.part_lse[static_cast<size_t>(sl) * kTileM + r] =
          l > 0.f ? (m_ref + lg2(l)) * 0.69314718055994531f : -INFINITY;
      if constexpr (kMerge) tail_merge_arrive(p, U.mt * p.Hkv + U.g, lane);
      if (p.stamps && r == 0) p.stamps[2 * sl + 1] = static_cast<long long>(globaltimer_ns());
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if constexpr (kMerge) tail_merge<kD>(p, &c.merge_slot);
}

}  // namespace

int fwd2_smem_bytes() { return kSmemBytes; }

cudaError_t launch_fwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                        int grid, cudaStream_t stream) {
  auto kern = p.tile_mask ? (p.o ? fwd2_kernel<true, true> : fwd2_kernel<false, true>)
                          : (p.o ? fwd2_kernel<true, false> : fwd2_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, 384, kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace skv
