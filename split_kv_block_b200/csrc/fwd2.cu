// Split-KV forward on sm_100a (head_dim 64 and 128): two query tiles per CTA,
// scores in 64-key sub-tiles with two score buffers per query tile.
//
// Per forward unit: the partial softmax attention of one 128-row query tile
// over one item's key range, its normalized partial output and log-sum-exp
// ("Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion
// Drafter Training", section "Split-KV's Core Mechanism"; the masking rules
// are stated in fwd.cu), arranged so that the tensor core does not wait for
// the softmax:
//   * a work unit is a pair of forward units of the same item; every 128-key
//     K/V tile loaded by TMA serves both query tiles;
//   * scores come in sub-tiles of 64 keys (S = Q K^T with N = 64). Each query
//     tile has two 64-column score buffers in TMEM and its O (D columns).
//     P overwrites the first 32 columns of its buffer (bf16 pairs) and feeds
//     O += P V from TMEM. While the softmax works on one buffer, the next
//     sub-tile's S is computed into the other, so a tile's softmax runs from
//     sub-tile to sub-tile without waiting for its own PV and S MMAs;
//   * one MMA-issuing warp per query tile (warps 1 and 3). Each runs its
//     tile's fixed sequence S(0), S(1), PV(0), S(2), PV(1), S(3), ... with
//     blocking waits, and the tensor core interleaves the two streams;
//   * lazy rescaling: a row's reference maximum moves only when a sub-tile
//     maximum exceeds it by more than 8 (log2 units), so every P is at most
//     2^8 and O is rarely touched; the final normalization uses the same
//     reference, so the result is exact.
// Warp roles: 0 scheduler + TMA producer, 1 and 3 MMA issuers of tiles 0 and
// 1, 2 TMEM allocator, 4..7 softmax of tile 0, 8..11 softmax of tile 1.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"
#include "tail_merge.cuh"

namespace skv {
namespace {

constexpr int kSub = 64;  // keys per score sub-tile

struct Ctl {
  uint64_t sched_full[2], sched_empty[2];
  uint64_t q_full[2], q_empty[2];  // per query tile
  uint64_t k_full[2], k_empty[2];  // per K stage (two issuers release it)
  uint64_t v_full[2], v_empty[2];  // per V stage (two issuers release it)
  uint64_t s_full[2][2];           // [tile][buffer]: S sub-tile in TMEM
  uint64_t p_full[2][2];           // [tile][buffer]: P in TMEM (128 arrivals)
  uint64_t pv_done[2][2];          // [tile][buffer]: O += P V from this buffer completed
  uint64_t o_free[2];              // per query tile: epilogue has read O (128 arrivals)
  uint64_t final_mma[2];
  int32_t sched[2];
  uint32_t tmem_base;
  int32_t merge_slot;  // tail merge: slot being merged (broadcast)
};
// Shared memory of the head_dim-D kernel: Q of both query tiles, two K and two V stages. A tile is 128
// rows of D bf16, stored as D / 64 column groups of 128 rows x 128 bytes (one 128-byte swizzle atom per
// row), 16 KB each.
template <int D>
struct FwdLayout {
  static constexpr int kHalves = D / 64;              // 64-column groups of a row
  static constexpr int kTileBytes = 128 * D * 2;      // a 128 x D bf16 tile
  static constexpr int kQ0 = 0;                       // Q of tile 0 and tile 1
  static constexpr int kK0 = kQ0 + 2 * kTileBytes;    // two K stages
  static constexpr int kV0 = kK0 + 2 * kTileBytes;    // two V stages
  static constexpr int kCtl = kV0 + 2 * kTileBytes;
  static constexpr int kSmemBytes = kCtl + static_cast<int>(sizeof(Ctl));
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t col_s(int t, int b) { return 128u * t + 64u * b; }  // score buffer b of tile t
__device__ __forceinline__ uint32_t col_o(int t) { return 256u + 128u * t; }            // O of tile t

// descriptor offset (16-byte units) of K-step ks inside a K-major SW128 tile of 128 rows
__device__ __forceinline__ uint64_t kmaj(int ks) {
  return static_cast<uint64_t>(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
}

// Maximum of a 64-column score row: four independent three-input chains.
__device__ __forceinline__ float row_max64(const uint32_t (&sv)[64]) {
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < 64; i += 2) mx[(i >> 1) & 3] = fmax3(mx[(i >> 1) & 3], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
  return fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
}

// P = 2^(s sl2 - m_use) over one 64-column score row (masked entries are -inf -> 0), stored as bf16
// pairs into the first 32 TMEM columns at tS; returns the row sum. With kMax it also returns, in
// raw_max, the maximum of the raw scores (three-input maxima on the ALU pipe beside the exponentials).
template <bool kMax>
__device__ __forceinline__ float exp_row64(const uint32_t (&sv)[64], float sl2, float m_use, uint32_t tS,
                                           float& raw_max) {
  float rs[4] = {0.f, 0.f, 0.f, 0.f};
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int cc = 0; cc < 64; cc += 32) {
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

// kMerge: the LSE merge runs in the kernel's tail (skv_attn_fwd_merged). kMask: a block-sparse mask;
// every role walks the pair's list of live key tiles and the softmax masks the rows whose block is off.
template <int D, bool kMerge, bool kMask>
__global__ void __launch_bounds__(384, 1)
    fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr int kD = D, kTileBytes = L::kTileBytes, kQ0 = L::kQ0, kK0 = L::kK0, kV0 = L::kV0;
  extern __shared__ __align__(1024) uint8_t smem[];
  Ctl& c = *reinterpret_cast<Ctl*>(smem + L::kCtl);
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
      mbar_init(&c.sched_empty[i], 2 + 8);  // both issuers and the eight softmax warps
      mbar_init(&c.q_full[i], 1);
      mbar_init(&c.q_empty[i], 1);
      mbar_init(&c.k_full[i], 1);
      mbar_init(&c.k_empty[i], 2);
      mbar_init(&c.v_full[i], 1);
      mbar_init(&c.v_empty[i], 2);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&c.s_full[i][b], 1);
        mbar_init(&c.p_full[i][b], 128);
        mbar_init(&c.pv_done[i][b], 1);
      }
      mbar_init(&c.o_free[i], 128);
      mbar_init(&c.final_mma[i], 1);
    }
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
          for (int db = 0; db < L::kHalves; ++db)
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
          for (int db = 0; db < L::kHalves; ++db)
            tma_load_3d(smem + kK0 + st * kTileBytes + db * 16384, &tmK, &c.k_full[st], db * 64, kvh, kb - kshift);
          ++k_iss;
          if (use >= 1 && !mbar_wait(&c.v_empty[st], (use - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&c.v_full[st], kTileBytes);
          for (int db = 0; db < L::kHalves; ++db)
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
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------ MMA issuer of query tile t
    // All 32 lanes run the loop (counters stay warp-uniform); one elected lane issues the MMAs and commits.
    const int t = warp == 1 ? 0 : 1;
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16(128, kSub, false, false);  // S = Q K^T over 64 keys
    constexpr uint32_t idO = idesc_bf16(128, kD, false, true);     // O += P V (P from TMEM)
    constexpr uint64_t kTileDesc = kTileBytes >> 4;
    const uint64_t dQ = sdesc_sw128(smem_u32(smem + kQ0), 16, 1024) + t * kTileDesc;
    const uint64_t dK0 = sdesc_sw128(smem_u32(smem + kK0), 16, 1024);
    const uint64_t dV0 = sdesc_sw128(smem_u32(smem + kV0), 16384, 1024);
    // Phase parities (bit b: buffer b) and whether buffer b has held a PV yet. Bit fields, not arrays, so
    // that nothing indexed by the buffer number leaves registers.
    uint32_t p_par = 0, pv_par = 0, pv_any = 0;
    uint32_t n_units = 0, kv = 0, q_use = 0, unit_cnt = 0;
    bool ok = true;
    // K (or V) stage of the unit's key tile j is released by both issuers; an issuer whose partner tile
    // is absent from the pair arrives for it as well (the phase still completes only after its MMAs).
    auto release = [&](uint64_t* bar, bool solo) {
      if (leader) {
        umma_commit(bar);
        if (solo) mbar_arrive(bar);
      }
    };
    while (ok) {
      const int slot = n_units & 1;
      if (!mbar_wait_warp(&c.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
      const int u = c.sched[slot];
      __syncwarp();
      if (leader) mbar_arrive(&c.sched_empty[slot]);
      if (u < 0) break;
      const FwdPair pr = p.pairs[u];
      const int nt = kMask ? p.pair_tile_off[u + 1] - p.pair_tile_off[u] : (pr.kend - pr.kbeg + kTileN - 1) / kTileN;
      ++n_units;
      if (pr.slot[t] < 0) {  // odd tile count: the partner issuer releases K and V alone
        kv += nt;
        continue;
      }
      const bool solo = pr.slot[1 - t] < 0;
      // sub-tiles: two per key tile, the last key tile's second one dropped when no key of the pair reaches it
      const int ns = kMask ? 2 * nt : (pr.kend - pr.kbeg + kSub - 1) / kSub;
      if (!mbar_wait_warp(&c.q_full[t], q_use & 1, status, lim)) break;
      // S of sub-tile s into buffer s & 1 (its previous PV has completed)
      auto issue_s = [&](int s) -> bool {
        const int b = s & 1, j = s >> 1;
        const uint32_t kt = kv + j;
        if (((pv_any >> b) & 1) && !mbar_wait_warp(&c.pv_done[t][b], ((pv_par >> b) & 1) ^ 1, status, lim))
          return false;
        if (b == 0 && !mbar_wait_warp(&c.k_full[kt & 1], (kt >> 1) & 1, status, lim)) return false;
        tc_fence_after();
        if (leader) {
          const uint64_t dk = dK0 + (kt & 1) * kTileDesc + static_cast<uint64_t>(b * (kSub * 128 >> 4));
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) umma_bf16(tmem + col_s(t, b), dQ + kmaj(ks), dk + kmaj(ks), idS, ks > 0);
          umma_commit(&c.s_full[t][b]);
          if (s + 1 == ns) umma_commit(&c.q_empty[t]);
        }
        __syncwarp();
        if (b == 1 || s + 1 == ns) release(&c.k_empty[kt & 1], solo);  // last sub-tile reading this K tile
        __syncwarp();
        return true;
      };
      for (int s = 0; s < 2 && s < ns && ok; ++s) ok = issue_s(s);
      for (int s = 0; s < ns && ok; ++s) {
        const int b = s & 1, j = s >> 1;
        const uint32_t vt = kv + j;
        // O += P V once the softmax has written P of sub-tile s
        if (!mbar_wait_warp(&c.p_full[t][b], (p_par >> b) & 1, status, lim)) { ok = false; break; }
        p_par ^= 1u << b;
        if (s == 0 && unit_cnt >= 1 && !mbar_wait_warp(&c.o_free[t], (unit_cnt - 1) & 1, status, lim)) {
          ok = false;
          break;
        }
        if (b == 0 && !mbar_wait_warp(&c.v_full[vt & 1], (vt >> 1) & 1, status, lim)) { ok = false; break; }
        tc_fence_after();
        if (leader) {
          const uint64_t dv = dV0 + (vt & 1) * kTileDesc;
#pragma unroll
          for (int kk = 0; kk < kSub / 16; ++kk)
            umma_bf16_ts(tmem + col_o(t), tmem + col_s(t, b) + 8 * kk, dv + (((4 * b + kk) * 2048) >> 4), idO,
                         (s > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&c.pv_done[t][b]);
        }
        __syncwarp();
        pv_par ^= 1u << b;
        pv_any |= 1u << b;
        if (b == 1 || s + 1 == ns) release(&c.v_empty[vt & 1], solo);  // last sub-tile reading this V tile
        __syncwarp();
        // the next S into this buffer
        if (s + 2 < ns) ok = issue_s(s + 2);
      }
      if (!ok) break;
      // the partner's half of the releases when the partner tile is absent is done above (solo)
      kv += nt;
      ++q_use;
      ++unit_cnt;
    }
    if (leader) umma_commit(&c.final_mma[t]);
    __syncwarp();
    mbar_wait_warp(&c.final_mma[t], 0, nullptr, lim);
  } else if (warp >= 4) {
    // ---------------------------------------------- softmax + epilogue of tile t
    const int t = (warp - 4) >> 2;         // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS0 = tmem + lane_off + col_s(t, 0), tO = tmem + lane_off + col_o(t);
    const float sl2 = p.scale_log2;
    uint32_t n_units = 0, s_par = 0, pv_par = 0;  // bit b: phase parity of buffer b
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
      const int ns = kMask ? 2 * nt : (pr.kend - pr.kbeg + kSub - 1) / kSub;
      const int sl = pr.slot[t];
      const FwdUnit U = p.units[sl];
      const MTile M = p.mtiles[U.mt];
      if (p.stamps && r == 0) p.stamps[2 * sl] = static_cast<long long>(globaltimer_ns());
      const int tl = r / p.G;
      const bool valid = tl < M.ntok;
      const int row_end = valid ? min(p.tok_kend[M.tok0 + tl], U.kend) : pr.kbeg;
      float m_ref = -INFINITY, l = 0.f;  // reference maximum (log2 units) and running sum
      bool ok = true;
      for (int s = 0; s < ns; ++s) {
        const int b = s & 1;
        const uint32_t tS = tS0 + 64u * b;
        if (!mbar_wait_warp(&c.s_full[t][b], (s_par >> b) & 1, status, lim)) { ok = false; break; }
        s_par ^= 1u << b;
        tc_fence_after();
        const int kt = kMask ? p.live_tiles[p.pair_tile_off[u] + (s >> 1)] : pr.kbeg + (s >> 1) * kTileN;
        int lim_c = row_end - (kt + b * kSub);  // valid columns of this row in the sub-tile
        if (kMask && valid && !((mask_word(p.tile_mask, p.mask_words, M, kt, tl) >> (tl & 31)) & 1u))
          lim_c = 0;  // the row's block is off
        uint32_t sv[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        if (lim_c < 64) {  // masked keys of this row: -inf
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= lim_c) sv[i] = __float_as_uint(-INFINITY);
        }
        float raw;
        if (s == 0) {
          // first sub-tile of the unit: the reference is its maximum (-inf for a row without keys)
          m_ref = row_max64(sv) * sl2;
          l = exp_row64<false>(sv, sl2, m_ref == -INFINITY ? 0.f : m_ref, tS, raw);
        } else {
          const float add = exp_row64<true>(sv, sl2, m_ref == -INFINITY ? 0.f : m_ref, tS, raw);
          const float tmax = raw * sl2;
          const bool move = tmax > m_ref + 8.f;
          if (__any_sync(0xffffffffu, move)) {
            const float m_new = move ? tmax : m_ref;
            const float alpha = move ? ex2(m_ref - m_new) : 1.f;  // m_ref = -inf -> 0
            // O may still be accumulating the previous sub-tile's PV: wait for it (no later PV can start
            // before this sub-tile's P is written)
            const int pb = b ^ 1;
            if (!mbar_wait_warp(&c.pv_done[t][pb], ((pv_par >> pb) & 1) ^ 1, status, lim)) { ok = false; break; }
            tc_fence_after();
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
            l = l * alpha + exp_row64<false>(sv, sl2, m_ref == -INFINITY ? 0.f : m_ref, tS, raw);
          } else {
            l += add;
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&c.p_full[t][b]);
        pv_par ^= 1u << b;  // the PV of this P is the next completion of buffer b's pv_done
      }
      if (!ok) break;
      // epilogue: O / l and the natural-log LSE of the partial. The last PV's completion covers every
      // earlier one (same accumulator, issued in order by one thread).
      const int lb = (ns - 1) & 1;
      if (!mbar_wait_warp(&c.pv_done[t][lb], ((pv_par >> lb) & 1) ^ 1, status, lim)) break;
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

template <int D>
cudaError_t launch_fwd2_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                          int grid, cudaStream_t stream) {
  auto kern = p.tile_mask ? (p.o ? fwd2_kernel<D, true, true> : fwd2_kernel<D, false, true>)
                          : (p.o ? fwd2_kernel<D, true, false> : fwd2_kernel<D, false, false>);
  constexpr int smem = FwdLayout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 384, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_fwd2(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const FwdParams& p, int grid, cudaStream_t stream) {
  return d == 64 ? launch_fwd2_d<64>(tq, tk, tv, p, grid, stream) : launch_fwd2_d<128>(tq, tk, tv, p, grid, stream);
}

}  // namespace skv
