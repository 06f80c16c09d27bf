// Split-KV backward on sm_100a (head_dim 64; head_dim 128 runs the pipelined
// kernel of bwd2.cu).
//
// Gradients through the split ("Split-KV: Breaking the Context Parallelism
// Bottleneck in Diffusion Drafter Training", section "Split-KV's Core
// Mechanism": the split result is strictly consistent with the unsharded
// one, which is what gradient correctness needs). Per backward work unit (a
// tile of <= 128 keys of one item, one kv-head) the kernel loops over the
// live 128-row query tiles of the sample and, with P recomputed from the
// merged LSE:
//   S^T  = K Q^T                 (TMEM, lanes = keys)
//   dP^T = V dO^T                (TMEM)
//   P^T  = exp(S^T / sqrt(d) - LSE),  dS^T = P^T (dP^T - D)   (registers -> smem, bf16)
//   dV  += P^T dO,  dK += dS^T Q (TMEM accumulators for the whole unit)
//   dQ   = dS K                  (TMEM, lanes = rows) -> fp32 reduction into the
//                                 dQ accumulator shared by all items
// dK/dV of the unit's keys are written once, at the end of the unit. The
// 1/sqrt(d) factor of dK is applied there, the one of dQ at the final cast.
//
// Warp roles: warp 0 scheduler + TMA producer, warp 1 MMA issuer, warp 2
// TMEM allocator, warps 4..7 softmax-gradient / dQ drain / dK-dV epilogue
// (thread = TMEM lane).
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace skv {

template <int D>
struct BwdSmem {
  static constexpr int kTile = 128 * D * 2;  // one 128 x D bf16 tile
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;
  static constexpr int kDO = kQ + kTile;
  static constexpr int kPt = kDO + kTile;      // P^T  [128 keys][128 rows] bf16
  static constexpr int kDSt = kPt + 128 * 128 * 2;  // dS^T [128 keys][128 rows] bf16
  static constexpr int kEnd = kDSt + 128 * 128 * 2;
  static constexpr int kDyn = kEnd + 1024;
};

struct BwdShared {
  uint64_t sched_full[2], sched_empty[2];
  uint64_t kv_full, kv_empty, q_full, q_empty;
  uint64_t sdp_full, pds_full, dq_full, dq_free, acc_free;
  uint64_t meta_full[2];  // row metadata of a query tile staged by the 128 softmax threads
  uint64_t final_mma;
  int32_t sched[2];
  uint32_t tmem_base;
  float lse2[2][128];   // log2-domain LSE of the tile rows (+inf for absent rows)
  float delta[2][128];  // D of the tile rows
  int32_t kend[2][128]; // absolute key end of the tile rows
};

// kDet: dQ added in ascending key order under turn counters. kMask: a
// block-sparse mask (rows whose block is off attend no key of the unit); the
// deterministic backward still walks the query tiles the mask turns off, so
// that every unit below a tile's largest anchor takes its turn on that tile.
template <int D, bool kDet, bool kMask>
__global__ void __launch_bounds__(256, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const BwdParams p) {
  using L = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ BwdShared sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kDBlocks = D / 64;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 128, kColDV = 256, kColDK = 256 + D;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.sched_full[i], 1);
      mbar_init(&sh.sched_empty[i], 5);
      mbar_init(&sh.meta_full[i], 128);
    }
    mbar_init(&sh.kv_full, 1);
    mbar_init(&sh.kv_empty, 1);
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, 1);
    mbar_init(&sh.sdp_full, 1);
    mbar_init(&sh.pds_full, 128);
    mbar_init(&sh.dq_full, 1);
    mbar_init(&sh.dq_free, 128);
    mbar_init(&sh.acc_free, 128);
    mbar_init(&sh.final_mma, 1);
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint64_t lim = p.timeout_ns;
  int* status = p.status;

  if (warp == 0) {
    // ------------------------------------------------ scheduler + producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      int part = static_cast<int>((static_cast<long long>(blockIdx.x) * p.P) / gridDim.x);
      int visited = 0;
      uint32_t n_units = 0, qc = 0;
      bool ok = true;
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
        if (n_units >= 2 && !mbar_wait(&sh.sched_empty[slot], ((n_units >> 1) - 1) & 1, status, lim)) break;
        sh.sched[slot] = u;
        mbar_arrive(&sh.sched_full[slot]);
        if (u < 0) break;
        const BwdUnit U = p.units[u];
        if (n_units >= 1 && !mbar_wait(&sh.kv_empty, (n_units - 1) & 1, status, lim)) break;
        mbar_arrive_expect_tx(&sh.kv_full, 2 * L::kTile);
        for (int db = 0; db < kDBlocks; ++db) {
          tma_load_3d(smem + L::kK + db * (128 * 128), &tmK, &sh.kv_full, db * 64, U.kvh, U.kbeg - U.kshift);
          tma_load_3d(smem + L::kV + db * (128 * 128), &tmV, &sh.kv_full, db * 64, U.kvh, U.kbeg - U.kshift);
        }
        ++n_units;
        for (int mt = U.mt_begin; mt < U.mt_end; ++mt) {
          const MTile M = p.mtiles[mt];
          if (!tile_live<kMask && !kDet>(p, M, U.kbeg)) continue;
          if (qc >= 1 && !mbar_wait(&sh.q_empty, (qc - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&sh.q_full, 2 * L::kTile);
          for (int db = 0; db < kDBlocks; ++db) {
            tma_load_3d(smem + L::kQ + db * (128 * 128), &tmQ, &sh.q_full, db * 64, U.g * p.G, M.tok0);
            tma_load_3d(smem + L::kDO + db * (128 * 128), &tmDO, &sh.q_full, db * 64, U.g * p.G, M.tok0);
          }
          ++qc;
        }
      }
      if (n_units > 0) mbar_wait(&sh.kv_full, (n_units - 1) & 1, nullptr, lim);
      if (qc > 0) mbar_wait(&sh.q_full, (qc - 1) & 1, nullptr, lim);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // All 32 lanes run the loop (stage indices and descriptors stay warp-uniform); one elected lane issues
    // the MMAs and their commits.
    {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t idKV = idesc_bf16(128, D, false, true);    // dV, dK
      constexpr uint32_t idQ = idesc_bf16(128, D, true, true);      // dQ
      // operand descriptors at their buffers' starts; K steps are byte offsets
      const uint64_t dK_k = sdesc_sw128(smem_u32(smem + L::kK), 16, 1024);
      const uint64_t dV_k = sdesc_sw128(smem_u32(smem + L::kV), 16, 1024);
      const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
      const uint64_t dDO_k = sdesc_sw128(smem_u32(smem + L::kDO), 16, 1024);
      const uint64_t dPt_k = sdesc_sw128(smem_u32(smem + L::kPt), 16, 1024);
      const uint64_t dDSt_k = sdesc_sw128(smem_u32(smem + L::kDSt), 16, 1024);
      const uint64_t dDO_mn = sdesc_sw128(smem_u32(smem + L::kDO), 128 * 128, 1024);
      const uint64_t dQ_mn = sdesc_sw128(smem_u32(smem + L::kQ), 128 * 128, 1024);
      const uint64_t dDSt_mn = sdesc_sw128(smem_u32(smem + L::kDSt), 128 * 128, 1024);
      const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + L::kK), 128 * 128, 1024);
      uint32_t n_units = 0, qc = 0;
      bool ok = true;
      while (ok) {
        const int slot = n_units & 1;
        if (!mbar_wait_warp(&sh.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
        const int u = sh.sched[slot];
        __syncwarp();
        if (leader) mbar_arrive(&sh.sched_empty[slot]);
        if (u < 0) break;
        const BwdUnit U = p.units[u];
        if (!mbar_wait_warp(&sh.kv_full, n_units & 1, status, lim)) break;
        tc_fence_after();
        bool first = true;
        for (int mt = U.mt_begin; mt < U.mt_end && ok; ++mt) {
          if (!tile_live<kMask && !kDet>(p, p.mtiles[mt], U.kbeg)) continue;
          if (!mbar_wait_warp(&sh.q_full, qc & 1, status, lim)) { ok = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
              umma_bf16(tmem + kColS, sdesc_add(dK_k, off), sdesc_add(dQ_k, off), idS, ks > 0);
            }
          }
          __syncwarp();
          if (qc >= 1 && !mbar_wait_warp(&sh.dq_free, (qc - 1) & 1, status, lim)) { ok = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t off = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
              umma_bf16(tmem + kColDP, sdesc_add(dV_k, off), sdesc_add(dDO_k, off), idS, ks > 0);
            }
            umma_commit(&sh.sdp_full);
          }
          __syncwarp();
          if (!mbar_wait_warp(&sh.pds_full, qc & 1, status, lim)) { ok = false; break; }
          if (first && n_units >= 1 && !mbar_wait_warp(&sh.acc_free, (n_units - 1) & 1, status, lim)) { ok = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks) {  // reduction over the tile rows
              const uint32_t aoff = (ks >> 2) * (128 * 128) + (ks & 3) * 32;
              const uint32_t acc = (!first || ks > 0) ? 1u : 0u;
              umma_bf16(tmem + kColDV, sdesc_add(dPt_k, aoff), sdesc_add(dDO_mn, ks * 2048), idKV, acc);
              umma_bf16(tmem + kColDK, sdesc_add(dDSt_k, aoff), sdesc_add(dQ_mn, ks * 2048), idKV, acc);
            }
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks)  // reduction over the tile keys
              umma_bf16(tmem + kColDQ, sdesc_add(dDSt_mn, ks * 2048), sdesc_add(dK_mn, ks * 2048), idQ, ks > 0);
            umma_commit(&sh.q_empty);
            umma_commit(&sh.dq_full);
          }
          __syncwarp();
          first = false;
          ++qc;
        }
        if (leader) umma_commit(&sh.kv_empty);
        __syncwarp();
        ++n_units;
      }
      if (leader) umma_commit(&sh.final_mma);
      __syncwarp();
      mbar_wait_warp(&sh.final_mma, 0, nullptr, lim);
    }
  } else if (warp >= 4) {
    // ------------------------------- softmax gradient, dQ drain, dK/dV epilogue
    const int t = tid - 128;  // TMEM lane: key for S^T/dP^T/dV/dK, row for dQ
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16);
    uint8_t* sPt = smem + L::kPt;
    uint8_t* sDSt = smem + L::kDSt;
    constexpr float kLog2e = 1.4426950408889634f;
    uint32_t n_units = 0, qc = 0;
    bool ok = true;
    while (ok) {
      const int slot = n_units & 1;
      if (!mbar_wait_warp(&sh.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
      const int u = sh.sched[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sched_empty[slot]);
      if (u < 0) break;
      const BwdUnit U = p.units[u];
      if (p.stamps && t == 0) p.stamps[2 * u] = static_cast<long long>(globaltimer_ns());
      const int nkeys = U.kend - U.kbeg;
      const int my_key = U.kbeg + t;
      const bool key_ok = t < nkeys;
      bool had_tiles = false;
      for (int mt = U.mt_begin; mt < U.mt_end; ++mt) {
        const MTile M = p.mtiles[mt];
        if (!tile_live<kMask && !kDet>(p, M, U.kbeg)) continue;
        had_tiles = true;
        const int b2 = qc & 1;
        const int tl = t / p.G;
        const bool row_ok = tl < M.ntok;
        const int token = M.tok0 + tl;
        const int h = U.g * p.G + t % p.G;
        sh.lse2[b2][t] = row_ok ? p.lse[static_cast<size_t>(token) * p.Hq + h] * kLog2e : INFINITY;
        sh.delta[b2][t] = row_ok ? p.delta[static_cast<size_t>(token) * p.Hq + h] : 0.f;
        const bool row_on =
            row_ok && (!kMask || ((mask_word(p.tile_mask, p.mask_words, M, U.kbeg, tl) >> (tl & 31)) & 1u));
        sh.kend[b2][t] = row_on ? p.tok_kend[token] : -1;
        mbar_arrive(&sh.meta_full[b2]);
        if (!mbar_wait_warp(&sh.meta_full[b2], (qc >> 1) & 1, status, lim)) { ok = false; break; }
        if (!mbar_wait_warp(&sh.sdp_full, qc & 1, status, lim)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t vs[32], vd[32];
          tmem_ld32(lane_base + kColS + c, vs);
          tmem_ld32(lane_base + kColDP + c, vd);
          tmem_wait_ld();
          float pr[32], ds[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int r = c + i;
            const bool live = key_ok && my_key < sh.kend[b2][r];
            const float pv = live ? ex2(__uint_as_float(vs[i]) * p.scale_log2 - sh.lse2[b2][r]) : 0.f;
            pr[i] = pv;
            ds[i] = pv * (__uint_as_float(vd[i]) - sh.delta[b2][r]);
          }
          // rows c..c+31 of key t: block c / 64, 16-byte chunks (c % 64) / 8 + 0..3
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t off = (c >> 6) * (128 * 128) + sw128_off(t, ((c & 63) >> 3) + q);
            uint4 wp, wd;
            wp.x = pack_bf16(pr[8 * q + 0], pr[8 * q + 1]);
            wp.y = pack_bf16(pr[8 * q + 2], pr[8 * q + 3]);
            wp.z = pack_bf16(pr[8 * q + 4], pr[8 * q + 5]);
            wp.w = pack_bf16(pr[8 * q + 6], pr[8 * q + 7]);
            wd.x = pack_bf16(ds[8 * q + 0], ds[8 * q + 1]);
            wd.y = pack_bf16(ds[8 * q + 2], ds[8 * q + 3]);
            wd.z = pack_bf16(ds[8 * q + 4], ds[8 * q + 5]);
            wd.w = pack_bf16(ds[8 * q + 6], ds[8 * q + 7]);
            *reinterpret_cast<uint4*>(sPt + off) = wp;
            *reinterpret_cast<uint4*>(sDSt + off) = wd;
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.pds_full);
        // dQ of this query tile: lane t = row t
        if (!mbar_wait_warp(&sh.dq_full, qc & 1, status, lim)) { ok = false; break; }
        tc_fence_after();
        float* dst = p.dq_acc + (static_cast<size_t>(token) * p.Hq + h) * D;
        // deterministic mode: this warp's 32 rows are added after every lower-ranked unit of the sample and
        // kv head has added its own (ascending key order); the turn fixes the order in which the fp32
        // reductions reach each address
        int32_t* turn = kDet ? p.turn + (static_cast<size_t>(mt) * p.Hkv + U.g) * 8 + (warp & 3) : nullptr;
        const bool my_turn = kDet && turn_wait(turn, p.rank[u], status, lim, lane);
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t v[32];
          tmem_ld32(lane_base + kColDQ + c, v);
          tmem_wait_ld();
          if (row_ok && (!kDet || my_turn)) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              atomicAdd(reinterpret_cast<float4*>(dst + c + i),
                        make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                                    __uint_as_float(v[i + 3])));
          }
        }
        if (kDet && my_turn) turn_pass(turn, p.rank[u] + 1, lane);
        tc_fence_before();
        mbar_arrive(&sh.dq_free);
        ++qc;
      }
      if (!ok) break;
      // dK, dV of the unit's keys (every MMA of the unit completed: dq_full above)
      tc_fence_after();
      const size_t krow = (static_cast<size_t>(my_key - U.kshift) * p.kv_heads + U.kvh) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t vv[32], vk[32];
        tmem_ld32(lane_base + kColDV + c, vv);
        tmem_ld32(lane_base + kColDK + c, vk);
        tmem_wait_ld();
        if (!had_tiles) {  // no query tile attends the unit's keys (a block mask): their gradients are zero
#pragma unroll
          for (int i = 0; i < 32; ++i) vv[i] = vk[i] = 0u;
        }
        if (key_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 a, b;
            a.x = pack_bf16(__uint_as_float(vv[i]), __uint_as_float(vv[i + 1]));
            a.y = pack_bf16(__uint_as_float(vv[i + 2]), __uint_as_float(vv[i + 3]));
            a.z = pack_bf16(__uint_as_float(vv[i + 4]), __uint_as_float(vv[i + 5]));
            a.w = pack_bf16(__uint_as_float(vv[i + 6]), __uint_as_float(vv[i + 7]));
            b.x = pack_bf16(__uint_as_float(vk[i]) * p.scale, __uint_as_float(vk[i + 1]) * p.scale);
            b.y = pack_bf16(__uint_as_float(vk[i + 2]) * p.scale, __uint_as_float(vk[i + 3]) * p.scale);
            b.z = pack_bf16(__uint_as_float(vk[i + 4]) * p.scale, __uint_as_float(vk[i + 5]) * p.scale);
            b.w = pack_bf16(__uint_as_float(vk[i + 6]) * p.scale, __uint_as_float(vk[i + 7]) * p.scale);
            *reinterpret_cast<uint4*>(p.dv + krow + c + i) = a;
            *reinterpret_cast<uint4*>(p.dk + krow + c + i) = b;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.acc_free);
      if (p.stamps && t == 0) p.stamps[2 * u + 1] = static_cast<long long>(globaltimer_ns());
      ++n_units;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}


cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdParams& p, int grid, cudaStream_t stream) {
  if (d == 128) return launch_bwd2(tq, tk, tv, tdo, p, grid, stream);
  const bool m = p.tile_mask != nullptr;
  auto k = p.det ? (m ? bwd_kernel<64, true, true> : bwd_kernel<64, true, false>)
                 : (m ? bwd_kernel<64, false, true> : bwd_kernel<64, false, false>);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdSmem<64>::kDyn);
  if (e != cudaSuccess) return e;
  k<<<grid, 256, BwdSmem<64>::kDyn, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

}  // namespace skv
