// Split-KV forward on sm_100a: for every forward work unit (one item's key
// range x one 128-row query tile of one kv-head group) computes the partial
// attention of the tile's rows over the range and writes the normalized
// partial output (fp32) and its log-sum-exp.
//
// Source: "Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion
// Drafter Training", section "Split-KV's Core Mechanism" (each KV shard's
// local attention is computed for the global query set and aggregated
// through query-sized tensors); "Split-KV: Efficient Context Parallelism for
// Training Diffusion Drafters", Abstract (block-sparse mask over the context,
// exact result).
//
// Structure: persistent CTAs, one per SM; each CTA starts on one virtual
// partition's work queue and moves to the next partition when its own is
// drained. Warp roles:
//   warp 0      scheduler + TMA producer (Q tile, double-buffered K and V)
//   warp 1      tcgen05.mma issuer: S = Q K^T into TMEM (double-buffered),
//               O += P V into TMEM
//   warp 2      TMEM allocator
//   warps 4..7  softmax, O rescale and epilogue; thread = query row
// Masking: row r of the tile sees keys < its anchor end; rows beyond the
// sample's tokens see none. A row with no key in the unit gets LSE = -inf and
// O = 0.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"
#include "tail_merge.cuh"

namespace skv {

template <int D>
struct FwdSmem {
  static constexpr int kQBytes = kTileM * D * 2;   // 128 rows x D bf16
  static constexpr int kKVBytes = kTileN * D * 2;  // 128 keys x D bf16
  static constexpr int kPBytes = kTileM * kTileN * 2;
  static constexpr int kQ = 0;
  static constexpr int kK0 = kQ + kQBytes;
  static constexpr int kV0 = kK0 + 2 * kKVBytes;
  static constexpr int kP = kV0 + 2 * kKVBytes;
  static constexpr int kEnd = kP + kPBytes;
  static constexpr int kDyn = kEnd + 1024;  // slack for 1024-byte alignment
};

struct FwdBarriers {
  uint64_t sched_full[2], sched_empty[2];
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];
  uint64_t p_full, o_done, o_free;
  uint64_t final_mma;
  int32_t sched[2];
  uint32_t tmem_base;
  int32_t merge_slot;  // tail merge: slot being merged (broadcast)
};

// kMerge: the LSE merge runs in the kernel's tail (skv_attn_fwd_merged).
// kMask: a block-sparse mask; every role walks the unit's list of live key
// tiles and the softmax masks the rows whose block is off.
template <int D, bool kMerge, bool kMask>
__global__ void __launch_bounds__(256, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ FwdBarriers bars;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kDBlocks = D / 64;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sched_full[i], 1);
      mbar_init(&bars.sched_empty[i], 5);
      mbar_init(&bars.k_full[i], 1);
      mbar_init(&bars.k_empty[i], 1);
      mbar_init(&bars.v_full[i], 1);
      mbar_init(&bars.v_empty[i], 1);
      mbar_init(&bars.s_full[i], 1);
    }
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.o_done, 1);
    mbar_init(&bars.o_free, 128);
    mbar_init(&bars.final_mma, 1);
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const uint64_t lim = p.timeout_ns;
  int* status = p.status;

  if (warp == 0) {
    // ------------------------------------------------ scheduler + producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int part = static_cast<int>((static_cast<long long>(blockIdx.x) * p.P) / gridDim.x);
      int visited = 0;
      uint32_t n_units = 0, kv = 0, k_issued = 0, v_issued = 0, q_issued = 0;
      bool ok = true;
      while (ok) {
        int u = -1;
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
        const int slot = n_units & 1;
        if (n_units >= 2 && !mbar_wait(&bars.sched_empty[slot], ((n_units >> 1) - 1) & 1, status, lim)) break;
        bars.sched[slot] = u;
        mbar_arrive(&bars.sched_full[slot]);
        if (u < 0) break;
        const FwdUnit U = p.units[u];
        const MTile M = p.mtiles[U.mt];
        if (n_units >= 1 && !mbar_wait(&bars.q_empty, (n_units - 1) & 1, status, lim)) break;
        mbar_arrive_expect_tx(&bars.q_full, L::kQBytes);
        for (int db = 0; db < kDBlocks; ++db)
          tma_load_3d(smem + L::kQ + db * (kTileM * 128), &tmQ, &bars.q_full, db * 64, U.g * p.G, M.tok0);
        ++q_issued;
        const int nt_p = kMask ? p.unit_tile_off[u + 1] - p.unit_tile_off[u] : (U.kend - U.kbeg + kTileN - 1) / kTileN;
        for (int jt = 0; jt < nt_p; ++jt, ++kv) {
          const int kb = kMask ? p.live_tiles[p.unit_tile_off[u] + jt] : U.kbeg + jt * kTileN;
          const int st = kv & 1;
          const uint32_t use = kv >> 1;
          if (use >= 1 && !mbar_wait(&bars.k_empty[st], (use - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.k_full[st], L::kKVBytes);
          for (int db = 0; db < kDBlocks; ++db)
            tma_load_3d(smem + L::kK0 + st * L::kKVBytes + db * (kTileN * 128), &tmK, &bars.k_full[st], db * 64,
                        U.kvh, kb - U.kshift);
          ++k_issued;
          if (use >= 1 && !mbar_wait(&bars.v_empty[st], (use - 1) & 1, status, lim)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.v_full[st], L::kKVBytes);
          for (int db = 0; db < kDBlocks; ++db)
            tma_load_3d(smem + L::kV0 + st * L::kKVBytes + db * (kTileN * 128), &tmV, &bars.v_full[st], db * 64,
                        U.kvh, kb - U.kshift);
          ++v_issued;
        }
        ++n_units;
      }
      // Let every load this thread issued land before the CTA can exit.
      for (int st = 0; st < 2; ++st) {
        const uint32_t ku = (k_issued + 1 - st) >> 1, vu = (v_issued + 1 - st) >> 1;  // loads into stage st
        if (ku > 0) mbar_wait(&bars.k_full[st], (ku - 1) & 1, nullptr, lim);
        if (vu > 0) mbar_wait(&bars.v_full[st], (vu - 1) & 1, nullptr, lim);
      }
      if (q_issued > 0) mbar_wait(&bars.q_full, (q_issued - 1) & 1, nullptr, lim);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // All 32 lanes run the loop (stage indices and descriptors stay warp-uniform); one elected lane issues
    // the MMAs and their commits.
    {
      const bool leader = elect_one();
      constexpr uint32_t idS = idesc_bf16(kTileM, kTileN, false, false);
      constexpr uint32_t idO = idesc_bf16(kTileM, D, false, true);
      // operand descriptors at their buffers' starts; K steps and stages are byte offsets
      const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + L::kQ), 16, 1024);
      const uint64_t dK_k = sdesc_sw128(smem_u32(smem + L::kK0), 16, 1024);
      const uint64_t dP_k = sdesc_sw128(smem_u32(smem + L::kP), 16, 1024);
      const uint64_t dV_mn = sdesc_sw128(smem_u32(smem + L::kV0), kTileN * 128, 1024);
      uint32_t n_units = 0, kv = 0, tcount = 0, pcount = 0;
      bool ok = true;
      while (ok) {
        const int slot = n_units & 1;
        if (!mbar_wait_warp(&bars.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
        const int u = bars.sched[slot];
        __syncwarp();
        if (leader) mbar_arrive(&bars.sched_empty[slot]);
        if (u < 0) break;
        const FwdUnit U = p.units[u];
        const int nt = kMask ? p.unit_tile_off[u + 1] - p.unit_tile_off[u] : (U.kend - U.kbeg + kTileN - 1) / kTileN;
        if (!mbar_wait_warp(&bars.q_full, n_units & 1, status, lim)) break;
        tc_fence_after();
        auto issue_s = [&](uint32_t t_index, uint32_t kv_index) -> bool {
          const int st = kv_index & 1;
          if (!mbar_wait_warp(&bars.k_full[st], (kv_index >> 1) & 1, status, lim)) return false;
          tc_fence_after();
          const uint32_t dS = tmem + ((t_index & 1) ? kColS1 : kColS0);
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t off = (ks >> 2) * (kTileM * 128) + (ks & 3) * 32;
              umma_bf16(dS, sdesc_add(dQ_k, off), sdesc_add(dK_k, st * L::kKVBytes + off), idS, ks > 0);
            }
            umma_commit(&bars.k_empty[st]);
            umma_commit(&bars.s_full[t_index & 1]);
          }
          __syncwarp();
          return true;
        };
        if (!issue_s(tcount, kv)) break;
        for (int j = 0; j < nt && ok; ++j) {
          const uint32_t tj = tcount + j, kvj = kv + j;
          if (j + 1 < nt) {
            if (!issue_s(tj + 1, kvj + 1)) { ok = false; break; }
          }
          if (leader && j + 1 == nt) umma_commit(&bars.q_empty);
          __syncwarp();
          if (!mbar_wait_warp(&bars.p_full, pcount & 1, status, lim)) { ok = false; break; }
          ++pcount;
          const int st = kvj & 1;
          if (!mbar_wait_warp(&bars.v_full[st], (kvj >> 1) & 1, status, lim)) { ok = false; break; }
          if (j == 0 && n_units >= 1 && !mbar_wait_warp(&bars.o_free, (n_units - 1) & 1, status, lim)) { ok = false; break; }
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int ks = 0; ks < kTileN / 16; ++ks) {
              const uint32_t aoff = (ks >> 2) * (kTileM * 128) + (ks & 3) * 32;
              umma_bf16(tmem + kColO, sdesc_add(dP_k, aoff), sdesc_add(dV_mn, st * L::kKVBytes + ks * 2048), idO,
                        (j > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit(&bars.v_empty[st]);
            umma_commit(&bars.o_done);
          }
          __syncwarp();
        }
        tcount += nt;
        kv += nt;
        ++n_units;
      }
      // every MMA issued by this thread completes before TMEM is released
      if (leader) umma_commit(&bars.final_mma);
      __syncwarp();
      mbar_wait_warp(&bars.final_mma, 0, nullptr, lim);
    }
  } else if (warp >= 4) {
    // ------------------------------------------- softmax / correction / epilogue
    const int r = tid - 128;               // row in the tile == TMEM lane
    const int wq = warp - 4;               // TMEM lane quarter of this warp
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    uint8_t* sP = smem + L::kP;
    uint32_t n_units = 0, tcount = 0, pv = 0;
    while (true) {
      const int slot = n_units & 1;
      if (!mbar_wait_warp(&bars.sched_full[slot], (n_units >> 1) & 1, status, lim)) break;
      const int u = bars.sched[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sched_empty[slot]);
      if (u < 0) break;
      const FwdUnit U = p.units[u];
      const MTile M = p.mtiles[U.mt];
      if (p.stamps && r == 0) p.stamps[2 * u] = static_cast<long long>(globaltimer_ns());
      const int tl = r / p.G;
      const bool valid = tl < M.ntok;
      const int row_end = valid ? min(p.tok_kend[M.tok0 + tl], U.kend) : U.kbeg;
      const int nt = kMask ? p.unit_tile_off[u + 1] - p.unit_tile_off[u] : (U.kend - U.kbeg + kTileN - 1) / kTileN;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nt; ++j) {
        const uint32_t tj = tcount + j;
        if (!mbar_wait_warp(&bars.s_full[tj & 1], (tj >> 1) & 1, status, lim)) { ok = false; break; }
        tc_fence_after();
        const int kb = kMask ? p.live_tiles[p.unit_tile_off[u] + j] : U.kbeg + j * kTileN;
        int lim_c = row_end - kb;  // valid columns in this tile
        if (kMask && valid && !((mask_word(p.tile_mask, p.mask_words, M, kb, tl) >> (tl & 31)) & 1u))
          lim_c = 0;  // the row's block is off
        float s[kTileN];
        const uint32_t scol = (tj & 1) ? kColS1 : kColS0;
#pragma unroll
        for (int c = 0; c < kTileN; c += 32) {
          uint32_t v[32];
          tmem_ld32(lane_base + scol + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c + i] = (c + i < lim_c) ? __uint_as_float(v[i]) * p.scale_log2 : -INFINITY;
        }
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < kTileN; ++c) mt = fmaxf(mt, s[c]);
        const float m_new = fmaxf(m, mt);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = ex2(m - m_use);   // m = -inf -> 0
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < kTileN; ++c) {
          s[c] = ex2(s[c] - m_use);
          rs += s[c];
        }
        l = l * alpha + rs;
        // PV of the previous tile must be done before O is rescaled and the P
        // buffer is overwritten.
        if (j > 0) {
          if (!mbar_wait_warp(&bars.o_done, pv & 1, status, lim)) { ok = false; break; }
          ++pv;
          tc_fence_after();
          const bool need = __any_sync(0xffffffffu, alpha != 1.f);
          if (need) {
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t v[32];
              tmem_ld32(lane_base + kColO + c, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
              tmem_st32(lane_base + kColO + c, v);
            }
            tmem_wait_st();
          }
        }
        m = m_new;
        // P (bf16) into the K-major A-operand tile: row r, keys in two 64-key blocks
#pragma unroll
        for (int c8 = 0; c8 < kTileN / 8; ++c8) {
          uint4 w;
          w.x = pack_bf16(s[c8 * 8 + 0], s[c8 * 8 + 1]);
          w.y = pack_bf16(s[c8 * 8 + 2], s[c8 * 8 + 3]);
          w.z = pack_bf16(s[c8 * 8 + 4], s[c8 * 8 + 5]);
          w.w = pack_bf16(s[c8 * 8 + 6], s[c8 * 8 + 7]);
          *reinterpret_cast<uint4*>(sP + (c8 >> 3) * (kTileM * 128) + sw128_off(r, c8 & 7)) = w;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars.p_full);
      }
      if (!ok) break;
      // epilogue: O / l and LSE (natural log) of the partial
      if (!mbar_wait_warp(&bars.o_done, pv & 1, status, lim)) break;
      ++pv;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      float* orow = p.part_o + (static_cast<size_t>(u) * kTileM + r) * D;
      const uint64_t pol = l2_policy_evict_last();
      __nv_bfloat16* orow16 = reinterpret_cast<__nv_bfloat16*>(p.part_o) + (static_cast<size_t>(u) * kTileM + r) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t v[32];
        tmem_ld32(lane_base + kColO + c, v);
        tmem_wait_ld();
        if (p.partial_bf16) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const uint4 w = make_uint4(pack_bf16(__uint_as_float(v[i]) * inv_l, __uint_as_float(v[i + 1]) * inv_l),
                                       pack_bf16(__uint_as_float(v[i + 2]) * inv_l, __uint_as_float(v[i + 3]) * inv_l),
                                       pack_bf16(__uint_as_float(v[i + 4]) * inv_l, __uint_as_float(v[i + 5]) * inv_l),
                                       pack_bf16(__uint_as_float(v[i + 6]) * inv_l, __uint_as_float(v[i + 7]) * inv_l));
            if (p.partials_l2_last)
              st_global_v4u_hint(orow16 + c + i, w, pol);
            else
              *reinterpret_cast<uint4*>(orow16 + c + i) = w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 o4 = make_float4(__uint_as_float(v[i]) * inv_l, __uint_as_float(v[i + 1]) * inv_l,
                                    __uint_as_float(v[i + 2]) * inv_l, __uint_as_float(v[i + 3]) * inv_l);
            if (p.partials_l2_last)
              st_global_v4_hint(orow + c + i, o4, pol);
            else
              *reinterpret_cast<float4*>(orow + c + i) = o4;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.o_free);
      p.part_lse[static_cast<size_t>(u) * kTileM + r] = l > 0.f ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
      if constexpr (kMerge) tail_merge_arrive(p, U.mt * p.Hkv + U.g, lane);
      if (p.stamps && r == 0) p.stamps[2 * u + 1] = static_cast<long long>(globaltimer_ns());
      tcount += nt;
      ++n_units;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if constexpr (kMerge) tail_merge<D>(p, &bars.merge_slot);
}

int fwd_smem_bytes(int d) { return d == 64 ? FwdSmem<64>::kDyn : FwdSmem<128>::kDyn; }

// head_dim 64 runs the one-tile kernel above; head_dim 128 the two-tile kernel of fwd2.cu
cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int grid, cudaStream_t stream) {
  if (d == 128) return launch_fwd2(tq, tk, tv, p, grid, stream);
  auto k = p.tile_mask ? (p.o ? fwd_kernel<64, true, true> : fwd_kernel<64, false, true>)
                       : (p.o ? fwd_kernel<64, true, false> : fwd_kernel<64, false, false>);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdSmem<64>::kDyn);
  if (e != cudaSuccess) return e;
  k<<<grid, 256, FwdSmem<64>::kDyn, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

int fwd_grid(int d, int sms, long long n_units, long long n_pairs) {
  const long long work = d == 128 ? n_pairs : n_units;
  return static_cast<int>(work < sms ? work : sms);
}

}  // namespace skv
