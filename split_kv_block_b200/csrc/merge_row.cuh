// The exact log-sum-exp merge of one query row, shared by the standalone
// merge kernel and the merge that runs in the forward kernel's tail.
//
// Source: "Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion
// Drafter Training", section "Split-KV's Core Mechanism" (the partial results
// of every KV shard are combined through query-sized tensors) and
// "Split-KV: Efficient Context Parallelism for Training Diffusion Drafters",
// Abstract (exact). For one (query tile, kv head, row), over the tile's
// partials c in ascending key order:
//   m = max_c LSE_c, den = sum_c exp(LSE_c - m),
//   O = sum_c exp(LSE_c - m) O_c / den, LSE = m + ln den.
// Partials with LSE_c = -inf weigh 0. One warp per row: lane i owns d/32
// consecutive elements, so every partial row is read as whole 128-byte lines.
// Partials are read through L2 only (ld.global.cg): in the forward's tail
// other SMs of the same launch wrote them.
#pragma once
#include <cuda_bf16.h>

#include "plan_layout.h"
#include "sm100.cuh"

namespace skv {

template <int D>
struct MergeVec;
template <>
struct MergeVec<128> {
  static constexpr int N = 4;
};
template <>
struct MergeVec<64> {
  static constexpr int N = 2;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// A partial row is read once and is dead afterwards: it is loaded with the
// L2 evict_first policy, so it leaves L2 before data that is still needed.
// kB16: the partial outputs are stored as bf16 (row of D elements, 2 bytes
// each), otherwise as fp32.
template <int D, bool kB16>
__device__ __forceinline__ void merge_load_row(const float* part_o, size_t row, int lane,
                                               float (&x)[MergeVec<D>::N], uint64_t pol) {
  if constexpr (kB16) {
    const auto* src = reinterpret_cast<const __nv_bfloat16*>(part_o) + row * D;
    if constexpr (D == 128) {
      const uint2 t = ld_cg_u2_hint(src + lane * 4, pol);
      x[0] = bf16_lo(t.x); x[1] = bf16_hi(t.x); x[2] = bf16_lo(t.y); x[3] = bf16_hi(t.y);
    } else {
      const uint32_t t = ld_cg_u1_hint(src + lane * 2, pol);
      x[0] = bf16_lo(t); x[1] = bf16_hi(t);
    }
  } else {
    const float* src = part_o + row * D;
    if constexpr (D == 128) {
      const float4 t = ld_cg_v4_hint(src + lane * 4, pol);
      x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
      const float2 t = ld_cg_v2_hint(src + lane * 2, pol);
      x[0] = t.x; x[1] = t.y;
    }
  }
}

template <int D>
__device__ __forceinline__ void merge_store_row(__nv_bfloat16* dst, int lane, const float (&x)[MergeVec<D>::N]) {
  if constexpr (D == 128) {
    uint2 t;
    t.x = pack_bf16(x[0], x[1]);
    t.y = pack_bf16(x[2], x[3]);
    *reinterpret_cast<uint2*>(dst + lane * 4) = t;
  } else {
    *reinterpret_cast<uint32_t*>(dst + lane * 2) = pack_bf16(x[0], x[1]);
  }
}

// Merges row r of slot (query tile mt, kv head g) = mt * Hkv + g; the whole
// warp calls it. Rows past the tile's tokens are skipped.
template <int D, bool kB16>
__device__ __forceinline__ void merge_row(const MTile& M, int g, int r, int lane, int G, int Hq, int c0, int c1,
                                          const int32_t* __restrict__ merge_list, const float* part_o,
                                          const float* part_lse, __nv_bfloat16* o, float* lse) {
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.69314718055994531f;
  const int tl = r / G;
  if (tl >= M.ntok) return;
  const int token = M.tok0 + tl;
  const int h = g * G + r % G;
  // The lanes fetch the partials' indices and LSEs in parallel (lane i: partials c0 + i, c0 + i + 32, ...),
  // so the only per-partial memory traffic left in the accumulation loop is the partial output row.
  float m = -INFINITY;
  for (int c = c0 + lane; c < c1; c += 32)
    m = fmaxf(m, __ldcg(part_lse + static_cast<size_t>(merge_list[c]) * kTileM + r));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[MergeVec<D>::N] = {};
  float den = 0.f;
  const uint64_t pol = l2_policy_evict_first();
  if (m != -INFINITY) {
    for (int base = c0; base < c1; base += 32) {
      const int cnt = min(32, c1 - base);
      int my_u = 0;
      float my_w = 0.f;  // weight exp(LSE_c - m); 0 for a dead partial (LSE = -inf)
      if (lane < cnt) {
        my_u = merge_list[base + lane];
        my_w = ex2((__ldcg(part_lse + static_cast<size_t>(my_u) * kTileM + r) - m) * kLog2e);
      }
      float ws = my_w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
      den += ws;
      // ascending key order; eight independent row loads in flight per step (the additions stay in
      // sequence, one partial after the other)
      for (int j = 0; j < cnt; j += 8) {
        float x[8][MergeVec<D>::N];
        float w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int uk = __shfl_sync(0xffffffffu, my_u, (j + k) & 31);
          w[k] = __shfl_sync(0xffffffffu, my_w, (j + k) & 31);
          if (j + k < cnt && w[k] != 0.f) {
            merge_load_row<D, kB16>(part_o, static_cast<size_t>(uk) * kTileM + r, lane, x[k], pol);
          } else {
            w[k] = 0.f;
#pragma unroll
            for (int i = 0; i < MergeVec<D>::N; ++i) x[k][i] = 0.f;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
          for (int i = 0; i < MergeVec<D>::N; ++i) acc[i] += w[k] * x[k][i];
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int i = 0; i < MergeVec<D>::N; ++i) acc[i] *= inv;
  merge_store_row<D>(o + (static_cast<size_t>(token) * Hq + h) * D, lane, acc);
  if (lane == 0) lse[static_cast<size_t>(token) * Hq + h] = den > 0.f ? m + lg2(den) * kLn2 : -INFINITY;
}

}  // namespace skv
