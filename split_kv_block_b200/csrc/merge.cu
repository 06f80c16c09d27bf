// Memory-bound kernels around the split-KV attention:
//   * the exact log-sum-exp merge of per-chunk partials ("Split-KV's Core
//     Mechanism": partial results of every KV shard aggregated through
//     query-sized tensors; exact, per the Abstract);
//   * the backward preprocess D = rowsum(dO * O) with the zeroing of the fp32
//     dQ accumulator;
//   * the final dQ rounding to bf16 (the sum over chunks happened in fp32).
// One warp per (query token, head) row, each lane owning d/32 consecutive
// elements so every row is read and written as whole 128-byte lines.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace skv {

namespace {

template <int D>
struct Vec;
template <>
struct Vec<128> {
  static constexpr int N = 4;
};
template <>
struct Vec<64> {
  static constexpr int N = 2;
};

template <int D>
__device__ __forceinline__ void load_row(const float* src, int lane, float (&x)[Vec<D>::N]) {
  if constexpr (D == 128) {
    float4 t = *reinterpret_cast<const float4*>(src + lane * 4);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  } else {
    float2 t = *reinterpret_cast<const float2*>(src + lane * 2);
    x[0] = t.x; x[1] = t.y;
  }
}

template <int D>
__device__ __forceinline__ void load_row_bf16(const __nv_bfloat16* src, int lane, float (&x)[Vec<D>::N]) {
  if constexpr (D == 128) {
    uint2 t = *reinterpret_cast<const uint2*>(src + lane * 4);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&t.x), b = *reinterpret_cast<__nv_bfloat162*>(&t.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
  } else {
    uint32_t t = *reinterpret_cast<const uint32_t*>(src + lane * 2);
    float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&t));
    x[0] = fa.x; x[1] = fa.y;
  }
}

template <int D>
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, int lane, const float (&x)[Vec<D>::N]) {
  if constexpr (D == 128) {
    uint2 t;
    t.x = pack_bf16(x[0], x[1]);
    t.y = pack_bf16(x[2], x[3]);
    *reinterpret_cast<uint2*>(dst + lane * 4) = t;
  } else {
    *reinterpret_cast<uint32_t*>(dst + lane * 2) = pack_bf16(x[0], x[1]);
  }
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

// Per (query tile, kv head, row): m = max LSE_c, LSE = m + ln sum exp(LSE_c - m),
// O = sum exp(LSE_c - LSE) O_c over the tile's partials in ascending key order.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.n_rows) return;
  const int r = static_cast<int>(row % kTileM);
  const long long slot = row / kTileM;  // mt * Hkv + g
  const int g = static_cast<int>(slot % p.Hkv);
  const int mt = static_cast<int>(slot / p.Hkv);
  const MTile M = p.mtiles[mt];
  const int tl = r / p.G;
  if (tl >= M.ntok) return;
  const int token = M.tok0 + tl;
  const int h = g * p.G + r % p.G;
  const int c0 = p.merge_off[slot], c1 = p.merge_off[slot + 1];
  // The lanes fetch the partials' indices and LSEs in parallel (lane i: partials c0 + i, c0 + i + 32, ...),
  // so the only per-partial memory traffic left in the accumulation loop is the partial output row.
  float m = -INFINITY;
  for (int c = c0 + lane; c < c1; c += 32) m = fmaxf(m, p.part_lse[static_cast<size_t>(p.merge_list[c]) * kTileM + r]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[Vec<D>::N] = {};
  float den = 0.f;
  if (m != -INFINITY) {
    for (int base = c0; base < c1; base += 32) {
      const int cnt = min(32, c1 - base);
      int my_u = 0;
      float my_w = 0.f;  // weight exp(LSE_c - m); 0 for a dead partial (LSE = -inf)
      if (lane < cnt) {
        my_u = p.merge_list[base + lane];
        my_w = ex2((p.part_lse[static_cast<size_t>(my_u) * kTileM + r] - m) * kLog2e);
      }
      float ws = my_w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
      den += ws;
      // ascending key order; four independent row loads in flight per step
      for (int j = 0; j < cnt; j += 4) {
        float x[4][Vec<D>::N];
        float w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int uk = __shfl_sync(0xffffffffu, my_u, (j + k) & 31);
          w[k] = __shfl_sync(0xffffffffu, my_w, (j + k) & 31);
          if (j + k < cnt && w[k] != 0.f) {
            load_row<D>(p.part_o + (static_cast<size_t>(uk) * kTileM + r) * D, lane, x[k]);
          } else {
            w[k] = 0.f;
#pragma unroll
            for (int i = 0; i < Vec<D>::N; ++i) x[k][i] = 0.f;
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int i = 0; i < Vec<D>::N; ++i) acc[i] += w[k] * x[k][i];
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int i = 0; i < Vec<D>::N; ++i) acc[i] *= inv;
  store_row_bf16<D>(p.o + (static_cast<size_t>(token) * p.Hq + h) * D, lane, acc);
  if (lane == 0) p.lse[static_cast<size_t>(token) * p.Hq + h] = den > 0.f ? m + lg2(den) * kLn2 : -INFINITY;
}

// D = rowsum(dO * O) per (token, head); zeroes that row of the dQ accumulator.
template <int D>
// Blocks [0, main_blocks): one warp per row. Blocks past them zero the dead key ranges of dK and
// dV, 16 bytes per thread per step.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                       float* delta, float* dq_acc, long long n_rows,
                                                       unsigned main_blocks, const int64_t* dead, int n_samples,
                                                       long long row_chunks, uint4* dk, uint4* dv) {
  if (blockIdx.x >= main_blocks) {
    const long long zid = static_cast<long long>(blockIdx.x - main_blocks) * blockDim.x + threadIdx.x;
    const long long zstride = static_cast<long long>(gridDim.x - main_blocks) * blockDim.x;
    for (int b = 0; b < n_samples; ++b) {
      const long long k0 = dead[2 * b], k1 = dead[2 * b + 1];
      if (k1 <= k0) continue;
      const long long n = (k1 - k0) * row_chunks;
      uint4* zk = dk + k0 * row_chunks;
      uint4* zv = dv + k0 * row_chunks;
      for (long long i = zid; i < n; i += zstride) {
        zk[i] = make_uint4(0u, 0u, 0u, 0u);
        zv[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  float a[Vec<D>::N], b[Vec<D>::N];
  load_row_bf16<D>(o + row * D, lane, a);
  load_row_bf16<D>(dout + row * D, lane, b);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < Vec<D>::N; ++i) s += a[i] * b[i];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) delta[row] = s;
  float* z = dq_acc + row * D + lane * Vec<D>::N;
  if constexpr (D == 128)
    *reinterpret_cast<float4*>(z) = make_float4(0.f, 0.f, 0.f, 0.f);
  else
    *reinterpret_cast<float2*>(z) = make_float2(0.f, 0.f);
}

// dq = bf16(scale * dq_acc), 4 elements per thread.
__global__ void __launch_bounds__(256) dq_cast_kernel(const float* acc, __nv_bfloat16* dq, float scale, long long n4) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(acc)[i];
    uint2 t;
    t.x = pack_bf16(x.x * scale, x.y * scale);
    t.y = pack_bf16(x.z * scale, x.w * scale);
    reinterpret_cast<uint2*>(dq)[i] = t;
  }
}

}  // namespace

cudaError_t launch_merge(int d, const MergeParams& p, cudaStream_t stream) {
  if (p.n_rows == 0) return cudaSuccess;
  const long long blocks = (p.n_rows * 32 + 255) / 256;
  if (d == 64)
    merge_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  else
    merge_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep(int d, const __nv_bfloat16* o, const __nv_bfloat16* dout, float* delta, float* dq_acc,
                            long long n_rows, const int64_t* dead, int n_samples, int64_t dead_rows,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int hkv, cudaStream_t stream) {
  const long long main_blocks = (n_rows * 32 + 255) / 256;
  const long long row_chunks = static_cast<long long>(hkv) * d * 2 / 16;  // 16-byte chunks per key row
  long long zero_blocks = (dead_rows * row_chunks + 255) / 256;
  if (zero_blocks > 148 * 4) zero_blocks = 148 * 4;
  const long long blocks = main_blocks + zero_blocks;
  if (blocks == 0) return cudaSuccess;
  auto* zk = reinterpret_cast<uint4*>(dk);
  auto* zv = reinterpret_cast<uint4*>(dv);
  if (d == 64)
    bwd_prep_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        o, dout, delta, dq_acc, n_rows, static_cast<unsigned>(main_blocks), dead, n_samples, row_chunks, zk, zv);
  else
    bwd_prep_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        o, dout, delta, dq_acc, n_rows, static_cast<unsigned>(main_blocks), dead, n_samples, row_chunks, zk, zv);
  return cudaGetLastError();
}

cudaError_t launch_dq_cast(const float* dq_acc, __nv_bfloat16* dq, float scale, long long n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const long long n4 = n / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  dq_cast_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(dq_acc, dq, scale, n4);
  return cudaGetLastError();
}

}  // namespace skv
