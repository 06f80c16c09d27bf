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
#include "merge_row.cuh"
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

// Per (query tile, kv head, row): m = max LSE_c, LSE = m + ln sum exp(LSE_c - m),
// O = sum exp(LSE_c - LSE) O_c over the tile's partials in ascending key order.
template <int D, bool kB16>
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.n_rows) return;
  const int r = static_cast<int>(row % kTileM);
  const long long slot = row / kTileM;  // mt * Hkv + g
  const int g = static_cast<int>(slot % p.Hkv);
  const int mt = static_cast<int>(slot / p.Hkv);
  merge_row<D, kB16>(p.mtiles[mt], g, r, lane, p.G, p.Hq, p.merge_off[slot], p.merge_off[slot + 1],
                     p.merge_list, p.part_o, p.part_lse, p.o, p.lse);
}

// D = rowsum(dO * O) per (token, head); zeroes that row of the dQ accumulator.
template <int D>
// Blocks [0, main_blocks): one warp per row. Blocks past them zero the dead row ranges of dK and
// dV, 16 bytes per thread per step.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                                       float* delta, float* dq_acc, long long n_rows,
                                                       unsigned main_blocks, const int64_t* dead, int n_dead,
                                                       long long row_chunks, uint4* dk, uint4* dv) {
  if (blockIdx.x >= main_blocks) {
    const long long zid = static_cast<long long>(blockIdx.x - main_blocks) * blockDim.x + threadIdx.x;
    const long long zstride = static_cast<long long>(gridDim.x - main_blocks) * blockDim.x;
    for (int i = 0; i < n_dead; ++i) {
      const long long k0 = dead[2 * i], k1 = dead[2 * i + 1];
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

// dq = scale * dq_acc in fp32 (a rank's partial dQ, summed over ranks afterwards), 4 elements per thread.
__global__ void __launch_bounds__(256) dq_scale_kernel(const float* acc, float* dq, float scale, long long n4) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(acc)[i];
    reinterpret_cast<float4*>(dq)[i] = make_float4(x.x * scale, x.y * scale, x.z * scale, x.w * scale);
  }
}

// Combine of R rank partials per (token, head) row, ranks in order r = 0 .. R-1:
//   m = max_r LSE_r, den = sum_r exp(LSE_r - m), O = sum_r exp(LSE_r - m) O_r / den, LSE = m + ln den.
// A rank without keys for the row has LSE_r = -inf and weighs 0. One warp per row, lanes over d.
template <int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(const __nv_bfloat16* o_parts, const float* lse_parts,
                                                          int n_parts, long long n_rows, __nv_bfloat16* o,
                                                          float* lse) {
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.69314718055994531f;
  constexpr int N = D / 32;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  float m = -INFINITY;
  for (int r = lane; r < n_parts; r += 32) m = fmaxf(m, lse_parts[static_cast<size_t>(r) * n_rows + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[N] = {};
  float den = 0.f;
  if (m != -INFINITY) {
    for (int r = 0; r < n_parts; ++r) {
      const float l = lse_parts[static_cast<size_t>(r) * n_rows + row];
      if (l == -INFINITY) continue;
      const float w = ex2((l - m) * kLog2e);
      den += w;
      const __nv_bfloat16* src = o_parts + (static_cast<size_t>(r) * n_rows + row) * D + lane * N;
      if constexpr (N == 4) {
        const uint2 t = *reinterpret_cast<const uint2*>(src);
        acc[0] += w * __uint_as_float(t.x << 16);
        acc[1] += w * __uint_as_float(t.x & 0xffff0000u);
        acc[2] += w * __uint_as_float(t.y << 16);
        acc[3] += w * __uint_as_float(t.y & 0xffff0000u);
      } else {
        const uint32_t t = *reinterpret_cast<const uint32_t*>(src);
        acc[0] += w * __uint_as_float(t << 16);
        acc[1] += w * __uint_as_float(t & 0xffff0000u);
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* dst = o + static_cast<size_t>(row) * D + lane * N;
  if constexpr (N == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) lse[row] = den > 0.f ? m + lg2(den) * kLn2 : -INFINITY;
}

// dq = bf16(sum_r dq_parts[r]), ranks in order, 4 elements per thread.
__global__ void __launch_bounds__(256) dq_combine_kernel(const float* parts, int n_parts, long long n4,
                                                         __nv_bfloat16* dq) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < n_parts; ++r) {
      const float4 x = reinterpret_cast<const float4*>(parts)[static_cast<size_t>(r) * n4 + i];
      s.x += x.x;
      s.y += x.y;
      s.z += x.z;
      s.w += x.w;
    }
    reinterpret_cast<uint2*>(dq)[i] = make_uint2(pack_bf16(s.x, s.y), pack_bf16(s.z, s.w));
  }
}

}  // namespace

cudaError_t launch_dq_scale(const float* dq_acc, float* dq, float scale, long long n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const long long n4 = n / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  dq_scale_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(dq_acc, dq, scale, n4);
  return cudaGetLastError();
}

cudaError_t launch_lse_combine(int d, const __nv_bfloat16* o_parts, const float* lse_parts, int n_parts,
                               long long n_rows, __nv_bfloat16* o, float* lse, cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const long long blocks = (n_rows * 32 + 255) / 256;
  if (d == 64)
    lse_combine_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(o_parts, lse_parts, n_parts, n_rows, o, lse);
  else
    lse_combine_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(o_parts, lse_parts, n_parts, n_rows, o,
                                                                             lse);
  return cudaGetLastError();
}

cudaError_t launch_dq_combine(const float* parts, int n_parts, long long n, __nv_bfloat16* dq, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const long long n4 = n / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  dq_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(parts, n_parts, n4, dq);
  return cudaGetLastError();
}

cudaError_t launch_merge(int d, const MergeParams& p, cudaStream_t stream) {
  if (p.n_rows == 0) return cudaSuccess;
  const long long blocks = (p.n_rows * 32 + 255) / 256;
  auto kern = d == 64 ? (p.partial_bf16 ? merge_kernel<64, true> : merge_kernel<64, false>)
                      : (p.partial_bf16 ? merge_kernel<128, true> : merge_kernel<128, false>);
  kern<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep(int d, const __nv_bfloat16* o, const __nv_bfloat16* dout, float* delta, float* dq_acc,
                            long long n_rows, const int64_t* dead, int n_dead, int64_t dead_rows,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int kv_heads, cudaStream_t stream) {
  const long long main_blocks = (n_rows * 32 + 255) / 256;
  const long long row_chunks = static_cast<long long>(kv_heads) * d * 2 / 16;  // 16-byte chunks per key row
  long long zero_blocks = (dead_rows * row_chunks + 255) / 256;
  if (zero_blocks > 148 * 4) zero_blocks = 148 * 4;
  const long long blocks = main_blocks + zero_blocks;
  if (blocks == 0) return cudaSuccess;
  auto* zk = reinterpret_cast<uint4*>(dk);
  auto* zv = reinterpret_cast<uint4*>(dv);
  if (d == 64)
    bwd_prep_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        o, dout, delta, dq_acc, n_rows, static_cast<unsigned>(main_blocks), dead, n_dead, row_chunks, zk, zv);
  else
    bwd_prep_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        o, dout, delta, dq_acc, n_rows, static_cast<unsigned>(main_blocks), dead, n_dead, row_chunks, zk, zv);
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
