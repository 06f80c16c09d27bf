// LPT placement on the device ("Split-KV: Breaking the Context Parallelism
// Bottleneck in Diffusion Drafter Training", section "LPT Scheduling: Load
// Balancing with Real Attention Costs": items sorted longest first, each
// placed on the currently least-loaded partition; "Split-KV: Efficient
// Context Parallelism for Training Diffusion Drafters", Abstract: planned
// every step).
//
// The same placement as the host planner, bit for bit: items sorted by
// (cost descending, index ascending) and each given to the partition with the
// smallest (load, index). One CTA:
//   * a bitonic sort of the (cost, index) pairs in shared memory (all
//     threads; the item count padded to a power of two with entries that sort
//     last);
//   * the greedy placement by one warp. Lane l owns partitions l, l + 32, ...
//     and keeps the smallest (load, index) among them; a step reduces the 32
//     lane minima across the warp, and only the lane that owns the chosen
//     partition recomputes its minimum.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "kernels.h"

namespace skv {
namespace {

constexpr int kLptThreads = 1024;

// a sorts before b: longer first, then lower index
__device__ __forceinline__ bool before(long long ca, int ia, long long cb, int ib) {
  return ca > cb || (ca == cb && ia < ib);
}

__global__ void __launch_bounds__(kLptThreads) lpt_place_kernel(const int64_t* __restrict__ costs, int n, int n_pad,
                                                                int P, int32_t* __restrict__ partition,
                                                                int64_t* __restrict__ loads_out) {
  extern __shared__ __align__(16) unsigned char sm[];
  long long* cost = reinterpret_cast<long long*>(sm);
  int* idx = reinterpret_cast<int*>(cost + n_pad);
  long long* load = reinterpret_cast<long long*>(idx + n_pad);
  const int tid = threadIdx.x;
  for (int i = tid; i < n_pad; i += kLptThreads) {
    cost[i] = i < n ? static_cast<long long>(costs[i]) : -1;  // padding sorts after every item (costs >= 0)
    idx[i] = i;
  }
  for (int p = tid; p < P; p += kLptThreads) load[p] = 0;
  __syncthreads();
  // bitonic sort into (cost desc, index asc)
  for (int k = 2; k <= n_pad; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n_pad; i += kLptThreads) {
        const int l = i ^ j;
        if (l > i) {
          const bool up = (i & k) == 0;  // this run ascends in the "before" order
          const bool swap = up ? before(cost[l], idx[l], cost[i], idx[i]) : before(cost[i], idx[i], cost[l], idx[l]);
          if (swap) {
            const long long c = cost[i];
            cost[i] = cost[l];
            cost[l] = c;
            const int t = idx[i];
            idx[i] = idx[l];
            idx[l] = t;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid >= 32) return;
  const int lane = tid;
  // this lane's smallest (load, index) among its partitions
  auto lane_min = [&](long long& bl, int& bp) {
    bl = LLONG_MAX;
    bp = INT_MAX;
    for (int p = lane; p < P; p += 32)
      if (load[p] < bl) {  // ascending p: the first of equal loads has the lower index
        bl = load[p];
        bp = p;
      }
  };
  long long my_l;
  int my_p;
  lane_min(my_l, my_p);
  for (int r = 0; r < n; ++r) {
    long long bl = my_l;
    int bp = my_p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const long long ol = __shfl_xor_sync(0xffffffffu, bl, off);
      const int op = __shfl_xor_sync(0xffffffffu, bp, off);
      if (ol < bl || (ol == bl && op < bp)) {
        bl = ol;
        bp = op;
      }
    }
    const int item = idx[r];
    if (lane == (bp & 31)) {
      load[bp] += cost[r];
      partition[item] = bp;
      lane_min(my_l, my_p);
    }
    __syncwarp();
  }
  for (int p = lane; p < P; p += 32) loads_out[p] = load[p];
}

}  // namespace
}  // namespace skv

using namespace skv;

extern "C" int skv_lpt_place_device(const int64_t* costs, int64_t n_items, int32_t n_partitions, int32_t* partition,
                                    int64_t* loads, skv_stream_t stream) {
  if (n_items < 0 || n_partitions < 1 || !loads || (n_items > 0 && (!costs || !partition))) return SKV_EINVAL;
  if (n_items > SKV_LPT_DEVICE_MAX_ITEMS || n_partitions > SKV_LPT_DEVICE_MAX_PARTITIONS) return SKV_EUNSUPPORTED;
  int n_pad = 2;  // a power of two, at least 2 so that the loads array after cost and idx is 8-byte aligned
  while (n_pad < n_items) n_pad <<= 1;
  const size_t smem = static_cast<size_t>(n_pad) * (sizeof(long long) + sizeof(int)) +
                      static_cast<size_t>(n_partitions) * sizeof(long long);
  cudaError_t e = cudaFuncSetAttribute(lpt_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e == cudaSuccess) {
    lpt_place_kernel<<<1, kLptThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        costs, static_cast<int>(n_items), n_pad, n_partitions, partition, loads);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  return SKV_OK;
}
