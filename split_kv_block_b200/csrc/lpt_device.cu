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
//     after every item);
//   * the greedy placement by one warp, one item per step. Lane l owns
//     partitions l, l + 32, ... and holds the smallest (load, index) among
//     them; a step takes the minimum over the 32 lanes and adds the item's
//     cost to that partition.
// The greedy is a chain of dependent steps, so the step's latency is what
// counts. When every load stays below 2^51 (checked on the costs' sum), a
// lane's (load, index) is packed into one 64-bit key, load << 12 | index,
// whose order is the lexicographic one, and the warp minimum is two 32-bit
// `redux.sync` minima (high word, then the low word among the lanes holding
// the smallest high word) instead of a five-level shuffle tree over two
// words. Up to 128 partitions a lane keeps its loads in registers.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "kernels.h"

namespace skv {
namespace {

constexpr int kLptThreads = 1024;
constexpr long long kPackLimit = 1LL << 51;  // loads below this fit a key with a 12-bit partition index
constexpr unsigned kFull = 0xffffffffu;

// a sorts before b: longer first, then lower index
__device__ __forceinline__ bool before(long long ca, int ia, long long cb, int ib) {
  return ca > cb || (ca == cb && ia < ib);
}

__device__ __forceinline__ unsigned long long pack(long long load, int p) {
  return (static_cast<unsigned long long>(load) << 12) | static_cast<unsigned>(p);
}

// the smallest key over the warp
__device__ __forceinline__ unsigned long long warp_min_key(unsigned long long key) {
  const unsigned hi = static_cast<unsigned>(key >> 32);
  const unsigned mh = __reduce_min_sync(kFull, hi);
  const unsigned ml = __reduce_min_sync(kFull, hi == mh ? static_cast<unsigned>(key) : kFull);
  return (static_cast<unsigned long long>(mh) << 32) | ml;
}

// Packed keys, loads in registers: KP partitions per lane (P <= 32 KP).
template <int KP>
__device__ void greedy_regs(const long long* cost, const int* idx, int n, int P, int lane, int32_t* partition,
                            long long* load) {
  long long ld[KP];
#pragma unroll
  for (int j = 0; j < KP; ++j) ld[j] = 0;
  for (int r = 0; r < n; ++r) {
    const long long c = cost[r];
    const int item = idx[r];
    unsigned long long key = ~0ull;
#pragma unroll
    for (int j = 0; j < KP; ++j) {
      const int p = lane + 32 * j;
      const unsigned long long kj = pack(ld[j], p);
      if (p < P && kj < key) key = kj;
    }
    const int bp = static_cast<int>(warp_min_key(key) & 0xfffu);
#pragma unroll
    for (int j = 0; j < KP; ++j)
      if (lane + 32 * j == bp) ld[j] += c;
    if (lane == 0) partition[item] = bp;
  }
#pragma unroll
  for (int j = 0; j < KP; ++j)
    if (lane + 32 * j < P) load[lane + 32 * j] = ld[j];
  __syncwarp();
}

// Loads in shared memory (any P up to the limit): a lane keeps its smallest
// (load, index) and rescans its partitions only when it received the item.
template <bool kPacked>
__device__ void greedy_smem(const long long* cost, const int* idx, int n, int P, int lane, int32_t* partition,
                            long long* load) {
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
    int bp;
    if constexpr (kPacked) {
      const unsigned long long key = my_p < P ? pack(my_l, my_p) : ~0ull;
      bp = static_cast<int>(warp_min_key(key) & 0xfffu);
    } else {
      long long bl = my_l;
      bp = my_p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const long long ol = __shfl_xor_sync(kFull, bl, off);
        const int op = __shfl_xor_sync(kFull, bp, off);
        if (ol < bl || (ol == bl && op < bp)) {
          bl = ol;
          bp = op;
        }
      }
    }
    if (lane == (bp & 31)) {
      load[bp] += cost[r];
      partition[idx[r]] = bp;
      lane_min(my_l, my_p);
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kLptThreads) lpt_place_kernel(const int64_t* __restrict__ costs, int n, int n_pad,
                                                                int P, int32_t* __restrict__ partition,
                                                                int64_t* __restrict__ loads_out) {
  extern __shared__ __align__(16) unsigned char sm[];
  long long* cost = reinterpret_cast<long long*>(sm);
  int* idx = reinterpret_cast<int*>(cost + n_pad);
  long long* load = reinterpret_cast<long long*>(idx + n_pad);
  __shared__ unsigned long long total;
  __shared__ int unpackable;
  const int tid = threadIdx.x;
  if (tid == 0) {
    total = 0;
    unpackable = 0;
  }
  __syncthreads();
  // Padding sorts after every item whatever its cost (LLONG_MIN, ties broken by the larger index), so the
  // first n sorted entries are the items. Each thread's partial sum of costs below 2^51 stays below 2^55,
  // and their sum over 1024 threads below 2^61: no overflow before the check.
  unsigned long long mine = 0;
  bool bad = false;
  for (int i = tid; i < n_pad; i += kLptThreads) {
    const long long c = i < n ? static_cast<long long>(costs[i]) : LLONG_MIN;
    cost[i] = c;
    idx[i] = i;
    if (i < n) {
      bad |= c < 0 || c >= kPackLimit;
      mine += bad ? 0ull : static_cast<unsigned long long>(c);
    }
  }
  bad |= mine >= static_cast<unsigned long long>(kPackLimit);
  for (int p = tid; p < P; p += kLptThreads) load[p] = 0;
  if (bad) atomicOr(&unpackable, 1);
  else if (mine) atomicAdd(&total, mine);
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
  // every load is at most the sum of the costs
  const bool packed = !unpackable && total < static_cast<unsigned long long>(kPackLimit);
  if (packed && P <= 32) greedy_regs<1>(cost, idx, n, P, lane, partition, load);
  else if (packed && P <= 64) greedy_regs<2>(cost, idx, n, P, lane, partition, load);
  else if (packed && P <= 128) greedy_regs<4>(cost, idx, n, P, lane, partition, load);
  else if (packed) greedy_smem<true>(cost, idx, n, P, lane, partition, load);
  else greedy_smem<false>(cost, idx, n, P, lane, partition, load);
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
