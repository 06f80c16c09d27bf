// The LSE merge inside the forward launch.
//
// Every forward unit writes its partial output and LSE for one (query tile,
// kv head) slot. When the last unit of a slot has written its partial, the
// slot goes on a completion list in global memory. A CTA that has no forward
// work left takes blocks of eight rows of those slots, in completion order,
// and merges them exactly (merge_row.cuh: max-shifted sum of exponentials,
// ascending key order), one row per warp. So the merge runs in the scheduling tail
// of the persistent forward, on SMs that would otherwise idle, while the
// slot's partials are recent in L2; no separate merge launch is needed.
// Source of the merge: "Split-KV: Breaking the Context Parallelism Bottleneck
// in Diffusion Drafter Training", section "Split-KV's Core Mechanism"
// (partials combined through query-sized tensors, exact).
//
// Ordering: the threads that wrote a unit's partial fence, synchronize their
// warp, and lane 0 of each of the unit's four warps fences again and
// increments the slot's arrival count (release pattern); the thread that
// completes the count fences (acquire pattern) and publishes the slot with a
// release store. The merging CTA acquires the list entry, then its threads
// read the partials through L2 (ld.global.cg). Waits are bounded: a slot that
// does not appear within the kernel's wait limit records SKV_ETIMEOUT, and a
// recorded error anywhere ends the wait at once.
#pragma once
#include <cuda_bf16.h>

#include "kernels.h"
#include "merge_row.cuh"
#include "sm100.cuh"

namespace skv {

// Called by every thread of the four warps that wrote one unit's partial
// (one row each), after its own writes; lane 0 of each warp reports the warp.
__device__ __forceinline__ void tail_merge_arrive(const FwdParams& p, int slot, int lane) {
  __threadfence();
  __syncwarp();
  if (lane == 0) {
    __threadfence();
    const int n = 4 * (p.merge_off[slot + 1] - p.merge_off[slot]);
    if (atomicAdd(&p.arrive[slot], 1) == n - 1) {
      __threadfence();
      const int i = atomicAdd(&p.merge_ctr[0], 1);
      st_release_gpu(&p.ready[i], slot + 1);
    }
  }
}

// The t-th completed slot, or -1 when an error was recorded or the wait gave up.
__device__ __forceinline__ int tail_merge_wait(const FwdParams& p, int t) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    const int v = ld_acquire_gpu(&p.ready[t]);
    if (v != 0) return v - 1;
    if (*reinterpret_cast<volatile int*>(p.status) != 0) return -1;
    if (globaltimer_ns() - t0 > p.timeout_ns) {
      atomicCAS(p.status, 0, kStatusTimeout);
      return -1;
    }
    __nanosleep(200);
  }
}

// Run by every thread of the CTA once its forward roles have finished.
// Tickets are (completed slot, block of kTailRows rows): the rows of a slot
// that completes late are merged by several CTAs at once, one row per warp.
// `s_slot` is a shared-memory word for the broadcast.
constexpr int kTailRows = 8;

template <int D>
__device__ __forceinline__ void tail_merge(const FwdParams& p, int* s_slot) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kBlocks = kTileM / kTailRows;
  while (true) {
    __syncthreads();  // the previous ticket's broadcast has been read
    if (tid == 0) {
      int v = -1;
      if (*reinterpret_cast<volatile int*>(p.status) == 0) {
        const int k = atomicAdd(&p.merge_ctr[1], 1);
        if (k < p.n_slots * kBlocks) {
          const int slot = tail_merge_wait(p, k / kBlocks);
          if (slot >= 0) v = slot * kBlocks + k % kBlocks;
        }
      }
      *s_slot = v;
    }
    __syncthreads();
    const int v = *s_slot;
    if (v < 0) break;
    const int slot = v / kBlocks, r = (v % kBlocks) * kTailRows + warp;
    if (warp < kTailRows) {
      const int mt = slot / p.Hkv, g = slot - mt * p.Hkv;
      if (p.partial_bf16)
        merge_row<D, true>(p.mtiles[mt], g, r, lane, p.G, p.Hq, p.merge_off[slot], p.merge_off[slot + 1],
                           p.merge_list, p.part_o, p.part_lse, p.o, p.lse);
      else
        merge_row<D, false>(p.mtiles[mt], g, r, lane, p.G, p.Hq, p.merge_off[slot], p.merge_off[slot + 1],
                            p.merge_list, p.part_o, p.part_lse, p.o, p.lse);
    }
  }
}

}  // namespace skv
