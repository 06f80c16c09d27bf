// sm_100a building blocks written as inline PTX: mbarriers with bounded waits,
// TMA tiled loads, tcgen05 (TMEM alloc, MMA, commit, ld/st, fences) and the
// shared-memory matrix descriptors the tensor core reads operands through.
//
// Layout conventions used by every kernel in this library:
//   * a bf16 tile of R rows x 64 columns is stored as R rows of 128 bytes with
//     the 128-byte swizzle (16-byte chunk c of row r lives at chunk c ^ (r & 7));
//     tiles wider than 64 columns are stacked 64-column blocks, block stride
//     R * 128 bytes. TMA with CU_TENSOR_MAP_SWIZZLE_128B writes exactly this.
//   * such a tile is a K-major operand when its rows are the M/N index and its
//     columns are the reduction index, and an MN-major operand when its rows
//     are the reduction index and its columns the M/N index.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace skv {

// ---------------------------------------------------------------- status word
// Error codes a kernel can leave in the device status word (see skv.h).
constexpr int kStatusTimeout = 6;   // SKV_ETIMEOUT
constexpr int kStatusBadPlan = 7;   // SKV_EDEVICE

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, giving up after `limit_ns`
// nanoseconds of wall time. On give-up it records kStatusTimeout in *status
// (first error wins) and returns false; the caller then abandons its loop.
// With a status word, it also returns false as soon as any other thread has
// recorded an error, so that every role of a failing CTA leaves quickly.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint64_t next_check = t0 + 20000;
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    // the status word is a global load: read it (and the limit) only once the wait has lasted 20 us, so that
    // a phase completing during that load's latency is not noticed late in ordinary waits
    const uint64_t now = globaltimer_ns();
    if (now < next_check) continue;
    next_check = now + 20000;
    // another role already gave up: leave too
    if (status && *reinterpret_cast<volatile int*>(status) != 0) return false;
    if (now - t0 > limit_ns) {
      if (status) atomicCAS(status, 0, kStatusTimeout);
      return false;
    }
  }
}

// Warp-uniform bounded wait: every lane of the warp gets the same verdict, so
// a warp never splits across a later warp-collective instruction.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, int* status, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, status, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------- cross-CTA flags (global)
__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int32_t* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Deterministic accumulation: the whole warp waits until the global turn
// counter `turn` holds `want` (lane 0 polls with acquire loads), bounded by
// `limit_ns` of %globaltimer time. On give-up it records kStatusTimeout; it
// also gives up at once when another thread has recorded an error. The
// verdict is the same on every lane.
__device__ __forceinline__ bool turn_wait(const int32_t* turn, int want, int* status, uint64_t limit_ns, int lane) {
  int ok = 1;
  if (lane == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(turn) != want) {
      if (*reinterpret_cast<volatile int*>(status) != 0) {
        ok = 0;
        break;
      }
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicCAS(status, 0, kStatusTimeout);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Hands the turn on: every lane's earlier writes are made visible at GPU
// scope before lane 0 stores `next` with release semantics.
__device__ __forceinline__ void turn_pass(int32_t* turn, int next, int lane) {
  __threadfence();
  __syncwarp();
  if (lane == 0) {
    __threadfence();
    st_release_gpu(turn, next);
  }
}

// ------------------------------------------------------- block-sparse mask
// The mask word of (query tile M, key block starting at absolute key kb) that
// holds token tl of the tile; bit tl % 32 says whether the token attends keys
// of the block.
template <class Tile>
__device__ __forceinline__ uint32_t mask_word(const uint32_t* tile_mask, int mask_words, const Tile& M, int kb,
                                              int tl) {
  return tile_mask[static_cast<size_t>(M.mbase + ((kb - M.kbase) >> 7)) * mask_words + (tl >> 5)];
}
// Whether any token of tile M attends a key of the block starting at kb.
template <class Tile>
__device__ __forceinline__ bool mask_block_live(const uint32_t* tile_mask, int mask_words, const Tile& M, int kb) {
  const uint32_t* w = tile_mask + static_cast<size_t>(M.mbase + ((kb - M.kbase) >> 7)) * mask_words;
  uint32_t any = 0;
  for (int i = 0; i < mask_words; ++i) any |= w[i];
  return any != 0;
}

// Whether query tile M has a row that attends a key of the key tile starting
// at kb (a backward unit's keys): some anchor of the tile lies past kb and,
// with a block-sparse mask, some token's block is on. Every role of a
// backward kernel walks the query tiles with this one test, so all of them
// agree on the sequence.
template <bool kMask, class Params, class Tile>
__device__ __forceinline__ bool tile_live(const Params& p, const Tile& M, int kb) {
  return M.kmax > kb && (!kMask || mask_block_live(p.tile_mask, p.mask_words, M, kb));
}

// ---------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ------------------------------------------------------------ L2 residency
// Cache policies for L2-hinted accesses (createpolicy, sm_80+): evict_last
// keeps lines ahead of normally-cached data, evict_first makes them the first
// to go.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_global_v4_hint(float* dst, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void st_global_v4u_hint(void* dst, uint4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w), "l"(pol)
               : "memory");
}
__device__ __forceinline__ uint2 ld_cg_u2_hint(const void* src, uint64_t pol) {
  uint2 v;
  asm volatile("ld.global.cg.L2::cache_hint.v2.b32 {%0, %1}, [%2], %3;" : "=r"(v.x), "=r"(v.y) : "l"(src), "l"(pol)
               : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_cg_u1_hint(const void* src, uint64_t pol) {
  uint32_t v;
  asm volatile("ld.global.cg.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(v) : "l"(src), "l"(pol) : "memory");
  return v;
}
// Loads through L2 only (.cg), with an L2 cache policy.
__device__ __forceinline__ float4 ld_cg_v4_hint(const float* src, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.cg.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(src), "l"(pol)
               : "memory");
  return v;
}
__device__ __forceinline__ float2 ld_cg_v2_hint(const float* src, uint64_t pol) {
  float2 v;
  asm volatile("ld.global.cg.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;" : "=f"(v.x), "=f"(v.y) : "l"(src), "l"(pol)
               : "memory");
  return v;
}

// -------------------------------------------------------------- async proxy
// Makes this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core operand reads, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- tcgen05
// Whole-warp TMEM allocation; the column base is written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A * B^T with A (M x K) and B (N x K) described by shared-memory
// descriptors, bf16 inputs, fp32 accumulate. One thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with the A operand read from TMEM: M rows = 128 TMEM lanes, each
// 32-bit column holds two consecutive K elements (low half = even k); one
// instruction consumes 8 columns (K = 16) starting at a_tmem.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// True on one lane of the converged warp (elect.sync). An MMA-issuing warp runs
// its loop on all 32 lanes, so that stage indices and descriptors are
// warp-uniform values, and issues the MMAs from the elected lane: the same
// instruction stream issued from a single-lane branch costs 20 to 45 % more
// cycles per N=64 MMA on the tensor pipe.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.b32 %0, 1, 0, P;\n\t}" : "=r"(pred));
  return pred != 0;
}

// Arrives once on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, dense.
// a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                                    // D format: f32
         | (1u << 7)                                  // A format: bf16
         | (1u << 10)                                 // B format: bf16
         | ((a_mn ? 1u : 0u) << 15)                   // A major
         | ((b_mn ? 1u : 0u) << 16)                   // B major
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   K-major operand : sbo = byte distance between 8-row groups (1024 for
//                     128-byte rows); lbo unused (16).
//   MN-major operand: lbo = byte distance between 64-element MN blocks,
//                     sbo = byte distance between groups of 8 K rows.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// The descriptor of the same operand `bytes` further on (a K step, a row block,
// a pipeline stage): the start-address field holds address >> 4 in 14 bits,
// and every shared-memory address is below 2^18, so the field never carries.
__device__ __forceinline__ uint64_t sdesc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets TMEM lane
// (32 * (warp % 4) + t), register j holds column (col + j).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------- fast math
// Maximum of three floats in one instruction (three-input max.f32, sm_100);
// same throughput as the two-input form, so a row maximum takes half the issues.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// Hardware base-2 exponential / logarithm (MUFU.EX2 / MUFU.LG2).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` inside a 128-byte-swizzled
// 64-column block.
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t c) {
  return r * 128u + (((c ^ (r & 7u)) & 7u) << 4);
}

}  // namespace skv
