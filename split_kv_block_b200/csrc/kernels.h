// Kernel parameter blocks and launchers (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cuda_bf16.h>

#include "plan_layout.h"

namespace skv {

struct FwdParams {
  const MTile* mtiles;
  const int32_t* tok_kend;
  const FwdUnit* units;
  const int32_t* part_off;  // [P+1] units of each work queue
  const FwdPair* pairs;     // pairs of forward units (two query tiles per CTA)
  const int32_t* pair_off;  // [P+1] pairs of each work queue
  int32_t* counters;        // [P] queue heads, zero at launch (P: the plan's work queues)
  int* status;
  float* part_o;            // [n_fwd][128][d], fp32 or (partial_bf16) bf16 elements
  float* part_lse;          // [n_fwd][128]
  int partial_bf16;         // partial outputs stored as bf16 (SKV_PLAN_PARTIALS_BF16)
  long long* stamps;        // optional [2 n_fwd] %globaltimer start/end per unit
  unsigned long long timeout_ns;
  int P;                    // work queues of the plan
  int G;
  float scale_log2;         // log2(e) / sqrt(d)
  int partials_l2_last;     // store the partials with the L2 evict_last policy (they fit in L2 beside K/V)
  // block-sparse mask (kernels compiled with kMask): per (tile, block) token words, and the live key tiles
  // of every forward pair (head_dim 128) or unit (head_dim 64) as first keys
  const uint32_t* tile_mask;
  const int32_t* pair_tile_off;  // [n_pairs + 1]
  const int32_t* unit_tile_off;  // [n_fwd + 1]
  const int32_t* live_tiles;
  int mask_words;
  // LSE merge in the same launch (tail_merge.cuh) when o != nullptr; partials only otherwise.
  const int32_t* merge_off;   // [n_slots + 1]: units of slot (query tile, kv head) = mt * Hkv + g
  const int32_t* merge_list;  // forward unit ids per slot, ascending key order
  int32_t* arrive;            // [n_slots] warps that have written their unit's partial rows, zero at launch
  int32_t* ready;             // [n_slots] slot + 1 of the i-th completed slot, zero at launch
  int32_t* merge_ctr;         // [2] completed slots, merge tickets taken; zero at launch
  __nv_bfloat16* o;           // [Nq][Hq][d] merged output, or nullptr
  float* lse;                 // [Nq][Hq]
  int n_slots;                // slots with at least one unit (every slot has one)
  int Hkv, Hq;
};

struct MergeParams {
  const MTile* mtiles;
  const int32_t* merge_off;
  const int32_t* merge_list;
  const float* part_o;      // fp32 or (partial_bf16) bf16 elements
  const float* part_lse;
  int partial_bf16;
  __nv_bfloat16* o;         // [Nq][Hq][d]
  float* lse;               // [Nq][Hq]
  long long n_rows;         // n_mtiles * Hkv * 128
  int Hkv, G, Hq;
};

struct BwdParams {
  const MTile* mtiles;
  const int32_t* tok_kend;
  const BwdUnit* units;
  const int32_t* part_off;
  int32_t* counters;
  int* status;
  const float* lse;         // [Nq][Hq] natural-log LSE of the merged forward
  const float* delta;       // [Nq][Hq] D = rowsum(dO * O)
  float* dq_acc;            // [Nq][Hq][d] fp32, zero at launch
  __nv_bfloat16* dk;        // [kv_rows][kv_heads][d] (the K/V buffers' layout)
  __nv_bfloat16* dv;
  int kv_heads;             // heads per K/V row: Hkv for a full plan, 1 for a shard plan
  const uint32_t* tile_mask;  // block-sparse mask (kernels compiled with kMask): per (tile, block) token words
  int mask_words;
  long long* stamps;
  unsigned long long timeout_ns;
  // Deterministic dQ (det != 0): units are taken from det_order through counters[0] instead of the
  // work queues, and each warp adds its dQ rows (fp32 reductions that complete before the turn passes)
  // once the turn counter of its (query tile, kv head, warp) equals the unit's rank, so the fp32 sum
  // over key tiles runs in ascending key order whatever the timing.
  const int32_t* rank;      // [n_bwd]
  const int32_t* det_order; // [n_bwd]
  int32_t* turn;            // [n_mtiles * Hkv][8], zero at launch
  int n_bwd;
  int det;
  int P, G, Hq, Hkv;
  int lgG;                  // log2(G); G = Hq / Hkv is a power of two
  float scale;              // 1 / sqrt(d)
  float scale_log2;         // log2(e) / sqrt(d)
};

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int grid, cudaStream_t stream);
cudaError_t launch_fwd2(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const FwdParams& p, int grid, cudaStream_t stream);  // pairs of query tiles
// CTAs of the forward launch: one per SM, at most one per pair of forward units
int fwd_grid(int sms, long long n_pairs);
cudaError_t launch_merge(int d, const MergeParams& p, cudaStream_t stream);
// D = rowsum(dO * O) and the zeroed dQ accumulator per (token, head) row; also zeroes dK/dV of
// the K/V rows no query attends to (rows dead[2i] .. dead[2i+1] for i < n_dead, device array;
// kv_heads heads per row).
cudaError_t launch_bwd_prep(int d, const __nv_bfloat16* o, const __nv_bfloat16* dout, float* delta, float* dq_acc,
                            long long n_rows, const int64_t* dead, int n_dead, int64_t dead_rows,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int kv_heads, cudaStream_t stream);
cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdParams& p, int grid, cudaStream_t stream);
cudaError_t launch_bwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                        const BwdParams& p, int grid, cudaStream_t stream);  // head_dim 128
cudaError_t launch_dq_cast(const float* dq_acc, __nv_bfloat16* dq, float scale, long long n, cudaStream_t stream);
cudaError_t launch_dq_scale(const float* dq_acc, float* dq, float scale, long long n, cudaStream_t stream);
// Context parallelism: combine of the ranks' (O_r, LSE_r), and the sum of the ranks' fp32 dQ partials.
cudaError_t launch_lse_combine(int d, const __nv_bfloat16* o_parts, const float* lse_parts, int n_parts,
                               long long n_rows, __nv_bfloat16* o, float* lse, cudaStream_t stream);
cudaError_t launch_dq_combine(const float* parts, int n_parts, long long n, __nv_bfloat16* dq, cudaStream_t stream);

// Helpers of the API layer shared with other entry-point files.
int skv_record_cuda_error(int cuda_error);  // remembers the error, returns SKV_ECUDA
int skv_make_tile_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_h, int box_rows);

}  // namespace skv
