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
  const int32_t* part_off;  // [P+1]
  const FwdPair* pairs;     // head_dim 128 kernel: pairs of units
  const int32_t* pair_off;  // [P+1]
  int32_t* counters;        // [P] queue heads, zero at launch
  int* status;
  float* part_o;            // [n_fwd][128][d]
  float* part_lse;          // [n_fwd][128]
  long long* stamps;        // optional [2 n_fwd] %globaltimer start/end per unit
  unsigned long long timeout_ns;
  int P;
  int G;
  float scale_log2;         // log2(e) / sqrt(d)
};

struct MergeParams {
  const MTile* mtiles;
  const int32_t* merge_off;
  const int32_t* merge_list;
  const float* part_o;
  const float* part_lse;
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
  __nv_bfloat16* dk;        // [Ltot][Hkv][d]
  __nv_bfloat16* dv;
  long long* stamps;
  unsigned long long timeout_ns;
  int P, G, Hq, Hkv;
  int lgG;                  // log2(G); G = Hq / Hkv is a power of two
  float scale;              // 1 / sqrt(d)
  float scale_log2;         // log2(e) / sqrt(d)
};

int fwd_smem_bytes(int d);
int bwd_smem_bytes(int d);
cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int grid, cudaStream_t stream);
cudaError_t launch_fwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                        int grid, cudaStream_t stream);  // head_dim 128: pairs of query tiles
int fwd2_smem_bytes();
// CTAs of the forward launch: one per SM, at most one per work unit (pair for head_dim 128)
int fwd_grid(int d, int sms, long long n_units, long long n_pairs);
cudaError_t launch_merge(int d, const MergeParams& p, cudaStream_t stream);
// D = rowsum(dO * O) and the zeroed dQ accumulator per (token, head) row; also zeroes dK/dV of
// the keys no query attends to (dead[2b] .. dead[2b+1] of every sample, device array).
cudaError_t launch_bwd_prep(int d, const __nv_bfloat16* o, const __nv_bfloat16* dout, float* delta, float* dq_acc,
                            long long n_rows, const int64_t* dead, int n_samples, int64_t dead_rows,
                            __nv_bfloat16* dk, __nv_bfloat16* dv, int hkv, cudaStream_t stream);
cudaError_t launch_bwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdParams& p, int grid, cudaStream_t stream);
cudaError_t launch_bwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                        const BwdParams& p, int grid, cudaStream_t stream);  // head_dim 128
int bwd2_smem_bytes();
cudaError_t launch_dq_cast(const float* dq_acc, __nv_bfloat16* dq, float scale, long long n, cudaStream_t stream);

// Helpers of the API layer shared with other entry-point files.
int skv_record_cuda_error(int cuda_error);  // remembers the error, returns SKV_ECUDA
int skv_make_tile_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_h, int box_rows);

}  // namespace skv
