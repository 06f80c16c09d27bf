// Split-KV forward: launch of the forward kernel (fwd2.cu) for head_dim 64 and
// 128, and the grid it runs on.
//
// Source: "Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion
// Drafter Training", section "Split-KV's Core Mechanism" (each KV shard's
// local attention is computed for the global query set and aggregated
// through query-sized tensors); "Split-KV: Efficient Context Parallelism for
// Training Diffusion Drafters", Abstract (block-sparse mask over the context,
// exact result). Per forward unit (one item's key range x one 128-row query
// tile of one kv-head group) the kernel writes the tile rows' normalized
// partial output and log-sum-exp; masking: row r sees keys below its anchor
// end (and, with a block mask, only the blocks its anchor attends); rows past
// the sample's tokens see none; a row with no key in the unit gets LSE = -inf
// and O = 0.
#include <cuda_runtime.h>

#include "kernels.h"

namespace skv {

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdParams& p, int grid, cudaStream_t stream) {
  return launch_fwd2(d, tq, tk, tv, p, grid, stream);
}

// one persistent CTA per SM, at most one per pair of forward units
int fwd_grid(int sms, long long n_pairs) { return static_cast<int>(n_pairs < sms ? n_pairs : sms); }

}  // namespace skv
