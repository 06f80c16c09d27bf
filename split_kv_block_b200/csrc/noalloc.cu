// skv_attn_fwd_noalloc: the split-KV forward plus LSE merge for callers that
// cannot allocate device memory.
//
// Who needs it: code that is handed only input and output pointers by a host
// framework that owns every byte of device memory (a plugin or extension
// with no allocator of its own), and latency-critical callers for which
// cudaMalloc/cudaFree are off limits because they may synchronize the whole
// device and stall work on other streams. Such callers cannot provide the
// workspace that skv_attn_fwd needs.
//
// How: the workspace (status word, device copy of the plan's work lists,
// queue counters, per-chunk partial outputs and LSEs) lives in the
// file-scope array below, allocated by the CUDA runtime when this library's
// device code is loaded and held by every GPU that loads the library until the
// process exits. This entry point calls no allocating routine: the plan's
// device section is copied with a plain cudaMemcpyAsync from the caller's
// buffer, and the status word and queue counters are cleared with
// cudaMemsetAsync on every call (the array keeps the previous call's
// contents; the partials are fully rewritten before they are read).
//
// Set-up: the first call on a device looks up the array's device address
// (cudaGetSymbolAddress, which may load this library's device code); make
// that first call before any stream capture. All calls share the one array
// per device, so calls whose work overlaps on the GPU (other streams, other
// host threads) race on it. Problems whose workspace exceeds the array are
// rejected with SKV_ESCRATCH before anything is enqueued. A device-side wait
// that gives up ends the kernels early and leaves its error in the status
// word at the start of the array, which skv_noalloc_status reads back.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "kernels.h"
#include "plan_layout.h"

namespace skv {
namespace {

constexpr size_t kNoAllocScratchBytes = SKV_NOALLOC_SCRATCH_BYTES;  // 32 MiB per GPU

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device, with that device current, and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace skv

using namespace skv;

extern "C" int skv_attn_fwd_noalloc(const void* plan, const skv_problem* prob, const void* q, const void* k,
                                    const void* v, void* o, float* lse, skv_stream_t stream_) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  if (h->masked == 2) return SKV_EUNSUPPORTED;  // key tiles do not line up with the mask's blocks
  if (!q || !k || !v || !o || !lse) return SKV_EINVAL;
  for (const void* ptr : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(lse)})
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return SKV_EINVAL;
  const WsLayout w = ws_layout(*h);
  if (w.fwd_end > kNoAllocScratchBytes) return SKV_ESCRATCH;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  void* ws = nullptr;
  cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  uint8_t* base = static_cast<uint8_t*>(ws);
  // zero what must start at zero: status word and queue counters
  e = cudaMemsetAsync(base + w.status, 0, w.control, stream);  // status word and queue counters
  if (e == cudaSuccess && h->dev.bytes > 0)
    e = cudaMemcpyAsync(base + w.dev, static_cast<const uint8_t*>(plan) + h->dev_off, h->dev.bytes,
                        cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  if (h->n_fwd == 0) return SKV_OK;

  CUtensorMap tq, tk, tv;
  rc = skv_make_tile_map(&tq, q, h->Nq, h->Hq, h->d, h->G, h->tile_tokens);
  if (rc == SKV_OK) rc = skv_make_tile_map(&tk, k, h->kv_rows, h->kv_heads, h->d, 1, kTileN);
  if (rc == SKV_OK) rc = skv_make_tile_map(&tv, v, h->kv_rows, h->kv_heads, h->d, 1, kTileN);
  if (rc != SKV_OK) return rc;
  const uint8_t* dev = base + w.dev;
  FwdParams p{};
  p.mtiles = reinterpret_cast<const MTile*>(dev + h->dev.mtiles);
  p.tok_kend = reinterpret_cast<const int32_t*>(dev + h->dev.tok_kend);
  p.units = reinterpret_cast<const FwdUnit*>(dev + h->dev.fwd_units);
  p.part_off = reinterpret_cast<const int32_t*>(dev + h->dev.fwd_part_off);
  p.pairs = reinterpret_cast<const FwdPair*>(dev + h->dev.fwd_pairs);
  p.pair_off = reinterpret_cast<const int32_t*>(dev + h->dev.fwd_pair_off);
  p.counters = reinterpret_cast<int32_t*>(base + w.counters);
  p.status = reinterpret_cast<int*>(base + w.status);
  p.part_o = reinterpret_cast<float*>(base + w.fwd_o);
  p.part_lse = reinterpret_cast<float*>(base + w.fwd_lse);
  p.partial_bf16 = (h->policy & SKV_PLAN_PARTIALS_BF16) ? 1 : 0;
  if (h->masked) {
    p.tile_mask = reinterpret_cast<const uint32_t*>(dev + h->dev.tile_mask);
    p.pair_tile_off = reinterpret_cast<const int32_t*>(dev + h->dev.pair_tile_off);
    p.unit_tile_off = reinterpret_cast<const int32_t*>(dev + h->dev.unit_tile_off);
    p.live_tiles = reinterpret_cast<const int32_t*>(dev + h->dev.live_tiles);
    p.mask_words = h->mask_words;
  }
  p.stamps = nullptr;
  p.timeout_ns = 2000000000ull;
  p.P = h->n_queues;
  p.G = h->G;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(h->d)));
  int dev_id = 0, sms = 0;
  e = cudaGetDevice(&dev_id);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_id);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  const int grid = fwd_grid(sms, h->n_fwd_pairs);
  e = launch_fwd(h->d, tq, tk, tv, p, grid, stream);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));

  MergeParams m{};
  m.mtiles = p.mtiles;
  m.merge_off = reinterpret_cast<const int32_t*>(dev + h->dev.merge_off);
  m.merge_list = reinterpret_cast<const int32_t*>(dev + h->dev.merge_list);
  m.part_o = p.part_o;
  m.part_lse = p.part_lse;
  m.partial_bf16 = p.partial_bf16;
  m.o = static_cast<__nv_bfloat16*>(o);
  m.lse = lse;
  m.n_rows = h->n_mtiles * h->Hkv * kTileM;
  m.Hkv = h->Hkv;
  m.G = h->G;
  m.Hq = h->Hq;
  e = launch_merge(h->d, m, stream);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  return SKV_OK;
}

extern "C" int skv_noalloc_status(skv_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  void* ws = nullptr;
  cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  int st = 0;
  e = cudaMemcpyAsync(&st, ws, sizeof(int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return skv_record_cuda_error(static_cast<int>(e));
  return st;
}
