// C ABI entry points: argument checks, workspace layout, plan upload,
// tensor maps and kernel launches. See include/skv.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <algorithm>
#include <vector>

#include "kernels.h"
#include "plan_layout.h"

namespace skv {
namespace {

thread_local int g_last_cuda = 0;
long long* g_fwd_stamps = nullptr;
long long* g_bwd_stamps = nullptr;
cudaEvent_t g_ev[3][2] = {};  // per SKV_KERNEL_*: start, end

cudaError_t mark(int kernel, int which, cudaStream_t stream) {
  return g_ev[kernel][which] ? cudaEventRecord(g_ev[kernel][which], stream) : cudaSuccess;
}
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s per device-side wait
constexpr uint64_t kPartialsL2Bytes = 64ull << 20;          // half of the 126 MB L2

int cuda_fail(cudaError_t e) {
  g_last_cuda = static_cast<int>(e);
  return SKV_ECUDA;
}

// ------------------------------------------------------------ plan upload
// The plan's device section is copied into the workspace from a pinned
// staging slot owned by the library; each slot is reused only after the copy
// that read it has completed, so the caller may reuse its plan buffer as soon
// as a call returns. The slots are mapped host memory (portable, so a kernel
// on any GPU of the process reads them), and the copy is a kernel that reads
// them over the bus: on B200 a copy-engine transfer between two kernels of one
// stream took about 9 us of stream time for any size up to 160 KB, and the
// kernel takes 2.5 to 5 us less per call on the 160 KB plan of a 32K context.
struct Staging {
  void* host = nullptr;
  size_t cap = 0;
  cudaEvent_t done = nullptr;
  bool pending = false;
};
constexpr int kSlots = 4;
constexpr int kMaxDevices = 64;
std::mutex g_stage_mu;
// Slots per device: a slot's event belongs to the device it was created on.
Staging g_stage[kMaxDevices][kSlots];
int g_stage_next[kMaxDevices] = {};
std::vector<void*> g_retired;  // outgrown staging buffers, released with the process

// Copies `total` bytes from mapped host memory `src` to device memory `dst`
// (both 16-byte aligned): 16 bytes per thread and step, the last total % 16
// bytes by the first threads of block 0.
__global__ void __launch_bounds__(256) upload_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                     size_t n16, size_t total) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride) dst[i] = src[i];
  const size_t tail = total - n16 * 16;
  if (blockIdx.x == 0 && threadIdx.x < tail)
    reinterpret_cast<uint8_t*>(dst)[n16 * 16 + threadIdx.x] =
        reinterpret_cast<const uint8_t*>(src)[n16 * 16 + threadIdx.x];
}

// Copies `zeros` zero bytes followed by the n bytes at src to dst, in one
// launch of upload_kernel from the staging slot.
int upload(const void* src, size_t n, void* dst, cudaStream_t stream, size_t zeros = 0) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return SKV_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_stage_mu);
  Staging& s = g_stage[dev][g_stage_next[dev]];
  g_stage_next[dev] = (g_stage_next[dev] + 1) % kSlots;
  if (s.pending) {
    e = cudaEventSynchronize(s.done);
    if (e != cudaSuccess) return cuda_fail(e);
    s.pending = false;
  }
  if (!s.done) {
    e = cudaEventCreateWithFlags(&s.done, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  const size_t total = zeros + n;
  if (s.cap < total) {
    // Grow geometrically and keep the old buffer until exit: cudaFreeHost
    // synchronizes the device, which would stall the caller's pipeline
    // whenever a larger plan arrives (plans change size every step when the
    // anchors are redrawn).
    size_t cap = size_t(1) << 20;
    while (cap < total) cap <<= 1;
    void* fresh = nullptr;
    e = cudaHostAlloc(&fresh, cap, cudaHostAllocMapped | cudaHostAllocPortable);
    if (e != cudaSuccess) return cuda_fail(e);
    if (s.host) g_retired.push_back(s.host);
    s.host = fresh;
    s.cap = cap;
  }
  std::memset(s.host, 0, zeros);
  std::memcpy(static_cast<uint8_t*>(s.host) + zeros, src, n);
  void* src_dev = nullptr;
  e = cudaHostGetDevicePointer(&src_dev, s.host, 0);
  if (e != cudaSuccess) return cuda_fail(e);
  const size_t n16 = total / 16;
  const int grid = static_cast<int>(std::max<size_t>(1, std::min<size_t>(2 * 148, (n16 + 255) / 256)));
  upload_kernel<<<grid, 256, 0, stream>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src_dev), n16, total);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaEventRecord(s.done, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  s.pending = true;
  return SKV_OK;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// bf16 tensor [rows][heads][d] seen as a 3-D map with a {64, box_h, box_rows}
// box and the 128-byte swizzle: one box fills box_h * box_rows rows of 128
// bytes of shared memory.
int make_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_h, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return SKV_ECUDA;
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0) return SKV_EINVAL;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(heads) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_h), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SKV_OK : SKV_ECUDA;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <class T>
T* at(void* base, uint64_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}
template <class T>
const T* at(const void* base, uint64_t off) {
  return reinterpret_cast<const T*>(static_cast<const uint8_t*>(base) + off);
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

// Device plan copy + zeroed control block and queue counters. `full` also
// uploads the arrays only the deterministic backward reads.
int prepare_ws(const PlanHeader& h, const void* plan, void* ws, const WsLayout& w, cudaStream_t stream,
               bool full = false) {
  // The control block (status word, queue and merge counters) is cleared and the plan's device section
  // copied behind it by one host-to-device copy: zeros up to the device section, then the section.
  const uint64_t n = full ? h.dev.bytes : h.dev.base_bytes;
  if (n > 0) return upload(static_cast<const uint8_t*>(plan) + h.dev_off, n, at<uint8_t>(ws, w.status), stream, w.dev);
  const cudaError_t e = cudaMemsetAsync(at<uint8_t>(ws, w.status), 0, w.control, stream);
  return e == cudaSuccess ? SKV_OK : cuda_fail(e);
}

}  // namespace

int skv_record_cuda_error(int cuda_error) { return cuda_fail(static_cast<cudaError_t>(cuda_error)); }

int skv_make_tile_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_h, int box_rows) {
  return make_map(map, base, rows, heads, d, box_h, box_rows);
}

}  // namespace skv

using namespace skv;

extern "C" const char* skv_strerror(int code) {
  switch (code) {
    case SKV_OK: return "ok";
    case SKV_EINVAL: return "invalid argument";
    case SKV_EWORKSPACE: return "buffer smaller than required";
    case SKV_EUNSUPPORTED: return "unsupported problem (head_dim, group size or sizes)";
    case SKV_ECUDA: return "CUDA runtime error";
    case SKV_EPLAN: return "not a plan written by skv_plan";
    case SKV_ETIMEOUT: return "a device-side wait timed out";
    case SKV_EDEVICE: return "a kernel found an inconsistent work list";
    case SKV_ESCRATCH: return "workspace exceeds the library's static scratch (SKV_NOALLOC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

extern "C" int skv_last_cuda_error(void) { return g_last_cuda; }

extern "C" int skv_set_unit_timer(void* fwd_stamps, void* bwd_stamps) {
  g_fwd_stamps = static_cast<long long*>(fwd_stamps);
  g_bwd_stamps = static_cast<long long*>(bwd_stamps);
  return SKV_OK;
}

extern "C" int skv_set_timing_events(int kernel, void* start_event, void* end_event) {
  if (kernel < SKV_KERNEL_FWD || kernel > SKV_KERNEL_BWD) return SKV_EINVAL;
  if ((start_event == nullptr) != (end_event == nullptr)) return SKV_EINVAL;
  g_ev[kernel][0] = static_cast<cudaEvent_t>(start_event);
  g_ev[kernel][1] = static_cast<cudaEvent_t>(end_event);
  return SKV_OK;
}

namespace {

// Forward launch shared by skv_attn_fwd (partials only, o == nullptr) and
// skv_attn_fwd_merged (partials merged into o / lse in the same launch).
int run_fwd(const PlanHeader* h, const void* plan, const void* q, const void* k, const void* v, void* ws,
            size_t ws_bytes, void* o, float* lse, cudaStream_t stream) {
  if (h->masked == 2) return SKV_EUNSUPPORTED;  // key tiles do not line up with the mask's blocks
  // a shard plan may own no key rows at all (more ranks than items): its K/V buffers may then be empty
  if (!q || !ws || (h->kv_rows > 0 && (!k || !v))) return SKV_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || reinterpret_cast<uintptr_t>(ws) % 256 != 0)
    return SKV_EINVAL;
  if (o && (!lse || !aligned16(o) || !aligned16(lse))) return SKV_EINVAL;
  const WsLayout w = ws_layout(*h);
  if (ws_bytes < w.fwd_end) return SKV_EWORKSPACE;
  int rc = prepare_ws(*h, plan, ws, w, stream);
  if (rc != SKV_OK) return rc;
  if (h->n_fwd == 0) return SKV_OK;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, h->Nq, h->Hq, h->d, h->G, h->tile_tokens)) != SKV_OK) return rc;
  if ((rc = make_map(&tk, k, h->kv_rows, h->kv_heads, h->d, 1, kTileN)) != SKV_OK) return rc;
  if ((rc = make_map(&tv, v, h->kv_rows, h->kv_heads, h->d, 1, kTileN)) != SKV_OK) return rc;
  const uint8_t* dev = at<uint8_t>(ws, w.dev);
  FwdParams p{};
  p.mtiles = at<MTile>(dev, h->dev.mtiles);
  p.tok_kend = at<int32_t>(dev, h->dev.tok_kend);
  p.units = at<FwdUnit>(dev, h->dev.fwd_units);
  p.part_off = at<int32_t>(dev, h->dev.fwd_part_off);
  p.pairs = at<FwdPair>(dev, h->dev.fwd_pairs);
  p.pair_off = at<int32_t>(dev, h->dev.fwd_pair_off);
  p.counters = at<int32_t>(ws, w.counters);
  p.status = at<int>(ws, w.status);
  p.part_o = at<float>(ws, w.fwd_o);
  p.part_lse = at<float>(ws, w.fwd_lse);
  p.partial_bf16 = (h->policy & SKV_PLAN_PARTIALS_BF16) ? 1 : 0;
  p.stamps = g_fwd_stamps;
  p.timeout_ns = kTimeoutNs;
  p.P = h->n_queues;
  p.G = h->G;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(h->d)));
  if (h->masked) {
    p.tile_mask = at<uint32_t>(dev, h->dev.tile_mask);
    p.pair_tile_off = at<int32_t>(dev, h->dev.pair_tile_off);
    p.unit_tile_off = at<int32_t>(dev, h->dev.unit_tile_off);
    p.live_tiles = at<int32_t>(dev, h->dev.live_tiles);
    p.mask_words = h->mask_words;
  }
  // partials that fit in half of L2 are kept there (evict_last) until the merge reads them
  p.partials_l2_last = (w.fwd_end - w.fwd_o) <= kPartialsL2Bytes ? 1 : 0;
  if (o) {
    p.merge_off = at<int32_t>(dev, h->dev.merge_off);
    p.merge_list = at<int32_t>(dev, h->dev.merge_list);
    p.arrive = at<int32_t>(ws, w.arrive);
    p.ready = at<int32_t>(ws, w.ready);
    p.merge_ctr = at<int32_t>(ws, w.merge_ctr);
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.n_slots = static_cast<int>(h->n_mtiles * h->Hkv);
    p.Hkv = h->Hkv;
    p.Hq = h->Hq;
  }
  int sms = num_sms();
  if (sms <= 0) return cuda_fail(cudaGetLastError());
  const int grid = fwd_grid(sms, h->n_fwd_pairs);
  cudaError_t e = mark(SKV_KERNEL_FWD, 0, stream);
  if (e == cudaSuccess) e = launch_fwd(h->d, tq, tk, tv, p, grid, stream);
  if (e == cudaSuccess) e = mark(SKV_KERNEL_FWD, 1, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return SKV_OK;
}

}  // namespace

extern "C" int skv_attn_fwd(const void* plan, const skv_problem* prob, const void* q, const void* k,
                            const void* v, void* ws, size_t ws_bytes, skv_stream_t stream_) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  return run_fwd(h, plan, q, k, v, ws, ws_bytes, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream_));
}

extern "C" int skv_attn_fwd_merged(const void* plan, const skv_problem* prob, const void* q, const void* k,
                                   const void* v, void* o, float* lse, void* ws, size_t ws_bytes,
                                   skv_stream_t stream_) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  if (!o || !lse) return SKV_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (h->empty_slots > 0) {
    // a shard plan whose rank has no unit for some query tiles: those rows are merged (O = 0,
    // LSE = -inf) by the merge kernel, launched after the forward
    rc = run_fwd(h, plan, q, k, v, ws, ws_bytes, nullptr, nullptr, stream);
    return rc != SKV_OK ? rc : skv_lse_merge(plan, prob, ws, o, lse, stream_);
  }
  return run_fwd(h, plan, q, k, v, ws, ws_bytes, o, lse, stream);
}

extern "C" int skv_lse_merge(const void* plan, const skv_problem* prob, const void* ws, void* o, float* lse,
                             skv_stream_t stream_) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  if (h->masked == 2) return SKV_EUNSUPPORTED;
  if (!ws || !o || !lse || !aligned16(o) || !aligned16(lse)) return SKV_EINVAL;
  const WsLayout w = ws_layout(*h);
  const uint8_t* dev = at<uint8_t>(ws, w.dev);
  MergeParams p{};
  p.mtiles = at<MTile>(dev, h->dev.mtiles);
  p.merge_off = at<int32_t>(dev, h->dev.merge_off);
  p.merge_list = at<int32_t>(dev, h->dev.merge_list);
  p.part_o = at<float>(ws, w.fwd_o);
  p.part_lse = at<float>(ws, w.fwd_lse);
  p.partial_bf16 = (h->policy & SKV_PLAN_PARTIALS_BF16) ? 1 : 0;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.n_rows = h->n_mtiles * h->Hkv * kTileM;
  p.Hkv = h->Hkv;
  p.G = h->G;
  p.Hq = h->Hq;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  cudaError_t e = mark(SKV_KERNEL_MERGE, 0, stream);
  if (e == cudaSuccess) e = launch_merge(h->d, p, stream);
  if (e == cudaSuccess) e = mark(SKV_KERNEL_MERGE, 1, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return SKV_OK;
}

namespace {

// dq_f32: write dQ as fp32 (this plan's contribution, to be summed over ranks) instead of bf16.
int run_bwd(const PlanHeader* h, const void* plan, const void* q, const void* k, const void* v, const void* o,
            const float* lse, const void* dout, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
            cudaStream_t stream, bool det, bool dq_f32 = false) {
  int rc = SKV_OK;
  if (h->masked == 2) return SKV_EUNSUPPORTED;  // key tiles do not line up with the mask's blocks
  if (!q || !o || !lse || !dout || !dq || !ws) return SKV_EINVAL;
  if (h->kv_rows > 0 && (!k || !v || !dk || !dv)) return SKV_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || reinterpret_cast<uintptr_t>(ws) % 256 != 0)
    return SKV_EINVAL;
  const WsLayout w = ws_layout(*h);
  if (ws_bytes < w.bwd_end) return SKV_EWORKSPACE;
  rc = prepare_ws(*h, plan, ws, w, stream, det);
  if (rc != SKV_OK) return rc;
  cudaError_t e;
  if (det) {
    e = cudaMemsetAsync(at<uint8_t>(ws, w.bwd_turn), 0, w.bwd_end - w.bwd_turn, stream);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  float* delta = at<float>(ws, w.bwd_delta);
  float* dq_acc = at<float>(ws, w.bwd_dq);
  const long long n_rows = h->Nq * h->Hq;
  // D, the zeroed dQ accumulator, and zero dK/dV for the keys no query attends to (the plan's
  // dead ranges, in the device section) in one launch
  int64_t dead_rows = 0;
  const int64_t* dead = at<int64_t>(plan, h->dead_off);
  for (int i = 0; i < h->n_dead; ++i) dead_rows += std::max<int64_t>(0, dead[2 * i + 1] - dead[2 * i]);
  e = launch_bwd_prep(h->d, static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), delta,
                      dq_acc, n_rows, at<int64_t>(at<uint8_t>(ws, w.dev), h->dev.dead), h->n_dead, dead_rows,
                      static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), h->kv_heads, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  if (h->n_bwd > 0) {
    CUtensorMap tq, tk, tv, tdo;
    if ((rc = make_map(&tq, q, h->Nq, h->Hq, h->d, h->G, h->tile_tokens)) != SKV_OK) return rc;
    if ((rc = make_map(&tdo, dout, h->Nq, h->Hq, h->d, h->G, h->tile_tokens)) != SKV_OK) return rc;
    if ((rc = make_map(&tk, k, h->kv_rows, h->kv_heads, h->d, 1, kTileN)) != SKV_OK) return rc;
    if ((rc = make_map(&tv, v, h->kv_rows, h->kv_heads, h->d, 1, kTileN)) != SKV_OK) return rc;
    const uint8_t* dev = at<uint8_t>(ws, w.dev);
    BwdParams p{};
    p.mtiles = at<MTile>(dev, h->dev.mtiles);
    p.tok_kend = at<int32_t>(dev, h->dev.tok_kend);
    p.units = at<BwdUnit>(dev, h->dev.bwd_units);
    p.part_off = at<int32_t>(dev, h->dev.bwd_part_off);
    p.counters = at<int32_t>(ws, w.counters) + h->P;
    p.status = at<int>(ws, w.status);
    p.lse = lse;
    p.delta = delta;
    p.dq_acc = dq_acc;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.kv_heads = h->kv_heads;
    if (h->masked) {
      p.tile_mask = at<uint32_t>(dev, h->dev.tile_mask);
      p.mask_words = h->mask_words;
    }
    p.stamps = g_bwd_stamps;
    p.timeout_ns = kTimeoutNs;
    if (det) {
      p.rank = at<int32_t>(dev, h->dev.bwd_rank);
      p.det_order = at<int32_t>(dev, h->dev.bwd_det_order);
      p.turn = at<int32_t>(ws, w.bwd_turn);
      p.n_bwd = static_cast<int>(h->n_bwd);
      p.det = 1;
    }
    p.P = h->n_queues;
    p.G = h->G;
    p.Hq = h->Hq;
    p.Hkv = h->Hkv;
    p.lgG = 0;
    while ((1 << p.lgG) < h->G) ++p.lgG;
    p.scale =static_cast<float>(1.0 / std::sqrt(static_cast<double>(h->d)));
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(h->d)));
    int sms = num_sms();
    if (sms <= 0) return cuda_fail(cudaGetLastError());
    const int grid = static_cast<int>(std::min<int64_t>(sms, h->n_bwd));
    e = mark(SKV_KERNEL_BWD, 0, stream);
    if (e == cudaSuccess) e = launch_bwd(h->d, tq, tk, tv, tdo, p, grid, stream);
    if (e == cudaSuccess) e = mark(SKV_KERNEL_BWD, 1, stream);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  const float dq_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(h->d)));
  e = dq_f32 ? launch_dq_scale(dq_acc, static_cast<float*>(dq), dq_scale, n_rows * h->d, stream)
             : launch_dq_cast(dq_acc, static_cast<__nv_bfloat16*>(dq), dq_scale, n_rows * h->d, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return SKV_OK;
}

}  // namespace

extern "C" int skv_attn_bwd(const void* plan, const skv_problem* prob, const void* q, const void* k,
                            const void* v, const void* o, const float* lse, const void* dout, void* dq, void* dk,
                            void* dv, void* ws, size_t ws_bytes, skv_stream_t stream) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  return run_bwd(h, plan, q, k, v, o, lse, dout, dq, dk, dv, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                 false);
}

extern "C" int skv_attn_bwd_deterministic(const void* plan, const skv_problem* prob, const void* q, const void* k,
                                          const void* v, const void* o, const float* lse, const void* dout,
                                          void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                          skv_stream_t stream) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  return run_bwd(h, plan, q, k, v, o, lse, dout, dq, dk, dv, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                 true);
}

extern "C" int skv_attn_bwd_partial(const void* plan, const skv_problem* prob, const void* q, const void* k,
                                    const void* v, const void* o, const float* lse, const void* dout, float* dq,
                                    void* dk, void* dv, void* ws, size_t ws_bytes, skv_stream_t stream) {
  int rc = SKV_OK;
  const PlanHeader* h = checked_plan(plan, prob, &rc);
  if (!h) return rc;
  return run_bwd(h, plan, q, k, v, o, lse, dout, dq, dk, dv, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                 false, true);
}

extern "C" int skv_lse_combine(const void* o_parts, const float* lse_parts, int n_parts, int64_t n_rows,
                               int head_dim, void* o, float* lse, skv_stream_t stream) {
  if (n_parts < 1 || n_rows < 0 || (head_dim != 64 && head_dim != 128)) return SKV_EINVAL;
  if (n_rows > 0 && (!o_parts || !lse_parts || !o || !lse)) return SKV_EINVAL;
  if (!aligned16(o_parts) || !aligned16(o) || reinterpret_cast<uintptr_t>(lse_parts) % 4 != 0 ||
      reinterpret_cast<uintptr_t>(lse) % 4 != 0)
    return SKV_EINVAL;
  cudaError_t e = launch_lse_combine(head_dim, static_cast<const __nv_bfloat16*>(o_parts), lse_parts, n_parts, n_rows,
                                     static_cast<__nv_bfloat16*>(o), lse, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SKV_OK : cuda_fail(e);
}

extern "C" int skv_dq_combine(const float* dq_parts, int n_parts, int64_t n, void* dq, skv_stream_t stream) {
  if (n_parts < 1 || n < 0 || n % 4 != 0) return SKV_EINVAL;
  if (n > 0 && (!dq_parts || !dq || !aligned16(dq_parts) || !aligned16(dq))) return SKV_EINVAL;
  cudaError_t e = launch_dq_combine(dq_parts, n_parts, n, static_cast<__nv_bfloat16*>(dq),
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SKV_OK : cuda_fail(e);
}

extern "C" int skv_status(const void* ws, skv_stream_t stream_) {
  if (!ws) return SKV_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int st = 0;
  cudaError_t e = cudaMemcpyAsync(&st, ws, sizeof(int), cudaMemcpyDeviceToHost, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return st;
}
