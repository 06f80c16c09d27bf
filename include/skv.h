/*
 * skv.h — C ABI of libskv.so: split-KV block-sparse cross-attention on B200.
 *
 * The operation (sources: the web pages "Split-KV: Efficient Context
 * Parallelism for Training Diffusion Drafters", arXiv 2611.05926, Abstract;
 * and "Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion
 * Drafter Training", sections "Split-KV's Core Mechanism" and "LPT
 * Scheduling"): short draft-query blocks, one block of `block_q` tokens per
 * sampled anchor, cross-attend to a much longer context under a block-sparse
 * mask. The context K/V is split into chunks; every chunk yields a partial
 * output and log-sum-exp for the whole query set, and the partials are merged
 * exactly with a query-sized combine. Chunks are placed on P partitions by a
 * longest-processing-time-first planner weighted by realized attention cost.
 *
 * Readings fixed by this library where the pages give no formula:
 *   - the block of anchor a (1 <= a <= L_b) attends to keys [0, a) of its own
 *     sample's context; scale 1/sqrt(head_dim); LSE is the natural log;
 *   - q-head h uses kv-head h / (Hq / Hkv);
 *   - item = (sample b, chunk c, kv-head g, key sub-chunk s); its cost is the
 *     number of unmasked (query token, key) pairs times the q-heads per
 *     kv-head; LPT sorts by (cost desc, b, c, g, s) and gives each item to the
 *     partition with the smallest (load, index);
 *   - the static split gives partition p the packed context tokens
 *     [floor(p T / P), floor((p + 1) T / P)).
 *
 * Data layout (all device tensors contiguous, caller-owned):
 *   q, o, dout, dq : bf16 [Nq][Hq][d], Nq = anchor_offsets[B] * block_q; the
 *                    block of anchor j is tokens [j * block_q, (j+1) * block_q)
 *   k, v, dk, dv   : bf16 [Ltot][Hkv][d], Ltot = ctx_offsets[B]
 *   lse            : fp32 [Nq][Hq]
 *
 * Errors: every call returns an skv_status code; nothing throws across the
 * ABI. Calls that take a stream only enqueue work; errors found on the device
 * (a wait that gave up, a malformed plan) land in a status word inside the
 * workspace, read back by skv_status(). Arguments are checked before any
 * launch: bad values return SKV_EINVAL, unsupported shapes SKV_EUNSUPPORTED.
 *
 * Memory: the library allocates no device memory. The caller provides the
 * workspace `ws` (device, 256-byte aligned) sized by skv_plan_size(). For the
 * plan uploads the library keeps four pinned, mapped host staging slots per
 * device (grown on demand, released when the process exits); a call copies
 * the plan's device section into a slot before it returns, and a small kernel
 * on the call's stream copies the slot into `ws`.
 */
#ifndef SKV_H_
#define SKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* skv_stream_t; /* a cudaStream_t; NULL = legacy default stream */

enum skv_status_code {
  SKV_OK = 0,
  SKV_EINVAL = 1,       /* an argument is out of range or inconsistent */
  SKV_EWORKSPACE = 2,   /* buffer smaller than the size skv_plan_size() gave */
  SKV_EUNSUPPORTED = 3, /* valid problem this build does not run (head_dim, group size, sizes) */
  SKV_ECUDA = 4,        /* a CUDA runtime call failed (see skv_last_cuda_error) */
  SKV_EPLAN = 5,        /* plan buffer not written by skv_plan, or for another problem */
  SKV_ETIMEOUT = 6,     /* a device-side wait gave up; results are invalid */
  SKV_EDEVICE = 7,      /* a kernel found an inconsistent work list; results are invalid */
  SKV_ESCRATCH = 8      /* skv_attn_fwd_noalloc: workspace larger than SKV_NOALLOC_SCRATCH_BYTES */
};

enum skv_plan_policy {
  SKV_PLAN_LPT = 0,    /* cost-aware LPT over (b, c, g, s) items ("LPT Scheduling") */
  SKV_PLAN_STATIC = 1, /* equal-token contiguous split, the baseline LPT replaces */
  /* LPT with a cost calibrated to the executed work: query rows in tiles of
   * 128 / G tokens x G heads, an item's keys in tiles of 128 from its start,
   * and 128 * 128 per (query tile, key tile) block in which some token
   * attends some key. Same items and tie-break as SKV_PLAN_LPT; the items'
   * costs and the loads are in these units. Under a block mask it needs the
   * items to start on 128-key blocks (SKV_EUNSUPPORTED otherwise). */
  SKV_PLAN_LPT_TILES = 2,
  /* Flag, OR-ed into either policy: the forward stores each chunk's partial
   * output in bf16 instead of fp32 (the partial LSE stays fp32), halving the
   * partials' memory traffic and workspace. A partial output is a convex
   * combination of bf16 value rows, so rounding it adds at most 2^-9 times
   * the largest |V| to the merged output (about 1.1e-2 for N(0,1) values)
   * and nothing to the LSE. skv_plan_size, the forward and the merge read
   * the format from the plan. */
  SKV_PLAN_PARTIALS_BF16 = 0x100,
  /* Flag, OR-ed into any policy: the kernels of a full plan take their work
   * units from one queue per partition (a CTA starts on the queue of
   * partition floor(i P / grid) and moves to the next when it is empty)
   * instead of the default single queue that holds every item, each item's
   * units together: samples in the order of their costliest item, a
   * sample's items in placement order (costliest first). The items, costs,
   * partitions and loads do not change. On one GPU the default is faster:
   * the CTAs that share the queue run neighbouring units at the same time,
   * so an item's K/V tiles are read by many CTAs while they are in L2, not
   * by the few CTAs of one partition one after another (on the 128K
   * workload the forward's DRAM reads drop from 5.4x to 1.04x the K/V
   * bytes), and only one or two samples' queries and gradients are in use
   * at a time. A shard plan always has one queue. */
  SKV_PLAN_PARTITION_QUEUES = 0x200
};

/* One split-KV problem. Host pointers; read during the call only. */
typedef struct {
  int32_t num_samples;           /* B >= 1 */
  const int64_t* ctx_offsets;    /* [B+1], ctx_offsets[0] = 0, L_b = ctx_offsets[b+1] - ctx_offsets[b] >= 1 */
  const int32_t* anchor_offsets; /* [B+1], anchor_offsets[0] = 0, non-decreasing */
  const int64_t* anchors;        /* [anchor_offsets[B]], 1 <= a <= L_b; any order, duplicates allowed */
  int32_t block_q;               /* draft tokens per anchor, >= 1 */
  int32_t chunk_kv;              /* KV chunk length C >= 1 */
  int32_t sub_chunks;            /* LPT items split each chunk into this many key ranges; C % sub_chunks == 0 */
  int32_t num_partitions;        /* P >= 1 virtual partitions (the pages' CP ranks) */
  int32_t num_q_heads;           /* Hq */
  int32_t num_kv_heads;          /* Hkv; Hq % Hkv == 0 and 128 % (Hq / Hkv) == 0 */
  int32_t head_dim;              /* d in {64, 128} */
  /* Optional block-sparse mask over the context (NULL: the prefix mask alone).
   * Row j (one per anchor, mask_stride bytes) holds one byte per block of 128
   * keys of the anchor's sample: the block of anchor j attends key k (sample-
   * relative) iff k < a_j and key_block_mask[j * mask_stride + k / 128] != 0.
   * A block left with no key gets O = 0, LSE = -inf and no gradient. Needs
   * mask_stride >= ceil(L_b / 128) for every sample (SKV_EINVAL otherwise).
   * Plans of any policy carry the masked costs and loads; the kernel calls
   * need every item to start on a 128-key block of its sample (LPT with
   * chunk_kv / sub_chunks a multiple of 128) and return SKV_EUNSUPPORTED for
   * other plans (the static split's pieces, for instance). */
  const uint8_t* key_block_mask;
  int32_t mask_stride;
} skv_problem;

/* One planned work item (a view into the plan buffer). */
typedef struct {
  int32_t b, c, g, sub;        /* sample, chunk, kv-head, sub-chunk (static: piece index in the chunk) */
  int64_t key_begin, key_end;  /* absolute key range in the packed context, [begin, end) */
  int64_t cost;                /* unmasked (query, key) pairs x q-heads of the group */
  int32_t partition;           /* partition the planner placed the item on */
  int32_t order;               /* position in the placement order (LPT: longest first) */
  int64_t kv_row;              /* row of key_begin in the K/V buffers the kernels read: key_begin for a
                                  full plan; for a shard plan the item's first row in the shard buffer
                                  (one kv head per row), or -1 for items of other partitions */
} skv_item;

/*
 * skv_plan_size — sizes for one problem under one policy.
 * Outputs (any may be NULL): number of items, bytes of the host plan buffer,
 * device workspace bytes for skv_attn_fwd + skv_lse_merge, and for
 * skv_attn_bwd. One workspace of max(ws_fwd, ws_bwd) bytes serves a
 * forward, merge and backward issued in that order on one stream.
 * Returns SKV_EINVAL / SKV_EUNSUPPORTED for a problem skv_plan would reject.
 */
int skv_plan_size(const skv_problem* prob, int policy, size_t* n_items, size_t* plan_bytes,
                  size_t* ws_fwd_bytes, size_t* ws_bwd_bytes);

/*
 * skv_plan — realized cost of every item (pages: "LPT Scheduling", cost each
 * KV block actually incurs), placement by `policy`, and the work lists the
 * kernels read. Host only, deterministic: the same problem gives the same
 * bytes. `plan` is a caller-owned host buffer of plan_bytes (from
 * skv_plan_size); `partition_load` (may be NULL) receives [P] int64 loads.
 */
int skv_plan(const skv_problem* prob, int policy, void* plan, size_t plan_bytes, int64_t* partition_load);

/*
 * Context parallelism across GPUs ("Split-KV: Breaking the Context
 * Parallelism Bottleneck in Diffusion Drafter Training", section "Split-KV's
 * Core Mechanism: Decoupling Communication from Context Length"; "Split-KV:
 * Efficient Context Parallelism for Training Diffusion Drafters", Abstract):
 * the P partitions of an LPT plan are the ranks. Each rank keeps the key/
 * value rows of its own items, sees the whole (small) query set, computes its
 * partial output and LSE over its items and its share of dQ, and only
 * query-sized tensors cross ranks: the (O_r, LSE_r) pairs, combined exactly
 * by skv_lse_combine, and the dQ shares, summed by skv_dq_combine. dK and dV
 * stay on the rank that owns the keys.
 *
 * skv_plan_shard_size / skv_plan_shard — the plan of rank `partition` (0 <=
 * partition < P): the global plan's items and placement, with only that
 * partition's items turned into work units, all on one work queue. The
 * rank's K/V (and dK/dV) buffers hold the rows of its items, one kv head per
 * row, items in (b, c, g, s) order: item i occupies rows [kv_row, kv_row +
 * key_end - key_begin) of a bf16 [kv_rows][1][d] buffer (skv_plan_items gives
 * kv_row; skv_plan_kv_layout gives kv_rows). Queries, outputs, LSE and dO
 * keep the full problem's layout. Every call below accepts such a plan with
 * the full problem; skv_attn_fwd + skv_lse_merge then give the rank's
 * (O_r, LSE_r) (rows without keys on the rank: O_r = 0, LSE_r = -inf), and
 * skv_attn_bwd_partial its dQ share and its items' dK/dV. Same arguments and
 * errors as skv_plan_size / skv_plan, plus SKV_EINVAL for a partition out of
 * range.
 */
int skv_plan_shard_size(const skv_problem* prob, int policy, int partition, size_t* n_items, size_t* plan_bytes,
                        size_t* ws_fwd_bytes, size_t* ws_bwd_bytes);
int skv_plan_shard(const skv_problem* prob, int policy, int partition, void* plan, size_t plan_bytes,
                   int64_t* partition_load);

/* Layout of the K/V (and dK/dV) buffers a plan's kernels read: kv_rows rows
 * of kv_heads heads of head_dim bf16 each (Ltot and Hkv for a full plan;
 * the shard's key count and 1 for a shard plan), and the plan's shard (-1
 * for a full plan). Any pointer may be NULL. */
int skv_plan_kv_layout(const void* plan, int64_t* kv_rows, int32_t* kv_heads, int32_t* shard);

/* Limits of skv_lpt_place_device (one CTA, its shared memory). */
#define SKV_LPT_DEVICE_MAX_ITEMS 16384
#define SKV_LPT_DEVICE_MAX_PARTITIONS 4096

/*
 * skv_lpt_place_device — the LPT placement of skv_plan computed on the GPU
 * ("Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion
 * Drafter Training", section "LPT Scheduling": longest first onto the
 * least-loaded partition; planned every step), for callers whose item costs
 * are on the device. costs: device int64 [n_items] (>= 0), items in the order
 * whose index breaks ties (skv_plan's (b, c, g, sub) order); writes partition
 * (device int32 [n_items]) and loads (device int64 [n_partitions]). Items go
 * longest first, ties by lower index, each to the partition with the smallest
 * (load, index): the same bits as skv_plan's partitions and partition loads.
 * One CTA (a bitonic sort in shared memory, then one warp places the items).
 * SKV_EUNSUPPORTED beyond SKV_LPT_DEVICE_MAX_ITEMS items or
 * SKV_LPT_DEVICE_MAX_PARTITIONS partitions; SKV_EINVAL for NULL pointers or
 * n_partitions < 1. Enqueued on `stream`.
 */
int skv_lpt_place_device(const int64_t* costs, int64_t n_items, int32_t n_partitions, int32_t* partition,
                         int64_t* loads, skv_stream_t stream);

/* Items of a plan in (b, c, g, sub) order; *items points into `plan`. */
int skv_plan_items(const void* plan, const skv_item** items, size_t* n_items);

/* Virtual partition of every work unit of a plan, in the order the unit
 * timer (skv_set_unit_timer) indexes its stamps: fwd_part receives
 * [n_fwd_units] and bwd_part [n_bwd_units] int32 values in [0, P) (host
 * buffers, caller-owned, sized from skv_plan_stats; either may be NULL).
 * With the stamps, it gives the realized busy time of each partition: the
 * measured counterpart of the LPT loads ("Split-KV: Breaking the Context
 * Parallelism Bottleneck in Diffusion Drafter Training", section "LPT
 * Scheduling: Load Balancing with Real Attention Costs").
 * Returns SKV_EINVAL for a NULL plan, SKV_EPLAN for a buffer that is not a
 * plan of this library version. */
int skv_plan_unit_partitions(const void* plan, int32_t* fwd_part, int32_t* bwd_part);

/* Scalars of a plan: total cost (sum over items), number of forward work
 * units (item x 128-row query tile pairs with unmasked keys), number of
 * backward work units (item x 128-key tiles with unmasked queries),
 * imbalance max/mean - 1 of the partition loads. Any pointer may be NULL. */
int skv_plan_stats(const void* plan, int64_t* total_cost, int64_t* n_fwd_units, int64_t* n_bwd_units,
                   double* imbalance);

/*
 * Plan and problem. Every call that runs kernels takes the plan together
 * with `prob`, the problem the caller's tensors are shaped for (host, read
 * during the call only). The plan must have been written by skv_plan for that
 * same problem: same scalars, context offsets, anchor offsets and anchors
 * (skv_plan stores a 64-bit hash of them in the plan). Otherwise the call
 * returns SKV_EPLAN before it enqueues anything, so a plan never drives the
 * kernels over tensors of another problem's sizes. NULL plan or prob:
 * SKV_EINVAL.
 */

/*
 * skv_attn_fwd — split-KV forward ("Split-KV: Breaking the Context
 * Parallelism Bottleneck in Diffusion Drafter Training", section "Split-KV's
 * Core Mechanism": every KV chunk's local attention for the global query
 * set). For every forward work unit, writes the chunk's normalized partial
 * output (fp32) and LSE into the workspace. Copies the device part of `plan`
 * into `ws` first (the caller may reuse `plan` once the call returns).
 * q, k, v: device bf16 in the layouts above. Enqueued on `stream`.
 */
int skv_attn_fwd(const void* plan, const skv_problem* prob, const void* q, const void* k, const void* v, void* ws,
                 size_t ws_bytes, skv_stream_t stream);

/*
 * skv_lse_merge — exact query-sized combine of the partials left in `ws` by
 * skv_attn_fwd (same plan, same stream order). Source: "Split-KV: Breaking
 * the Context Parallelism Bottleneck in Diffusion Drafter Training", section
 * "Split-KV's Core Mechanism" (the partial results of every KV shard are
 * aggregated through query-sized tensors, with results strictly consistent
 * with the unsharded computation) and "Split-KV: Efficient Context
 * Parallelism for Training Diffusion Drafters", Abstract (exact). Per
 * (token, q-head):
 *   m = max_c LSE_c, LSE = m + ln sum_c exp(LSE_c - m),
 *   O = sum_c exp(LSE_c - LSE) O_c, chunks taken in ascending key order.
 * Writes o (device bf16 [Nq][Hq][d]) and lse (device fp32 [Nq][Hq]).
 */
int skv_lse_merge(const void* plan, const skv_problem* prob, const void* ws, void* o, float* lse,
                  skv_stream_t stream);

/*
 * skv_attn_fwd_merged — skv_attn_fwd and skv_lse_merge in one kernel launch
 * (same passages as those two calls). Every forward work unit writes its
 * partial into `ws` as skv_attn_fwd does; as soon as all units of a (query
 * tile, kv head) have written theirs, a CTA of the same launch that has no
 * forward work left merges that tile's rows into o and lse, with the
 * arithmetic and ascending key order of skv_lse_merge. So the merge runs in
 * the forward's scheduling tail, while the partials are recent in L2, and o
 * and lse are bitwise equal to those of skv_attn_fwd + skv_lse_merge (the
 * partials stay in `ws` as well). Outputs: o (device bf16 [Nq][Hq][d]), lse
 * (device fp32 [Nq][Hq]). The workspace is the forward's (ws_fwd_bytes).
 * Waits across CTAs are bounded like every other wait: a tile whose partials
 * do not all arrive within the limit records SKV_ETIMEOUT in the status word.
 * Enqueued on `stream`.
 */
int skv_attn_fwd_merged(const void* plan, const skv_problem* prob, const void* q, const void* k, const void* v,
                        void* o, float* lse, void* ws, size_t ws_bytes, skv_stream_t stream);

/*
 * skv_attn_bwd — gradients of the attention through the split. Source:
 * "Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion Drafter
 * Training", section "Split-KV's Core Mechanism" (the split is exact, which
 * gradient correctness relies on; key/value shards stay where they are and
 * only query-sized tensors are combined) and "Split-KV: Efficient Context
 * Parallelism for Training Diffusion Drafters", Abstract. Per KV item,
 * probabilities are recomputed with the merged LSE and D = rowsum(dO * O);
 * dK/dV of every key are written by the one item that owns it (zero for keys
 * no query attends to); dQ is summed over items in fp32 inside the workspace,
 * then rounded to bf16.
 * Inputs: q, k, v, o (bf16), lse (fp32, from skv_lse_merge), dout (bf16).
 * Outputs: dq, dk, dv (bf16, fully overwritten). Enqueued on `stream`.
 */
int skv_attn_bwd(const void* plan, const skv_problem* prob, const void* q, const void* k, const void* v,
                 const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv, void* ws,
                 size_t ws_bytes, skv_stream_t stream);

/*
 * skv_attn_bwd_deterministic — skv_attn_bwd with dQ summed over the key
 * tiles in one fixed order, so that two runs of the same problem give the
 * same dQ bits (dK and dV are bitwise reproducible in both calls: every key's
 * gradient is written by the one unit that owns it). Reading of the pages:
 * dQ = sum over KV chunks of the chunks' dQ contributions ("Split-KV:
 * Breaking the Context Parallelism Bottleneck in Diffusion Drafter Training",
 * section "Split-KV's Core Mechanism"), taken here in ascending key order, in
 * fp32. skv_attn_bwd adds the contributions with fp32 atomics in whatever
 * order the work units finish, which is faster but reproducible only to
 * rounding. Here the units are taken from one queue in (sample, key tile,
 * kv head) order, and each warp adds its rows of a query tile's dQ once every
 * unit with a lower key tile of the same sample and kv head has added its
 * own (a turn counter per query tile, kv head and warp, waited on with the
 * bounded wait of every kernel). Same arguments, layouts and workspace size
 * as skv_attn_bwd.
 */
int skv_attn_bwd_deterministic(const void* plan, const skv_problem* prob, const void* q, const void* k,
                               const void* v, const void* o, const float* lse, const void* dout, void* dq,
                               void* dk, void* dv, void* ws, size_t ws_bytes, skv_stream_t stream);

/*
 * skv_attn_bwd_partial — skv_attn_bwd with dQ written in fp32 (device
 * [Nq][Hq][d], scaled): the plan's share of dQ, to be summed over ranks with
 * skv_dq_combine. For a shard plan it is the rank's share (its keys' part of
 * every query's gradient); dk and dv are the shard's rows (kv_rows x 1 x d).
 * Same arguments, layouts and workspace as skv_attn_bwd otherwise.
 */
int skv_attn_bwd_partial(const void* plan, const skv_problem* prob, const void* q, const void* k, const void* v,
                         const void* o, const float* lse, const void* dout, float* dq, void* dk, void* dv, void* ws,
                         size_t ws_bytes, skv_stream_t stream);

/*
 * skv_lse_combine — exact combine of the ranks' partial outputs (the
 * query-sized aggregation of "Split-KV's Core Mechanism"): per row i of
 * n_rows = Nq * Hq, over ranks r = 0 .. n_parts-1 in order,
 *   m = max_r LSE_r, LSE = m + ln sum_r exp(LSE_r - m),
 *   O = sum_r exp(LSE_r - LSE) O_r; ranks with LSE_r = -inf weigh nothing.
 * o_parts: device bf16 [n_parts][n_rows][head_dim] (the all-gathered rank
 * outputs of skv_lse_merge), lse_parts: device fp32 [n_parts][n_rows];
 * writes o (bf16 [n_rows][head_dim]) and lse (fp32 [n_rows]). head_dim 64 or
 * 128; SKV_EINVAL otherwise or for misaligned pointers. Enqueued on `stream`.
 */
int skv_lse_combine(const void* o_parts, const float* lse_parts, int n_parts, int64_t n_rows, int head_dim,
                    void* o, float* lse, skv_stream_t stream);

/*
 * skv_dq_combine — dQ = sum over ranks of their fp32 shares (from
 * skv_attn_bwd_partial), ranks in order r = 0 .. n_parts-1, rounded once to
 * bf16. dq_parts: device fp32 [n_parts][n]; dq: device bf16 [n]; n a
 * multiple of 4 (Nq * Hq * head_dim). Enqueued on `stream`.
 */
int skv_dq_combine(const float* dq_parts, int n_parts, int64_t n, void* dq, skv_stream_t stream);

/*
 * skv_status — synchronizes `stream`, reads the status word in `ws` and
 * returns it (SKV_OK when no kernel reported an error since the last
 * skv_attn_fwd/skv_attn_bwd reset it). SKV_ECUDA if the synchronize failed.
 */
int skv_status(const void* ws, skv_stream_t stream);

/* Static text for a status code. */
const char* skv_strerror(int code);

/* Last CUDA runtime error code seen by this thread's calls (0 if none). */
int skv_last_cuda_error(void);

/* Realized per-partition busy time: while set (non-NULL), the forward /
 * backward kernels record, per work unit u, its %globaltimer start and end
 * (ns) into stamps[2u], stamps[2u+1] (device int64 [2 * n_units],
 * caller-owned). NULL disables. Process-wide setting. */
int skv_set_unit_timer(void* fwd_stamps, void* bwd_stamps);

enum skv_kernel_id { SKV_KERNEL_FWD = 0, SKV_KERNEL_MERGE = 1, SKV_KERNEL_BWD = 2 };

/* Kernel timing: while set, the library records the caller-created CUDA
 * events `start` / `end` (cudaEvent_t) on the launch stream immediately
 * before and after every launch of the given kernel (the forward attention
 * kernel, with its merge for skv_attn_fwd_merged; the LSE merge kernel; or
 * the backward attention kernel). NULL disables. Process-wide setting. */
int skv_set_timing_events(int kernel, void* start_event, void* end_event);

/* Size of the library-owned scratch array used by skv_attn_fwd_noalloc. */
#define SKV_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * skv_attn_fwd_noalloc — skv_attn_fwd followed by skv_lse_merge, for callers
 * that cannot allocate device memory. The pages have no counterpart of this
 * call; it is a deployment convenience of this library.
 *
 * Which callers: code given only input and output pointers by a host
 * framework that owns all device memory (a plugin without an allocator of
 * its own), and latency-critical code that must not call cudaMalloc/cudaFree
 * because they can synchronize the device and stall other streams. Neither
 * can provide the workspace skv_attn_fwd needs.
 *
 * The workspace lives instead in one file-scope device array of
 * SKV_NOALLOC_SCRATCH_BYTES (32 MiB) per GPU, held by every GPU that loads the
 * library until the process exits. The call allocates nothing: no
 * cudaMalloc, cudaFree, pinned staging or library allocator. The caller
 * passes the plan (host, from skv_plan), q, k, v (device bf16) and the outputs
 * o (device bf16 [Nq][Hq][d]) and lse (device fp32 [Nq][Hq]), as for
 * skv_attn_fwd + skv_lse_merge, and `prob`, the problem the plan was made for
 * (SKV_EPLAN otherwise, before anything is enqueued). The plan's device
 * section is copied from `plan` with one cudaMemcpyAsync, with no staging of
 * the library's own. From pageable host memory that copy may block the
 * calling thread until earlier work on `stream` has drained, and it cannot be
 * recorded inside a stream capture. Keep the plan in pinned memory instead
 * (page-locked by the caller's framework) and leave it unchanged until
 * `stream` has passed this call.
 *
 * The first call on a device looks up the array's device address (this may
 * load the library's device code); make it before any stream capture.
 * Every call shares the array and it keeps the last call's contents; the
 * call clears what must start at zero. Calls whose GPU work overlaps (other
 * streams or threads) race on the array. Returns SKV_ESCRATCH, before
 * enqueuing anything, when the problem's forward workspace (ws_fwd_bytes of
 * skv_plan_size) exceeds SKV_NOALLOC_SCRATCH_BYTES. A device-side wait that
 * gives up ends the kernels early and leaves SKV_ETIMEOUT in the status word
 * inside the array; read it with skv_noalloc_status.
 */
int skv_attn_fwd_noalloc(const void* plan, const skv_problem* prob, const void* q, const void* k, const void* v,
                         void* o, float* lse, skv_stream_t stream);

/*
 * skv_noalloc_status — the status word left in the library's scratch array
 * (on the current device) by the last skv_attn_fwd_noalloc call: SKV_OK, or
 * the error a kernel of that call recorded (SKV_ETIMEOUT, SKV_EDEVICE), in
 * which case o and lse of that call are invalid. Synchronizes `stream` and
 * copies the 4-byte word to host memory; allocates nothing. Returns
 * SKV_ECUDA if the copy or the synchronize failed. Like the scratch array,
 * the word is shared by every call on the device: read it before the next
 * skv_attn_fwd_noalloc call clears it. The pages have no counterpart of this
 * call.
 */
int skv_noalloc_status(skv_stream_t stream);

/*
 * skv_wait_selftest — exercises, without any fault, the bounded device-side
 * wait every kernel of this library uses. One CTA waits on a shared-memory
 * mbarrier phase for at most `limit_ns` nanoseconds of %globaltimer time:
 *   * arrive != 0: the CTA completes the phase itself first, the wait
 *     succeeds and the status word stays SKV_OK;
 *   * arrive == 0: nothing completes the phase, the wait gives up and records
 *     SKV_ETIMEOUT in the status word, exactly as a stalled pipeline stage of
 *     the attention kernels would. The device context stays usable.
 * The outcome is read with skv_status(ws, stream). The pages have no
 * counterpart of this call; it tests this library's failure detection.
 * ws: device buffer of at least 256 bytes, 256-byte aligned, caller-owned;
 * its status word is cleared first. limit_ns: 1 .. 10^10. A wait checks its
 * limit (and the status word) only once it has lasted 20 us, and every 20 us
 * after that, so it gives up between limit_ns and max(limit_ns, 20 us) + 20 us.
 * Returns SKV_EINVAL for a NULL or misaligned ws or a limit out of range,
 * SKV_ECUDA when the launch fails, SKV_OK otherwise.
 */
int skv_wait_selftest(void* ws, uint64_t limit_ns, int arrive, skv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SKV_H_ */
