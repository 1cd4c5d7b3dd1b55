/*
 * ep_balance.h — C ABI of the B200 expert-balance library (libep_b200.so).
 *
 * One microbatch and one MoE layer of UltraEP-style real-time expert load
 * balancing, with the expert-parallel group of R ranks simulated as data on one
 * GPU.  Sources, by page title and section:
 *
 *   [U] "300 µs to level MoE expert load: Xiaohongshu UltraEP" (UltraEP page)
 *       §"Getting the real load of the current layer after the Gate",
 *       §"Quota decides replicas and token split together",
 *       §"Shared redundant slots manage dynamic replicas",
 *       §"Reusing the forward plan for weight restore and gradient reduction".
 *   [W] "Improving DeepEP MoE Load Balance in SGLang with Waterfill and LPLB"
 *       §"Waterfill" (waterline, slack, per-token draw, local preference,
 *       fallback) and §"Shared expert fusion" (one extra slot per rank).
 *
 * Conventions shared by every call:
 *   - Pointers named d_* are device pointers, h_* host pointers.  The caller owns
 *     all device memory (workspace, inputs, outputs, weights, slots); it must
 *     outlive the plan.  The plan handle owns only host state.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call except ep_read_layer_stats is asynchronous on that stream and
 *     performs no host synchronisation; plan data stays on the device.
 *   - Host-side argument errors return immediately with no work enqueued.
 *     Device-side anomalies never trap: kernels set bits of the layer's device
 *     status word (EP_DEV_*), read back by ep_read_layer_stats.
 *   - Integer results are bit-exact and deterministic (independent of grid
 *     size and run); the one floating-point operation (gradient reduction)
 *     adds in a fixed order.
 *   - All functions are thread-compatible: one plan must not be used from two
 *     host threads at once.  Calls on one plan that overlap on the GPU race.
 */
#ifndef EP_BALANCE_H_
#define EP_BALANCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EP_ABI_VERSION 2

/* Exported symbols of libep_b200.so (everything else is hidden). */
#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

typedef int32_t ep_status_t;
enum {
  EP_OK = 0,
  EP_ERR_INVALID_ARGUMENT = 1,   /* null pointer, out-of-range layer or rank range, bad size */
  EP_ERR_UNSUPPORTED = 2,        /* shape outside the supported limits below */
  EP_ERR_CUDA = 3,               /* a CUDA runtime call or launch failed */
  EP_ERR_WORKSPACE_TOO_SMALL = 4,
  EP_ERR_NOT_PLANNED = 5,        /* layer was never balanced (host-side bookkeeping) */
  EP_ERR_DEVICE_STATUS = 6       /* ep_read_layer_stats found a device status bit set */
};

/* Device status bits (ep_layer_stats.status). */
#define EP_DEV_BAD_ID 1        /* a top-k id outside [0, E): not counted, its row is -1 */
#define EP_DEV_ITER_CAP 2      /* a cap candidate hit the solver's iteration bound */
#define EP_DEV_WAIT_TIMEOUT 4  /* a bounded wait ran out (the bulk-copy dispatch variant's
                                  mbarrier waits; the default kernels never wait) */
#define EP_DEV_OUT_CAPACITY 8  /* a dispatch row fell outside the caller's output buffer */
#define EP_DEV_INCONSISTENT 16 /* an assignment found no rerouting segment (internal check) */

/* Stop reasons of the quota solve (ep_layer_stats.stop_reason). */
#define EP_STOP_BALANCED 0      /* every rank at or below the cap */
#define EP_STOP_SLOT_LIMITED 1  /* an over-cap rank could not shed load because every
                                   rank with room had its redundant slots full */
#define EP_STOP_QUOTA_LIMITED 2 /* an over-cap rank could not shed load: no receiver had
                                   room for the minimum quota, or its natives were below it */
#define EP_STOP_ITER_CAP 3

/*
 * Problem description.  Supported limits (else EP_ERR_UNSUPPORTED):
 *   1 <= R <= 128, 1 <= E <= 1024, natives per rank ceil(E/R) <= 32,
 *   1 <= K <= 16, T >= 0, R*T*(K+1) < 2^31, 0 <= S <= 8, m >= 1,
 *   1 <= J <= 16, hidden >= 8 with hidden*2 a multiple of 16 bytes,
 *   expert_weight_elems >= 0 and a multiple of 8,
 *   R*S*ceil(expert_weight_elems/16) < 2^32, num_layers >= 1,
 *   0 <= waterfill_bonus_permille <= 1000, rerouting_mode in {0, 1},
 *   solver_iter_limit >= 0.
 * Native placement is fixed: rank q hosts the contiguous block of experts
 * [q*(E/R) + min(q, E%R), ... + E/R + (q < E%R)) ([U] §"Shared redundant
 * slots": every logical expert keeps one fixed native instance).
 */
typedef struct ep_config {
  int32_t num_ranks;                /* R: simulated EP ranks */
  int32_t num_experts;              /* E: logical routed experts */
  int32_t top_k;                    /* K */
  int32_t tokens_per_rank;          /* T */
  int32_t slots_per_rank;           /* S: redundant slots per rank ([U] §"Quota") */
  int32_t min_replica_quota;        /* m: minimum quota of a new replica ([U]: 1024) */
  int32_t hidden;                   /* bf16 elements per hidden-state row */
  int32_t num_layers;               /* depth of the per-layer plan cache */
  int32_t num_cap_candidates;       /* J: caps ceil(A(200+j)/(200R)), j < J */
  int32_t shared_expert;            /* 1: one Waterfill shared-expert slot per token ([W]) */
  int32_t waterfill_bonus_permille; /* local preference B = ceil(H*bonus/1000) */
  int32_t waterfill_all_ranks;      /* 0: candidates = own rank + ranks the token visits
                                       (communication-conservative set, [W]); 1: all ranks
                                       ([W]'s all-rank mode) */
  int64_t expert_weight_elems;      /* Wn: bf16 elements of one expert (3*hidden*ffn) */
  uint64_t waterfill_seed;          /* seed of the per-token SplitMix64 draw */
  uint64_t sampling_seed;           /* seed of the per-assignment draw of rerouting_mode 1 */
  int32_t rerouting_mode;           /* EP_REROUTE_LOCAL_FIRST or EP_REROUTE_SAMPLED */
  int32_t solver_iter_limit;        /* 0: the solver's bound 4(R*S + R + E) + 64; > 0: this
                                       bound instead (drives EP_DEV_ITER_CAP in tests) */
} ep_config;

/* Rerouting modes (ep_config.rerouting_mode).  Both use the same quota solve.
 * LOCAL_FIRST ([U] §"Quota"): each source rank's assignments of an expert use
 * the instance on the source's own rank up to its quota, the rest fill the
 * remote instances in instance order up to their remaining quotas; every
 * instance receives exactly its quota.
 * SAMPLED ([W] §"LPLB": the per-expert split, normalised to a distribution
 * over the expert's physical instances, from which each token samples one):
 * assignment a = (r*T + t)*K + k of expert e picks instance i of e with
 * probability quota_i / total_e, drawn as h = SplitMix64(sampling_seed + a),
 * u = ((h >> 32) * total_e) >> 32, i = first instance in instance order whose
 * running quota sum exceeds u; an expert with one instance takes no draw.  An
 * instance then receives as many rows as it drew (ep_layer_view.inst_count);
 * rows inside an instance stay ordered by (source rank, t, k).  Waterfill's
 * load score remains the solve's planned per-rank load. */
#define EP_REROUTE_LOCAL_FIRST 0
#define EP_REROUTE_SAMPLED 1

/* Per-layer results, device-resident; copied to the host by ep_read_layer_stats. */
typedef struct ep_layer_stats {
  int32_t status;            /* EP_DEV_* bits */
  int32_t cap_idx;           /* chosen cap candidate j */
  int32_t stop_reason;       /* EP_STOP_* of the chosen candidate */
  int32_t tight_stop_reason; /* EP_STOP_* of candidate j = 0 (the cap nearest the mean) */
  int32_t replicas;          /* replicas placed */
  int32_t realized_max;      /* max per-rank routed rows actually dispatched: after_max,
                                except in the sampled rerouting mode */
  int64_t cap;               /* cap C of the chosen candidate */
  int64_t assignments;       /* A: counted (valid) (token, k) assignments */
  int64_t rows;              /* dispatch rows: A, plus R*T with a shared expert */
  int64_t before_max;        /* max per-rank load with natives only */
  int64_t after_max;         /* max per-rank routed load after balancing */
} ep_layer_stats;

/*
 * Device pointers into the plan workspace for one layer (valid until the
 * workspace is freed; contents valid after ep_balance_layer completes on the
 * stream).  G = Gmax + S + shared columns per rank; global instance index
 * i = q*G + col, "instance order" = ascending i.  int32 everywhere.
 */
typedef struct ep_layer_view {
  const int32_t* load;          /* [R][E] load matrix L[r][e] ([U] §"real load") */
  const int32_t* expert_total;  /* [E] per-expert assignments */
  const int32_t* rank_load_before; /* [R] natives-only load W0 */
  const int32_t* rank_load;     /* [R] routed load W after the solve */
  const int32_t* inst_expert;   /* [R][G] expert of each instance: natives ascending, -1
                                   padding, slots in creation order (-1 empty), E = shared */
  const int32_t* inst_quota;    /* [R][G] quota (tokens) of each instance */
  const int32_t* inst_off;      /* [R*G+1] first dispatch row of each instance */
  const int32_t* rank_row_begin;/* [R+1] first dispatch row of each destination rank */
  const int32_t* dst_row;       /* [R][T][K] dispatch row of each (token, k), -1 if bad id */
  const int32_t* shared_rank;   /* [R][T] Waterfill rank of each token (NULL if none) */
  const int32_t* shared_row;    /* [R][T] dispatch row of the shared slot (NULL if none) */
  const int32_t* cand_max_load; /* [J] each cap candidate's max rank load */
  const int32_t* cand_replicas; /* [J] each candidate's replica count */
  const int32_t* cand_stop;     /* [J] each candidate's stop reason */
  const int32_t* replica_list;  /* [R*S] slot index q*S+s of every replica, grouped by expert
                                   (ascending), instance order inside an expert */
  const int32_t* replica_expert_ptr; /* [E+1] CSR offsets of replica_list by expert */
  const ep_layer_stats* stats;  /* device copy of the layer's stats */
  const int32_t* inst_count;    /* [R][G] rows each instance receives (inst_off's steps):
                                   inst_quota itself except in the sampled rerouting mode */
  int32_t Gmax, G;              /* natives per rank (max) and columns per rank */
} ep_layer_view;

typedef struct ep_plan ep_plan; /* opaque */

/* Workspace bytes a plan for `cfg` needs (device memory the caller allocates,
 * 256-byte aligned).  EP_ERR_UNSUPPORTED / EP_ERR_INVALID_ARGUMENT on a bad cfg. */
EP_API ep_status_t ep_plan_workspace_bytes(const ep_config* cfg, size_t* bytes);

/* Create a plan over caller-owned device workspace `d_workspace` (>= the size
 * above, 256-byte aligned).  Uses the current CUDA device.  Writes *out.
 * The copy kernels (dispatch, combine, staging, reduction) size their grids
 * by the device's SM count; if the environment variable EP_GRID_SMS holds an
 * integer in [1, 4096] when the plan is created, that count is used instead.
 * No result depends on it (every output element is written by one thread of
 * a grid-stride loop); it exists to test exactly that.
 * If EP_DISPATCH_IMPL is "bulk" when the plan is created, ep_dispatch_layout
 * and ep_dispatch_tokens move the rows with the bulk-copy (TMA) engine through
 * a ring of shared-memory row buffers instead of staging them in registers
 * (same results; measured slower on B200, kept to reproduce that
 * measurement).  It falls back to the register path when four rows do not
 * fit in shared memory or K + 1 > 32. */
EP_API ep_status_t ep_plan_create(const ep_config* cfg, void* d_workspace, size_t workspace_bytes,
                           ep_plan** out);

EP_API void ep_plan_destroy(ep_plan* plan);

/*
 * Balance one layer ([U] §"Getting the real load", §"Quota", local-first
 * rerouting; [W] §"Waterfill" when shared_expert = 1): from gate top-k ids
 * d_topk_ids [R][T][K] int32 (device, C-contiguous), build the load matrix,
 * solve replica placement and per-instance quotas, reroute local-first, and
 * assign every (token, k) its dispatch row, all into the layer's slot of the
 * plan cache (overwriting it).  Every rank would compute this identically.
 * Calls on one plan share its scratch: they must not overlap on the GPU (one
 * stream, or streams ordered by events).  The first call of a plan zeroes the
 * scratch accumulators with one cudaMemsetAsync on `stream`; a call whose
 * launch fails (EP_ERR_CUDA) makes the next call zero them again.
 */
EP_API ep_status_t ep_balance_layer(ep_plan* plan, int32_t layer, const int32_t* d_topk_ids,
                             void* stream);

/* Device pointers of a layer's cached plan (no GPU work). */
EP_API ep_status_t ep_layer_view_get(const ep_plan* plan, int32_t layer, ep_layer_view* out);

/* Copy a layer's stats to the host; synchronises `stream`.  Returns
 * EP_ERR_DEVICE_STATUS (after filling *h_out) if any status bit is set. */
EP_API ep_status_t ep_read_layer_stats(ep_plan* plan, int32_t layer, ep_layer_stats* h_out,
                                void* stream);

/*
 * Token dispatch layout ([U]: dispatch starts once replicas are in place; [W]
 * §"Shared expert fusion": the shared slot sits beside each rank's routed
 * experts).  out[row - rank_row_begin[b]] = hidden[r*T + t] for every row of
 * destination ranks [b, e) = [dst_rank_begin, dst_rank_end): a bitwise copy of
 * bf16 rows of `hidden` elements.  d_hidden [R*T][hidden], d_out must hold the
 * rank range's rows; out_rows_capacity is its size in rows (rows beyond it are
 * skipped and flag EP_DEV_OUT_CAPACITY).  The whole layout is b = 0, e = R.
 */
EP_API ep_status_t ep_dispatch_layout(ep_plan* plan, int32_t layer, const void* d_hidden, void* d_out,
                               int64_t out_rows_capacity, int32_t dst_rank_begin,
                               int32_t dst_rank_end, void* stream);

/*
 * Token-range dispatch: the rows of source tokens n in [token_begin,
 * token_end) only (n = r*T + t), for every destination rank:
 * out[row] = hidden[n] for each dispatch row (routed and shared) of those
 * tokens; rows of other tokens are not touched.  The pages have no
 * counterpart: it lets a caller dispatch the tokens whose hidden states have
 * arrived while the rest are still being copied in.  d_hidden is the whole
 * [R*T][hidden] buffer (only the range's rows are read); d_out holds the whole
 * layout (rows_total rows), out_rows_capacity its size in rows (rows beyond it
 * are skipped and flag EP_DEV_OUT_CAPACITY).  An empty range does nothing.
 * Errors: EP_ERR_INVALID_ARGUMENT for token_begin < 0, token_end > R*T,
 * token_begin > token_end, a null or non-16-byte-aligned buffer (for a
 * non-empty range); EP_ERR_NOT_PLANNED before ep_balance_layer.
 */
EP_API ep_status_t ep_dispatch_tokens(ep_plan* plan, int32_t layer, const void* d_hidden,
                               int64_t token_begin, int64_t token_end, void* d_out,
                               int64_t out_rows_capacity, void* stream);

/*
 * Replica weight staging ([U] §"Shared redundant slots": hot experts' weights
 * are written into the reserved slots, shared by all layers; backward re-stages
 * from the cached forward plan): d_slots[q][s] = d_native_w[expert of slot (q,s)]
 * for every slot the layer filled; empty slots are untouched.  d_native_w
 * [E][Wn] bf16, d_slots [R][S][Wn] bf16 (the cross-layer shared buffer).
 */
EP_API ep_status_t ep_stage_replicas(ep_plan* plan, int32_t layer, const void* d_native_w,
                              void* d_slots, void* stream);

/*
 * Replica gradient reduction ([U] §"Reusing the forward plan": replica
 * gradients are reduced into the native expert's gradient buffer, then the
 * redundant gradient buffer is cleared): for every expert e with replicas and
 * every element j, acc = native[e][j]; acc = acc + (float)g[replica][j] for the
 * replicas in instance order, one fp32 add at a time (round to nearest even);
 * native[e][j] = acc; then the layer's filled slot gradients are zeroed.
 * d_slot_grads [R][S][Wn] of grad_dtype (0 = bf16, 1 = fp32), d_native_grads
 * [E][Wn] fp32.
 */
EP_API ep_status_t ep_reduce_replica_grads(ep_plan* plan, int32_t layer, void* d_slot_grads,
                                    int32_t grad_dtype, float* d_native_grads, void* stream);

/*
 * Combine, the reverse of ep_dispatch_layout ([W] §"Shared expert fusion":
 * routed and shared experts share one dispatch -> grouped GEMM -> combine
 * flow; [U]: dispatch by the rerouting plan): after expert compute, dispatch
 * row i of d_expert_out [rows][hidden] bf16 holds its expert's output for the
 * (token, k) that was sent there.  For every token n = r*T + t:
 *   out[n] = sum over k ascending of w[r][t][k] * x[dst_row[r][t][k]]
 *            (+ x[shared_row[r][t]] with weight 1 when the layer has a shared
 *            expert),
 * accumulated in fp32, one fused multiply-add per k in ascending k, the shared
 * row added last; rows of dropped ids (-1) contribute nothing.  d_weights
 * [R][T][K] fp32 (the gate's top-k weights); d_out [R*T][hidden] of out_dtype
 * (0 = bf16, round to nearest even; 1 = fp32).  All buffers 16-byte aligned.
 */
EP_API ep_status_t ep_combine(ep_plan* plan, int32_t layer, const void* d_expert_out,
                              const float* d_weights, void* d_out, int32_t out_dtype,
                              void* stream);

/*
 * Standalone Waterfill ([W] §"Waterfill"): for routed per-rank loads d_load [R]
 * (int32) and the destination rank of every routed assignment d_dst_rank
 * [R][T][K] (int32, -1 = none), pick each token's shared-expert rank:
 * H = ceil((sum L + R*T)/R), slack S_r = max(H - L_r, 0), B = ceil(H*bonus/1000);
 * candidates = own rank, then the other ranks the token visits, ascending; draw
 * proportional to slack (+B on the own rank) with u = ((h>>32)*sum)>>32,
 * h = SplitMix64(seed + r*T + t); with no slack, the least-loaded candidate
 * unless the own rank is within B of it.  flags bit 0 (EP_WATERFILL_ALL_RANKS):
 * every rank is a candidate ([W]'s all-rank mode), own rank first.  Writes
 * d_pick [R][T] and d_count [R] (tokens per rank).  Limits: R <= 128, K <= 16,
 * R*T*(K+1) < 2^31.
 */
#define EP_WATERFILL_ALL_RANKS 1
EP_API ep_status_t ep_waterfill(int32_t R, int32_t T, int32_t K, const int32_t* d_load,
                         const int32_t* d_dst_rank, uint64_t seed, int32_t bonus_permille,
                         int32_t flags, int32_t* d_pick, int32_t* d_count, void* stream);

/*
 * Waterfill re-run of a cached layer ([W] §"Waterfill"; [U] §"Reusing the
 * forward plan": the layer's routed plan is kept and reused): re-draws every
 * token's shared-expert rank of `layer` with `seed` in place of the plan's
 * waterfill_seed — same candidates, waterline, slack, local preference and
 * fallback as the pass inside ep_balance_layer, on the layer's routed rows and
 * planned per-rank loads — and lays the shared columns out again.  Every rank's
 * block keeps its routed rows in order; blocks shift with the new shared-column
 * sizes, so the layer's dst_row, shared_rank, shared_row, the shared columns'
 * inst_quota / inst_count, inst_off, rank_row_begin and stats.rows are all
 * rewritten.  The result equals ep_balance_layer on the same ids with
 * waterfill_seed = seed.  EP_ERR_UNSUPPORTED without a shared expert,
 * EP_ERR_NOT_PLANNED before the layer's ep_balance_layer.  Uses the plan's
 * scratch: must not overlap other calls on the plan.  Asynchronous on `stream`.
 */
EP_API ep_status_t ep_waterfill_layer(ep_plan* plan, int32_t layer, uint64_t seed, void* stream);

/*
 * Load matrix without allocation.  The pages have no counterpart: this exists
 * for callers that cannot allocate device memory on this path (engines that
 * reserve nearly all device memory up front, embedded callers without an
 * allocator, loops where an allocation would synchronise the device).
 * Computes d_load[r][e] = number of (t, k) with d_topk_ids[r][t][k] == e — the
 * same values as ep_layer_view.load after ep_balance_layer — from d_topk_ids
 * [R][T][K] int32 into d_load [R][E] int32 (both caller-owned device memory).
 * d_status (device int32, may be NULL) is set to EP_DEV_BAD_ID if an id was
 * outside [0, E), else 0; such ids are not counted.
 * It calls no allocator: its only scratch, R*ceil(T/128)*E int32 sub-chunk
 * counts, lives in a fixed device array of EP_LOAD_STATIC_MAX_SCRATCH int32
 * (4 MiB) that every GPU loading the library holds until the process exits;
 * larger shapes return EP_ERR_UNSUPPORTED.  The first call on each device looks
 * up the array's address (cudaGetSymbolAddress) — make that first call before
 * any stream capture.  The address is cached with the id of the CUDA context
 * it belongs to; after a device reset the next call looks it up again, so make
 * that call, too, before any capture.  All calls on a device share the array;
 * calls that overlap on the GPU race and must be serialised by the caller.
 * Limits: R >= 1, 1 <= E <= 1024, 1 <= K <= 16, T >= 0, R*T*K < 2^31,
 * R*E < 2^31.  Asynchronous on `stream`; EP_ERR_CUDA reports a failure of this
 * call's own memset or launches only (an error left pending by earlier,
 * unrelated work is not reported and not cleared).
 */
#define EP_LOAD_STATIC_MAX_SCRATCH (1 << 20)
EP_API ep_status_t ep_load_matrix_static(int32_t R, int32_t E, int32_t K, int32_t T,
                                         const int32_t* d_topk_ids, int32_t* d_load,
                                         int32_t* d_status, void* stream);

EP_API const char* ep_status_string(ep_status_t status);
EP_API int32_t ep_abi_version(void);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* EP_BALANCE_H_ */
