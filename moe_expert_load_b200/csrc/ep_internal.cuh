// Internal definitions shared by the CUDA translation units of libep_b200.
// Not part of the public ABI (include/ep_balance.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep_balance.h"

namespace ep {

constexpr int kSubT = 128;      // tokens per sub-chunk of the static load-matrix variant
constexpr int kPlanSubT = 64;   // tokens per sub-chunk of the plan kernels (one warp each)
constexpr int kPlanWarps = 8;   // sub-chunks (warps) per block of the plan kernels
constexpr int kMaxR = 128;      // ranks (4 words of 32 per warp lane)
constexpr int kRW = 4;          // rank words per lane: lane owns ranks lane + 32*k
constexpr int kMaxE = 1024;
constexpr int kMaxK = 16;
constexpr int kMaxS = 8;
constexpr int kMaxJ = 16;
constexpr int kMaxNat = 32;     // natives per rank: one warp lane each in the solver
constexpr int kNoRank = 0xFF;   // "no destination" in uint8 rank buffers

// Problem dimensions, passed by value to every kernel.
struct Dims {
  int R, E, K, T;
  int S, m, J;
  int Gmax, G, sh;   // natives per rank (max), columns per rank, shared column present
  int nsub;          // sub-chunks per rank = ceil(T / kPlanSubT)
  int bonus;         // Waterfill local preference, permille
  int hidden;        // bf16 elements per hidden row
  int all_ranks;     // Waterfill candidates: every rank
  uint64_t seed;     // Waterfill draw seed
  int64_t Wn;        // bf16 elements per expert
  int sampled;       // rerouting mode: 1 = each assignment samples an instance
  int iter_limit;    // > 0: the solver's iteration bound instead of 4(RS+R+E)+64
  uint64_t sseed;    // seed of the sampled mode's per-assignment draw
  int nkey;          // sampled mode: key space E + R*S (expert-major instance keys)
  int solve_smem;    // dynamic shared memory of the solve launch (set at plan creation)
  int fix_grid;      // blocks of the shared-slot fix-up: those resident at once (plan creation)
};

// One layer's slot in the plan cache (all device pointers).
struct LayerBuf {
  int32_t* load;          // [R][E]
  int32_t* expert_total;  // [E]
  int32_t* W0;            // [R]
  int32_t* W;             // [R]
  int32_t* inst_expert;   // [R][G]
  int32_t* inst_quota;    // [R][G]
  int32_t* inst_off;      // [R*G+1]
  int32_t* rank_base;     // [R+1]
  int32_t* dst_row;       // [R][T][K]
  int32_t* shared_rank;   // [R][T] or null
  int32_t* shared_row;    // [R][T] or null
  int32_t* cand;          // [3][J]: max load, replicas, stop reason
  int32_t* rep_list;      // [R*S] slot ids grouped by expert, instance order within
  int32_t* rep_eptr;      // [E+1]
  int32_t* rep_nexp;      // [1] number of replicated experts
  int32_t* rep_experts;   // [R*S] replicated experts, ascending
  int32_t* inst_count;    // [R][G] rows per instance (sampled mode; else inst_quota)
  ep_layer_stats* stats;
};

// Scratch shared by all layers, reused by every balance call.
struct Scratch {
  int32_t* sub_cnt;   // [R][nsub][E] per-sub-chunk counts
  int32_t* blk_cnt;   // [R][ceil(nsub/kPlanWarps)][E] per-block counts
  int32_t* wsub_cnt;  // [R][R*nsub] shared-slot counts per (dest rank, sub-chunk), then bases
  int32_t* seg_rec;   // [R][E][8] per (source rank, expert): the first two segments
                      // and where the third begins, as two int4 records
  int32_t* seg_ord;   // [E][3R] first ordinal of the segment
  int32_t* seg_rank;  // [E][3R] destination rank
  int32_t* seg_base;  // [E][3R] first row minus first ordinal: absolute without a shared
                      // expert, relative to the destination rank's block with one
  int32_t* inst_rel;  // [R*G] first row of an instance inside its rank's block
  int32_t* slack;     // [R] Waterfill slack
  int32_t* wf;        // [2] Waterfill H, B
  int32_t* sbase;     // [R] first row of each rank's shared column
  int32_t* shared_tot;  // [R] shared-slot rows per destination rank
  uint8_t* asg_rank;    // [R][T][K] destination rank of each assignment (shared expert only)
  // Accumulators that are zero whenever no balance call is running: the
  // histogram adds into the load matrix, the rerouting copies it out to the
  // layer and zeroes it again, the solve moves the status bits, and the
  // arrival ticket resets itself.
  int32_t* acc_load;    // [R][E]
  int32_t* acc_misc;    // [0] status bits of the histogram, [1] arrival ticket
  // Sampled rerouting mode only.  An instance key is kappa = e + rep_eptr[e] + j
  // for the j-th instance of expert e in instance order (E + R*S keys at most).
  int32_t* smp_tot;     // [R][nkey] draws per (source rank, key): an accumulator,
                        // zero between calls like the ones above
  int32_t* smp_cum;     // [nkey] running quota sum of the key's expert, inclusive
  int32_t* smp_inst;    // [nkey] global instance index of the key
  uint16_t* smp_key;    // [R][T][K] key drawn by each assignment (0xFFFF: dropped id)
  int32_t* smp_sub;     // [R][nsub][nkey] draws per sub-chunk
  int32_t* smp_blk;     // [R][ceil(nsub/kPlanWarps)][nkey] draws per block
  int32_t* smp_row0;    // [R][nkey] first row of (source rank, key) (rank-relative
                        // with a shared expert)
  int32_t* rank_rows;   // [R] routed rows per destination rank
  int32_t* prev_base;   // [R+1] a cached layer's rank bases before a Waterfill re-run
};

// ---- native placement: contiguous balanced blocks ---------------------------
__host__ __device__ __forceinline__ int nat_count(int q, int E, int R) {
  return E / R + (q < E % R ? 1 : 0);
}
__host__ __device__ __forceinline__ int nat_first(int q, int E, int R) {
  return q * (E / R) + (q < E % R ? q : E % R);
}
__host__ __device__ __forceinline__ int home_of(int e, int E, int R) {
  const int base = E / R, rem = E % R;
  const int big = rem * (base + 1);  // experts held by the first rem ranks
  return e < big ? e / (base + 1) : rem + (e - big) / base;
}

// Let kernel f request up to the device's opt-in shared memory per block:
// static + dynamic shared memory may not exceed it, so the dynamic allowance is
// the opt-in maximum minus f's static shared memory.
template <typename F>
inline cudaError_t allow_max_dynamic_smem(F* f, int max_smem) {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, f);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              max_smem - (int)a.sharedSizeBytes);
}

// ---- launchers (defined in the .cu files) ----------------------------------
cudaError_t launch_balance(const Dims& d, const LayerBuf& L, const Scratch& s,
                           const int32_t* ids, cudaStream_t st);
cudaError_t launch_dispatch(const Dims& d, const LayerBuf& L, const void* hidden, void* out,
                            int64_t cap_rows, int rank_begin, int rank_end, int64_t token_begin,
                            int64_t token_end, int num_sms, int bulk, cudaStream_t st);
cudaError_t launch_combine(const Dims& d, const LayerBuf& L, const void* x, const float* w, void* out,
                           int out_f32, int num_sms, cudaStream_t st);
cudaError_t launch_stage(const Dims& d, const LayerBuf& L, const void* native_w, void* slots,
                         int num_sms, cudaStream_t st);
cudaError_t launch_reduce(const Dims& d, const LayerBuf& L, void* slot_grads, int grad_f32,
                          float* native_grads, int num_sms, cudaStream_t st);
cudaError_t launch_waterfill_layer(const Dims& d, const LayerBuf& L, const Scratch& s,
                                   cudaStream_t st);
cudaError_t launch_waterfill(int R, int T, int K, const int32_t* load, const int32_t* dst_rank,
                             uint64_t seed, int bonus, int all_ranks, int32_t* pick, int32_t* count,
                             cudaStream_t st);

}  // namespace ep
