// HBM-bound data movement for sm_100a: dispatch permutation of hidden rows,
// replica weight staging into the shared slots, replica gradient reduction.
//
// Dispatch (UltraEP page, "300 µs to level MoE expert load": token dispatch
// starts once replicas are in place; Waterfill page §"Shared expert fusion":
// the shared slot is one more column of every rank's block) and staging
// (§"Shared redundant slots manage dynamic replicas"; §"Streaming
// communication kernels": a persistent kernel pulls fixed-size tiles from a
// device-side task list, double-buffered) are whole-row / whole-tile bit copies.
// Both move data with the Blackwell bulk-copy engine: one warp per CTA issues
// cp.async.bulk global->shared loads completing on an mbarrier, then
// cp.async.bulk shared->global stores, one per destination, so each source
// byte is read from HBM once and written once per destination.  No load uses
// cluster multicast.  Every mbarrier wait is bounded; on timeout the kernel
// sets EP_DEV_WAIT_TIMEOUT, waits (bounded) for the copies it issued and exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
#ifndef EP_COPY_STAGES
#define EP_COPY_STAGES 4
#endif
#ifndef EP_PERMUTE_SMEM_BUDGET
#define EP_PERMUTE_SMEM_BUDGET (200 * 1024)
#endif
constexpr int kStages = EP_COPY_STAGES;     // row / tile buffers per CTA
constexpr uint32_t kWaitSpins = 1u << 20;   // try_wait polls before giving up
constexpr int kStageTile = 16384;           // bytes per staging tile

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
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
// Bounded, warp-uniform wait on an mbarrier phase: every lane observes the
// completed phase (each lane may then issue bulk stores reading the buffer);
// false for the whole warp after kWaitSpins polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitSpins; ++i)
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  return false;
}
// Bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Bulk copy shared -> global, tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// All but the newest group of this thread have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// a6: dispatch permutation.  Each CTA (one warp) owns a contiguous range of
// tokens.  Token row n is loaded once into a stage buffer; lane k < K stores it
// to dispatch row dst_row[n][k], lane K to the shared-slot row, if the row falls
// in the destination-rank window [row_lo, row_hi).  Rows for a token are loaded
// only if at least one of its destinations is in the window.  The destination
// rows of a token are fetched when its load is issued, kStages tokens ahead.
// ---------------------------------------------------------------------------
struct PermuteArgs {
  const uint8_t* hidden;
  uint8_t* out;
  const int32_t* dst_row;
  const int32_t* shared_row;  // null without a shared expert
  const int32_t* rank_base;
  ep_layer_stats* stats;
  int64_t N;
  int64_t cap_rows;
  uint32_t row_bytes;
  int K;
  int rank_begin, rank_end;
};

__global__ void __launch_bounds__(32) k_permute(PermuteArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint8_t* buf = smem + 128;
  const int lane = threadIdx.x;
  const int row_lo = a.rank_base[a.rank_begin];
  const int row_hi = a.rank_base[a.rank_end];
  const int64_t per = (a.N + gridDim.x - 1) / gridDim.x;
  const int64_t n0 = (int64_t)blockIdx.x * per;
  const int64_t cnt = n0 < a.N ? min(per, a.N - n0) : 0;
  if (cnt <= 0) return;
  if (lane == 0) {
#pragma unroll
    for (int u = 0; u < kStages; ++u) mbar_init(&bars[u], 1);
    fence_barrier_init();
  }
  __syncwarp();
  const bool store_lane = lane < a.K || (lane == a.K && a.shared_row != nullptr);
  const uint32_t rb = a.row_bytes;
  // Per stage u: this lane's destination row of the token in the stage (or -1),
  // whether the token was loaded, and the barrier's next parity.
  int drow[kStages];
  bool need[kStages];
  uint32_t parity = 0;  // bit u: parity of stage u
  auto fetch_row = [&](int64_t n) -> int {
    int d = -1;
    if (lane < a.K) d = a.dst_row[n * a.K + lane];
    else if (store_lane) d = a.shared_row[n];
    return (d >= row_lo && d < row_hi) ? d : -1;
  };
  auto issue = [&](int u, int64_t i) {
    drow[u] = fetch_row(n0 + i);
    need[u] = __any_sync(kFull, drow[u] >= 0);
    if (need[u] && lane == 0) {
      mbar_expect_tx(&bars[u], rb);
      bulk_load(buf + (size_t)u * rb, a.hidden + (n0 + i) * (int64_t)rb, rb, &bars[u]);
    }
  };
#pragma unroll
  for (int u = 0; u < kStages; ++u) {
    need[u] = false;
    drow[u] = -1;
    if (u < cnt) issue(u, u);
  }
  bool timed_out = false, overflow = false;
  for (int64_t i0 = 0; i0 < cnt && !timed_out; i0 += kStages) {
#pragma unroll
    for (int u = 0; u < kStages; ++u) {
      const int64_t i = i0 + u;
      if (i >= cnt || timed_out) break;
      if (need[u]) {
        if (!mbar_wait(&bars[u], (parity >> u) & 1u)) {
          timed_out = true;
          break;
        }
        parity ^= 1u << u;
        const int d = drow[u];
        if (d >= 0) {
          const int64_t o = (int64_t)(d - row_lo);
          if (o < a.cap_rows) bulk_store(a.out + o * rb, buf + (size_t)u * rb, rb);
          else overflow = true;
        }
      }
      bulk_commit();
      // Refill the previous stage: its stores were committed one step ago.
      const int up = (u + kStages - 1) % kStages;
      const int64_t inext = i - 1 + kStages;
      if (i >= 1 && inext < cnt) {
        bulk_wait_read_1();
        __syncwarp();
        issue(up, inext);
      }
    }
  }
  bulk_wait_all();
  if (timed_out) {
    // Drain the loads still in flight (bounded) before the CTA exits.
#pragma unroll
    for (int u = 0; u < kStages; ++u)
      if (need[u]) mbar_wait(&bars[u], (parity >> u) & 1u);
    if (lane == 0) atomicOr(&a.stats->status, EP_DEV_WAIT_TIMEOUT);
  }
  if (__any_sync(kFull, overflow) && lane == 0) atomicOr(&a.stats->status, EP_DEV_OUT_CAPACITY);
}

// ---------------------------------------------------------------------------
// a7: replica weight staging as persistent tile streaming.  Task t = (replicated
// expert i, tile) from the device-side replica lists; the tile is loaded once and
// stored to every slot that holds a replica of the expert.
// ---------------------------------------------------------------------------
struct StageArgs {
  const uint8_t* native_w;
  uint8_t* slots;
  const int32_t* rep_nexp;
  const int32_t* rep_experts;
  const int32_t* rep_eptr;
  const int32_t* rep_list;
  ep_layer_stats* stats;
  int64_t expert_bytes;
};

__global__ void __launch_bounds__(32) k_stage(StageArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  uint8_t* buf = smem + 128;
  const int lane = threadIdx.x;
  const int64_t tiles = (a.expert_bytes + kStageTile - 1) / kStageTile;
  const int64_t total = (int64_t)a.rep_nexp[0] * tiles;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * per;
  const int64_t cnt = t0 < total ? min(per, total - t0) : 0;
  if (cnt <= 0) return;
  if (lane == 0) {
#pragma unroll
    for (int u = 0; u < kStages; ++u) mbar_init(&bars[u], 1);
    fence_barrier_init();
  }
  __syncwarp();
  uint32_t parity = 0;
  auto tile_of = [&](int64_t i, int& e, int64_t& off, uint32_t& bytes) {
    const int64_t t = t0 + i;
    const int64_t xi = t / tiles;
    off = (t - xi * tiles) * kStageTile;
    e = a.rep_experts[xi];
    bytes = (uint32_t)min((int64_t)kStageTile, a.expert_bytes - off);
  };
  auto issue = [&](int u, int64_t i) {
    if (lane == 0) {
      int e;
      int64_t off;
      uint32_t bytes;
      tile_of(i, e, off, bytes);
      mbar_expect_tx(&bars[u], bytes);
      bulk_load(buf + (size_t)u * kStageTile, a.native_w + (int64_t)e * a.expert_bytes + off, bytes,
                &bars[u]);
    }
  };
#pragma unroll
  for (int u = 0; u < kStages; ++u)
    if (u < cnt) issue(u, u);
  bool timed_out = false;
  for (int64_t i0 = 0; i0 < cnt && !timed_out; i0 += kStages) {
#pragma unroll
    for (int u = 0; u < kStages; ++u) {
      const int64_t i = i0 + u;
      if (i >= cnt || timed_out) break;
      if (!mbar_wait(&bars[u], (parity >> u) & 1u)) {
        timed_out = true;
        break;
      }
      parity ^= 1u << u;
      int e;
      int64_t off;
      uint32_t bytes;
      tile_of(i, e, off, bytes);
      const int p0 = a.rep_eptr[e], p1 = a.rep_eptr[e + 1];
      for (int p = p0 + lane; p < p1; p += 32)
        bulk_store(a.slots + (int64_t)a.rep_list[p] * a.expert_bytes + off,
                   buf + (size_t)u * kStageTile, bytes);
      bulk_commit();
      const int up = (u + kStages - 1) % kStages;
      const int64_t inext = i - 1 + kStages;
      if (i >= 1 && inext < cnt) {
        bulk_wait_read_1();
        __syncwarp();
        issue(up, inext);
      }
    }
  }
  bulk_wait_all();
  if (timed_out) {
    if (lane == 0) atomicOr(&a.stats->status, EP_DEV_WAIT_TIMEOUT);
  }
}

// ---------------------------------------------------------------------------
// a8: replica gradient reduction.  Task = (replicated expert, 2048 elements);
// thread = 8 consecutive elements.  acc = native; acc += replica in instance
// order, one round-to-nearest fp32 add at a time; then the replica gradients
// are zeroed.
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 256;

// The replica lists of the layer (at most R*S slots) are staged in shared
// memory once per block, so the streaming loops have no dependent global
// lookups.  Clearing a replica gradient in the thread that has just loaded it
// stalls the load/store pipeline on the in-flight line (measured: ~1.1 TB/s);
// so k_reduce only loads replica gradients, and k_clear_replicas zeroes them
// afterwards (together ~6 TB/s).
constexpr int kMaxRepSlots = kMaxR * kMaxS;

struct RepTables {
  int32_t exp[kMaxRepSlots];      // replicated expert i
  int32_t ptr[kMaxRepSlots + 1];  // its replicas: slot[ptr[i] .. ptr[i+1])
  int32_t slot[kMaxRepSlots];     // slot index q*S + s, instance order
};

__device__ __forceinline__ int stage_rep_tables(RepTables& t, const int32_t* rep_nexp,
                                                const int32_t* rep_experts, const int32_t* rep_eptr,
                                                const int32_t* rep_list, int E) {
  const int nexp = rep_nexp[0];
  for (int i = threadIdx.x; i < nexp; i += blockDim.x) {
    const int e = rep_experts[i];
    t.exp[i] = e;
    t.ptr[i] = rep_eptr[e];
  }
  const int nrep = rep_eptr[E];
  if (threadIdx.x == 0) t.ptr[nexp] = nrep;
  for (int i = threadIdx.x; i < nrep; i += blockDim.x) t.slot[i] = rep_list[i];
  __syncthreads();
  return nexp;
}

// 8 gradient values of one replica: bf16 in one 16-byte word, fp32 in two.
template <bool F32>
struct Raw8 {
  uint4 a, b;
};

template <bool F32>
__device__ __forceinline__ Raw8<F32> load8(const void* g, int64_t base) {
  Raw8<F32> r;
  if (F32) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(g) + base);
    r.a = p[0];
    r.b = p[1];
  } else {
    r.a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g) + base);
    r.b = r.a;
  }
  return r;
}

template <bool F32>
__device__ __forceinline__ void add8(float (&acc)[8], const Raw8<F32>& r) {
  const uint32_t w[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float v = F32 ? __uint_as_float(w[i])
                        : __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
    acc[i] = __fadd_rn(acc[i], v);  // instance order, one round-to-nearest add each
  }
}

template <bool F32>
__global__ void __launch_bounds__(kReduceThreads)
k_reduce(const int32_t* __restrict__ rep_nexp, const int32_t* __restrict__ rep_experts,
         const int32_t* __restrict__ rep_eptr, const int32_t* __restrict__ rep_list,
         const void* __restrict__ slot_grads, float* __restrict__ native, int64_t Wn, int E) {
  constexpr int kB = F32 ? 4 : 8;  // replica loads issued together
  __shared__ RepTables t;
  const int nexp = stage_rep_tables(t, rep_nexp, rep_experts, rep_eptr, rep_list, E);
  const uint32_t vpe = (uint32_t)(Wn / 8);
  const uint32_t total = (uint32_t)nexp * vpe;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t v = blockIdx.x * blockDim.x + threadIdx.x; v < total; v += stride) {
    const uint32_t xi = v / vpe;
    const int64_t j = (int64_t)(v - xi * vpe) * 8;
    const int e = t.exp[xi];
    const int p0 = t.ptr[xi], p1 = t.ptr[xi + 1];
    float4* nat = reinterpret_cast<float4*>(native + (int64_t)e * Wn + j);
    const float4 n0 = nat[0], n1 = nat[1];
    float acc[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
    for (int p = p0; p < p1; p += kB) {
      Raw8<F32> r[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u)
        if (p + u < p1) r[u] = load8<F32>(slot_grads, (int64_t)t.slot[p + u] * Wn + j);
#pragma unroll
      for (int u = 0; u < kB; ++u)
        if (p + u < p1) add8<F32>(acc, r[u]);
    }
    nat[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    nat[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// Zero every filled replica slot's gradient (16-byte stores).
__global__ void __launch_bounds__(kReduceThreads)
k_clear_replicas(const int32_t* __restrict__ rep_nexp, const int32_t* __restrict__ rep_experts,
                 const int32_t* __restrict__ rep_eptr, const int32_t* __restrict__ rep_list,
                 uint4* slot_grads, int64_t slot_words, int E) {
  __shared__ RepTables t;
  stage_rep_tables(t, rep_nexp, rep_experts, rep_eptr, rep_list, E);
  const int nrep = rep_eptr[E];
  const uint64_t total = (uint64_t)nrep * (uint64_t)slot_words;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t w = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; w < total; w += stride) {
    const uint64_t p = w / (uint64_t)slot_words;
    slot_grads[(uint64_t)t.slot[p] * slot_words + (w - p * slot_words)] = make_uint4(0u, 0u, 0u, 0u);
  }
}

int permute_ctas_per_sm(uint32_t row_bytes) {
  const size_t smem = 128 + (size_t)kStages * row_bytes;
  int c = (int)((size_t)EP_PERMUTE_SMEM_BUDGET / smem);
  if (c > 16) c = 16;
  if (c < 1) c = 1;
  return c;
}

}  // namespace

cudaError_t set_copy_attributes(int max_smem) {
  cudaError_t e = allow_max_dynamic_smem(k_permute, max_smem);
  if (e != cudaSuccess) return e;
  return allow_max_dynamic_smem(k_stage, max_smem);
}

cudaError_t launch_dispatch(const Dims& d, const LayerBuf& L, const void* hidden, void* out,
                            int64_t cap_rows, int rank_begin, int rank_end, int num_sms,
                            cudaStream_t st) {
  PermuteArgs a;
  a.hidden = static_cast<const uint8_t*>(hidden);
  a.out = static_cast<uint8_t*>(out);
  a.dst_row = L.dst_row;
  a.shared_row = d.sh ? L.shared_row : nullptr;
  a.rank_base = L.rank_base;
  a.stats = L.stats;
  a.N = (int64_t)d.R * d.T;
  a.cap_rows = cap_rows;
  a.row_bytes = (uint32_t)d.hidden * 2u;
  a.K = d.K;
  a.rank_begin = rank_begin;
  a.rank_end = rank_end;
  if (a.N == 0) return cudaSuccess;
  const int per_sm = permute_ctas_per_sm(a.row_bytes);
  int64_t grid = (int64_t)num_sms * per_sm;
  if (grid > a.N) grid = a.N;
  const size_t smem = 128 + (size_t)kStages * a.row_bytes;
  k_permute<<<(unsigned)grid, 32, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_stage(const Dims& d, const LayerBuf& L, const void* native_w, void* slots,
                         int num_sms, cudaStream_t st) {
  if (d.Wn == 0 || d.S == 0) return cudaSuccess;
  StageArgs a;
  a.native_w = static_cast<const uint8_t*>(native_w);
  a.slots = static_cast<uint8_t*>(slots);
  a.rep_nexp = L.rep_nexp;
  a.rep_experts = L.rep_experts;
  a.rep_eptr = L.rep_eptr;
  a.rep_list = L.rep_list;
  a.stats = L.stats;
  a.expert_bytes = d.Wn * 2;
  k_stage<<<(unsigned)(num_sms * 3), 32, 128 + kStages * kStageTile, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_reduce(const Dims& d, const LayerBuf& L, void* slot_grads, int grad_f32,
                          float* native_grads, int num_sms, cudaStream_t st) {
  if (d.Wn == 0 || d.S == 0) return cudaSuccess;
  int per_sm = 0;
  cudaError_t e = grad_f32 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_reduce<true>,
                                                                          kReduceThreads, 0)
                           : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_reduce<false>,
                                                                          kReduceThreads, 0);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(num_sms * (per_sm > 0 ? per_sm : 1));
  if (grad_f32)
    k_reduce<true><<<grid, kReduceThreads, 0, st>>>(L.rep_nexp, L.rep_experts, L.rep_eptr,
                                                    L.rep_list, slot_grads, native_grads, d.Wn, d.E);
  else
    k_reduce<false><<<grid, kReduceThreads, 0, st>>>(L.rep_nexp, L.rep_experts, L.rep_eptr,
                                                     L.rep_list, slot_grads, native_grads, d.Wn, d.E);
  const int64_t slot_words = d.Wn * (grad_f32 ? 4 : 2) / 16;
  k_clear_replicas<<<(unsigned)(num_sms * 4), kReduceThreads, 0, st>>>(
      L.rep_nexp, L.rep_experts, L.rep_eptr, L.rep_list, static_cast<uint4*>(slot_grads), slot_words,
      d.E);
  return cudaGetLastError();
}

}  // namespace ep
