// HBM-bound data movement for sm_100a: dispatch permutation of hidden rows,
// its reverse (the gate-weighted combine), replica weight staging into the
// shared slots, replica gradient reduction.
//
// Dispatch (UltraEP page, "300 µs to level MoE expert load": token dispatch
// starts once replicas are in place; Waterfill page §"Shared expert fusion":
// the shared slot is one more column of every rank's block) and staging
// (§"Shared redundant slots manage dynamic replicas"; §"Streaming
// communication kernels": a persistent kernel pulls fixed-size tiles from a
// device-side task list) are whole-row / whole-tile bit copies in which each
// source byte is read from HBM once and written once per destination: a warp
// stages a slice of the row (or tile) in registers with vector loads and
// stores it to every destination with vector stores.  See k_permute for the
// measurements that chose this over bulk-copy (TMA) staging through shared
// memory.  Nothing here waits on another thread, block or device.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// a6: dispatch permutation.  One warp per token at a time (grid-stride over
// the tokens [n0, N) of the call): lanes 0..K-1 fetch the token's K dispatch rows, lane K its
// shared-slot row, keeping those inside the destination-rank window
// [row_lo, row_hi); the warp loads the bf16 row once into registers (32-byte
// vector loads, 4 KiB per pass, where the row size and both buffers are
// 32-byte aligned; else 16-byte loads, 8 KiB per pass) and stores it to every
// kept row with vector stores of the same width.  Tokens with no row in the
// window are not read.
//
// Measured on B200 (qwen, 19.3 GB per launch): this register-staged form moves
// 6.1-6.2 TB/s with 16-byte vectors; the same copy with bulk-copy (TMA) loads into shared memory
// and bulk stores stayed at 5.6-5.7 TB/s for every stage count (2-8) and
// occupancy tried, and TMA loads with vector stores from shared memory at
// 5.3-5.5 TB/s, so the bulk-copy engine is not used for this 1:K fan-out.
// ---------------------------------------------------------------------------
struct PermuteArgs {
  const uint4* hidden;
  uint4* out;
  const int32_t* dst_row;
  const int32_t* shared_row;  // null without a shared expert
  const int32_t* rank_base;
  ep_layer_stats* stats;
  int64_t n0, N;  // tokens [n0, N)
  int64_t cap_rows;
  int row16;  // 16-byte words per row
  int K;
  int rank_begin, rank_end;
};

constexpr int kPermuteThreads = 128;

// 32-byte vectors (ld/st.global.v8.b32, sm_100): rows and both buffers must be
// 32-byte aligned.
struct Vec32 {
  uint32_t x[8];
};
__device__ __forceinline__ Vec32 load32(const Vec32* p) {
  Vec32 v;
  asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v.x[0]), "=r"(v.x[1]), "=r"(v.x[2]), "=r"(v.x[3]), "=r"(v.x[4]),
                 "=r"(v.x[5]), "=r"(v.x[6]), "=r"(v.x[7])
               : "l"(p));
  return v;
}
__device__ __forceinline__ void store32(Vec32* p, const Vec32& v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.x[0]),
               "r"(v.x[1]), "r"(v.x[2]), "r"(v.x[3]), "r"(v.x[4]), "r"(v.x[5]), "r"(v.x[6]),
               "r"(v.x[7])
               : "memory");
}
__device__ __forceinline__ uint4 load32(const uint4* p) { return *p; }
__device__ __forceinline__ void store32(uint4* p, const uint4& v) { *p = v; }

// Words per lane per pass: 4 x 32 B (4 KiB per warp pass) with 32-byte
// vectors, 16 x 16 B (8 KiB) otherwise.  Measured on the qwen / dsv3 layers:
// 6.28-6.30 / 6.22-6.25 TB/s with 4 x 32 B, 6.13 / 6.09 with 16 x 16 B, 5.7 /
// 5.6 with 8 x 32 B (114 registers, lower occupancy).
template <typename W>
struct PermuteShape {
  static constexpr int kWordsPerLane = sizeof(W) == 32 ? 4 : 16;
};

template <typename W>
__global__ void __launch_bounds__(kPermuteThreads) k_permute(PermuteArgs a) {
  constexpr int kWPL = PermuteShape<W>::kWordsPerLane;
  const int lane = threadIdx.x & 31;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int row_lo = a.rank_base[a.rank_begin];
  const int row_hi = a.rank_base[a.rank_end];
  const int roww = a.row16 * 16 / (int)sizeof(W);  // words of W per row
  const W* hidden = reinterpret_cast<const W*>(a.hidden);
  W* out = reinterpret_cast<W*>(a.out);
  bool overflow = false;
  for (int64_t n = a.n0 + (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); n < a.N; n += nw) {
    int d = -1;
    if (lane < a.K) d = a.dst_row[n * a.K + lane];
    else if (lane == a.K && a.shared_row != nullptr) d = a.shared_row[n];
    d = (d >= row_lo && d < row_hi) ? d - row_lo : -1;
    if (d >= a.cap_rows) {
      overflow = true;
      d = -1;
    }
    const unsigned m = __ballot_sync(kFull, d >= 0);
    if (!m) continue;
    const W* src = hidden + n * roww;
    for (int c0 = 0; c0 < roww; c0 += kWPL * 32) {
      W v[kWPL];
#pragma unroll
      for (int k = 0; k < kWPL; ++k) {
        const int idx = c0 + k * 32 + lane;
        if (idx < roww) v[k] = load32(src + idx);
      }
      unsigned mm = m;
      while (mm) {
        const int from = __ffs(mm) - 1;
        mm &= mm - 1;
        W* dst = out + (int64_t)__shfl_sync(kFull, d, from) * roww;
#pragma unroll
        for (int k = 0; k < kWPL; ++k) {
          const int idx = c0 + k * 32 + lane;
          if (idx < roww) store32(dst + idx, v[k]);
        }
      }
    }
  }
  if (__any_sync(kFull, overflow) && lane == 0) atomicOr(&a.stats->status, EP_DEV_OUT_CAPACITY);
}

// ---------------------------------------------------------------------------
// a6, bulk-copy variant (EP_DISPATCH_IMPL=bulk at plan creation): the same
// permutation moved by the bulk-copy (TMA) engine instead of registers.  One
// warp per CTA keeps a ring of NST row buffers in shared memory; lane 0 loads
// token j's row with cp.async.bulk (completion counted on the stage's
// mbarrier) LA tokens ahead of storing it, and stores each kept row with
// cp.async.bulk from shared memory, one bulk group per token; a stage is
// reused once the group that last read it has finished reading (NST - LA
// groups of slack).  Loads carry no multicast.  Every mbarrier wait is
// bounded: on timeout the kernel flags EP_DEV_WAIT_TIMEOUT, stops issuing,
// waits (bounded) for the loads it has in flight and returns.
// ---------------------------------------------------------------------------
constexpr int kBulkStages = 4;      // row buffers per CTA
constexpr int kBulkAhead = 2;       // tokens loaded ahead of the one being stored
constexpr uint32_t kBulkSpinLimit = 1u << 22;  // polls of one mbarrier before giving up

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait for the phase with the given parity; false on timeout
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kBulkSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_addr(src_smem)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <int NST, int LA>
__global__ void __launch_bounds__(32) k_permute_bulk(PermuteArgs a) {
  static_assert(LA >= 1 && LA < NST, "stores need slack behind the loads");
  extern __shared__ __align__(128) uint8_t bbuf[];
  __shared__ __align__(8) uint64_t bar[NST];
  __shared__ int32_t sd[NST][kMaxK + 1];
  __shared__ uint32_t smask[NST];
  const int lane = threadIdx.x;
  const uint32_t row_bytes = (uint32_t)a.row16 * 16u;
  const int row_lo = a.rank_base[a.rank_begin];
  const int row_hi = a.rank_base[a.rank_end];
  const uint8_t* hidden = reinterpret_cast<const uint8_t*>(a.hidden);
  uint8_t* out = reinterpret_cast<uint8_t*>(a.out);
  if (lane == 0) {
    for (int st = 0; st < NST; ++st) mbar_init(&bar[st], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const int64_t first = a.n0 + blockIdx.x;
  const int64_t count = first < a.N ? (a.N - first + gridDim.x - 1) / gridDim.x : 0;
  uint32_t phase = 0, inflight = 0;  // lane 0: per-stage parity and loads in flight
  bool overflow = false, timeout = false;
  for (int64_t j = 0; j < count + LA; ++j) {
    // store token j - LA: wait for its row, then one bulk store per kept row
    const int64_t js = j - LA;
    if (js >= 0 && lane == 0) {
      const int st = (int)(js % NST);
      const uint32_t m = smask[st];
      if (m) {
        if (mbar_wait(&bar[st], (phase >> st) & 1u)) {
          phase ^= 1u << st;
          inflight &= ~(1u << st);
          uint32_t mm = m;
          while (mm) {
            const int from = __ffs(mm) - 1;
            mm &= mm - 1;
            bulk_store(out + (int64_t)sd[st][from] * row_bytes, bbuf + (size_t)st * row_bytes,
                       row_bytes);
          }
        } else {
          timeout = true;
        }
      }
      bulk_commit();  // one group per token, possibly empty
    }
    timeout = __shfl_sync(kFull, timeout ? 1 : 0, 0) != 0;
    if (timeout) break;  // the same on every lane
    // issue token j into stage j % NST
    if (j < count) {
      const int st = (int)(j % NST);
      const int64_t n = first + j * gridDim.x;
      int d = -1;
      if (lane < a.K) d = a.dst_row[n * a.K + lane];
      else if (lane == a.K && a.shared_row != nullptr) d = a.shared_row[n];
      d = (d >= row_lo && d < row_hi) ? d - row_lo : -1;
      if (d >= a.cap_rows) {
        overflow = true;
        d = -1;
      }
      const unsigned m = __ballot_sync(kFull, d >= 0);
      // the stage's previous token, j - NST, was stored NST - LA iterations ago:
      // once at most NST - LA newer groups are pending, its group has
      // finished reading the buffer
      if (lane == 0) bulk_wait_read<NST - LA>();
      __syncwarp();
      if (lane <= a.K) sd[st][lane] = d;
      if (lane == 0) {
        smask[st] = m;
        if (m) {
          mbar_expect_tx(&bar[st], row_bytes);
          bulk_load(bbuf + (size_t)st * row_bytes, hidden + n * (int64_t)row_bytes, row_bytes,
                    &bar[st]);
          inflight |= 1u << st;
        }
      }
    }
    __syncwarp();
  }
  if (lane == 0) {
    // after a timeout, loads may still be in flight: wait for them (bounded)
    for (int st = 0; st < NST; ++st)
      if ((inflight >> st) & 1u) mbar_wait(&bar[st], (phase >> st) & 1u);
    bulk_wait_all();
    if (timeout) atomicOr(&a.stats->status, EP_DEV_WAIT_TIMEOUT);
  }
  if (__any_sync(kFull, overflow) && lane == 0) atomicOr(&a.stats->status, EP_DEV_OUT_CAPACITY);
}

// ---------------------------------------------------------------------------
// Combine: the reverse of the dispatch.  One warp per token at a time
// (grid-stride): lanes 0..K-1 fetch the token's dispatch rows and gate
// weights, lane K its shared-slot row; the warp walks the hidden dimension in
// passes of 1024 elements (four 16-byte words per lane) and, per pass, loads
// one k's row at a time before its fused multiply-adds, keeping
// acc = fma(w_k, x_k, acc) in ascending k and adding the shared row last.
// The grid is exactly the resident blocks (SMs x occupancy).  Measured on the
// qwen / dsv3 layers (bf16 out): 4.5 / 4.3 TB/s with two words x four rows in
// flight and twice the resident grid; 6.7 / 6.4 TB/s in this shape, which
// keeps 79 registers and three blocks per SM.
// ---------------------------------------------------------------------------
struct CombineArgs {
  const uint4* x;        // [rows][row16] bf16 expert outputs
  const float* w;        // [N][K]
  const int32_t* dst_row;
  const int32_t* shared_row;  // null without a shared expert
  const int32_t* rank_base;   // [R+1]: rank_base[R] = rows of the layout
  void* out;             // [N][hidden] bf16 or fp32
  int64_t N;
  int row16;
  int K;
  int R;
  int out_f32;
};

constexpr int kCombineThreads = 256;
constexpr int kCW = 4;   // 16-byte words per lane per pass
constexpr int kCK = 1;   // rows whose loads are issued together

__device__ __forceinline__ void fma_bf16x8(float* acc, const uint4 v, float w) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = __fmaf_rn(w, __uint_as_float(u[i] << 16), acc[2 * i]);
    acc[2 * i + 1] = __fmaf_rn(w, __uint_as_float(u[i] & 0xffff0000u), acc[2 * i + 1]);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__global__ void __launch_bounds__(kCombineThreads) k_combine(CombineArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int row16 = a.row16;
  const int rows = a.rank_base[a.R];  // rows of the layout: anything else is not read
  for (int64_t n = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; n < a.N; n += nw) {
    int d = -1;
    float wk = 0.f;
    if (lane < a.K) {
      d = a.dst_row[n * a.K + lane];
      wk = a.w[n * a.K + lane];
      if (d >= rows) d = -1;
    }
    int ds = a.shared_row ? a.shared_row[n] : -1;
    if (ds >= rows) ds = -1;
    for (int c0 = 0; c0 < row16; c0 += kCW * 32) {
      float acc[kCW * 8];
#pragma unroll
      for (int i = 0; i < kCW * 8; ++i) acc[i] = 0.f;
      for (int k0 = 0; k0 < a.K; k0 += kCK) {
        uint4 v[kCK][kCW];
        int dk[kCK];
        float wkk[kCK];
#pragma unroll
        for (int j = 0; j < kCK; ++j) {
          dk[j] = __shfl_sync(kFull, d, (k0 + j) & 31);
          wkk[j] = __shfl_sync(kFull, wk, (k0 + j) & 31);
          if (k0 + j >= a.K) dk[j] = -1;
#pragma unroll
          for (int c = 0; c < kCW; ++c) {
            const int idx = c0 + c * 32 + lane;
            if (dk[j] >= 0 && idx < row16) v[j][c] = a.x[(int64_t)dk[j] * row16 + idx];
          }
        }
#pragma unroll
        for (int j = 0; j < kCK; ++j)
          if (dk[j] >= 0) {
#pragma unroll
            for (int c = 0; c < kCW; ++c)
              if (c0 + c * 32 + lane < row16) fma_bf16x8(acc + c * 8, v[j][c], wkk[j]);
          }
      }
      if (ds >= 0) {
#pragma unroll
        for (int c = 0; c < kCW; ++c) {
          const int idx = c0 + c * 32 + lane;
          if (idx < row16) {
            const uint4 v = a.x[(int64_t)ds * row16 + idx];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[c * 8 + 2 * i] = __fadd_rn(acc[c * 8 + 2 * i], __uint_as_float(u[i] << 16));
              acc[c * 8 + 2 * i + 1] =
                  __fadd_rn(acc[c * 8 + 2 * i + 1], __uint_as_float(u[i] & 0xffff0000u));
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kCW; ++c) {
        const int idx = c0 + c * 32 + lane;
        if (idx >= row16) continue;
        const float* f = acc + c * 8;
        if (a.out_f32) {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + (n * row16 + idx) * 8);
          o[0] = make_float4(f[0], f[1], f[2], f[3]);
          o[1] = make_float4(f[4], f[5], f[6], f[7]);
        } else {
          reinterpret_cast<uint4*>(a.out)[n * row16 + idx] =
              make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                         pack_bf16x2(f[6], f[7]));
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a7: replica weight staging as persistent tile streaming.  The device-side
// task list is (replicated expert i, 8 KiB tile); a warp takes tasks
// grid-stride, loads the tile of the native expert once into registers and
// stores it to every slot holding a replica of that expert (a hot expert is
// read once however many replicas it has).  Measured on B200: 1.0 ms for the
// dsv3 layer's 51 replicas of 84 MiB, vs 1.5 ms with bulk-copy tiles through
// shared memory.
// ---------------------------------------------------------------------------
struct StageArgs {
  const uint4* native_w;
  uint4* slots;
  const int32_t* rep_nexp;
  const int32_t* rep_experts;
  const int32_t* rep_eptr;
  const int32_t* rep_list;
  int64_t words;  // 16-byte words per expert
};

constexpr int kStageThreads = 256;
constexpr int kTileWordsPerLane = 16;  // 8 KiB tile per warp

__global__ void __launch_bounds__(kStageThreads) k_stage(StageArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  constexpr int64_t kTile = kTileWordsPerLane * 32;
  const int64_t tiles = (a.words + kTile - 1) / kTile;
  const int64_t total = (int64_t)a.rep_nexp[0] * tiles;
  for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < total; t += nw) {
    const int64_t xi = t / tiles;
    const int64_t c0 = (t - xi * tiles) * kTile;
    const int e = a.rep_experts[xi];
    const int p0 = a.rep_eptr[e], p1 = a.rep_eptr[e + 1];
    const uint4* src = a.native_w + (int64_t)e * a.words;
    uint4 v[kTileWordsPerLane];
#pragma unroll
    for (int k = 0; k < kTileWordsPerLane; ++k) {
      const int64_t idx = c0 + k * 32 + lane;
      if (idx < a.words) v[k] = src[idx];
    }
    for (int p = p0; p < p1; ++p) {
      uint4* dst = a.slots + (int64_t)a.rep_list[p] * a.words;
#pragma unroll
      for (int k = 0; k < kTileWordsPerLane; ++k) {
        const int64_t idx = c0 + k * 32 + lane;
        if (idx < a.words) dst[idx] = v[k];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a8: replica gradient reduction.  Thread = 16 consecutive elements of one
// replicated expert, grid-stride over (replicated expert, element pair).
// acc = native; acc += replica in instance order, one round-to-nearest fp32
// add at a time; then the replica gradients are zeroed.
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 128;

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

// A thread owns 16 consecutive elements (two 8-element vectors; the second is
// absent in an expert's last pair when Wn % 16 == 8) and loads up to four
// replicas' vectors before adding them.  Measured on the qwen / dsv3 layers
// (bf16 grads, with the clearing kernel): one vector and eight replicas in
// flight, 256 threads: 5.4 / 5.5 TB/s; this shape with 128-thread blocks:
// 6.5 / 6.7 TB/s.  Wider (four vectors) or deeper (six or eight replicas)
// forms lose occupancy to registers and were slower.
template <bool F32>
__global__ void __launch_bounds__(kReduceThreads)
k_reduce(const int32_t* __restrict__ rep_nexp, const int32_t* __restrict__ rep_experts,
         const int32_t* __restrict__ rep_eptr, const int32_t* __restrict__ rep_list,
         const void* __restrict__ slot_grads, float* __restrict__ native, int64_t Wn, int E) {
  constexpr int kB = F32 ? 2 : 4;  // replicas whose loads are issued together
  __shared__ RepTables t;
  const int nexp = stage_rep_tables(t, rep_nexp, rep_experts, rep_eptr, rep_list, E);
  const uint32_t ppe = (uint32_t)((Wn + 15) / 16);  // element pairs of vectors per expert
  const uint32_t total = (uint32_t)nexp * ppe;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t v = blockIdx.x * blockDim.x + threadIdx.x; v < total; v += stride) {
    const uint32_t xi = v / ppe;
    const int64_t j = (int64_t)(v - xi * ppe) * 16;
    const bool two = j + 8 < Wn;
    const int e = t.exp[xi];
    const int p0 = t.ptr[xi], p1 = t.ptr[xi + 1];
    float4* nat = reinterpret_cast<float4*>(native + (int64_t)e * Wn + j);
    float acc[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !two) break;
      const float4 n0 = nat[2 * h], n1 = nat[2 * h + 1];
      acc[h][0] = n0.x; acc[h][1] = n0.y; acc[h][2] = n0.z; acc[h][3] = n0.w;
      acc[h][4] = n1.x; acc[h][5] = n1.y; acc[h][6] = n1.z; acc[h][7] = n1.w;
    }
    for (int p = p0; p < p1; p += kB) {
      Raw8<F32> r[kB][2];
#pragma unroll
      for (int u = 0; u < kB; ++u)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (p + u < p1 && (h == 0 || two))
            r[u][h] = load8<F32>(slot_grads, (int64_t)t.slot[p + u] * Wn + j + 8 * h);
#pragma unroll
      for (int u = 0; u < kB; ++u)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (p + u < p1 && (h == 0 || two)) add8<F32>(acc[h], r[u][h]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !two) break;
      nat[2 * h] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      nat[2 * h + 1] = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
    }
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


}  // namespace

cudaError_t set_copy_attributes(int max_smem) {
  // only the bulk-copy dispatch variant uses dynamic shared memory
  return allow_max_dynamic_smem(k_permute_bulk<kBulkStages, kBulkAhead>, max_smem);
}

cudaError_t launch_dispatch(const Dims& d, const LayerBuf& L, const void* hidden, void* out,
                            int64_t cap_rows, int rank_begin, int rank_end, int64_t token_begin,
                            int64_t token_end, int num_sms, int bulk, cudaStream_t st) {
  PermuteArgs a;
  a.hidden = static_cast<const uint4*>(hidden);
  a.out = static_cast<uint4*>(out);
  a.dst_row = L.dst_row;
  a.shared_row = d.sh ? L.shared_row : nullptr;
  a.rank_base = L.rank_base;
  a.stats = L.stats;
  a.n0 = token_begin;
  a.N = token_end;
  a.cap_rows = cap_rows;
  a.row16 = d.hidden * 2 / 16;
  a.K = d.K;
  a.rank_begin = rank_begin;
  a.rank_end = rank_end;
  if (a.N <= a.n0) return cudaSuccess;
  // 12 blocks of 4 warps per SM, about twice what is resident at once:
  // measured 6.0 (8), 6.1-6.2 (12) and 6.1 (16) TB/s on the qwen layer;
  // a short token range needs no more than one warp per token
  const int64_t warps = (a.N - a.n0);
  if (bulk) {
    const size_t smem = (size_t)kBulkStages * a.row16 * 16;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, k_permute_bulk<kBulkStages, kBulkAhead>, 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm > 0 && a.K + 1 <= 32) {
      const int64_t cap = (int64_t)num_sms * per_sm;
      const int64_t grid = warps < cap ? warps : cap;
      k_permute_bulk<kBulkStages, kBulkAhead><<<(unsigned)grid, 32, smem, st>>>(a);
      return cudaPeekAtLastError();
    }
    // rows too large for the ring: the register-staged form below
  }
  const int64_t blocks = (warps + kPermuteThreads / 32 - 1) / (kPermuteThreads / 32);
  const int64_t grid = blocks < (int64_t)num_sms * 12 ? blocks : (int64_t)num_sms * 12;
  const bool w32 = a.row16 % 2 == 0 && (reinterpret_cast<uintptr_t>(hidden) & 31u) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  if (w32)
    k_permute<Vec32><<<(unsigned)grid, kPermuteThreads, 0, st>>>(a);
  else
    k_permute<uint4><<<(unsigned)grid, kPermuteThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Dims& d, const LayerBuf& L, const void* x, const float* w, void* out,
                           int out_f32, int num_sms, cudaStream_t st) {
  CombineArgs a;
  a.x = static_cast<const uint4*>(x);
  a.w = w;
  a.dst_row = L.dst_row;
  a.shared_row = d.sh ? L.shared_row : nullptr;
  a.rank_base = L.rank_base;
  a.R = d.R;
  a.out = out;
  a.N = (int64_t)d.R * d.T;
  a.row16 = d.hidden * 2 / 16;
  a.K = d.K;
  a.out_f32 = out_f32;
  if (a.N == 0) return cudaSuccess;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_combine, kCombineThreads, 0);
  if (e != cudaSuccess) return e;
  k_combine<<<(unsigned)(num_sms * (per_sm > 0 ? per_sm : 1)), kCombineThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_stage(const Dims& d, const LayerBuf& L, const void* native_w, void* slots,
                         int num_sms, cudaStream_t st) {
  if (d.Wn == 0 || d.S == 0) return cudaSuccess;
  StageArgs a;
  a.native_w = static_cast<const uint4*>(native_w);
  a.slots = static_cast<uint4*>(slots);
  a.rep_nexp = L.rep_nexp;
  a.rep_experts = L.rep_experts;
  a.rep_eptr = L.rep_eptr;
  a.rep_list = L.rep_list;
  a.words = d.Wn * 2 / 16;
  k_stage<<<(unsigned)(num_sms * 8), kStageThreads, 0, st>>>(a);
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
