// Balance-plan kernels for sm_100a: load matrix, quota solve, local-first
// rerouting, token assignment and the Waterfill shared slot.
//
// What each kernel computes follows the UltraEP page ("300 µs to level MoE
// expert load"): §"Getting the real load of the current layer after the Gate"
// (global load matrix, identical deterministic solve on every rank),
// §"Quota decides replicas and token split together" (quota per instance,
// replica creation under S slots per rank / one instance per rank / minimum
// quota, local instance first then remote instances by remaining quota), and
// the Waterfill page §"Waterfill" (waterline H, slack, per-token draw).
// Everything is integer arithmetic; all orders are fixed, so results are
// bit-identical run to run and independent of the grid size.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>

#include "ep_internal.cuh"

namespace cg = cooperative_groups;

namespace ep {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarpsPerBlock = kPlanWarps;
// experts per thread when a block of the plan kernels covers all E <= kMaxE
constexpr int kExpPerThread = kMaxE / (kWarpsPerBlock * 32);

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Lanes of the warp whose key equals this lane's, for keys below 2^nbits
// (nbits <= 12): the intersection of one ballot per key bit.  Measured on
// B200 in the sampled-mode assignment (qwen / dsv3 plan 93 -> 87 / 148 -> 141
// us against match.any); in the local-first assignment and the Waterfill pass
// it was slower (stress 168 -> 194 us) and match.any stays there.
__device__ __forceinline__ unsigned match_bits(int key, int nbits) {
  unsigned m = kFull;
#pragma unroll
  for (int b = 0; b < 12; ++b) {
    if (b >= nbits) break;  // warp-uniform
    const bool bit = (key >> b) & 1;
    const unsigned bal = __ballot_sync(kFull, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the state is advanced by the
// golden-gamma increment and finished with the variant-13 mixer.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor runs; pdl_wait() blocks until
// the predecessor grid has completed and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr int kBatch = 16;     // ids per lane in flight in k_hist (a whole sub-chunk for K <= 8)
constexpr int kAsgBatch = 8;   // ids per lane per pass in k_assign

// ---------------------------------------------------------------------------
// a1: load histogram.  A block owns up to 8 consecutive sub-chunks of
// kPlanSubT tokens of one source rank, one per warp.  Each warp loads its whole
// sub-chunk at once (for K <= 8 four 16-byte vectors of ids per lane, when the
// rank's ids are 16-byte aligned; else 16 single ids) and counts it into a private
// shared-memory histogram with shared atomic adds; the warp writes its row of
// counts and the block writes the sum of its rows (the two levels of bases of
// the stable ordinals, used by k_assign).  The block then adds its sum to the
// load-matrix accumulator with integer atomics (order-independent, so the
// result is deterministic); it is zero on entry, the solve sums its columns
// into the expert totals and the rerouting moves it into the layer.  The first kernel
// of the plan: a plain launch, so the ids are complete when it starts.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 6)
k_hist(const int32_t* __restrict__ ids, Dims d, Scratch s) {
  extern __shared__ int32_t sm_hist[];
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbpr = (d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int r = blockIdx.x / nbpr, b = blockIdx.x - r * nbpr;
  const int sub = b * kWarpsPerBlock + warp;
  const int E = d.E, K = d.K;
  int32_t* hist = sm_hist + warp * E;
  for (int e = lane; e < E; e += 32) hist[e] = 0;
  __syncwarp();
  int bad = 0;
  if (sub < d.nsub) {
    const int t0 = sub * kPlanSubT, t1 = min(d.T, t0 + kPlanSubT);
    const int32_t* src = ids + (int64_t)r * d.T * K;
    const int a1 = t1 * K;
    const int32_t* p = src + t0 * K;
    const int n = a1 - t0 * K;
    auto count = [&](int v, bool in) {
      if (!in) return;
      if (v < 0 || v >= E) ++bad;
      else atomicAdd(&hist[v], 1);  // integer: order-independent
    };
    if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
      // 16-byte loads: a lane takes 4 consecutive ids, 4 vectors in flight
      // (a whole sub-chunk for K <= 8); a vector that would cross the end of
      // the sub-chunk is read id by id
      for (int q0 = 0; q0 < n; q0 += 16 * 32) {
        int4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = q0 + 4 * (u * 32 + lane);
          if (q + 3 < n) {
            w[u] = __ldg(reinterpret_cast<const int4*>(p + q));
          } else {
            w[u].x = q < n ? __ldg(p + q) : -1;
            w[u].y = q + 1 < n ? __ldg(p + q + 1) : -1;
            w[u].z = q + 2 < n ? __ldg(p + q + 2) : -1;
            w[u].w = -1;
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = q0 + 4 * (u * 32 + lane);
          count(w[u].x, q < n);
          count(w[u].y, q + 1 < n);
          count(w[u].z, q + 2 < n);
          count(w[u].w, q + 3 < n);
        }
      }
    } else {
      for (int a = t0 * K; a < a1; a += kBatch * 32) {  // one pass for K <= 8, two for K <= 16
        int v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int idx = a + u * 32 + lane;
          v[u] = idx < a1 ? __ldg(src + idx) : -1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) count(v[u], a + u * 32 + lane < a1);
      }
    }
    __syncwarp();
    int32_t* out = s.sub_cnt + ((int64_t)r * d.nsub + sub) * E;
    for (int e = lane; e < E; e += 32) out[e] = hist[e];
  }
  __syncthreads();
  int32_t* blk = s.blk_cnt + ((int64_t)r * nbpr + b) * E;
  int csum[kExpPerThread];
#pragma unroll
  for (int u = 0; u < kExpPerThread; ++u) {
    const int e = threadIdx.x + u * blockDim.x;
    csum[u] = 0;
    if (e < E) {
#pragma unroll
      for (int w = 0; w < kWarpsPerBlock; ++w) csum[u] += sm_hist[w * E + e];
      blk[e] = csum[u];
    }
  }
  // ids outside [0, E): the status bit, and their count, from which the solve
  // takes the number of assignments without a reduction of its own
  const int nbad = (int)__reduce_add_sync(kFull, (unsigned)bad);
  if (nbad && lane == 0) {
    atomicOr(&s.acc_misc[0], EP_DEV_BAD_ID);
    atomicAdd(&s.acc_misc[2], nbad);
  }
#pragma unroll
  for (int u = 0; u < kExpPerThread; ++u) {
    const int e = threadIdx.x + u * blockDim.x;
    if (e < E && csum[u]) atomicAdd(&s.acc_load[r * E + e], csum[u]);
  }
}


// Warp argmax over the ranks lane + 32k (k < RW) with ok[k] set: the largest
// v, smallest rank on ties.  When every v is below 2^24 the value and the rank
// travel in one key, v * 128 + (127 - rank), and one redux finds both;
// otherwise a max redux and a ballot per word.  Returns vmax = 0 when no rank
// is ok (the rank returned is then meaningless).
template <int RW>
__device__ __forceinline__ int warp_argmax_rank(const unsigned (&v)[RW], const bool (&ok)[RW],
                                                bool pack, int lane, unsigned& vmax) {
  if (pack) {
    unsigned key = 0;
#pragma unroll
    for (int k = 0; k < RW; ++k)
      if (ok[k]) key = max(key, (v[k] << 7) | (unsigned)(127 - (lane + 32 * k)));
    key = __reduce_max_sync(kFull, key);
    vmax = key >> 7;
    return 127 - (int)(key & 127u);
  }
  unsigned mx = 0;
#pragma unroll
  for (int k = 0; k < RW; ++k)
    if (ok[k]) mx = max(mx, v[k]);
  vmax = __reduce_max_sync(kFull, mx);
  int q = -1;
#pragma unroll
  for (int k = 0; k < RW; ++k) {
    const unsigned b = __ballot_sync(kFull, ok[k] && v[k] == vmax);
    if (q < 0 && b) q = 32 * k + __ffs(b) - 1;
  }
  return q;
}

// ---------------------------------------------------------------------------
// a2: quota solve.  A thread-block cluster of ceil(J/4) CTAs, one SM each;
// cap-candidate warp j (warp j%4 of CTA j/4; warps 4-7 of every CTA help with
// the setup and the table emit) runs the greedy at cap
// C_j = ceil(A (200 + j) / (200 R)).  Greedy step: the most-loaded rank p that is
// not stuck (smallest index on ties) gives min(max(W_p - C, m), slack_r, Q_e) of
// its native e — natives tried by quota descending, then expert ascending, only
// those with quota >= m — to a new replica on the rank r with the largest slack
// C - W_r >= m among ranks with a free slot and no instance of e (smallest index
// on ties).  If no native of p can move, p is stuck.  The run with the smallest
// (max load, replicas, j) wins.  A lane owns ranks lane + 32k (k < RW, the
// number of 32-rank words) and keeps their load, slot table and flags in
// registers; native quotas live in shared memory.
// ---------------------------------------------------------------------------
constexpr int kSolveWarps = 4;                     // cap candidates per CTA: one per SM partition
// plus as many helper warps, which wait at the barrier during the greedy and
// halve the per-thread work of the setup and of the winner's table emit
constexpr int kSolveThreads = 2 * kSolveWarps * 32;

template <int SMAX, int RW, bool PACK>
__global__ void __launch_bounds__(kSolveThreads, 1) k_solve(Dims d, LayerBuf L, Scratch s) {
  extern __shared__ int32_t sm[];
  int32_t* Tot = sm;              // [E]
  int32_t* Qn_all = sm + d.E;     // [kSolveWarps][E]: this CTA's candidates' native quotas
  int32_t* cnt_e = Qn_all + kSolveWarps * d.E;  // [E+1]
  int32_t* s_rel = cnt_e + d.E + 1;     // [R*G] rank-relative first rows
  int32_t* s_iex = s_rel + d.R * d.G;   // [R*G] the winner's instance table: experts
  int32_t* s_iqu = s_iex + d.R * d.G;   // [R*G] and quotas
  __shared__ int32_t s_W0[kMaxR];
  __shared__ int32_t s_Wf[kMaxR];
  __shared__ int32_t s_se[kMaxR * kMaxS];
  __shared__ int32_t s_sq[kMaxR * kMaxS];
  __shared__ int32_t s_cmax[kMaxJ], s_crep[kMaxJ], s_cstop[kMaxJ];
  __shared__ int32_t s_best, s_iter_cap_hit, s_tight, s_any_cap, s_bmax;
  __shared__ int32_t s_base[kMaxR + 1];
  __shared__ int32_t s_wsum[kMaxJ];

  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank(), ncta = (int)cluster.num_blocks();
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int R = d.R, E = d.E, S = d.S, m = d.m;
  // native placement: rank q holds [q*eb + min(q, er), +eb + (q < er)); one
  // division here rather than one per greedy step
  const int eb = E / R, er = E - (E / R) * R;

  // wait first: the rerouting, launched at this trigger, may then read the
  // histogram's load matrix before waiting for the solve
  pdl_wait();
  pdl_trigger();
  const int hist_status = s.acc_misc[0];  // the histogram's status bits of this call
  // A: every assignment with an id in [0, E) (the histogram counts the others)
  const int A = (int)((int64_t)R * d.T * d.K - s.acc_misc[2]);
  // expert totals: the load matrix's columns summed over source ranks (the
  // histogram adds only into the load matrix: one total per expert would
  // take an atomic from every block of the grid).  CTA c of the cluster sums
  // experts [c*E/n, (c+1)*E/n): nslice adjacent lanes (a power of two) share
  // an expert, each summing ranks slice, slice + nslice, ... with sixteen
  // loads in flight, and a shuffle reduction leaves the total with the
  // group's first lane; every CTA then reads the other CTAs' totals from
  // their shared memory.
  const int e_lo = crank * E / ncta, e_hi = (crank + 1) * E / ncta, ne = e_hi - e_lo;
  for (int e = tid; e <= E; e += nthr) cnt_e[e] = 0;  // the winner's replica counts, at the end
  if (tid == 0) s_iter_cap_hit = 0;
  if (ne > 0) {
    int nslice = 1;
    while (nslice < 32 && 2 * nslice * ne <= nthr) nslice *= 2;
    for (int t0 = 0; t0 < nslice * ne; t0 += nthr) {  // warp-uniform rounds
      const int t = t0 + tid;
      const bool in = t < nslice * ne;
      const int e = e_lo + t / nslice, sl = t % nslice;
      int acc = 0;
      if (in)
        for (int r = sl; r < R; r += 16 * nslice) {
          int v[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int q = r + u * nslice;
            v[u] = q < R ? s.acc_load[q * E + e] : 0;
          }
#pragma unroll
          for (int u = 0; u < 16; ++u) acc += v[u];
        }
      for (int o = nslice / 2; o > 0; o >>= 1) acc += __shfl_down_sync(kFull, acc, o, nslice);
      if (in && sl == 0) Tot[e] = acc;
    }
  }
  cluster.sync();
  for (int e = tid; e < E; e += nthr) {
    if (e >= e_lo && e < e_hi) continue;
    int c = 0;
    while (e >= (c + 1) * E / ncta) ++c;  // the CTA whose range holds e
    Tot[e] = *cluster.map_shared_rank(&Tot[e], c);
  }
  __syncthreads();
  // (the totals, W0 and the statistics reach global memory only in the
  // winner's last phase: no global store is queued ahead of the greedy's
  // shared-memory loads)
  if (tid < R) {
    const int f = tid * eb + min(tid, er), n = eb + (tid < er ? 1 : 0);
    int w = 0;
    for (int i = 0; i < n; ++i) w += Tot[f + i];
    s_W0[tid] = w;
  }
  __syncthreads();

  // ---- one greedy run per warp: candidate j = crank * kSolveWarps + warp ----
  const int j = crank * kSolveWarps + warp;
  const bool solver = warp < kSolveWarps && j < d.J;
  const int64_t den = 200LL * R;
  const int C = (int)(((int64_t)A * (200 + j) + den - 1) / den);
  int Wr[RW], used[RW], se[RW][SMAX], sq[RW][SMAX];
  int replicas = 0, stop = -1, maxW = 0;
  if (solver) {
    int32_t* Qn = Qn_all + warp * E;
    for (int e = lane; e < E; e += 32) Qn[e] = Tot[e];
    unsigned stuck = 0, slotlim = 0;
#pragma unroll
    for (int k = 0; k < RW; ++k) {
      const int q = lane + 32 * k;
      Wr[k] = q < R ? s_W0[q] : 0;
      used[k] = 0;
#pragma unroll
      for (int t = 0; t < SMAX; ++t) { se[k][t] = -1; sq[k][t] = 0; }
    }
    __syncwarp();
    const int iter_cap = d.iter_limit > 0 ? d.iter_limit : 4 * (R * S + R + E) + 64;
    // every key value is a load, a slack or a quota, at most C <= 1.08 A: below
    // 2^25 whenever R*T*K < 2^24 (the host's choice of PACK), so value and
    // index travel in one 32-bit redux key
    constexpr bool pack = PACK;
    for (int it = 0;; ++it) {
      if (it >= iter_cap) { stop = EP_STOP_ITER_CAP; break; }
      unsigned wv[RW];
      bool wok[RW];
#pragma unroll
      for (int k = 0; k < RW; ++k) {
        wv[k] = (unsigned)Wr[k];
        wok[k] = lane + 32 * k < R && !((stuck >> k) & 1u);
      }
      unsigned uvmax;
      const int p = warp_argmax_rank<RW>(wv, wok, pack, lane, uvmax);
      const int vmax = (int)uvmax;
      if (vmax <= C) break;
      const int ex = vmax - C;
      const int nf = p * eb + min(p, er), nc = eb + (p < er ? 1 : 0);
      const int myQ = lane < nc ? Qn[nf + lane] : 0;
      bool tried = false, moved = false;
      for (;;) {
        // the donor's untried native with the largest quota >= m (smallest e on ties)
        const unsigned cq = (lane < nc && !tried && myQ >= m) ? (unsigned)myQ : 0u;
        unsigned qmax;
        int li;
        if (pack) {
          const unsigned key = __reduce_max_sync(kFull, cq ? (cq << 5) | (unsigned)(31 - lane) : 0u);
          qmax = key >> 5;
          li = 31 - (int)(key & 31u);
        } else {
          qmax = __reduce_max_sync(kFull, cq);
          li = __ffs(__ballot_sync(kFull, cq == qmax)) - 1;
        }
        if (qmax == 0) break;
        const int e = nf + li;
        // receivers: free slot, no instance of e, slack >= m
        unsigned sv[RW];
        bool ok[RW];
#pragma unroll
        for (int k = 0; k < RW; ++k) {
          const int q = lane + 32 * k;
          bool h = false;
#pragma unroll
          for (int t = 0; t < SMAX; ++t) h |= (se[k][t] == e);
          ok[k] = q < R && q != p && used[k] < S && !h && C - Wr[k] >= m;
          sv[k] = (unsigned)(C - Wr[k]);
        }
        unsigned smax;
        const int rr = warp_argmax_rank<RW>(sv, ok, pack, lane, smax);
        if (smax == 0) {
          if (lane == li) tried = true;
          // no rank other than p has a free slot and slack >= m at all: every
          // other native fails the same way
          bool any_r = false;
#pragma unroll
          for (int k = 0; k < RW; ++k) {
            const int q = lane + 32 * k;
            any_r |= q < R && q != p && used[k] < S && C - Wr[k] >= m;
          }
          if (!__any_sync(kFull, any_r)) break;
          continue;
        }
        const int x = min(min(max(ex, m), (int)smax), (int)qmax);
#pragma unroll
        for (int k = 0; k < RW; ++k) {
          const int q = lane + 32 * k;
          if (q == p) Wr[k] -= x;
          if (q == rr) {
            Wr[k] += x;
#pragma unroll
            for (int t = 0; t < SMAX; ++t) {
              const bool here = (t == used[k]);
              se[k][t] = here ? e : se[k][t];
              sq[k][t] = here ? x : sq[k][t];
            }
            used[k] += 1;
          }
        }
        if (lane == li) Qn[e] = (int)qmax - x;
        ++replicas;
        moved = true;
        break;
      }
      if (!moved) {
        bool fr = false;
#pragma unroll
        for (int k = 0; k < RW; ++k)
          fr |= (lane + 32 * k < R && used[k] == S && C - Wr[k] >= m);
        const bool full_receiver = __any_sync(kFull, fr);
        const bool native_big = __any_sync(kFull, lane < nc && myQ >= m);
#pragma unroll
        for (int k = 0; k < RW; ++k)
          if (lane + 32 * k == p) {
            stuck |= 1u << k;
            if (full_receiver && native_big) slotlim |= 1u << k;
          }
      }
      __syncwarp();
    }
    unsigned wm = 0;
    bool sl = false;
#pragma unroll
    for (int k = 0; k < RW; ++k)
      if (lane + 32 * k < R) {
        wm = max(wm, (unsigned)Wr[k]);
        sl |= ((stuck >> k) & 1u) && ((slotlim >> k) & 1u) && Wr[k] > C;
      }
    maxW = (int)__reduce_max_sync(kFull, wm);
    const bool any_sl = __any_sync(kFull, sl);
    if (stop != EP_STOP_ITER_CAP)
      stop = maxW <= C ? EP_STOP_BALANCED : (any_sl ? EP_STOP_SLOT_LIMITED : EP_STOP_QUOTA_LIMITED);
    if (lane == 0) {
      s_cmax[j] = maxW;
      s_crep[j] = replicas;
      s_cstop[j] = stop;
      L.cand[j] = maxW;
      L.cand[d.J + j] = replicas;
      L.cand[2 * d.J + j] = stop;
      if (stop == EP_STOP_ITER_CAP) atomicOr(&s_iter_cap_hit, 1);
    }
  }
  cluster.sync();
  if (warp == 0) {  // smallest (max load, replicas, j), read from the candidates' CTAs
    const int owner = lane / kSolveWarps;
    const bool cand = lane < d.J;
    const unsigned cmax = cand ? (unsigned)*cluster.map_shared_rank(&s_cmax[lane], owner) : 0u;
    const unsigned crep = cand ? (unsigned)*cluster.map_shared_rank(&s_crep[lane], owner) : 0u;
    const int cstop0 = *cluster.map_shared_rank(&s_cstop[0], 0);
    const bool cap_hit = lane < ncta && *cluster.map_shared_rank(&s_iter_cap_hit, lane);
    const unsigned k1 = cand ? cmax : 0xffffffffu;
    const unsigned m1 = __reduce_min_sync(kFull, k1);
    const unsigned k2 = (cand && k1 == m1) ? crep * 32u + (unsigned)lane : 0xffffffffu;
    const unsigned m2 = __reduce_min_sync(kFull, k2);
    const bool any_cap = __any_sync(kFull, cap_hit);
    if (lane == 0) {
      s_best = (int)(m2 & 31u);
      s_tight = cstop0;
      s_any_cap = any_cap ? 1 : 0;
    }
  }
  // every remote read above is done before any CTA leaves; only the winner's
  // CTA lays the plan out
  cluster.sync();
  if (crank != s_best / kSolveWarps) return;
  __shared__ int32_t s_wst[4];  // the winner's stop reason, replicas, cap, max load
  if (solver && j == s_best) {
    if (lane == 0) {
      s_wst[0] = stop;
      s_wst[1] = replicas;
      s_wst[2] = C;
      s_wst[3] = maxW;
    }
#pragma unroll
    for (int k = 0; k < RW; ++k) {
      const int q = lane + 32 * k;
      if (q < R) {
        s_Wf[q] = Wr[k];
#pragma unroll
        for (int t = 0; t < SMAX; ++t)
          if (t < S) { s_se[q * S + t] = se[k][t]; s_sq[q * S + t] = sq[k][t]; }
      }
    }
  }
  __syncthreads();

  // ---- emit the winner's instance table ----
  // Everything is laid out in shared memory first and written to global
  // memory in one last phase; the layout takes two barriers.  Thread q walks
  // rank q's columns once (expert, quota, rank-relative first row, and the
  // replica count of the column's expert); the last warp scans the ranks'
  // routed rows into the ranks' first rows.  (With only the solve's four warps
  // on the SM, each barrier-separated phase costs its full dependency chain:
  // clock readings put the earlier five-phase layout at 0.8-1.6 us a phase.)
  const int G = d.G, Gmax = d.Gmax;
  const int32_t* Qw = Qn_all + (s_best % kSolveWarps) * E;
  if (tid < R) {
    const int q = tid, nf = q * eb + min(q, er), nn = eb + (q < er ? 1 : 0);
    int run = 0;
    for (int col = 0; col < G; ++col) {
      int ex = -1, qu = 0;
      if (col < Gmax) {
        if (col < nn) { ex = nf + col; qu = Qw[ex]; }
      } else if (col < Gmax + S) {
        ex = s_se[q * S + col - Gmax];
        qu = s_sq[q * S + col - Gmax];
        if (ex >= 0) atomicAdd(&cnt_e[ex], 1);
      } else {
        ex = E;  // the shared-expert column
      }
      s_iex[q * G + col] = ex;
      s_iqu[q * G + col] = qu;
      s_rel[q * G + col] = run;
      run += qu;
    }
  }
  if (warp == kSolveThreads / 32 - 1) {  // a warp with no rank of its own above
    // first row of each rank's block (routed rows only; a shared column moves
    // it later), and the largest load before balancing
    int carry = 0, bm = 0;
    for (int q0 = 0; q0 < R; q0 += 32) {
      const int q = q0 + lane;
      const int v = q < R ? s_Wf[q] : 0;
      if (q < R) bm = max(bm, s_W0[q]);
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (q < R) s_base[q] = carry + incl - v;
      carry += __shfl_sync(kFull, incl, 31);
    }
    bm = (int)__reduce_max_sync(kFull, (unsigned)bm);
    if (lane == 0) {
      s_base[R] = carry;
      s_bmax = bm;
    }
  }
  __syncthreads();
  // replica lists grouped by expert (CSR): the offsets rep_eptr and the list
  // of replicated experts come from one block-wide exclusive scan of
  // (replicas of e) | (e has replicas) << 16 — both sums stay below 2^16 —
  // and k_reroute writes each expert's slots into its part of the list
  constexpr int kIPT = (kMaxE + 1 + kSolveThreads - 1) / kSolveThreads;
  int vals[kIPT], local = 0;
#pragma unroll
  for (int u = 0; u < kIPT; ++u) {
    const int e = tid * kIPT + u;
    const int c = e < E ? cnt_e[e] : 0;
    vals[u] = c | (c > 0 ? 1 << 16 : 0);
    local += vals[u];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  int wbase = 0;  // the earlier warps' sums
  for (int w = 0; w < warp; ++w) wbase += s_wsum[w];

  // ---- the global writes ----
  if (tid == 0) {
    ep_layer_stats* st = L.stats;
    st->status = hist_status | (s_any_cap ? EP_DEV_ITER_CAP : 0);
    s.acc_misc[0] = 0;  // zero again for the next call
    s.acc_misc[2] = 0;
    st->before_max = s_bmax;
    st->cap_idx = s_best;
    st->stop_reason = s_wst[0];
    st->tight_stop_reason = s_tight;
    st->replicas = s_wst[1];
    st->cap = s_wst[2];
    st->assignments = A;
    st->after_max = s_wst[3];
    st->realized_max = s_wst[3];
  }
  for (int e = tid; e < E; e += nthr) L.expert_total[e] = Tot[e];
  for (int q = tid; q < R; q += nthr) {
    L.W0[q] = s_W0[q];
    L.W[q] = s_Wf[q];
    s.rank_rows[q] = s_Wf[q];  // routed rows per rank (the sampled mode recounts them)
  }
  int run = wbase + incl - local;
#pragma unroll
  for (int u = 0; u < kIPT; ++u) {
    const int e = tid * kIPT + u;
    if (e <= E) L.rep_eptr[e] = run & 0xffff;
    if (e < E && (vals[u] & 0xffff)) L.rep_experts[run >> 16] = e;
    if (e == E) L.rep_nexp[0] = run >> 16;
    run += vals[u];
  }
  for (int i = tid; i < R * G; i += nthr) {
    L.inst_expert[i] = s_iex[i];
    L.inst_quota[i] = s_iqu[i];
    s.inst_rel[i] = s_rel[i];
    if (!d.sh) L.inst_off[i] = s_base[i / G] + s_rel[i];
  }
  if (!d.sh) {
    if (tid == 0) L.inst_off[R * G] = s_base[R];
    for (int q = tid; q <= R; q += nthr) L.rank_base[q] = s_base[q];
    if (tid == 0) L.stats->rows = s_base[R];
  } else {
    // Waterfill waterline on the routed loads: H = ceil((sum W + N)/R),
    // B = ceil(H * bonus / 1000), slack = max(H - W, 0).
    const int64_t N = (int64_t)R * d.T;
    const int64_t H = ((int64_t)A + N + R - 1) / R;
    if (tid == 0) {
      s.wf[0] = (int)H;
      s.wf[1] = (int)((H * d.bonus + 999) / 1000);
    }
    for (int q = tid; q < R; q += nthr) s.slack[q] = (int)max(H - (int64_t)s_Wf[q], (int64_t)0);
  }
}

// ---------------------------------------------------------------------------
// a3: local-first rerouting, one warp per expert.  Instances of e (native plus
// replicas) in instance order; each source rank first uses the instance on its
// own rank up to its quota; the residual demands, laid end to end in source
// order, fill the residual quotas laid end to end in instance order.  The
// output is, per (expert, source), the ordered segments (first ordinal,
// destination rank, first row minus first ordinal), and per (source, expert) a
// 32-byte record of the first two segments that the token assignment copies
// with one coalesced load.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_reroute(Dims d, LayerBuf L, Scratch s) {
  __shared__ int32_t s_irank[kWarpsPerBlock][kMaxR];  // instance j: rank
  __shared__ int32_t s_irel[kWarpsPerBlock][kMaxR];   // instance j: rank-relative first row
  __shared__ int32_t s_iq[kWarpsPerBlock][kMaxR];     // instance j: quota, then residual
  __shared__ int32_t s_ipq[kWarpsPerBlock][kMaxR];    // instance j: start of residual interval
  __shared__ int32_t s_iloc[kWarpsPerBlock][kMaxR];   // instance j: local take
  __shared__ int32_t s_jof[kWarpsPerBlock][kMaxR];    // rank -> instance j or -1
  __shared__ int32_t s_igi[kWarpsPerBlock][kMaxR];    // instance j: global instance index
  __shared__ int32_t s_rbw[kWarpsPerBlock][kMaxR + 1];  // first row of each rank, per warp
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kWarpsPerBlock + warp;
  const int R = d.R, E = d.E, G = d.G, S = d.S;
  // the load column of e: the histogram had completed before the solve
  // triggered this launch, so it is read before waiting for the solve (which
  // reads the load matrix too: it is copied out and zeroed only after the wait)
  int lcol[kRW];
#pragma unroll
  for (int k = 0; k < kRW; ++k) {
    const int r = lane + 32 * k;
    lcol[k] = (e < E && r < R) ? s.acc_load[r * E + e] : 0;
  }
  pdl_wait();
  if (e >= d.E) return;
  // Every load of the solve's tables that does not depend on another is
  // issued first, together: the native's entry, the replica list's offset and
  // the first 32 replica slots' entries (all slots for R*S <= 32).
  const int h = home_of(e, E, R);
  const int hcol = e - nat_first(h, E, R);
  const int nat_rel = s.inst_rel[h * G + hcol], nat_q = L.inst_quota[h * G + hcol];
  const int rep_off = L.rep_eptr[e];
  bool hit0 = false;
  int rel0 = 0, quota0 = 0;
  if (lane < R * S) {
    const int q = lane / S, col = d.Gmax + (lane - q * S);
    hit0 = L.inst_expert[q * G + col] == e;
    rel0 = s.inst_rel[q * G + col];
    quota0 = L.inst_quota[q * G + col];
  }
  int32_t* s_rb = s_rbw[warp];
  if (!d.sh && !d.sampled)  // issued now, read once the segments are written
    for (int q = lane; q <= d.R; q += 32) s_rb[q] = L.rank_base[q];
  int32_t* irank = s_irank[warp];
  int32_t* irel = s_irel[warp];
  int32_t* iq = s_iq[warp];
  int32_t* ipq = s_ipq[warp];
  int32_t* iloc = s_iloc[warp];
  int32_t* jof = s_jof[warp];
  int32_t* igi = s_igi[warp];

#pragma unroll
  for (int k = 0; k < kRW; ++k) {
    const int r = lane + 32 * k;
    if (r < R) {
      L.load[r * E + e] = lcol[k];
      s.acc_load[r * E + e] = 0;  // zero again for the next call
    }
  }
  for (int q = lane; q < R; q += 32) jof[q] = -1;
  __syncwarp();
  // instances in instance order: the replica slots holding e (scanned in slot
  // order, i.e. rank order; none is on the home rank h) with the native placed
  // after the replicas on ranks below h.  Every slot's entries are loaded in
  // one round, independent of each other.
  int nrep = 0, np = 0;
  int32_t* rlist = L.rep_list + rep_off;  // e's part of the replica list
  for (int i0 = 0; i0 < R * S; i0 += 32) {
    const int i = i0 + lane;
    const int q = i / S, col = d.Gmax + (i - (i / S) * S);
    bool hit = i0 == 0 && hit0;
    int rel = i0 == 0 ? rel0 : 0, quota = i0 == 0 ? quota0 : 0;
    if (i0 > 0 && i < R * S) {
      hit = L.inst_expert[q * G + col] == e;
      rel = s.inst_rel[q * G + col];
      quota = L.inst_quota[q * G + col];
    }
    const unsigned m = __ballot_sync(kFull, hit);
    if (hit) {
      rlist[nrep + __popc(m & lanemask_lt())] = i;  // slot order = instance order
      const int j = nrep + __popc(m & lanemask_lt()) + (q > h ? 1 : 0);
      irank[j] = q;
      irel[j] = rel;
      iq[j] = quota;
      jof[q] = j;
      igi[j] = q * G + col;
    }
    nrep += __popc(m);
    np += __popc(__ballot_sync(kFull, hit && q < h));
  }
  if (lane == 0) {
    irank[np] = h;
    irel[np] = nat_rel;
    iq[np] = nat_q;
    jof[h] = np;
    igi[np] = h * G + hcol;
  }
  const int ninst = nrep + 1;
  __syncwarp();
  if (d.sampled) {
    // the sampled mode needs, per instance key e + rep_eptr[e] + j, the running
    // quota sum of e's instances in instance order and the instance's index
    const int kb = e + L.rep_eptr[e];
    int carry = 0;
    for (int j0 = 0; j0 < ninst; j0 += 32) {
      const int j = j0 + lane;
      const int v = j < ninst ? iq[j] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (j < ninst) {
        s.smp_cum[kb + j] = carry + incl;
        s.smp_inst[kb + j] = igi[j];
      }
      carry += __shfl_sync(kFull, incl, 31);
    }
    return;
  }
  // local take and residual demand of every source rank (lane owns r = lane + 32k)
  int Dr[kRW], locr[kRW];
#pragma unroll
  for (int k = 0; k < kRW; ++k) {
    const int r = lane + 32 * k;
    Dr[k] = 0;
    locr[k] = 0;
    if (r < R) {
      const int l = lcol[k];
      const int j = jof[r];
      const int loc = j >= 0 ? min(l, iq[j]) : 0;
      locr[k] = loc;
      Dr[k] = l - loc;
      if (j >= 0) iloc[j] = loc;
    }
  }
  __syncwarp();
  // residual quotas and their exclusive prefix in instance order
  {
    int carry = 0;
    for (int j0 = 0; j0 < ninst; j0 += 32) {
      const int j = j0 + lane;
      const int v = j < ninst ? iq[j] - iloc[j] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (j < ninst) { iq[j] = v; ipq[j] = carry + incl - v; }
      carry += __shfl_sync(kFull, incl, 31);
    }
  }
  __syncwarp();
  // exclusive prefix of residual demand in source order
  int PD[kRW];
  {
    int carry = 0;
#pragma unroll
    for (int k = 0; k < kRW; ++k) {
      int incl = Dr[k];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      PD[k] = carry + incl - Dr[k];
      carry += __shfl_sync(kFull, incl, 31);
    }
  }
  // first instance whose residual interval ends after PD (binary search)
  auto first_after = [&](int x) {
    int lo = 0, hi = ninst;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ipq[mid] + iq[mid] > x) hi = mid; else lo = mid + 1;
    }
    return lo;
  };
  // pass 1: segment count per source, prefix in source order
  int cnt[kRW], j0r[kRW];
#pragma unroll
  for (int k = 0; k < kRW; ++k) {
    cnt[k] = 0;
    j0r[k] = 0;
    const int r = lane + 32 * k;
    if (r < R) {
      cnt[k] = locr[k] > 0 ? 1 : 0;
      if (Dr[k] > 0) {
        const int end = PD[k] + Dr[k];
        int j = first_after(PD[k]);
        j0r[k] = j;
        for (; j < ninst && ipq[j] < end; ++j) cnt[k] += iq[j] > 0;
      }
    }
  }
  int segbase[kRW];
  {
    int carry = 0;
#pragma unroll
    for (int k = 0; k < kRW; ++k) {
      int incl = cnt[k];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      segbase[k] = carry + incl - cnt[k];
      carry += __shfl_sync(kFull, incl, 31);
    }
  }
  // pass 2: write the segments
  int32_t* sord = s.seg_ord + (int64_t)e * 3 * R;
  int32_t* srank = s.seg_rank + (int64_t)e * 3 * R;
  int32_t* sbase = s.seg_base + (int64_t)e * 3 * R;
  // a segment's rows start at its destination rank's first row (without a
  // shared expert; with one, k_fixup adds it later) plus its offset there
  const bool absolute = !d.sh;
#pragma unroll
  for (int k = 0; k < kRW; ++k) {
    const int r = lane + 32 * k;
    if (r >= R) continue;
    int w = segbase[k];
    // the record of (r, e) for the token assignment: {first row base
    // (INT_MIN: no segment), second segment's first ordinal (INT_MAX: none),
    // first rank, 0} and {second rank | segment count << 8, second row base,
    // third segment's first ordinal (INT_MAX: none), index of the last
    // segment in the lists}
    int4 r0 = make_int4(INT_MIN, INT_MAX, 0, 0);
    int4 r1 = make_int4(cnt[k] << 8, 0, INT_MAX, e * 3 * R + w + cnt[k] - 1);
    auto put = [&](int ord, int rank, int base) {
      const int i = w - segbase[k];
      if (i == 0) {
        r0.x = base;
        r0.z = rank;
      } else if (i == 1) {
        r0.y = ord;
        r1.x |= rank;
        r1.y = base;
      } else if (i == 2) {
        r1.z = ord;
      }
      sord[w] = ord;
      srank[w] = rank;
      sbase[w] = base;
      ++w;
    };
    if (locr[k] > 0) {
      const int j = jof[r];
      const int before = min(max(PD[k] - ipq[j], 0), iq[j]);  // remote rows of earlier sources
      put(0, r, (absolute ? s_rb[r] : 0) + irel[j] + before);
    }
    if (Dr[k] > 0) {
      const int end = PD[k] + Dr[k];
      for (int j = j0r[k]; j < ninst && ipq[j] < end; ++j) {
        if (iq[j] <= 0) continue;
        const int lo = max(PD[k], ipq[j]);
        const int c = irank[j];
        const int ord = locr[k] + (lo - PD[k]);
        put(ord, c, (absolute ? s_rb[c] : 0) + irel[j] + (c < r ? iloc[j] : 0) + (lo - ipq[j]) - ord);
      }
    }
    int4* rec = reinterpret_cast<int4*>(s.seg_rec) + ((int64_t)r * E + e) * 2;
    rec[0] = r0;
    rec[1] = r1;
  }
}

// Every rank below R set (all-rank Waterfill candidates).
__device__ __forceinline__ void mask_all(unsigned (&mask)[kRW], int R) {
#pragma unroll
  for (int w = 0; w < kRW; ++w) {
    const int n = min(max(R - 32 * w, 0), 32);
    mask[w] = n == 32 ? 0xffffffffu : ((1u << n) - 1u);
  }
}

// Set / clear bit q of a 4-word rank mask without a dynamic word index.
__device__ __forceinline__ void mask_set(unsigned (&mask)[kRW], int q) {
  const unsigned bit = 1u << (q & 31);
#pragma unroll
  for (int w = 0; w < kRW; ++w) mask[w] |= (q >> 5) == w ? bit : 0u;
}
__device__ __forceinline__ void mask_clear(unsigned (&mask)[kRW], int q) {
  const unsigned bit = 1u << (q & 31);
#pragma unroll
  for (int w = 0; w < kRW; ++w) mask[w] &= (q >> 5) == w ? ~bit : ~0u;
}

// ---------------------------------------------------------------------------
// a5 device side: the Waterfill pick of one token.  cand mask holds the ranks
// the token visits; the own rank r comes first, the others ascending.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int wf_pick(int r, int64_t token, const unsigned (&mask)[kRW],
                                       const int32_t* slack, const int32_t* W, int B,
                                       uint64_t seed) {
  int64_t sumS = slack[r];
#pragma unroll
  for (int w = 0; w < kRW; ++w) {
    unsigned b = mask[w];
    while (b) {
      const int c = 32 * w + __ffs(b) - 1;
      b &= b - 1;
      sumS += slack[c];
    }
  }
  if (sumS > 0) {
    const uint64_t h = splitmix64(seed + (uint64_t)token);
    const uint64_t u = ((h >> 32) * (uint64_t)(sumS + B)) >> 32;
    int64_t acc = (int64_t)slack[r] + B;
    if ((uint64_t)acc > u) return r;
    int last = r;
#pragma unroll
    for (int w = 0; w < kRW; ++w) {
      unsigned b = mask[w];
      while (b) {
        const int c = 32 * w + __ffs(b) - 1;
        b &= b - 1;
        acc += slack[c];
        last = c;
        if ((uint64_t)acc > u) return c;
      }
    }
    return last;
  }
  int lo = r;
#pragma unroll
  for (int w = 0; w < kRW; ++w) {
    unsigned b = mask[w];
    while (b) {
      const int c = 32 * w + __ffs(b) - 1;
      b &= b - 1;
      if (W[c] < W[lo] || (W[c] == W[lo] && c < lo)) lo = c;
    }
  }
  return W[r] <= W[lo] + B ? r : lo;
}

// a5 for one warp's sub-chunk of source rank r (tokens [t0, t1)): dr holds the
// destination rank of each of the sub-chunk's assignments (kNoRank if none);
// every token picks its shared-expert rank (wf_pick) and gets its ordinal among
// the sub-chunk's tokens with the same pick (match.any groups, in token order);
// the sub-chunk's pick counts per destination rank go to wsub_cnt for
// k_shared_scan, and k_fixup turns the ordinals into rows.
__device__ __forceinline__ void waterfill_subchunk(const Dims& d, const LayerBuf& L, const Scratch& s,
                                                   int r, int sub, int t0, int t1,
                                                   const uint8_t* dr, int32_t* wrun,
                                                   const int32_t* s_slack, const int32_t* s_W,
                                                   int lane) {
  const int R = d.R, K = d.K;
  const int gw = r * d.nsub + sub;
  for (int q = lane; q < R; q += 32) wrun[q] = 0;
  __syncwarp();
  const int B = s.wf[1];
  for (int t = t0; t < t1; t += 32) {
    const int tt = t + lane;
    int c = -1;
    if (tt < t1) {
      unsigned mask[kRW] = {0u, 0u, 0u, 0u};
      if (d.all_ranks) {
        mask_all(mask, R);
      } else {
        for (int k = 0; k < K; ++k) {
          const int q = dr[(tt - t0) * K + k];
          if (q != kNoRank) mask_set(mask, q);
        }
      }
      mask_clear(mask, r);
      c = wf_pick(r, (int64_t)r * d.T + tt, mask, s_slack, s_W, B, d.seed);
    }
    const unsigned peers = __match_any_sync(kFull, c);
    const int rk = __popc(peers & lanemask_lt());
    const int o = c >= 0 ? wrun[c] + rk : 0;
    __syncwarp();
    if (c >= 0 && lane == __ffs(peers) - 1) wrun[c] = o + __popc(peers);
    __syncwarp();
    if (tt < t1) {
      L.shared_rank[(int64_t)r * d.T + tt] = c;
      L.shared_row[(int64_t)r * d.T + tt] = o;  // ordinal inside (c, sub-chunk) for now
    }
  }
  __syncwarp();
  for (int q = lane; q < R; q += 32) s.wsub_cnt[(int64_t)q * R * d.nsub + gw] = wrun[q];
}

// ---------------------------------------------------------------------------
// a4 (+a5): token assignment.  A block owns up to 8 consecutive sub-chunks of
// one source rank r (one per warp).  The stable ordinal of (t, k) among rank
// r's assignments of expert e = the counts of the rank's earlier blocks + those
// of the block's earlier warps + the warp's running count + the rank inside
// the 32-lane match.any group; these need only the ids and the histogram, so
// the block computes them before waiting for the rerouting (while the solve
// runs).  After the wait it copies rank r's per-expert segment records (the
// first two segments and where the third begins) into shared memory, and each
// ordinal selects its segment and thus its row.
// PASS 0 (no shared expert): rows.  PASS 1 (shared expert): rows relative to
// the destination rank's block and the destination ranks, then the Waterfill
// pick of every token, its ordinal among the sub-chunk's tokens with that pick,
// and the sub-chunk's pick counts per destination rank; k_fixup adds the rank
// bases once the shared columns are laid out.
// ---------------------------------------------------------------------------
// The token assignment keeps an assignment's expert (<= E <= 1024, 11 bits)
// and ordinal in one word when every ordinal of a source rank is below 2^21.
__host__ __device__ __forceinline__ bool assign_packed(const Dims& d) {
  return (int64_t)d.T * d.K <= ((int64_t)1 << 21);
}

template <int PASS>
struct AssignCtx {
  const int2* sge;       // [E+1] per expert: first row base (INT_MIN: none), second
                         // segment's first ordinal (slot E: dummy)
  const uint8_t* rk0;    // [E+1] first segment's destination rank (PASS 1)
  const int4* rec1;      // [E] second segment, where the third begins, last segment
  const int32_t* gord;   // the rerouting's segment lists in global memory
  const int32_t* gbase;
  const int32_t* grk;
  int32_t* drow;         // dst_row of the source rank
  uint8_t* grank;        // destination-rank bytes of the source rank (PASS 1)
  uint8_t* dr;           // the sub-chunk's destination ranks in shared memory (PASS 1)
  int a0, E;
};

// The row (and destination rank) of ordinal o of expert e; ok is false for a
// dropped id or an expert without segments.  The segment is the last one that
// starts at or before o: the first two are in shared memory (the first in an
// 8-byte record), a third or later one (rare: a source rank's demand spread
// over several remote instances) is found in the rerouting's list in global
// memory.
template <int PASS>
__device__ __forceinline__ void assign_finish(const AssignCtx<PASS>& c, int e, int o, bool valid,
                                              int idx, bool& inconsistent) {
  const int2 g = c.sge[e];
  int b = g.x, q = PASS > 0 ? c.rk0[e] : 0;
  if (o >= g.y) {
    const int4 h = c.rec1[e];
    b = h.y;
    q = h.x & 0xff;
    if (o >= h.z) {
      const int third = h.w - (h.x >> 8) + 3;
      int si = h.w;
      while (si > third && c.gord[si] > o) --si;
      b = c.gbase[si];
      if (PASS > 0) q = c.grk[si];
    }
  }
  const bool has = g.x != INT_MIN;
  const bool ok = valid && has;
  inconsistent |= valid && !has;
  c.drow[idx] = ok ? b + o : -1;
  if (PASS > 0) {
    const uint8_t rank = ok ? (uint8_t)q : (uint8_t)kNoRank;
    c.dr[idx - c.a0] = rank;
    c.grank[idx] = rank;
  }
}

// The stable ordinals of one warp's sub-chunk [a0, a1) of the source rank's
// assignments, in rounds of 32: an assignment's ordinal is its expert's
// running count plus its rank inside the round's match.any group (the group's
// leader advances the count).  Only the ids and the histogram's counts enter,
// so this runs before the wait for the rerouting.  so/se receive each
// assignment's ordinal and expert (E for a dropped id); when every ordinal is
// below 2^21 (pk) both travel in so as o | e << 21 and se is unused.  v holds
// the first batch of ids.
__device__ __forceinline__ void assign_ordinals(const int32_t* __restrict__ src, int32_t* run,
                                                int a0, int a1, int E, int lane, unsigned lt,
                                                bool pk, int (&v)[kAsgBatch], int32_t* so,
                                                uint16_t* se) {
  for (int a = a0; a < a1; a += kAsgBatch * 32) {
    if (a != a0) {
#pragma unroll
      for (int u = 0; u < kAsgBatch; ++u) {
        const int idx = a + u * 32 + lane;
        v[u] = idx < a1 ? __ldg(src + idx) : -1;
      }
    }
#pragma unroll
    for (int u = 0; u < kAsgBatch; ++u) {
      if (a + u * 32 >= a1) break;  // warp-uniform
      const int idx = a + u * 32 + lane;
      const bool in = idx < a1;
      const int e = in && v[u] >= 0 && v[u] < E ? v[u] : E;
      const unsigned peers = __match_any_sync(kFull, e);
      const int o = run[e] + __popc(peers & lt);
      __syncwarp();
      if (lane == __ffs(peers) - 1) run[e] = o + __popc(peers);  // the leader's o is the count
      __syncwarp();
      if (in) {
        if (pk) {
          so[idx - a0] = (int32_t)((unsigned)o | ((unsigned)e << 21));
        } else {
          so[idx - a0] = o;
          se[idx - a0] = (uint16_t)e;
        }
      }
    }
  }
}

template <int PASS>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 6)
k_assign(const int32_t* __restrict__ ids, Dims d, LayerBuf L, Scratch s) {
  extern __shared__ __align__(16) int32_t sm[];
  __shared__ int32_t s_slack[kMaxR];
  __shared__ int32_t s_W[kMaxR];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthr = blockDim.x;
  const int R = d.R, E = d.E, K = d.K;
  const int nbpr = (d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int r = blockIdx.x / nbpr;
  const int sub0 = (blockIdx.x - r * nbpr) * kWarpsPerBlock;
  const int sub = sub0 + warp;
  const bool active = sub < d.nsub;
  // the rerouting's records of source rank r (see k_reroute); slot E of the
  // first table and of the running counts is a dummy that dropped ids (and
  // lanes past the end of the sub-chunk) share
  int4* rec1 = reinterpret_cast<int4*>(sm);             // [E]
  int2* sge = reinterpret_cast<int2*>(rec1 + E);        // [E+1]
  uint8_t* rk0 = reinterpret_cast<uint8_t*>(sge + E + 1);  // [E+1] (PASS 1)
  int32_t* base0 = sm + 4 * E + 2 * (E + 1) + (PASS > 0 ? (E + 4) / 4 : 0);  // [E]
  const int nsa = kPlanSubT * K;                        // assignments per sub-chunk
  const bool pk = assign_packed(d);                     // expert and ordinal in one word
  const int per_warp = E + 1 + nsa + (pk ? 0 : (nsa + 1) / 2) + (PASS > 0 ? R + (nsa + 3) / 4 : 0);
  int32_t* run = base0 + E + warp * per_warp;           // [E+1] running ordinals
  int32_t* so = run + E + 1;                            // [nsa] ordinals (| expert << 21)
  uint16_t* se = reinterpret_cast<uint16_t*>(so + nsa); // [nsa] experts (E: dropped), !pk
  int32_t* wrun = so + nsa + (pk ? 0 : (nsa + 1) / 2);  // [R] running shared ordinals
  uint8_t* dr = reinterpret_cast<uint8_t*>(wrun + R);   // [nsa] destination ranks

  // The first batch of ids is an input no kernel of the plan writes: fetch it
  // before waiting for the predecessor grid.
  const int t0 = active ? sub * kPlanSubT : 0, t1 = active ? min(d.T, t0 + kPlanSubT) : 0;
  const int a0 = t0 * K, a1 = t1 * K;
  const int64_t rbase = (int64_t)r * d.T * K;
  int v[kAsgBatch];
#pragma unroll
  for (int u = 0; u < kAsgBatch; ++u) {
    const int idx = a0 + u * 32 + lane;
    v[u] = idx < a1 ? __ldg(ids + rbase + idx) : -1;
  }
  pdl_trigger();

  // Before waiting: the histogram's counts.  The histogram finished before the
  // solve passed its own wait and triggered the rerouting, whose trigger
  // launched this grid, so its block and sub-chunk counts are complete here.
  // The exclusive base of the block's first sub-chunk (earlier blocks of this
  // rank), then each warp's running counts (plus the block's earlier warps),
  // then the warp's ordinals.  On a plan of one layer this overlaps the solve,
  // which occupies a few SMs and leaves the rest to these blocks.
  for (int e = tid; e < E; e += nthr) base0[e] = 0;
  __syncthreads();
  const int32_t* cnt_r = s.sub_cnt + (int64_t)r * d.nsub * E;
  {
    const int32_t* blk_r = s.blk_cnt + (int64_t)r * nbpr * E;
    const int n = (sub0 / kWarpsPerBlock) * E;
    for (int i = tid; i < n; i += nthr * 8) {
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int ii = i + u * nthr;
        c[u] = ii < n ? blk_r[ii] : 0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int ii = i + u * nthr;
        if (c[u]) atomicAdd(&base0[ii % E], c[u]);
      }
    }
  }
  __syncthreads();
  if (active) {
    for (int e = lane; e < E; e += 32) {
      int c[kWarpsPerBlock];  // the block's earlier warps' counts, loaded together
#pragma unroll
      for (int w = 0; w < kWarpsPerBlock; ++w)
        c[w] = w < warp ? cnt_r[(int64_t)(sub0 + w) * E + e] : 0;
      int acc = base0[e];
#pragma unroll
      for (int w = 0; w < kWarpsPerBlock; ++w) acc += c[w];
      run[e] = acc;
    }
    if (lane == 0) run[E] = 0;
    __syncwarp();
    assign_ordinals(ids + rbase, run, a0, a1, E, lane, lanemask_lt(), pk, v, so, se);
  }
  pdl_wait();

  // rank r's segment records (the rerouting's output), and with a shared
  // expert the Waterfill slack and loads
  {
    const int4* rec = reinterpret_cast<const int4*>(s.seg_rec) + (int64_t)r * E * 2;
    for (int i = tid; i < 2 * E; i += nthr) {
      const int4 x = rec[i];
      if (i & 1) {
        rec1[i >> 1] = x;
      } else {
        sge[i >> 1] = make_int2(x.x, x.y);
        if (PASS > 0) rk0[i >> 1] = (uint8_t)x.z;
      }
    }
    if (tid == 0) sge[E] = make_int2(0, INT_MAX);
  }
  if (PASS > 0)
    for (int q = tid; q < R; q += nthr) {
      s_slack[q] = s.slack[q];
      s_W[q] = L.W[q];
    }
  __syncthreads();
  if (!active) return;

  // Each assignment's ordinal selects its segment and thus its row: the
  // expert's segment record first (dropped ids share the dummy slot E).
  bool inconsistent = false;
  AssignCtx<PASS> c{sge, rk0, rec1, s.seg_ord, s.seg_base, s.seg_rank, L.dst_row + rbase,
                    PASS > 0 ? s.asg_rank + rbase : nullptr, dr, a0, E};
  __syncwarp();
#pragma unroll 4
  for (int i = lane; i < a1 - a0; i += 32) {
    const unsigned w = (unsigned)so[i];
    const int e = pk ? (int)(w >> 21) : se[i], o = pk ? (int)(w & 0x1FFFFFu) : (int)w;
    assign_finish<PASS>(c, e, o, e < E, a0 + i, inconsistent);
  }
  if (__any_sync(kFull, inconsistent) && lane == 0) atomicOr(&L.stats->status, EP_DEV_INCONSISTENT);
  if (PASS > 0) waterfill_subchunk(d, L, s, r, sub, t0, t1, dr, wrun, s_slack, s_W, lane);
}

// ---------------------------------------------------------------------------
// Sampled rerouting ("Waterfill and LPLB" page, section "LPLB": the per-expert
// split, normalised to a distribution over the expert's physical instances,
// from which every token samples one instance).  An instance key is
// kappa = e + rep_eptr[e] + j for the j-th instance of e in instance order, so
// the keys of one expert are contiguous and there are E + replicas of them.
//
// k_sample: same blocks as k_hist.  Each assignment a = (r*T + t)*K + k of
// expert e draws its key: with more than one instance,
// h = SplitMix64(sampling_seed + a), u = ((h >> 32) * total_e) >> 32 and the
// key is the first of e's keys whose running quota sum exceeds u (binary
// search); with one instance, that instance.  The warp counts its keys in a
// shared histogram and writes the sub-chunk's row of counts; the block writes
// its sum and adds it into the per-(source rank, key) accumulator.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
k_sample(const int32_t* __restrict__ ids, Dims d, LayerBuf L, Scratch s) {
  extern __shared__ int32_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthr = blockDim.x;
  const int E = d.E, K = d.K, NK = d.nkey;
  const int nbpr = (d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int r = blockIdx.x / nbpr, b = blockIdx.x - r * nbpr;
  const int sub = b * kWarpsPerBlock + warp;
  int32_t* s_cum = sm;                 // [NK]
  int32_t* s_eptr = s_cum + NK;        // [E+1]
  int32_t* s_tot = s_eptr + E + 1;     // [E]
  int32_t* hists = s_tot + E;          // [warps][NK]
  int32_t* hist = hists + warp * NK;
  // the first batch of ids is an input no kernel of the plan writes: fetch it
  // before waiting
  const bool active = sub < d.nsub;
  const int t0 = active ? sub * kPlanSubT : 0, t1 = active ? min(d.T, t0 + kPlanSubT) : 0;
  const int64_t rbase = (int64_t)r * d.T * K;
  const int a1 = t1 * K;
  int v[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int idx = t0 * K + u * 32 + lane;
    v[u] = idx < a1 ? __ldg(ids + rbase + idx) : -1;
  }
  pdl_trigger();
  pdl_wait();
  for (int e = tid; e <= E; e += nthr) s_eptr[e] = L.rep_eptr[e];
  for (int e = tid; e < E; e += nthr) s_tot[e] = L.expert_total[e];
  __syncthreads();
  const int nk = E + s_eptr[E];  // keys in use
  for (int i = tid; i < nk; i += nthr) s_cum[i] = s.smp_cum[i];
  for (int i = lane; i < nk; i += 32) hist[i] = 0;
  __syncthreads();
  if (active) {
    for (int a = t0 * K; a < a1; a += kBatch * 32) {
      if (a != t0 * K) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int idx = a + u * 32 + lane;
          v[u] = idx < a1 ? __ldg(ids + rbase + idx) : -1;
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = a + u * 32 + lane;
        if (idx >= a1) continue;
        const int e = v[u];
        int key = 0xFFFF;
        if (e >= 0 && e < E) {
          const int kb = e + s_eptr[e];
          const int n = 1 + s_eptr[e + 1] - s_eptr[e];
          int lo = 0;
          if (n > 1) {
            const uint64_t h = splitmix64(d.sseed + (uint64_t)(rbase + idx));
            const int u32 = (int)(((h >> 32) * (uint64_t)s_tot[e]) >> 32);
            int hi = n - 1;  // s_cum[kb + n - 1] = total > u: the answer exists
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              if (s_cum[kb + mid] > u32) hi = mid; else lo = mid + 1;
            }
          }
          key = kb + lo;
          atomicAdd(&hist[key], 1);
        }
        s.smp_key[rbase + idx] = (uint16_t)key;
      }
    }
    __syncwarp();
    int32_t* out = s.smp_sub + ((int64_t)r * d.nsub + sub) * NK;
    for (int i = lane; i < nk; i += 32) out[i] = hist[i];
  }
  __syncthreads();
  int32_t* blk = s.smp_blk + ((int64_t)r * nbpr + b) * NK;
  for (int i = tid; i < nk; i += nthr) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kWarpsPerBlock; ++w) c += hists[w * NK + i];
    blk[i] = c;
    if (c) atomicAdd(&s.smp_tot[r * NK + i], c);
  }
}

// k_sample_layout: one CTA, a thread per key (consecutive keys read
// consecutive words of each source rank's row, eight rows in flight).  Pass 1:
// the key's draws summed over source ranks, which is its instance's row
// count.  Then the rank-relative first row of every instance, each rank's
// routed rows and the dispatch layout (without a shared expert; with one,
// k_shared_scan lays the ranks out).  Pass 2: the first row of every (source
// rank, key) — the instance's first row plus the draws of earlier sources —
// absolute or rank-relative; the accumulator is zeroed for the next call.
constexpr int kLayoutThreads = 1024;

__global__ void __launch_bounds__(kLayoutThreads) k_sample_layout(Dims d, LayerBuf L, Scratch s) {
  extern __shared__ int32_t sm[];
  __shared__ int32_t s_base[kMaxR + 1];
  __shared__ int32_t s_nk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = d.R, E = d.E, G = d.G, NK = d.nkey, RG = d.R * d.G;
  const int routed = d.Gmax + d.S;
  int32_t* s_kcnt = sm;            // [NK] draws per key
  int32_t* s_kinst = s_kcnt + NK;  // [NK] instance of the key
  int32_t* s_icnt = s_kinst + NK;  // [R*G] rows per instance
  int32_t* s_rel = s_icnt + RG;    // [R*G] rank-relative first row
  // wait first: the assignment pass, launched at this trigger, may then read
  // the sampling pass's draws before waiting for this layout
  pdl_wait();
  pdl_trigger();
  if (tid == 0) s_nk = E + L.rep_eptr[E];
  for (int i = tid; i < RG; i += kLayoutThreads) s_icnt[i] = 0;
  __syncthreads();
  const int nk = s_nk;
  for (int k = tid; k < nk; k += kLayoutThreads) {  // consecutive keys: coalesced rows
    int sum = 0, r = 0;
    for (; r + 8 <= R; r += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = s.smp_tot[(r + u) * NK + k];
#pragma unroll
      for (int u = 0; u < 8; ++u) sum += v[u];
    }
    for (; r < R; ++r) sum += s.smp_tot[r * NK + k];
    s_kcnt[k] = sum;
    s_kinst[k] = s.smp_inst[k];
  }
  __syncthreads();
  for (int k = tid; k < nk; k += kLayoutThreads) {
    const int i = s_kinst[k];
    if (i >= 0 && i < RG) s_icnt[i] = s_kcnt[k];  // each routed instance has one key
  }
  __syncthreads();
  for (int i = tid; i < RG; i += kLayoutThreads) L.inst_count[i] = s_icnt[i];
  if (tid < R) {
    int run = 0;
    for (int col = 0; col < G; ++col) {
      s_rel[tid * G + col] = run;
      s.inst_rel[tid * G + col] = run;
      if (col < routed) run += s_icnt[tid * G + col];
    }
    s.rank_rows[tid] = run;
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0, mx = 0;
    for (int q0 = 0; q0 < R; q0 += 32) {
      const int q = q0 + lane;
      const int v = q < R ? s.rank_rows[q] : 0;
      mx = max(mx, v);
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (q < R) s_base[q] = carry + incl - v;
      carry += __shfl_sync(kFull, incl, 31);
    }
    mx = (int)__reduce_max_sync(kFull, (unsigned)mx);
    if (lane == 0) {
      s_base[R] = carry;
      L.stats->realized_max = mx;
    }
  }
  __syncthreads();
  if (!d.sh) {
    for (int i = tid; i < RG; i += kLayoutThreads) L.inst_off[i] = s_base[i / G] + s_rel[i];
    if (tid == 0) {
      L.inst_off[RG] = s_base[R];
      L.stats->rows = s_base[R];
    }
    for (int q = tid; q <= R; q += kLayoutThreads) L.rank_base[q] = s_base[q];
  }
  for (int k = tid; k < nk; k += kLayoutThreads) {
    const int i = s_kinst[k];
    if (i < 0 || i >= RG) continue;  // every key has an instance; guard the tables anyway
    int run = d.sh ? s_rel[i] : s_base[i / G] + s_rel[i];
    int r = 0;
    for (; r + 8 <= R; r += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = s.smp_tot[(r + u) * NK + k];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        s.smp_row0[(r + u) * NK + k] = run;
        s.smp_tot[(r + u) * NK + k] = 0;  // zero again for the next call
        run += v[u];
      }
    }
    for (; r < R; ++r) {
      const int v = s.smp_tot[r * NK + k];
      s.smp_row0[r * NK + k] = run;
      s.smp_tot[r * NK + k] = 0;
      run += v;
    }
  }
}

// k_sample_assign: same blocks as k_assign.  The row of an assignment with key
// kappa is the first row of (r, kappa) plus its ordinal among rank r's
// assignments with that key in (t, k) order: the counts of the rank's earlier
// blocks and the block's earlier warps, the warp's running count and the rank
// inside the 32-lane match.any group.  The ordinals need only the draws, so
// they are computed before the wait (while the layout kernel runs); after it
// the first rows are added.  SH: rows relative to the destination rank's block
// and the destination rank bytes, then the Waterfill picks
// (waterfill_subchunk), exactly as k_assign<1>.
__host__ __device__ __forceinline__ bool sample_assign_packed(const Dims& d) {
  // ordinal and key (< 2^12 with the dummy) in one word
  return (int64_t)d.T * d.K <= ((int64_t)1 << 20);
}

template <int SH>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
k_sample_assign(Dims d, LayerBuf L, Scratch s) {
  extern __shared__ __align__(16) int32_t sm[];
  __shared__ int32_t s_slack[kMaxR];
  __shared__ int32_t s_W[kMaxR];
  __shared__ int32_t s_nk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthr = blockDim.x;
  const int R = d.R, E = d.E, K = d.K, NK = d.nkey, G = d.G;
  const int nbpr = (d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int r = blockIdx.x / nbpr;
  const int sub0 = (blockIdx.x - r * nbpr) * kWarpsPerBlock;
  const int sub = sub0 + warp;
  const bool active = sub < d.nsub;
  int32_t* s_row0 = sm;                        // [NK] first row of (r, key)
  int32_t* s_krank = s_row0 + NK;              // [NK] destination rank of the key (SH)
  int32_t* base0 = s_krank + (SH ? NK : 0);    // [NK] draws of the rank's earlier blocks
  const int nsa = kPlanSubT * K;
  const bool pk = sample_assign_packed(d);
  const int per_warp = NK + nsa + (pk ? 0 : (nsa + 1) / 2) + (SH ? R + (nsa + 3) / 4 : 0);
  int32_t* run = base0 + NK + warp * per_warp; // [NK] running ordinals
  int32_t* so = run + NK;                      // [nsa] ordinals (| key << 20)
  uint16_t* sk = reinterpret_cast<uint16_t*>(so + nsa);  // [nsa] keys (!pk)
  int32_t* wrun = so + nsa + (pk ? 0 : (nsa + 1) / 2);   // [R] running shared ordinals (SH)
  uint8_t* dr = reinterpret_cast<uint8_t*>(wrun + R);    // [nsa] ranks (SH)
  pdl_trigger();
  // Before waiting: the draws (the sampling pass had completed before the
  // layout passed its own wait and launched this grid) — the exclusive base
  // of the block's first sub-chunk and each warp's running counts.
  if (tid == 0) s_nk = E + L.rep_eptr[E];
  __syncthreads();
  const int nk = s_nk;
  {
    const int32_t* blk_r = s.smp_blk + (int64_t)r * nbpr * NK;
    const int nb = sub0 / kWarpsPerBlock;
    for (int k = tid; k < nk; k += nthr) {
      int acc = 0;
      for (int b0 = 0; b0 < nb; b0 += 8) {  // eight loads in flight
        int c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) c[u] = b0 + u < nb ? blk_r[(int64_t)(b0 + u) * NK + k] : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) acc += c[u];
      }
      base0[k] = acc;
      if (SH) s_krank[k] = s.smp_inst[k] / G;
    }
  }
  __syncthreads();
  const int32_t* cnt_r = s.smp_sub + (int64_t)r * d.nsub * NK;
  if (active) {
    for (int k = lane; k < nk; k += 32) {
      int c[kWarpsPerBlock];
#pragma unroll
      for (int w = 0; w < kWarpsPerBlock; ++w)
        c[w] = w < warp ? cnt_r[(int64_t)(sub0 + w) * NK + k] : 0;
      int acc = base0[k];
#pragma unroll
      for (int w = 0; w < kWarpsPerBlock; ++w) acc += c[w];
      run[k] = acc;
    }
  }
  const int t0 = active ? sub * kPlanSubT : 0, t1 = active ? min(d.T, t0 + kPlanSubT) : 0;
  const int a0 = t0 * K, a1 = t1 * K;
  const int64_t rbase = (int64_t)r * d.T * K;
  if (active) {
    __syncwarp();
    for (int a = a0; a < a1; a += kAsgBatch * 32) {
      int v[kAsgBatch];
#pragma unroll
      for (int u = 0; u < kAsgBatch; ++u) {
        const int idx = a + u * 32 + lane;
        v[u] = idx < a1 ? (int)s.smp_key[rbase + idx] : 0xFFFF;
      }
#pragma unroll
      for (int u = 0; u < kAsgBatch; ++u) {
        if (a + u * 32 >= a1) break;
        const int idx = a + u * 32 + lane;
        const int key = v[u] < nk ? v[u] : nk;  // nk: a dropped id
        const unsigned peers = match_bits(key, 32 - __clz(nk));
        const int rk = __popc(peers & lanemask_lt());
        const int o = key < nk ? run[key] + rk : 0;
        __syncwarp();
        if (key < nk && lane == __ffs(peers) - 1) run[key] = o + __popc(peers);
        __syncwarp();
        if (idx < a1) {
          if (pk) {
            so[idx - a0] = (int32_t)((unsigned)o | ((unsigned)key << 20));
          } else {
            so[idx - a0] = o;
            sk[idx - a0] = (uint16_t)key;
          }
        }
      }
    }
  }
  pdl_wait();
  for (int k = tid; k < nk; k += nthr) s_row0[k] = s.smp_row0[r * NK + k];
  if (SH)
    for (int q = tid; q < R; q += nthr) {
      s_slack[q] = s.slack[q];
      s_W[q] = L.W[q];
    }
  __syncthreads();
  if (!active) return;
#pragma unroll 4
  for (int i = lane; i < a1 - a0; i += 32) {
    const unsigned w = (unsigned)so[i];
    const int key = pk ? (int)(w >> 20) : sk[i], o = pk ? (int)(w & 0xFFFFFu) : (int)w;
    const bool ok = key < nk;
    L.dst_row[rbase + a0 + i] = ok ? s_row0[key] + o : -1;
    if (SH) {
      const uint8_t q = ok ? (uint8_t)s_krank[key] : (uint8_t)kNoRank;
      dr[i] = q;
      s.asg_rank[rbase + a0 + i] = q;
    }
  }
  if (SH) {
    __syncwarp();
    waterfill_subchunk(d, L, s, r, sub, t0, t1, dr, wrun, s_slack, s_W, lane);
  }
}

// ---------------------------------------------------------------------------
// Waterfill re-run of a cached layer.  k_wf_layer_prep (one CTA) rebuilds from
// the layer's cache what the shared-slot pass reads from the scratch: routed
// rows per rank and each instance's rank-relative first row (from the row
// counts), the waterline H = ceil((A + N)/R), the local preference B and the
// slack of every rank (from the planned loads), and keeps the old rank bases.
// k_wf_layer (the blocks of k_assign) turns each routed row back into its
// destination rank and rank-relative row, then draws the sub-chunk's shared
// ranks (waterfill_subchunk); k_shared_scan and k_fixup lay the ranks out again.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_wf_layer_prep(Dims d, LayerBuf L, Scratch s) {
  __shared__ int32_t s_A;
  pdl_trigger();
  const int tid = threadIdx.x;
  const int R = d.R, G = d.G, routed = d.Gmax + d.S;
  if (tid == 0) s_A = (int32_t)L.stats->assignments;
  for (int q = tid; q <= R; q += blockDim.x) s.prev_base[q] = L.rank_base[q];
  __syncthreads();
  const int64_t N = (int64_t)R * d.T;
  const int64_t H = ((int64_t)s_A + N + R - 1) / R;
  if (tid == 0) {
    s.wf[0] = (int)H;
    s.wf[1] = (int)((H * d.bonus + 999) / 1000);
  }
  for (int q = tid; q < R; q += blockDim.x) {
    int run = 0;
    for (int col = 0; col < G; ++col) {
      s.inst_rel[q * G + col] = run;
      if (col < routed) run += L.inst_count[q * G + col];
    }
    s.rank_rows[q] = run;
    s.slack[q] = (int)max(H - (int64_t)L.W[q], (int64_t)0);
  }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_wf_layer(Dims d, LayerBuf L, Scratch s) {
  extern __shared__ __align__(16) int32_t sm[];
  __shared__ int32_t s_slack[kMaxR];
  __shared__ int32_t s_W[kMaxR];
  __shared__ int32_t s_pb[kMaxR + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthr = blockDim.x;
  const int R = d.R, K = d.K;
  const int nbpr = (d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const int r = blockIdx.x / nbpr;
  const int sub = (blockIdx.x - r * nbpr) * kWarpsPerBlock + warp;
  const int per_warp = R + (kPlanSubT * K + 3) / 4;
  int32_t* wrun = sm + warp * per_warp;                 // [R]
  uint8_t* dr = reinterpret_cast<uint8_t*>(wrun + R);   // [kPlanSubT*K]
  pdl_trigger();
  pdl_wait();
  for (int q = tid; q < R; q += nthr) {
    s_slack[q] = s.slack[q];
    s_W[q] = L.W[q];
  }
  for (int q = tid; q <= R; q += nthr) s_pb[q] = s.prev_base[q];
  __syncthreads();
  if (sub >= d.nsub) return;
  const int t0 = sub * kPlanSubT, t1 = min(d.T, t0 + kPlanSubT);
  const int a0 = t0 * K, a1 = t1 * K;
  const int64_t rbase = (int64_t)r * d.T * K;
  for (int idx = a0 + lane; idx < a1; idx += 32) {
    const int row = L.dst_row[rbase + idx];
    uint8_t q8 = (uint8_t)kNoRank;
    if (row >= 0) {
      int lo = 0, hi = R - 1;  // the last rank whose block starts at or before row
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pb[mid] <= row) lo = mid; else hi = mid - 1;
      }
      q8 = (uint8_t)lo;
      L.dst_row[rbase + idx] = row - s_pb[lo];
    }
    dr[idx - a0] = q8;
    s.asg_rank[rbase + idx] = q8;
  }
  __syncwarp();
  waterfill_subchunk(d, L, s, r, sub, t0, t1, dr, wrun, s_slack, s_W, lane);
}

// Shared-slot layout: block c scans destination rank c's pick counts over
// (source rank, sub-chunk) — rows ordered by (source rank, token) — in place;
// the last block to finish (arrival ticket, no waiting) lays out every rank's
// block: routed rows followed by its shared column.
constexpr int kScanThreads = 256;
constexpr int kScanItems = 8;

__global__ void __launch_bounds__(kScanThreads) k_shared_scan(Dims d, LayerBuf L, Scratch s) {
  __shared__ int32_t s_wsum[kScanThreads / 32];
  __shared__ int32_t s_carry;
  __shared__ int32_t s_last;
  __shared__ int32_t s_base[kMaxR + 1];
  // wait first: the fix-up, launched at this trigger, may then read the
  // assignment pass's rows and rank bytes before waiting for this scan
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = d.R, G = d.G;
  const int c = blockIdx.x;
  const int n = R * d.nsub;
  int32_t* col = s.wsub_cnt + (int64_t)c * n;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < n; b0 += kScanThreads * kScanItems) {
    const int i0 = b0 + tid * kScanItems;
    int v[kScanItems], local = 0;
#pragma unroll
    for (int u = 0; u < kScanItems; ++u) {
      v[u] = i0 + u < n ? col[i0 + u] : 0;
      local += v[u];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int run = s_carry + incl - local;
    for (int w = 0; w < warp; ++w) run += s_wsum[w];
#pragma unroll
    for (int u = 0; u < kScanItems; ++u) {
      if (i0 + u < n) col[i0 + u] = run;
      run += v[u];
    }
    __syncthreads();
    if (tid == kScanThreads - 1) s_carry = run;
    __syncthreads();
  }
  if (tid == 0) {
    s.shared_tot[c] = s_carry;
    __threadfence();
    s_last = atomicAdd(&s.acc_misc[1], 1) == R - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) s.acc_misc[1] = 0;  // every block has arrived: reset for the next call
  if (warp == 0) {
    int carry = 0;
    for (int q0 = 0; q0 < R; q0 += 32) {
      const int q = q0 + lane;
      const int v = q < R ? s.rank_rows[q] + s.shared_tot[q] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (q < R) s_base[q] = carry + incl - v;
      carry += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) s_base[R] = carry;
  }
  __syncthreads();
  const int scol = d.Gmax + d.S;
  for (int i = tid; i < R * G; i += kScanThreads) {
    const int q = i / G, cc = i - (i / G) * G;
    if (cc == scol) {
      L.inst_quota[i] = s.shared_tot[q];
      L.inst_count[i] = s.shared_tot[q];
      L.inst_off[i] = s_base[q] + s.rank_rows[q];
    } else {
      L.inst_off[i] = s_base[q] + s.inst_rel[i];
    }
  }
  for (int q = tid; q <= R; q += kScanThreads) {
    L.rank_base[q] = s_base[q];
    if (q < R) s.sbase[q] = s_base[q] + s.rank_rows[q];
  }
  if (tid == 0) {
    L.inst_off[R * G] = s_base[R];
    L.stats->rows = s_base[R];
  }
}

// Shared expert, once the shared columns are laid out: every routed row gets
// its destination rank's first row added, and every shared-slot row (still
// the token's ordinal among its sub-chunk's tokens with the same pick) gets
// its column's first row plus the picks of that rank in earlier (source rank,
// sub-chunk) pairs.  Elementwise; four routed rows per 16-byte access.
constexpr int kFixThreads = 256;

__global__ void __launch_bounds__(kFixThreads) k_fixup(Dims d, LayerBuf L, Scratch s) {
  __shared__ int32_t s_rb[kMaxR + 1];
  __shared__ int32_t s_sb[kMaxR];
  pdl_trigger();
  const int R = d.R;
  const int64_t A = (int64_t)R * d.T * d.K;
  const int N = R * d.T;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  // dst_row and the rank bytes both start 256-byte aligned
  const int64_t A4 = A / 4;
  int4* row4 = reinterpret_cast<int4*>(L.dst_row);
  const uint32_t* rk4 = reinterpret_cast<const uint32_t*>(s.asg_rank);
  // the first rows and rank bytes: the assignment pass that wrote them had
  // completed before the shared scan passed its wait and launched this grid
  int4 v0 = make_int4(0, 0, 0, 0);
  uint32_t q0w = 0;
  if (i0 < A4) {
    v0 = row4[i0];
    q0w = rk4[i0];
  }
  pdl_wait();
  for (int q = threadIdx.x; q <= R; q += blockDim.x) {
    s_rb[q] = L.rank_base[q];
    if (q < R) s_sb[q] = s.sbase[q];
  }
  __syncthreads();
  for (int64_t i = i0; i < A4; i += stride) {
    int4 v = i == i0 ? v0 : row4[i];
    const uint32_t q = i == i0 ? q0w : rk4[i];
    const int q0 = q & 0xffu, q1 = (q >> 8) & 0xffu, q2 = (q >> 16) & 0xffu, q3 = q >> 24;
    // a rank byte is a rank below R, or kNoRank for a dropped assignment;
    // anything else leaves the row alone
    if (q0 < R) v.x += s_rb[q0];
    if (q1 < R) v.y += s_rb[q1];
    if (q2 < R) v.z += s_rb[q2];
    if (q3 < R) v.w += s_rb[q3];
    row4[i] = v;
  }
  for (int64_t i = 4 * A4 + i0; i < A; i += stride) {
    const int q = s.asg_rank[i];
    if (q < R) L.dst_row[i] += s_rb[q];
  }
  const int n = R * d.nsub;
  for (int64_t t = i0; t < N; t += stride) {
    const int c = L.shared_rank[t];
    if ((unsigned)c >= (unsigned)R) continue;  // every pick is a rank; guard the tables anyway
    const int r = (int)t / d.T, tt = (int)t - r * d.T;
    L.shared_row[t] += s_sb[c] + s.wsub_cnt[(int64_t)c * n + r * d.nsub + tt / kPlanSubT];
  }
}

// Standalone Waterfill: one thread per token; the waterline is recomputed per
// block from the loads (R <= 128 values).
__global__ void __launch_bounds__(256)
k_waterfill(int R, int T, int K, const int32_t* __restrict__ load,
            const int32_t* __restrict__ dst_rank, uint64_t seed, int bonus, int all_ranks,
            int32_t* __restrict__ pick, int32_t* __restrict__ count) {
  __shared__ int32_t s_load[kMaxR], s_slack[kMaxR];
  __shared__ int64_t s_sum;
  if (threadIdx.x == 0) s_sum = 0;
  __syncthreads();
  for (int q = threadIdx.x; q < R; q += blockDim.x) {
    s_load[q] = load[q];
    atomicAdd(reinterpret_cast<unsigned long long*>(&s_sum), (unsigned long long)load[q]);
  }
  __syncthreads();
  const int64_t N = (int64_t)R * T;
  const int64_t H = (s_sum + N + R - 1) / R;
  const int B = (int)((H * bonus + 999) / 1000);
  for (int q = threadIdx.x; q < R; q += blockDim.x)
    s_slack[q] = (int)max(H - (int64_t)s_load[q], (int64_t)0);
  __syncthreads();
  const int64_t tok = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tok >= N) return;
  const int r = (int)(tok / T);
  unsigned mask[kRW] = {0u, 0u, 0u, 0u};
  if (all_ranks) {
    mask_all(mask, R);
  } else {
    for (int k = 0; k < K; ++k) {
      const int q = dst_rank[tok * K + k];
      if (q >= 0 && q < R) mask_set(mask, q);
    }
  }
  mask_clear(mask, r);
  const int c = wf_pick(r, tok, mask, s_slack, s_load, B, seed);
  pick[tok] = c;
  atomicAdd(&count[c], 1);
}

size_t sample_smem(const Dims& d) {
  return sizeof(int32_t) * ((size_t)d.nkey * (1 + kWarpsPerBlock) + 2 * (size_t)d.E + 1);
}
size_t sample_layout_smem(const Dims& d) {
  return sizeof(int32_t) * (2 * (size_t)d.nkey + 2 * (size_t)d.R * d.G);
}
size_t sample_assign_smem(const Dims& d) {
  const size_t nsa = (size_t)kPlanSubT * d.K;
  const size_t per_warp = d.nkey + nsa + (sample_assign_packed(d) ? 0 : (nsa + 1) / 2) +
                          (d.sh ? d.R + (nsa + 3) / 4 : 0);
  return sizeof(int32_t) *
         ((size_t)d.nkey * (d.sh ? 3 : 2) + (size_t)kWarpsPerBlock * per_warp);
}
size_t wf_layer_smem(const Dims& d) {
  return sizeof(int32_t) * (size_t)kWarpsPerBlock * (d.R + (kPlanSubT * d.K + 3) / 4);
}
size_t solve_smem(const Dims& d) {
  return sizeof(int32_t) *
         ((size_t)d.E * (1 + kSolveWarps) + ((size_t)d.E + 1) + 3 * (size_t)d.R * d.G);
}
size_t hist_smem(const Dims& d) { return sizeof(int32_t) * (size_t)kWarpsPerBlock * d.E; }
size_t assign_smem(const Dims& d, int pass) {
  const size_t nsa = (size_t)kPlanSubT * d.K;
  const size_t per_warp = (size_t)d.E + 1 + nsa + (assign_packed(d) ? 0 : (nsa + 1) / 2) +
                          (pass > 0 ? d.R + (nsa + 3) / 4 : 0);
  return sizeof(int32_t) * (4 * (size_t)d.E + 2 * ((size_t)d.E + 1) +
                            (pass > 0 ? ((size_t)d.E + 4) / 4 : 0) + d.E +
                            (size_t)kWarpsPerBlock * per_warp);
}

// Launch with programmatic stream serialisation: the kernel may begin while
// its predecessor in the stream is still running and waits for it in pdl_wait().
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace

// Allow every kernel the device's opt-in shared-memory maximum once, so that
// plans of any shape can coexist (each launch still requests only its own size),
// and prefer the largest shared-memory carveout for all of them.  The kernels of
// one plan run side by side under programmatic dependent launch (the token
// assignment's blocks compute their ordinals while the solve and the rerouting
// run), and an SM configured with a smaller carveout for a kernel that needs
// little shared memory could not take an assignment block until it drained.
template <typename F>
cudaError_t allow_plan_kernel(F* f, int max_smem) {
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
  return e != cudaSuccess ? e : allow_max_dynamic_smem(f, max_smem);
}
template <typename F>
cudaError_t prefer_max_carveout(F* f) {
  return cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}
template <int SMAX, bool PACK>
cudaError_t allow_solve_pack(int max_smem) {
  cudaError_t e;
  if ((e = allow_plan_kernel(k_solve<SMAX, 1, PACK>, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_solve<SMAX, 2, PACK>, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_solve<SMAX, 3, PACK>, max_smem)) != cudaSuccess) return e;
  return allow_plan_kernel(k_solve<SMAX, 4, PACK>, max_smem);
}
template <int SMAX>
cudaError_t allow_solve(int max_smem) {
  cudaError_t e = allow_solve_pack<SMAX, true>(max_smem);
  return e != cudaSuccess ? e : allow_solve_pack<SMAX, false>(max_smem);
}

cudaError_t set_plan_attributes(int max_smem) {
  cudaError_t e;
  if ((e = allow_solve<1>(max_smem)) != cudaSuccess) return e;
  if ((e = allow_solve<2>(max_smem)) != cudaSuccess) return e;
  if ((e = allow_solve<4>(max_smem)) != cudaSuccess) return e;
  if ((e = allow_solve<8>(max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_hist, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_assign<0>, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_assign<1>, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_sample, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_sample_layout, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_sample_assign<0>, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_sample_assign<1>, max_smem)) != cudaSuccess) return e;
  if ((e = allow_plan_kernel(k_wf_layer, max_smem)) != cudaSuccess) return e;
  if ((e = prefer_max_carveout(k_reroute)) != cudaSuccess) return e;
  if ((e = prefer_max_carveout(k_shared_scan)) != cudaSuccess) return e;
  if ((e = prefer_max_carveout(k_fixup)) != cudaSuccess) return e;
  return prefer_max_carveout(k_wf_layer_prep);
}

// The solve's dynamic shared memory: the whole of what the SM allows a block,
// so that no other block shares the SM of a solve CTA.  Each cap candidate's
// greedy is a serial chain of dependent steps; while it runs, the token
// assignment's blocks compute their ordinals on every other SM, and on the
// solve's SMs they would take issue slots from the chain.
//
// The fix-up's grid: the blocks that are resident at once.  Its blocks wait
// for the shared scan before their grid-stride loop, so a second wave of
// blocks would start only as the first one leaves.
cudaError_t plan_launch_shapes(Dims& d, int max_smem, int sms) {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, k_solve<1, 1, true>);
  if (e != cudaSuccess) return e;
  const size_t need = solve_smem(d), all = (size_t)max_smem - a.sharedSizeBytes;
  d.solve_smem = (int)(need > all ? need : all);
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_fixup, kFixThreads, 0);
  if (e != cudaSuccess) return e;
  d.fix_grid = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
  return cudaSuccess;
}

// The solve: a cluster of ceil(J / kSolveWarps) CTAs (one cap candidate per
// warp, at most four per SM), launched as a programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), unsigned ctas, unsigned block, size_t smem,
                               cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = ctas;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int SMAX>
cudaError_t launch_solve_rw(const Dims& d, const LayerBuf& L, const Scratch& s, cudaStream_t st) {
  const size_t ss = (size_t)d.solve_smem;
  const unsigned nt = kSolveThreads;
  const unsigned nc = (unsigned)((d.J + kSolveWarps - 1) / kSolveWarps);
  const int rw = (d.R + 31) / 32;
  if ((int64_t)d.R * d.T * d.K < ((int64_t)1 << 24)) {
    if (rw <= 1) return launch_pdl_cluster(k_solve<SMAX, 1, true>, nc, nt, ss, st, d, L, s);
    if (rw == 2) return launch_pdl_cluster(k_solve<SMAX, 2, true>, nc, nt, ss, st, d, L, s);
    if (rw == 3) return launch_pdl_cluster(k_solve<SMAX, 3, true>, nc, nt, ss, st, d, L, s);
    return launch_pdl_cluster(k_solve<SMAX, 4, true>, nc, nt, ss, st, d, L, s);
  }
  if (rw <= 1) return launch_pdl_cluster(k_solve<SMAX, 1, false>, nc, nt, ss, st, d, L, s);
  if (rw == 2) return launch_pdl_cluster(k_solve<SMAX, 2, false>, nc, nt, ss, st, d, L, s);
  if (rw == 3) return launch_pdl_cluster(k_solve<SMAX, 3, false>, nc, nt, ss, st, d, L, s);
  return launch_pdl_cluster(k_solve<SMAX, 4, false>, nc, nt, ss, st, d, L, s);
}

cudaError_t launch_solve(const Dims& d, const LayerBuf& L, const Scratch& s, cudaStream_t st) {
  if (d.S <= 1) return launch_solve_rw<1>(d, L, s, st);
  if (d.S <= 2) return launch_solve_rw<2>(d, L, s, st);
  if (d.S <= 4) return launch_solve_rw<4>(d, L, s, st);
  return launch_solve_rw<8>(d, L, s, st);
}

cudaError_t launch_shared_layout(const Dims& d, const LayerBuf& L, const Scratch& s,
                                 cudaStream_t st);

cudaError_t launch_balance(const Dims& d, const LayerBuf& L, const Scratch& s, const int32_t* ids,
                           cudaStream_t st) {
  // the histogram is a plain launch (it reads the caller's ids at once); every
  // later kernel is a programmatic dependent launch of its predecessor
  cudaError_t err = cudaSuccess;
  const unsigned nblk = (unsigned)(d.R * ((d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock));
  const unsigned bt = kWarpsPerBlock * 32;
  if (nblk > 0) {
    k_hist<<<nblk, bt, hist_smem(d), st>>>(ids, d, s);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  err = launch_solve(d, L, s, st);
  if (err != cudaSuccess) return err;
  err = launch_pdl(k_reroute, (unsigned)((d.E + kWarpsPerBlock - 1) / kWarpsPerBlock), bt, 0, st, d,
                   L, s);
  if (err != cudaSuccess) return err;
  if (d.sampled) {
    // sampled rerouting: draw keys, lay the instances out, then the rows
    if (nblk > 0) err = launch_pdl(k_sample, nblk, bt, sample_smem(d), st, ids, d, L, s);
    if (err != cudaSuccess) return err;
    err = launch_pdl(k_sample_layout, 1, kLayoutThreads, sample_layout_smem(d), st, d, L, s);
    if (err != cudaSuccess) return err;
    if (nblk > 0)
      err = d.sh ? launch_pdl(k_sample_assign<1>, nblk, bt, sample_assign_smem(d), st, d, L, s)
                 : launch_pdl(k_sample_assign<0>, nblk, bt, sample_assign_smem(d), st, d, L, s);
    if (err != cudaSuccess) return err;
  }
  if (!d.sh) {
    if (!d.sampled && nblk > 0)
      err = launch_pdl(k_assign<0>, nblk, bt, assign_smem(d, 0), st, ids, d, L, s);
  } else {
    if (!d.sampled && nblk > 0)
      err = launch_pdl(k_assign<1>, nblk, bt, assign_smem(d, 1), st, ids, d, L, s);
    if (err != cudaSuccess) return err;
    err = launch_shared_layout(d, L, s, st);
  }
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_shared_layout(const Dims& d, const LayerBuf& L, const Scratch& s,
                                 cudaStream_t st) {
  cudaError_t err = launch_pdl(k_shared_scan, (unsigned)d.R, kScanThreads, 0, st, d, L, s);
  if (err != cudaSuccess) return err;
  const int64_t A4 = (int64_t)d.R * d.T * d.K / 4, N = (int64_t)d.R * d.T;
  const int64_t work = A4 > N ? A4 : N;
  const int64_t fblk = (work + kFixThreads - 1) / kFixThreads;
  if (work > 0)
    err = launch_pdl(k_fixup, (unsigned)(fblk < d.fix_grid ? fblk : d.fix_grid), kFixThreads, 0, st,
                     d, L, s);
  return err;
}

cudaError_t launch_waterfill_layer(const Dims& d, const LayerBuf& L, const Scratch& s,
                                   cudaStream_t st) {
  k_wf_layer_prep<<<1, 256, 0, st>>>(d, L, s);
  cudaError_t err = cudaPeekAtLastError();
  if (err != cudaSuccess) return err;
  const unsigned nblk = (unsigned)(d.R * ((d.nsub + kWarpsPerBlock - 1) / kWarpsPerBlock));
  if (nblk > 0)
    err = launch_pdl(k_wf_layer, nblk, kWarpsPerBlock * 32, wf_layer_smem(d), st, d, L, s);
  if (err != cudaSuccess) return err;
  return launch_shared_layout(d, L, s, st);
}

cudaError_t launch_waterfill(int R, int T, int K, const int32_t* load, const int32_t* dst_rank,
                             uint64_t seed, int bonus, int all_ranks, int32_t* pick, int32_t* count,
                             cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(count, 0, sizeof(int32_t) * (size_t)R, st);
  if (err != cudaSuccess) return err;
  const int64_t N = (int64_t)R * T;
  if (N > 0)
    k_waterfill<<<(unsigned)((N + 255) / 256), 256, 0, st>>>(R, T, K, load, dst_rank, seed, bonus,
                                                             all_ranks, pick, count);
  return cudaGetLastError();
}

}  // namespace ep
