/*
 * CPU oracle of the UltraEP-style balance + dispatch plan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library; it is a plain, slow,
 * single-threaded restatement of the method, step by step, in the order the
 * pages give it:
 *
 *   "300 µs to level MoE expert load" (UltraEP page)
 *     - section "Getting the real load of the current layer after the Gate":
 *       the global load matrix of one microbatch and layer, solved identically
 *       on every rank;
 *     - section "Quota decides replicas and token split together": the quota
 *       solve (each step may create a replica or update the quota
 *       distribution), its constraints (S redundant slots per rank, no logical
 *       expert twice on one rank, a minimum quota of new replicas), and
 *       local-first rerouting followed by remote instances by remaining quota;
 *     - section "Shared redundant slots manage dynamic replicas": one native
 *       instance per logical expert plus zero or more replicas held in per-rank
 *       slots, reused across layers;
 *     - section "Reusing the forward plan": backward re-stages replica weights
 *       from the cached plan, reduces replica gradients into the native
 *       expert's gradient buffer and then clears the replica buffer.
 *   "Waterfill and LPLB" page, section "LPLB": the per-expert split over
 *     its physical instances, normalised to a probability distribution, from
 *     which every token routed to a replicated expert samples one instance
 *     (the sampling rerouting mode, in place of local-first rerouting);
 *   "Waterfill and LPLB" page, section "Waterfill": the waterline
 *     H = ceil((sum_r L_r + N) / R), slack S_r = max(H - L_r, 0), per-token
 *     sampling proportional to slack among the local rank and the ranks the
 *     token already visits, with a small local preference and a fallback to a
 *     clearly lighter candidate when no candidate has slack; section "Shared
 *     expert fusion": the shared expert is one more slot per rank.
 *
 * Every open point of the pages is fixed by a stated reading (tie-breaks,
 * the cap candidates, the order of tokens within an instance, the hash of the
 * Waterfill draw).  Integer work is exact (int64 here).  The only floating
 * point is the replica-gradient reduction, done in fp32 — the precision the
 * page's 72 MB fp32 gradient space per 36 MB bf16 weight slot fixes — one
 * add at a time in instance order.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_NO_MEM 2

/* stop reasons of one greedy run */
#define STOP_BALANCED 0
#define STOP_SLOT_LIMITED 1
#define STOP_QUOTA_LIMITED 2
#define STOP_ITER_CAP 3

/* status bits of a plan */
#define ST_BAD_ID 1
#define ST_ITER_CAP 2

typedef struct {
  int32_t R, E, K, T;     /* ranks, experts, top-k, tokens per rank */
  int32_t S, m;           /* redundant slots per rank, minimum replica quota */
  int32_t J;              /* number of cap candidates */
  int32_t shared_expert;  /* 1: one Waterfill shared-expert slot per token */
  int32_t bonus_permille; /* local preference of the Waterfill draw */
  int32_t all_ranks;      /* 1: Waterfill candidates are all ranks, not only visited ones */
  uint64_t seed;          /* Waterfill draw seed */
  int32_t sampling;       /* 1: every (token, k) samples an instance of its expert with
                             probability proportional to the instance's quota */
  int32_t iter_limit;     /* > 0: replaces the greedy's iteration bound (tests of the bound) */
  uint64_t sampling_seed; /* seed of the per-assignment draw of the sampling mode */
} orc_cfg;

typedef struct {
  int32_t Gmax, G;        /* natives per rank (max), columns per rank */
  int32_t cap_idx;        /* chosen cap candidate j */
  int32_t stop_reason;    /* of the chosen candidate */
  int64_t cap;            /* C_j of the chosen candidate */
  int64_t A;              /* counted (valid) assignments */
  int64_t before_max;     /* max_q W0[q] */
  int64_t after_max;      /* max_q W[q] */
  int32_t replicas;       /* replicas created */
  int32_t status;         /* ST_* bits */
  int64_t rows;           /* total dispatch rows (A, plus N with a shared expert) */
  int64_t realized_max;   /* max per-rank routed rows actually dispatched */
} orc_stats;

/* ---- O1: native placement, contiguous balanced blocks ------------------ */
static int32_t nat_count(int32_t q, int32_t E, int32_t R) {
  return E / R + (q < E % R ? 1 : 0);
}
static int32_t nat_first(int32_t q, int32_t E, int32_t R) {
  return q * (E / R) + (q < E % R ? q : E % R);
}
static int32_t home_rank(int32_t e, int32_t E, int32_t R) {
  /* the rank whose block [first, first+count) contains e, by walking */
  for (int32_t q = 0; q < R; ++q)
    if (e >= nat_first(q, E, R) && e < nat_first(q, E, R) + nat_count(q, E, R)) return q;
  return -1;
}

int32_t orc_gmax(int32_t E, int32_t R) { return E / R + (E % R ? 1 : 0); }

/* ---- O2: load matrix --------------------------------------------------- */
/* L[r][e] = number of (t,k) on source rank r with id e; ids outside [0,E)
 * are not counted and reported. */
int64_t orc_load_matrix(int32_t R, int32_t E, int32_t K, int32_t T, const int32_t* ids,
                        int64_t* L) {
  int64_t bad = 0;
  memset(L, 0, sizeof(int64_t) * (size_t)R * E);
  for (int32_t r = 0; r < R; ++r)
    for (int64_t a = 0; a < (int64_t)T * K; ++a) {
      int32_t e = ids[(int64_t)r * T * K + a];
      if (e < 0 || e >= E) { ++bad; continue; }
      L[(int64_t)r * E + e] += 1;
    }
  return bad;
}

/* ---- O10 helper: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) --------- */
/* One output of the generator whose state is x: advance the state by the
 * golden-gamma increment, then apply the variant-13 finaliser. */
uint64_t orc_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* ---- O10 helper: the Waterfill waterline -------------------------------- */
/* H = ceil((sum_r L_r + N) / R), slack S_r = max(H - L_r, 0) and the local
 * preference B = ceil(H * bonus / 1000). */
void orc_waterline(int32_t R, int64_t N, const int64_t* load, int32_t bonus_permille,
                   int64_t* H_out, int64_t* B_out, int64_t* slack) {
  int64_t sumL = 0;
  for (int32_t q = 0; q < R; ++q) sumL += load[q];
  const int64_t H = (sumL + N + R - 1) / R;
  for (int32_t q = 0; q < R; ++q) slack[q] = H - load[q] > 0 ? H - load[q] : 0;
  *H_out = H;
  *B_out = (H * bonus_permille + 999) / 1000;
}

/* Shared-slot rank of one token: cand[0] is the token's own rank, cand[1..nc)
 * the other ranks it already visits, ascending.  Draw proportional to slack
 * (own rank + B) with the SplitMix64 output of seed + token index; with no
 * slack among the candidates, the least-loaded candidate unless the own rank
 * is within B of it (ties to the smallest rank). */
static int32_t waterfill_pick(const int32_t* cand, int32_t nc, const int64_t* load,
                              const int64_t* slack, int64_t B, uint64_t seed, int64_t token) {
  int64_t sumS = 0;
  for (int32_t u = 0; u < nc; ++u) sumS += slack[cand[u]];
  if (sumS > 0) {
    const uint64_t h = orc_splitmix64(seed + (uint64_t)token);
    const uint64_t u64 = ((h >> 32) * (uint64_t)(sumS + B)) >> 32;
    int64_t acc = 0;
    for (int32_t u = 0; u < nc; ++u) {
      acc += slack[cand[u]] + (u == 0 ? B : 0);
      if ((uint64_t)acc > u64) return cand[u];
    }
    return cand[nc - 1]; /* unreachable: u64 < sumS + B */
  }
  int32_t lo = cand[0];
  for (int32_t u = 1; u < nc; ++u)
    if (load[cand[u]] < load[lo] || (load[cand[u]] == load[lo] && cand[u] < lo)) lo = cand[u];
  return (load[cand[0]] <= load[lo] + B) ? cand[0] : lo;
}

/* candidate list of a token: own rank, then the distinct other ranks it
 * visits ascending — or, in all-rank mode, every other rank ascending */
static int32_t waterfill_candidates(int32_t r, const int32_t* ranks, int32_t K, int32_t R,
                                    int32_t all_ranks, int32_t* cand) {
  int32_t nc = 0;
  cand[nc++] = r;
  if (all_ranks) {
    for (int32_t q = 0; q < R; ++q)
      if (q != r) cand[nc++] = q;
    return nc;
  }
  for (int32_t k = 0; k < K; ++k) {
    const int32_t q = ranks[k];
    if (q < 0 || q >= R) continue;
    int dup = 0;
    for (int32_t u = 0; u < nc; ++u) dup |= (cand[u] == q);
    if (!dup) cand[nc++] = q;
  }
  for (int32_t u = 2; u < nc; ++u) {
    int32_t v = cand[u], w = u - 1;
    while (w >= 1 && cand[w] > v) { cand[w + 1] = cand[w]; --w; }
    cand[w + 1] = v;
  }
  return nc;
}

/* ---- O4: one greedy run at cap C --------------------------------------- */
typedef struct {
  int64_t* W;      /* [R] per-rank load */
  int64_t* Qn;     /* [E] native quota */
  int32_t* slot_e; /* [R][S] expert in slot, -1 if empty */
  int64_t* slot_q; /* [R][S] quota of the replica in the slot */
  int32_t* used;   /* [R] filled slots */
  int32_t replicas;
  int32_t stop;
  int64_t maxW;
} greedy_state;

static int holds(const orc_cfg* c, const greedy_state* g, int32_t e, int32_t r) {
  if (home_rank(e, c->E, c->R) == r) return 1;
  for (int32_t s = 0; s < g->used[r]; ++s)
    if (g->slot_e[(int64_t)r * c->S + s] == e) return 1;
  return 0;
}

static void greedy(const orc_cfg* c, const int64_t* Tot, const int64_t* W0, int64_t C,
                   greedy_state* g, char* stuck, char* slotlim, int32_t* order) {
  const int32_t R = c->R, E = c->E, S = c->S;
  const int64_t m = c->m;
  for (int32_t q = 0; q < R; ++q) { g->W[q] = W0[q]; g->used[q] = 0; stuck[q] = 0; slotlim[q] = 0; }
  for (int32_t e = 0; e < E; ++e) g->Qn[e] = Tot[e];
  for (int64_t i = 0; i < (int64_t)R * S; ++i) { g->slot_e[i] = -1; g->slot_q[i] = 0; }
  g->replicas = 0;
  g->stop = -1;
  const int64_t iter_cap = c->iter_limit > 0 ? c->iter_limit : 4 * ((int64_t)R * S + R + E) + 64;
  for (int64_t it = 0;; ++it) {
    if (it >= iter_cap) { g->stop = STOP_ITER_CAP; break; }
    /* 1. most loaded rank that is not stuck, smallest index on ties */
    int32_t p = -1;
    for (int32_t q = 0; q < R; ++q)
      if (!stuck[q] && (p < 0 || g->W[q] > g->W[p])) p = q;
    if (p < 0 || g->W[p] <= C) break;
    const int64_t ex = g->W[p] - C;
    /* 2. natives of p by (quota descending, expert ascending) */
    const int32_t f = nat_first(p, E, R), n = nat_count(p, E, R);
    for (int32_t i = 0; i < n; ++i) order[i] = f + i;
    for (int32_t i = 1; i < n; ++i) { /* insertion sort */
      int32_t v = order[i], j = i - 1;
      while (j >= 0 && (g->Qn[order[j]] < g->Qn[v] ||
                        (g->Qn[order[j]] == g->Qn[v] && order[j] > v))) {
        order[j + 1] = order[j];
        --j;
      }
      order[j + 1] = v;
    }
    int moved = 0;
    for (int32_t i = 0; i < n && !moved; ++i) {
      const int32_t e = order[i];
      if (g->Qn[e] <= 0) continue;
      /* a new replica on the rank with the largest slack among those with a
       * free slot, no instance of e and slack >= m (smallest rank on ties).
       * Adding to an existing replica never arises: a replica is created
       * either filling its receiver to C, ending the donor's excess, or
       * exhausting the native quota, and only the native's rank donates e. */
      int32_t best = -1;
      for (int32_t r = 0; r < R; ++r) {
        if (g->used[r] >= S || holds(c, g, e, r) || C - g->W[r] < m) continue;
        if (best < 0 || C - g->W[best] < C - g->W[r]) best = r;
      }
      if (best >= 0) {
        int64_t x = ex > m ? ex : m;
        if (C - g->W[best] < x) x = C - g->W[best];
        if (g->Qn[e] < x) x = g->Qn[e];
        if (x >= m) {
          const int64_t s = (int64_t)best * S + g->used[best];
          g->slot_e[s] = e;
          g->slot_q[s] = x;
          g->used[best] += 1;
          g->replicas += 1;
          g->W[p] -= x;
          g->W[best] += x;
          g->Qn[e] -= x;
          moved = 1;
        }
      }
    }
    if (!moved) {
      /* 3. p cannot give anything away any more */
      stuck[p] = 1;
      int full_receiver = 0, native_big = 0;
      for (int32_t r = 0; r < R; ++r)
        if (g->used[r] == S && C - g->W[r] >= m) full_receiver = 1;
      for (int32_t i = 0; i < n; ++i)
        if (g->Qn[f + i] >= m) native_big = 1;
      slotlim[p] = (char)(full_receiver && native_big);
    }
  }
  g->maxW = 0;
  for (int32_t q = 0; q < R; ++q)
    if (g->W[q] > g->maxW) g->maxW = g->W[q];
  if (g->stop != STOP_ITER_CAP) {
    if (g->maxW <= C) {
      g->stop = STOP_BALANCED;
    } else {
      g->stop = STOP_QUOTA_LIMITED;
      for (int32_t q = 0; q < R; ++q)
        if (stuck[q] && g->W[q] > C && slotlim[q]) g->stop = STOP_SLOT_LIMITED;
    }
  }
}

/* ---- the whole plan ---------------------------------------------------- */
/*
 * Outputs (caller-allocated):
 *   L        [R][E]            load matrix (O2)
 *   Tot      [E]               per-expert totals
 *   W0, W    [R]               per-rank load before / after the solve (O3, O4)
 *   inst_expert [R][G] int32   instance table (O5); -1 empty, E = shared column
 *   inst_quota  [R][G]         quota of each instance (the solve's split)
 *   inst_count  [R][G]         rows each instance receives: its quota, except in the
 *                              sampling mode, where it is the number of draws it got
 *   inst_off    [R*G+1]        exclusive prefix of inst_count, in instance order (O8)
 *   dst_inst    [R][T][K]      global instance index of each assignment, -1 if invalid
 *   dst_row     [R][T][K]      dispatch row of each assignment (O7, O8), -1 if invalid
 *   shared_rank [R][T]         Waterfill rank of each token's shared slot (O10), or NULL
 *   shared_row  [R][T]         dispatch row of the shared slot, or NULL
 *   cand_maxW, cand_repl, cand_stop [J]   each cap candidate's result
 */
int orc_plan(const orc_cfg* c, const int32_t* ids, int64_t* L, int64_t* Tot, int64_t* W0,
             int64_t* W, int32_t* inst_expert, int64_t* inst_quota, int64_t* inst_count,
             int64_t* inst_off, int32_t* dst_inst, int64_t* dst_row, int32_t* shared_rank,
             int64_t* shared_row, int64_t* cand_maxW, int32_t* cand_repl, int32_t* cand_stop,
             orc_stats* st) {
  const int32_t R = c->R, E = c->E, K = c->K, T = c->T, S = c->S;
  if (R < 1 || E < 1 || K < 1 || T < 0 || S < 0 || c->m < 1 || c->J < 1) return ORC_BAD_ARG;
  const int32_t Gmax = orc_gmax(E, R);
  const int32_t sh = c->shared_expert ? 1 : 0;
  const int32_t G = Gmax + S + sh;
  memset(st, 0, sizeof(*st));
  st->Gmax = Gmax;
  st->G = G;

  /* O2, O3 */
  const int64_t bad = orc_load_matrix(R, E, K, T, ids, L);
  if (bad) st->status |= ST_BAD_ID;
  int64_t A = 0;
  for (int32_t e = 0; e < E; ++e) {
    Tot[e] = 0;
    for (int32_t r = 0; r < R; ++r) Tot[e] += L[(int64_t)r * E + e];
    A += Tot[e];
  }
  st->A = A;
  for (int32_t q = 0; q < R; ++q) {
    W0[q] = 0;
    for (int32_t i = 0; i < nat_count(q, E, R); ++i) W0[q] += Tot[nat_first(q, E, R) + i];
    if (W0[q] > st->before_max) st->before_max = W0[q];
  }

  /* O4: greedy at each cap candidate, keep the lexicographically smallest
   * (max load, replicas, candidate index). */
  greedy_state g, best;
  char* stuck = (char*)malloc((size_t)R);
  char* slotlim = (char*)malloc((size_t)R);
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(Gmax + 1));
  greedy_state* gs[2] = {&g, &best};
  for (int k = 0; k < 2; ++k) {
    gs[k]->W = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    gs[k]->Qn = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    gs[k]->slot_e = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R * S + 1));
    gs[k]->slot_q = (int64_t*)malloc(sizeof(int64_t) * (size_t)(R * S + 1));
    gs[k]->used = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
  }
  int32_t best_j = -1;
  int64_t best_C = 0;
  for (int32_t j = 0; j < c->J; ++j) {
    /* C_j = ceil(A * (200 + j) / (200 R)): caps from the mean upward in 0.5 % steps */
    const int64_t num = A * (200 + j), den = 200 * (int64_t)R;
    const int64_t C = (num + den - 1) / den;
    greedy(c, Tot, W0, C, &g, stuck, slotlim, order);
    cand_maxW[j] = g.maxW;
    cand_repl[j] = g.replicas;
    cand_stop[j] = g.stop;
    if (g.stop == STOP_ITER_CAP) st->status |= ST_ITER_CAP;
    if (best_j < 0 || g.maxW < best.maxW || (g.maxW == best.maxW && g.replicas < best.replicas)) {
      greedy_state tmp = best;
      best = g;
      g = tmp;
      best_j = j;
      best_C = C;
    }
  }
  st->cap_idx = best_j;
  st->cap = best_C;
  st->stop_reason = best.stop;
  st->replicas = best.replicas;
  st->after_max = best.maxW;
  for (int32_t q = 0; q < R; ++q) W[q] = best.W[q];

  /* O5: instance table */
  for (int32_t q = 0; q < R; ++q) {
    for (int32_t col = 0; col < G; ++col) {
      inst_expert[(int64_t)q * G + col] = -1;
      inst_quota[(int64_t)q * G + col] = 0;
    }
    for (int32_t i = 0; i < nat_count(q, E, R); ++i) {
      const int32_t e = nat_first(q, E, R) + i;
      inst_expert[(int64_t)q * G + i] = e;
      inst_quota[(int64_t)q * G + i] = best.Qn[e];
    }
    for (int32_t s = 0; s < best.used[q]; ++s) {
      inst_expert[(int64_t)q * G + Gmax + s] = best.slot_e[(int64_t)q * S + s];
      inst_quota[(int64_t)q * G + Gmax + s] = best.slot_q[(int64_t)q * S + s];
    }
    if (sh) inst_expert[(int64_t)q * G + Gmax + S] = E;
  }

  /* O6: local-first take, then remote fill in instance order.
   * flow[r][i] for the instances of one expert at a time (dense [R][R]),
   * pos_start[r][i] = rows of instance i that precede source r. */
  int32_t* inst_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)R); /* instance of e on rank, or -1 */
  int64_t* flow = (int64_t*)malloc(sizeof(int64_t) * (size_t)R * R);
  int64_t* Qp = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
  int64_t* D = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
  /* per (r, e): the ordered list of (instance, count, first row within instance) */
  /* per expert at most R local segments and 2R-1 remote overlaps */
  int64_t seg_cap = 3 * (int64_t)R * E + 1;
  int32_t* seg_inst = (int32_t*)malloc(sizeof(int32_t) * (size_t)seg_cap);
  int64_t* seg_cnt = (int64_t*)malloc(sizeof(int64_t) * (size_t)seg_cap);
  int64_t* seg_pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)seg_cap);
  /* segments are appended per expert, then indexed per (r, e) */
  int64_t* tmp_ptr = (int64_t*)malloc(sizeof(int64_t) * (size_t)R * E);
  int64_t nseg = 0;
  for (int32_t e = 0; e < E; ++e) {
    for (int32_t r = 0; r < R; ++r) inst_of[r] = -1;
    for (int32_t q = 0; q < R; ++q)
      for (int32_t col = 0; col < Gmax + S; ++col)
        if (inst_expert[(int64_t)q * G + col] == e) inst_of[q] = q * G + col;
    for (int32_t r = 0; r < R; ++r) {
      const int64_t l = L[(int64_t)r * E + e];
      const int32_t i = inst_of[r];
      const int64_t loc = (i >= 0) ? (l < inst_quota[i] ? l : inst_quota[i]) : 0;
      D[r] = l - loc;
      Qp[r] = (i >= 0) ? inst_quota[i] - loc : 0;
      for (int32_t q = 0; q < R; ++q) flow[(int64_t)r * R + q] = 0;
      if (i >= 0) flow[(int64_t)r * R + r] = loc;
    }
    /* two-pointer merge of demands (ascending source rank) and residual quotas
     * (ascending instance index = ascending rank) */
    {
      int32_t r = 0, q = 0;
      int64_t dleft = R > 0 ? D[0] : 0, qleft = R > 0 ? Qp[0] : 0;
      while (r < R && q < R) {
        if (dleft == 0) { ++r; if (r < R) dleft = D[r]; continue; }
        if (qleft == 0) { ++q; if (q < R) qleft = Qp[q]; continue; }
        const int64_t x = dleft < qleft ? dleft : qleft;
        flow[(int64_t)r * R + q] += x; /* r != q here: a source with residual
                                          demand has no residual local quota */
        dleft -= x;
        qleft -= x;
      }
    }
    /* segments of each source r: local first, then remote in instance order;
     * position of r within instance q: flows of sources r' < r into q */
    for (int32_t r = 0; r < R; ++r) {
      tmp_ptr[(int64_t)r * E + e] = nseg;
      /* local */
      if (inst_of[r] >= 0 && flow[(int64_t)r * R + r] > 0) {
        int64_t pos = 0;
        for (int32_t r2 = 0; r2 < r; ++r2) pos += flow[(int64_t)r2 * R + r];
        seg_inst[nseg] = inst_of[r];
        seg_cnt[nseg] = flow[(int64_t)r * R + r];
        seg_pos[nseg] = pos;
        ++nseg;
      }
      for (int32_t q = 0; q < R; ++q) {
        if (q == r || flow[(int64_t)r * R + q] == 0) continue;
        int64_t pos = 0;
        for (int32_t r2 = 0; r2 < r; ++r2) pos += flow[(int64_t)r2 * R + q];
        seg_inst[nseg] = inst_of[q];
        seg_cnt[nseg] = flow[(int64_t)r * R + q];
        seg_pos[nseg] = pos;
        ++nseg;
      }
    }
  }

  /* O7: materialise onto tokens, ascending (t, k) per (source, expert) */
  int64_t* cur_seg = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  int64_t* cur_used = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  int64_t* dst_pos = (int64_t*)malloc(sizeof(int64_t) * ((size_t)R * T * K + 1));
  if (!c->sampling) {
    for (int32_t r = 0; r < R; ++r) {
      for (int32_t e = 0; e < E; ++e) { cur_seg[e] = tmp_ptr[(int64_t)r * E + e]; cur_used[e] = 0; }
      for (int64_t a = 0; a < (int64_t)T * K; ++a) {
        const int64_t idx = (int64_t)r * T * K + a;
        const int32_t e = ids[idx];
        if (e < 0 || e >= E) { dst_inst[idx] = -1; dst_pos[idx] = -1; continue; }
        while (cur_used[e] == seg_cnt[cur_seg[e]]) { ++cur_seg[e]; cur_used[e] = 0; }
        dst_inst[idx] = seg_inst[cur_seg[e]];
        dst_pos[idx] = seg_pos[cur_seg[e]] + cur_used[e];
        ++cur_used[e];
      }
    }
  }

  /* Sampling mode ("Waterfill and LPLB" page, section "LPLB"): the solve's
   * split of each expert over its instances, divided by the expert's total, is
   * a probability distribution over the instances; every (token, k) draws one
   * instance from it independently, and an expert with a single instance maps
   * to it without a draw.  The draw is made reproducible with a counter-based
   * hash of the assignment index a = (r*T + t)*K + k:
   * h = SplitMix64(sampling_seed + a), u = ((h >> 32) * total) >> 32, and the
   * pick is the first instance, in instance order, whose running quota sum
   * exceeds u.  Rows of an instance keep the order (source rank, t, k). */
  int64_t* run = (int64_t*)calloc((size_t)R * G, sizeof(int64_t));
  if (c->sampling) {
    /* instances of each expert in instance order (natives and replicas) */
    int64_t* eptr = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
    int32_t* elist = (int32_t*)malloc(sizeof(int32_t) * ((size_t)R * G + 1));
    for (int64_t i = 0; i < (int64_t)R * G; ++i) {
      const int32_t e = inst_expert[i];
      if (e >= 0 && e < E) eptr[e + 1] += 1;
    }
    for (int32_t e = 0; e < E; ++e) eptr[e + 1] += eptr[e];
    int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * ((size_t)E + 1));
    for (int32_t e = 0; e <= E; ++e) fill[e] = eptr[e];
    for (int64_t i = 0; i < (int64_t)R * G; ++i) {
      const int32_t e = inst_expert[i];
      if (e >= 0 && e < E) elist[fill[e]++] = (int32_t)i;
    }
    for (int64_t idx = 0; idx < (int64_t)R * T * K; ++idx) {
      const int32_t e = ids[idx];
      if (e < 0 || e >= E) { dst_inst[idx] = -1; dst_pos[idx] = -1; continue; }
      const int64_t n = eptr[e + 1] - eptr[e];
      int32_t pick = elist[eptr[e]];
      if (n > 1) {
        const uint64_t h = orc_splitmix64(c->sampling_seed + (uint64_t)idx);
        const uint64_t u = ((h >> 32) * (uint64_t)Tot[e]) >> 32;
        int64_t acc = 0;
        for (int64_t j = 0; j < n; ++j) {
          acc += inst_quota[elist[eptr[e] + j]];
          if ((uint64_t)acc > u) { pick = elist[eptr[e] + j]; break; }
        }
      }
      dst_inst[idx] = pick;
      dst_pos[idx] = run[pick]++; /* assignments are visited in (r, t, k) order */
    }
    free(eptr);
    free(elist);
    free(fill);
  }

  /* O10: Waterfill shared-expert slot of each token.  The load score of a
   * rank is its routed load W after the solve; in the sampling mode that is
   * the planned (expected) load, the realised one being known only after every
   * draw. */
  int64_t* shared_cnt = (int64_t*)calloc((size_t)R, sizeof(int64_t));
  if (sh) {
    int64_t H, B;
    int64_t* slack = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    orc_waterline(R, (int64_t)R * T, W, c->bonus_permille, &H, &B, slack);
    int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K + R + 1));
    int32_t* ranks = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
    for (int32_t r = 0; r < R; ++r)
      for (int32_t t = 0; t < T; ++t) {
        for (int32_t k = 0; k < K; ++k) {
          const int32_t i = dst_inst[((int64_t)r * T + t) * K + k];
          ranks[k] = i < 0 ? -1 : i / G;
        }
        const int32_t nc = waterfill_candidates(r, ranks, K, R, c->all_ranks, cand);
        const int32_t pick = waterfill_pick(cand, nc, W, slack, B, c->seed, (int64_t)r * T + t);
        shared_rank[(int64_t)r * T + t] = pick;
        shared_cnt[pick] += 1;
      }
    free(slack);
    free(cand);
    free(ranks);
    for (int32_t q = 0; q < R; ++q) inst_quota[(int64_t)q * G + Gmax + S] = shared_cnt[q];
  }

  /* rows each instance receives: the quota, or the draws it got */
  for (int64_t i = 0; i < (int64_t)R * G; ++i) {
    const int shared_col = sh && (i % G) == Gmax + S;
    inst_count[i] = (c->sampling && !shared_col) ? run[i] : inst_quota[i];
  }
  st->realized_max = 0;
  for (int32_t q = 0; q < R; ++q) {
    int64_t w = 0;
    for (int32_t col = 0; col < Gmax + S; ++col) w += inst_count[(int64_t)q * G + col];
    if (w > st->realized_max) st->realized_max = w;
  }

  /* O8: row layout */
  inst_off[0] = 0;
  for (int64_t i = 0; i < (int64_t)R * G; ++i) inst_off[i + 1] = inst_off[i] + inst_count[i];
  st->rows = inst_off[(int64_t)R * G];
  for (int64_t a = 0; a < (int64_t)R * T * K; ++a)
    dst_row[a] = dst_inst[a] < 0 ? -1 : inst_off[dst_inst[a]] + dst_pos[a];
  if (sh) {
    int64_t* run = (int64_t*)calloc((size_t)R, sizeof(int64_t));
    for (int32_t r = 0; r < R; ++r)
      for (int32_t t = 0; t < T; ++t) {
        const int32_t q = shared_rank[(int64_t)r * T + t];
        shared_row[(int64_t)r * T + t] = inst_off[(int64_t)q * G + Gmax + S] + run[q]++;
      }
    free(run);
  }

  free(shared_cnt);
  free(run);
  free(dst_pos);
  free(cur_seg);
  free(cur_used);
  free(tmp_ptr);
  free(seg_inst);
  free(seg_cnt);
  free(seg_pos);
  free(D);
  free(Qp);
  free(flow);
  free(inst_of);
  for (int k = 0; k < 2; ++k) {
    free(gs[k]->W);
    free(gs[k]->Qn);
    free(gs[k]->slot_e);
    free(gs[k]->slot_q);
    free(gs[k]->used);
  }
  free(stuck);
  free(slotlim);
  free(order);
  return ORC_OK;
}

/* ---- O3 + O4 alone: the quota solve from the per-expert totals ---------- */
/* The same greedy at the same cap candidates and the same selection as
 * orc_plan, without the load matrix, the rerouting or the layout: what a
 * solve-latency comparison with another replication rule times.  Writes the
 * chosen candidate's per-rank loads W[R]; returns its replica count (or -1). */
int32_t orc_quota_solve(int32_t R, int32_t E, int32_t S, int32_t m, int32_t J, const int64_t* Tot,
                        int64_t* W, int64_t* max_out) {
  if (R < 1 || E < 1 || S < 0 || m < 1 || J < 1) return -1;
  orc_cfg c;
  memset(&c, 0, sizeof c);
  c.R = R; c.E = E; c.S = S; c.m = m; c.J = J; c.K = 1;
  int64_t* W0 = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
  int64_t A = 0;
  for (int32_t e = 0; e < E; ++e) A += Tot[e];
  for (int32_t q = 0; q < R; ++q) {
    W0[q] = 0;
    for (int32_t i = 0; i < nat_count(q, E, R); ++i) W0[q] += Tot[nat_first(q, E, R) + i];
  }
  greedy_state g, best;
  char* stuck = (char*)malloc((size_t)R);
  char* slotlim = (char*)malloc((size_t)R);
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(orc_gmax(E, R) + 1));
  greedy_state* gs[2] = {&g, &best};
  for (int k = 0; k < 2; ++k) {
    gs[k]->W = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    gs[k]->Qn = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    gs[k]->slot_e = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R * S + 1));
    gs[k]->slot_q = (int64_t*)malloc(sizeof(int64_t) * (size_t)(R * S + 1));
    gs[k]->used = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
  }
  int32_t best_j = -1;
  for (int32_t j = 0; j < J; ++j) {
    const int64_t num = A * (200 + j), den = 200 * (int64_t)R;
    greedy(&c, Tot, W0, (num + den - 1) / den, &g, stuck, slotlim, order);
    if (best_j < 0 || g.maxW < best.maxW || (g.maxW == best.maxW && g.replicas < best.replicas)) {
      greedy_state tmp = best;
      best = g;
      g = tmp;
      best_j = j;
    }
  }
  for (int32_t q = 0; q < R; ++q) W[q] = best.W[q];
  *max_out = best.maxW;
  const int32_t replicas = best.replicas;
  for (int k = 0; k < 2; ++k) {
    free(gs[k]->W);
    free(gs[k]->Qn);
    free(gs[k]->slot_e);
    free(gs[k]->slot_q);
    free(gs[k]->used);
  }
  free(W0);
  free(stuck);
  free(slotlim);
  free(order);
  return replicas;
}

/* ---- O10 standalone: Waterfill for given per-rank loads and routes ------ */
/* load[R]: routed load per rank; dst_rank[R][T][K]: destination rank of each
 * routed assignment (-1 = none).  Writes pick[R][T] and count[R]. */
int orc_waterfill(int32_t R, int32_t T, int32_t K, const int64_t* load, const int32_t* dst_rank,
                  uint64_t seed, int32_t bonus_permille, int32_t all_ranks, int32_t* pick_out,
                  int64_t* count) {
  int64_t H, B;
  int64_t* slack = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
  int32_t* cand = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K + R + 1));
  orc_waterline(R, (int64_t)R * T, load, bonus_permille, &H, &B, slack);
  for (int32_t q = 0; q < R; ++q) count[q] = 0;
  for (int32_t r = 0; r < R; ++r)
    for (int32_t t = 0; t < T; ++t) {
      const int32_t nc =
          waterfill_candidates(r, dst_rank + ((int64_t)r * T + t) * K, K, R, all_ranks, cand);
      const int32_t pick = waterfill_pick(cand, nc, load, slack, B, seed, (int64_t)r * T + t);
      pick_out[(int64_t)r * T + t] = pick;
      count[pick] += 1;
    }
  free(slack);
  free(cand);
  return ORC_OK;
}

/* ---- O9: permute (bit copy of whole rows) ------------------------------ */
void orc_permute(int64_t N, int32_t K, int64_t row_bytes, const uint8_t* hidden,
                 const int64_t* dst_row, const int64_t* shared_row, uint8_t* out) {
  for (int64_t n = 0; n < N; ++n) {
    for (int32_t k = 0; k < K; ++k) {
      const int64_t d = dst_row[n * K + k];
      if (d >= 0) memcpy(out + d * row_bytes, hidden + n * row_bytes, (size_t)row_bytes);
    }
    if (shared_row) memcpy(out + shared_row[n] * row_bytes, hidden + n * row_bytes, (size_t)row_bytes);
  }
}

/* ---- EPLB+ comparison baseline ------------------------------------------ */
/* UltraEP page, section "Quota decides replicas and token split together":
 * EPLB+ uses the same exact per-layer loads but EPLB-style replication and
 * round-robin rerouting.  Reading (the page does not spell EPLB out): every
 * redundant slot is filled, one at a time, with a replica of the expert whose
 * load per instance T[e]/n[e] is largest (smallest e on ties) among experts
 * that still fit somewhere, placed on the rank with the smallest estimated
 * load sum_i T[e_i]/n[e_i] that has a free slot and no instance of the expert
 * (smallest rank on ties); then each expert's tokens are split round robin
 * over its instances in instance order (the first T[e] mod n instances get one
 * more).  Writes the instance table like orc_plan and W[R]; returns the number
 * of replicas placed. */
int32_t orc_eplb_plus(int32_t R, int32_t E, int32_t S, const int64_t* Tot, int32_t* inst_expert,
                      int64_t* inst_quota, int64_t* W) {
  const int32_t Gmax = orc_gmax(E, R), G = Gmax + S;
  int32_t* n = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int32_t* used = (int32_t*)calloc((size_t)R, sizeof(int32_t));
  double* est = (double*)calloc((size_t)R, sizeof(double));
  for (int32_t e = 0; e < E; ++e) n[e] = 1;
  for (int32_t q = 0; q < R; ++q)
    for (int32_t col = 0; col < G; ++col) {
      inst_expert[(int64_t)q * G + col] = -1;
      inst_quota[(int64_t)q * G + col] = 0;
    }
  for (int32_t q = 0; q < R; ++q)
    for (int32_t i = 0; i < nat_count(q, E, R); ++i)
      inst_expert[(int64_t)q * G + i] = nat_first(q, E, R) + i;
  int32_t placed = 0;
  for (int32_t round = 0; round < R * S; ++round) {
    /* estimated load of each rank with the current instance counts */
    for (int32_t q = 0; q < R; ++q) {
      est[q] = 0.0;
      for (int32_t col = 0; col < G; ++col) {
        const int32_t e = inst_expert[(int64_t)q * G + col];
        if (e >= 0) est[q] += (double)Tot[e] / n[e];
      }
    }
    int32_t best_e = -1, best_r = -1;
    for (int32_t e = 0; e < E; ++e) {
      /* candidate only if some rank has a free slot and no instance of e */
      int32_t r_for_e = -1;
      for (int32_t q = 0; q < R; ++q) {
        if (used[q] >= S) continue;
        int holds_e = 0;
        for (int32_t col = 0; col < G; ++col) holds_e |= inst_expert[(int64_t)q * G + col] == e;
        if (holds_e) continue;
        if (r_for_e < 0 || est[q] < est[r_for_e]) r_for_e = q;
      }
      if (r_for_e < 0) continue;
      /* largest T[e]/n[e]: compare T[e]*n[b] > T[b]*n[e] exactly */
      if (best_e < 0 || Tot[e] * n[best_e] > Tot[best_e] * n[e]) {
        best_e = e;
        best_r = r_for_e;
      }
    }
    if (best_e < 0) break;
    inst_expert[(int64_t)best_r * G + Gmax + used[best_r]] = best_e;
    used[best_r] += 1;
    n[best_e] += 1;
    ++placed;
  }
  /* round robin over the instances of each expert, in instance order */
  int32_t* seen = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int32_t q = 0; q < R; ++q) W[q] = 0;
  for (int64_t i = 0; i < (int64_t)R * G; ++i) {
    const int32_t e = inst_expert[i];
    if (e < 0) continue;
    const int64_t quota = Tot[e] / n[e] + (seen[e] < Tot[e] % n[e] ? 1 : 0);
    seen[e] += 1;
    inst_quota[i] = quota;
    W[i / G] += quota;
  }
  free(seen);
  free(n);
  free(used);
  free(est);
  return placed;
}

/* ---- combine (reverse of the dispatch, with gate weights) -------------- */
/* After expert compute each dispatch row holds its expert's output for one
 * (token, k) (or the shared expert's output for the token).  The token's
 * output is the gate-weighted sum of its routed rows plus its shared-expert
 * row with weight 1 (the shared expert is not gated), computed here exactly
 * enough in fp64: out[n][h] = sum_k w[n][k] * x[dst_row[n][k]][h]
 * (+ x[shared_row[n]][h]); rows of -1 (dropped ids) contribute nothing. */
static double bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

void orc_combine(int64_t N, int32_t K, int32_t H, const uint16_t* x, const int64_t* dst_row,
                 const float* w, const int64_t* shared_row, double* out) {
  for (int64_t n = 0; n < N; ++n)
    for (int32_t h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int32_t k = 0; k < K; ++k) {
        const int64_t d = dst_row[n * K + k];
        if (d >= 0) acc += (double)w[n * K + k] * bf16_to_f64(x[d * H + h]);
      }
      if (shared_row) acc += bf16_to_f64(x[shared_row[n] * H + h]);
      out[n * H + h] = acc;
    }
}

/* ---- O11: stage replica weights (bit copy) ----------------------------- */
void orc_stage(int32_t R, int32_t S, int32_t G, int32_t Gmax, const int32_t* inst_expert,
               int64_t elem_bytes, const uint8_t* native_w, uint8_t* slots) {
  for (int32_t q = 0; q < R; ++q)
    for (int32_t s = 0; s < S; ++s) {
      const int32_t e = inst_expert[(int64_t)q * G + Gmax + s];
      if (e >= 0)
        memcpy(slots + ((int64_t)q * S + s) * elem_bytes, native_w + (int64_t)e * elem_bytes,
               (size_t)elem_bytes);
    }
}

/* ---- O12: reduce replica gradients into the native fp32 buffer --------- */
static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* grad_is_f32 = 0: slot gradients are bf16 (uint16 bits); 1: fp32. */
void orc_reduce_grads(int32_t R, int32_t S, int32_t G, int32_t Gmax, const int32_t* inst_expert,
                      int64_t elems, int32_t grad_is_f32, void* slot_grads, float* native_grads) {
  for (int32_t q = 0; q < R; ++q) /* instance order = (rank, slot) ascending */
    for (int32_t s = 0; s < S; ++s) {
      const int32_t e = inst_expert[(int64_t)q * G + Gmax + s];
      if (e < 0) continue;
      float* acc = native_grads + (int64_t)e * elems;
      const int64_t base = ((int64_t)q * S + s) * elems;
      for (int64_t j = 0; j < elems; ++j) {
        const float v = grad_is_f32 ? ((float*)slot_grads)[base + j]
                                    : bf16_to_f32(((uint16_t*)slot_grads)[base + j]);
        acc[j] = acc[j] + v;
      }
      if (grad_is_f32)
        memset((float*)slot_grads + base, 0, sizeof(float) * (size_t)elems);
      else
        memset((uint16_t*)slot_grads + base, 0, sizeof(uint16_t) * (size_t)elems);
    }
}
