// Host side of the C ABI declared in include/ep_balance.h: configuration
// checks, the workspace layout (per-layer plan cache + shared scratch), and the
// entry points, each of which only validates arguments and enqueues kernels.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "ep_internal.cuh"

namespace ep {
cudaError_t set_plan_attributes(int max_smem);
cudaError_t plan_launch_shapes(Dims& d, int max_smem, int sms);
cudaError_t set_copy_attributes(int max_smem);
}  // namespace ep

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Byte offsets of every array, relative to the workspace base.
struct Layout {
  // per layer (offset inside one layer block)
  size_t load, expert_total, W0, W, inst_expert, inst_quota, inst_off, rank_base, dst_row,
      shared_rank, shared_row, cand, rep_list, rep_eptr, rep_nexp, rep_experts, inst_count, stats;
  size_t layer_bytes;
  // scratch (absolute)
  size_t sub_cnt, blk_cnt, wsub_cnt, seg_rec, seg_ord, seg_rank, seg_base, inst_rel, slack, wf, sbase,
      shared_tot, asg_rank, smp_cum, smp_inst, smp_key, smp_sub, smp_blk, smp_row0, rank_rows,
      prev_base,
      acc_load, acc_misc, smp_tot;
  size_t acc_end;  // end of the accumulators zeroed before a plan's first balance call
  size_t scratch_bytes;
  size_t total;
};

struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = align_up(off + (bytes ? bytes : 1));
    return o;
  }
};

ep_status_t make_dims(const ep_config* c, ep::Dims* d) {
  if (!c) return EP_ERR_INVALID_ARGUMENT;
  const int R = c->num_ranks, E = c->num_experts, K = c->top_k, T = c->tokens_per_rank;
  if (R < 1 || E < 1 || K < 1 || T < 0 || c->slots_per_rank < 0 || c->min_replica_quota < 1 ||
      c->num_layers < 1 || c->num_cap_candidates < 1 || c->hidden < 1 ||
      c->expert_weight_elems < 0 || c->waterfill_bonus_permille < 0 ||
      (c->shared_expert != 0 && c->shared_expert != 1) ||
      (c->waterfill_all_ranks != 0 && c->waterfill_all_ranks != 1) ||
      (c->rerouting_mode != EP_REROUTE_LOCAL_FIRST && c->rerouting_mode != EP_REROUTE_SAMPLED) ||
      c->solver_iter_limit < 0)
    return EP_ERR_INVALID_ARGUMENT;
  const int Gmax = E / R + (E % R ? 1 : 0);
  if (R > ep::kMaxR || E > ep::kMaxE || Gmax > ep::kMaxNat || K > ep::kMaxK ||
      c->slots_per_rank > ep::kMaxS || c->num_cap_candidates > ep::kMaxJ ||
      c->waterfill_bonus_permille > 1000 || c->hidden < 8 || (c->hidden * 2) % 16 != 0 ||
      c->expert_weight_elems % 8 != 0)
    return EP_ERR_UNSUPPORTED;
  if ((int64_t)R * T * (K + 1) >= (int64_t)INT32_MAX) return EP_ERR_UNSUPPORTED;
  // the gradient reduction indexes (replica slot, 16-element pair) in 32 bits
  if ((int64_t)R * c->slots_per_rank * ((c->expert_weight_elems + 15) / 16) >= ((int64_t)1 << 32))
    return EP_ERR_UNSUPPORTED;
  // Waterfill draw weights stay below 2^32: (K + 2) * H with H <= ceil((A + N) / R) + 1
  const int64_t H = ((int64_t)T * (K + 1) * R + R - 1) / R + 1;
  if ((int64_t)(K + 2) * H >= ((int64_t)1 << 32)) return EP_ERR_UNSUPPORTED;
  d->R = R;
  d->E = E;
  d->K = K;
  d->T = T;
  d->S = c->slots_per_rank;
  d->m = c->min_replica_quota;
  d->J = c->num_cap_candidates;
  d->Gmax = Gmax;
  d->sh = c->shared_expert;
  d->G = Gmax + d->S + d->sh;
  d->nsub = (T + ep::kPlanSubT - 1) / ep::kPlanSubT;
  d->bonus = c->waterfill_bonus_permille;
  d->all_ranks = c->waterfill_all_ranks;
  d->hidden = c->hidden;
  d->seed = c->waterfill_seed;
  d->Wn = c->expert_weight_elems;
  d->sampled = c->rerouting_mode == EP_REROUTE_SAMPLED;
  d->iter_limit = c->solver_iter_limit;
  d->sseed = c->sampling_seed;
  d->nkey = E + R * d->S;  // at most 1024 + 128 * 8 keys: they fit the uint16 key buffer
  d->solve_smem = 0;       // set at plan creation, from the device's shared-memory limit
  d->fix_grid = 1;         // set at plan creation, from the device's SM count
  return EP_OK;
}

Layout make_layout(const ep::Dims& d, int num_layers) {
  Layout L{};
  const size_t i4 = sizeof(int32_t);
  Bump b;
  L.stats = b.take(sizeof(ep_layer_stats));
  L.load = b.take(i4 * d.R * d.E);
  L.expert_total = b.take(i4 * d.E);
  L.W0 = b.take(i4 * d.R);
  L.W = b.take(i4 * d.R);
  L.inst_expert = b.take(i4 * d.R * d.G);
  L.inst_quota = b.take(i4 * d.R * d.G);
  L.inst_off = b.take(i4 * ((size_t)d.R * d.G + 1));
  L.rank_base = b.take(i4 * (d.R + 1));
  L.dst_row = b.take(i4 * (size_t)d.R * d.T * d.K);
  L.shared_rank = b.take(d.sh ? i4 * (size_t)d.R * d.T : 0);
  L.shared_row = b.take(d.sh ? i4 * (size_t)d.R * d.T : 0);
  L.cand = b.take(i4 * 3 * d.J);
  L.rep_list = b.take(i4 * ((size_t)d.R * d.S + 1));
  L.rep_eptr = b.take(i4 * (d.E + 1));
  L.rep_nexp = b.take(i4);
  L.rep_experts = b.take(i4 * ((size_t)d.R * d.S + 1));
  L.inst_count = b.take(d.sampled ? i4 * d.R * d.G : 0);
  L.layer_bytes = b.off;
  Bump s;
  s.off = L.layer_bytes * (size_t)num_layers;
  L.sub_cnt = s.take(i4 * (size_t)d.R * d.nsub * d.E);
  L.blk_cnt = s.take(i4 * (size_t)d.R * ((d.nsub + ep::kPlanWarps - 1) / ep::kPlanWarps) * d.E);
  L.wsub_cnt = s.take(d.sh ? i4 * (size_t)d.R * d.R * d.nsub : 0);
  L.seg_rec = s.take(i4 * 8 * (size_t)d.R * d.E);
  L.seg_ord = s.take(i4 * (size_t)d.E * 3 * d.R);
  L.seg_rank = s.take(i4 * (size_t)d.E * 3 * d.R);
  L.seg_base = s.take(i4 * (size_t)d.E * 3 * d.R);
  L.inst_rel = s.take(i4 * (size_t)d.R * d.G);
  L.slack = s.take(i4 * d.R);
  L.wf = s.take(i4 * 2);
  L.sbase = s.take(i4 * d.R);
  L.shared_tot = s.take(i4 * d.R);
  L.asg_rank = s.take(d.sh ? (size_t)d.R * d.T * d.K : 0);
  const size_t nblk = (d.nsub + ep::kPlanWarps - 1) / ep::kPlanWarps;
  const size_t nk = d.sampled ? (size_t)d.nkey : 0;
  L.smp_cum = s.take(i4 * nk);
  L.smp_inst = s.take(i4 * nk);
  L.smp_key = s.take(d.sampled ? sizeof(uint16_t) * (size_t)d.R * d.T * d.K : 0);
  L.smp_sub = s.take(i4 * (size_t)d.R * d.nsub * nk);
  L.smp_blk = s.take(i4 * (size_t)d.R * nblk * nk);
  L.smp_row0 = s.take(i4 * (size_t)d.R * nk);
  L.rank_rows = s.take(i4 * d.R);
  L.prev_base = s.take(i4 * (d.R + 1));
  // contiguous: zeroed together once, before the plan's first balance call
  L.acc_load = s.take(i4 * (size_t)d.R * d.E);
  L.acc_misc = s.take(i4 * 4);
  L.smp_tot = s.take(i4 * (size_t)d.R * nk);
  L.acc_end = s.off;
  L.total = s.off;
  L.scratch_bytes = s.off - L.layer_bytes * (size_t)num_layers;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct ep_plan {
  ep_config cfg;
  ep::Dims d;
  Layout lay;
  char* ws;
  size_t ws_bytes;
  int device;
  int num_sms;
  int dispatch_bulk;       // EP_DISPATCH_IMPL=bulk: the bulk-copy (TMA) dispatch variant
  unsigned char* planned;  // per layer: balanced at least once
  bool acc_zero;           // the scratch accumulators are known to be zero
};

namespace {

int32_t* at(const ep_plan* p, size_t off) { return reinterpret_cast<int32_t*>(p->ws + off); }

ep::LayerBuf layer_buf(const ep_plan* p, int layer) {
  const size_t b = p->lay.layer_bytes * (size_t)layer;
  const Layout& l = p->lay;
  ep::LayerBuf L;
  L.load = at(p, b + l.load);
  L.expert_total = at(p, b + l.expert_total);
  L.W0 = at(p, b + l.W0);
  L.W = at(p, b + l.W);
  L.inst_expert = at(p, b + l.inst_expert);
  L.inst_quota = at(p, b + l.inst_quota);
  L.inst_off = at(p, b + l.inst_off);
  L.rank_base = at(p, b + l.rank_base);
  L.dst_row = at(p, b + l.dst_row);
  L.shared_rank = p->d.sh ? at(p, b + l.shared_rank) : nullptr;
  L.shared_row = p->d.sh ? at(p, b + l.shared_row) : nullptr;
  L.cand = at(p, b + l.cand);
  L.rep_list = at(p, b + l.rep_list);
  L.rep_eptr = at(p, b + l.rep_eptr);
  L.rep_nexp = at(p, b + l.rep_nexp);
  L.rep_experts = at(p, b + l.rep_experts);
  L.inst_count = p->d.sampled ? at(p, b + l.inst_count) : L.inst_quota;
  L.stats = reinterpret_cast<ep_layer_stats*>(p->ws + b + l.stats);
  return L;
}

ep::Scratch scratch(const ep_plan* p) {
  const Layout& l = p->lay;
  ep::Scratch s;
  s.sub_cnt = at(p, l.sub_cnt);
  s.blk_cnt = at(p, l.blk_cnt);
  s.wsub_cnt = p->d.sh ? at(p, l.wsub_cnt) : nullptr;
  s.seg_rec = at(p, l.seg_rec);
  s.seg_ord = at(p, l.seg_ord);
  s.seg_rank = at(p, l.seg_rank);
  s.seg_base = at(p, l.seg_base);
  s.inst_rel = at(p, l.inst_rel);
  s.slack = at(p, l.slack);
  s.wf = at(p, l.wf);
  s.sbase = at(p, l.sbase);
  s.shared_tot = at(p, l.shared_tot);
  s.asg_rank = p->d.sh ? reinterpret_cast<uint8_t*>(p->ws + l.asg_rank) : nullptr;
  s.acc_load = at(p, l.acc_load);
  s.acc_misc = at(p, l.acc_misc);
  const bool smp = p->d.sampled;
  s.smp_tot = smp ? at(p, l.smp_tot) : nullptr;
  s.smp_cum = smp ? at(p, l.smp_cum) : nullptr;
  s.smp_inst = smp ? at(p, l.smp_inst) : nullptr;
  s.smp_key = smp ? reinterpret_cast<uint16_t*>(p->ws + l.smp_key) : nullptr;
  s.smp_sub = smp ? at(p, l.smp_sub) : nullptr;
  s.smp_blk = smp ? at(p, l.smp_blk) : nullptr;
  s.smp_row0 = smp ? at(p, l.smp_row0) : nullptr;
  s.rank_rows = at(p, l.rank_rows);
  s.prev_base = at(p, l.prev_base);
  return s;
}

ep_status_t check_layer(const ep_plan* p, int32_t layer) {
  if (!p) return EP_ERR_INVALID_ARGUMENT;
  if (layer < 0 || layer >= p->cfg.num_layers) return EP_ERR_INVALID_ARGUMENT;
  return EP_OK;
}

ep_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t ep_abi_version(void) { return EP_ABI_VERSION; }

const char* ep_status_string(ep_status_t s) {
  switch (s) {
    case EP_OK: return "ok";
    case EP_ERR_INVALID_ARGUMENT: return "invalid argument";
    case EP_ERR_UNSUPPORTED: return "unsupported configuration";
    case EP_ERR_CUDA: return "CUDA error";
    case EP_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case EP_ERR_NOT_PLANNED: return "layer not balanced yet";
    case EP_ERR_DEVICE_STATUS: return "device status bit set";
    default: return "unknown status";
  }
}

ep_status_t ep_plan_workspace_bytes(const ep_config* cfg, size_t* bytes) {
  if (!bytes) return EP_ERR_INVALID_ARGUMENT;
  ep::Dims d;
  const ep_status_t st = make_dims(cfg, &d);
  if (st != EP_OK) return st;
  *bytes = make_layout(d, cfg->num_layers).total;
  return EP_OK;
}

ep_status_t ep_plan_create(const ep_config* cfg, void* d_workspace, size_t workspace_bytes,
                           ep_plan** out) {
  if (!out || !d_workspace) return EP_ERR_INVALID_ARGUMENT;
  *out = nullptr;
  ep::Dims d;
  ep_status_t st = make_dims(cfg, &d);
  if (st != EP_OK) return st;
  if ((reinterpret_cast<uintptr_t>(d_workspace) & (kAlign - 1)) != 0) return EP_ERR_INVALID_ARGUMENT;
  const Layout lay = make_layout(d, cfg->num_layers);
  if (workspace_bytes < lay.total) return EP_ERR_WORKSPACE_TOO_SMALL;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return EP_ERR_CUDA;
  // EP_GRID_SMS replaces the SM count the copy kernels size their grids by
  // (results never depend on it; tests use it to check exactly that)
  if (const char* env = getenv("EP_GRID_SMS")) {
    const long v = strtol(env, nullptr, 10);
    if (v > 0 && v <= 4096) sms = (int)v;
  }
  int max_smem = 0;
  if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return EP_ERR_CUDA;
  if (ep::set_plan_attributes(max_smem) != cudaSuccess) return EP_ERR_CUDA;
  {
    int dev_sms = 0;  // the device's own count: the plan kernels' grids are not overridden
    if (cudaDeviceGetAttribute(&dev_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return EP_ERR_CUDA;
    if (ep::plan_launch_shapes(d, max_smem, dev_sms) != cudaSuccess) return EP_ERR_CUDA;
  }
  if (ep::set_copy_attributes(max_smem) != cudaSuccess) return EP_ERR_CUDA;
  ep_plan* p = new (std::nothrow) ep_plan;
  if (!p) return EP_ERR_INVALID_ARGUMENT;
  p->planned = new (std::nothrow) unsigned char[cfg->num_layers];
  if (!p->planned) {
    delete p;
    return EP_ERR_INVALID_ARGUMENT;
  }
  memset(p->planned, 0, (size_t)cfg->num_layers);
  p->cfg = *cfg;
  p->d = d;
  p->lay = lay;
  p->ws = static_cast<char*>(d_workspace);
  p->ws_bytes = workspace_bytes;
  p->device = dev;
  p->num_sms = sms;
  {
    const char* impl = getenv("EP_DISPATCH_IMPL");
    p->dispatch_bulk = impl && strcmp(impl, "bulk") == 0;
  }
  p->acc_zero = false;
  *out = p;
  return EP_OK;
}

void ep_plan_destroy(ep_plan* plan) {
  if (!plan) return;
  delete[] plan->planned;
  delete plan;
}

ep_status_t ep_balance_layer(ep_plan* plan, int32_t layer, const int32_t* d_topk_ids,
                             void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!d_topk_ids && plan->d.T > 0) return EP_ERR_INVALID_ARGUMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!plan->acc_zero) {
    // the workspace arrives uninitialised; after this every balance call
    // leaves the accumulators zero for the next
    const Layout& l = plan->lay;
    const size_t bytes = l.acc_end - l.acc_load;
    st = cuda_status(cudaMemsetAsync(plan->ws + l.acc_load, 0, bytes, s));
    if (st != EP_OK) return st;
    plan->acc_zero = true;
  }
  st = cuda_status(ep::launch_balance(plan->d, layer_buf(plan, layer), scratch(plan), d_topk_ids, s));
  if (st == EP_OK) plan->planned[layer] = 1;
  else plan->acc_zero = false;  // a partly launched chain may leave them non-zero
  return st;
}

ep_status_t ep_layer_view_get(const ep_plan* plan, int32_t layer, ep_layer_view* out) {
  const ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!out) return EP_ERR_INVALID_ARGUMENT;
  const ep::LayerBuf L = layer_buf(plan, layer);
  out->load = L.load;
  out->expert_total = L.expert_total;
  out->rank_load_before = L.W0;
  out->rank_load = L.W;
  out->inst_expert = L.inst_expert;
  out->inst_quota = L.inst_quota;
  out->inst_off = L.inst_off;
  out->rank_row_begin = L.rank_base;
  out->dst_row = L.dst_row;
  out->shared_rank = L.shared_rank;
  out->shared_row = L.shared_row;
  out->cand_max_load = L.cand;
  out->cand_replicas = L.cand + plan->d.J;
  out->cand_stop = L.cand + 2 * plan->d.J;
  out->replica_list = L.rep_list;
  out->replica_expert_ptr = L.rep_eptr;
  out->stats = L.stats;
  out->inst_count = L.inst_count;
  out->Gmax = plan->d.Gmax;
  out->G = plan->d.G;
  return EP_OK;
}

ep_status_t ep_read_layer_stats(ep_plan* plan, int32_t layer, ep_layer_stats* h_out,
                                void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!h_out) return EP_ERR_INVALID_ARGUMENT;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ep::LayerBuf L = layer_buf(plan, layer);
  if (cudaMemcpyAsync(h_out, L.stats, sizeof(ep_layer_stats), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return EP_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return EP_ERR_CUDA;
  return h_out->status ? EP_ERR_DEVICE_STATUS : EP_OK;
}

ep_status_t ep_dispatch_layout(ep_plan* plan, int32_t layer, const void* d_hidden, void* d_out,
                               int64_t out_rows_capacity, int32_t dst_rank_begin,
                               int32_t dst_rank_end, void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  if (dst_rank_begin < 0 || dst_rank_end > plan->d.R || dst_rank_begin > dst_rank_end ||
      out_rows_capacity < 0)
    return EP_ERR_INVALID_ARGUMENT;
  if ((int64_t)plan->d.R * plan->d.T > 0 && (!d_hidden || !d_out)) return EP_ERR_INVALID_ARGUMENT;
  if (!aligned16(d_hidden) || !aligned16(d_out)) return EP_ERR_INVALID_ARGUMENT;
  if (dst_rank_begin == dst_rank_end) return EP_OK;
  return cuda_status(ep::launch_dispatch(plan->d, layer_buf(plan, layer), d_hidden, d_out,
                                         out_rows_capacity, dst_rank_begin, dst_rank_end, 0,
                                         (int64_t)plan->d.R * plan->d.T, plan->num_sms,
                                         plan->dispatch_bulk, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_dispatch_tokens(ep_plan* plan, int32_t layer, const void* d_hidden, int64_t token_begin,
                               int64_t token_end, void* d_out, int64_t out_rows_capacity,
                               void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  const int64_t N = (int64_t)plan->d.R * plan->d.T;
  if (token_begin < 0 || token_end > N || token_begin > token_end || out_rows_capacity < 0)
    return EP_ERR_INVALID_ARGUMENT;
  if (token_begin == token_end) return EP_OK;
  if (!d_hidden || !d_out || !aligned16(d_hidden) || !aligned16(d_out)) return EP_ERR_INVALID_ARGUMENT;
  return cuda_status(ep::launch_dispatch(plan->d, layer_buf(plan, layer), d_hidden, d_out,
                                         out_rows_capacity, 0, plan->d.R, token_begin, token_end,
                                         plan->num_sms, plan->dispatch_bulk,
                                         static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_combine(ep_plan* plan, int32_t layer, const void* d_expert_out, const float* d_weights,
                       void* d_out, int32_t out_dtype, void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  if (out_dtype != 0 && out_dtype != 1) return EP_ERR_INVALID_ARGUMENT;
  if ((int64_t)plan->d.R * plan->d.T > 0 && (!d_expert_out || !d_weights || !d_out))
    return EP_ERR_INVALID_ARGUMENT;
  if (!aligned16(d_expert_out) || !aligned16(d_out) ||
      (reinterpret_cast<uintptr_t>(d_weights) & 3u) != 0)
    return EP_ERR_INVALID_ARGUMENT;
  return cuda_status(ep::launch_combine(plan->d, layer_buf(plan, layer), d_expert_out, d_weights,
                                        d_out, out_dtype, plan->num_sms,
                                        static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_stage_replicas(ep_plan* plan, int32_t layer, const void* d_native_w,
                              void* d_slots, void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  if (plan->d.Wn > 0 && plan->d.S > 0 && (!d_native_w || !d_slots)) return EP_ERR_INVALID_ARGUMENT;
  if (!aligned16(d_native_w) || !aligned16(d_slots)) return EP_ERR_INVALID_ARGUMENT;
  return cuda_status(ep::launch_stage(plan->d, layer_buf(plan, layer), d_native_w, d_slots,
                                      plan->num_sms, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_reduce_replica_grads(ep_plan* plan, int32_t layer, void* d_slot_grads,
                                    int32_t grad_dtype, float* d_native_grads, void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  if (grad_dtype != 0 && grad_dtype != 1) return EP_ERR_INVALID_ARGUMENT;
  if (plan->d.Wn > 0 && plan->d.S > 0 && (!d_slot_grads || !d_native_grads))
    return EP_ERR_INVALID_ARGUMENT;
  if (!aligned16(d_slot_grads) || !aligned16(d_native_grads)) return EP_ERR_INVALID_ARGUMENT;
  return cuda_status(ep::launch_reduce(plan->d, layer_buf(plan, layer), d_slot_grads, grad_dtype,
                                       d_native_grads, plan->num_sms,
                                       static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_waterfill(int32_t R, int32_t T, int32_t K, const int32_t* d_load,
                         const int32_t* d_dst_rank, uint64_t seed, int32_t bonus_permille,
                         int32_t flags, int32_t* d_pick, int32_t* d_count, void* stream) {
  if (R < 1 || T < 0 || K < 0 || bonus_permille < 0 || (flags & ~EP_WATERFILL_ALL_RANKS) != 0)
    return EP_ERR_INVALID_ARGUMENT;
  if (R > ep::kMaxR || K > ep::kMaxK || bonus_permille > 1000) return EP_ERR_UNSUPPORTED;
  if ((int64_t)R * T * (K + 1) >= (int64_t)INT32_MAX) return EP_ERR_UNSUPPORTED;
  if (!d_load || !d_count) return EP_ERR_INVALID_ARGUMENT;
  if (T > 0 && (!d_pick || (K > 0 && !d_dst_rank))) return EP_ERR_INVALID_ARGUMENT;
  return cuda_status(ep::launch_waterfill(R, T, K, d_load, d_dst_rank, seed, bonus_permille,
                                          flags & EP_WATERFILL_ALL_RANKS, d_pick, d_count,
                                          static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_waterfill_layer(ep_plan* plan, int32_t layer, uint64_t seed, void* stream) {
  ep_status_t st = check_layer(plan, layer);
  if (st != EP_OK) return st;
  if (!plan->d.sh) return EP_ERR_UNSUPPORTED;
  if (!plan->planned[layer]) return EP_ERR_NOT_PLANNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!plan->acc_zero) {  // the shared scan's arrival ticket must start at zero
    const Layout& l = plan->lay;
    st = cuda_status(cudaMemsetAsync(plan->ws + l.acc_load, 0, l.acc_end - l.acc_load, s));
    if (st != EP_OK) return st;
    plan->acc_zero = true;
  }
  ep::Dims d = plan->d;
  d.seed = seed;
  st = cuda_status(ep::launch_waterfill_layer(d, layer_buf(plan, layer), scratch(plan), s));
  if (st != EP_OK) plan->acc_zero = false;
  return st;
}

}  // extern "C"
