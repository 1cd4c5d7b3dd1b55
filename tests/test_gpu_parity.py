"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer outputs must be bit-exact; the gradient reduction too, since both sides
add in the same fixed order in fp32.  Sizes span several sub-chunks and a
ragged tail; the five named workloads run at full size.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_b200 import EpError, Plan, config_from_workload, ep_waterfill
from tests.gpu_helpers import compare_plan, fetch, gpu_plan, oracle_plan
from tests.invariants import check_plan
from workloads import get_config, topk_ids

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "qwen", "dsv3", "stress"])
def test_plan_parity_full_configs(name):
    w = get_config(name)
    ids = topk_ids(w)
    o = oracle_plan(w, ids)
    plan = gpu_plan(w, ids)
    compare_plan(fetch(plan), o, w)


def test_plan_parity_large_counts():
    # R*T*K = 2^24 assignments: load, slack and quota values too wide for the
    # solver's one-redux argmax keys, so it takes the two-step (max, ballot) path
    w = get_config("stress").replace(R=64, T=32768, S=2, distinct=True, hot_frac=None, seed=6001)
    assert w.A == 1 << 24
    ids = topk_ids(w)
    o = oracle_plan(w, ids)
    plan = gpu_plan(w, ids)
    compare_plan(fetch(plan), o, w)
    assert o.replicas > 0


def _skewed_topk(rng, R, T, E, K, zipf_s):
    """Distinct top-K ids per token from a Zipf-skewed popularity (Gumbel top-k)."""
    logp = -zipf_s * np.log(np.arange(1, E + 1, dtype=np.float64))
    logp = logp[rng.permutation(E)]
    g = rng.gumbel(size=(R * T, E)) + logp
    ids = np.argpartition(-g, K - 1, axis=1)[:, :K]
    return ids.reshape(R, T, K).astype(np.int32)


@pytest.mark.parametrize("R,E,K,T,S,m,shared", [
    (128, 1024, 16, 96, 8, 1, False),   # every limit at once: 4 rank words, 8 slots, 8 natives
    (128, 1024, 16, 96, 8, 16, True),
    (128, 128, 16, 200, 8, 4, True),    # one native per rank
    (32, 1024, 8, 300, 2, 8, False),    # 32 natives per rank (the solver's lane limit)
    (1, 32, 16, 500, 8, 1, True),       # a single rank
])
def test_plan_parity_maximum_shapes(R, E, K, T, S, m, shared):
    rng = np.random.default_rng(R * 7919 + E + K + S)
    ids = _skewed_topk(rng, R, T, E, K, 1.3)
    w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=m, J=16, shared_expert=shared)
    o = oracle_plan(w, ids)
    compare_plan(fetch(gpu_plan(w, ids)), o, w)


@pytest.mark.parametrize("K,T,m,shared", [(8, 600, 1, False), (16, 300, 4, True)])
def test_plan_parity_every_slot_filled(K, T, m, shared):
    # rank 0's 32 natives (the solver's lane limit) carry all the load, so the
    # greedy moves whole experts until each of the 3 other ranks holds 8
    # replicas (every slot of the 8-slot layout in use)
    R, E, S = 4, 128, 8
    rng = np.random.default_rng(5)
    logp = np.full(E, -8.0)
    logp[:32] = 0.0
    g = rng.gumbel(size=(R * T, E)) + logp
    ids = np.argpartition(-g, K - 1, axis=1)[:, :K].reshape(R, T, K).astype(np.int32)
    w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=m, J=16, shared_expert=shared)
    o = oracle_plan(w, ids)
    assert (o.inst_expert[1:, o.Gmax:o.Gmax + S] >= 0).all()
    compare_plan(fetch(gpu_plan(w, ids)), o, w)


def test_stage_and_reduce_every_slot_filled():
    # the 24-replica plan above: staging copies each filled slot's expert, the
    # reduction adds up to 3 replicas per expert in instance order
    R, E, S, K, T, Wn = 4, 128, 8, 8, 600, 1000
    rng = np.random.default_rng(5)
    logp = np.full(E, -8.0)
    logp[:32] = 0.0
    g = rng.gumbel(size=(R * T, E)) + logp
    ids = np.argpartition(-g, K - 1, axis=1)[:, :K].reshape(R, T, K).astype(np.int32)
    w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=1, J=16)
    plan = gpu_plan(w, ids, expert_weight_elems=Wn)
    o = oracle_plan(w, ids)
    native = torch.from_numpy(rng.integers(-30000, 30000, (E, Wn)).astype(np.int16)).cuda()
    slots = torch.full((R, S, Wn), 3, dtype=torch.int16, device="cuda")
    plan.stage_replicas(0, native.view(torch.bfloat16), slots.view(torch.bfloat16))
    g32 = (rng.standard_normal((R, S, Wn)) * 1e-2).astype(np.float32)
    g_np = (g32.view(np.uint32) >> 16).astype(np.uint16)
    g_t = torch.from_numpy(g_np.view(np.int16)).cuda().view(torch.bfloat16)
    nat_np = rng.standard_normal((E, Wn)).astype(np.float32)
    nat_t = torch.from_numpy(nat_np).cuda()
    plan.reduce_replica_grads(0, g_t, nat_t)
    torch.cuda.synchronize()
    want_slots = np.full((R, S, Wn), 3, np.int16)
    oracle.stage(o, native.cpu().numpy(), want_slots)
    np.testing.assert_array_equal(slots.cpu().numpy(), want_slots)
    want_nat, want_g = nat_np.copy(), g_np.copy()
    oracle.reduce_grads(o, want_g, want_nat)
    np.testing.assert_array_equal(nat_t.cpu().numpy().view(np.uint32), want_nat.view(np.uint32))
    np.testing.assert_array_equal(g_t.view(torch.int16).cpu().numpy().view(np.uint16), want_g)


def test_plan_parity_sweep_layers_cached():
    w = get_config("sweep")
    layers = [0, 1, 3, 47, 93]
    plan = Plan(config_from_workload(w, num_layers=w.layers))
    ids_by_layer = {l: topk_ids(w, l) for l in layers}
    for l in layers:
        gpu_plan(w, ids_by_layer[l], plan=plan, layer=l)
    # every cached layer still holds its own plan after later layers ran
    for l in layers:
        compare_plan(fetch(plan, l), oracle_plan(w, ids_by_layer[l]), w)


def _random_case(rng):
    R = int(rng.integers(1, 20))
    E = int(rng.integers(max(1, R // 2), min(32 * R, 300) + 1))
    K = int(rng.integers(1, 10))
    T = int(rng.integers(0, 700))
    S = int(rng.integers(0, 5))
    m = int(rng.choice([1, 3, 16, 64]))
    shared = bool(rng.integers(0, 2))
    J = int(rng.integers(1, 17))
    skew = rng.dirichlet(np.ones(E) * 0.2)
    ids = rng.choice(E, size=(R, T, K), p=skew).astype(np.int32)
    return R, E, K, T, S, m, shared, J, ids


def test_plan_parity_random_shapes():
    rng = np.random.default_rng(2024)
    for case in range(40):
        R, E, K, T, S, m, shared, J, ids = _random_case(rng)
        w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=m, J=J, shared_expert=shared)
        o = oracle_plan(w, ids)
        g = fetch(gpu_plan(w, ids))
        compare_plan(g, o, w)


def test_plan_parity_random_shapes_wide():
    # the rest of the shape space: up to 8 slots and 16 experts per token,
    # repeated experts in a token, Waterfill over all ranks
    rng = np.random.default_rng(4242)
    for case in range(30):
        R = int(rng.integers(1, 40))
        E = int(rng.integers(1, min(32 * R, 400) + 1))
        K = int(rng.integers(1, min(E, 16) + 1))
        T = int(rng.integers(0, 500))
        S = int(rng.integers(4, 9))
        m = int(rng.choice([1, 4, 32]))
        shared = bool(rng.integers(0, 2))
        all_ranks = bool(rng.integers(0, 2))
        p_e = rng.dirichlet(np.full(E, 0.3))
        if rng.integers(0, 2):
            g = rng.gumbel(size=(R * T, E)) + np.log(p_e + 1e-12)
            ids = np.argsort(-g, axis=1)[:, :K].reshape(R, T, K).astype(np.int32)
        else:
            ids = rng.choice(E, size=(R, T, K), p=p_e).astype(np.int32)
        w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=m, J=16, shared_expert=shared,
                                       waterfill_all_ranks=all_ranks)
        o = oracle_plan(w, ids)
        compare_plan(fetch(gpu_plan(w, ids)), o, w)


def test_plan_parity_bad_ids_and_ragged_tail():
    w = get_config("tiny").replace(T=1000, shared_expert=True)
    ids = topk_ids(get_config("tiny"))[:, :1000].copy()
    ids[0, 3, 1] = w.E
    ids[3, 999, 0] = -7
    o = oracle_plan(w, ids)
    plan = gpu_plan(w, ids)
    g = fetch(plan)
    compare_plan(g, o, w)
    assert g["stats"]["status"] & 1
    assert g["dst_row"][0, 3, 1] == -1


@pytest.mark.parametrize("shared", [False, True])
def test_plan_state_does_not_carry_between_calls(shared):
    # one plan, one layer, several calls in a row with different ids (one with
    # bad ids, one empty-looking skew, then the first again): every call must
    # equal the oracle on its own ids, and a status bit of one call must not
    # survive into the next
    base = get_config("tiny").replace(T=1000, shared_expert=shared)
    rng = np.random.default_rng(11)
    good = topk_ids(get_config("tiny"))[:, :1000].copy()
    bad = good.copy()
    bad[1, 5, 0] = base.E + 3
    skew = np.zeros_like(good)
    skew[..., 1] = 1
    shuffled = rng.permutation(good.reshape(-1)).reshape(good.shape).astype(np.int32)
    plan = Plan(config_from_workload(base, num_layers=2))
    for ids in (good, bad, skew, shuffled, good):
        for layer in (0, 1):
            gpu_plan(base, ids, plan=plan, layer=layer)
            g = fetch(plan, layer)
            compare_plan(g, oracle_plan(base, ids), base)
            assert (g["stats"]["status"] & 1) == (1 if ids is bad else 0)


def test_plan_deterministic():
    w = get_config("dsv3")
    ids = topk_ids(w)
    a = fetch(gpu_plan(w, ids))
    b = fetch(gpu_plan(w, ids))
    for k in ("dst_row", "shared_row", "inst_quota", "inst_expert", "load"):
        np.testing.assert_array_equal(a[k], b[k])


def test_results_do_not_depend_on_the_copy_grids(monkeypatch):
    # the same layer through plans whose copy kernels run on grids sized for 3
    # and for 1000 SMs instead of the device's: every output bitwise equal
    w = get_config("dsv3").replace(T=1000)
    ids = topk_ids(get_config("dsv3"))[:, :1000].copy()
    Wn = 3 * 7168 * 2
    g = torch.Generator(device="cuda")
    g.manual_seed(31)
    hidden = torch.randn((w.N, w.hidden), generator=g, device="cuda").to(torch.bfloat16)
    native = torch.randn((w.E, Wn), generator=g, device="cuda").to(torch.bfloat16)
    grads = (torch.randn((w.R, w.S, Wn), generator=g, device="cuda") * 1e-2).to(torch.bfloat16)
    gates = torch.rand((w.R, w.T, w.K), generator=g, device="cuda")
    outs = []
    for sms in (None, "3", "1000"):
        if sms is None:
            monkeypatch.delenv("EP_GRID_SMS", raising=False)
        else:
            monkeypatch.setenv("EP_GRID_SMS", sms)
        plan = gpu_plan(w, ids, expert_weight_elems=Wn)
        disp = plan.dispatch_layout(0, hidden)
        slots = torch.zeros((w.R, w.S, Wn), dtype=torch.bfloat16, device="cuda")
        plan.stage_replicas(0, native, slots)
        gr = grads.clone()
        nat = torch.ones((w.E, Wn), dtype=torch.float32, device="cuda")
        plan.reduce_replica_grads(0, gr, nat)
        y = plan.combine(0, disp, gates, out_dtype=torch.float32)
        torch.cuda.synchronize()
        outs.append([t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)
                     for t in (disp, slots, gr, nat, y)] + [plan.view(0)["dst_row"].clone()])
    monkeypatch.delenv("EP_GRID_SMS", raising=False)
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)


def test_plan_invariants_on_gpu_output():
    w = get_config("qwen")
    ids = topk_ids(w)
    g = fetch(gpu_plan(w, ids))
    check_plan(ids, w.E, w.S, w.m, Gmax=g["Gmax"], G=g["G"], W=g["rank_load"],
               inst_expert=g["inst_expert"], inst_quota=g["inst_quota"], inst_off=g["inst_off"],
               dst_row=g["dst_row"], cap=g["stats"]["cap"])
    ratio = g["stats"]["after_max"] * w.R / g["stats"]["assignments"]
    assert ratio <= 1.05 or g["stats"]["tight_stop_reason"] == 1


# ---- sampled rerouting ("Waterfill and LPLB" page, section "LPLB") ---------------
@pytest.mark.parametrize("name", ["tiny", "qwen", "dsv3", "stress"])
def test_plan_parity_sampled_full_configs(name):
    w = get_config(name).replace(sampled_rerouting=True)
    ids = topk_ids(get_config(name))
    o = oracle_plan(w, ids)
    g = fetch(gpu_plan(w, ids))
    compare_plan(g, o, w)
    if o.replicas:
        assert (o.inst_count != o.inst_quota).any()  # the draws are not the quotas


def test_plan_parity_sampled_random_shapes():
    rng = np.random.default_rng(777)
    for case in range(30):
        R, E, K, T, S, m, shared, J, ids = _random_case(rng)
        if case % 3 == 0 and T:
            ids[0, 0, 0] = E  # a dropped id
        w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=m, J=J, shared_expert=shared,
                                       sampled_rerouting=True, sampling_seed=int(rng.integers(0, 2**62)),
                                       waterfill_all_ranks=bool(case % 2))
        o = oracle_plan(w, ids)
        compare_plan(fetch(gpu_plan(w, ids)), o, w)


@pytest.mark.parametrize("R,E,K,T,S,shared", [
    (128, 1024, 16, 40, 8, True),   # the largest key space: E + R*S = 2048 keys
    (4, 128, 8, 600, 8, False),     # every slot filled
])
def test_plan_parity_sampled_maximum_shapes(R, E, K, T, S, shared):
    rng = np.random.default_rng(R + E + S)
    if R == 4:
        logp = np.full(E, -8.0)
        logp[:32] = 0.0
        g = rng.gumbel(size=(R * T, E)) + logp
        ids = np.argpartition(-g, K - 1, axis=1)[:, :K].reshape(R, T, K).astype(np.int32)
    else:
        ids = _skewed_topk(rng, R, T, E, K, 1.3)
    w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=1, J=16, shared_expert=shared,
                                   sampled_rerouting=True, sampling_seed=99)
    o = oracle_plan(w, ids)
    compare_plan(fetch(gpu_plan(w, ids)), o, w)


def test_sampled_dispatch_matches_oracle():
    w = get_config("tiny").replace(T=777, shared_expert=True, sampled_rerouting=True)
    ids = topk_ids(get_config("tiny"))[:, :777].copy()
    plan = gpu_plan(w, ids)
    hidden = _hidden(w, 9)
    out = plan.dispatch_layout(0, hidden)
    torch.cuda.synchronize()
    o = oracle_plan(w, ids)
    want = oracle.permute(o, hidden.view(torch.int16).cpu().numpy())
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy()[: o.rows], want)
    assert plan.read_layer_stats(0)["status"] == 0


# ---- the solver's iteration bound -------------------------------------------------
@pytest.mark.parametrize("name,limit", [("qwen", 2), ("dsv3", 5), ("tiny", 1)])
def test_iteration_bound_sets_status_and_keeps_a_valid_plan(name, limit):
    # a bound smaller than the moves the greedy needs: every candidate stops
    # there, the status bit is set and the plan is still a valid layout equal
    # to the oracle's under the same bound
    w = get_config(name)
    ids = topk_ids(w)
    o = oracle_plan(w, ids, iter_limit=limit)
    assert o.status & oracle.ST_ITER_CAP
    plan = gpu_plan(w, ids, solver_iter_limit=limit)
    g = fetch(plan)
    compare_plan(g, o, w)
    assert g["stats"]["status"] & 2  # EP_DEV_ITER_CAP
    assert (g["cand_stop"] == 3).any()
    check_plan(ids, w.E, w.S, w.m, Gmax=g["Gmax"], G=g["G"], W=g["rank_load"],
               inst_expert=g["inst_expert"], inst_quota=g["inst_quota"], inst_off=g["inst_off"],
               dst_row=g["dst_row"], cap=g["stats"]["cap"], shared_rank=g["shared_rank"],
               shared_row=g["shared_row"])
    # the next call without the bound (another plan, same ids) is clean
    assert plan.read_layer_stats(0)["status"] & 2
    assert fetch(gpu_plan(w, ids))["stats"]["status"] == 0


# ---- dispatch permutation ------------------------------------------------------
def _hidden(w, seed=0):
    g = torch.Generator(device="cuda")
    g.manual_seed(1234 + seed)
    return torch.randn((w.N, w.hidden), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("shared,hidden_dim,out_offset", [
    (False, 256, 0), (True, 256, 0),   # 32-byte rows and buffers: 32-byte vectors
    (False, 264, 0),                   # 528-byte rows: 16-byte vectors
    (True, 256, 8),                    # output 16 bytes past a 32-byte boundary
])
def test_dispatch_matches_oracle_small(shared, hidden_dim, out_offset):
    w = get_config("tiny").replace(T=777, shared_expert=shared, hidden=hidden_dim)
    ids = topk_ids(get_config("tiny"))[:, :777].copy()
    plan = gpu_plan(w, ids)
    hidden = _hidden(w)
    rows = w.A + (w.N if shared else 0)
    flat = torch.zeros(rows * w.hidden + out_offset, dtype=torch.bfloat16, device="cuda")
    out = flat[out_offset:].view(rows, w.hidden)
    assert (out.data_ptr() % 32 == 0) == (out_offset == 0)
    plan.dispatch_layout(0, hidden, out=out)
    torch.cuda.synchronize()
    o = oracle_plan(w, ids)
    want = oracle.permute(o, hidden.view(torch.int16).cpu().numpy())
    got = out.view(torch.int16).cpu().numpy()[: o.rows]
    np.testing.assert_array_equal(got, want)
    assert plan.read_layer_stats(0)["status"] == 0


def test_dispatch_full_qwen_round_trip():
    w = get_config("qwen")
    ids = topk_ids(w)
    plan = gpu_plan(w, ids)
    hidden = _hidden(w)
    out = torch.full((w.A, w.hidden), -1.0, dtype=torch.bfloat16, device="cuda")
    plan.dispatch_layout(0, hidden, out=out)
    torch.cuda.synchronize()
    dst = plan.view(0)["dst_row"].reshape(w.N, w.K).long()
    for k in range(w.K):  # gather back by dst_row: bitwise the source rows
        assert torch.equal(out[dst[:, k]].view(torch.int16), hidden.view(torch.int16))
    assert plan.read_layer_stats(0)["status"] == 0


def _rows_hold_tokens(out, lo, hi, rows_np, hidden, chunk=1 << 15):
    """out[row - lo] == hidden[n] (bitwise) for every token n whose oracle row
    `rows_np[n]` lies in [lo, hi); returns how many rows were checked."""
    n_all = np.nonzero((rows_np >= lo) & (rows_np < hi))[0]
    for a in range(0, len(n_all), chunk):
        n = torch.from_numpy(n_all[a:a + chunk]).cuda()
        r = torch.from_numpy(rows_np[n_all[a:a + chunk]] - lo).cuda()
        assert torch.equal(out[r].view(torch.int16), hidden[n].view(torch.int16))
    return len(n_all)


def _count_unwritten(out, sentinel=-1, chunk=1 << 16):
    bad = 0
    o16 = out.view(torch.int16)
    for a in range(0, o16.shape[0], chunk):
        bad += int((o16[a:a + chunk] == sentinel).all(dim=1).sum())
    return bad


def test_dispatch_dsv3_full_matches_oracle_rows():
    # the whole DeepSeek-V3-shaped layer (routed and shared rows, 33.8 GB):
    # every token's row, at the position the oracle's layout gives it, holds
    # the token's hidden state, and no row is left unwritten
    w = get_config("dsv3")
    ids = topk_ids(w)
    o = oracle_plan(w, ids)
    plan = gpu_plan(w, ids)
    hidden = _hidden(w, 6)
    out = torch.full((o.rows, w.hidden), -1, dtype=torch.int16, device="cuda")
    plan.dispatch_layout(0, hidden, out=out.view(torch.bfloat16))
    torch.cuda.synchronize()
    dst = o.dst_row.reshape(w.N, w.K)
    checked = sum(_rows_hold_tokens(out, 0, o.rows, np.ascontiguousarray(dst[:, k]), hidden)
                  for k in range(w.K))
    checked += _rows_hold_tokens(out, 0, o.rows, o.shared_row.reshape(w.N), hidden)
    assert checked == o.rows == w.A + w.N
    assert _count_unwritten(out) == 0
    assert plan.read_layer_stats(0)["status"] == 0


def test_dispatch_stress_rank_windows_match_oracle_rows():
    # the stress layer's 135 GB layout does not fit one GPU next to its input:
    # it is dispatched in destination-rank windows; each window holds exactly
    # the oracle's rows of those ranks
    w = get_config("stress")
    ids = topk_ids(w)
    o = oracle_plan(w, ids)
    plan = gpu_plan(w, ids)
    hidden = _hidden(w, 7)
    rb = o.inst_off[np.arange(w.R + 1) * o.G]
    dst = o.dst_row.reshape(w.N, w.K)
    cols = [np.ascontiguousarray(dst[:, k]) for k in range(w.K)]
    total = 0
    for b, e in [(0, 18), (18, 37), (37, 72)]:
        lo, hi = int(rb[b]), int(rb[e])
        out = torch.full((hi - lo, w.hidden), -1, dtype=torch.int16, device="cuda")
        plan.dispatch_layout(0, hidden, out=out.view(torch.bfloat16), rank_begin=b, rank_end=e)
        torch.cuda.synchronize()
        checked = sum(_rows_hold_tokens(out, lo, hi, c, hidden) for c in cols)
        assert checked == hi - lo
        assert _count_unwritten(out) == 0
        total += checked
        del out
        torch.cuda.empty_cache()
    assert total == o.rows == w.A
    assert plan.read_layer_stats(0)["status"] == 0


def test_dispatch_rank_windows_concatenate():
    w = get_config("dsv3")
    ids = topk_ids(w)
    plan = gpu_plan(w, ids)
    hidden = _hidden(w, 1)
    full = plan.dispatch_layout(0, hidden)
    rb = plan.view(0)["rank_row_begin"].cpu().numpy()
    parts = []
    for b, e in [(0, 5), (5, 23), (23, 24), (24, 64)]:
        n = int(rb[e] - rb[b])
        parts.append(plan.dispatch_layout(0, hidden, rank_begin=b, rank_end=e, out_rows=max(n, 1))[:n])
    torch.cuda.synchronize()
    cat = torch.cat(parts)
    rows = int(rb[-1])
    assert torch.equal(cat.view(torch.int16), full[:rows].view(torch.int16))
    assert plan.read_layer_stats(0)["status"] == 0


@pytest.mark.parametrize("shared", [False, True])
def test_dispatch_token_ranges_match_oracle(shared):
    # ragged source-token chunks, each written into the same buffer, give the
    # oracle's permutation; a chunk writes only its own tokens' rows
    w = get_config("tiny").replace(T=777, shared_expert=shared)
    ids = topk_ids(get_config("tiny"))[:, :777].copy()
    plan = gpu_plan(w, ids)
    hidden = _hidden(w, 2)
    o = oracle_plan(w, ids)
    want = oracle.permute(o, hidden.view(torch.int16).cpu().numpy())
    rows = w.A + (w.N if shared else 0)
    out = torch.zeros((rows, w.hidden), dtype=torch.bfloat16, device="cuda")
    cuts = [0, 1, 500, 2047, 2048, 3000, w.N]
    plan.dispatch_tokens(0, hidden, out, 500, 2047)
    torch.cuda.synchronize()
    got = out.view(torch.int16).cpu().numpy()
    mine = np.zeros(rows, bool)
    dst = o.dst_row.reshape(w.N, w.K)[500:2047]
    mine[dst.ravel()] = True
    if shared:
        mine[o.shared_row.reshape(w.N)[500:2047]] = True
    np.testing.assert_array_equal(got[mine], want[mine])
    assert not got[~mine].any()
    for b, e in zip(cuts[:-1], cuts[1:]):
        plan.dispatch_tokens(0, hidden, out, b, e)
    plan.dispatch_tokens(0, hidden, out, 7, 7)  # empty range: nothing
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy(), want)
    assert plan.read_layer_stats(0)["status"] == 0


@pytest.mark.parametrize("shared,hidden_dim", [(False, 256), (True, 264), (True, 7168)])
def test_bulk_copy_dispatch_variant_matches_oracle(monkeypatch, shared, hidden_dim):
    # the bulk-copy (TMA) variant of the dispatch, chosen at plan creation:
    # the whole layout, destination-rank windows and source-token ranges give
    # the oracle's bytes
    monkeypatch.setenv("EP_DISPATCH_IMPL", "bulk")
    w = get_config("tiny").replace(T=777, shared_expert=shared, hidden=hidden_dim)
    ids = topk_ids(get_config("tiny"))[:, :777].copy()
    plan = gpu_plan(w, ids)
    monkeypatch.delenv("EP_DISPATCH_IMPL")
    hidden = _hidden(w, 11)
    o = oracle_plan(w, ids)
    want = oracle.permute(o, hidden.view(torch.int16).cpu().numpy())
    out = plan.dispatch_layout(0, hidden)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy()[: o.rows], want)
    rb = o.inst_off[np.arange(w.R + 1) * o.G]
    for b, e in [(0, 1), (1, 4)]:
        n = int(rb[e] - rb[b])
        part = plan.dispatch_layout(0, hidden, rank_begin=b, rank_end=e, out_rows=max(n, 1))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(part.view(torch.int16).cpu().numpy()[:n], want[rb[b]:rb[e]])
    out2 = torch.zeros_like(out)
    for lo, hi in [(0, 5), (5, 1500), (1500, w.N)]:
        plan.dispatch_tokens(0, hidden, out2, lo, hi)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out2.view(torch.int16).cpu().numpy()[: o.rows], want)
    assert plan.read_layer_stats(0)["status"] == 0


def test_bulk_copy_dispatch_variant_full_qwen_round_trip(monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_IMPL", "bulk")
    w = get_config("qwen")
    ids = topk_ids(w)
    plan = gpu_plan(w, ids)
    monkeypatch.delenv("EP_DISPATCH_IMPL")
    hidden = _hidden(w, 12)
    out = torch.full((w.A, w.hidden), -1.0, dtype=torch.bfloat16, device="cuda")
    plan.dispatch_layout(0, hidden, out=out)
    torch.cuda.synchronize()
    o = oracle_plan(w, ids)
    dst = o.dst_row.reshape(w.N, w.K)
    for k in range(w.K):  # the oracle's rows hold the tokens
        assert _rows_hold_tokens(out, 0, o.rows, np.ascontiguousarray(dst[:, k]), hidden) == w.N
    assert plan.read_layer_stats(0)["status"] == 0


def test_dispatch_tokens_argument_errors():
    w = get_config("tiny")
    plan = Plan(config_from_workload(w))
    hidden = _hidden(w)
    out = torch.empty((w.A, w.hidden), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(EpError) as ei:
        plan.dispatch_tokens(0, hidden, out, 0, 10)
    assert ei.value.status == 5  # not planned yet
    plan.balance_layer(0, torch.from_numpy(topk_ids(w)).cuda())
    for b, e in [(-1, 3), (5, 4), (0, w.N + 1)]:
        with pytest.raises(EpError) as ei:
            plan.dispatch_tokens(0, hidden, out, b, e)
        assert ei.value.status == 1
    plan.dispatch_tokens(0, hidden, out, 0, w.N)
    torch.cuda.synchronize()
    assert plan.read_layer_stats(0)["status"] == 0


def test_balance_and_dispatch_replay_from_cuda_graph():
    # the plan chain (programmatic dependent launches) and the dispatch,
    # captured once and replayed on new ids written into the same buffer
    w = get_config("tiny").replace(T=1000, shared_expert=True)
    base = topk_ids(get_config("tiny"))[:, :1000].copy()
    rng = np.random.default_rng(3)
    sets = [base, rng.permutation(base.reshape(-1)).reshape(base.shape).astype(np.int32),
            np.ascontiguousarray(base[:, ::-1])]
    plan = Plan(config_from_workload(w))
    ids_buf = torch.from_numpy(sets[1]).cuda()
    hidden = _hidden(w, 4)
    out = torch.zeros((w.A + w.N, w.hidden), dtype=torch.bfloat16, device="cuda")
    plan.balance_layer(0, ids_buf)  # outside the graph: the plan's first call
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        plan.balance_layer(0, ids_buf)
        plan.dispatch_layout(0, hidden, out=out)
    for ids in sets:
        ids_buf.copy_(torch.from_numpy(ids))
        graph.replay()
        torch.cuda.synchronize()
        o = oracle_plan(w, ids)
        compare_plan(fetch(plan), o, w)
        want = oracle.permute(o, hidden.view(torch.int16).cpu().numpy())
        np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy()[: o.rows], want)
    del graph


def test_dispatch_capacity_overflow_is_flagged_not_written():
    w = get_config("tiny")
    ids = topk_ids(w)
    plan = gpu_plan(w, ids)
    hidden = _hidden(w)
    guard = torch.zeros((w.A + 64, w.hidden), dtype=torch.bfloat16, device="cuda")
    out = guard[:100]
    plan.dispatch_layout(0, hidden, out=out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(guard[100:]) == 0
    st = plan.read_layer_stats(0)
    assert st["status"] & 8


# ---- replica staging and gradient reduction -----------------------------------
def test_stage_replicas_qwen():
    # which expert each slot must hold comes from the oracle's plan, not from
    # the plan under test
    w = get_config("qwen")
    ids = topk_ids(w)
    plan = gpu_plan(w, ids)
    o = oracle_plan(w, ids)
    Wn = w.expert_elems
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    native = torch.randint(-32768, 32767, (w.E, Wn), generator=g, device="cuda", dtype=torch.int16)
    slots = torch.full((w.R, w.S, Wn), 7, dtype=torch.int16, device="cuda")
    plan.stage_replicas(0, native.view(torch.bfloat16), slots.view(torch.bfloat16))
    torch.cuda.synchronize()
    filled = 0
    for q in range(w.R):
        for s in range(w.S):
            e = int(o.inst_expert[q, o.Gmax + s])
            if e >= 0:
                filled += 1
                assert torch.equal(slots[q, s], native[e])
            else:
                assert bool((slots[q, s] == 7).all())
    assert filled == o.replicas == plan.read_layer_stats(0)["replicas"] > 0


@pytest.mark.parametrize("grad_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("Wn", [3 * 7168 * 9, 1000, 8])
def test_reduce_grads_bit_exact(grad_dtype, Wn):
    # small experts, same routing as dsv3; 1000 and 8 leave a lone 8-element
    # vector at the end of each expert (Wn % 16 == 8)
    w = get_config("dsv3")
    ids = topk_ids(w)
    plan = gpu_plan(w, ids, expert_weight_elems=Wn)
    rng = np.random.default_rng(3)
    g32 = (rng.standard_normal((w.R, w.S, Wn)) * 1e-2).astype(np.float32)
    if grad_dtype == "bf16":
        g_np = (g32.view(np.uint32) >> 16).astype(np.uint16)
        g_t = torch.from_numpy(g_np.view(np.int16)).cuda().view(torch.bfloat16)
    else:
        g_np = g32
        g_t = torch.from_numpy(g32).cuda()
    nat_np = rng.standard_normal((w.E, Wn)).astype(np.float32)
    nat_t = torch.from_numpy(nat_np).cuda()
    plan.reduce_replica_grads(0, g_t, nat_t)
    torch.cuda.synchronize()
    o = oracle_plan(w, ids)
    want_nat = nat_np.copy()
    want_g = g_np.copy()
    oracle.reduce_grads(o, want_g, want_nat)
    got_nat = nat_t.cpu().numpy()
    np.testing.assert_array_equal(got_nat.view(np.uint32), want_nat.view(np.uint32))
    got_g = g_t.view(torch.int16).cpu().numpy().view(np.uint16) if grad_dtype == "bf16" else g_t.cpu().numpy()
    np.testing.assert_array_equal(got_g, want_g)


# ---- standalone Waterfill -------------------------------------------------------
@pytest.mark.parametrize("all_ranks", [False, True])
def test_waterfill_standalone_parity(all_ranks):
    rng = np.random.default_rng(77)
    for R, T, K in [(4, 1000, 2), (64, 4096, 8), (7, 333, 5), (128, 50, 16), (33, 100, 0)]:
        load = rng.integers(0, 5 * T, size=R).astype(np.int32)
        dst = rng.integers(-1, R, size=(R, T, max(K, 1))).astype(np.int32)[:, :, :K].copy()
        for seed, bonus in [(1, 10), (2**63 + 5, 0), (99, 500)]:
            pick, count = ep_waterfill(torch.from_numpy(load).cuda(), torch.from_numpy(dst).cuda(),
                                       seed=seed, bonus_permille=bonus, all_ranks=all_ranks)
            torch.cuda.synchronize()
            wp, wc = oracle.waterfill(load, dst, seed=seed, bonus_permille=bonus, all_ranks=all_ranks)
            np.testing.assert_array_equal(pick.cpu().numpy(), wp)
            np.testing.assert_array_equal(count.cpu().numpy(), wc)


def test_waterfill_hand_worked_draws_on_gpu():
    # the hand-worked picks of tests/golden/waterfill_worked_draws.json, drawn
    # by the device kernel (the expected values are the golden file's)
    import json
    import os

    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "waterfill_worked_draws.json")))
    load = np.array(g["load"], dtype=np.int32)
    for d in g["draws"]:
        dst = np.full((g["R"], g["T"], g["K"]), -1, np.int32)
        dst[d["r"], 0] = d["routes"]
        pick, _ = ep_waterfill(torch.from_numpy(load).cuda(), torch.from_numpy(dst).cuda(),
                               seed=int(d["seed"]), bonus_permille=d["bonus_permille"])
        torch.cuda.synchronize()
        assert int(pick.cpu().numpy()[d["r"], 0]) == d["pick"], d


@pytest.mark.parametrize("name,all_ranks,sampled", [
    ("dsv3", False, False), ("tiny", True, False), ("dsv3", False, True)])
def test_waterfill_layer_rerun_equals_a_fresh_balance(name, all_ranks, sampled):
    # a cached layer re-drawn with another seed equals the oracle's plan of the
    # same ids with that seed; another layer balanced in between (it rewrites
    # the plan's scratch) does not matter
    w0 = get_config(name).replace(shared_expert=True, waterfill_all_ranks=all_ranks,
                                  sampled_rerouting=sampled)
    ids = topk_ids(get_config(name))
    other = np.ascontiguousarray(ids[::-1])
    plan = Plan(config_from_workload(w0, num_layers=2))
    gpu_plan(w0, ids, plan=plan, layer=0)
    gpu_plan(w0, other, plan=plan, layer=1)
    for seed in (12345, 2**64 - 3):
        plan.waterfill_layer(0, seed)
        torch.cuda.synchronize()
        w1 = w0.replace(waterfill_seed=seed)
        compare_plan(fetch(plan, 0), oracle_plan(w1, ids), w1)
    compare_plan(fetch(plan, 1), oracle_plan(w0, other), w0)  # untouched
    plan.waterfill_layer(0, w0.waterfill_seed)  # back to the plan's own seed
    torch.cuda.synchronize()
    compare_plan(fetch(plan, 0), oracle_plan(w0, ids), w0)


def test_waterfill_layer_errors():
    w = get_config("tiny")
    plan = Plan(config_from_workload(w))
    with pytest.raises(EpError) as ei:
        plan.waterfill_layer(0, 1)
    assert ei.value.status == 2  # no shared expert
    ws = w.replace(shared_expert=True)
    plan = Plan(config_from_workload(ws, num_layers=2))
    with pytest.raises(EpError) as ei:
        plan.waterfill_layer(0, 1)
    assert ei.value.status == 5  # not balanced yet
    with pytest.raises(EpError) as ei:
        plan.waterfill_layer(2, 1)
    assert ei.value.status == 1


def test_plan_parity_waterfill_all_ranks():
    for name in ("dsv3", "tiny"):
        w = get_config(name).replace(shared_expert=True, waterfill_all_ranks=True)
        ids = topk_ids(get_config(name))
        o = oracle_plan(w, ids)
        compare_plan(fetch(gpu_plan(w, ids)), o, w)


# ---- errors are reported, not trapped --------------------------------------------
def test_errors_are_status_codes():
    w = get_config("tiny")
    with pytest.raises(EpError) as ei:
        Plan(config_from_workload(w.replace(R=129)))
    assert ei.value.status == 2
    plan = Plan(config_from_workload(w))
    with pytest.raises(EpError) as ei:
        plan.dispatch_layout(0, _hidden(w))
    assert ei.value.status == 5  # not planned yet
    ids = torch.from_numpy(topk_ids(w)).cuda()
    with pytest.raises(EpError) as ei:
        plan.balance_layer(1, ids)
    assert ei.value.status == 1
    plan.balance_layer(0, ids)
    with pytest.raises(EpError):
        plan.dispatch_layout(0, _hidden(w), rank_begin=3, rank_end=2)


def test_plans_of_different_shapes_coexist():
    # a plan with 14 KiB rows created before a plan with 512 B rows must still
    # launch its dispatch (per-kernel shared-memory limits are plan independent)
    wa = get_config("dsv3").replace(T=300)
    ida = topk_ids(get_config("dsv3"))[:, :300].copy()
    pa = gpu_plan(wa, ida)
    wb = get_config("tiny")
    pb = gpu_plan(wb, topk_ids(wb))
    ha = _hidden(wa)
    out = pa.dispatch_layout(0, ha)
    pb.dispatch_layout(0, _hidden(wb))
    torch.cuda.synchronize()
    dst = pa.view(0)["dst_row"].reshape(wa.N, wa.K).long()
    assert torch.equal(out[dst[:, 0]].view(torch.int16), ha.view(torch.int16))
    assert pa.read_layer_stats(0)["status"] == 0 and pb.read_layer_stats(0)["status"] == 0


# ---- combine (reverse of the dispatch) ------------------------------------------
def _combine_bound(x_bits, dst, w, srow):
    """sum over terms of |w x| (the scale of the fp32 rounding error)."""
    ax = (x_bits & 0x7FFF).astype(np.uint16)  # |x| in bf16 bits
    return oracle.combine_tokens(ax, dst, np.abs(w), srow)


@pytest.mark.parametrize("name,shared,out_dtype,sample", [
    ("tiny", False, "f32", None), ("tiny", True, "f32", None), ("tiny", True, "bf16", None),
    ("qwen", False, "bf16", 700), ("dsv3", True, "f32", 500)])
def test_combine_matches_oracle(name, shared, out_dtype, sample):
    w_cfg = get_config(name).replace(shared_expert=shared)
    ids = topk_ids(get_config(name))
    if name == "tiny":
        ids = ids.copy()
        ids[2, 5, 1] = -1  # a dropped id contributes nothing
    plan = gpu_plan(w_cfg, ids)
    rows = plan.read_layer_stats(0)["rows"]
    g = torch.Generator(device="cuda")
    g.manual_seed(21)
    x = torch.randn((rows, w_cfg.hidden), generator=g, device="cuda").to(torch.bfloat16)
    wts = torch.rand((w_cfg.R, w_cfg.T, w_cfg.K), generator=g, device="cuda")
    dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    y = plan.combine(0, x, wts, out_dtype=dt)
    torch.cuda.synchronize()
    # the rows each token's terms come from: the oracle's layout
    o = oracle_plan(w_cfg, ids)
    assert o.rows == rows
    N = w_cfg.N
    toks = np.arange(N) if sample is None else np.random.default_rng(5).choice(N, sample, replace=False)
    dst = o.dst_row.reshape(N, w_cfg.K)[toks]
    srow = None if not shared else o.shared_row.reshape(N)[toks]
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    wn = wts.reshape(N, w_cfg.K).cpu().numpy()[toks]
    want = oracle.combine_tokens(xb, dst, wn, srow)
    bound = _combine_bound(xb, dst, wn, srow)
    got = y.float().cpu().numpy()[toks].astype(np.float64)
    # fp32: K+1 rounded fma/add steps, each within 2^-24 of the running sum
    tol = 2.0**-20 * bound
    if out_dtype == "bf16":  # plus one round-to-nearest to 8 significant bits
        tol = tol + 2.0**-8 * np.abs(want)
    assert (np.abs(got - want) <= tol + 1e-30).all(), float(np.max(np.abs(got - want) - tol))
