"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties the oracle to a value or property fixed by the pages or by
mathematics: hand-worked cases (tests/golden), numpy routines, brute force,
closed forms and invariants.  No expected value here comes from the CUDA path.
"""
import json
import os

import numpy as np
import pytest

import oracle
from tests.bruteforce import brute_force_opt, native_home
from tests.invariants import check_plan
from workloads import get_config, topk_ids

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _plan_cfg(cfg, ids, **kw):
    args = dict(E=cfg.E, S=cfg.S, m=cfg.m, J=cfg.J, shared_expert=cfg.shared_expert,
                seed=cfg.waterfill_seed, bonus_permille=cfg.waterfill_bonus_permille)
    args.update(kw)
    return oracle.plan(ids, **args)


def _check(p, ids, E, S, m):
    return check_plan(ids, E, S, m, Gmax=p.Gmax, G=p.G, W=p.W, inst_expert=p.inst_expert,
                      inst_quota=p.inst_quota, inst_off=p.inst_off, dst_row=p.dst_row,
                      cap=p.cap, stop=p.stop_name, shared_rank=p.shared_rank,
                      shared_row=p.shared_row)


# ---- load matrix: numpy bincount ------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "qwen"])
def test_load_matrix_is_bincount(name):
    cfg = get_config(name)
    ids = topk_ids(cfg)
    L, bad = oracle.load_matrix(ids, cfg.E)
    assert bad == 0
    for r in range(cfg.R):
        assert (L[r] == np.bincount(ids[r].ravel(), minlength=cfg.E)).all()


def test_load_matrix_skips_bad_ids():
    rng = np.random.default_rng(3)
    ids = rng.integers(-2, 10, size=(3, 17, 3)).astype(np.int32)
    L, bad = oracle.load_matrix(ids, 8)
    ok = (ids >= 0) & (ids < 8)
    assert bad == int((~ok).sum())
    for r in range(3):
        assert (L[r] == np.bincount(ids[r][ok[r]], minlength=8)).all()


# ---- hand-worked cases ------------------------------------------------------
@pytest.mark.parametrize("case", _golden("quota_worked_examples.json")["cases"],
                         ids=lambda c: c["name"])
def test_worked_examples(case):
    ids = np.array(case["ids"], dtype=np.int32).reshape(case["R"], case["T"], case["K"])
    p = oracle.plan(ids, E=case["E"], S=case["S"], m=case["m"], J=case["J"])
    x = case["expect"]
    assert p.Tot.tolist() == x["Tot"]
    assert p.W0.tolist() == x["W0"]
    assert p.W.tolist() == x["W"]
    assert p.cap_idx == x["cap_idx"] and p.cap == x["cap"]
    assert p.replicas == x["replicas"]
    assert p.stop_name == x["stop"]
    assert p.inst_expert.tolist() == x["inst_expert"]
    assert p.inst_quota.tolist() == x["inst_quota"]
    if "inst_off" in x:
        assert p.inst_off.tolist() == x["inst_off"]
    if "dst_row" in x:
        assert p.dst_row.reshape(case["R"], -1).tolist() == x["dst_row"]
    if "cand_maxW_prefix" in x:
        n = len(x["cand_maxW_prefix"])
        assert p.cand_maxW[:n].tolist() == x["cand_maxW_prefix"]
        assert [oracle.STOP_NAMES[s] for s in p.cand_stop[:n]] == x["cand_stop_prefix"]
    _check(p, ids, case["E"], case["S"], case["m"])


def test_waterline_closed_form():
    for c in _golden("waterfill_closed_form.json")["cases"]:
        H, B, slack = oracle.waterline(np.array(c["load"]), c["N"], bonus_permille=0)
        assert H == c["H"] and slack.tolist() == c["slack"] and B == 0


def test_waterline_bonus_rounds_up():
    # B = ceil(H * bonus / 1000): H = 6 with 10 permille -> 0.06 -> 1; 500 permille -> 3
    assert oracle.waterline(np.array([10, 2, 6, 0]), 6, 10)[1] == 1
    assert oracle.waterline(np.array([10, 2, 6, 0]), 6, 500)[1] == 3
    assert oracle.waterline(np.array([10, 2, 6, 0]), 6, 0)[1] == 0


def test_splitmix64_published_vector():
    g = _golden("splitmix64.json")
    gamma = 0x9E3779B97F4A7C15
    got = [oracle.splitmix64(g["seed"] + i * gamma) for i in range(len(g["outputs"]))]
    assert got == [int(v) for v in g["outputs"]]


def test_slot_sizing_matches_page():
    g = _golden("slot_sizing.json")
    cfg = get_config("qwen")
    assert cfg.hidden == g["hidden"] and cfg.ffn == g["ffn"]
    assert cfg.expert_elems * 2 == g["weight_bytes_per_slot"]
    assert cfg.expert_elems * 4 == g["fp32_grad_bytes_per_slot"]
    assert (cfg.expert_elems * 6) >> 20 == g["total_mib_per_slot"]
    total_gib = g["layers"] * cfg.expert_elems * 6 / 2**30
    assert abs(total_gib - g["per_layer_total_gib_approx"]) < 0.05
    assert get_config("sweep").layers == g["layers"]


# ---- brute force on tiny inputs ---------------------------------------------
def _random_tiny(rng):
    R = int(rng.integers(2, 5))
    E = int(rng.integers(R, 9))
    S = 1 if R == 4 else int(rng.integers(1, 3))
    if S == 2:
        E = min(E, 6)
    m = int(rng.choice([1, 2, 4]))
    A = int(rng.integers(4, 49))
    T = -(-A // R)
    p = rng.dirichlet(np.ones(E) * 0.3)
    ids = rng.choice(E, size=(R, T, 1), p=p).astype(np.int32)
    return ids, E, S, m


def test_bruteforce_bounds_the_greedy():
    rng = np.random.default_rng(11)
    gaps = []
    for _ in range(120):
        ids, E, S, m = _random_tiny(rng)
        R = ids.shape[0]
        p = oracle.plan(ids, E=E, S=S, m=m, J=16)
        _check(p, ids, E, S, m)
        opt = brute_force_opt(p.Tot.tolist(), R, S, m)
        assert p.after_max >= opt, "oracle reports a load below the exact optimum"
        assert p.after_max == p.W.max()
        lb = -(-p.A // R)
        assert opt >= lb
        gaps.append(p.after_max - opt)
    # the greedy is a heuristic; on these skewed micro loads it is exact most of the time
    assert np.mean(np.array(gaps) == 0) > 0.6


def test_greedy_exact_with_unit_minimum_and_ample_slots():
    # m = 1 and S >= E: every over-cap rank always finds a receiver with slack and a free
    # slot, so the first cap ceil(A/R) -- the exact optimum -- is reached.
    rng = np.random.default_rng(5)
    for _ in range(60):
        R = int(rng.integers(2, 6))
        E = int(rng.integers(R, 12))
        ids = rng.choice(E, size=(R, int(rng.integers(1, 40)), 2),
                         p=rng.dirichlet(np.ones(E) * 0.4)).astype(np.int32)
        p = oracle.plan(ids, E=E, S=E, m=1, J=4)
        _check(p, ids, E, E, 1)
        assert p.after_max == -(-p.A // R)
        assert p.stop_name == "BALANCED" and p.cap_idx == 0


def test_bruteforce_helper_on_known_case():
    # fig_ep4 loads with S=1, m=2: the optimum is ceil(36/4) = 9 (reached by the worked case)
    assert brute_force_opt([20, 4, 3, 3, 2, 2, 1, 1], 4, 1, 2) == 9
    # one hot expert, no slots: nothing can move
    assert brute_force_opt([9, 0, 0], 3, 0, 1) == 9
    assert native_home(8, 3) == [0, 0, 0, 1, 1, 1, 2, 2]


# ---- special cases ------------------------------------------------------------
def test_no_slots_is_stable_counting_sort():
    cfg = get_config("tiny")
    ids = topk_ids(cfg)
    p = oracle.plan(ids, E=cfg.E, S=0, m=cfg.m, J=cfg.J)
    assert p.replicas == 0 and (p.W == p.W0).all()
    # every expert has its native instance only; rows ordered by (expert, source, t, k)
    expect = np.empty(ids.size, np.int64)
    expect[np.argsort(ids.ravel(), kind="stable")] = np.arange(ids.size)
    assert (p.dst_row.ravel() == expect).all()


def test_no_slots_random_shapes():
    rng = np.random.default_rng(9)
    for _ in range(20):
        R = int(rng.integers(1, 7))
        E = int(rng.integers(1, 20))
        ids = rng.integers(0, E, size=(R, int(rng.integers(0, 30)), int(rng.integers(1, 5)))).astype(np.int32)
        p = oracle.plan(ids, E=E, S=0, m=3, J=3)
        expect = np.empty(ids.size, np.int64)
        # natives are contiguous blocks in expert order, so instance order = expert order
        expect[np.argsort(ids.ravel(), kind="stable")] = np.arange(ids.size)
        assert (p.dst_row.ravel() == expect).all()


def test_balanced_input_needs_no_replica():
    # every rank already at the mean: the first cap is met immediately
    R, E, T, K = 4, 8, 64, 2
    ids = np.tile(np.arange(E, dtype=np.int32), R * T * K // E).reshape(R, T, K)
    p = oracle.plan(ids, E=E, S=1, m=4, J=16)
    assert p.replicas == 0 and p.stop_name == "BALANCED" and p.cap_idx == 0
    assert (p.W == p.A // R).all()


def test_empty_input():
    ids = np.zeros((3, 0, 4), np.int32)
    p = oracle.plan(ids, E=6, S=1, m=2, J=4)
    assert p.A == 0 and p.rows == 0 and p.replicas == 0 and p.stop_name == "BALANCED"


def test_bad_ids_are_dropped_and_flagged():
    cfg = get_config("tiny")
    ids = topk_ids(cfg).copy()
    ids[0, 5, 1] = cfg.E
    ids[2, 7, 0] = -1
    p = _plan_cfg(cfg, ids)
    assert p.status & oracle.ST_BAD_ID
    assert p.A == ids.size - 2
    assert p.dst_row[0, 5, 1] == -1 and p.dst_row[2, 7, 0] == -1
    _check(p, ids, cfg.E, cfg.S, cfg.m)


def test_iteration_cap_never_hit():
    for name in ["tiny", "qwen", "dsv3"]:
        cfg = get_config(name)
        p = _plan_cfg(cfg, topk_ids(cfg))
        assert not (p.status & oracle.ST_ITER_CAP)
        assert (p.cand_stop != 3).all()


# ---- invariants at full size ---------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "qwen", "dsv3"])
def test_invariants_full_configs(name):
    cfg = get_config(name)
    ids = topk_ids(cfg)
    p = _plan_cfg(cfg, ids)
    _check(p, ids, cfg.E, cfg.S, cfg.m)
    assert p.rows == cfg.A + (cfg.N if cfg.shared_expert else 0)
    ratio = p.after_max * cfg.R / p.A
    assert ratio <= 1.05 or p.cand_stop[0] == 1, (name, ratio, p.stop_name)


def test_invariants_random_shapes():
    # 150 small random problems across the supported shape space: ragged E/R,
    # 0..8 slots, 1..16 experts per token (with and without repeats), every
    # minimum quota, shared expert in both candidate modes
    rng = np.random.default_rng(8080)
    for case in range(150):
        R = int(rng.integers(1, 13))
        E = int(rng.integers(1, min(32 * R, 200) + 1))
        K = int(rng.integers(1, min(E, 16) + 1))
        T = int(rng.integers(0, 160))
        S = int(rng.integers(0, 9))
        m = int(rng.choice([1, 2, 5, 20]))
        shared = bool(rng.integers(0, 2))
        all_ranks = bool(rng.integers(0, 2))
        p_e = rng.dirichlet(np.full(E, 0.3))
        if rng.integers(0, 2):  # distinct experts per token
            g = rng.gumbel(size=(R * T, E)) + np.log(p_e + 1e-12)
            ids = np.argsort(-g, axis=1)[:, :K].reshape(R, T, K).astype(np.int32)
        else:  # independent draws, repeats allowed
            ids = rng.choice(E, size=(R, T, K), p=p_e).astype(np.int32)
        p = oracle.plan(ids, E=E, S=S, m=m, J=16, shared_expert=shared, seed=case,
                        bonus_permille=10, all_ranks=all_ranks)
        check_plan(ids, E, S, m, Gmax=p.Gmax, G=p.G, W=p.W, inst_expert=p.inst_expert,
                   inst_quota=p.inst_quota, inst_off=p.inst_off, dst_row=p.dst_row, cap=p.cap,
                   stop=p.stop_name, shared_rank=p.shared_rank, shared_row=p.shared_row,
                   all_ranks=all_ranks)
        assert p.rows == R * T * K + (R * T if shared else 0)


@pytest.mark.slow
def test_invariants_stress():
    cfg = get_config("stress")
    ids = topk_ids(cfg)
    p = _plan_cfg(cfg, ids)
    _check(p, ids, cfg.E, cfg.S, cfg.m)
    assert p.before_max * cfg.R / p.A > 20
    assert p.after_max * cfg.R / p.A <= 1.05


def test_sweep_layers_sampled():
    cfg = get_config("sweep")
    for layer in (0, 3, 47, 93):
        ids = topk_ids(cfg, layer)
        p = _plan_cfg(cfg, ids)
        _check(p, ids, cfg.E, cfg.S, cfg.m)
        ratio = p.after_max * cfg.R / p.A
        assert ratio <= 1.05 or p.cand_stop[0] == 1, (layer, ratio)


# ---- Waterfill ------------------------------------------------------------------
def _dst_ranks(R, T, K, rng, p_none=0.0):
    d = rng.integers(0, R, size=(R, T, K)).astype(np.int32)
    d[rng.random((R, T, K)) < p_none] = -1
    return d


def test_waterfill_all_slack_on_one_candidate():
    # loads [50, 50, 50, 0], N = 8: H = ceil(158/4) = 40, slack only on rank 3; with no
    # local bonus every token whose candidates include rank 3 must pick it
    R, T, K = 4, 2, 2
    rng = np.random.default_rng(1)
    dst = _dst_ranks(R, T, K, rng)
    load = np.array([50, 50, 50, 0])
    pick, cnt = oracle.waterfill(load, dst, seed=7, bonus_permille=0)
    for r in range(R):
        for t in range(T):
            cands = {r} | set(dst[r, t].tolist())
            if 3 in cands:
                assert pick[r, t] == 3
            else:
                # fallback: least loaded candidate, own rank kept on ties (B = 0)
                assert pick[r, t] == r
    assert cnt.sum() == R * T


def test_waterfill_hand_worked_draws():
    # three picks worked by hand from the published SplitMix64 vector
    # (tests/golden/waterfill_worked_draws.json): a draw on an interval
    # boundary, the first of the other candidates, and the local preference
    g = json.load(open(os.path.join(GOLDEN, "waterfill_worked_draws.json")))
    load = np.array(g["load"])
    H, B0, slack = oracle.waterline(load, g["R"] * g["T"], 0)
    assert H == 8 and B0 == 0 and slack.tolist() == [0, 2, 6, 0]
    for d in g["draws"]:
        dst = np.full((g["R"], g["T"], g["K"]), -1, np.int32)
        dst[d["r"], 0] = d["routes"]
        pick, cnt = oracle.waterfill(load, dst, seed=int(d["seed"]), bonus_permille=d["bonus_permille"])
        assert int(pick[d["r"], 0]) == d["pick"], d
        assert cnt.sum() == g["R"] * g["T"]


def test_waterfill_fallback_prefers_clearly_lighter():
    # loads [12, 10, 10, 0] with N = 4: H = ceil(36/4) = 9, no slack on ranks 0..2.
    # Token on rank 0 visiting rank 1 only: candidates {0, 1}, min load 10 on rank 1.
    load = np.array([12, 10, 10, 0])
    dst = np.full((4, 1, 1), -1, np.int32)
    dst[0, 0, 0] = 1
    dst[1, 0, 0] = 2  # candidates {1, 2}: equal loads, keep own rank
    dst[2, 0, 0] = 3  # rank 3 has slack -> the slack draw
    # B = ceil(9 * 10 / 1000) = 1: 12 > 10 + 1, so rank 1 is clearly lighter
    pick, _ = oracle.waterfill(load, dst, seed=1, bonus_permille=10)
    assert pick[0, 0] == 1 and pick[1, 0] == 1
    # B = ceil(9 * 300 / 1000) = 3: 12 <= 10 + 3, keep the own rank
    pick, _ = oracle.waterfill(load, dst, seed=1, bonus_permille=300)
    assert pick[0, 0] == 0 and pick[1, 0] == 1
    # rank 3 has no load: a token on rank 3 with no routes picks itself by slack
    assert pick[3, 0] == 3


def test_waterfill_proportional_to_slack():
    # every rank-0 token has candidates {0, 1}; with no local bonus the share that picks
    # rank 0 must match slack_0 / (slack_0 + slack_1) within a 5-sigma binomial bound
    R, T = 2, 40000
    N = R * T
    load = np.array([N // 2 + 10, N // 2 - 10])  # H = N, slack = [N/2 - 10, N/2 + 10]
    H, B, slack = oracle.waterline(load, N, 0)
    assert H == N and B == 0 and slack.tolist() == [N // 2 - 10, N // 2 + 10]
    load = np.array([3 * N // 4, N // 4])  # slack 1 : 3
    H, B, slack = oracle.waterline(load, N, 0)
    assert slack[1] == 3 * slack[0]
    dst = np.zeros((R, T, 1), np.int32)
    dst[0, :, 0] = 1
    dst[1, :, 0] = 0
    pick, _ = oracle.waterfill(load, dst, seed=12345, bonus_permille=0)
    p0 = slack[0] / (slack[0] + slack[1])
    assert abs(float((pick[0] == 0).mean()) - p0) < 5 * np.sqrt(p0 * (1 - p0) / T)
    # the local bonus moves the split toward the own rank: (slack_0 + B) / (sum + B)
    pick_b, _ = oracle.waterfill(load, dst, seed=12345, bonus_permille=100)
    _, Bb, sb = oracle.waterline(load, N, 100)
    pb = (sb[0] + Bb) / (sb[0] + sb[1] + Bb)
    assert abs(float((pick_b[0] == 0).mean()) - pb) < 5 * np.sqrt(pb * (1 - pb) / T)


def test_waterfill_draw_is_per_token_and_deterministic():
    R, T, K = 3, 100, 3
    rng = np.random.default_rng(2)
    dst = _dst_ranks(R, T, K, rng, 0.2)
    load = np.array([30, 10, 5])
    a, ca = oracle.waterfill(load, dst, seed=99)
    b, cb = oracle.waterfill(load, dst, seed=99)
    assert (a == b).all() and (ca == cb).all()
    c, _ = oracle.waterfill(load, dst, seed=100)
    assert (a != c).any()
    # a token's pick depends on its own routes only: perturb another token
    dst2 = dst.copy()
    dst2[1, 50] = (dst2[1, 50] + 1) % R
    d, _ = oracle.waterfill(load, dst2, seed=99)
    mask = np.ones((R, T), bool)
    mask[1, 50] = False
    assert (a[mask] == d[mask]).all()


def test_waterfill_in_plan_matches_standalone():
    cfg = get_config("tiny").replace(shared_expert=True)
    ids = topk_ids(cfg)
    p = _plan_cfg(cfg, ids)
    dst_rank = np.where(p.dst_inst >= 0, p.dst_inst // p.G, -1).astype(np.int32)
    pick, cnt = oracle.waterfill(p.W, dst_rank, seed=cfg.waterfill_seed,
                                 bonus_permille=cfg.waterfill_bonus_permille)
    assert (pick == p.shared_rank).all()
    assert (cnt == p.inst_quota[:, -1]).all()
    _check(p, ids, cfg.E, cfg.S, cfg.m)


def test_waterfill_lowers_the_peak():
    # without redundant slots the routed load stays skewed; moving shared-expert work to
    # slack ranks must lower the worst rank below "shared expert always local"
    cfg = get_config("dsv3")
    ids = topk_ids(cfg)
    p = _plan_cfg(cfg, ids, S=0)
    total = p.W + p.inst_quota[:, -1]
    local_only = p.W + cfg.T
    assert total.max() < local_only.max()
    assert total.sum() == cfg.A + cfg.N
    H, _, slack = oracle.waterline(p.W, cfg.N, cfg.waterfill_bonus_permille)
    # ranks above the waterline only keep the shared work of their own tokens at most
    over = p.W >= H
    assert (p.inst_quota[over, -1] <= cfg.T).all()


# ---- permute, stage, gradient reduction ---------------------------------------
def test_permute_round_trip():
    cfg = get_config("tiny").replace(shared_expert=True)
    ids = topk_ids(cfg)
    p = _plan_cfg(cfg, ids)
    rng = np.random.default_rng(4)
    hidden = rng.integers(0, 2**16, size=(cfg.N, cfg.hidden), dtype=np.uint16)
    out = oracle.permute(p, hidden)
    d = p.dst_row.reshape(cfg.N, cfg.K)
    for k in range(cfg.K):
        assert (out[d[:, k]] == hidden).all()
    assert (out[p.shared_row.ravel()] == hidden).all()


def test_stage_copies_exact_bytes():
    cfg = get_config("tiny")
    p = _plan_cfg(cfg, topk_ids(cfg))
    elems = 1000
    rng = np.random.default_rng(6)
    w = rng.integers(0, 2**16, size=(cfg.E, elems), dtype=np.uint16)
    slots = np.full((cfg.R, cfg.S, elems), 0xBEEF, np.uint16)
    oracle.stage(p, w, slots)
    for q in range(cfg.R):
        for s in range(cfg.S):
            e = p.inst_expert[q, p.Gmax + s]
            if e >= 0:
                assert (slots[q, s] == w[e]).all()
            else:
                assert (slots[q, s] == 0xBEEF).all()


@pytest.mark.parametrize("grad_dtype", ["bf16", "f32"])
def test_reduce_grads_is_sequential_fp32_sum(grad_dtype):
    cfg = get_config("qwen")
    p = _plan_cfg(cfg, topk_ids(cfg))
    elems = 257
    rng = np.random.default_rng(8)
    g32 = (rng.standard_normal((cfg.R, cfg.S, elems)) * 1e-2).astype(np.float32)
    if grad_dtype == "bf16":
        g = (g32.view(np.uint32) >> 16).astype(np.uint16)
        gval = (g.astype(np.uint32) << 16).view(np.float32)
    else:
        g = g32.copy()
        gval = g32
    native = rng.standard_normal((cfg.E, elems)).astype(np.float32)
    expect = native.copy()
    for q in range(cfg.R):  # instance order
        for s in range(cfg.S):
            e = p.inst_expert[q, p.Gmax + s]
            if e >= 0:
                expect[e] = np.add(expect[e], gval[q, s], dtype=np.float32)
    got = native.copy()
    gg = g.copy()
    oracle.reduce_grads(p, gg, got)
    assert (got.view(np.uint32) == expect.view(np.uint32)).all()
    filled = p.inst_expert[:, p.Gmax:p.Gmax + p.S] >= 0
    assert (gg[filled] == 0).all()
    assert (gg[~filled] == g[~filled]).all()
    assert p.replicas > 0


# ---- combine (reverse of the dispatch) -------------------------------------------
def _bf16_bits(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((u + ((u >> 16) & 1) + 0x7FFF) >> 16).astype(np.uint16)


def _bits_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("shared", [False, True])
def test_combine_is_adjoint_of_dispatch(shared):
    # dispatching hidden rows and combining them back with gate weights w gives
    # (sum_k w_k + [shared]) * hidden exactly (each dispatch row is a copy)
    cfg = get_config("tiny").replace(shared_expert=shared)
    ids = topk_ids(cfg)
    p = _plan_cfg(cfg, ids)
    rng = np.random.default_rng(12)
    hidden = _bf16_bits(rng.standard_normal((cfg.N, cfg.hidden)))
    x = oracle.permute(p, hidden)
    w = rng.random((cfg.R, cfg.T, cfg.K)).astype(np.float32)
    y = oracle.combine(p, x, w)
    scale = w.reshape(cfg.N, cfg.K).astype(np.float64).sum(1) + (1.0 if shared else 0.0)
    np.testing.assert_allclose(y, scale[:, None] * _bits_f64(hidden), rtol=1e-14, atol=0)


def test_combine_is_linear_and_skips_dropped_rows():
    cfg = get_config("tiny")
    ids = topk_ids(cfg).copy()
    ids[1, 10, 0] = -1  # dropped id: its weight must not matter
    p = _plan_cfg(cfg, ids)
    rng = np.random.default_rng(13)
    xa = _bf16_bits(rng.standard_normal((p.rows, 16)))
    xb = _bf16_bits(rng.standard_normal((p.rows, 16)))
    w = rng.random((cfg.R, cfg.T, cfg.K)).astype(np.float32)
    ya, yb = oracle.combine(p, xa, w), oracle.combine(p, xb, w)
    # linear in the gate weights: doubling w doubles the output exactly
    np.testing.assert_array_equal(oracle.combine(p, xa, 2 * w), 2 * ya)
    w2 = w.copy()
    w2[1, 10, 0] = 1e6
    np.testing.assert_array_equal(oracle.combine(p, xa, w2), ya)
    # all-ones expert outputs: each token gets the sum of the weights of its valid ids
    ones = _bf16_bits(np.ones((p.rows, 16)))
    valid = (np.asarray(ids) >= 0).reshape(-1, cfg.K)
    expect = (w.reshape(-1, cfg.K).astype(np.float64) * valid).sum(1)
    np.testing.assert_allclose(oracle.combine(p, ones, w), np.repeat(expect[:, None], 16, 1), rtol=1e-14)
    # additive in the expert outputs (exact sums of small integers)
    xi = _bf16_bits(rng.integers(-8, 8, size=(p.rows, 16)).astype(np.float64))
    xj = _bf16_bits(rng.integers(-8, 8, size=(p.rows, 16)).astype(np.float64))
    xij = _bf16_bits(_bits_f64(xi) + _bits_f64(xj))
    wi = np.ones_like(w)
    np.testing.assert_array_equal(oracle.combine(p, xij, wi), oracle.combine(p, xi, wi) + oracle.combine(p, xj, wi))
    assert yb.shape == ya.shape


# ---- Waterfill all-rank mode ----------------------------------------------------
def test_waterfill_all_ranks_single_slack_rank():
    # only rank 3 has slack and there is no local bonus: in all-rank mode every
    # token picks it, whatever ranks it visits (conservative mode would not)
    R, T, K = 4, 50, 2
    dst = _dst_ranks(R, T, K, np.random.default_rng(3))
    load = np.array([500, 500, 500, 0])
    pick, cnt = oracle.waterfill(load, dst, seed=11, bonus_permille=0, all_ranks=True)
    assert (pick == 3).all() and cnt.tolist() == [0, 0, 0, R * T]
    pick_c, _ = oracle.waterfill(load, dst, seed=11, bonus_permille=0, all_ranks=False)
    assert (pick_c != 3).any()


def test_waterfill_all_ranks_proportional():
    # uniform-slack ranks except rank 0 (no slack): picks spread over ranks 1..3
    # in proportion to slack, within a 5-sigma binomial bound per rank
    R, T = 4, 30000
    load = np.array([5 * T, 0, T // 2, T])
    H, B, slack = oracle.waterline(load, R * T, 0)
    dst = np.full((R, T, 1), -1, np.int32)
    pick, _ = oracle.waterfill(load, dst, seed=4, bonus_permille=0, all_ranks=True)
    p = slack / slack.sum()
    n = R * T
    for q in range(R):
        f = float((pick == q).mean())
        assert abs(f - p[q]) <= 5 * np.sqrt(max(p[q] * (1 - p[q]), 1e-12) / n) + 1e-12
    assert p[0] == 0 and (pick == 0).sum() == 0


def test_waterfill_all_ranks_flattens_more():
    # more freedom than the conservative set: the worst rank (routed + shared)
    # is no higher, and the spread is tighter, on the dsv3 layer without slots
    cfg = get_config("dsv3")
    ids = topk_ids(cfg)
    pc = _plan_cfg(cfg, ids, S=0)
    pa = _plan_cfg(cfg, ids, S=0, all_ranks=True)
    tc = pc.W + pc.inst_quota[:, -1]
    ta = pa.W + pa.inst_quota[:, -1]
    assert ta.max() <= tc.max() and ta.std() < tc.std()
    check_plan(ids, cfg.E, 0, cfg.m, Gmax=pa.Gmax, G=pa.G, W=pa.W, inst_expert=pa.inst_expert,
               inst_quota=pa.inst_quota, inst_off=pa.inst_off, dst_row=pa.dst_row, cap=pa.cap,
               stop=pa.stop_name, shared_rank=pa.shared_rank, shared_row=pa.shared_row,
               all_ranks=True)


# ---- EPLB+ comparison baseline and LP cross-check ------------------------------
def test_eplb_plus_worked_example():
    g = _golden("quota_worked_examples.json")["eplb_plus_fig_ep4"]
    ie, iq, W, n = oracle.eplb_plus(np.array(g["Tot"]), g["R"], g["S"])
    assert ie.tolist() == g["inst_expert"] and iq.tolist() == g["inst_quota"]
    assert W.tolist() == g["W"] and n == g["replicas"]


@pytest.mark.parametrize("name", ["qwen", "dsv3"])
def test_eplb_plus_is_a_valid_round_robin_plan(name):
    cfg = get_config(name)
    p = _plan_cfg(cfg, topk_ids(cfg))
    ie, iq, W, n = oracle.eplb_plus(p.Tot, cfg.R, cfg.S)
    Gm = p.Gmax
    assert n == cfg.R * cfg.S  # EPLB-style: every redundant slot is used
    per_e = {}
    for q in range(cfg.R):
        held = [int(e) for e in ie[q] if e >= 0]
        assert len(held) == len(set(held))
        assert (ie[q, Gm:] >= 0).sum() <= cfg.S
        assert W[q] == iq[q].sum()
        for col in range(ie.shape[1]):
            if ie[q, col] >= 0:
                per_e.setdefault(int(ie[q, col]), []).append(int(iq[q, col]))
    for e, qs in per_e.items():
        assert sum(qs) == p.Tot[e]
        assert max(qs) - min(qs) <= 1 and qs == sorted(qs, reverse=True)  # round robin


def test_lp_bound_is_met_on_the_worked_case():
    from oracle.lplb import min_max_split

    case = _golden("quota_worked_examples.json")["cases"][0]
    ids = np.array(case["ids"], dtype=np.int32).reshape(case["R"], case["T"], case["K"])
    p = oracle.plan(ids, E=case["E"], S=case["S"], m=case["m"], J=case["J"])
    M, x = min_max_split(p.Tot, p.inst_expert, p.Gmax, p.S, m_replica=case["m"])
    assert abs(M - 9.0) < 1e-9 and p.after_max == 9


@pytest.mark.parametrize("name", ["tiny", "qwen", "dsv3"])
def test_greedy_split_is_never_below_the_lp_bound(name):
    # for the greedy's own placement, no split (LP relaxation, replicas >= m)
    # has a smaller worst rank; the greedy's split is feasible for that LP
    from oracle.lplb import min_max_split

    cfg = get_config(name)
    p = _plan_cfg(cfg, topk_ids(cfg))
    M, _ = min_max_split(p.Tot, p.inst_expert, p.Gmax, p.S, m_replica=cfg.m)
    assert p.after_max >= M - 1e-6
    assert p.after_max <= 1.06 * M  # and close to it on these workloads


# ---- sampling rerouting mode ("Waterfill and LPLB" page, section "LPLB") --------
def _fig_ep4():
    case = next(c for c in _golden("quota_worked_examples.json")["cases"] if c["name"] == "fig_ep4")
    return case, np.array(case["ids"], dtype=np.int32).reshape(case["R"], case["T"], case["K"])


def test_sampling_hand_worked_draws():
    g = _golden("sampling_worked_example.json")
    case, ids = _fig_ep4()
    for d in g["draws"]:
        p = oracle.plan(ids, E=case["E"], S=case["S"], m=case["m"], J=case["J"], sampling=True,
                        sampling_seed=int(d["seed"]))
        assert p.dst_inst[d["r"], d["t"], d["k"]] == d["instance"], d


def _sampled(cfg, ids, seed=77, **kw):
    return _plan_cfg(cfg, ids, sampling=True, sampling_seed=seed, **kw)


def _check_sampled(p, ids, E, S):
    from tests.invariants import check_sampled_rows

    check_sampled_rows(ids, E, Gmax=p.Gmax, G=p.G, S=S, inst_expert=p.inst_expert,
                       inst_quota=p.inst_quota, inst_count=p.inst_count, inst_off=p.inst_off,
                       dst_row=p.dst_row, shared_rank=p.shared_rank, shared_row=p.shared_row)


@pytest.mark.parametrize("name", ["tiny", "qwen", "dsv3"])
def test_sampling_keeps_the_solve_and_gives_valid_rows(name):
    cfg = get_config(name)
    ids = topk_ids(cfg)
    det = _plan_cfg(cfg, ids)
    p = _sampled(cfg, ids)
    # the solve is the same in both modes; only the token-to-instance step differs
    for f in ("L", "Tot", "W0", "W", "inst_expert", "cand_maxW", "cand_repl", "cand_stop"):
        np.testing.assert_array_equal(getattr(p, f), getattr(det, f), err_msg=f)
    sc = det.Gmax + det.S  # the shared column's quota depends on the routed ranks
    np.testing.assert_array_equal(p.inst_quota[:, :sc], det.inst_quota[:, :sc])
    assert (p.cap_idx, p.replicas, p.after_max, p.A) == (det.cap_idx, det.replicas, det.after_max, det.A)
    _check_sampled(p, ids, cfg.E, cfg.S)
    np.testing.assert_array_equal(det.inst_count, det.inst_quota)
    assert det.realized_max == det.after_max
    routed = p.inst_count[:, :sc].sum(axis=1)
    assert p.realized_max == routed.max()
    if p.replicas:  # the draws do move tokens off the deterministic rows
        assert (p.dst_inst != det.dst_inst).any()


def test_sampling_without_slots_is_the_counting_sort():
    # one instance per expert: no draw, rows in (expert, source, t, k) order
    rng = np.random.default_rng(12)
    for _ in range(10):
        R = int(rng.integers(1, 6))
        E = int(rng.integers(1, 16))
        ids = rng.integers(0, E, size=(R, int(rng.integers(0, 40)), int(rng.integers(1, 4)))).astype(np.int32)
        p = oracle.plan(ids, E=E, S=0, m=2, J=4, sampling=True, sampling_seed=5)
        expect = np.empty(ids.size, np.int64)
        expect[np.argsort(ids.ravel(), kind="stable")] = np.arange(ids.size)
        assert (p.dst_row.ravel() == expect).all()


def test_sampling_proportional_to_quota():
    # each replicated expert's tokens split over its instances in proportion
    # to the quotas: every realised count within 5 binomial sigma of its quota
    cfg = get_config("qwen")
    ids = topk_ids(cfg)
    p = _sampled(cfg, ids, seed=2026)
    checked = 0
    for e in range(cfg.E):
        cols = np.argwhere(p.inst_expert[:, :p.Gmax + cfg.S] == e)
        if len(cols) < 2:
            continue
        tot = int(p.Tot[e])
        for q, c in cols:
            pr = p.inst_quota[q, c] / tot
            sigma = np.sqrt(tot * pr * (1 - pr))
            assert abs(int(p.inst_count[q, c]) - int(p.inst_quota[q, c])) <= 5 * sigma + 1
            checked += 1
    assert checked > p.replicas  # every replica plus its native


def test_sampling_draw_depends_only_on_seed_and_assignment():
    cfg = get_config("tiny")
    ids = topk_ids(cfg)
    a = _sampled(cfg, ids, seed=3)
    b = _sampled(cfg, ids, seed=3)
    c = _sampled(cfg, ids, seed=4)
    np.testing.assert_array_equal(a.dst_row, b.dst_row)
    assert (a.dst_inst != c.dst_inst).any()
    # swap two tokens of one rank: loads, quotas and every other draw stay
    ids2 = ids.copy()
    ids2[1, [10, 700]] = ids2[1, [700, 10]]
    d = _sampled(cfg, ids2, seed=3)
    np.testing.assert_array_equal(d.inst_quota, a.inst_quota)
    keep = np.ones(ids.shape, bool)
    keep[1, [10, 700]] = False
    np.testing.assert_array_equal(d.dst_inst[keep], a.dst_inst[keep])


def test_sampling_random_shapes():
    rng = np.random.default_rng(31)
    for _ in range(40):
        R = int(rng.integers(1, 9))
        E = int(rng.integers(1, min(32 * R, 60) + 1))
        K = int(rng.integers(1, 6))
        T = int(rng.integers(0, 120))
        S = int(rng.integers(0, 4))
        shared = bool(rng.integers(0, 2))
        ids = rng.choice(E, size=(R, T, K), p=rng.dirichlet(np.full(E, 0.3))).astype(np.int32)
        if T and rng.integers(0, 2):
            ids[0, 0, 0] = E  # a dropped id
        p = oracle.plan(ids, E=E, S=S, m=int(rng.choice([1, 4])), J=8, shared_expert=shared,
                        sampling=True, sampling_seed=int(rng.integers(0, 2**63)))
        _check_sampled(p, ids, E, S)


# ---- the greedy's iteration bound ----------------------------------------------
def test_iteration_limit_stops_the_greedy_and_keeps_a_valid_plan():
    cfg = get_config("qwen")
    ids = topk_ids(cfg)
    full = _plan_cfg(cfg, ids)
    assert full.replicas >= 3
    p = _plan_cfg(cfg, ids, iter_limit=2)
    assert p.status & oracle.ST_ITER_CAP
    assert (p.cand_stop == 3).all()  # every candidate needed more than two moves
    assert (p.cand_repl <= 2).all()
    assert p.stop_name == "ITER_CAP"
    _check(p, ids, cfg.E, cfg.S, cfg.m)


@pytest.mark.parametrize("name", ["qwen", "dsv3"])
def test_quota_solve_alone_matches_the_plan(name):
    # the solve-latency comparison times the same solve the plan runs
    cfg = get_config(name)
    p = _plan_cfg(cfg, topk_ids(cfg))
    W, mx, rep = oracle.quota_solve(p.Tot, cfg.R, cfg.S, cfg.m, cfg.J)
    np.testing.assert_array_equal(W, p.W)
    assert (mx, rep) == (p.after_max, p.replicas)
