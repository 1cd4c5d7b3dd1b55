"""Shared helpers of the GPU tests: run the CUDA path through the C ABI and the
oracle on the same seeded input, and compare element by element."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_expert_load_b200 import Plan, config_from_workload


def oracle_plan(w, ids, **kw):
    args = dict(E=w.E, S=w.S, m=w.m, J=w.J, shared_expert=w.shared_expert,
                seed=w.waterfill_seed, bonus_permille=w.waterfill_bonus_permille,
                all_ranks=w.waterfill_all_ranks, sampling=w.sampled_rerouting,
                sampling_seed=w.sampling_seed)
    args.update(kw)
    return oracle.plan(ids, **args)


def gpu_plan(w, ids_np, layers=1, layer=0, plan=None, **cfg_overrides):
    if plan is None:
        plan = Plan(config_from_workload(w, num_layers=layers, **cfg_overrides))
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).cuda()
    plan.balance_layer(layer, ids)
    torch.cuda.synchronize()
    return plan


def fetch(plan, layer=0):
    v = plan.view(layer)
    out = {k: (t.cpu().numpy() if isinstance(t, torch.Tensor) else t) for k, t in v.items()}
    out["stats"] = plan.read_layer_stats(layer)
    return out


def compare_plan(g, o, w):
    """Element-by-element equality of every plan output (bit-exact, integers)."""
    R, T, K = o.R, o.T, o.K
    assert g["G"] == o.G and g["Gmax"] == o.Gmax
    np.testing.assert_array_equal(g["load"], o.L)
    np.testing.assert_array_equal(g["expert_total"], o.Tot)
    np.testing.assert_array_equal(g["rank_load_before"], o.W0)
    np.testing.assert_array_equal(g["rank_load"], o.W)
    np.testing.assert_array_equal(g["cand_max_load"], o.cand_maxW)
    np.testing.assert_array_equal(g["cand_replicas"], o.cand_repl)
    np.testing.assert_array_equal(g["cand_stop"], o.cand_stop)
    np.testing.assert_array_equal(g["inst_expert"], o.inst_expert)
    np.testing.assert_array_equal(g["inst_quota"], o.inst_quota)
    np.testing.assert_array_equal(g["inst_count"], o.inst_count)
    np.testing.assert_array_equal(g["inst_off"], o.inst_off)
    np.testing.assert_array_equal(g["dst_row"], o.dst_row)
    if o.shared_rank is not None:
        np.testing.assert_array_equal(g["shared_rank"], o.shared_rank)
        np.testing.assert_array_equal(g["shared_row"], o.shared_row)
    # rank blocks: first row of each destination rank
    G = o.G
    np.testing.assert_array_equal(g["rank_row_begin"], o.inst_off[np.arange(R + 1) * G])
    st = g["stats"]
    assert st["cap_idx"] == o.cap_idx
    assert st["cap"] == o.cap
    assert st["stop_reason"] == o.stop_reason
    assert st["tight_stop_reason"] == o.cand_stop[0]
    assert st["replicas"] == o.replicas
    assert st["assignments"] == o.A
    assert st["rows"] == o.rows
    assert st["before_max"] == o.before_max
    assert st["after_max"] == o.after_max
    assert st["realized_max"] == o.realized_max
    # replica lists grouped by expert, instance order inside an expert
    S, Gm = o.S, o.Gmax
    ptr = g["replica_expert_ptr"]
    lst = g["replica_list"]
    for e in range(o.E):
        want = [q * S + s for q in range(R) for s in range(S) if o.inst_expert[q, Gm + s] == e]
        assert lst[ptr[e]:ptr[e + 1]].tolist() == want
    bad = int(((o.status & oracle.ST_BAD_ID) != 0))
    assert (st["status"] & 1) == bad
