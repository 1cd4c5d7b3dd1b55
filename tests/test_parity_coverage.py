"""The GPU parity cases reach the paths they exist to test.

The token assignment finds an assignment's row in one of three ways: the first
rerouting segment of its (source rank, expert), the second one, or, when the
source rank's demand spreads over three or more instances, a search of the
rerouting's segment list in global memory.  A (source rank, expert) pair's
segments are the runs of equal destination instances in its assignments'
(token, k) order, so the oracle's instance per assignment tells how many there
are.  These checks run the oracle alone (no GPU) on inputs that GPU parity
tests use, and fail if a case stops reaching the rare path."""
import numpy as np

from tests.gpu_helpers import oracle_plan
from workloads import get_config, topk_ids


def _max_segments(ids: np.ndarray, dst_inst: np.ndarray, E: int) -> int:
    R = ids.shape[0]
    best = 0
    for r in range(R):
        e = ids[r].reshape(-1)
        inst = dst_inst[r].reshape(-1)
        ok = (e >= 0) & (e < E)
        order = np.argsort(e[ok], kind="stable")  # (t, k) order within each expert
        es, ins = e[ok][order], inst[ok][order]
        if es.size == 0:
            continue
        new_run = np.ones(es.size, dtype=bool)
        new_run[1:] = (es[1:] != es[:-1]) | (ins[1:] != ins[:-1])
        runs = np.bincount(es[new_run], minlength=E)
        best = max(best, int(runs.max()))
    return best


def test_segment_runs_match_a_direct_count():
    # the vectorised count against a plain loop on a small case
    w = get_config("tiny")
    ids = topk_ids(w)
    o = oracle_plan(w, ids)
    best = 0
    for r in range(w.R):
        last = {}
        runs = {}
        for t in range(w.T):
            for k in range(w.K):
                e = int(ids[r, t, k])
                g = int(o.dst_inst[r, t, k])
                if last.get(e) != g:
                    runs[e] = runs.get(e, 0) + 1
                    last[e] = g
        best = max([best, *runs.values()])
    assert _max_segments(ids, o.dst_inst, w.E) == best


def test_full_stress_parity_reaches_a_third_segment():
    # test_plan_parity_full_configs[stress]: the hot expert's demand from one
    # source rank overlaps several of its instances
    w = get_config("stress")
    ids = topk_ids(w)
    o = oracle_plan(w, ids)
    assert _max_segments(ids, o.dst_inst, w.E) >= 3


def test_random_shape_parity_reaches_a_fourth_segment():
    # test_plan_parity_random_shapes: at least one case walks the global
    # segment list past the third segment
    from tests.test_gpu_parity import _random_case

    rng = np.random.default_rng(2024)
    best = 0
    for _ in range(40):
        R, E, K, T, S, m, shared, J, ids = _random_case(rng)
        w = get_config("tiny").replace(R=R, E=E, K=K, T=T, S=S, m=m, J=J, shared_expert=shared)
        best = max(best, _max_segments(ids, oracle_plan(w, ids).dst_inst, E))
    assert best >= 4
