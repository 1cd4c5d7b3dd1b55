"""ep_load_matrix_static: the load matrix for callers that cannot allocate.

Serving engines that reserve nearly all device memory up front, embedded C
callers without an allocator, and loops where an allocation would synchronise
the device cannot use an entry point that needs a caller-allocated workspace.
ep_load_matrix_static keeps its scratch in a fixed device array inside the
library instead.  These tests call it through the C ABI and check it against
the load matrix the existing entry point (ep_balance_layer) produces, on two
calls in a row, so that contents left in the shared array by one call cannot
leak into the next.  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from moe_expert_load_b200 import _abi
from workloads import get_config, topk_ids

MAX_SCRATCH = 1 << 20  # EP_LOAD_STATIC_MAX_SCRATCH in include/ep_balance.h


def _fn():
    lib = _abi.load()
    f = lib.ep_load_matrix_static
    f.restype = ctypes.c_int32
    f.argtypes = [ctypes.c_int32] * 4 + [ctypes.c_void_p] * 3 + [ctypes.c_void_p]
    return f


def _static_load(ids: torch.Tensor, E: int):
    R, T, K = ids.shape
    load = torch.full((R, E), -1, dtype=torch.int32, device=ids.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=ids.device)
    rc = _fn()(R, E, K, T, ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(load.data_ptr()),
               ctypes.c_void_p(status.data_ptr()),
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, rc
    return load, status


def _existing_load(w, ids: torch.Tensor):
    from moe_expert_load_b200 import Plan, config_from_workload

    plan = Plan(config_from_workload(w, num_layers=1))
    plan.balance_layer(0, ids)
    return plan.view(0)["load"].clone()


@pytest.mark.gpu
def test_static_load_matrix_matches_balance_layer_twice():
    cases = []
    for name in ("qwen", "dsv3"):
        w = get_config(name)
        ids = topk_ids(w)
        if name == "dsv3":  # second call: other shape, two ids out of range
            ids = ids.copy()
            ids[1, 2, 3] = w.E
            ids[60, 4000, 0] = -3
        cases.append((w, torch.from_numpy(ids).cuda()))
    results = [_static_load(ids, w.E) for w, ids in cases]  # two calls in a row
    torch.cuda.synchronize()
    for (w, ids), (load, status) in zip(cases, results):
        want = _existing_load(w, ids)
        torch.cuda.synchronize()
        assert torch.equal(load, want)
        bad = int(((ids < 0) | (ids >= w.E)).any())
        assert int(status.item()) == bad
    # the counts themselves: one bincount per source rank
    w, ids = cases[0]
    ref = np.stack([np.bincount(r.ravel(), minlength=w.E) for r in ids.cpu().numpy()])
    np.testing.assert_array_equal(results[0][0].cpu().numpy(), ref)


@pytest.mark.gpu
def test_static_load_matrix_ragged_tail_and_empty():
    # T = 1000 leaves a partial last sub-chunk of 104 tokens and K = 3 makes
    # the ids of a sub-chunk end inside a 32-lane pass; T = 0 writes zeros
    rng = np.random.default_rng(17)
    R, E, K, T = 3, 40, 3, 1000
    ids_np = rng.integers(0, E, size=(R, T, K)).astype(np.int32)
    ids_np[2, 999, 2] = E + 1  # the very last id is out of range
    for _ in range(2):  # twice in a row on the shared array
        load, status = _static_load(torch.from_numpy(ids_np).cuda(), E)
        torch.cuda.synchronize()
        ref = np.stack([np.bincount(r.ravel()[r.ravel() < E], minlength=E) for r in ids_np])
        np.testing.assert_array_equal(load.cpu().numpy(), ref)
        assert int(status.item()) == 1
    empty = torch.empty((5, 0, 4), dtype=torch.int32, device="cuda")
    load, status = _static_load(empty, 16)
    torch.cuda.synchronize()
    assert not load.any() and int(status.item()) == 0


def test_static_load_matrix_rejects_shapes_beyond_its_scratch():
    f = _fn()
    w = get_config("stress")  # 72 * 128 * 256 sub-chunk counts > 2^20
    assert w.R * -(-w.T // 128) * w.E > MAX_SCRATCH
    assert f(w.R, w.E, w.K, w.T, None, None, None, None) == 2
    assert f(0, 8, 2, 10, None, None, None, None) == 1
    assert f(4, 8, 2, 10, None, None, None, None) == 1  # null pointers
    # with T = 0 the scratch bound holds for any R, so R * E itself is bounded
    assert f(3_000_000, 1024, 2, 0, None, None, None, None) == 2
