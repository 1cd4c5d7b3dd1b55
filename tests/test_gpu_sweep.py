"""The 94-layer sweep through the plan cache, forward and backward, against
the oracle.

UltraEP page, section "Reusing the forward plan for weight restore and
gradient reduction": the backward pass walks the layers in reverse order and,
for each layer, re-stages the replica weights from that layer's cached forward
plan into the one set of redundant slots, reduces the replica gradients into
the native experts' gradients and clears the replica gradient buffer; section
"Shared redundant slots manage dynamic replicas": the slots are shared by all
layers.  Here every one of the 94 layers is balanced into one plan, each
cached plan is compared with the oracle after all layers ran, and the reverse
walk is compared byte for byte (staging) and bit for bit (fp32 reduction,
fixed order on both sides) with the oracle applied in the same order to host
copies of the same buffers.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_b200 import Plan, config_from_workload
from tests.gpu_helpers import compare_plan, fetch, oracle_plan
from workloads import get_config, topk_ids

pytestmark = pytest.mark.gpu

# small experts keep the walk cheap; % 16 == 8 exercises the reduction's tail
WN = 3 * 4096 * 2 + 8


def _all_layer_ids(w):
    with ThreadPoolExecutor(8) as ex:  # numpy releases the GIL in the samplers
        return list(ex.map(lambda l: topk_ids(w, l), range(w.layers)))


def test_sweep_forward_cache_and_backward_replay_match_oracle():
    w = get_config("sweep")
    assert w.layers == 94
    ids = _all_layer_ids(w)
    plan = Plan(config_from_workload(w, num_layers=w.layers, expert_weight_elems=WN))
    dev_ids = torch.empty((w.R, w.T, w.K), dtype=torch.int32, device="cuda")
    for l in range(w.layers):  # forward: one balance call per layer, one id buffer
        dev_ids.copy_(torch.from_numpy(ids[l]))
        plan.balance_layer(l, dev_ids)
    torch.cuda.synchronize()
    plans = [oracle_plan(w, ids[l]) for l in range(w.layers)]
    for l in range(w.layers):  # every cached layer still holds its own plan
        compare_plan(fetch(plan, l), plans[l], w)
    assert sum(p.replicas for p in plans) > w.layers  # the walk has work to do

    rng = np.random.default_rng(94)
    native = rng.integers(-30000, 30000, (w.E, WN)).astype(np.int16)
    native_t = torch.from_numpy(native).cuda()
    slots_host = np.full((w.R, w.S, WN), 5, np.int16)  # the one shared slot buffer
    slots_t = torch.from_numpy(slots_host.copy()).cuda()
    gnat_host = (rng.standard_normal((w.E, WN)) * 1e-3).astype(np.float32)
    gnat_t = torch.from_numpy(gnat_host.copy()).cuda()
    gslot_t = torch.empty((w.R, w.S, WN), dtype=torch.int16, device="cuda")
    for l in reversed(range(w.layers)):
        p = plans[l]
        # weight restore from the cached forward plan of layer l
        plan.stage_replicas(l, native_t.view(torch.bfloat16), slots_t.view(torch.bfloat16))
        oracle.stage(p, native, slots_host)
        # this layer's replica gradients (bf16 bits of N(0, 1e-2) samples)
        g32 = (rng.standard_normal((w.R, w.S, WN)) * 1e-2).astype(np.float32)
        g_host = (g32.view(np.uint32) >> 16).astype(np.uint16)
        gslot_t.copy_(torch.from_numpy(g_host.view(np.int16)))
        plan.reduce_replica_grads(l, gslot_t.view(torch.bfloat16), gnat_t)
        oracle.reduce_grads(p, g_host, gnat_host)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(slots_t.cpu().numpy(), slots_host, err_msg=f"layer {l}")
        np.testing.assert_array_equal(gslot_t.cpu().numpy().view(np.uint16), g_host,
                                      err_msg=f"layer {l}")
        np.testing.assert_array_equal(gnat_t.cpu().numpy().view(np.uint32),
                                      gnat_host.view(np.uint32), err_msg=f"layer {l}")
        # every filled slot's gradient is clear after the layer's reduction
        filled = p.inst_expert[:, p.Gmax:p.Gmax + w.S] >= 0
        assert not g_host[filled].any()
    for l in range(w.layers):
        assert plan.read_layer_stats(l)["status"] == 0
