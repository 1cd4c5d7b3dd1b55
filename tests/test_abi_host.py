"""Host-side checks of the C ABI (no GPU work): the library loads, exports every
symbol include/*.h declares, and validates configurations on the host."""
import ctypes
import glob
import os
import re

import pytest

from moe_expert_load_b200 import (_abi, config_from_workload, ep_abi_version, ep_plan_workspace_bytes,
                                  ep_status_string)
from moe_expert_load_b200 import build as lib_build
from moe_expert_load_b200 import EpError
from workloads import CONFIGS, get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    lib_build.build()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"^EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", src, flags=re.M))
    return names


def test_every_declared_symbol_is_exported():
    declared = _declared()
    assert len(declared) >= 12
    lib = ctypes.CDLL(_abi.library_path())
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(_abi.EXPORTS)


def test_only_declared_symbols_are_exported():
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", _abi.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == _declared()


def test_abi_version_and_strings():
    assert ep_abi_version() == 2
    lib = _abi.load()
    assert lib.ep_status_string(2) == b"unsupported configuration"


def test_struct_sizes_match_header():
    # ep_config: 12 int32 + int64 + 2 uint64 + 2 int32; ep_layer_stats: 6 int32 + 5 int64
    assert ctypes.sizeof(_abi.EpConfig) == 80
    assert ctypes.sizeof(_abi.EpLayerStats) == 64


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_workspace_sizes(name):
    w = get_config(name)
    n = ep_plan_workspace_bytes(config_from_workload(w))
    # at least the per-layer dispatch rows, at most a few hundred MiB
    assert n >= 4 * w.A * w.layers
    assert n < 512 << 20


@pytest.mark.parametrize("field,value,code", [
    ("num_ranks", 129, 2), ("num_ranks", 0, 1), ("num_experts", 1025, 2), ("top_k", 17, 2),
    ("slots_per_rank", 9, 2), ("num_cap_candidates", 17, 2), ("hidden", 12, 2),
    ("expert_weight_elems", 12, 2), ("min_replica_quota", 0, 1), ("waterfill_all_ranks", 2, 1),
    ("waterfill_bonus_permille", 1001, 2), ("shared_expert", 2, 1), ("tokens_per_rank", -1, 1),
    ("rerouting_mode", 2, 1), ("solver_iter_limit", -1, 1),
])
def test_config_validation(field, value, code):
    c = config_from_workload(get_config("tiny"))
    setattr(c, field, value)
    with pytest.raises(EpError) as ei:
        ep_plan_workspace_bytes(c)
    assert ei.value.status == code


def test_reduction_index_limit():
    # (replica slots) x (16-element pairs per expert) must stay below 2^32
    c = config_from_workload(get_config("tiny"), num_ranks=128, slots_per_rank=8,
                             expert_weight_elems=1 << 26)
    with pytest.raises(EpError) as ei:
        ep_plan_workspace_bytes(c)
    assert ei.value.status == 2
    c.expert_weight_elems = (1 << 26) - 16
    assert ep_plan_workspace_bytes(c) > 0


def test_natives_per_rank_limit():
    c = config_from_workload(get_config("tiny"), num_experts=33 * 4)
    with pytest.raises(EpError):
        ep_plan_workspace_bytes(c)
    c = config_from_workload(get_config("tiny"), num_experts=32 * 4)
    assert ep_plan_workspace_bytes(c) > 0


def test_create_rejects_small_or_misaligned_workspace():
    lib = _abi.load()
    c = config_from_workload(get_config("tiny"))
    n = ep_plan_workspace_bytes(c)
    h = ctypes.c_void_p()
    # no CUDA call is reached: both checks happen before any device query
    assert lib.ep_plan_create(ctypes.byref(c), ctypes.c_void_p(256), n - 1, ctypes.byref(h)) == 4
    assert lib.ep_plan_create(ctypes.byref(c), ctypes.c_void_p(300), n, ctypes.byref(h)) == 1
    assert lib.ep_plan_create(ctypes.byref(c), None, n, ctypes.byref(h)) == 1


def test_product_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "moe_expert_load_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h")):
            assert "oracle" not in open(path).read().lower(), path


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "ep_balance.h"
int main(void) {
  ep_config c;
  memset(&c, 0, sizeof c);
  c.num_ranks = 4; c.num_experts = 8; c.top_k = 2; c.tokens_per_rank = 1024;
  c.slots_per_rank = 1; c.min_replica_quota = 64; c.hidden = 256; c.num_layers = 1;
  c.num_cap_candidates = 16; c.expert_weight_elems = 3 * 256 * 512;
  c.waterfill_bonus_permille = 10; c.waterfill_seed = 1;
  size_t n = 0;
  ep_status_t st = ep_plan_workspace_bytes(&c, &n);
  c.num_ranks = 0;
  size_t m = 0;
  ep_status_t bad = ep_plan_workspace_bytes(&c, &m);
  printf("%d %zu %d %s %d\n", (int)st, n, (int)bad, ep_status_string(bad), (int)ep_abi_version());
  return 0;
}
"""


def test_plain_c_caller_links_and_runs(tmp_path):
    # the boundary is a C ABI: a C99 program includes the header, links the
    # library and calls its host-only entry points (no GPU needed)
    import subprocess

    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(_abi.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lep_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    want = ep_plan_workspace_bytes(config_from_workload(get_config("tiny"), waterfill_seed=1))
    assert out[0] == "0" and int(out[1]) == want
    assert out[2] == "1" and " ".join(out[3:-1]) == ep_status_string(1)
    assert int(out[-1]) == ep_abi_version()
