"""ctypes mirror of include/ep_balance.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

from . import build as _build

EP_OK = 0
EP_ERR_INVALID_ARGUMENT = 1
EP_ERR_UNSUPPORTED = 2
EP_ERR_CUDA = 3
EP_ERR_WORKSPACE_TOO_SMALL = 4
EP_ERR_NOT_PLANNED = 5
EP_ERR_DEVICE_STATUS = 6

EP_DEV_BAD_ID = 1
EP_DEV_ITER_CAP = 2
EP_DEV_WAIT_TIMEOUT = 4
EP_DEV_OUT_CAPACITY = 8
EP_DEV_INCONSISTENT = 16

EP_REROUTE_LOCAL_FIRST = 0
EP_REROUTE_SAMPLED = 1

STOP_NAMES = {0: "BALANCED", 1: "SLOT_LIMITED", 2: "QUOTA_LIMITED", 3: "ITER_CAP"}

# Every entry point include/ep_balance.h declares.
EXPORTS = (
    "ep_plan_workspace_bytes", "ep_plan_create", "ep_plan_destroy", "ep_balance_layer",
    "ep_layer_view_get", "ep_read_layer_stats", "ep_dispatch_layout", "ep_stage_replicas",
    "ep_reduce_replica_grads", "ep_waterfill", "ep_status_string", "ep_abi_version",
    "ep_load_matrix_static", "ep_combine", "ep_dispatch_tokens", "ep_waterfill_layer",
)


class EpConfig(ctypes.Structure):
    _fields_ = [
        ("num_ranks", ctypes.c_int32), ("num_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("tokens_per_rank", ctypes.c_int32),
        ("slots_per_rank", ctypes.c_int32), ("min_replica_quota", ctypes.c_int32),
        ("hidden", ctypes.c_int32), ("num_layers", ctypes.c_int32),
        ("num_cap_candidates", ctypes.c_int32), ("shared_expert", ctypes.c_int32),
        ("waterfill_bonus_permille", ctypes.c_int32), ("waterfill_all_ranks", ctypes.c_int32),
        ("expert_weight_elems", ctypes.c_int64), ("waterfill_seed", ctypes.c_uint64),
        ("sampling_seed", ctypes.c_uint64), ("rerouting_mode", ctypes.c_int32),
        ("solver_iter_limit", ctypes.c_int32),
    ]


class EpLayerStats(ctypes.Structure):
    _fields_ = [
        ("status", ctypes.c_int32), ("cap_idx", ctypes.c_int32),
        ("stop_reason", ctypes.c_int32), ("tight_stop_reason", ctypes.c_int32),
        ("replicas", ctypes.c_int32), ("realized_max", ctypes.c_int32),
        ("cap", ctypes.c_int64), ("assignments", ctypes.c_int64), ("rows", ctypes.c_int64),
        ("before_max", ctypes.c_int64), ("after_max", ctypes.c_int64),
    ]


_VIEW_PTRS = (
    "load", "expert_total", "rank_load_before", "rank_load", "inst_expert", "inst_quota",
    "inst_off", "rank_row_begin", "dst_row", "shared_rank", "shared_row", "cand_max_load",
    "cand_replicas", "cand_stop", "replica_list", "replica_expert_ptr", "stats", "inst_count",
)


class EpLayerView(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _VIEW_PTRS] + [
        ("Gmax", ctypes.c_int32), ("G", ctypes.c_int32),
    ]


_lib = None


class LibraryMissing(RuntimeError):
    pass


def library_path() -> str:
    return _build.LIB


def load():
    """Load libep_b200.so; raise if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if not os.path.exists(path):
        raise LibraryMissing(
            f"{path} is missing: build it with `python -m moe_expert_load_b200.build` "
            "(this package has no CPU or Python fallback)")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I32 = ctypes.c_int32
    I64 = ctypes.c_int64
    S = ctypes.c_int32  # ep_status_t
    sig = {
        "ep_plan_workspace_bytes": (S, [ctypes.POINTER(EpConfig), ctypes.POINTER(ctypes.c_size_t)]),
        "ep_plan_create": (S, [ctypes.POINTER(EpConfig), P, ctypes.c_size_t, ctypes.POINTER(P)]),
        "ep_plan_destroy": (None, [P]),
        "ep_balance_layer": (S, [P, I32, P, P]),
        "ep_layer_view_get": (S, [P, I32, ctypes.POINTER(EpLayerView)]),
        "ep_read_layer_stats": (S, [P, I32, ctypes.POINTER(EpLayerStats), P]),
        "ep_dispatch_layout": (S, [P, I32, P, P, I64, I32, I32, P]),
        "ep_dispatch_tokens": (S, [P, I32, P, I64, I64, P, I64, P]),
        "ep_stage_replicas": (S, [P, I32, P, P, P]),
        "ep_reduce_replica_grads": (S, [P, I32, P, I32, P, P]),
        "ep_waterfill": (S, [I32, I32, I32, P, P, ctypes.c_uint64, I32, I32, P, P, P]),
        "ep_combine": (S, [P, I32, P, P, P, I32, P]),
        "ep_waterfill_layer": (S, [P, I32, ctypes.c_uint64, P]),
        "ep_status_string": (ctypes.c_char_p, [S]),
        "ep_abi_version": (I32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
