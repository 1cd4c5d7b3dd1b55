"""B200 expert-balance library: Python binding of libep_b200.so.

The functions here carry the C ABI's names and only marshal arguments: torch
CUDA tensors are passed as raw device pointers, the current torch stream as the
cudaStream_t.  Every step of the path runs in the library's CUDA kernels; if
the library is not built, importing the entry points raises (no fallback).

    plan = Plan(config_from_workload(get_config("qwen")))
    plan.balance_layer(0, ids)                  # ep_balance_layer
    out = plan.dispatch_layout(0, hidden)       # ep_dispatch_layout
    plan.dispatch_tokens(0, hidden, out, 0, n)  # ep_dispatch_tokens (source-token range)
    plan.stage_replicas(0, native_w, slots)     # ep_stage_replicas
    plan.reduce_replica_grads(0, g_slots, g_native)
    plan.waterfill_layer(0, seed)               # ep_waterfill_layer (shared expert)
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _abi
from ._abi import (EP_DEV_BAD_ID, EP_DEV_ITER_CAP, EP_DEV_OUT_CAPACITY, EP_DEV_WAIT_TIMEOUT,
                   EP_ERR_DEVICE_STATUS, EP_OK, STOP_NAMES, EpConfig, LibraryMissing)

__all__ = [
    "EpConfig", "EpError", "LibraryMissing", "Plan", "config_from_workload",
    "ep_plan_workspace_bytes", "ep_waterfill", "ep_status_string", "ep_abi_version",
    "STOP_NAMES", "EP_DEV_BAD_ID", "EP_DEV_ITER_CAP", "EP_DEV_WAIT_TIMEOUT", "EP_DEV_OUT_CAPACITY",
]


class EpError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {ep_status_string(status)} ({status})")


def _check(fn: str, status: int) -> None:
    if status != EP_OK:
        raise EpError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def ep_status_string(status: int) -> str:
    return _abi.load().ep_status_string(status).decode()


def ep_abi_version() -> int:
    return int(_abi.load().ep_abi_version())


def config_from_workload(w, num_layers: Optional[int] = None, **overrides) -> EpConfig:
    """ep_config for a workloads.WorkloadConfig (sizes only; no arithmetic)."""
    c = EpConfig(
        num_ranks=w.R, num_experts=w.E, top_k=w.K, tokens_per_rank=w.T,
        slots_per_rank=w.S, min_replica_quota=w.m, hidden=w.hidden,
        num_layers=num_layers if num_layers is not None else w.layers,
        num_cap_candidates=w.J, shared_expert=int(bool(w.shared_expert)),
        waterfill_bonus_permille=w.waterfill_bonus_permille,
        waterfill_all_ranks=int(getattr(w, "waterfill_all_ranks", False)),
        expert_weight_elems=w.expert_elems, waterfill_seed=w.waterfill_seed,
        sampling_seed=getattr(w, "sampling_seed", 0),
        rerouting_mode=1 if getattr(w, "sampled_rerouting", False) else 0,
    )
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def ep_plan_workspace_bytes(cfg: EpConfig) -> int:
    n = ctypes.c_size_t()
    _check("ep_plan_workspace_bytes", _abi.load().ep_plan_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)))
    return int(n.value)


class Plan:
    """Owns the device workspace (a torch uint8 tensor) and the ep_plan handle."""

    def __init__(self, cfg: EpConfig, device: Optional[torch.device] = None):
        self.lib = _abi.load()
        self.cfg = cfg
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        nbytes = ep_plan_workspace_bytes(cfg)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
            base = self.workspace.data_ptr()
            self._ws_off = (-base) % 256
            handle = ctypes.c_void_p()
            _check("ep_plan_create", self.lib.ep_plan_create(
                ctypes.byref(cfg), ctypes.c_void_p(base + self._ws_off), nbytes, ctypes.byref(handle)))
        self.handle = handle
        self.R, self.E, self.K, self.T = cfg.num_ranks, cfg.num_experts, cfg.top_k, cfg.tokens_per_rank
        self.S, self.J = cfg.slots_per_rank, cfg.num_cap_candidates
        self.shared = bool(cfg.shared_expert)

    def close(self) -> None:
        if getattr(self, "handle", None):
            self.lib.ep_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover - interpreter shutdown order varies
        try:
            self.close()
        except Exception:
            pass

    # -- entry points --------------------------------------------------------
    def balance_layer(self, layer: int, topk_ids: torch.Tensor, stream=None) -> None:
        """ep_balance_layer: topk_ids int32 [R][T][K] on the plan's device."""
        if topk_ids.dtype != torch.int32 or tuple(topk_ids.shape) != (self.R, self.T, self.K):
            raise ValueError(f"topk_ids must be int32 [{self.R}, {self.T}, {self.K}]")
        _check("ep_balance_layer", self.lib.ep_balance_layer(self.handle, layer, _ptr(topk_ids), _stream(stream)))

    def read_layer_stats(self, layer: int, stream=None, raise_on_status: bool = False) -> dict:
        """ep_read_layer_stats (synchronises the stream)."""
        st = _abi.EpLayerStats()
        rc = self.lib.ep_read_layer_stats(self.handle, layer, ctypes.byref(st), _stream(stream))
        if rc not in (EP_OK, EP_ERR_DEVICE_STATUS) or (raise_on_status and rc != EP_OK):
            raise EpError("ep_read_layer_stats", rc)
        return {f: getattr(st, f) for f, _ in _abi.EpLayerStats._fields_}

    def view(self, layer: int) -> dict:
        """ep_layer_view_get, returned as int32 tensors aliasing the workspace."""
        v = _abi.EpLayerView()
        _check("ep_layer_view_get", self.lib.ep_layer_view_get(self.handle, layer, ctypes.byref(v)))
        R, E, T, K, G, S, J = self.R, self.E, self.T, self.K, v.G, self.S, self.J
        shapes = {
            "load": (R, E), "expert_total": (E,), "rank_load_before": (R,), "rank_load": (R,),
            "inst_expert": (R, G), "inst_quota": (R, G), "inst_off": (R * G + 1,),
            "rank_row_begin": (R + 1,), "dst_row": (R, T, K), "shared_rank": (R, T),
            "shared_row": (R, T), "cand_max_load": (J,), "cand_replicas": (J,), "cand_stop": (J,),
            "replica_list": (R * S,), "replica_expert_ptr": (E + 1,), "inst_count": (R, G),
        }
        base = self.workspace.data_ptr()
        out = {"G": v.G, "Gmax": v.Gmax}
        for name, shape in shapes.items():
            p = getattr(v, name)
            if not p:
                out[name] = None
                continue
            off = p - base
            n = 1
            for s in shape:
                n *= s
            out[name] = self.workspace[off:off + 4 * n].view(torch.int32).view(shape)
        return out

    def waterfill_layer(self, layer: int, seed: int, stream=None) -> None:
        """ep_waterfill_layer: re-draw the layer's shared-expert ranks with `seed`."""
        _check("ep_waterfill_layer", self.lib.ep_waterfill_layer(
            self.handle, layer, ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), _stream(stream)))

    def dispatch_layout(self, layer: int, hidden: torch.Tensor, out: Optional[torch.Tensor] = None,
                        rank_begin: int = 0, rank_end: Optional[int] = None, out_rows: Optional[int] = None,
                        stream=None) -> torch.Tensor:
        """ep_dispatch_layout: rows of destination ranks [rank_begin, rank_end)."""
        rank_end = self.R if rank_end is None else rank_end
        if out is None:
            if out_rows is None:
                out_rows = self.R * self.T * (self.K + (1 if self.shared else 0))
            out = torch.empty((out_rows, hidden.shape[1]), dtype=hidden.dtype, device=hidden.device)
        _check("ep_dispatch_layout", self.lib.ep_dispatch_layout(
            self.handle, layer, _ptr(hidden), _ptr(out), out.shape[0], rank_begin, rank_end, _stream(stream)))
        return out

    def dispatch_tokens(self, layer: int, hidden: torch.Tensor, out: torch.Tensor, token_begin: int,
                        token_end: int, stream=None) -> torch.Tensor:
        """ep_dispatch_tokens: every dispatch row of source tokens [token_begin, token_end)."""
        _check("ep_dispatch_tokens", self.lib.ep_dispatch_tokens(
            self.handle, layer, _ptr(hidden), token_begin, token_end, _ptr(out), out.shape[0],
            _stream(stream)))
        return out

    def combine(self, layer: int, expert_out: torch.Tensor, weights: torch.Tensor,
                out: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
        """ep_combine: gate-weighted sum of each token's dispatch rows (+ shared row)."""
        if weights.dtype != torch.float32 or tuple(weights.shape) != (self.R, self.T, self.K):
            raise ValueError(f"weights must be float32 [{self.R}, {self.T}, {self.K}]")
        out = _combine_out(self, expert_out, out, out_dtype)
        if out.dtype == torch.bfloat16:
            dt = 0
        elif out.dtype == torch.float32:
            dt = 1
        else:
            raise ValueError("out must be bfloat16 or float32")
        _check("ep_combine", self.lib.ep_combine(
            self.handle, layer, _ptr(expert_out), _ptr(weights), _ptr(out), dt, _stream(stream)))
        return out

    def stage_replicas(self, layer: int, native_w: torch.Tensor, slots: torch.Tensor, stream=None) -> None:
        """ep_stage_replicas: native_w bf16 [E][Wn] -> slots bf16 [R][S][Wn]."""
        _check("ep_stage_replicas", self.lib.ep_stage_replicas(
            self.handle, layer, _ptr(native_w), _ptr(slots), _stream(stream)))

    def reduce_replica_grads(self, layer: int, slot_grads: torch.Tensor, native_grads: torch.Tensor,
                             stream=None) -> None:
        """ep_reduce_replica_grads: slot_grads bf16/fp32 [R][S][Wn] into native_grads fp32 [E][Wn]."""
        if native_grads.dtype != torch.float32:
            raise ValueError("native_grads must be float32")
        if slot_grads.dtype == torch.bfloat16:
            dt = 0
        elif slot_grads.dtype == torch.float32:
            dt = 1
        else:
            raise ValueError("slot_grads must be bfloat16 or float32")
        _check("ep_reduce_replica_grads", self.lib.ep_reduce_replica_grads(
            self.handle, layer, _ptr(slot_grads), dt, _ptr(native_grads), _stream(stream)))


def _combine_out(plan, expert_out, out, out_dtype):
    if out is None:
        out = torch.empty((plan.R * plan.T, expert_out.shape[1]), dtype=out_dtype, device=expert_out.device)
    return out


def ep_waterfill(load: torch.Tensor, dst_rank: torch.Tensor, seed: int, bonus_permille: int = 10,
                 all_ranks: bool = False, stream=None):
    """Standalone Waterfill: load int32 [R], dst_rank int32 [R][T][K] -> (pick [R][T], count [R])."""
    R, T, K = dst_rank.shape
    pick = torch.empty((R, T), dtype=torch.int32, device=dst_rank.device)
    count = torch.empty((R,), dtype=torch.int32, device=dst_rank.device)
    _check("ep_waterfill", _abi.load().ep_waterfill(
        R, T, K, _ptr(load), _ptr(dst_rank), ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), bonus_permille,
        1 if all_ranks else 0, _ptr(pick), _ptr(count), _stream(stream)))
    return pick, count
