"""CPU oracle of the UltraEP-style balance + dispatch plan (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (``moe_expert_load_b200``)
never does, and this package never imports the product.  The arithmetic lives
in ``ep_oracle.c`` (plain single-threaded C, compiled by ``oracle/build.py``);
this module only marshals numpy arrays.

Pinned by the ``-m "not gpu"`` tests against: numpy bincount (load matrix),
hand-worked cases (quota solve, rerouting, Waterfill closed form), brute-force
min-max enumeration on tiny inputs, the stable counting sort that rerouting
reduces to with no redundant slots, published SplitMix64 outputs, invariants
(quota conservation, cap, slot and uniqueness constraints, bijection,
round trip) and a numpy float32 sequential sum for the gradient reduction.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import numpy as np

from . import build as _build

STOP_NAMES = {0: "BALANCED", 1: "SLOT_LIMITED", 2: "QUOTA_LIMITED", 3: "ITER_CAP"}
ST_BAD_ID = 1
ST_ITER_CAP = 2


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("R", ctypes.c_int32), ("E", ctypes.c_int32), ("K", ctypes.c_int32), ("T", ctypes.c_int32),
        ("S", ctypes.c_int32), ("m", ctypes.c_int32), ("J", ctypes.c_int32),
        ("shared_expert", ctypes.c_int32), ("bonus_permille", ctypes.c_int32),
        ("all_ranks", ctypes.c_int32), ("seed", ctypes.c_uint64),
        ("sampling", ctypes.c_int32), ("iter_limit", ctypes.c_int32),
        ("sampling_seed", ctypes.c_uint64),
    ]


class _Stats(ctypes.Structure):
    _fields_ = [
        ("Gmax", ctypes.c_int32), ("G", ctypes.c_int32), ("cap_idx", ctypes.c_int32),
        ("stop_reason", ctypes.c_int32), ("cap", ctypes.c_int64), ("A", ctypes.c_int64),
        ("before_max", ctypes.c_int64), ("after_max", ctypes.c_int64),
        ("replicas", ctypes.c_int32), ("status", ctypes.c_int32), ("rows", ctypes.c_int64),
        ("realized_max", ctypes.c_int64),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        P = ctypes.c_void_p
        lib.orc_plan.argtypes = [ctypes.POINTER(_Cfg), P] + [P] * 15 + [ctypes.POINTER(_Stats)]
        lib.orc_plan.restype = ctypes.c_int
        lib.orc_load_matrix.argtypes = [ctypes.c_int32] * 4 + [P, P]
        lib.orc_load_matrix.restype = ctypes.c_int64
        lib.orc_splitmix64.argtypes = [ctypes.c_uint64]
        lib.orc_splitmix64.restype = ctypes.c_uint64
        lib.orc_gmax.argtypes = [ctypes.c_int32, ctypes.c_int32]
        lib.orc_gmax.restype = ctypes.c_int32
        lib.orc_waterline.argtypes = [ctypes.c_int32, ctypes.c_int64, P, ctypes.c_int32, P, P, P]
        lib.orc_waterline.restype = None
        lib.orc_waterfill.argtypes = [ctypes.c_int32] * 3 + [P, P, ctypes.c_uint64, ctypes.c_int32,
                                                             ctypes.c_int32, P, P]
        lib.orc_waterfill.restype = ctypes.c_int
        lib.orc_permute.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int64, P, P, P, P]
        lib.orc_permute.restype = None
        lib.orc_combine.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, P, P, P, P, P]
        lib.orc_combine.restype = None
        lib.orc_quota_solve.argtypes = [ctypes.c_int32] * 5 + [P, P, P]
        lib.orc_quota_solve.restype = ctypes.c_int32
        lib.orc_eplb_plus.argtypes = [ctypes.c_int32] * 3 + [P, P, P, P]
        lib.orc_eplb_plus.restype = ctypes.c_int32
        lib.orc_stage.argtypes = [ctypes.c_int32] * 4 + [P, ctypes.c_int64, P, P]
        lib.orc_stage.restype = None
        lib.orc_reduce_grads.argtypes = [ctypes.c_int32] * 4 + [P, ctypes.c_int64, ctypes.c_int32, P, P]
        lib.orc_reduce_grads.restype = None
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


@dataclasses.dataclass
class Plan:
    R: int
    E: int
    K: int
    T: int
    S: int
    Gmax: int
    G: int
    L: np.ndarray  # [R][E] int64
    Tot: np.ndarray  # [E]
    W0: np.ndarray  # [R]
    W: np.ndarray  # [R]
    inst_expert: np.ndarray  # [R][G] int32
    inst_quota: np.ndarray  # [R][G] int64: the solve's split (shared column: its rows)
    inst_count: np.ndarray  # [R][G] int64: rows each instance receives
    inst_off: np.ndarray  # [R*G+1] int64
    dst_inst: np.ndarray  # [R][T][K] int32
    dst_row: np.ndarray  # [R][T][K] int64
    shared_rank: Optional[np.ndarray]  # [R][T] int32
    shared_row: Optional[np.ndarray]  # [R][T] int64
    cand_maxW: np.ndarray
    cand_repl: np.ndarray
    cand_stop: np.ndarray
    cap_idx: int
    cap: int
    stop_reason: int
    A: int
    before_max: int
    after_max: int
    replicas: int
    status: int
    rows: int
    realized_max: int

    @property
    def stop_name(self) -> str:
        return STOP_NAMES[self.stop_reason]


def gmax(E: int, R: int) -> int:
    return int(_load().orc_gmax(E, R))


def plan(ids: np.ndarray, *, E: int, S: int, m: int, J: int = 16, shared_expert: bool = False,
         seed: int = 0, bonus_permille: int = 10, all_ranks: bool = False, sampling: bool = False,
         sampling_seed: int = 0, iter_limit: int = 0) -> Plan:
    """Whole balance + dispatch plan of one layer from gate ids [R][T][K].

    sampling: each (token, k) draws an instance of its expert with probability
    quota / expert total (the LPLB-style dispatch) instead of the local-first
    rerouting; iter_limit > 0 replaces the greedy's iteration bound."""
    lib = _load()
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    R, T, K = ids.shape
    cfg = _Cfg(R=R, E=E, K=K, T=T, S=S, m=m, J=J, shared_expert=int(bool(shared_expert)),
               bonus_permille=bonus_permille, all_ranks=int(bool(all_ranks)),
               seed=seed & 0xFFFFFFFFFFFFFFFF, sampling=int(bool(sampling)),
               iter_limit=int(iter_limit), sampling_seed=sampling_seed & 0xFFFFFFFFFFFFFFFF)
    Gm = gmax(E, R)
    G = Gm + S + (1 if shared_expert else 0)
    L = np.zeros((R, E), np.int64)
    Tot = np.zeros(E, np.int64)
    W0 = np.zeros(R, np.int64)
    W = np.zeros(R, np.int64)
    inst_expert = np.zeros((R, G), np.int32)
    inst_quota = np.zeros((R, G), np.int64)
    inst_count = np.zeros((R, G), np.int64)
    inst_off = np.zeros(R * G + 1, np.int64)
    dst_inst = np.zeros((R, T, K), np.int32)
    dst_row = np.zeros((R, T, K), np.int64)
    shared_rank = np.zeros((R, T), np.int32) if shared_expert else None
    shared_row = np.zeros((R, T), np.int64) if shared_expert else None
    cand_maxW = np.zeros(J, np.int64)
    cand_repl = np.zeros(J, np.int32)
    cand_stop = np.zeros(J, np.int32)
    st = _Stats()
    rc = lib.orc_plan(ctypes.byref(cfg), _p(ids), _p(L), _p(Tot), _p(W0), _p(W), _p(inst_expert),
                      _p(inst_quota), _p(inst_count), _p(inst_off), _p(dst_inst), _p(dst_row),
                      _p(shared_rank),
                      _p(shared_row), _p(cand_maxW), _p(cand_repl), _p(cand_stop), ctypes.byref(st))
    if rc != 0:
        raise ValueError(f"oracle rejected the configuration (code {rc})")
    return Plan(R=R, E=E, K=K, T=T, S=S, Gmax=st.Gmax, G=st.G, L=L, Tot=Tot, W0=W0, W=W,
                inst_expert=inst_expert, inst_quota=inst_quota, inst_count=inst_count,
                inst_off=inst_off,
                dst_inst=dst_inst, dst_row=dst_row, shared_rank=shared_rank, shared_row=shared_row,
                cand_maxW=cand_maxW, cand_repl=cand_repl, cand_stop=cand_stop,
                cap_idx=st.cap_idx, cap=st.cap, stop_reason=st.stop_reason, A=st.A,
                before_max=st.before_max, after_max=st.after_max, replicas=st.replicas,
                status=st.status, rows=st.rows, realized_max=st.realized_max)


def load_matrix(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    R, T, K = ids.shape
    L = np.zeros((R, E), np.int64)
    bad = _load().orc_load_matrix(R, E, K, T, _p(ids), _p(L))
    return L, int(bad)


def splitmix64(x: int) -> int:
    return int(_load().orc_splitmix64(x & 0xFFFFFFFFFFFFFFFF))


def waterline(load: np.ndarray, N: int, bonus_permille: int = 10):
    """Waterfill waterline H, local preference B and per-rank slack."""
    load = np.ascontiguousarray(load, dtype=np.int64)
    slack = np.zeros(load.shape[0], np.int64)
    H = ctypes.c_int64()
    B = ctypes.c_int64()
    _load().orc_waterline(load.shape[0], N, _p(load), bonus_permille, ctypes.byref(H),
                          ctypes.byref(B), _p(slack))
    return int(H.value), int(B.value), slack


def waterfill(load: np.ndarray, dst_rank: np.ndarray, *, seed: int, bonus_permille: int = 10,
              all_ranks: bool = False):
    """Standalone Waterfill: shared-slot rank per token and per-rank counts."""
    load = np.ascontiguousarray(load, dtype=np.int64)
    dst_rank = np.ascontiguousarray(dst_rank, dtype=np.int32)
    R, T, K = dst_rank.shape
    pick = np.zeros((R, T), np.int32)
    count = np.zeros(R, np.int64)
    rc = _load().orc_waterfill(R, T, K, _p(load), _p(dst_rank), seed & 0xFFFFFFFFFFFFFFFF,
                               bonus_permille, int(bool(all_ranks)), _p(pick), _p(count))
    if rc != 0:
        raise ValueError("oracle waterfill rejected its arguments")
    return pick, count


def permute(p: Plan, hidden: np.ndarray) -> np.ndarray:
    """out[dst_row] = hidden row, as raw bytes; hidden [N][row] of any dtype."""
    hidden = np.ascontiguousarray(hidden)
    N = hidden.shape[0]
    out = np.zeros((p.rows,) + hidden.shape[1:], hidden.dtype)
    row_bytes = hidden.strides[0]
    dst = np.ascontiguousarray(p.dst_row.reshape(N, p.K))
    srow = None if p.shared_row is None else np.ascontiguousarray(p.shared_row.reshape(N))
    _load().orc_permute(N, p.K, row_bytes, _p(hidden), _p(dst), _p(srow), _p(out))
    return out


def permute_range(p: Plan, hidden_rows: np.ndarray, n0: int, out: np.ndarray) -> None:
    """Dispatch tokens [n0, n0 + len(hidden_rows)) of the layer into `out` (all rows)."""
    hidden_rows = np.ascontiguousarray(hidden_rows)
    n = hidden_rows.shape[0]
    assert out.flags.c_contiguous and out.strides[0] == hidden_rows.strides[0]
    dst = np.ascontiguousarray(p.dst_row.reshape(-1, p.K)[n0:n0 + n])
    srow = None if p.shared_row is None else np.ascontiguousarray(p.shared_row.reshape(-1)[n0:n0 + n])
    _load().orc_permute(n, p.K, hidden_rows.strides[0], _p(hidden_rows), _p(dst), _p(srow), _p(out))


def quota_solve(Tot: np.ndarray, R: int, S: int, m: int, J: int = 16):
    """The quota solve alone from per-expert totals: (W [R], max load, replicas)."""
    Tot = np.ascontiguousarray(Tot, dtype=np.int64)
    W = np.zeros(R, np.int64)
    mx = ctypes.c_int64()
    n = _load().orc_quota_solve(R, Tot.shape[0], S, m, J, _p(Tot), _p(W), ctypes.byref(mx))
    if n < 0:
        raise ValueError("oracle quota_solve rejected its arguments")
    return W, int(mx.value), int(n)


def eplb_plus(Tot: np.ndarray, R: int, S: int):
    """EPLB+ comparison baseline: (inst_expert [R][G], inst_quota [R][G], W [R], replicas)."""
    Tot = np.ascontiguousarray(Tot, dtype=np.int64)
    E = Tot.shape[0]
    G = gmax(E, R) + S
    ie = np.zeros((R, G), np.int32)
    iq = np.zeros((R, G), np.int64)
    W = np.zeros(R, np.int64)
    n = _load().orc_eplb_plus(R, E, S, _p(Tot), _p(ie), _p(iq), _p(W))
    return ie, iq, W, int(n)


def combine_tokens(expert_out: np.ndarray, dst_row: np.ndarray, weights: np.ndarray,
                   shared_row: Optional[np.ndarray] = None) -> np.ndarray:
    """fp64 combine of selected tokens: dst_row / weights [n][K], shared_row [n]."""
    x = np.ascontiguousarray(expert_out, dtype=np.uint16)
    dst = np.ascontiguousarray(dst_row, dtype=np.int64)
    n, K = dst.shape
    wt = np.ascontiguousarray(weights, dtype=np.float32).reshape(n, K)
    srow = None if shared_row is None else np.ascontiguousarray(shared_row, dtype=np.int64).reshape(n)
    out = np.zeros((n, x.shape[1]), np.float64)
    _load().orc_combine(n, K, x.shape[1], _p(x), _p(dst), _p(wt), _p(srow), _p(out))
    return out


def combine(p: Plan, expert_out: np.ndarray, weights: np.ndarray) -> np.ndarray:
    """fp64 combine: gate-weighted sum of each token's routed rows, plus its
    shared-expert row with weight 1.  expert_out: bf16 bits (uint16) [rows][H];
    weights: float32 [R][T][K].  Returns float64 [N][H]."""
    x = np.ascontiguousarray(expert_out, dtype=np.uint16)
    H = x.shape[1]
    N = p.R * p.T
    dst = np.ascontiguousarray(p.dst_row.reshape(N, p.K), dtype=np.int64)
    wt = np.ascontiguousarray(weights.reshape(N, p.K), dtype=np.float32)
    srow = None if p.shared_row is None else np.ascontiguousarray(p.shared_row.reshape(N), dtype=np.int64)
    out = np.zeros((N, H), np.float64)
    _load().orc_combine(N, p.K, H, _p(x), _p(dst), _p(wt), _p(srow), _p(out))
    return out


def stage(p: Plan, native_w: np.ndarray, slots: np.ndarray) -> None:
    """slots[q][s] = native_w[expert of slot (q, s)] for every filled slot (in place)."""
    native_w = np.ascontiguousarray(native_w)
    assert slots.flags.c_contiguous
    ie = np.ascontiguousarray(p.inst_expert, dtype=np.int32)
    _load().orc_stage(p.R, p.S, p.G, p.Gmax, _p(ie), native_w.strides[0], _p(native_w), _p(slots))


def reduce_grads(p: Plan, slot_grads: np.ndarray, native_grads: np.ndarray) -> None:
    """native_grads[e] += replica grads in instance order, then zero them (in place)."""
    assert slot_grads.flags.c_contiguous and native_grads.flags.c_contiguous
    assert native_grads.dtype == np.float32
    is_f32 = 1 if slot_grads.dtype == np.float32 else 0
    if not is_f32:
        assert slot_grads.dtype == np.uint16
    elems = native_grads.shape[1]
    ie = np.ascontiguousarray(p.inst_expert, dtype=np.int32)
    _load().orc_reduce_grads(p.R, p.S, p.G, p.Gmax, _p(ie), elems, is_f32, _p(slot_grads),
                             _p(native_grads))
