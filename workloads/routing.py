"""Seeded synthetic gate outputs and bf16 payloads.

Routing recipe (stand-in for real routing traces, which are not available):

* Per layer, a seeded permutation pi of the E experts fixes which expert is
  hot; expert pi[j] has popularity proportional to (j+1)^-s (finite Zipf).
* Distinct top-k per token is drawn by Gumbel-top-k, i.e. weighted sampling
  without replacement, and the k columns are ordered by descending score as a
  router's sorted top-k output would be.
* The stress workload draws each (token, k) independently: with probability
  hot_frac the hot expert pi[0], otherwise Zipf(s) over the other E-1 experts.
  Duplicates within a token are allowed there (a single expert cannot take 40 %
  of assignments under distinct top-8).
* The 94-layer sweep draws its per-layer exponent uniformly from [0.8, 1.6]
  with the generator seeded by (seed - 1) and layer l uses seed + l.

Every array is produced by numpy's PCG64 generator, so the oracle and the CUDA
path see identical ids.
"""
from __future__ import annotations

import numpy as np

from .configs import WorkloadConfig

_CHUNK_TOKENS = 1 << 15


def _layer_params(cfg: WorkloadConfig, layer: int):
    if cfg.layers > 1:
        s_all = np.random.default_rng(cfg.seed - 1).uniform(0.8, 1.6, size=cfg.layers)
        return cfg.seed + layer, float(s_all[layer])
    if layer != 0:
        raise ValueError(f"workload {cfg.name} has a single layer")
    return cfg.seed, cfg.zipf_s


def _zipf_probs(n: int, s: float) -> np.ndarray:
    w = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return w / w.sum()


def topk_ids(cfg: WorkloadConfig, layer: int = 0) -> np.ndarray:
    """Gate top-k expert ids, int32 [R][T][K], C-contiguous."""
    seed, s = _layer_params(cfg, layer)
    rng = np.random.default_rng(seed)
    E, K, N = cfg.E, cfg.K, cfg.N
    perm = rng.permutation(E)
    out = np.empty((N, K), dtype=np.int32)
    if cfg.hot_frac is not None:
        p_rest = _zipf_probs(E - 1, s)
        cdf = np.cumsum(p_rest)
        cdf[-1] = 1.0
        for a in range(0, N, _CHUNK_TOKENS):
            b = min(N, a + _CHUNK_TOKENS)
            hot = rng.random((b - a, K)) < cfg.hot_frac
            rest = np.searchsorted(cdf, rng.random((b - a, K)), side="right")
            rest = np.minimum(rest, E - 2)
            out[a:b] = np.where(hot, perm[0], perm[1 + rest])
    elif cfg.distinct:
        if K > E:
            raise ValueError("distinct top-k needs K <= E")
        p = np.empty(E, dtype=np.float64)
        p[perm] = _zipf_probs(E, s)
        logp = np.log(p).astype(np.float32)
        for a in range(0, N, _CHUNK_TOKENS):
            b = min(N, a + _CHUNK_TOKENS)
            score = rng.gumbel(size=(b - a, E)).astype(np.float32) + logp
            if K < E:
                top = np.argpartition(-score, K - 1, axis=1)[:, :K]
            else:
                top = np.broadcast_to(np.arange(E), (b - a, E)).copy()
            order = np.argsort(-np.take_along_axis(score, top, axis=1), axis=1, kind="stable")
            out[a:b] = np.take_along_axis(top, order, axis=1)
    else:
        p = np.empty(E, dtype=np.float64)
        p[perm] = _zipf_probs(E, s)
        cdf = np.cumsum(p)
        cdf[-1] = 1.0
        for a in range(0, N, _CHUNK_TOKENS):
            b = min(N, a + _CHUNK_TOKENS)
            out[a:b] = np.minimum(np.searchsorted(cdf, rng.random((b - a, K)), side="right"), E - 1)
    return out.reshape(cfg.R, cfg.T, K)


def _bf16_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, std^2) samples, round-to-nearest-even."""
    x = (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).view(np.uint32)
    rounding = ((x >> 16) & 1) + np.uint32(0x7FFF)
    return ((x + rounding) >> 16).astype(np.uint16)


def hidden_states_np(cfg: WorkloadConfig, seed: int = 0) -> np.ndarray:
    """bf16 N(0,1) hidden states as uint16 bit patterns, [N][hidden]."""
    return _bf16_normal(np.random.default_rng(cfg.seed * 7 + 1 + seed), (cfg.N, cfg.hidden), 1.0)


def expert_weights_np(cfg: WorkloadConfig, elems: int | None = None, seed: int = 0) -> np.ndarray:
    """bf16 N(0,1) native expert weights as uint16 bit patterns, [E][elems]."""
    n = cfg.expert_elems if elems is None else elems
    return _bf16_normal(np.random.default_rng(cfg.seed * 7 + 2 + seed), (cfg.E, n), 1.0)


def replica_grads_np(cfg: WorkloadConfig, elems: int, seed: int = 0) -> np.ndarray:
    """bf16 N(0, 1e-4) slot gradients as uint16 bit patterns, [R][S][elems]."""
    return _bf16_normal(np.random.default_rng(cfg.seed * 7 + 3 + seed), (cfg.R, cfg.S, elems), 1e-2)
