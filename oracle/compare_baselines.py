"""UltraEP-style greedy vs the EPLB+ baseline vs the LP bound, on the seeded
workloads (TEST INFRASTRUCTURE: runs the oracle only).

    python -m oracle.compare_baselines [--sweep-layers 94]

The UltraEP page (section "Quota decides replicas and token split together")
reports, against EPLB+ (exact loads, EPLB-style replication, round-robin
rerouting), mean imbalance 1.19 -> 1.03 and 57.9 % fewer redundant slots used.
This prints the same two quantities for this repository's greedy and its EPLB+
reading, plus the LP optimum of the min-max split for the greedy's placement.
"""
from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from oracle.lplb import min_max_split  # noqa: E402
from workloads import get_config, topk_ids  # noqa: E402


def _best_time(fn, reps=5):
    """Smallest wall time of fn over reps runs (one host thread)."""
    best = float("inf")
    for _ in range(reps):
        t0 = time.perf_counter()
        fn()
        best = min(best, time.perf_counter() - t0)
    return best


def one(cfg, ids, timing=True):
    p = oracle.plan(ids, E=cfg.E, S=cfg.S, m=cfg.m, J=cfg.J)
    mean = p.A / cfg.R
    _, _, W, n = oracle.eplb_plus(p.Tot, cfg.R, cfg.S)
    M, _ = min_max_split(p.Tot, p.inst_expert, p.Gmax, p.S, m_replica=cfg.m)
    r = dict(before=p.before_max / mean, greedy=p.after_max / mean, greedy_slots=p.replicas,
             eplb=W.max() / mean, eplb_slots=n, lp=M / mean)
    if timing:  # the two replication rules alone, from the same per-expert totals
        r["greedy_ms"] = 1e3 * _best_time(lambda: oracle.quota_solve(p.Tot, cfg.R, cfg.S, cfg.m, cfg.J))
        r["eplb_ms"] = 1e3 * _best_time(lambda: oracle.eplb_plus(p.Tot, cfg.R, cfg.S))
    return r


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--sweep-layers", type=int, default=94)
    args = ap.parse_args()
    rows = []
    for name in ("qwen", "dsv3", "stress"):
        cfg = get_config(name)
        rows.append((name, one(cfg, topk_ids(cfg))))
    cfg = get_config("sweep")
    sw = [one(cfg, topk_ids(cfg, l), timing=l < 8) for l in range(args.sweep_layers)]
    agg = {k: float(np.mean([r[k] for r in sw if k in r])) for k in sw[0]}
    rows.append((f"sweep (mean of {args.sweep_layers} layers)", agg))
    print("| workload | max/mean before | greedy max/mean | greedy replicas | EPLB+ max/mean | "
          "EPLB+ replicas | LP bound (greedy placement) | greedy solve ms | EPLB+ solve ms |")
    print("|---|---|---|---|---|---|---|---|---|")
    for name, r in rows:
        print(f"| {name} | {r['before']:.3f} | {r['greedy']:.3f} | {r['greedy_slots']:.1f} | "
              f"{r['eplb']:.3f} | {r['eplb_slots']:.1f} | {r['lp']:.3f} | {r['greedy_ms']:.3f} | "
              f"{r['eplb_ms']:.3f} |")
    print("\nsolve latency: one host thread, best of 5 runs, from the same per-expert totals "
          "(sweep: mean over its first 8 layers)")
    slots_cut = 1 - agg["greedy_slots"] / agg["eplb_slots"]
    print(f"\nsweep: mean imbalance EPLB+ {agg['eplb']:.3f} -> greedy {agg['greedy']:.3f}; "
          f"redundant slots used {100 * slots_cut:.1f} % fewer")


if __name__ == "__main__":
    main()
