"""LP cross-check of a quota split (TEST INFRASTRUCTURE, like the rest of oracle/).

Waterfill and LPLB page, section "LPLB": for a fixed replica placement, the
per-batch split that minimises the largest per-rank load is a small linear
program (minimise M subject to: each expert's instance quotas sum to its
load, each rank's quotas sum to at most M).  Solved here with scipy's HiGHS
for a placement taken from an instance table, optionally with the minimum
quota m on replica instances.  Its optimum bounds from below the largest
per-rank load any split of that placement can reach, so the greedy's split
can be measured against it.
"""
from __future__ import annotations

import numpy as np
from scipy.optimize import linprog


def min_max_split(Tot, inst_expert, Gmax: int, S: int, m_replica: int = 0):
    """Optimal max per-rank load (LP relaxation) for the placement in inst_expert.

    Tot [E]; inst_expert [R][G] with natives in columns [0, Gmax) and replicas
    in [Gmax, Gmax+S).  Returns (M, x) with x the per-instance quotas."""
    ie = np.asarray(inst_expert)
    R = ie.shape[0]
    inst = [(q, col, int(ie[q, col])) for q in range(R) for col in range(Gmax + S)
            if ie[q, col] >= 0 and ie[q, col] < len(Tot)]
    n = len(inst)
    E = len(Tot)
    # variables: x_0..x_{n-1}, M ; minimise M
    c = np.zeros(n + 1)
    c[-1] = 1.0
    A_eq = np.zeros((E, n + 1))
    for j, (_, _, e) in enumerate(inst):
        A_eq[e, j] = 1.0
    b_eq = np.asarray(Tot, dtype=np.float64)
    A_ub = np.zeros((R, n + 1))
    for j, (q, _, _) in enumerate(inst):
        A_ub[q, j] = 1.0
    A_ub[:, -1] = -1.0
    b_ub = np.zeros(R)
    bounds = [(m_replica if col >= Gmax else 0.0, None) for (_, col, _) in inst] + [(0.0, None)]
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, A_eq=A_eq, b_eq=b_eq, bounds=bounds, method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return float(res.x[-1]), res.x[:-1]
