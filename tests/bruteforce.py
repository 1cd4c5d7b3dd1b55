"""Exact minimum of the worst-rank load by exhaustive enumeration (tiny inputs).

Independent of the oracle: it shares no code with it and solves the problem
the quota solve approximates (UltraEP page, section "Quota decides replicas and
token split together"): place replicas into at most S redundant slots per rank,
never two instances of one logical expert on a rank, give every placed replica
at least m tokens, split each expert's load over its instances, and minimise the
largest per-rank load.

For a fixed placement, pre-assign m tokens to every replica (the lower bound);
what remains is a transportation problem with unbounded expert->rank edges, and
by Hall's / Gale's supply-demand theorem a cap M is feasible iff every set Y of
experts satisfies  rest(Y) <= sum over ranks r in N(Y) of (M - pre[r]), and
M >= pre[r] for all r.  The smallest feasible M is therefore a maximum over the
2^E expert subsets, which this module evaluates directly.
"""
from __future__ import annotations

import itertools
from typing import List, Sequence, Tuple


def native_home(E: int, R: int) -> List[int]:
    """Contiguous balanced native blocks: first E % R ranks hold one more."""
    base, rem = divmod(E, R)
    home = []
    for q in range(R):
        home += [q] * (base + (1 if q < rem else 0))
    return home


def min_cap_for_placement(tot: Sequence[int], home: Sequence[int], repl: Sequence[Tuple[int, int]],
                          R: int, m: int) -> int:
    """Smallest max rank load for a fixed replica placement [(expert, rank)], or -1."""
    E = len(tot)
    rest = list(tot)
    pre = [0] * R
    ranks_of = [{home[e]} for e in range(E)]
    for e, r in repl:
        rest[e] -= m
        pre[r] += m
        ranks_of[e].add(r)
    if min(rest) < 0:
        return -1
    best = max(pre)
    for mask in range(1, 1 << E):
        need = 0
        nb = set()
        for e in range(E):
            if mask >> e & 1:
                need += rest[e]
                nb |= ranks_of[e]
        total = need + sum(pre[r] for r in nb)
        best = max(best, -(-total // len(nb)))
    return best


def placements(E: int, R: int, S: int, home: Sequence[int]):
    """Every assignment of at most S distinct non-native experts to each rank."""
    per_rank = []
    for q in range(R):
        cands = [e for e in range(E) if home[e] != q]
        opts = []
        for k in range(S + 1):
            opts += list(itertools.combinations(cands, k))
        per_rank.append(opts)
    for choice in itertools.product(*per_rank):
        yield [(e, q) for q, es in enumerate(choice) for e in es]


def brute_force_opt(tot: Sequence[int], R: int, S: int, m: int) -> int:
    """Exact optimum of the worst-rank load over all placements and splits."""
    E = len(tot)
    home = native_home(E, R)
    best = None
    for repl in placements(E, R, S, home):
        c = min_cap_for_placement(tot, home, repl, R, m)
        if c >= 0 and (best is None or c < best):
            best = c
    return best
