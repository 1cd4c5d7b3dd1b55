"""Property checks of a balance + dispatch plan, written from the pages' rules.

Independent of the oracle's code: these functions only look at the plan's
outputs (instance table, quotas, dispatch rows) and check what the UltraEP page
(section "Quota decides replicas and token split together") and the Waterfill
page (section "Waterfill") require of any valid plan:

* per-expert quota conservation, minimum replica quota, at most S replicas per
  rank, no logical expert twice on one rank, one fixed native per expert;
* the per-rank load equals the sum of the rank's quotas and no receiving rank
  exceeds the cap;
* every (token, k) lands in exactly one row of an instance of its own logical
  expert (a bijection onto the rows), same-rank instances are filled first, the
  residual demands fill the remote instances in instance order (north-west
  corner rule: no two flows cross), and rows inside an instance follow the
  source order;
* the Waterfill shared slot of a token is on its own rank or on a rank the token
  already visits (any rank in all-rank mode).
"""
from __future__ import annotations

import numpy as np


def native_blocks(E: int, R: int):
    base, rem = divmod(E, R)
    first = [q * base + min(q, rem) for q in range(R)]
    count = [base + (1 if q < rem else 0) for q in range(R)]
    return first, count


def check_plan(ids: np.ndarray, E: int, S: int, m: int, *, Gmax: int, G: int, W, inst_expert,
               inst_quota, inst_off, dst_row, cap=None, stop=None, shared_rank=None,
               shared_row=None, W0=None, all_ranks=False):
    ids = np.asarray(ids)
    R, T, K = ids.shape
    inst_expert = np.asarray(inst_expert).reshape(R, G)
    inst_quota = np.asarray(inst_quota, dtype=np.int64).reshape(R, G)
    inst_off = np.asarray(inst_off, dtype=np.int64).reshape(-1)
    dst_row = np.asarray(dst_row, dtype=np.int64).reshape(R, T, K)
    W = np.asarray(W, dtype=np.int64)
    sh = G - Gmax - S
    assert sh in (0, 1)
    valid = (ids >= 0) & (ids < E)
    L = np.stack([np.bincount(ids[r][valid[r]].ravel(), minlength=E) for r in range(R)])
    Tot = L.sum(0)

    # native placement and slot structure
    first, count = native_blocks(E, R)
    for q in range(R):
        nat = inst_expert[q, :Gmax]
        assert list(nat[: count[q]]) == list(range(first[q], first[q] + count[q])), "native block"
        assert (nat[count[q]:] == -1).all() and (inst_quota[q, count[q]:Gmax] == 0).all()
        slots = inst_expert[q, Gmax:Gmax + S]
        filled = slots[slots >= 0]
        n_filled = len(filled)
        assert (slots[n_filled:] == -1).all(), "slots fill in order"
        assert (inst_quota[q, Gmax + n_filled:Gmax + S] == 0).all()
        held = list(nat[: count[q]]) + list(filled)
        assert len(set(held)) == len(held), "no logical expert twice on one rank"
        assert ((filled >= 0) & (filled < E)).all()
        assert (inst_quota[q, Gmax:Gmax + n_filled] >= m).all(), "replica below minimum quota"
        assert W[q] == inst_quota[q, :Gmax + S].sum(), "rank load = sum of its quotas"
        if sh:
            assert inst_expert[q, Gmax + S] == E
    assert (inst_quota >= 0).all()
    per_e = np.zeros(E, np.int64)
    for q in range(R):
        for col in range(Gmax + S):
            e = inst_expert[q, col]
            if e >= 0:
                per_e[e] += inst_quota[q, col]
    assert (per_e == Tot).all(), "per-expert quota conservation"
    if cap is not None:
        for q in range(R):
            if (inst_expert[q, Gmax:Gmax + S] >= 0).any():
                assert W[q] <= cap, "a receiving rank is above the cap"
        if stop == "BALANCED":
            assert W.max(initial=0) <= cap

    # row layout: exclusive prefix of quotas in instance order
    flat_q = inst_quota.reshape(-1)
    assert inst_off[0] == 0 and (np.diff(inst_off) == flat_q).all()
    rows = int(inst_off[-1])

    # bijection and "row is an instance of the token's expert"
    d = dst_row[valid]
    assert (dst_row[~valid] == -1).all()
    all_rows = d
    if sh:
        all_rows = np.concatenate([d, np.asarray(shared_row, dtype=np.int64).ravel()])
    assert len(all_rows) == rows
    assert (np.sort(all_rows) == np.arange(rows)).all(), "rows are a bijection"
    inst_of_row = np.searchsorted(inst_off, np.arange(rows), side="right") - 1
    inst_flat_e = inst_expert.reshape(-1)
    inst_a = inst_of_row[d]
    assert (inst_flat_e[inst_a] == ids[valid]).all(), "row hosts another expert"

    # rows inside an instance follow (source rank, t, k)
    flat_idx = np.arange(R * T * K).reshape(R, T, K)[valid]
    order = np.argsort(d)
    inst_sorted = inst_a[order]
    src_sorted = flat_idx[order]
    same = inst_sorted[1:] == inst_sorted[:-1]
    assert (src_sorted[1:][same] > src_sorted[:-1][same]).all(), "row order inside an instance"

    # local first, remote fill in instance order (no crossing flows)
    NI = R * G
    rank_of_inst = inst_a // G
    src_rank = np.repeat(np.arange(R), T * K).reshape(R, T, K)[valid]
    uniq, cnt = np.unique(src_rank.astype(np.int64) * NI + inst_a, return_counts=True)
    F = dict(zip(uniq.tolist(), cnt.tolist()))
    for q in range(R):
        for col in range(Gmax + S):
            i = q * G + col
            e = inst_flat_e[i]
            if e >= 0:
                assert F.get(q * NI + i, 0) == min(L[q, e], flat_q[i]), "local instance first"
    remote_by_e = {}
    for key in uniq.tolist():
        r, i = divmod(key, NI)
        if i // G != r:
            remote_by_e.setdefault(int(inst_flat_e[i]), []).append((r, i))
    for e, pairs in remote_by_e.items():
        for (r1, i1) in pairs:
            for (r2, i2) in pairs:
                if r1 < r2 and i1 > i2:
                    raise AssertionError("remote flows cross (not filled in instance order)")
    # per (source, expert), in token order: the local block, then instances non-decreasing
    e_a = ids[valid]
    order = np.lexsort((flat_idx, e_a, src_rank))
    grp = (src_rank[order].astype(np.int64) * E + e_a[order])
    is_loc = (rank_of_inst[order] == src_rank[order]).astype(np.int8)
    ins = inst_a[order]
    same = grp[1:] == grp[:-1]
    assert not ((is_loc[1:] > is_loc[:-1]) & same).any(), "local assignments come first"
    both_remote = (is_loc[1:] == 0) & (is_loc[:-1] == 0) & same
    assert not ((ins[1:] < ins[:-1]) & both_remote).any(), "remote instances in instance order"

    if sh:
        sr = np.asarray(shared_rank).reshape(R, T)
        srow = np.asarray(shared_row, dtype=np.int64).reshape(R, T)
        rank_k = np.full((R, T, K), -1, np.int64)
        rank_k[valid] = rank_of_inst
        own = sr == np.arange(R)[:, None]
        visits = (rank_k == sr[:, :, None]).any(axis=2)
        if all_ranks:
            assert ((sr >= 0) & (sr < R)).all()
        else:
            assert (own | visits).all(), "shared slot outside the candidate set"
        counts = np.bincount(sr.ravel(), minlength=R)
        assert (inst_quota[:, Gmax + S] == counts).all()
        # shared rows ordered by (source rank, t) inside each rank's shared column
        for q in range(R):
            rr = srow[sr == q]
            assert (np.diff(rr) > 0).all()
            if len(rr):
                assert rr[0] == inst_off[q * G + Gmax + S]
    return dict(L=L, Tot=Tot)



def check_sampled_rows(ids: np.ndarray, E: int, *, Gmax: int, G: int, S: int, inst_expert,
                       inst_quota, inst_count, inst_off, dst_row, shared_rank=None,
                       shared_row=None):
    """Rows of the sampling rerouting mode ("Waterfill and LPLB" page, section
    "LPLB": each token of a replicated expert samples one of its physical
    instances).  Whatever the draws, the rows must be a bijection, each row
    must sit in an instance of its token's expert, the rows an instance
    receives must be what the layout gives it, an instance the split gives no
    tokens can never be drawn, an expert with one instance keeps all its
    tokens there, and rows inside an instance follow (source rank, t, k)."""
    ids = np.asarray(ids)
    R, T, K = ids.shape
    inst_expert = np.asarray(inst_expert).reshape(R, G)
    inst_quota = np.asarray(inst_quota, dtype=np.int64).reshape(R, G)
    inst_count = np.asarray(inst_count, dtype=np.int64).reshape(R, G)
    inst_off = np.asarray(inst_off, dtype=np.int64).reshape(-1)
    dst_row = np.asarray(dst_row, dtype=np.int64).reshape(R, T, K)
    sh = G - Gmax - S
    valid = (ids >= 0) & (ids < E)
    Tot = np.bincount(ids[valid].ravel(), minlength=E)
    assert inst_off[0] == 0 and (np.diff(inst_off) == inst_count.reshape(-1)).all()
    rows = int(inst_off[-1])
    d = dst_row[valid]
    assert (dst_row[~valid] == -1).all()
    all_rows = d if not sh else np.concatenate([d, np.asarray(shared_row, np.int64).ravel()])
    assert len(all_rows) == rows
    assert (np.sort(all_rows) == np.arange(rows)).all(), "rows are a bijection"
    inst_of_row = np.searchsorted(inst_off, np.arange(rows), side="right") - 1
    flat_e = inst_expert.reshape(-1)
    inst_a = inst_of_row[d]
    assert (flat_e[inst_a] == ids[valid]).all(), "row hosts another expert"
    n_inst = np.zeros(E, np.int64)
    got = np.zeros(E, np.int64)
    for q in range(R):
        for col in range(Gmax + S):
            e = inst_expert[q, col]
            if e >= 0:
                n_inst[e] += 1
                got[e] += inst_count[q, col]
                if inst_quota[q, col] == 0:
                    assert inst_count[q, col] == 0, "an instance with no quota was drawn"
    assert (got == Tot).all(), "every assignment of an expert lands in one of its instances"
    for q in range(R):
        for col in range(Gmax + S):
            e = inst_expert[q, col]
            if e >= 0 and n_inst[e] == 1:
                assert inst_count[q, col] == Tot[e], "single instance keeps all its tokens"
    flat_idx = np.arange(R * T * K).reshape(R, T, K)[valid]
    order = np.argsort(d)
    same = inst_a[order][1:] == inst_a[order][:-1]
    src = flat_idx[order]
    assert (src[1:][same] > src[:-1][same]).all(), "row order inside an instance"
    if sh:
        sr = np.asarray(shared_rank).reshape(R, T)
        counts = np.bincount(sr.ravel(), minlength=R)
        assert (inst_count[:, Gmax + S] == counts).all()
        assert (inst_quota[:, Gmax + S] == counts).all()
