"""Pins of the selection-row checker ``oracle.selection_is_admissible`` (CPU).

The GPU and the oracle sum their fp32 dot products in different orders, so at a
near-tie (R10: relative gap below 1e-3 between the K_l-th and (K_l+1)-th score
of a pruning level) they may keep different blocks. The GPU tests accept such a
row only if the checker finds it well formed and reachable by the descent with
the near-ties resolved some way. These tests tie the checker to facts fixed
outside it:

* brute force: with tolerance 0 and inputs built to give many exactly equal
  scores, the rows it accepts are exactly the results of the descent under
  every way of breaking equal scores (each level's kept set enumerated as
  every K_l-subset whose lowest score is not below the highest score left
  out);
* the oracle's own rows are accepted, on random shapes with and without forced
  blocks and per-level budgets;
* doctored rows are rejected: a repeated block, a dropped slot, unsorted
  entries, a block after the padding, a future block, a missing forced block,
  a swap with a block far below the cut, and a child of a parent the descent
  did not keep;
* a planted near-tie one level above the blocks, resolved the other way,
  descends into other children: that row is accepted, its neighbours are not.
"""
import itertools

import numpy as np
import pytest

import oracle

F32 = np.float32


def _brute_force_rows(qbar, levels, factor, topk, last):
    """Every result of the descent under every way of breaking equal scores (fp64 scores of exact
    inputs): at each level, any K_l-subset S of the candidates with min over S >= max outside S."""
    n0 = levels[0].shape[0]
    top = len(levels) - 1

    def span_lo(l, c):
        return c * factor ** l

    def node_vec(l, c):
        lo, hi = span_lo(l, c), min((c + 1) * factor ** l, n0) - 1
        if hi <= last:
            return levels[l][c].astype(np.float64)
        return levels[0][lo:last + 1].astype(np.float64).mean(axis=0)

    results = set()

    def go(l, cands):
        s = {c: float(node_vec(l, c) @ qbar.astype(np.float64)) for c in cands}
        if len(cands) <= topk:
            subsets = [tuple(cands)]
        else:
            subsets = []
            for S in itertools.combinations(cands, topk):
                out = [s[c] for c in cands if c not in S]
                if min(s[c] for c in S) >= max(out):
                    subsets.append(S)
        for S in subsets:
            if l == 0:
                results.add(tuple(sorted(S)))
                continue
            n_below = levels[l - 1].shape[0]
            nxt = sorted(ch for c in S for ch in range(c * factor, min(c * factor + factor, n_below))
                         if span_lo(l - 1, ch) <= last)
            go(l - 1, nxt)

    go(top, [c for c in range(levels[top].shape[0]) if span_lo(top, c) <= last])
    return results


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_exact_ties_accepts_exactly_the_tie_resolutions(seed, causal):
    """nb = 16 blocks of one key each, factor 2 (levels 16, 8, 4, 2), K = 3; every key is one of
    three small integer patterns, so block means, node means and dot products are exact in fp32
    and equal scores abound at every level."""
    rng = np.random.Generator(np.random.PCG64(100 + seed))
    patterns = np.array([[2, 0, 1], [0, 2, 1], [1, 1, 0]], dtype=F32)
    keys = patterns[rng.integers(0, 3, size=16)]
    factor, topk = 2, 3
    levels = oracle.build_pyramid(keys, 1, factor)
    assert [lev.shape[0] for lev in levels] == [16, 8, 4, 2]
    n_ambiguous = 0
    for trial in range(4):
        qbar = rng.integers(-2, 3, size=3).astype(F32)
        for last in ([15] if not causal else [2, 5, 9, 15]):
            allowed = _brute_force_rows(qbar, levels, factor, topk, last)
            n_ambiguous += len(allowed) > 1
            want = oracle.select_blocks(qbar, levels, factor, topk, last)["idx"]
            assert tuple(want) in allowed
            eligible = list(range(last + 1))
            for size in {min(topk, len(eligible)) - 1, min(topk, len(eligible))} - {0}:
                for row in itertools.combinations(eligible, size):
                    padded = list(row) + [-1] * (topk - size)
                    ok, why = oracle.selection_is_admissible(qbar, levels, factor, topk, last, padded, rel_tol=0.0)
                    assert ok == (row in allowed), (trial, last, row, why, sorted(allowed))
    assert n_ambiguous > 0, "the inputs gave no equal scores at a cut"


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("forced", [0, 1, 3])
def test_oracle_rows_are_admissible(seed, forced):
    rng = np.random.Generator(np.random.PCG64(200 + seed))
    nb, block, factor, topk = int(rng.integers(5, 40)), 4, int(rng.integers(2, 5)), int(rng.integers(1, 7))
    causal = bool(seed % 2)
    q = rng.standard_normal((1, 2, nb * block, 8)).astype(F32)
    k = rng.standard_normal((1, 1, nb * block, 8)).astype(F32)
    sizes = oracle.level_sizes(nb, factor)
    budgets = [topk] + [int(rng.integers(1, topk + 3)) for _ in sizes[1:]]
    for bud in (None, budgets):
        r = oracle.forward(q, k, k, block, factor, topk, causal, budgets=bud, forced=forced)
        for i in range(nb):
            last = i if causal else nb - 1
            fset = oracle.forced_set(forced, i, topk)
            for tol in (0.0, 1e-3):
                ok, why = oracle.selection_is_admissible(r["qbar"][0, 0, i], r["pyramid"][0][0], factor, topk,
                                                         last, r["idx"][0, 0, i], budgets=bud, forced=fset,
                                                         rel_tol=tol)
                assert ok, (i, tol, why)


def _clear_rows(seed=7, nb=48, block=4, factor=4, topk=6, causal=True):
    """Random inputs and the oracle's rows with no near-tie at any level (margin >= 1e-3)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((1, 1, nb * block, 16)).astype(F32)
    k = rng.standard_normal((1, 1, nb * block, 16)).astype(F32)
    r = oracle.forward(q, k, k, block, factor, topk, causal)
    rows = [i for i in range(nb) if r["margin"][0, 0, i] >= 1e-3 and (i + 1 if causal else nb) > topk + 2]
    assert len(rows) > 10
    return r, rows, factor, topk, causal, nb


def test_doctored_rows_are_rejected():
    r, rows, factor, topk, causal, nb = _clear_rows()
    levels = r["pyramid"][0][0]

    def check(i, row, forced=None):
        last = i if causal else nb - 1
        return oracle.selection_is_admissible(r["qbar"][0, 0, i], levels, factor, topk, last, row, forced=forced)

    for i in rows:
        good = [int(x) for x in r["idx"][0, 0, i]]
        assert check(i, good)[0]
        kept = [x for x in good if x >= 0]
        last = i if causal else nb - 1
        outside = [j for j in range(last + 1) if j not in kept]
        doctored = {
            "repeated": sorted(kept[:-1] + [kept[0]]) + [-1] * (topk - len(kept)),
            "dropped slot": kept[:-1] + [-1] * (topk - len(kept) + 1),
            "unsorted": kept[::-1] + [-1] * (topk - len(kept)),
            "block after padding": kept[:-2] + [-1, kept[-1]] + [-1] * (topk - len(kept)),
            "future block": sorted(kept[:-1] + [last + 1]) + [-1] * (topk - len(kept)) if last + 1 < nb else None,
        }
        for what, row in doctored.items():
            if row is None:
                continue
            assert not check(i, row[:topk])[0], (i, what, row)
        # every single swap of a kept block for a block left out changes a row with no near-tie
        for t in range(len(kept)):
            for j in outside:
                swapped = sorted(kept[:t] + kept[t + 1:] + [j]) + [-1] * (topk - len(kept))
                assert not check(i, swapped)[0], (i, kept[t], j)
        # a forced block the row does not hold
        if outside:
            assert not check(i, good, forced=[outside[0]])[0]


def test_near_tie_one_level_up_may_descend_into_other_children():
    """16 one-key blocks, factor 4 (levels 16, 4), K = 2, scores = first key component.
    Level 1 node means: 4.75, 3.0, 2.999625 (relative gap 1.25e-4 to node 1: a near-tie), 0.
    Keeping node 1 (the oracle) gives blocks [0, 1]; keeping node 2 instead gives [0, 9]."""
    first = [10, 9, 0, 0, 3, 3, 3, 3, 1, 10.9985, 0, 0, 0, 0, 0, 0]
    keys = np.zeros((16, 2), dtype=F32)
    keys[:, 0] = first
    levels = oracle.build_pyramid(keys, 1, 4)
    assert [lev.shape[0] for lev in levels] == [16, 4]
    qbar = np.array([1.0, 0.0], dtype=F32)
    r = oracle.select_blocks(qbar, levels, 4, 2, 15)
    assert r["idx"] == [0, 1] and r["margin"] < 1e-3

    def ok(row, tol=1e-3):
        return oracle.selection_is_admissible(qbar, levels, 4, 2, 15, row, rel_tol=tol)[0]

    assert ok([0, 1]) and ok([0, 9])
    for row in ([0, 4], [1, 9], [0, 12], [9, 13], [1, 2], [0, 8]):
        assert not ok(row), row
    # without tolerance only the oracle's own resolution remains
    assert ok([0, 1], 0.0) and not ok([0, 9], 0.0)


def test_gpu_harness_rejects_a_doctored_near_tie_row():
    """The GPU tests' row check (``gpu_util.check_selection``) on the planted near-tie above, with
    the GPU's rows stood in for by hand: the other resolution of the tie passes; a near-tie row
    with a repeated block, a dropped slot or a block far below the cut fails."""
    import workloads
    from tests import gpu_util as gu
    first = [10, 9, 0, 0, 3, 3, 3, 3, 1, 10.9985, 0, 0, 0, 0, 0, 0]
    keys = np.zeros((16, 2), dtype=F32)
    keys[:, 0] = first
    levels = oracle.build_pyramid(keys, 1, 4)
    qbar = np.array([1.0, 0.0], dtype=F32)
    r = oracle.select_blocks(qbar, levels, 4, 2, 15)
    # one decode row over 16 one-key blocks, factor 4, K = 2
    w = workloads.Workload("planted-near-tie", 1, 1, 1, 1, 16, 2, 1, 4, 2, 0, "iid", 0)
    ref = {"idx": np.array(r["idx"], dtype=np.int32).reshape(1, 1, 1, 2),
           "margin": np.array([[[r["margin"]]]]), "qbar": qbar.reshape(1, 1, 1, 2), "pyramid": [[levels]]}
    assert gu.check_selection(ref["idx"], ref, w) == (1, 0)
    assert gu.check_selection(np.array([0, 9]).reshape(1, 1, 1, 2), ref, w) == (1, 1)
    for row in ([0, 0], [0, -1], [0, 4], [9, 0]):
        with pytest.raises(AssertionError):
            gu.check_selection(np.array(row).reshape(1, 1, 1, 2), ref, w)
