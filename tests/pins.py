"""Checks that tie the CPU oracle to facts fixed outside it.

Each check takes the oracle module as an argument so that the mutation tests
can run the same check against an oracle with a planted mistake and see it
fail. A check returns None when the pin holds and raises AssertionError
otherwise. The facts come from the definitions on the pages (pooling means,
dense softmax attention, online-softmax merge) and from mathematics (brute
force on tiny inputs, closed forms, invariants); none is a retyped copy of the
oracle's own formula.
"""
from __future__ import annotations

import math

import numpy as np


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _bf16_exact(x):
    from workloads import bf16_to_f32, round_bf16
    return bf16_to_f32(round_bf16(np.asarray(x, dtype=np.float32)))


def rand_qkv(seed, B, Hq, Hkv, Nq, N, D):
    g = _rng(seed)
    q = _bf16_exact(g.standard_normal((B, Hq, Nq, D)))
    k = _bf16_exact(g.standard_normal((B, Hkv, N, D)))
    v = _bf16_exact(g.standard_normal((B, Hkv, N, D)))
    return q, k, v


# ----------------------------------------------------------------------------- P2 pyramid means

def check_pyramid_means(o, seed=7, n_blocks=37, block=16, factor=4, D=24):
    """Every node equals the fp64 mean of all keys it covers; a node with f full
    children equals the fp64 mean of its children (ragged tail included)."""
    g = _rng(seed)
    keys = _bf16_exact(g.standard_normal((n_blocks * block, D)) * 3.0 + 0.5)
    levels = o.build_pyramid(keys, block, factor)
    width = 1
    for l, lev in enumerate(levels):
        n_l = -(-n_blocks // width)
        assert lev.shape == (n_l, D), (l, lev.shape)
        for c in range(n_l):
            lo, hi = c * width * block, min((c + 1) * width, n_blocks) * block
            ref = keys[lo:hi].astype(np.float64).mean(axis=0)
            assert np.allclose(lev[c], ref, rtol=1e-5, atol=1e-5), (l, c)
            if l > 0 and (c + 1) * factor <= levels[l - 1].shape[0] and (c + 1) * width <= n_blocks:
                kids = levels[l - 1][c * factor:(c + 1) * factor].astype(np.float64).mean(axis=0)
                assert np.allclose(lev[c], kids, rtol=1e-5, atol=1e-5), (l, c)
        width *= factor
    assert levels[-1].shape[0] <= factor and (len(levels) == 1 or levels[-2].shape[0] > factor)


# ----------------------------------------------------------------------------- query summary

def check_query_summary(o, seed=8):
    g = _rng(seed)
    q = _bf16_exact(g.standard_normal((3, 40, 16)))
    qbar = o.query_summary(q, 8)
    assert qbar.shape == (5, 16)
    for i in range(5):
        ref = q[:, i * 8:(i + 1) * 8].astype(np.float64).reshape(-1, 16).mean(axis=0)
        assert np.allclose(qbar[i], ref, rtol=1e-6, atol=1e-6), i
    dec = o.query_summary(q[:, :1], 1)
    assert np.allclose(dec[0], q[:, 0].astype(np.float64).mean(axis=0), rtol=1e-6, atol=1e-6)


# ----------------------------------------------------------------------------- P1 dense reduction

def check_dense_reduction(o, seed=11, causal=True, per_qhead=False, decode=False,
                          B=1, Hq=4, Hkv=2, N=256, D=32, block=16, factor=4):
    """With K >= every eligible block, sparse attention is dense softmax attention (fp64 brute force)."""
    nq = 1 if decode else N
    q, k, v = rand_qkv(seed, B, Hq, Hkv, nq, N, D)
    res = o.forward(q, k, v, block, factor, N // block, causal, per_qhead=per_qhead)
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(D)
    for b in range(B):
        for h in range(Hq):
            pos = np.full(1, N - 1) if decode else np.arange(N)
            ref_o, ref_l = o_dense(q[b, h], pos, k[b, h // g], v[b, h // g], causal and not decode, scale)
            assert np.abs(res["O"][b, h] - ref_o).max() < 1e-5, (b, h)
            assert np.abs(res["lse"][b, h] - ref_l).max() < 1e-5, (b, h)


def o_dense(q, pos, k, v, causal, scale):
    """Textbook dense attention written out independently of the oracle (fp64)."""
    s = scale * (q.astype(np.float64) @ k.astype(np.float64).T)
    if causal:
        s[np.arange(k.shape[0])[None, :] > pos[:, None]] = -np.inf
    p = np.exp(s - s.max(axis=1, keepdims=True))
    out = (p @ v.astype(np.float64)) / p.sum(axis=1, keepdims=True)
    lse = np.log(np.exp(s - s.max(axis=1, keepdims=True)).sum(axis=1)) + s.max(axis=1)
    return out, lse


# ----------------------------------------------------------------------------- P3 cardinality

def check_cardinality(o, seed=12, causal=True, topk=6, N=512, block=16, factor=4):
    q, k, v = rand_qkv(seed, 1, 2, 1, N, N, 16)
    res = o.forward(q, k, v, block, factor, topk, causal)
    nb = N // block
    for i in range(nb):
        row = res["idx"][0, 0, i]
        eligible = i + 1 if causal else nb
        valid = row[row >= 0]
        assert len(valid) == min(topk, eligible), (i, row)
        assert np.all(row[len(valid):] == -1)
        assert len(set(valid.tolist())) == len(valid)
        assert np.all(np.diff(valid) > 0)
        assert valid.max() < eligible and valid.min() >= 0


# ----------------------------------------------------------------------------- P4 tie rule

def tie_case():
    """Key blocks 3, 9 and 12 are identical and point along the query; the rest are zero.

    nb = 16, f = 4, K = 2. At level 1 nodes 0, 2 and 3 tie exactly; the lower
    indices 0 and 2 are kept, and level 0 then keeps blocks 3 and 9. Exhaustive
    top-2 with the lower-index rule gives the same {3, 9}.
    """
    D, block = 8, 4
    k = np.zeros((16 * block, D), dtype=np.float32)
    pattern = np.array([1.0, 0.5, 0, 0, 0, 0, 0, 0], dtype=np.float32)
    for j in (3, 9, 12):
        k[j * block:(j + 1) * block] = pattern
    q = np.zeros((1, block, D), dtype=np.float32)
    q[0, :, 0] = 1.0
    return q, k, block, 4, 2, [3, 9]


def check_tie_rule(o):
    q, k, block, factor, topk, expect = tie_case()
    levels = o.build_pyramid(k, block, factor)
    qbar = o.query_summary(q, block)[0]
    r = o.select_blocks(qbar, levels, factor, topk, 15)
    assert r["idx"] == expect, r["idx"]
    assert r["margin"] == 0.0


# ----------------------------------------------------------------------------- P5/P6 exhaustive

def brute_topk(qbar, k_plane, block, topk, last):
    """Exhaustive top-K over the eligible level-0 blocks in fp64, lower index on ties; returns (idx, margin)."""
    nb = k_plane.shape[0] // block
    means = k_plane.astype(np.float64).reshape(nb, block, -1).mean(axis=1)
    s = means[:last + 1] @ qbar.astype(np.float64)
    order = sorted(range(last + 1), key=lambda j: (-s[j], j))
    if last + 1 <= topk:
        return sorted(order), math.inf
    a, b = s[order[topk - 1]], s[order[topk]]
    return sorted(order[:topk]), (a - b) / max(abs(a), abs(b), 1e-30)


def check_full_budgets(o, seed=13, causal=True, N=1024, block=16, factor=4, topk=8, D=16):
    """Descent with K_l = n_l at every coarse level equals exhaustive top-K at the finest level."""
    q, k, v = rand_qkv(seed, 1, 2, 1, N, N, D)
    levels = o.build_pyramid(k[0, 0], block, factor)
    budgets = [topk] + [lev.shape[0] for lev in levels[1:]]
    qbar = o.query_summary(q[0], block)
    nb = N // block
    checked = 0
    for i in range(nb):
        last = i if causal else nb - 1
        ref, margin = brute_topk(qbar[i], k[0, 0], block, topk, last)
        if margin < 1e-4:
            continue
        got = o.select_blocks(qbar[i], levels, factor, topk, last, budgets)["idx"]
        assert got == ref, (i, got, ref)
        checked += 1
    assert checked > nb // 2


def check_single_level(o, seed=14, N=512, block=16, topk=5, D=16):
    """f >= nb: the pyramid is level 0 alone and the descent is a flat top-K."""
    q, k, v = rand_qkv(seed, 1, 1, 1, N, N, D)
    nb = N // block
    levels = o.build_pyramid(k[0, 0], block, nb)
    assert len(levels) == 1
    qbar = o.query_summary(q[0], block)
    for i in range(nb):
        ref, margin = brute_topk(qbar[i], k[0, 0], block, topk, nb - 1)
        if margin < 1e-4:
            continue
        assert o.select_blocks(qbar[i], levels, nb, topk, nb - 1)["idx"] == ref


# ----------------------------------------------------------------------------- P7 masked dense

def check_masked_dense(o, seed=15, N=256, block=16, D=32, causal=True):
    """Attention over chosen blocks equals fp64 dense attention with -inf outside those blocks."""
    q, k, v = rand_qkv(seed, 1, 1, 1, N, N, D)
    g = _rng(seed + 1)
    scale = 1.0 / math.sqrt(D)
    for i in (0, 3, 15):
        blocks = sorted(set(g.choice(i + 1, size=min(4, i + 1), replace=False).tolist()) | {i})
        rows = np.arange(i * block, (i + 1) * block)
        out, lse = o.attend(q[0, 0, rows], rows, k[0, 0], v[0, 0], blocks, block, causal, scale)
        allowed = np.zeros((block, N), dtype=bool)
        for j in blocks:
            allowed[:, j * block:(j + 1) * block] = True
        s = scale * (q[0, 0, rows].astype(np.float64) @ k[0, 0].astype(np.float64).T)
        keep = allowed & (np.arange(N)[None, :] <= rows[:, None] if causal else True)
        s = np.where(keep, s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        ref = (p @ v[0, 0].astype(np.float64)) / p.sum(axis=1, keepdims=True)
        assert np.abs(out - ref).max() < 1e-5, i
        ref_lse = s.max(axis=1) + np.log(p.sum(axis=1))
        assert np.abs(lse - ref_lse).max() < 1e-5, i


# ----------------------------------------------------------------------------- P8 merge

def check_merge(o, seed=16, N=512, block=16, D=32):
    """Splitting the selected blocks into parts and merging by LSE equals the unsplit result."""
    q, k, v = rand_qkv(seed, 1, 1, 1, N, N, D)
    rows = np.arange(20 * block, 21 * block)
    blocks = [1, 4, 7, 8, 13, 19, 20]
    scale = 1.0 / math.sqrt(D)
    full_o, full_l = o.attend(q[0, 0, rows], rows, k[0, 0], v[0, 0], blocks, block, True, scale)
    for parts in ([[1, 4], [7, 8, 13], [19, 20]], [[1], [4, 7, 8, 13, 19, 20]], [[20], [1, 4, 7], [8], [13, 19]]):
        outs, lses = zip(*[o.attend(q[0, 0, rows], rows, k[0, 0], v[0, 0], p, block, True, scale) for p in parts])
        mo, ml = o.merge_partials(list(outs), list(lses))
        assert np.abs(mo - full_o).max() < 1e-5
        assert np.abs(ml - full_l).max() < 1e-5
    # a partial whose rows are all masked carries lse = -inf and weight 0
    lse_a = np.array([0.3, -1.0]); lse_b = np.array([1.2, 0.5])
    oa = np.array([[1.0, 0.0], [0.0, 2.0]]); ob = np.array([[0.0, 1.0], [4.0, 0.0]])
    mo, ml = o.merge_partials([oa, ob], [lse_a, lse_b])
    wa = np.exp(lse_a) / (np.exp(lse_a) + np.exp(lse_b))
    assert np.allclose(mo, wa[:, None] * oa + (1 - wa)[:, None] * ob, atol=1e-12)
    assert np.allclose(ml, np.log(np.exp(lse_a) + np.exp(lse_b)), atol=1e-12)


# ----------------------------------------------------------------------------- causality (R6)

def check_causal_partial_node(o, seed=17, N=1024, block=16, factor=4, D=16):
    """A node straddling the query block is summarised by the mean of its eligible keys only."""
    g = _rng(seed)
    k = _bf16_exact(g.standard_normal((N, D)))
    levels = o.build_pyramid(k, block, factor)
    nb = N // block
    for last in (0, 5, 17, 33, 62):
        for l in range(len(levels)):
            width = factor ** l
            c = last // width
            lo = c * width
            hi = min((c + 1) * width, nb) - 1
            ref = k[lo * block:(last + 1) * block].astype(np.float64).mean(axis=0)
            got = o.node_value(levels, factor, l, c, last)
            assert np.allclose(got, ref, rtol=1e-5, atol=1e-5), (last, l)
            if hi <= last:
                assert np.array_equal(got, levels[l][c])


def check_causal_invariance(o, seed=18, N=1024, block=16, factor=4, topk=5, D=16):
    """Changing keys after a query block changes neither its selection nor its output."""
    q, k, v = rand_qkv(seed, 1, 2, 1, N, N, D)
    base = o.forward(q, k, v, block, factor, topk, True)
    i = 21
    k2, v2 = k.copy(), v.copy()
    g = _rng(seed + 5)
    k2[0, 0, (i + 1) * block:] = _bf16_exact(g.standard_normal(((N // block - i - 1) * block, D)) * 4)
    v2[0, 0, (i + 1) * block:] = _bf16_exact(g.standard_normal(((N // block - i - 1) * block, D)))
    # plant a strong future block: a leak through a straddling node would pull its parent in
    k2[0, 0, (i + 2) * block:(i + 3) * block] = 50.0 * q[0].mean(axis=(0, 1))[None, :]
    alt = o.forward(q, k2, v2, block, factor, topk, True)
    for j in range(i + 1):
        assert np.array_equal(base["idx"][0, 0, j], alt["idx"][0, 0, j]), j
    rows = slice(0, (i + 1) * block)
    assert np.array_equal(base["O"][0, :, rows], alt["O"][0, :, rows])


# ----------------------------------------------------------------------------- P10 work bound

def check_work_bound(o, seed=19, N=4096, block=16, factor=4, topk=8, D=16):
    """Candidates scored per query block stay within n_top + sum_l K_l f (O(N log N))."""
    q, k, v = rand_qkv(seed, 1, 1, 1, N, N, D)
    levels = o.build_pyramid(k[0, 0], block, factor)
    qbar = o.query_summary(q[0], block)
    bound = levels[-1].shape[0] + (len(levels) - 1) * topk * factor
    nb = N // block
    for i in (0, 7, 100, nb - 1):
        r = o.select_blocks(qbar[i], levels, factor, topk, i)
        assert r["n_scored"] <= bound, (i, r["n_scored"], bound)
    r = o.select_blocks(qbar[nb - 1], levels, factor, topk, nb - 1)
    assert r["n_scored"] < nb


# ----------------------------------------------------------------------------- R16 forced blocks

def brute_topk_excluding(qbar, k_plane, block, topk, last, excluded):
    """Exhaustive top-K over eligible level-0 blocks not in `excluded` (fp64, lower index on ties)."""
    nb = k_plane.shape[0] // block
    means = k_plane.astype(np.float64).reshape(nb, block, -1).mean(axis=1)
    s = means[:last + 1] @ qbar.astype(np.float64)
    pool = [j for j in range(last + 1) if j not in excluded]
    order = sorted(pool, key=lambda j: (-s[j], j))
    if len(pool) <= topk:
        return sorted(order), math.inf
    if topk == 0:
        return [], math.inf
    a, b = s[order[topk - 1]], s[order[topk]]
    return sorted(order[:topk]), (a - b) / max(abs(a), abs(b), 1e-30)


def check_forced_full_budgets(o, forced, seed=21, causal=True, N=1024, block=16, factor=4, topk=8, D=16):
    """With K_l = n_l at the coarse levels, a selection with forced blocks F equals F plus the
    exhaustive top-(K - |F|) of the other eligible blocks."""
    q, k, v = rand_qkv(seed, 1, 2, 1, N, N, D)
    levels = o.build_pyramid(k[0, 0], block, factor)
    budgets = [topk] + [lev.shape[0] for lev in levels[1:]]
    qbar = o.query_summary(q[0], block)
    nb = N // block
    checked = 0
    for i in range(nb):
        last = i if causal else nb - 1
        fset = []
        if forced & 1:
            fset.append(0)
        if forced & 2 and i not in fset:
            fset.append(i)
        fset = fset[:topk]
        rest, margin = brute_topk_excluding(qbar[i], k[0, 0], block, topk - len(fset), last, fset)
        if margin < 1e-4:
            continue
        got = o.select_blocks(qbar[i], levels, factor, topk, last, budgets, o.forced_set(forced, i, topk))["idx"]
        assert got == sorted(rest + fset), (i, got, sorted(rest + fset))
        checked += 1
    assert checked > nb // 2


def check_forced_cardinality(o, seed=22, topk=3, N=512, block=16, factor=4):
    """Every row keeps min(K, eligible) distinct sorted blocks and holds its forced blocks."""
    q, k, v = rand_qkv(seed, 1, 2, 1, N, N, 16)
    nb = N // block
    for forced in (1, 2, 3):
        res = o.forward(q, k, v, block, factor, topk, True, forced=forced)
        for i in range(nb):
            row = res["idx"][0, 0, i]
            valid = row[row >= 0]
            assert len(valid) == min(topk, i + 1), (forced, i, row)
            assert np.all(np.diff(valid) > 0) and valid.max() <= i
            if forced & 1:
                assert 0 in valid
            if forced & 2:
                assert i in valid


def check_forced_budget_edges(o, seed=23, N=256, block=16, factor=4):
    """K = 1 with sink and local: the sink alone; K = 2: the sink and the query's own block."""
    q, k, v = rand_qkv(seed, 1, 1, 1, N, N, 16)
    nb = N // block
    r1 = o.forward(q, k, v, block, factor, 1, True, forced=3)["idx"][0, 0]
    assert np.all(r1[:, 0] == 0)
    r2 = o.forward(q, k, v, block, factor, 2, True, forced=3)["idx"][0, 0]
    for i in range(nb):
        assert r2[i].tolist() == ([0, -1] if i == 0 else [0, i]), (i, r2[i])


# ----------------------------------------------------------------------------- R17 spare KV capacity

def check_capacity_pyramid_means(o, seed=24, n_cap=37, block=16, factor=4, D=12):
    """Every node of a capacity pyramid is the fp64 mean of the keys it covers among the first
    kv_len rows, and 0 when it covers none of them."""
    rng = _rng(seed)
    k = _bf16_exact(rng.standard_normal((n_cap * block, D)))
    for nv in (0, 1, 5, 16, 21, n_cap):
        levels = o.build_pyramid_capacity(k, block, factor, nv * block)
        width = 1
        for l, lev in enumerate(levels):
            for c in range(lev.shape[0]):
                lo, hi = c * width * block, min((c + 1) * width, nv) * block
                expect = k[lo:hi].astype(np.float64).mean(axis=0) if hi > lo else np.zeros(D)
                assert np.allclose(lev[c], expect, atol=1e-5, rtol=1e-5), (nv, l, c)
            width *= factor


def check_capacity_decode_equals_exact(o, seed=25, n_cap=64, nv=39, block=16, factor=4, topk=5, D=16):
    """Decode on a cache with spare capacity selects what decode on the exact-length cache
    selects (outside near-ties) and gives the same attention."""
    q, k, v = rand_qkv(seed, 2, 4, 2, 1, n_cap * block, D)
    kv_len = nv * block
    cap = o.forward(q, k, v, block, factor, topk, False, kv_len=kv_len)
    exact = o.forward(q, k[:, :, :kv_len], v[:, :, :kv_len], block, factor, topk, False)
    same = np.all(cap["idx"] == exact["idx"], axis=-1)
    near = (cap["margin"] < 1e-3) | (exact["margin"] < 1e-3)
    assert np.all(same | near)
    assert same.sum() >= same.size // 2
    for b in range(2):
        for h in range(4):
            if same[b, h // 2, 0]:
                assert np.allclose(cap["O"][b, h], exact["O"][b, h], atol=1e-6)
    # the spare rows are never read: garbage there changes nothing
    k2, v2 = k.copy(), v.copy()
    k2[:, :, kv_len:] = 1e4
    v2[:, :, kv_len:] = -1e4
    cap2 = o.forward(q, k2, v2, block, factor, topk, False, kv_len=kv_len)
    assert np.array_equal(cap2["idx"], cap["idx"]) and np.array_equal(cap2["O"], cap["O"])


# ----------------------------------------------------------------------------- backward

def _loss_sparse(o, Q, K, V, W, idx, block, causal, scale):
    """sum(O * W) of the sparse attention step, from the fp64 dense softmax with a mask that
    keeps each query block's selected keys (an independent route to the same forward)."""
    B, Hq, N, D = Q.shape
    g = Hq // K.shape[1]
    total = 0.0
    for b in range(B):
        for h in range(Hq):
            allowed = np.zeros((N, N), dtype=bool)
            for i in range(N // block):
                for j in idx[b, h // g, i]:
                    if j >= 0:
                        allowed[i * block:(i + 1) * block, j * block:(j + 1) * block] = True
            out, _ = o.dense_attention(Q[b, h], np.arange(N), K[b, h // g], V[b, h // g], causal, scale, allowed)
            total += float((out * W[b, h]).sum())
    return total


def check_backward_finite_differences(o, seed=26, causal=True, B=1, Hq=2, Hkv=1, nb=4, block=8, D=8, topk=2):
    """dQ, dK, dV of the sparse step match central finite differences of sum(O * dO) taken
    through the fp64 dense forward with the selection as a mask."""
    rng = _rng(seed)
    N = nb * block
    Q, K, V = (rng.standard_normal((B, h, N, D)) for h in (Hq, Hkv, Hkv))
    W = rng.standard_normal((B, Hq, N, D))
    idx = np.full((B, Hkv, nb, topk), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            for i in range(nb):
                elig = i + 1 if causal else nb
                sel = np.sort(rng.choice(elig, size=min(topk, elig), replace=False))
                idx[b, h, i, :len(sel)] = sel
    scale = 0.7
    g = o.backward(Q, K, V, W, idx, block, causal, scale)
    eps = 1e-6
    for name, T in (("dQ", Q), ("dK", K), ("dV", V)):
        for _ in range(12):
            pos = tuple(int(rng.integers(0, n)) for n in T.shape)
            old = T[pos]
            T[pos] = old + eps
            lp = _loss_sparse(o, Q, K, V, W, idx, block, causal, scale)
            T[pos] = old - eps
            lm = _loss_sparse(o, Q, K, V, W, idx, block, causal, scale)
            T[pos] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[name][pos]) < 1e-6 + 1e-5 * abs(fd), (name, pos, fd, g[name][pos])


def check_backward_constant_values(o, seed=27, N=64, block=16, D=8):
    """When every key has the same value row, O does not depend on the scores: dQ = dK = 0,
    and dV sums P^T dO, so the value row's total gradient is the sum of dO over the queries."""
    rng = _rng(seed)
    Q = rng.standard_normal((1, 1, N, D))
    K = rng.standard_normal((1, 1, N, D))
    V = np.tile(rng.standard_normal(D), (1, 1, N, 1))
    W = rng.standard_normal((1, 1, N, D))
    nb = N // block
    idx = np.array([[[list(range(i + 1)) + [-1] * (nb - i - 1) for i in range(nb)]]], dtype=np.int32)
    g = o.backward(Q, K, V, W, idx, block, True, 0.5)
    assert np.abs(g["dQ"]).max() < 1e-12 and np.abs(g["dK"]).max() < 1e-12
    assert np.allclose(g["dV"][0, 0].sum(axis=0), W[0, 0].sum(axis=0), atol=1e-10)


def check_backward_gqa_sum(o, seed=28, N=64, block=16, D=8, topk=2):
    """A KV head's dK and dV are the sums over its query heads of each head's own gradients."""
    rng = _rng(seed)
    Q = rng.standard_normal((1, 2, N, D))
    K = rng.standard_normal((1, 1, N, D))
    V = rng.standard_normal((1, 1, N, D))
    W = rng.standard_normal((1, 2, N, D))
    nb = N // block
    idx = np.array([[[sorted(rng.choice(i + 1, size=min(topk, i + 1), replace=False).tolist())
                      + [-1] * (topk - min(topk, i + 1)) for i in range(nb)]]], dtype=np.int32)
    both = o.backward(Q, K, V, W, idx, block, True)
    one = [o.backward(Q[:, h:h + 1], K, V, W[:, h:h + 1], idx, block, True) for h in range(2)]
    assert np.allclose(both["dK"], one[0]["dK"] + one[1]["dK"], atol=1e-12)
    assert np.allclose(both["dV"], one[0]["dV"] + one[1]["dV"], atol=1e-12)
    assert np.allclose(both["dQ"][:, 1:], one[1]["dQ"], atol=1e-12)


ALL_PINS = {
    "pyramid_means": check_pyramid_means,
    "query_summary": check_query_summary,
    "dense_reduction_causal": lambda o: check_dense_reduction(o, causal=True),
    "dense_reduction_noncausal": lambda o: check_dense_reduction(o, causal=False, Hq=2, Hkv=2),
    "dense_reduction_per_qhead": lambda o: check_dense_reduction(o, causal=True, per_qhead=True),
    "dense_reduction_decode": lambda o: check_dense_reduction(o, decode=True, B=2),
    "cardinality_causal": lambda o: check_cardinality(o, causal=True),
    "cardinality_noncausal": lambda o: check_cardinality(o, causal=False),
    "tie_rule": check_tie_rule,
    "full_budgets_causal": lambda o: check_full_budgets(o, causal=True),
    "full_budgets_noncausal": lambda o: check_full_budgets(o, causal=False),
    "single_level": check_single_level,
    "masked_dense": check_masked_dense,
    "merge": check_merge,
    "causal_partial_node": check_causal_partial_node,
    "causal_invariance": check_causal_invariance,
    "work_bound": check_work_bound,
    "forced_sink_full_budgets": lambda o: check_forced_full_budgets(o, 1),
    "forced_local_full_budgets_noncausal": lambda o: check_forced_full_budgets(o, 2, causal=False),
    "forced_both_full_budgets": lambda o: check_forced_full_budgets(o, 3),
    "forced_cardinality": check_forced_cardinality,
    "forced_budget_edges": check_forced_budget_edges,
    "capacity_pyramid_means": check_capacity_pyramid_means,
    "capacity_decode_equals_exact": check_capacity_decode_equals_exact,
    "backward_finite_differences_causal": lambda o: check_backward_finite_differences(o, causal=True),
    "backward_finite_differences_noncausal_gqa": lambda o: check_backward_finite_differences(
        o, seed=29, causal=False, B=2, Hq=4, Hkv=2, nb=3, topk=2),
    "backward_constant_values": check_backward_constant_values,
    "backward_gqa_sum": check_backward_gqa_sum,
}
