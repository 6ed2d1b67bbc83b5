"""GPU path vs the CPU oracle on seeded inputs, through the C ABI.

Small shapes: every kernel variant (head dims 64/128, blocks 64/128, 1 or 2
tensor-core tiles per CTA, split head groups), causal and not, shared and
per-query-head selection, ragged pyramids, decode, ties and edge cases.
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
W = workloads.Workload

SMALL = {
    "tiny": workloads.WORKLOADS["tiny"],
    "gqa4-causal-ragged": W("gqa4-causal-ragged", 1, 8, 2, 37 * 64, 37 * 64, 128, 64, 4, 6, 1, "iid", 11),
    "gqa2-causal": W("gqa2-causal", 1, 4, 2, 20 * 64, 20 * 64, 128, 64, 4, 5, 1, "iid", 12),
    "gqa8-d64-causal": W("gqa8-d64-causal", 1, 16, 2, 24 * 64, 24 * 64, 64, 64, 4, 4, 1, "iid", 13),
    "mha-d128-b64-causal": W("mha-d128-b64-causal", 1, 3, 3, 33 * 64, 33 * 64, 128, 64, 4, 7, 1, "clustered", 14),
    "mha-d64-b128-f8": W("mha-d64-b128-f8", 1, 2, 2, 70 * 128, 70 * 128, 64, 128, 8, 9, 0, "iid", 15),
    "mha-d128-b128-f8-causal": W("mha-d128-b128-f8-causal", 1, 2, 2, 66 * 128, 66 * 128, 128, 128, 8, 10, 1,
                                 "clustered", 16),
    "gqa4-d64-noncausal": W("gqa4-d64-noncausal", 2, 8, 2, 18 * 64, 18 * 64, 64, 64, 4, 5, 0, "iid", 17),
    "gqa4-needle": W("gqa4-needle", 1, 8, 2, 256 * 64, 256 * 64, 128, 64, 4, 16, 1, "needle", 18),
    # fewer query blocks than the dense-scoring threshold: the sparse descent runs for prefill (as it
    # does for every prefill of at most 592 selection rows, the shapes above included)
    "gqa4-causal-short": W("gqa4-causal-short", 2, 8, 2, 13 * 64, 13 * 64, 128, 64, 4, 3, 1, "iid", 23),
    # more than 592 selection rows: the dense scoring and the warp descent
    "gqa2-dense-640": W("gqa2-dense-640", 2, 16, 8, 40 * 64, 40 * 64, 128, 64, 4, 6, 1, "iid", 24),
    "mha-d64-b128-dense": W("mha-d64-b128-dense", 2, 8, 8, 40 * 128, 40 * 128, 64, 128, 8, 9, 1, "clustered", 25),
    "decode-gqa4": W("decode-gqa4", 3, 8, 2, 1, 45 * 64, 128, 64, 4, 9, 0, "clustered", 19),
    "decode-d64-b128": W("decode-d64-b128", 2, 4, 4, 1, 40 * 128, 64, 128, 8, 6, 0, "iid", 20),
}
PER_QHEAD = {
    "perq-gqa4-causal": W("perq-gqa4-causal", 1, 8, 2, 21 * 64, 21 * 64, 128, 64, 4, 5, 1, "iid", 21),
    "perq-decode": W("perq-decode", 2, 8, 2, 1, 30 * 64, 128, 64, 4, 7, 0, "iid", 22),
    "perq-gqa4-dense": W("perq-gqa4-dense", 1, 16, 4, 40 * 64, 40 * 64, 128, 64, 4, 5, 1, "iid", 26),
}


def _run(w, cuda_device, per_qhead=False, topk=None, forced=0):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    if topk is not None:
        w = w.replace(topk=topk)
    shape = pisa.Shape.of(w, select_per_qhead=int(per_qhead), forced_blocks=forced)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    pyr = pisa.build_pyramid(shape, k)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, w.name)
    assert pisa.last_launch_count() >= 1
    Q, K, V = (gu.host_f32(x) for x in (q, k, v))
    ref = oracle.forward(Q, K, V, w.block, w.factor, w.topk, bool(w.causal), per_qhead=per_qhead, forced=forced)
    return shape, (Q, K, V), ref, gu.host_f32(o), gu.host_f32(lse), idx.cpu().numpy(), gu.host_f32(pyr)


@pytest.mark.parametrize("name", sorted(SMALL) + sorted(PER_QHEAD))
def test_forward_matches_oracle(name, cuda_device):
    per_q = name in PER_QHEAD
    w = PER_QHEAD[name] if per_q else SMALL[name]
    shape, (Q, K, V), ref, o, lse, idx, pyr = _run(w, cuda_device, per_qhead=per_q)
    import block_sparse_long_pisa_b200 as pisa
    _, offs = pisa.level_layout(shape)
    for b in range(w.batch):
        for h in range(w.heads_kv):
            gu.assert_pyramid_close(pyr[b, h], ref["pyramid"][b][h], offs)
    gu.check_selection(idx, ref, w, per_qhead=per_q)
    # attention checked against the oracle on the GPU's own selection
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, w.topk, bool(w.causal), per_qhead=per_q, idx_override=idx)
    gu.assert_output_close(o, ref_o["O"], lse, ref_o["lse"], name)
    if w.keys == "needle":
        for kvh in range(w.heads_kv):
            for (i, j) in workloads.needles(w, 0, kvh):
                assert j in idx[0, kvh, i], (kvh, i, j)


@pytest.mark.parametrize("name", ["gqa4-causal-ragged", "mha-d64-b128-f8", "decode-gqa4"])
def test_full_topk_is_dense_attention(name, cuda_device):
    """K >= number of blocks: every eligible block is selected and O is dense softmax attention."""
    w = SMALL[name]
    n0 = w.n_blocks
    shape, (Q, K, V), ref, o, lse, idx, _ = _run(w, cuda_device, topk=n0)
    g = w.group
    scale = 1.0 / math.sqrt(w.head_dim)
    for b in range(w.batch):
        for h in range(w.heads_q):
            pos = np.full(1, w.seq_kv - 1) if w.decode else np.arange(w.seq_q)
            d_o, d_l = oracle.dense_attention(Q[b, h], pos, K[b, h // g], V[b, h // g],
                                              bool(w.causal) and not w.decode, scale)
            gu.assert_output_close(o[b, h], d_o, lse[b, h], d_l, f"{name} b{b} h{h}")
    if not w.decode:
        nqb = w.seq_q // w.block
        for i in range(nqb):
            expect = list(range(i + 1)) if w.causal else list(range(n0))
            assert idx[0, 0, i, :len(expect)].tolist() == expect
            assert np.all(idx[0, 0, i, len(expect):] == -1)


@pytest.mark.parametrize("topk", [1, 2])
def test_small_topk(topk, cuda_device):
    w = SMALL["gqa4-causal-ragged"]
    shape, (Q, K, V), ref, o, lse, idx, _ = _run(w, cuda_device, topk=topk)
    gu.check_selection(idx, ref, w, topk=topk)
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, topk, True, idx_override=idx)
    gu.assert_output_close(o, ref_o["O"], lse, ref_o["lse"])


def _tie_inputs(device):
    """Key blocks 3, 9 and 12 identical and aligned with every query; all others zero.

    nb = 16, f = 4, K = 2: level-1 nodes 0, 2, 3 tie exactly; lower indices win
    at every level, so every query block must select exactly [3, 9].
    """
    import torch
    D, b, nb = 64, 64, 16
    k = torch.zeros((1, 1, nb * b, D), dtype=torch.bfloat16)
    pattern = torch.zeros(D)
    pattern[0], pattern[1] = 1.0, 0.5
    for j in (3, 9, 12):
        k[0, 0, j * b:(j + 1) * b] = pattern
    q = torch.zeros((1, 1, nb * b, D), dtype=torch.bfloat16)
    q[..., 0] = 1.0
    v = torch.randn((1, 1, nb * b, D), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    return [x.to(device) for x in (q, k, v)]


def test_exact_ties_go_to_lower_index(cuda_device):
    import block_sparse_long_pisa_b200 as pisa
    q, k, v = _tie_inputs(cuda_device)
    shape = pisa.Shape(1, 1, 1, 1024, 1024, 64, 64, 4, 2, causal=0)
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    idx = idx.cpu().numpy()
    assert np.all(idx[0, 0] == np.array([3, 9])), idx[0, 0]
    ref = oracle.forward(*(gu.host_f32(x) for x in (q, k, v)), 64, 4, 2, False)
    assert np.array_equal(idx, ref["idx"])


@pytest.mark.parametrize("name", ["gqa4-causal-ragged", "gqa2-dense-640"])
def test_full_budgets_equal_exhaustive_topk(name, cuda_device):
    """level_budget = n_l at every coarse level: the descent is exhaustive top-K (per-row and
    dense selection paths)."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL[name]
    shape = pisa.Shape.of(w)
    q, k = (gu.to_device(w, t, cuda_device) for t in ("q", "k"))
    sizes, _ = pisa.level_layout(shape)
    budgets = [w.topk] + sizes[1:]
    ws = pisa.new_workspace(shape, cuda_device)
    pyr = pisa.build_pyramid(shape, k)
    idx, marg = pisa.select_blocks(shape, q, pyr, ws, level_budget=budgets, margin=True)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws)
    idx = idx.cpu().numpy()
    Q, K = gu.host_f32(q), gu.host_f32(k)
    for h in range(w.heads_kv):
        qbar = oracle.query_summary(Q[0, h * w.group:(h + 1) * w.group], w.block)
        for i in range(w.seq_q // w.block):
            nb = i + 1
            means = K[0, h].astype(np.float64).reshape(-1, w.block, w.head_dim).mean(1)[:nb]
            s = means @ qbar[i].astype(np.float64)
            order = sorted(range(nb), key=lambda j: (-s[j], j))
            if nb > w.topk and (s[order[w.topk - 1]] - s[order[w.topk]]) < 1e-3 * abs(s[order[w.topk - 1]]):
                # a near-tie at the cut: the row must still be one the descent reaches
                levels = oracle.build_pyramid(K[0, h], w.block, w.factor)
                ok, why = oracle.selection_is_admissible(qbar[i], levels, w.factor, w.topk, i, idx[0, h, i],
                                                         budgets=budgets)
                assert ok, (h, i, why)
                continue
            expect = sorted(order[:w.topk])
            assert idx[0, h, i, :len(expect)].tolist() == expect, (h, i)


def test_sparse_attention_on_given_indices_and_bad_entries(cuda_device):
    """Arbitrary index rows: -1 padding is skipped, out-of-range or future blocks are skipped and reported,
    and a row with no valid block gives O = 0 and LSE = -inf."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL["gqa2-causal"]
    shape = pisa.Shape.of(w)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    nqb, K = w.seq_q // w.block, w.topk
    rng = np.random.Generator(np.random.PCG64(5))
    idx = np.full((1, w.heads_kv, nqb, K), -1, dtype=np.int32)
    for h in range(w.heads_kv):
        for i in range(nqb):
            n = int(rng.integers(1, min(K, i + 1) + 1))
            idx[0, h, i, :n] = np.sort(rng.choice(i + 1, size=n, replace=False))
    idx[0, 1, 4] = -1                       # empty row
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse = pisa.sparse_attention(shape, q, k, v, torch.from_numpy(idx).to(cuda_device), ws)
    st, _ = pisa.check_status(ws)
    assert st == pisa.OK
    Q, Kf, V = (gu.host_f32(x) for x in (q, k, v))
    ref = oracle.forward(Q, Kf, V, w.block, w.factor, K, True, idx_override=idx)
    o, lse = gu.host_f32(o), gu.host_f32(lse)
    g = w.group
    rows = slice(4 * w.block, 5 * w.block)
    assert np.all(o[0, g:2 * g, rows] == 0) and np.all(np.isneginf(lse[0, g:2 * g, rows]))
    keep = np.ones(o.shape, dtype=bool)
    keep[0, g:2 * g, rows] = False
    gu.assert_output_close(o[keep], ref["O"][keep], what="given indices")
    # a future block (causal) and an out-of-range block are skipped and reported
    bad = idx.copy()
    bad[0, 0, 2, -1] = 7                    # j > i for i = 2
    bad[0, 0, 3, -1] = 10 ** 6              # j >= n0
    o2, _ = pisa.sparse_attention(shape, q, k, v, torch.from_numpy(bad).to(cuda_device), ws)
    st, _ = pisa.check_status(ws)
    assert st == pisa.ERR_BAD_INDEX
    o2 = gu.host_f32(o2)
    np.testing.assert_array_equal(o2[0, :g, 2 * 64:4 * 64], o[0, :g, 2 * 64:4 * 64])
    assert pisa.check_status(ws)[0] == pisa.OK  # cleared after the read


def test_decode_split_merge_matches_unsplit(cuda_device):
    """Many splits (K = 40 blocks -> 10 splits) merged by LSE equal the oracle's single softmax."""
    w = W("decode-many-splits", 2, 4, 1, 1, 96 * 64, 128, 64, 4, 40, 0, "iid", 31)
    shape, (Q, K, V), ref, o, lse, idx, _ = _run(w, cuda_device)
    gu.check_selection(idx, ref, w)
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, idx_override=idx)
    gu.assert_output_close(o, ref_o["O"], lse, ref_o["lse"])


def test_repeated_calls_are_deterministic(cuda_device):
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL["gqa4-causal-ragged"]
    shape = pisa.Shape.of(w)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o1, l1, i1 = pisa.forward(shape, q, k, v, ws, idx=True)
    o2, l2, i2 = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    assert (i1 == i2).all() and (o1 == o2).all() and (l1 == l2).all()


@pytest.mark.parametrize("causal", [0, 1])
def test_growing_logits_rescale_running_max(causal, cuda_device):
    """Key blocks scaled by factors that jump from block to block, with every block selected: the
    row maximum grows past the lazy-rescale threshold at many key groups, sometimes in one
    64-key half of a group and sometimes in both, so the running max, O and the row sums are
    rescaled mid-row. The result must still be dense softmax attention."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    B, Hq, Hkv, nb, D, blk = 1, 8, 2, 24, 128, 64
    N = nb * blk
    gen = torch.Generator().manual_seed(41)
    scale = torch.empty(nb).uniform_(0.3, 1.0, generator=gen) * torch.linspace(0.5, 4.0, nb)
    scale[torch.randperm(nb, generator=gen)[:4]] *= 2.5
    q = torch.randn((B, Hq, N, D), generator=gen)
    k = torch.randn((B, Hkv, N, D), generator=gen) * scale.repeat_interleave(blk)[None, None, :, None]
    v = torch.randn((B, Hkv, N, D), generator=gen)
    q, k, v = (x.to(torch.bfloat16).to(cuda_device) for x in (q, k, v))
    shape = pisa.Shape(B, Hq, Hkv, N, N, D, blk, 4, nb, causal=causal)
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws)
    Q, K, V = (gu.host_f32(x) for x in (q, k, v))
    o, lse = gu.host_f32(o), gu.host_f32(lse)
    g = Hq // Hkv
    sc = 1.0 / math.sqrt(D)
    for h in range(Hq):
        d_o, d_l = oracle.dense_attention(Q[0, h], np.arange(N), K[0, h // g], V[0, h // g], bool(causal), sc)
        gu.assert_output_close(o[0, h], d_o, lse[0, h], d_l, f"causal={causal} h{h}")


FORCED_CASES = [("tiny", 3), ("gqa4-causal-ragged", 1), ("gqa4-causal-ragged", 2), ("gqa4-causal-ragged", 3),
                ("gqa4-causal-short", 3), ("decode-gqa4", 3), ("decode-d64-b128", 2), ("perq-gqa4-causal", 3),
                ("mha-d128-b128-f8-causal", 1), ("gqa2-dense-640", 3), ("perq-gqa4-dense", 3),
                ("mha-d64-b128-dense", 2)]


@pytest.mark.parametrize("name,forced", FORCED_CASES)
def test_forced_blocks_match_oracle(name, forced, cuda_device):
    """Selection variants (attention sink, local block, both) on both selection paths (dense
    prefill scoring, per-query-block descent for short prefill and decode) and per-query-head."""
    per_q = name in PER_QHEAD
    w = PER_QHEAD[name] if per_q else SMALL[name]
    shape, (Q, K, V), ref, o, lse, idx, _ = _run(w, cuda_device, per_qhead=per_q, forced=forced)
    gu.check_selection(idx, ref, w, per_qhead=per_q, forced=forced)
    nqb = 1 if w.decode else w.seq_q // w.block
    n0 = w.n_blocks
    for i in range(nqb):
        local = n0 - 1 if w.decode else i
        rows = idx[:, :, i]
        if forced & 1:
            assert np.all((rows == 0).any(axis=-1))
        if forced & 2:
            assert np.all((rows == local).any(axis=-1))
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, w.topk, bool(w.causal), per_qhead=per_q, idx_override=idx)
    gu.assert_output_close(o, ref_o["O"], lse, ref_o["lse"], name)


@pytest.mark.parametrize("topk", [1, 2])
def test_forced_blocks_fill_the_budget(topk, cuda_device):
    """K no larger than the forced blocks: K = 1 keeps the sink alone, K = 2 the sink and the
    query's own block, on both selection paths."""
    for name in ("gqa4-causal-ragged", "gqa4-causal-short", "gqa2-dense-640"):
        w = SMALL[name]
        _, _, ref, _, _, idx, _ = _run(w, cuda_device, topk=topk, forced=3)
        assert np.array_equal(idx, ref["idx"]), name
        nqb = w.seq_q // w.block
        for i in range(nqb):
            expect = [0] if topk == 1 else ([0, -1] if i == 0 else [0, i])
            assert np.all(idx[:, :, i] == np.array(expect)), (name, i)


def _capacity_cache(w, cap, cuda_device):
    """K and V of a decode workload placed in a cache of `cap` rows; the spare rows hold NaN,
    so any read past the keys would show in the results."""
    import torch
    k, v = (gu.to_device(w, t, cuda_device) for t in ("k", "v"))
    out = []
    for x in (k, v):
        c = torch.full((w.batch, w.heads_kv, cap, w.head_dim), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        c[:, :, :w.seq_kv] = x
        out.append(c)
    return out


def test_capacity_pyramid_build_and_append(cuda_device):
    """A cache with spare capacity: the pyramid built at one length matches the oracle; appending
    blocks (one at a time and several at once) gives the pyramid a build at the new length gives,
    bit for bit."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL["decode-gqa4"]                  # 45 blocks of 64 keys
    cap = 64 * 64
    kc, _ = _capacity_cache(w, cap, cuda_device)
    kc = torch.nan_to_num(kc, nan=0.0)        # rows past a length are never averaged, but keep them finite
    K = gu.host_f32(kc)

    def shape_at(n):
        return pisa.Shape(w.batch, w.heads_q, w.heads_kv, 1, n, w.head_dim, w.block, w.factor, w.topk,
                          kv_capacity=cap)
    lengths = [17 * 64, 18 * 64, 19 * 64, 30 * 64, 45 * 64]
    pyr = pisa.build_pyramid(shape_at(lengths[0]), kc)
    _, offs = pisa.level_layout(shape_at(lengths[0]))
    for n_old, n_new in zip(lengths, lengths[1:]):
        pisa.append_pyramid(shape_at(n_new), kc, pyr, n_old)
        fresh = pisa.build_pyramid(shape_at(n_new), kc)
        torch.cuda.synchronize()
        assert torch.equal(pyr, fresh), (n_old, n_new)
        got = gu.host_f32(pyr)
        for b in range(w.batch):
            for h in range(w.heads_kv):
                ref = oracle.build_pyramid_capacity(K[b, h], w.block, w.factor, n_new)
                gu.assert_pyramid_close(got[b, h], ref, offs)


def test_pyramid_top_levels_past_the_shared_memory_limit(cuda_device):
    """One plane of 21,000 key blocks: above the 64-block subtrees the pyramid has 441 rows
    (225 KB at head dim 128), more than the top-level kernel keeps in shared memory, so it forms
    those levels from global memory. The two-launch build equals the per-level path (an append
    from an empty cache) bit for bit, and the oracle within the pyramid tolerance."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    n0, D = 21000, 128
    shape = pisa.Shape(1, 1, 1, n0 * 64, n0 * 64, D, 64, 4, 64, causal=1)
    sizes, offs = pisa.level_layout(shape)
    assert sum(sizes[3:]) * D * 4 > 160 * 1024
    gen = torch.Generator(device=cuda_device).manual_seed(1234)
    k = torch.randn((1, 1, n0 * 64, D), generator=gen, device=cuda_device).to(torch.bfloat16)
    built = pisa.build_pyramid(shape, k)
    appended = torch.zeros_like(built)
    pisa.append_pyramid(shape, k, appended, 0)
    torch.cuda.synchronize()
    assert torch.equal(built, appended)
    levels = oracle.build_pyramid(gu.host_f32(k)[0, 0], 64, 4)
    gu.assert_pyramid_close(gu.host_f32(built)[0, 0], levels, offs)


@pytest.mark.parametrize("forced", [0, 3])
def test_decode_with_spare_capacity(forced, cuda_device):
    """Decode over a partly filled cache (spare rows hold NaN) matches the oracle's decode at the
    cache's current length."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL["decode-gqa4"]
    cap = 80 * 64
    kc, vc = _capacity_cache(w, cap, cuda_device)
    q = gu.to_device(w, "q", cuda_device)
    shape = pisa.Shape.of(w, kv_capacity=cap, forced_blocks=forced)
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, kc, vc, ws, idx=True)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws)
    Q, K, V = gu.host_f32(q), gu.host_f32(kc), gu.host_f32(vc)
    ref = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, kv_len=w.seq_kv, forced=forced)
    idx = idx.cpu().numpy()
    gu.check_selection(idx, ref, w, forced=forced, kv_len=w.seq_kv)
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, kv_len=w.seq_kv, idx_override=idx)
    o, lse = gu.host_f32(o), gu.host_f32(lse)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    gu.assert_output_close(o, ref_o["O"], lse, ref_o["lse"], "spare capacity")


@pytest.mark.parametrize("name,units", [("gqa4-d64-noncausal", 3), ("gqa4-causal-ragged", 8), ("decode-gqa4", 4)])
def test_session_pipelined_host_forward(name, units, cuda_device):
    """Session.forward with pinned host buffers splits the (batch, KV head) planes into ranges and
    overlaps their copies with the computation of other ranges: prefill results equal one
    pisa_forward on the whole device tensors bit for bit; decode (whose split count depends on the
    rows per call) matches the oracle on the device call's selection."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL[name]
    shape = pisa.Shape.of(w)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o_ref, _, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    sess = pisa.Session(shape, cuda_device, units=units)
    assert len(sess.ranges) == min(units, w.batch * w.heads_kv)
    for _ in range(2):
        out = sess.forward(hq, hk, hv)
        torch.cuda.synchronize()
        pisa.raise_on_device_error(sess.unit_ws)
        if w.decode:
            Q, K, V = (gu.host_f32(x) for x in (q, k, v))
            ref = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, idx_override=idx.cpu().numpy())
            gu.assert_output_close(out.float().numpy(), ref["O"], what=name)
        else:
            assert torch.equal(out, o_ref.cpu()), name


@pytest.mark.parametrize("name", ["gqa4-d64-noncausal", "gqa4-causal-ragged"])
def test_units_shard_without_changing_results(name, cuda_device):
    """The premise of sharding over GPUs: (batch, KV head) units are independent. A call on any
    subset of the units (one sequence of the batch, a range of KV heads with their query heads)
    gives exactly, bit for bit, what the call on the whole batch gives for those units, so a rank
    that processes its shard returns the single-process output for it."""
    import dataclasses
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = SMALL[name]
    if w.batch == 1:
        w = w.replace(batch=2)
    shape = pisa.Shape.of(w)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    o, lse, idx = pisa.forward(shape, q, k, v, pisa.new_workspace(shape, cuda_device), idx=True)
    g = w.heads_q // w.heads_kv
    shards = [(b, h0, h1) for b in range(w.batch) for (h0, h1) in ((0, 1), (1, w.heads_kv))]
    for b, h0, h1 in shards:
        sub = dataclasses.replace(shape, batch=1, heads_q=(h1 - h0) * g, heads_kv=h1 - h0)
        qs = q[b:b + 1, h0 * g:h1 * g].contiguous()
        ks, vs = k[b:b + 1, h0:h1].contiguous(), v[b:b + 1, h0:h1].contiguous()
        os_, ls, is_ = pisa.forward(sub, qs, ks, vs, pisa.new_workspace(sub, cuda_device), idx=True)
        torch.cuda.synchronize()
        assert torch.equal(os_, o[b:b + 1, h0 * g:h1 * g]), (name, b, h0, h1)
        assert torch.equal(ls, lse[b:b + 1, h0 * g:h1 * g]), (name, b, h0, h1)
        assert torch.equal(is_, idx[b:b + 1, h0:h1]), (name, b, h0, h1)
