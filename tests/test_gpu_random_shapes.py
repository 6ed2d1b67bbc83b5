"""A seeded sweep over random supported shapes, GPU against the oracle through the C ABI.

The named cases of the other GPU tests pick one shape per kernel variant; this sweep draws
shapes at random inside the library's limits (head dim 64/128, key blocks 64/128, pooling
factor 2/4/8, group size 1-8, 1-2 KV heads and sequences, 2-40 key blocks so that pyramids are
ragged, K from 1 to beyond the eligible blocks, causal or not, prefill or decode, shared or
per-query-head selection, forced sink and local blocks) so that a dispatch or index error tied
to one combination shows. Each shape: pyramid planes, selection rows (equal to the oracle's or
an admissible near-tie resolution), O and LSE on the GPU's own selection; every third prefill
shape also runs the backward against the oracle's gradients. A second test runs the selection of
every shape under random per-level budgets; a third puts the decode shapes in a cache with spare
capacity and checks the incremental pyramid against a fresh build.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
REL_MAX, REL_MEAN = 2e-2, 1e-3   # backward tolerance, as in test_gpu_backward.py


def _draw(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for k in range(n):
        D = int(rng.choice([64, 128]))
        blk = int(rng.choice([64, 128]))
        f = int(rng.choice([2, 4, 8]))
        hkv = int(rng.integers(1, 3))
        decode = bool(rng.random() < 0.25)
        g = int(rng.choice([1, 2, 3, 4, 8]))
        nb = int(rng.integers(2, 41))
        causal = 0 if decode else int(rng.random() < 0.6)
        topk = int(rng.integers(1, nb + 3))
        batch = int(rng.integers(1, 3))
        per_q = bool(rng.random() < 0.25)
        forced = int(rng.choice([0, 0, 1, 2, 3]))
        keys = str(rng.choice(["iid", "clustered"]))
        w = workloads.Workload(f"rand{k}-d{D}-b{blk}-f{f}-g{g}-nb{nb}-k{topk}{'-dec' if decode else ''}"
                               f"{'-causal' if causal else ''}{'-perq' if per_q else ''}-forced{forced}",
                               batch, hkv * g, hkv, 1 if decode else nb * blk, nb * blk, D, blk, f, topk, causal,
                               keys, 700 + k)
        cases.append((w, per_q, forced))
    return cases


CASES = _draw()


@pytest.mark.parametrize("case", range(len(CASES)), ids=[c[0].name for c in CASES])
def test_random_shape_matches_oracle(case, cuda_device):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w, per_q, forced = CASES[case]
    shape = pisa.Shape.of(w, select_per_qhead=int(per_q), forced_blocks=forced)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    pyr = pisa.build_pyramid(shape, k)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, w.name)
    Q, K, V = (gu.host_f32(x) for x in (q, k, v))
    ref = oracle.forward(Q, K, V, w.block, w.factor, w.topk, bool(w.causal), per_qhead=per_q, forced=forced)
    _, offs = pisa.level_layout(shape)
    pyr_h = gu.host_f32(pyr)
    for b in range(w.batch):
        for h in range(w.heads_kv):
            gu.assert_pyramid_close(pyr_h[b, h], ref["pyramid"][b][h], offs)
    idx_h = idx.cpu().numpy()
    gu.check_selection(idx_h, ref, w, per_qhead=per_q, forced=forced)
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, w.topk, bool(w.causal), per_qhead=per_q,
                           idx_override=idx_h)
    gu.assert_output_close(gu.host_f32(o), ref_o["O"], gu.host_f32(lse), ref_o["lse"], w.name)
    if w.decode or case % 3 != 0:
        return
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1000)
    do = torch.randn(tuple(q.shape), generator=g).to(torch.bfloat16).to(cuda_device)
    ws_b = torch.zeros(pisa.backward_workspace_size(shape), dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = pisa.sparse_attention_backward(shape, q, k, v, o, lse, do, idx, ws=ws_b)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws_b, "backward")
    grads = oracle.backward(Q, K, V, gu.host_f32(do), idx_h, w.block, bool(w.causal), per_qhead=per_q)
    for name, got in (("dQ", dq), ("dK", dk), ("dV", dv)):
        got = gu.host_f32(got).astype(np.float64)
        want = grads[name]
        scale = np.abs(want).max()
        err = np.abs(got - want)
        assert err.max() <= REL_MAX * scale, f"{w.name} {name}: max err {err.max():.3e} vs {scale:.3e}"
        assert err.mean() <= REL_MEAN * scale, f"{w.name} {name}: mean err {err.mean():.3e} vs {scale:.3e}"


@pytest.mark.parametrize("case", range(len(CASES)), ids=[c[0].name for c in CASES])
def test_random_level_budgets_match_oracle(case, cuda_device):
    """The same shapes with random per-level budgets K_l (level 0 keeps K; coarser levels keep
    between 1 and twice K nodes, capped by the level's size): every selection row equals the
    oracle's descent under those budgets, or is an admissible near-tie resolution of it."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w, per_q, forced = CASES[case]
    shape = pisa.Shape.of(w, select_per_qhead=int(per_q), forced_blocks=forced)
    sizes, _ = pisa.level_layout(shape)
    rng = np.random.default_rng(9000 + case)
    budgets = [w.topk] + [int(rng.integers(1, max(1, min(n, 2 * w.topk)) + 1)) for n in sizes[1:]]
    q, k = (gu.to_device(w, t, cuda_device) for t in ("q", "k"))
    ws = pisa.new_workspace(shape, cuda_device)
    pyr = pisa.build_pyramid(shape, k)
    idx = pisa.select_blocks(shape, q, pyr, ws, level_budget=budgets)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, w.name)
    Q, K = gu.host_f32(q), gu.host_f32(k)
    ref = oracle.forward(Q, K, K, w.block, w.factor, w.topk, bool(w.causal), per_qhead=per_q, budgets=budgets,
                         forced=forced)
    gu.check_selection(idx.cpu().numpy(), ref, w, per_qhead=per_q, budgets=budgets, forced=forced,
                       what=f"{w.name} budgets {budgets}")


DECODE_CASES = [c for c, (w, _, _) in enumerate(CASES) if w.decode]


@pytest.mark.parametrize("case", DECODE_CASES, ids=[CASES[c][0].name for c in DECODE_CASES])
def test_random_decode_with_spare_capacity_and_append(case, cuda_device):
    """The sweep's decode shapes in a cache with spare capacity (1-20 blocks, rows past the
    length hold NaN): decode matches the oracle at the cache's length, and a pyramid built at a
    shorter length and appended up to it equals the one built at it, bit for bit."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w, per_q, forced = CASES[case]
    rng = np.random.default_rng(9500 + case)
    cap = w.seq_kv + int(rng.integers(1, 21)) * w.block
    k, v = (gu.to_device(w, t, cuda_device) for t in ("k", "v"))
    kc, vc = (torch.full((w.batch, w.heads_kv, cap, w.head_dim), float("nan"), dtype=torch.bfloat16,
                         device=cuda_device) for _ in range(2))
    kc[:, :, :w.seq_kv] = k
    vc[:, :, :w.seq_kv] = v
    q = gu.to_device(w, "q", cuda_device)
    shape = pisa.Shape.of(w, select_per_qhead=int(per_q), forced_blocks=forced, kv_capacity=cap)
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, kc, vc, ws, idx=True)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, w.name)
    Q, K, V = gu.host_f32(q), gu.host_f32(kc), gu.host_f32(vc)
    ref = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, per_qhead=per_q, kv_len=w.seq_kv,
                         forced=forced)
    idx = idx.cpu().numpy()
    gu.check_selection(idx, ref, w, per_qhead=per_q, forced=forced, kv_len=w.seq_kv)
    ref_o = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, per_qhead=per_q, kv_len=w.seq_kv,
                           idx_override=idx)
    o, lse = gu.host_f32(o), gu.host_f32(lse)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    gu.assert_output_close(o, ref_o["O"], lse, ref_o["lse"], w.name)
    # append: from a shorter length (a multiple of the block) up to the cache's length
    n_old = int(rng.integers(0, w.seq_kv // w.block)) * w.block
    kz = torch.nan_to_num(kc, nan=0.0)
    at = lambda n: pisa.Shape.of(w.replace(seq_kv=n), select_per_qhead=int(per_q), kv_capacity=cap)
    pyr = pisa.build_pyramid(at(n_old), kz) if n_old > 0 else \
        torch.zeros(pisa.pyramid_size(at(w.seq_kv)) // 4, dtype=torch.float32, device=cuda_device)
    pisa.append_pyramid(at(w.seq_kv), kz, pyr, n_old)
    fresh = pisa.build_pyramid(at(w.seq_kv), kz)
    torch.cuda.synchronize()
    assert torch.equal(pyr.view(-1), fresh.view(-1)), (w.name, n_old)
