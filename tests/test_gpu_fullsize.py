"""Full-size workloads on the GPU, checked against the oracle on sampled outputs.

Each workload runs at its full size in the launch configuration bench.py
times (pisa_build_pyramid, pisa_select_blocks, pisa_sparse_attention on one
stream; pisa_forward must agree bit for bit). The oracle then recomputes, one
by one, sampled parts of the result from inputs regenerated on the host from
the same seeds: whole pyramid planes, the selections of sampled query blocks
(bit-exact except near-ties), and the attention rows of sampled query blocks
(on the GPU's own selection). The needle workload also checks that every
planted needle block is selected for its target query block.
"""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import gpu_util as gu

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _run(w, device):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    shape = pisa.Shape.of(w)
    q, k, v = (workloads.device_tensor(w, t, device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, device)
    pyr = pisa.build_pyramid(shape, k)
    idx = pisa.select_blocks(shape, q, pyr, ws)
    o, lse = pisa.sparse_attention(shape, q, k, v, idx, ws)
    o2, lse2, idx2 = pisa.forward(shape, q, k, v, pisa.new_workspace(shape, device), idx=True)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, w.name)
    assert torch.equal(idx, idx2) and torch.equal(o, o2) and torch.equal(lse, lse2)
    del q, k, v, o2, lse2, idx2
    return shape, pyr, idx.cpu().numpy(), o, lse


def _check_planes(w, shape, pyr, idx, o, lse, planes, n_sel, n_att, seed, extra_blocks=()):
    """Pyramid, selection and attention of sampled (batch, KV head) planes against the oracle."""
    import block_sparse_long_pisa_b200 as pisa
    _, offs = pisa.level_layout(shape)
    rng = np.random.Generator(np.random.PCG64(seed))
    nqb = shape.n_qblocks
    g = w.group
    scale = 1.0 / math.sqrt(w.head_dim)
    near_total = n_differ = n_rows = 0
    for (b, kvh) in planes:
        K = workloads.plane_f32(w, "k", b, kvh)
        V = workloads.plane_f32(w, "v", b, kvh)
        Qh = np.stack([workloads.plane_f32(w, "q", b, h) for h in range(kvh * g, (kvh + 1) * g)])
        levels = oracle.build_pyramid(K, w.block, w.factor)
        gu.assert_pyramid_close(gu.host_f32(pyr[b, kvh]), levels, offs)
        qbar = oracle.query_summary(Qh, 1 if w.decode else w.block)
        if w.decode:
            blocks_sel = [0]
        else:
            extra = [i for (i, _) in workloads.needles(w, b, kvh)] if w.keys == "needle" else []
            picks = rng.choice(nqb, size=min(n_sel, nqb), replace=False).tolist()
            blocks_sel = sorted(set(picks) | {0, nqb - 1} | set(extra) | set(extra_blocks))
        for i in blocks_sel:
            last = i if (w.causal and not w.decode) else w.n_blocks - 1
            r = oracle.select_blocks(qbar[i], levels, w.factor, w.topk, last)
            ref = np.full(w.topk, -1, dtype=np.int32)
            ref[:len(r["idx"])] = r["idx"]
            near_total += r["margin"] < gu.NEAR_TIE
            if not np.array_equal(idx[b, kvh, i], ref):
                # only a near-tie may differ, and the row must be one the descent reaches
                assert r["margin"] < gu.NEAR_TIE, (w.name, b, kvh, i, r["margin"])
                ok, why = oracle.selection_is_admissible(qbar[i], levels, w.factor, w.topk, last, idx[b, kvh, i])
                assert ok, (w.name, b, kvh, i, why, idx[b, kvh, i].tolist(), ref.tolist())
                n_differ += 1
            n_rows += 1
        att_blocks = blocks_sel if w.decode else sorted(rng.choice(blocks_sel, size=min(n_att, len(blocks_sel)),
                                                                   replace=False).tolist())
        for i in att_blocks:
            rows = np.arange(1) if w.decode else np.arange(i * w.block, (i + 1) * w.block)
            pos = np.full(1, w.seq_kv - 1) if w.decode else rows
            sel = [int(j) for j in idx[b, kvh, i] if j >= 0]
            for hh in range(g):
                h = kvh * g + hh
                ro, rl = oracle.attend(Qh[hh, rows], pos, K, V, sel, w.block, bool(w.causal) and not w.decode, scale)
                go = o[b, h, rows[0]:rows[-1] + 1].float().cpu().numpy()
                gl = lse[b, h, rows[0]:rows[-1] + 1].cpu().numpy()
                gu.assert_output_close(go, ro, gl, rl, f"{w.name} b{b} h{h} i{i}")
    print(f"selection {w.name}: {n_rows} sampled rows, {near_total} near-ties, {n_differ} differ from the oracle")
    return near_total


def test_causal32k(cuda_device):
    w = workloads.WORKLOADS["causal32k"]
    shape, pyr, idx, o, lse = _run(w, cuda_device)
    _check_planes(w, shape, pyr, idx, o, lse, [(0, 0), (0, 9), (0, 15)], 24, 6, 1)


def test_gqa128k_bench_configuration(cuda_device):
    w = workloads.WORKLOADS["gqa128k"]
    shape, pyr, idx, o, lse = _run(w, cuda_device)
    # the selection scores and descends 512 query blocks at a time: rows on both sides of each seam
    _check_planes(w, shape, pyr, idx, o, lse, [(0, 0), (0, 5)], 16, 6, 2,
                  extra_blocks=(511, 512, 1023, 1024, 1535, 1536))
    # every planted needle block is selected for its target query block, in every KV head
    for kvh in range(w.heads_kv):
        for (i, j) in workloads.needles(w, 0, kvh):
            assert j in idx[0, kvh, i], (kvh, i, j)


def test_long1m(cuda_device):
    w = workloads.WORKLOADS["long1m"]
    shape, pyr, idx, o, lse = _run(w, cuda_device)
    # 64 chunks of 128 query blocks
    _check_planes(w, shape, pyr, idx, o, lse, [(0, 3)], 12, 4, 3, extra_blocks=(127, 128, 4095, 4096))


def test_decode128k(cuda_device):
    w = workloads.WORKLOADS["decode128k"]
    shape, pyr, idx, o, lse = _run(w, cuda_device)
    _check_planes(w, shape, pyr, idx, o, lse, [(0, 0), (17, 3), (63, 7)], 1, 1, 4)


def test_gqa128k_backward_sampled(cuda_device):
    """The backward at the bench's full size (128K GQA, `bench.py --backward`): dQ of sampled query
    blocks and dK, dV of sampled key blocks (one with a list of ~90 query blocks x 4 heads, i.e.
    ~180 column-pass tiles) against the fp64 oracle, each part computed on its own from the rows
    and keys it depends on."""
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = workloads.WORKLOADS["gqa128k"]
    shape = pisa.Shape.of(w)
    q, k, v = (workloads.device_tensor(w, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    gen = torch.Generator(device="cpu").manual_seed(w.seed + 1000)
    do_h = torch.randn(tuple(q.shape), generator=gen).to(torch.bfloat16)
    do = do_h.to(cuda_device)
    ws_b = torch.zeros(pisa.backward_workspace_size(shape), dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = pisa.sparse_attention_backward(shape, q, k, v, o, lse, do, idx, ws=ws_b)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws, "forward")
    pisa.raise_on_device_error(ws_b, "backward")
    del o, lse, q, k, v
    idx_h = idx.cpu().numpy()
    B, g, blk, nqb = 0, w.group, w.block, shape.n_qblocks
    scale = 1.0 / math.sqrt(w.head_dim)
    t = np.arange(blk)
    rel_max, rel_mean = 2e-2, 1e-3

    def close(got, ref, what):
        err = np.abs(got - ref)
        top = np.abs(ref).max()
        assert err.max() <= rel_max * top, f"{what}: max err {err.max():.3e} vs max |ref| {top:.3e}"
        assert err.mean() <= rel_mean * top, f"{what}: mean err {err.mean():.3e} vs max |ref| {top:.3e}"

    for kvh in (0, 5):
        K = workloads.plane_f32(w, "k", B, kvh)
        V = workloads.plane_f32(w, "v", B, kvh)
        heads = list(range(kvh * g, (kvh + 1) * g))
        Qh = {h: workloads.plane_f32(w, "q", B, h) for h in heads}
        dOh = {h: do_h[B, h].float().numpy() for h in heads}

        def row_grads(i, h):
            sel = [int(j) for j in idx_h[B, kvh, i] if j >= 0]
            rows, q_pos, blocks = gu.compact_row_problem(sel, i, blk, True, t)
            qr = slice(i * blk, (i + 1) * blk)
            dq_r, dk_r, dv_r = oracle.attend_backward(Qh[h][qr], q_pos, K[rows], V[rows], blocks, blk, True,
                                                      scale, dOh[h][qr])
            return sel, dq_r, dk_r, dv_r

        # dQ of sampled query blocks (first, last, a needle target, random)
        rng = np.random.Generator(np.random.PCG64(40 + kvh))
        target = workloads.needles(w, B, kvh)[0][0]
        for i in sorted({0, nqb - 1, target} | set(rng.choice(nqb, size=3, replace=False).tolist())):
            for h in heads:
                _, dq_r, _, _ = row_grads(i, h)
                close(gu.host_f32(dq[B, h, i * blk:(i + 1) * blk]), dq_r, f"dQ kvh{kvh} h{h} i{i}")
        # dK, dV of sampled key blocks: sum over every (query block, head) whose selection holds it
        for j in ((nqb // 4 + 3, nqb - 1) if kvh == 0 else (nqb // 2 + 7, nqb - 1)):
            users = [i for i in range(j, nqb) if j in idx_h[B, kvh, i]]
            dk_ref = np.zeros((blk, w.head_dim))
            dv_ref = np.zeros((blk, w.head_dim))
            for i in users:
                for h in heads:
                    sel, _, dk_r, dv_r = row_grads(i, h)
                    m = sel.index(j)
                    dk_ref += dk_r[m * blk:(m + 1) * blk]
                    dv_ref += dv_r[m * blk:(m + 1) * blk]
            close(gu.host_f32(dk[B, kvh, j * blk:(j + 1) * blk]), dk_ref, f"dK kvh{kvh} j{j} ({len(users)} users)")
            close(gu.host_f32(dv[B, kvh, j * blk:(j + 1) * blk]), dv_ref, f"dV kvh{kvh} j{j} ({len(users)} users)")
