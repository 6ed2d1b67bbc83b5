"""Backward of the sparse attention step on the GPU against the fp64 oracle, through the C ABI.

The tolerance is relative to the largest gradient entry: the kernels round P and dS to bf16
before the dV, dQ and dK products (relative error 2^-9 per term) and write bf16 outputs
(another 2^-9), with fp32 accumulation; errors above 2 % of the largest entry, or a mean error
above 0.1 % of it, mean a wrong term, not rounding (measured on B200: at most 0.8 % and 0.02 %).
"""
import numpy as np
import pytest

import oracle
import workloads
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
W = workloads.Workload

CASES = {
    "gqa4-causal": W("bwd-gqa4-causal", 1, 8, 2, 20 * 64, 20 * 64, 128, 64, 4, 5, 1, "iid", 41),
    "gqa4-d64-noncausal": W("bwd-gqa4-d64", 2, 8, 2, 18 * 64, 18 * 64, 64, 64, 4, 4, 0, "iid", 42),
    # every shape runs both passes on tcgen05; the column pass takes a 128-key block as two
    # 64-key halves, and at head dim 64 pads the head-dim side of its MMAs to 128 lanes
    "mha-b128-causal": W("bwd-mha-b128", 1, 2, 2, 12 * 128, 12 * 128, 128, 128, 8, 4, 1, "clustered", 43),
    "gqa4-b128-noncausal": W("bwd-gqa4-b128", 2, 8, 2, 10 * 128, 10 * 128, 128, 128, 4, 3, 0, "iid", 47),
    "mha-d64-b64-causal": W("bwd-mha-d64", 1, 3, 3, 17 * 64, 17 * 64, 64, 64, 4, 6, 1, "clustered", 44),
    "gqa2-d64-b128-causal": W("bwd-gqa2-d64-b128", 1, 4, 2, 10 * 128, 10 * 128, 64, 128, 4, 3, 1, "clustered", 48),
    "gqa8-d128-noncausal": W("bwd-gqa8-d128", 2, 16, 2, 16 * 64, 16 * 64, 128, 64, 4, 6, 0, "clustered", 45),
    "mha-d128-b64-causal": W("bwd-mha-d128", 1, 2, 2, 15 * 64, 15 * 64, 128, 64, 4, 4, 1, "iid", 46),
}
REL_MAX, REL_MEAN = 2e-2, 1e-3


def _grads(w, cuda_device, per_qhead=False, forced=0):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    shape = pisa.Shape.of(w, select_per_qhead=int(per_qhead), forced_blocks=forced)
    q, k, v = (gu.to_device(w, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o, lse, idx = pisa.forward(shape, q, k, v, ws, idx=True)
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1000)
    do = torch.randn(tuple(q.shape), generator=g).to(torch.bfloat16).to(cuda_device)
    ws_b = torch.zeros(pisa.backward_workspace_size(shape), dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = pisa.sparse_attention_backward(shape, q, k, v, o, lse, do, idx, ws=ws_b)
    torch.cuda.synchronize()
    pisa.raise_on_device_error(ws)
    pisa.raise_on_device_error(ws_b, "backward")  # the backward kernels' status word
    return shape, (q, k, v, o, lse, do, idx), (dq, dk, dv)


def _close(got, ref, what):
    got = gu.host_f32(got).astype(np.float64)
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    assert err.max() <= REL_MAX * scale, f"{what}: max err {err.max():.3e} vs max |ref| {scale:.3e}"
    assert err.mean() <= REL_MEAN * scale, f"{what}: mean err {err.mean():.3e} vs max |ref| {scale:.3e}"


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name, cuda_device):
    w = CASES[name]
    shape, (q, k, v, o, lse, do, idx), (dq, dk, dv) = _grads(w, cuda_device)
    Q, K, V, dO = (gu.host_f32(x) for x in (q, k, v, do))
    ref = oracle.backward(Q, K, V, dO, idx.cpu().numpy(), w.block, bool(w.causal))
    _close(dq, ref["dQ"], f"{name} dQ")
    _close(dk, ref["dK"], f"{name} dK")
    _close(dv, ref["dV"], f"{name} dV")


@pytest.mark.parametrize("name", ["gqa4-causal", "gqa4-b128-noncausal", "gqa4-d64-noncausal"])
def test_backward_per_qhead_and_forced(name, cuda_device):
    w = CASES[name]
    shape, (q, k, v, o, lse, do, idx), (dq, dk, dv) = _grads(w, cuda_device, per_qhead=True, forced=3)
    Q, K, V, dO = (gu.host_f32(x) for x in (q, k, v, do))
    ref = oracle.backward(Q, K, V, dO, idx.cpu().numpy(), w.block, bool(w.causal), per_qhead=True)
    _close(dq, ref["dQ"], "per-qhead dQ")
    _close(dk, ref["dK"], "per-qhead dK")
    _close(dv, ref["dV"], "per-qhead dV")


@pytest.mark.parametrize("name", ["mha-d64-b64-causal", "mha-d128-b64-causal", "mha-b128-causal"])
def test_backward_full_topk_is_dense_gradient(name, cuda_device):
    """K = every block: the gradient of dense causal softmax attention (every key block's
    inverse list then holds every later query block)."""
    import torch
    w = CASES[name]
    w = w.replace(topk=w.n_blocks)
    shape, (q, k, v, o, lse, do, idx), (dq, dk, dv) = _grads(w, cuda_device)
    nb = w.n_blocks
    full = np.full((w.batch, w.heads_kv, nb, nb), -1, dtype=np.int32)
    for i in range(nb):
        full[:, :, i, :i + 1] = np.arange(i + 1)
    assert np.array_equal(idx.cpu().numpy(), full)
    Q, K, V, dO = (gu.host_f32(x) for x in (q, k, v, do))
    ref = oracle.backward(Q, K, V, dO, full, w.block, True)
    _close(dq, ref["dQ"], "dense dQ")
    _close(dk, ref["dK"], "dense dK")
    _close(dv, ref["dV"], "dense dV")


def test_backward_is_deterministic(cuda_device):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    w = CASES["gqa4-causal"]
    shape, (q, k, v, o, lse, do, idx), (dq, dk, dv) = _grads(w, cuda_device)
    dq2, dk2, dv2 = pisa.sparse_attention_backward(shape, q, k, v, o, lse, do, idx)
    torch.cuda.synchronize()
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
