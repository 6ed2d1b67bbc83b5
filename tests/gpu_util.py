"""Helpers for the GPU parity tests: seeded inputs on the device, oracle
references on the host, and the acceptance checks.

Acceptance (bf16 inputs, fp32 accumulation):
  * selected indices bit-exact, except query blocks whose oracle margin at a
    pruning level is below 1e-3 (near-ties), which are counted; a row that
    differs must still be well formed and reachable by the descent with its
    near-ties resolved the other way (``check_selection``);
  * O within max-abs 2e-2 and mean-abs 2e-3 of the oracle run on the GPU's own
    indices; LSE within 1e-3;
  * pyramid within 1e-5 absolute + 1e-5 relative.
"""
from __future__ import annotations

import numpy as np

import workloads

O_MAX, O_MEAN, LSE_TOL, PYR_TOL, NEAR_TIE = 2e-2, 2e-3, 1e-3, 1e-5, 1e-3


to_device = workloads.device_tensor


def host_f32(t):
    """fp32 numpy copy of a bf16/fp32 device tensor."""
    return t.float().cpu().numpy()


def check_selection(gpu_idx, ref, w, *, per_qhead=False, budgets=None, forced=0, topk=None, kv_len=None,
                    what=""):
    """Selection rows from the GPU against the oracle's `ref` (``oracle.forward`` on the same inputs).

    A row equal to the oracle's passes. A row that differs must be one the oracle's descent can
    reach when near-ties (R10) are resolved the other way: ``oracle.selection_is_admissible``
    checks that it is well formed (min(K, eligible) distinct ascending eligible blocks, then -1,
    forced blocks present) and replays the descent with every near-tie band open. Any other
    difference fails the test. Returns (near-tie rows, rows that differ) and prints both.
    """
    import oracle
    topk = w.topk if topk is None else topk
    g = w.heads_q // w.heads_kv
    n0 = (w.seq_kv if kv_len is None else kv_len) // w.block
    gpu_idx = np.asarray(gpu_idx)
    same = np.all(gpu_idx == ref["idx"], axis=-1)
    near = np.asarray(ref["margin"]) < NEAR_TIE
    bad = []
    for (b, hs, i) in zip(*np.nonzero(~same)):
        kvh = hs // g if per_qhead else hs
        last = n0 - 1 if (w.decode or not w.causal) else int(i)
        fset = oracle.forced_set(forced, n0 - 1 if w.decode else int(i), topk)
        ok, why = oracle.selection_is_admissible(ref["qbar"][b, hs, i], ref["pyramid"][b][kvh], w.factor, topk,
                                                 last, gpu_idx[b, hs, i], budgets=budgets, forced=fset)
        if not ok:
            bad.append(((int(b), int(hs), int(i)), why, gpu_idx[b, hs, i].tolist(), ref["idx"][b, hs, i].tolist()))
    n_near, n_diff = int(near.sum()), int((~same).sum())
    print(f"selection {what or w.name}: {same.size} rows, {n_near} near-ties, {n_diff} differ from the oracle")
    assert not bad, f"{len(bad)} selection rows not reachable by the descent: {bad[:3]}"
    return n_near, n_diff


def assert_output_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    err = np.abs(np.asarray(o_gpu, dtype=np.float64) - np.asarray(o_ref, dtype=np.float64))
    assert err.max() < O_MAX, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() < O_MEAN, f"{what}: O mean-abs {err.mean():.3e}"
    if lse_gpu is not None:
        le = np.abs(np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_ref, dtype=np.float64))
        assert le.max() < LSE_TOL, f"{what}: LSE max-abs {le.max():.3e}"


def assert_pyramid_close(pyr_gpu, levels_ref, offsets):
    for l, lev in enumerate(levels_ref):
        got = pyr_gpu[offsets[l]:offsets[l] + lev.shape[0]]
        err = np.abs(got - lev)
        assert np.all(err <= PYR_TOL + PYR_TOL * np.abs(lev)), f"level {l}: max err {err.max():.3e}"


def compact_row_problem(sel, i: int, block: int, causal: bool, t: np.ndarray):
    """Index plumbing for checking one query block on its own: the keys of its selected blocks
    `sel` (ascending) laid end to end, and query positions `t` (within block i) moved so that a
    causal mask over the compacted positions hides exactly what it hid in the full plane: every
    key of a block j < i stays visible, and in the diagonal block (j = i, which sorts last) key u
    is visible from query t >= u. Returns (key rows in the full plane, compacted query positions,
    compacted block ids)."""
    n = len(sel)
    key_rows = np.concatenate([np.arange(j * block, (j + 1) * block) for j in sel]) if n else np.zeros(0, int)
    if causal and n and sel[-1] == i:
        q_pos = (n - 1) * block + t
    else:
        q_pos = n * block + t
    return key_rows, q_pos, list(range(n))
