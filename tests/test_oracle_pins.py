"""The CPU oracle against facts fixed outside it (closed forms, brute force, invariants)."""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import pins


@pytest.mark.parametrize("name", sorted(pins.ALL_PINS))
def test_pin(name):
    pins.ALL_PINS[name](oracle.pisa_oracle)


def test_level_sizes_of_the_workloads():
    # R1 gives exactly the level chains the workload descriptions state
    assert oracle.level_sizes(64, 4) == [64, 16, 4]
    assert oracle.level_sizes(512, 4) == [512, 128, 32, 8, 2]
    assert oracle.level_sizes(2048, 4) == [2048, 512, 128, 32, 8, 2]
    assert oracle.level_sizes(8192, 8) == [8192, 1024, 128, 16, 2]
    assert oracle.level_sizes(5, 8) == [5]
    assert oracle.level_sizes(37, 4) == [37, 10, 3]


def test_workload_shapes_and_bf16():
    w = workloads.WORKLOADS["tiny"]
    q = workloads.plane_bf16(w, "q", 0, 1)
    assert q.shape == (4096, 64) and q.dtype == np.uint16
    # regenerating a slice gives the same bits; bf16 decode is exact
    assert np.array_equal(q[:4096], workloads.chunk_bf16(w, "q", 0, 1, 0))
    x = np.array([1.0, -2.5, 3.14159265, 1e-3, 65504.0], dtype=np.float32)
    r = workloads.bf16_to_f32(workloads.round_bf16(x))
    assert np.all(np.abs(r - x) <= np.abs(x) * 2.0 ** -8)
    # round to nearest even on an exact halfway case: 1 + 2^-8 -> 1.0, 1 + 3*2^-8 -> 1 + 2^-6
    h = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8], dtype=np.float32)
    assert workloads.bf16_to_f32(workloads.round_bf16(h)).tolist() == [1.0, 1 + 2 ** -6]


def test_whole_tensor_draw_is_thread_count_independent():
    w = workloads.WORKLOADS["tiny"].replace(seq_q=8192, seq_kv=8192)
    a = workloads.tensor_bf16(w, "k", threads=1)
    b = workloads.tensor_bf16(w, "k", threads=4)
    assert np.array_equal(a, b)


def test_clustered_keys_follow_their_centroid():
    w = workloads.WORKLOADS["causal32k"].replace(seq_q=4096, seq_kv=4096, heads_q=2, heads_kv=2)
    k = workloads.plane_f32(w, "k", 0, 1)
    cid = workloads._key_block_cluster(w, 0, 1)
    cent = workloads._centroids(w, 0, 1)
    resid = k.reshape(-1, w.block, w.head_dim) - cent[cid][:, None, :]
    assert abs(resid.std() - workloads.CLUSTER_NOISE_STD) < 0.01


def test_needle_recall_small():
    """P9 on a scaled-down needle workload: every planted needle block is selected for its target block."""
    w = workloads.WORKLOADS["gqa128k"].replace(heads_q=8, heads_kv=2, seq_q=16384, seq_kv=16384)
    found = total = 0
    for kvh in range(w.heads_kv):
        k = workloads.plane_f32(w, "k", 0, kvh)
        levels = oracle.build_pyramid(k, w.block, w.factor)
        for (i, j) in workloads.needles(w, 0, kvh):
            qrows = np.stack([workloads.plane_f32(w, "q", 0, h)[i * w.block:(i + 1) * w.block]
                              for h in range(kvh * w.group, (kvh + 1) * w.group)])
            qbar = oracle.query_summary(qrows, w.block)[0]
            sel = oracle.select_blocks(qbar, levels, w.factor, w.topk, i)["idx"]
            total += 1
            found += j in sel
            # needle keys have cosine 0.9 with the target direction
            d = qrows.astype(np.float64).reshape(-1, w.head_dim).sum(0)
            u = d / np.linalg.norm(d)
            blk = k[j * w.block:(j + 1) * w.block].astype(np.float64)
            cos = blk @ u / np.linalg.norm(blk, axis=1)
            assert np.all(np.abs(cos - 0.9) < 0.02)
    assert found == total == 16 * w.heads_kv


def test_oracle_forward_tiny_workload_structure():
    w = workloads.WORKLOADS["tiny"]
    q, k, v = workloads.qkv_f32(w)
    res = oracle.forward(q, k, v, w.block, w.factor, w.topk, bool(w.causal))
    assert res["idx"].shape == (1, 2, 64, 8)
    assert np.all(res["idx"] >= 0)
    assert np.all(np.diff(res["idx"], axis=-1) > 0)
    assert np.all(res["n_scored"] == 4 + 16 + 32)
    assert np.isfinite(res["O"]).all() and np.isfinite(res["lse"]).all()
    # each output row is a convex combination of selected values: |O| <= max |V|
    assert np.abs(res["O"]).max() <= np.abs(v).max() + 1e-5
    # lse is at least the max logit over the row's keys and at most that plus log(#keys)
    sc = 1.0 / math.sqrt(w.head_dim)
    b, h, i = 0, 1, 5
    blocks = res["idx"][b, h, i]
    keys = np.concatenate([k[b, h, j * 64:(j + 1) * 64] for j in blocks])
    s = sc * (q[b, h, i * 64:(i + 1) * 64].astype(np.float64) @ keys.T.astype(np.float64))
    lse = res["lse"][b, h, i * 64:(i + 1) * 64]
    assert np.all(lse >= s.max(1) - 1e-4) and np.all(lse <= s.max(1) + math.log(keys.shape[0]) + 1e-4)
