"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, sizes buffers, and rejects bad arguments before enqueuing anything.

Every compute call here fails validation on the host, so the fake pointers it
carries are never dereferenced or handed to a kernel.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import workloads

pisa = pytest.importorskip("block_sparse_long_pisa_b200")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"PISA_API\s+[\w\s\*]+?\b(pisa_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(pisa._lib, n), n
    assert set(names) == set(pisa.EXPORTED)


def shape_of(name, **kw):
    return pisa.Shape.of(workloads.WORKLOADS[name], **kw)


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
def test_level_layout_matches_the_level_rule(name):
    s = shape_of(name)
    sizes, offs = pisa.level_layout(s)
    assert sizes == oracle.level_sizes(s.n_blocks, s.factor)
    assert offs == list(np.cumsum([0] + sizes[:-1]))
    assert pisa.num_levels(s) == len(sizes)
    assert pisa.pyramid_size(s) == s.batch * s.heads_kv * sum(sizes) * s.head_dim * 4
    ws = pisa.workspace_size(s)
    assert ws >= 256 + pisa.pyramid_size(s)


@pytest.mark.parametrize("bad, code", [
    (dict(heads_q=6, heads_kv=4), pisa.ERR_INVALID_ARG),
    (dict(seq_kv=4096 + 32, seq_q=4096 + 32), pisa.ERR_INVALID_ARG),
    (dict(seq_q=2048), pisa.ERR_INVALID_ARG),
    (dict(factor=1), pisa.ERR_INVALID_ARG),
    (dict(topk=0), pisa.ERR_INVALID_ARG),
    (dict(causal=2), pisa.ERR_INVALID_ARG),
    (dict(batch=0), pisa.ERR_INVALID_ARG),
    (dict(head_dim=96), pisa.ERR_UNSUPPORTED),
    (dict(block=32), pisa.ERR_UNSUPPORTED),
    (dict(topk=2048, factor=4), pisa.ERR_UNSUPPORTED),
])
def test_invalid_shapes(bad, code):
    s = shape_of("tiny", **bad)
    n = ctypes.c_size_t()
    assert pisa._lib.pisa_workspace_size(ctypes.byref(s.c()), ctypes.byref(n)) == code
    assert pisa._lib.pisa_num_levels(ctypes.byref(s.c())) == -1
    assert pisa._lib.pisa_forward(ctypes.byref(s.c()), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1 << 40,
                                  None) == code


def test_null_and_misaligned_pointers_rejected():
    s = shape_of("tiny").c()
    big = 1 << 40
    f = pisa._lib
    assert f.pisa_forward(ctypes.byref(s), None, FAKE, FAKE, FAKE, None, None, FAKE, big, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_forward(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, None, None, big, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_forward(ctypes.byref(s), MISALIGNED, FAKE, FAKE, FAKE, None, None, FAKE, big,
                          None) == pisa.ERR_INVALID_ARG
    assert f.pisa_build_pyramid(ctypes.byref(s), None, FAKE, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_sparse_attention(ctypes.byref(s), FAKE, FAKE, FAKE, None, FAKE, None, FAKE, big,
                                   None) == pisa.ERR_INVALID_ARG
    assert f.pisa_select_blocks(ctypes.byref(s), FAKE, None, None, FAKE, None, FAKE, big, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_check_status(None, None, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_forward(None, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, big, None) == pisa.ERR_INVALID_ARG


def test_small_workspace_rejected():
    s = shape_of("tiny")
    need = pisa.workspace_size(s)
    f = pisa._lib
    c = s.c()
    assert f.pisa_forward(ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, None, None, FAKE, need - 1,
                          None) == pisa.ERR_WORKSPACE
    assert f.pisa_select_blocks(ctypes.byref(c), FAKE, FAKE, None, FAKE, None, FAKE, need - 1,
                                None) == pisa.ERR_WORKSPACE
    assert f.pisa_sparse_attention(ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need - 1,
                                   None) == pisa.ERR_WORKSPACE


def test_level_budget_checks():
    s = shape_of("tiny")
    c = s.c()
    n = pisa.num_levels(s)
    bad_first = (ctypes.c_int32 * n)(*([s.topk + 1] + [s.topk] * (n - 1)))
    assert pisa._lib.pisa_select_blocks(ctypes.byref(c), FAKE, FAKE, bad_first, FAKE, None, FAKE, 1 << 40,
                                        None) == pisa.ERR_INVALID_ARG
    too_wide = (ctypes.c_int32 * n)(*([s.topk] + [2000] * (n - 1)))
    assert pisa._lib.pisa_select_blocks(ctypes.byref(c), FAKE, FAKE, too_wide, FAKE, None, FAKE, 1 << 40,
                                        None) == pisa.ERR_UNSUPPORTED
    zero = (ctypes.c_int32 * n)(*([s.topk] + [0] * (n - 1)))
    assert pisa._lib.pisa_select_blocks(ctypes.byref(c), FAKE, FAKE, zero, FAKE, None, FAKE, 1 << 40,
                                        None) == pisa.ERR_INVALID_ARG


def test_status_strings():
    for code in range(7):
        assert pisa._lib.pisa_status_string(code).decode()
    assert pisa._lib.pisa_status_string(99).decode() == "unknown status"


def test_attention_pair_count_by_brute_force():
    s = pisa.Shape(1, 4, 2, 256, 256, 64, 64, 4, 3, causal=1)
    idx = np.array([[[[0, -1, -1], [0, 1, -1], [0, 1, 2], [1, 2, 3]]] * 2]).reshape(1, 2, 4, 3).astype(np.int32)
    brute = 0
    for h in range(4):
        for i in range(4):
            for t in range(64):
                q = i * 64 + t
                for j in idx[0, h // 2, i]:
                    if j >= 0:
                        brute += sum(1 for key in range(j * 64, j * 64 + 64) if key <= q)
    assert pisa.attention_pairs(idx, s) == brute


def _align256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("name", ["tiny", "causal32k", "gqa128k"])
def test_backward_workspace_layout(name):
    """Status word, Delta per query row, list offsets per key block, list entries, and the
    per-range counts of the parallel list fill (32 ranges of query blocks)."""
    s = shape_of(name)
    n0, nqb, g = s.n_blocks, s.n_qblocks, s.heads_q // s.heads_kv
    rsize = -(-nqb // 32)
    nranges = -(-nqb // rsize)
    o = 256
    o = _align256(o + s.batch * s.heads_q * s.seq_q * 4)
    o = _align256(o + s.batch * s.heads_kv * (n0 + 1) * 4)
    o = _align256(o + s.batch * s.heads_kv * nqb * s.topk * g * 4)
    o = _align256(o + s.batch * s.heads_kv * nranges * n0 * 4)
    assert pisa.backward_workspace_size(s) == o


def test_backward_argument_checks():
    s = shape_of("tiny")
    c = s.c()
    f = pisa._lib
    need = pisa.backward_workspace_size(s)
    args = [FAKE] * 10
    assert f.pisa_sparse_attention_backward(ctypes.byref(c), *args, FAKE, need - 1, None) == pisa.ERR_WORKSPACE
    for k in range(10):
        bad = list(args)
        bad[k] = None
        assert f.pisa_sparse_attention_backward(ctypes.byref(c), *bad, FAKE, need, None) == pisa.ERR_INVALID_ARG
        bad[k] = MISALIGNED
        assert f.pisa_sparse_attention_backward(ctypes.byref(c), *bad, FAKE, need, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_sparse_attention_backward(ctypes.byref(c), *args, None, need, None) == pisa.ERR_INVALID_ARG
    dec = shape_of("decode128k").c()
    n = ctypes.c_size_t()
    assert f.pisa_backward_workspace_size(ctypes.byref(dec), ctypes.byref(n)) == pisa.ERR_UNSUPPORTED


@pytest.mark.parametrize("bad", [
    dict(forced_blocks=4),                                    # unknown variant bit
    dict(seq_q=1, kv_capacity=4096 - 64),                     # capacity below seq_kv
    dict(seq_q=1, kv_capacity=8192 + 32),                     # capacity not a multiple of the block
    dict(kv_capacity=8192),                                   # spare capacity is a decode feature
])
def test_selection_variant_and_capacity_checks(bad):
    s = shape_of("tiny", **bad)
    n = ctypes.c_size_t()
    assert pisa._lib.pisa_workspace_size(ctypes.byref(s.c()), ctypes.byref(n)) == pisa.ERR_INVALID_ARG


def test_capacity_sets_the_pyramid_layout():
    s = shape_of("tiny", seq_q=1, kv_capacity=4 * 4096)
    sizes, offs = pisa.level_layout(s)
    assert sizes == oracle.level_sizes(4 * 4096 // s.block, s.factor)
    assert pisa.pyramid_size(s) == s.batch * s.heads_kv * sum(sizes) * s.head_dim * 4
    for forced in (1, 2, 3):
        assert pisa.workspace_size(shape_of("tiny", forced_blocks=forced)) > 0


def test_append_pyramid_argument_checks():
    s = shape_of("tiny", seq_q=1, kv_capacity=2 * 4096).c()
    f = pisa._lib
    assert f.pisa_append_pyramid(ctypes.byref(s), None, FAKE, 0, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_append_pyramid(ctypes.byref(s), FAKE, None, 0, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_append_pyramid(ctypes.byref(s), MISALIGNED, FAKE, 0, None) == pisa.ERR_INVALID_ARG
    assert f.pisa_append_pyramid(ctypes.byref(s), FAKE, MISALIGNED, 0, None) == pisa.ERR_INVALID_ARG
    for old in (-64, 4096 + 64, 32):  # negative, past seq_kv, not a whole block
        assert f.pisa_append_pyramid(ctypes.byref(s), FAKE, FAKE, old, None) == pisa.ERR_INVALID_ARG


def test_workspace_grows_no_faster_than_n_log_n():
    """The selection's score plane is scored and descended in chunks of query blocks, so the
    workspace of a causal prefill grows like the pyramid, the query summaries and the index rows
    (O(N)), not like nQB x total nodes (O(N^2)): the 1M-token workload stays within a few hundred MB,
    and from 128K to 1M to 4M tokens the growth stays within N log N."""
    import math
    shapes = {n: pisa.Shape(1, 8, 8, n, n, 128, 128, 8, 128, causal=1) for n in (1 << 17, 1 << 20, 1 << 22)}
    ws = {n: pisa.workspace_size(s) for n, s in shapes.items()}
    assert ws[1 << 20] < 512e6, ws[1 << 20]
    ns = sorted(ws)
    for a, b in zip(ns, ns[1:]):
        assert ws[b] / ws[a] <= (b * math.log(b)) / (a * math.log(a)), (a, b, ws[a], ws[b])
    # the bench workload too (GQA, 64-key blocks)
    assert pisa.workspace_size(pisa.Shape(1, 32, 8, 1 << 17, 1 << 17, 128, 64, 4, 64, causal=1)) < 300e6


def test_injected_launch_failure_after_argument_checks(monkeypatch):
    """With PISA_FAULT=launch the enqueuing calls still report argument errors first; the
    self-test's arguments are checked on the host too. (The injected PISA_ERR_CUDA itself, and
    that nothing is enqueued, are checked on a GPU.)"""
    monkeypatch.setenv("PISA_FAULT", "launch")
    fake = ctypes.c_void_p(1 << 20)
    bad = pisa.Shape(1, 3, 2, 4096, 4096, 64, 64, 4, 8)      # heads_q not a multiple of heads_kv
    assert pisa._lib.pisa_build_pyramid(ctypes.byref(bad.c()), fake, fake, None) == pisa.ERR_INVALID_ARG
    good = pisa.Shape(1, 2, 2, 4096, 4096, 64, 64, 4, 8)
    assert pisa._lib.pisa_build_pyramid(ctypes.byref(good.c()), fake, None, None) == pisa.ERR_INVALID_ARG
    assert pisa._lib.pisa_build_pyramid(ctypes.byref(good.c()), fake, fake, None) == pisa.ERR_CUDA
    assert pisa._lib.pisa_selftest_wait_timeout(fake, 0, None) == pisa.ERR_INVALID_ARG
    assert pisa._lib.pisa_selftest_wait_timeout(None, 10, None) == pisa.ERR_INVALID_ARG
    assert pisa._lib.pisa_selftest_wait_timeout(fake, 10, None) == pisa.ERR_CUDA
