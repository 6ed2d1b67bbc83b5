"""pisa_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers may not call cudaMalloc (code inside another framework's memory
pool, a plugin with no allocator of its own, a serving loop that must not
allocate once running). This entry point keeps its split-KV scratch in an
8 MiB device array built into the library. These tests call it through the C
ABI and check it against pisa_sparse_attention, which uses a caller
workspace, on two calls in a row (the array keeps the previous call's
contents). This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import workloads

pisa = pytest.importorskip("block_sparse_long_pisa_b200")

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3


def _decode_shape(batch=3, seq_kv=45 * 64, topk=9):
    w = workloads.Workload("noalloc-decode", batch, 8, 2, 1, seq_kv, 128, 64, 4, topk, 0, "clustered", 91)
    return w, pisa.Shape.of(w)


def test_rejects_shapes_beyond_the_builtin_scratch():
    # 64 sequences x 32 KV heads x 512 blocks: partials far above 8 MiB; checked before any GPU work
    s = pisa.Shape(64, 32, 32, 1, 131072, 128, 64, 4, 512)
    fake = ctypes.c_void_p(1 << 20)
    st = pisa._lib.pisa_decode_attention_noalloc(ctypes.byref(s.c()), fake, fake, fake, fake, fake, None, None)
    assert st == pisa.ERR_WORKSPACE
    prefill = pisa.Shape(1, 2, 2, 4096, 4096, 64, 64, 4, 8)
    st = pisa._lib.pisa_decode_attention_noalloc(ctypes.byref(prefill.c()), fake, fake, fake, fake, fake, None, None)
    assert st == pisa.ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_entry_point():
    import torch
    dev = torch.device("cuda:0")
    w, shape = _decode_shape()
    q, k, v = (workloads.device_tensor(w, t, dev) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, dev)
    pyr = pisa.build_pyramid(shape, k)
    idx = pisa.select_blocks(shape, q, pyr, ws)
    o_ref, l_ref = pisa.sparse_attention(shape, q, k, v, idx, ws)
    pisa.raise_on_device_error(ws)
    o_ref, l_ref = o_ref.float().cpu().numpy(), l_ref.cpu().numpy()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((w.batch, w.heads_q, 1), float("nan"), dtype=torch.float32, device=dev)
        st = pisa._lib.pisa_decode_attention_noalloc(ctypes.byref(shape.c()), q.data_ptr(), k.data_ptr(),
                                                     v.data_ptr(), idx.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                                     stream)
        assert st == pisa.OK, (call, pisa.STATUS.get(st))
        torch.cuda.synchronize()
        err = np.abs(o.float().cpu().numpy() - o_ref)
        assert err.max() < O_MAX and err.mean() < O_MEAN, (call, err.max(), err.mean())
        assert np.abs(lse.cpu().numpy() - l_ref).max() < LSE_TOL, call
