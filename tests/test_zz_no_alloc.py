"""pisa_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers may not call cudaMalloc (code inside another framework's memory
pool, a plugin with no allocator of its own, a serving loop that must not
allocate once running). This entry point keeps its split-KV scratch in an
8 MiB device array built into the library. These tests call it through the C
ABI and check it against the oracle and against pisa_sparse_attention, which
uses a caller workspace, on two calls in a row (the array keeps the previous
call's contents); a shape whose partials come within one split of the array's
end runs through the Python wrapper; the companion status call reports an
out-of-range block index. This file is named to be collected last.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import workloads

pisa = pytest.importorskip("block_sparse_long_pisa_b200")

O_MAX, O_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3
ARRAY_BYTES, STATUS_BYTES = 8 << 20, 256


def _decode_shape(batch=3, seq_kv=45 * 64, topk=9):
    w = workloads.Workload("noalloc-decode", batch, 8, 2, 1, seq_kv, 128, 64, 4, topk, 0, "clustered", 91)
    return w, pisa.Shape.of(w)


def _needed_bytes(s):
    """The size rule the header states for the built-in array."""
    hsel = s.heads_q if s.select_per_qhead else s.heads_kv
    gsel = 1 if s.select_per_qhead else s.heads_q // s.heads_kv
    rows = s.batch * hsel
    per_split = min(max(math.ceil(s.topk / math.ceil(592 / rows)), 2), 16)
    splits = math.ceil(s.topk / per_split)
    return STATUS_BYTES + rows * splits * gsel * (s.head_dim + 2) * 4


# 126 sequences x 8 KV heads (32 query heads), head dim 128, K = 64: 4 splits of 16 blocks, partials
# 8,386,560 bytes, 1,792 bytes short of the array's end (one more split row needs 2,080)
LIMIT = pisa.Shape(126, 32, 8, 1, 80 * 64, 128, 64, 4, 64)
OVER = pisa.Shape(127, 32, 8, 1, 80 * 64, 128, 64, 4, 64)


def test_rejects_shapes_beyond_the_builtin_scratch():
    import torch
    fake = ctypes.c_void_p(1 << 20)

    def call(s):
        return pisa._lib.pisa_decode_attention_noalloc(ctypes.byref(s.c()), fake, fake, fake, fake, fake, None, None)

    # 64 sequences x 32 KV heads x 512 blocks: partials far above 8 MiB; checked before any GPU work
    assert call(pisa.Shape(64, 32, 32, 1, 131072, 128, 64, 4, 512)) == pisa.ERR_WORKSPACE
    assert call(pisa.Shape(1, 2, 2, 4096, 4096, 64, 64, 4, 8)) == pisa.ERR_INVALID_ARG
    # the documented rule at its boundary: one split row past the end is refused
    assert _needed_bytes(LIMIT) <= ARRAY_BYTES < _needed_bytes(LIMIT) + 128 * 4 * 130
    assert _needed_bytes(OVER) > ARRAY_BYTES
    assert call(OVER) == pisa.ERR_WORKSPACE
    # the headline decode shape fits (4 splits, about 4.3 MB)
    assert _needed_bytes(pisa.Shape(64, 32, 8, 1, 131072, 128, 64, 4, 64)) < 4.3e6
    if not torch.cuda.is_available():
        # past the size check the call needs a device: with none it fails on the CUDA side
        assert call(LIMIT) == pisa.ERR_CUDA


def _oracle_rows(q, k, v, idx, b, h, g, block):
    """Oracle O and LSE of decode row (b, h) over the blocks its selection row lists."""
    K = k[b, h // g].float().cpu().numpy()
    V = v[b, h // g].float().cpu().numpy()
    qr = q[b, h].float().cpu().numpy()
    sel = [int(j) for j in idx[b, h // g, 0].tolist() if j >= 0]
    n = K.shape[0]
    return oracle.attend(qr, np.full(1, n - 1), K, V, sel, block, False, 1.0 / math.sqrt(q.shape[-1]))


def _close(o, l, ro, rl, what):
    err = np.abs(np.asarray(o, dtype=np.float64) - ro)
    assert err.max() < O_MAX and err.mean() < O_MEAN, (what, err.max(), err.mean())
    assert np.abs(np.asarray(l, dtype=np.float64) - rl).max() < LSE_TOL, what


@pytest.mark.gpu
def test_noalloc_decode_matches_oracle_and_workspace_entry_point():
    import torch
    dev = torch.device("cuda:0")
    w, shape = _decode_shape()
    q, k, v = (workloads.device_tensor(w, t, dev) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, dev)
    pyr = pisa.build_pyramid(shape, k)
    idx = pisa.select_blocks(shape, q, pyr, ws)
    o_ws, l_ws = pisa.sparse_attention(shape, q, k, v, idx, ws)
    pisa.raise_on_device_error(ws)
    o_ws, l_ws = o_ws.float().cpu().numpy(), l_ws.cpu().numpy()
    Q, K, V = (x.float().cpu().numpy() for x in (q, k, v))
    ref = oracle.forward(Q, K, V, w.block, w.factor, w.topk, False, idx_override=idx.cpu().numpy())
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((w.batch, w.heads_q, 1), float("nan"), dtype=torch.float32, device=dev)
        st = pisa._lib.pisa_decode_attention_noalloc(ctypes.byref(shape.c()), q.data_ptr(), k.data_ptr(),
                                                     v.data_ptr(), idx.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                                     stream)
        assert st == pisa.OK, (call, pisa.STATUS.get(st))
        assert pisa.decode_noalloc_check_status() == (pisa.OK, 0), call
        o_h, l_h = o.float().cpu().numpy(), lse.cpu().numpy()
        _close(o_h, l_h, ref["O"], ref["lse"], f"call {call} vs the oracle")
        _close(o_h, l_h, o_ws, l_ws, f"call {call} vs pisa_sparse_attention")


@pytest.mark.gpu
def test_noalloc_decode_at_the_array_limit():
    """Partials within one split of the array's end, through the Python wrapper, twice."""
    import torch
    dev = torch.device("cuda:0")
    s = LIMIT
    gen = torch.Generator(device=dev).manual_seed(93)
    q = torch.randn((s.batch, s.heads_q, 1, s.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    k = torch.randn((s.batch, s.heads_kv, s.seq_kv, s.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    v = torch.randn((s.batch, s.heads_kv, s.seq_kv, s.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    ws = pisa.new_workspace(s, dev)
    idx = pisa.select_blocks(s, q, pisa.build_pyramid(s, k), ws)
    o_ws, l_ws = pisa.sparse_attention(s, q, k, v, idx, ws)
    pisa.raise_on_device_error(ws)
    g = s.heads_q // s.heads_kv
    for call in range(2):
        o, lse = pisa.decode_attention_noalloc(s, q, k, v, idx)
        assert pisa.decode_noalloc_check_status() == (pisa.OK, 0), call
        _close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ws.float().cpu().numpy(), l_ws.cpu().numpy(),
               f"call {call} vs pisa_sparse_attention")
        # rows whose partials sit at the start, the middle and the very end of the array
        for b, h in ((0, 0), (63, 17), (s.batch - 1, s.heads_q - 1)):
            ro, rl = _oracle_rows(q, k, v, idx, b, h, g, s.block)
            _close(o[b, h].float().cpu().numpy(), lse[b, h].cpu().numpy(), ro, rl, f"call {call} b{b} h{h}")
    st = pisa._lib.pisa_decode_attention_noalloc(ctypes.byref(OVER.c()), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                 idx.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                                 torch.cuda.current_stream().cuda_stream)
    assert st == pisa.ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_status_reports_a_bad_index():
    """A selection row naming a block past the cache: the kernel skips it and records
    PISA_ERR_BAD_INDEX, which the companion call reports and clears; the next call with good
    indices reports nothing."""
    import torch
    dev = torch.device("cuda:0")
    w, shape = _decode_shape()
    q, k, v = (workloads.device_tensor(w, t, dev) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, dev)
    idx = pisa.select_blocks(shape, q, pisa.build_pyramid(shape, k), ws)
    bad = idx.clone()
    bad[1, 0, 0, -1] = 10 ** 6
    pisa.decode_attention_noalloc(shape, q, k, v, bad)
    st, detail = pisa.decode_noalloc_check_status()
    assert st == pisa.ERR_BAD_INDEX and detail >> 8 == 2, (st, hex(detail))
    assert pisa.decode_noalloc_check_status() == (pisa.OK, 0)
    pisa.decode_attention_noalloc(shape, q, k, v, bad)
    pisa.decode_attention_noalloc(shape, q, k, v, idx)
    assert pisa.decode_noalloc_check_status()[0] == pisa.OK
