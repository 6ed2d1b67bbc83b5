"""Failure paths on the GPU, in the forms that fault no GPU.

* Host-side launch-failure injection: with PISA_FAULT=launch every enqueuing call returns
  PISA_ERR_CUDA after its argument checks and enqueues nothing (no launch is counted, outputs stay
  as they were); once the variable is gone the same calls run and give the results they gave
  before.
* A bounded wait that runs out: the self-test kernel waits on an mbarrier that nothing completes;
  after its limit it records PISA_ERR_TIMEOUT (detail 0x501) in the workspace status word and
  returns, pisa_check_status reports and clears it, and the context stays usable for the next
  forward.
"""
import numpy as np
import pytest

import workloads
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

W = workloads.Workload("failure-gqa", 1, 8, 2, 20 * 64, 20 * 64, 128, 64, 4, 5, 1, "iid", 51)


def test_injected_launch_failure_enqueues_nothing(cuda_device, monkeypatch):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    shape = pisa.Shape.of(W)
    q, k, v = (gu.to_device(W, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o_ref, lse_ref, idx_ref = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    monkeypatch.setenv("PISA_FAULT", "launch")
    o = torch.full_like(q, 7.0)
    pyr = torch.zeros(pisa.pyramid_size(shape) // 4, dtype=torch.float32, device=cuda_device)
    calls = {
        "forward": lambda: pisa.forward(shape, q, k, v, ws, O=o),
        "build_pyramid": lambda: pisa.build_pyramid(shape, k),
        "select_blocks": lambda: pisa.select_blocks(shape, q, pyr, ws),
        "sparse_attention": lambda: pisa.sparse_attention(shape, q, k, v, idx_ref, ws, O=o),
        "selftest": lambda: pisa.selftest_wait_timeout(ws, 1000),
    }
    for name, call in calls.items():
        with pytest.raises(pisa.PisaError) as e:
            call()
        assert e.value.status == pisa.ERR_CUDA, name
        assert pisa.last_launch_count() == 0, name
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()), "an injected failure must leave the output untouched"
    assert pisa.check_status(ws) == (pisa.OK, 0)
    monkeypatch.delenv("PISA_FAULT")
    o2, lse2, idx2 = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    assert torch.equal(o2, o_ref) and torch.equal(lse2, lse_ref) and torch.equal(idx2, idx_ref)


def test_bounded_wait_timeout_is_reported(cuda_device):
    import torch
    import block_sparse_long_pisa_b200 as pisa
    shape = pisa.Shape.of(W)
    q, k, v = (gu.to_device(W, t, cuda_device) for t in ("q", "k", "v"))
    ws = pisa.new_workspace(shape, cuda_device)
    o_ref, lse_ref, _ = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    pisa.selftest_wait_timeout(ws, 3000)
    t1.record(stream)
    st, detail = pisa.check_status(ws)
    assert (st, detail) == (pisa.ERR_TIMEOUT, 0x501), (st, hex(detail))
    ms = t0.elapsed_time(t1)
    assert 3.0 <= ms < 1000.0, ms          # it waited its limit, then returned
    assert pisa.check_status(ws) == (pisa.OK, 0)
    # the context is still usable: the same forward gives the same result
    o2, lse2, _ = pisa.forward(shape, q, k, v, ws, idx=True)
    pisa.raise_on_device_error(ws)
    assert torch.equal(o2, o_ref) and torch.equal(lse2, lse_ref)
    assert np.isfinite(gu.host_f32(o2)).all()
