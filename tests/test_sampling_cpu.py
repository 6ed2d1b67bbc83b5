"""The compaction the full-size backward check uses (one query block's selected keys laid end to
end, positions moved) gives the same oracle gradients as the full-plane call."""
import numpy as np

import oracle
from tests import gpu_util as gu


def test_compacted_backward_equals_full_plane():
    rng = np.random.Generator(np.random.PCG64(31))
    block, nb, D = 8, 12, 16
    K = rng.standard_normal((nb * block, D))
    V = rng.standard_normal((nb * block, D))
    for (i, sel, causal) in [(9, [0, 3, 7, 9], True), (9, [1, 2, 5], True), (4, [0, 4, 8, 11], False)]:
        t = np.arange(block)
        Q = rng.standard_normal((block, D))
        dO = rng.standard_normal((block, D))
        dq, dk, dv = oracle.attend_backward(Q, i * block + t, K, V, sel, block, causal, 0.3, dO)
        rows, q_pos, blocks = gu.compact_row_problem(sel, i, block, causal, t)
        dq2, dk2, dv2 = oracle.attend_backward(Q, q_pos, K[rows], V[rows], blocks, block, causal, 0.3, dO)
        assert np.allclose(dq, dq2, atol=1e-12)
        assert np.allclose(dk[rows], dk2, atol=1e-12) and np.allclose(dv[rows], dv2, atol=1e-12)
        rest = np.setdiff1d(np.arange(nb * block), rows)
        assert not dk[rest].any() and not dv[rest].any()
