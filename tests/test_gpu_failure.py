"""Failure detection without a GPU fault: a bounded wait on an mbarrier phase that nothing
completes gives up on its own, reports SFA_ERR_TIMEOUT through the device status word, and
the context stays usable for the next call (the same bounded-wait loop guards every wait of
the attention, estimate and decode kernels)."""

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200 import sfa
from block_sparse_long_dual_b200.synthetic import make_inputs
from block_sparse_long_dual_b200.workloads import TINY

pytestmark = pytest.mark.gpu

SFA_ERR_TIMEOUT = 7


def test_wait_that_nothing_completes_times_out_and_context_survives():
    assert sfa.selftest_bounded_wait(500, complete=True) == 0
    assert sfa.selftest_bounded_wait(300, complete=False) == SFA_ERR_TIMEOUT
    # the context is still usable: a full small path runs and reports no device error
    w = TINY
    Q, K, V = make_inputs(w, seed=0)
    dev = torch.device("cuda")
    m = sfa.PrismAttention(batch=w.batch, heads_q=w.heads_q, heads_kv=w.heads_kv, seq_len=w.seq_len,
                           head_dim=w.head_dim, dtype=w.dtype, block=w.block, rope_base=w.rope_base,
                           band_split=w.band_split, k=w.k, flags=w.flags, device=dev)
    O = m(Q.to(dev), K.to(dev), V.to(dev))
    torch.cuda.synchronize()
    assert int(m.status.item()) == 0
    assert np.isfinite(O.cpu().numpy()).all()
