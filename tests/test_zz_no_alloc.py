"""sfa_block_scores_noalloc: the scoring entry point for callers that cannot allocate.

Plugin code hosted by a runtime that owns all device memory, or code in a
process whose memory another allocator has already reserved, cannot hand the
library a scratch workspace.  The no-allocation variant keeps its scratch in a
fixed 16 MiB device array inside the library.  This test calls it through the
C ABI twice in a row (a small shape, then a larger one, so the second call
reads scratch regions the first did not cover and runs on what the first left)
and checks each result against the workspace-taking sfa_block_scores: the
same kernels on the same inputs, so the outputs must be identical bit for bit.
It also checks that shapes over the limit are refused.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes
from ctypes import POINTER, c_int, c_uint, c_void_p

import pytest
import torch

from block_sparse_long_dual_b200 import sfa
from block_sparse_long_dual_b200.synthetic import make_inputs
from block_sparse_long_dual_b200.workloads import LLAMA_32K, TINY

pytestmark = pytest.mark.gpu

SFA_ERR_WORKSPACE = 5


def _noalloc(lib):
    fn = lib.sfa_block_scores_noalloc
    fn.restype = c_int
    fn.argtypes = [POINTER(sfa.Shape), c_void_p, c_void_p, POINTER(sfa.Rope), c_int, c_int, c_uint, c_void_p,
                   c_void_p, c_void_p, c_void_p]
    return fn


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_no_alloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = sfa.load()
    fn = _noalloc(lib)
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    for w in (TINY, LLAMA_32K):   # two calls in a row, the larger shape second
        Q, K, _ = make_inputs(w, seed=3)
        Qd, Kd = Q.to(dev), K.to(dev)
        cos, sin = sfa.rope_table(w.rope_base, w.seq_len, w.head_dim, device=dev)
        Qr_ref, Kr_ref, P_ref, _ = sfa.block_scores(Qd, Kd, cos, sin, band_split=w.band_split, block=w.block,
                                                    flags=w.flags)
        shape = sfa.make_shape(Qd, Kd)
        rope = sfa.Rope(cos.data_ptr(), sin.data_ptr(), 1)
        Qr, Kr = torch.empty_like(Qd), torch.empty_like(Kd)
        P = torch.full_like(P_ref, float("nan"))
        rc = fn(ctypes.byref(shape), _p(Qd), _p(Kd), ctypes.byref(rope), w.band_split, w.block, w.flags, _p(Qr),
                _p(Kr), _p(P), ctypes.c_void_p(stream.cuda_stream))
        assert rc == 0, lib.sfa_status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(Qr, Qr_ref) and torch.equal(Kr, Kr_ref)
        assert torch.equal(P, P_ref)


def test_no_alloc_refuses_shapes_over_the_limit():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = sfa.load()
    fn = _noalloc(lib)
    shape = sfa.Shape(1, 32, 8, 65536, 128, sfa.BF16)   # needs ~21 MiB of scratch
    assert lib.sfa_block_scores_workspace(ctypes.byref(shape), 128) > (16 << 20)
    d = ctypes.c_void_p(1 << 20)
    rope = sfa.Rope(d, d, 1)
    assert fn(ctypes.byref(shape), d, d, ctypes.byref(rope), 32, 128, 0, d, d, d, None) == SFA_ERR_WORKSPACE
