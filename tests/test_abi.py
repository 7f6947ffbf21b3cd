"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before touching the GPU (these run without a GPU)."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from block_sparse_long_dual_b200 import build as sfa_build
from block_sparse_long_dual_b200 import sfa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    sfa_build.build()
    return sfa.load()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?[\s\*])(sfa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sfa_block_scores", "sfa_select", "sfa_block_sparse_attn", "sfa_block_scores_select",
                     "sfa_block_sparse_attn_rope",
                     "sfa_rope_table",
                     "sfa_block_scores_workspace", "sfa_workspace_layout", "sfa_status_string", "sfa_version"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.sfa_version() >= 100
    for code in range(9):
        assert lib.sfa_status_string(code)
    assert lib.sfa_status_string(99) == b"unknown status"


def S(B=1, Hq=4, Hkv=2, L=1024, d=128, dt=sfa.BF16):
    return sfa.Shape(B, Hq, Hkv, L, d, dt)


@pytest.mark.parametrize("shape,block,code", [
    (S(L=1000), 128, 2),           # L not a multiple of the block
    (S(), 96, 2),                  # block not 64 / 128
    (S(d=96), 128, 2),             # head dim
    (S(Hq=6, Hkv=4), 128, 2),      # heads_q % heads_kv
    (S(dt=7), 128, 3),             # dtype
    (S(L=128 * 4096), 128, 4),     # nb > 2048
    (S(B=256, Hq=32, Hkv=8, L=1 << 18), 128, 4),   # B * Hq * L = 2^31 rows: past int32
    (S(B=0), 128, 2),
])
def test_shape_validation(lib, shape, block, code):
    assert lib.sfa_block_scores_workspace(ctypes.byref(shape), block) == 0
    off = (ctypes.c_size_t * 4)()
    assert lib.sfa_workspace_layout(ctypes.byref(shape), block, off) == code
    rope = sfa.Rope(None, None, 0)
    dummy = ctypes.c_void_p(256)
    assert lib.sfa_block_scores(ctypes.byref(shape), dummy, dummy, ctypes.byref(rope), 16, block, 0, None, None,
                                dummy, dummy, 1 << 30, None) == code
    assert lib.sfa_select(ctypes.byref(shape), block, dummy, 4, 0.0, 0, dummy, dummy, 64, None) == code
    assert lib.sfa_block_scores_select(ctypes.byref(shape), dummy, dummy, ctypes.byref(rope), 16, block, 0, 4, 0.0,
                                       None, None, None, dummy, dummy, 64, dummy, 1 << 30, None) == code
    assert lib.sfa_block_sparse_attn(ctypes.byref(shape), block, dummy, dummy, dummy, dummy, dummy, 8, 1, 0.0,
                                     dummy, None, None, None) == code


def test_row_limit_is_exclusive_at_2_to_the_31(lib):
    below = S(B=255, Hq=32, Hkv=8, L=1 << 18)          # 255 * 32 * 2^18 rows < 2^31
    nb = (1 << 18) // 128
    want = 255 * 32 * nb * 128 * 8                        # Qbar alone, float64
    assert lib.sfa_block_scores_workspace(ctypes.byref(below), 128) > want


def test_workspace_layout_matches_documented_sizes(lib):
    shape = S(B=2, Hq=4, Hkv=2, L=2048, d=128)
    nb = 16
    off = sfa.workspace_layout(shape, 128)
    assert off[0] == 0
    assert off[1] >= 2 * 4 * nb * 128 * 8 and off[1] % 256 == 0
    assert off[2] >= off[1] + 2 * 2 * nb * 128 * 8 and off[2] % 256 == 0
    assert off[3] >= off[2] + 2 * 6 * nb * 4 * 8 and off[3] % 256 == 0
    total = lib.sfa_block_scores_workspace(ctypes.byref(shape), 128)
    assert total >= off[3] + 2 * 4 * 2 * 8


def test_argument_validation_before_launch(lib):
    shape = S()
    d = ctypes.c_void_p(1 << 20)
    rope = sfa.Rope(d, d, 1)
    ws = lib.sfa_block_scores_workspace(ctypes.byref(shape), 128)
    bs = lib.sfa_block_scores
    # null Q / probs, band_split out of range, unknown flags, rope without rotated outputs
    assert bs(ctypes.byref(shape), None, d, ctypes.byref(rope), 16, 128, 0, d, d, d, d, ws, None) == 1
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 0, d, d, None, d, ws, None) == 1
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 65, 128, 0, d, d, d, d, ws, None) == 1
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), -1, 128, 0, d, d, d, d, ws, None) == 1
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 64, d, d, d, d, ws, None) == 1
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 32 | 2, d, d, d, d, ws, None) == 1  # block tau + no calib
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 32 | 8, d, d, d, d, ws, None) == 1
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 0, d, None, d, d, ws, None) == 1  # no K_rot
    # misaligned pointers
    assert bs(ctypes.byref(shape), ctypes.c_void_p((1 << 20) + 2), d, ctypes.byref(rope), 16, 128, 0, d, d, d, d,
              ws, None) == 1
    # workspace too small / missing / misaligned
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 0, d, d, d, d, ws - 1, None) == 5
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 0, d, d, d, None, ws, None) == 5
    assert bs(ctypes.byref(shape), d, d, ctypes.byref(rope), 16, 128, 0, d, d, d, ctypes.c_void_p((1 << 20) + 16),
              ws, None) == 5
    sel = lib.sfa_select
    nb = 8
    assert sel(ctypes.byref(shape), 128, d, -1, 0.0, 0, d, d, nb, None) == 1     # mass 0
    assert sel(ctypes.byref(shape), 128, d, -1, 1.5, 0, d, d, nb, None) == 1     # mass > 1
    assert sel(ctypes.byref(shape), 128, d, -1, 0.9, 0, d, d, nb - 1, None) == 1  # kmax < nb for mass
    assert sel(ctypes.byref(shape), 128, d, 3, 0.0, 0, d, d, 3, None) == 1       # kmax < k + 1
    assert sel(ctypes.byref(shape), 128, d, 3, 0.0, 1, d, d, 4, None) == 1       # kmax < k + 2 with sink
    assert sel(ctypes.byref(shape), 128, None, 3, 0.0, 0, d, d, 4, None) == 1
    assert sel(ctypes.byref(shape), 128, d, 3, 0.0, 64, d, d, 4, None) == 1      # unknown flag
    at = lib.sfa_block_sparse_attn
    assert at(ctypes.byref(shape), 128, d, d, d, d, d, 0, 1, 0.0, d, None, None, None) == 1  # kmax 0
    assert at(ctypes.byref(shape), 128, d, None, d, d, d, 4, 1, 0.0, d, None, None, None) == 1
    assert at(ctypes.byref(shape), 128, d, d, d, d, d, 4, 1, float("nan"), d, None, None, None) == 1
    assert lib.sfa_rope_table(0.0, 16, 64, d, d, None) == 1
    assert lib.sfa_rope_table(1e4, 16, 63, d, d, None) == 2
    assert lib.sfa_rope_table(1e4, 0, 64, d, d, None) == 2


def test_fused_scores_select_validation(lib):
    shape = S()  # nb = 8
    d = ctypes.c_void_p(1 << 20)
    rope = sfa.Rope(d, d, 1)
    ws = lib.sfa_block_scores_workspace(ctypes.byref(shape), 128)
    f = lib.sfa_block_scores_select
    R = ctypes.byref(rope)
    sh = ctypes.byref(shape)
    # score-side errors: null Q, band_split, unknown flag, rope outputs, workspace
    assert f(sh, None, d, R, 16, 128, 0, 4, 0.0, d, d, None, d, d, 5, d, ws, None) == 1
    assert f(sh, d, d, R, 65, 128, 0, 4, 0.0, d, d, None, d, d, 5, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 64, 4, 0.0, d, d, None, d, d, 6, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 0, 4, 0.0, d, None, None, d, d, 5, d, ws, None) == 1  # no K_rot
    assert f(sh, d, d, R, 16, 128, 0, 4, 0.0, d, d, None, d, d, 5, d, ws - 1, None) == 5
    # selection-side errors: null counts / idx, kmax too small, mass out of range
    assert f(sh, d, d, R, 16, 128, 0, 4, 0.0, d, d, None, None, d, 5, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 0, 4, 0.0, d, d, None, d, None, 5, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 0, 4, 0.0, d, d, None, d, d, 4, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 1, 4, 0.0, d, d, None, d, d, 5, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 0, -1, 0.0, d, d, None, d, d, 8, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 0, -1, 1.5, d, d, None, d, d, 8, d, ws, None) == 1
    assert f(sh, d, d, R, 16, 128, 0, -1, 0.9, d, d, None, d, d, 7, d, ws, None) == 1
    # probs may be NULL here, unlike sfa_block_scores
    assert lib.sfa_block_scores(sh, d, d, R, 16, 128, 0, d, d, None, d, ws, None) == 1


def test_attn_rope_validation(lib):
    shape = S()
    d = ctypes.c_void_p(1 << 20)
    f = lib.sfa_block_sparse_attn_rope
    sh = ctypes.byref(shape)
    good = sfa.Rope(d, d, 1)
    assert f(sh, 128, d, None, d, d, d, d, 8, 1, 0.0, d, None, None, None) == 1            # no tables
    assert f(sh, 128, d, ctypes.byref(sfa.Rope(d, d, 0)), d, d, d, d, 8, 1, 0.0, d, None, None, None) == 1
    assert f(sh, 128, d, ctypes.byref(sfa.Rope(None, d, 1)), d, d, d, d, 8, 1, 0.0, d, None, None, None) == 1
    assert f(sh, 128, d, ctypes.byref(sfa.Rope(ctypes.c_void_p((1 << 20) + 4), d, 1)), d, d, d, d, 8, 1, 0.0, d,
             None, None, None) == 1                                                       # misaligned table
    assert f(sh, 128, d, ctypes.byref(good), None, d, d, d, 8, 1, 0.0, d, None, None, None) == 1  # no K_rot
    assert f(sh, 128, d, ctypes.byref(good), d, d, d, d, 0, 1, 0.0, d, None, None, None) == 1     # kmax 0
    bad = S(L=1000)
    assert f(ctypes.byref(bad), 128, d, ctypes.byref(good), d, d, d, d, 8, 1, 0.0, d, None, None, None) == 2


def test_decode_validation(lib):
    d = ctypes.c_void_p(1 << 20)
    sh = S(B=2, Hq=8, Hkv=2, L=5000)
    fc = (ctypes.c_int * 8)(0, 5, 9, 63, 1, 2, 3, 4)
    ws = lib.sfa_decode_workspace(ctypes.byref(sh), 256)
    assert ws >= 2 * 8 * 2 * 256 * 8
    g = lib.sfa_decode_fc_gather
    assert g(ctypes.byref(S(B=2, Hq=8, Hkv=2, L=5000, dt=sfa.F32)), d, fc, 4, 0, 5000, d, None) == 3
    assert g(ctypes.byref(S(B=1, Hq=18, Hkv=2, L=50)), d, fc, 4, 0, 50, d, None) == 4  # group 9
    assert g(ctypes.byref(sh), d, fc, 3, 0, 5000, d, None) == 1                    # nfc % 4
    assert g(ctypes.byref(sh), d, fc, 68, 0, 5000, d, None) == 1                   # nfc > d/2 (rejected before fc is read)
    bad = (ctypes.c_int * 8)(0, 5, 9, 64, 1, 2, 3, 4)                             # pair 64 >= d/2
    assert g(ctypes.byref(sh), d, bad, 4, 0, 5000, d, None) == 1
    dup = (ctypes.c_int * 8)(0, 5, 5, 6, 1, 2, 3, 4)
    assert g(ctypes.byref(sh), d, dup, 4, 0, 5000, d, None) == 1
    assert g(ctypes.byref(sh), d, fc, 4, 4000, 1001, d, None) == 1                 # past L
    assert g(ctypes.byref(sh), d, fc, 4, -1, 10, d, None) == 1
    assert g(ctypes.byref(sh), d, None, 4, 0, 10, d, None) == 1
    s = lib.sfa_decode_select
    assert s(ctypes.byref(sh), d, d, fc, 4, 0, d, d, ws, None, None) == 1          # k = 0
    assert s(ctypes.byref(sh), d, d, fc, 4, 256, d, d, ws - 1, None, None) == 5
    assert s(ctypes.byref(sh), d, d, fc, 4, 256, d, None, ws, None, None) == 5
    assert s(ctypes.byref(sh), None, d, fc, 4, 256, d, d, ws, None, None) == 1
    a = lib.sfa_decode_attn
    assert a(ctypes.byref(sh), d, d, d, d, 0, 0.0, d, None, None, None) == 1        # k = 0
    assert a(ctypes.byref(sh), d, d, d, None, 8, 0.0, d, None, None, None) == 1
    assert a(ctypes.byref(sh), d, d, d, d, 8, float("inf"), d, None, None, None) == 1
    assert a(ctypes.byref(S(d=96)), d, d, d, d, 8, 0.0, d, None, None, None) == 2
    assert lib.sfa_decode_workspace(ctypes.byref(sh), 0) == 0


def test_selftest_validation(lib):
    d = ctypes.c_void_p(1 << 20)
    assert lib.sfa_selftest_bounded_wait(None, 100, 0, None) == 1
    assert lib.sfa_selftest_bounded_wait(d, 0, 0, None) == 1
    assert lib.sfa_selftest_bounded_wait(d, 20000, 0, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sfa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sfa, "_lib", None)
    with pytest.raises(ImportError):
        sfa.load()


def test_binding_checks_buffer_shapes_before_any_call():
    """The binding rejects a buffer of the wrong shape or dtype before the library sees its pointer."""
    t = torch.zeros((1, 2, 256, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        sfa._expect(torch.zeros((1, 2, 128, 64), dtype=torch.bfloat16), "Q_rot", t.shape, t.dtype)
    with pytest.raises(ValueError, match="float32"):
        sfa._expect(torch.zeros((4, 4), dtype=torch.float64), "probs", (4, 4), torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        sfa._expect(torch.zeros((4, 4), dtype=torch.float32), "probs", (4, 4), torch.float32)
    sfa._expect(None, "lse", (1,), torch.float32)  # optional buffers may be absent


class _FakeCuda:
    """Stands in for a CUDA tensor on a CPU-only host: only what the binding's checks read."""

    def __init__(self, index, shape=(1,), dtype=torch.int32):
        self.is_cuda = True
        self.device = torch.device("cuda", index)
        self.shape = torch.Size(shape)
        self.dtype = dtype

    def is_contiguous(self):
        return True

    def numel(self):
        return int(np.prod(self.shape))

    def dim(self):
        return len(self.shape)


def test_binding_rejects_buffers_of_another_device(lib, monkeypatch):
    """Every kernel launches on the current device, so a buffer, status word or stream of another
    device is refused before its pointer reaches the library."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    sfa._cuda(_FakeCuda(0), "q")
    with pytest.raises(ValueError, match="current CUDA device"):
        sfa._cuda(_FakeCuda(1), "q")
    with pytest.raises(ValueError, match="current CUDA device"):
        sfa._expect(_FakeCuda(1, (4,), torch.float32), "lse", (4,), torch.float32)
    sfa._status(None)
    sfa._status(_FakeCuda(0))
    with pytest.raises(ValueError, match="int32"):
        sfa._status(_FakeCuda(0, dtype=torch.float32))
    with pytest.raises(ValueError, match="current CUDA device"):
        sfa._status(_FakeCuda(1))
    sfa._workspace(_FakeCuda(0, (256,), torch.uint8))
    with pytest.raises(ValueError, match="uint8"):
        sfa._workspace(_FakeCuda(0, (64,), torch.int32))
    with pytest.raises(ValueError, match="current CUDA device"):
        sfa._workspace(_FakeCuda(1, (256,), torch.uint8))

    class OtherStream:
        device = torch.device("cuda", 1)
        cuda_stream = 0

    with pytest.raises(ValueError, match="current CUDA device"):
        sfa._stream(OtherStream())
    q = _FakeCuda(0, (1, 4, 128), torch.bfloat16)
    cache = _FakeCuda(1, (1, 1, 64, 128), torch.bfloat16)
    idx = _FakeCuda(0, (1, 4, 8), torch.int32)
    with pytest.raises(ValueError, match="current CUDA device"):
        sfa.decode_attn(q, cache, cache, idx)
