"""Python binding of the C-ABI library ``libsfa.so`` (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module only
checks tensor shapes / dtypes / devices, allocates outputs with PyTorch and
passes raw device pointers plus the current CUDA stream.  If the library is
missing it raises: there is no fallback.

Names follow include/sfa.h: ``rope_table``, ``block_scores``, ``select``,
``block_sparse_attn``; ``PrismAttention`` chains the three calls of the
estimate -> select -> attend path of "Prism: Spectral-Aware Block-Sparse
Attention" for one fixed layer shape with preallocated buffers.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int, c_int32, c_size_t, c_uint, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsfa.so")

F32, BF16 = 0, 1
KEEP_SINK, NO_CALIB, SINGLE_BAND, RELATIVE_CALIB, BAND_MAX, BLOCK_TAU = 1, 2, 4, 8, 16, 32
STATUS = {0: "SFA_OK", 1: "SFA_ERR_INVALID_ARG", 2: "SFA_ERR_SHAPE", 3: "SFA_ERR_DTYPE",
          4: "SFA_ERR_UNSUPPORTED", 5: "SFA_ERR_WORKSPACE", 6: "SFA_ERR_CUDA", 7: "SFA_ERR_TIMEOUT",
          8: "SFA_ERR_INDEX"}


class SfaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("heads_q", c_int32), ("heads_kv", c_int32),
                ("seq_len", c_int32), ("head_dim", c_int32), ("dtype", c_int32)]


class Rope(ctypes.Structure):
    _fields_ = [("cos", c_void_p), ("sin", c_void_p), ("apply", c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libsfa.so (built by ``block_sparse_long_dual_b200.build``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} not found: build it with `python -m block_sparse_long_dual_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.sfa_version.restype = c_int
    lib.sfa_status_string.restype = ctypes.c_char_p
    lib.sfa_status_string.argtypes = [c_int]
    lib.sfa_rope_table.restype = c_int
    lib.sfa_rope_table.argtypes = [c_double, c_int, c_int, c_void_p, c_void_p, c_void_p]
    lib.sfa_block_scores_workspace.restype = c_size_t
    lib.sfa_block_scores_workspace.argtypes = [POINTER(Shape), c_int]
    lib.sfa_workspace_layout.restype = c_int
    lib.sfa_workspace_layout.argtypes = [POINTER(Shape), c_int, POINTER(c_size_t)]
    lib.sfa_block_scores.restype = c_int
    lib.sfa_block_scores.argtypes = [POINTER(Shape), c_void_p, c_void_p, POINTER(Rope), c_int, c_int, c_uint,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
    lib.sfa_block_scores_select.restype = c_int
    lib.sfa_block_scores_select.argtypes = [POINTER(Shape), c_void_p, c_void_p, POINTER(Rope), c_int, c_int, c_uint,
                                            c_int, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_int, c_void_p, c_size_t, c_void_p]
    lib.sfa_select.restype = c_int
    lib.sfa_select.argtypes = [POINTER(Shape), c_int, c_void_p, c_int, c_float, c_uint, c_void_p, c_void_p,
                               c_int, c_void_p]
    lib.sfa_block_sparse_attn.restype = c_int
    lib.sfa_block_sparse_attn.argtypes = [POINTER(Shape), c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_int, c_int, c_float, c_void_p, c_void_p, c_void_p,
                                          c_void_p]
    lib.sfa_block_sparse_attn_rope.restype = c_int
    lib.sfa_block_sparse_attn_rope.argtypes = [POINTER(Shape), c_int, c_void_p, POINTER(Rope), c_void_p, c_void_p,
                                               c_void_p, c_void_p, c_int, c_int, c_float, c_void_p, c_void_p,
                                               c_void_p, c_void_p]
    lib.sfa_decode_workspace.restype = c_size_t
    lib.sfa_decode_workspace.argtypes = [POINTER(Shape), c_int]
    lib.sfa_decode_fc_gather.restype = c_int
    lib.sfa_decode_fc_gather.argtypes = [POINTER(Shape), c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p]
    lib.sfa_decode_select.restype = c_int
    lib.sfa_decode_select.argtypes = [POINTER(Shape), c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                      c_size_t, c_void_p, c_void_p]
    lib.sfa_decode_attn.restype = c_int
    lib.sfa_decode_attn.argtypes = [POINTER(Shape), c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_float,
                                    c_void_p, c_void_p, c_void_p, c_void_p]
    lib.sfa_selftest_bounded_wait.restype = c_int
    lib.sfa_selftest_bounded_wait.argtypes = [c_void_p, ctypes.c_uint, c_int, c_void_p]
    _lib = lib
    return lib


def _check(code: int, what: str):
    if code != 0:
        raise SfaError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cur = torch.cuda.current_device()
    if stream.device.index != cur:
        raise ValueError(f"stream belongs to {stream.device} but the current CUDA device is cuda:{cur}")
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _cuda(t: torch.Tensor, name: str):
    """A contiguous tensor on the current CUDA device: the library launches every kernel on the
    calling thread's current device, so a buffer of another device would be read through a foreign
    pointer."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current CUDA device is cuda:{cur}")


def _status(status):
    """The optional device status word: an int32 CUDA tensor with at least one element."""
    if status is None:
        return
    if status.dtype != torch.int32 or status.numel() < 1:
        raise ValueError("status must be an int32 tensor with at least one element")
    _cuda(status, "status")


def _workspace(workspace):
    if workspace.dtype != torch.uint8 or workspace.dim() != 1:
        raise ValueError("workspace must be a 1-D uint8 tensor")
    _cuda(workspace, "workspace")


def _expect(t, name: str, shape, dtype, device=None):
    """The library takes raw pointers, so every buffer's shape, dtype, layout and device is checked
    here before a kernel can read or write past it."""
    if t is None:
        return
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} must have shape {tuple(int(x) for x in shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    _cuda(t, name)
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def make_shape(Q: torch.Tensor, K: torch.Tensor) -> Shape:
    if Q.dim() != 4 or K.dim() != 4:
        raise ValueError("Q and K must be [B, H, L, d]")
    B, Hq, L, d = Q.shape
    if K.shape[0] != B or K.shape[2] != L or K.shape[3] != d or K.dtype != Q.dtype:
        raise ValueError("K must be [B, Hkv, L, d] with the dtype of Q")
    return Shape(B, Hq, K.shape[1], L, d, _dtype_code(Q))


def rope_table(base: float, seq_len: int, head_dim: int, device="cuda", stream=None):
    """cos/sin tables [seq_len, head_dim/2] float32 on ``device`` (sfa_rope_table)."""
    lib = load()
    cos = torch.empty((seq_len, head_dim // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    _check(lib.sfa_rope_table(float(base), seq_len, head_dim, _ptr(cos), _ptr(sin), _stream(stream)),
           "sfa_rope_table")
    return cos, sin


def workspace_bytes(shape: Shape, block: int) -> int:
    return int(load().sfa_block_scores_workspace(ctypes.byref(shape), block))


def workspace_layout(shape: Shape, block: int):
    off = (c_size_t * 4)()
    _check(load().sfa_workspace_layout(ctypes.byref(shape), block, off), "sfa_workspace_layout")
    return [int(x) for x in off]


def workspace_views(ws: torch.Tensor, shape: Shape, block: int):
    """Qbar, Kbar, energy, tau views of a workspace buffer (see include/sfa.h)."""
    off = workspace_layout(shape, block)
    nb = shape.seq_len // block
    B, Hq, Hkv, d = shape.batch, shape.heads_q, shape.heads_kv, shape.head_dim

    def view(i, n, dt, shp):
        nbytes = n * torch.tensor([], dtype=dt).element_size()
        return ws[off[i]:off[i] + nbytes].view(dt).view(*shp)

    return (view(0, B * Hq * nb * d, torch.float64, (B, Hq, nb, d)),
            view(1, B * Hkv * nb * d, torch.float64, (B, Hkv, nb, d)),
            view(2, B * (Hq + Hkv) * nb * 4, torch.float64, (B, Hq + Hkv, nb, 4)),
            view(3, B * Hq * 2, torch.float64, (B, Hq, 2)))


def _check_score_buffers(Q, K, cos, sin, apply_rope, Q_rot, K_rot, probs, workspace, nb):
    dev = Q.device
    _expect(K, "K", K.shape, Q.dtype, dev)
    if apply_rope:
        half = Q.shape[-1] // 2
        _expect(cos, "cos", (Q.shape[2], half), torch.float32, dev)
        _expect(sin, "sin", (Q.shape[2], half), torch.float32, dev)
        _expect(Q_rot, "Q_rot", Q.shape, Q.dtype, dev)
        _expect(K_rot, "K_rot", K.shape, K.dtype, dev)
    _expect(probs, "probs", (Q.shape[0], Q.shape[1], nb, nb), torch.float32, dev)
    _workspace(workspace)


def block_scores(Q, K, cos, sin, *, band_split: int, block: int, flags: int = 0, apply_rope: bool = True,
                 Q_rot=None, K_rot=None, probs=None, workspace=None, store_q_rot: bool = True, stream=None):
    """sfa_block_scores: returns (Q_rot, K_rot, probs, workspace).

    ``store_q_rot=False`` passes a NULL Q_rot (the rotated Q is not written; Q_rot is returned as None)."""
    lib = load()
    _cuda(Q, "Q"); _cuda(K, "K")
    shape = make_shape(Q, K)
    nb = shape.seq_len // block if block > 0 else 0
    if apply_rope and not store_q_rot:
        Q_rot = None
    elif apply_rope:
        Q_rot = torch.empty_like(Q) if Q_rot is None else Q_rot
        K_rot = torch.empty_like(K) if K_rot is None else K_rot
        _cuda(cos, "cos"); _cuda(sin, "sin")
    if probs is None:
        probs = torch.empty((shape.batch, shape.heads_q, nb, nb), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(shape, block), 256), dtype=torch.uint8, device=Q.device)
    _check_score_buffers(Q, K, cos, sin, apply_rope, Q_rot, K_rot, probs, workspace, nb)
    rope = Rope(cos.data_ptr() if apply_rope else None, sin.data_ptr() if apply_rope else None,
                1 if apply_rope else 0)
    _check(lib.sfa_block_scores(ctypes.byref(shape), _ptr(Q), _ptr(K), ctypes.byref(rope), band_split, block,
                                flags, _ptr(Q_rot) if apply_rope else None, _ptr(K_rot) if apply_rope else None,
                                _ptr(probs), _ptr(workspace), workspace.numel(), _stream(stream)),
           "sfa_block_scores")
    return (Q_rot if apply_rope else Q), (K_rot if apply_rope else K), probs, workspace


def block_scores_select(Q, K, cos, sin, *, band_split: int, block: int, k: int | None = None,
                        mass: float | None = None, flags: int = 0, apply_rope: bool = True, Q_rot=None, K_rot=None,
                        probs=None, want_probs: bool = False, kmax: int | None = None, counts=None, idx=None,
                        workspace=None, store_q_rot: bool = True, stream=None):
    """sfa_block_scores_select: returns (Q_rot, K_rot, probs or None, counts, idx, workspace)."""
    lib = load()
    _cuda(Q, "Q"); _cuda(K, "K")
    if (k is None) == (mass is None):
        raise ValueError("give exactly one of k / mass")
    shape = make_shape(Q, K)
    nb = shape.seq_len // block if block > 0 else 0
    if apply_rope and not store_q_rot:
        Q_rot = None
    elif apply_rope:
        Q_rot = torch.empty_like(Q) if Q_rot is None else Q_rot
        K_rot = torch.empty_like(K) if K_rot is None else K_rot
        _cuda(cos, "cos"); _cuda(sin, "sin")
    if probs is None and want_probs:
        probs = torch.empty((shape.batch, shape.heads_q, nb, nb), dtype=torch.float32, device=Q.device)
    kmax = kmax_for(nb, k, flags) if kmax is None else kmax
    if counts is None:
        counts = torch.empty((shape.batch, shape.heads_q, nb), dtype=torch.int32, device=Q.device)
    if idx is None:
        idx = torch.empty((shape.batch, shape.heads_q, nb, max(kmax, 1)), dtype=torch.int32, device=Q.device)
    if workspace is None:
        workspace = torch.empty(max(workspace_bytes(shape, block), 256), dtype=torch.uint8, device=Q.device)
    _check_score_buffers(Q, K, cos, sin, apply_rope, Q_rot, K_rot, probs, workspace, nb)
    _expect(counts, "counts", (shape.batch, shape.heads_q, nb), torch.int32, Q.device)
    _expect(idx, "idx", (shape.batch, shape.heads_q, nb, idx.shape[-1]), torch.int32, Q.device)
    if idx.shape[-1] < kmax:
        raise ValueError(f"idx rows hold {idx.shape[-1]} entries, kmax = {kmax}")
    rope = Rope(cos.data_ptr() if apply_rope else None, sin.data_ptr() if apply_rope else None,
                1 if apply_rope else 0)
    _check(lib.sfa_block_scores_select(ctypes.byref(shape), _ptr(Q), _ptr(K), ctypes.byref(rope), band_split,
                                       block, flags, -1 if k is None else int(k),
                                       0.0 if mass is None else float(mass),
                                       _ptr(Q_rot) if apply_rope else None, _ptr(K_rot) if apply_rope else None,
                                       _ptr(probs), _ptr(counts), _ptr(idx), kmax, _ptr(workspace),
                                       workspace.numel(), _stream(stream)), "sfa_block_scores_select")
    return (Q_rot if apply_rope else Q), (K_rot if apply_rope else K), probs, counts, idx, workspace


def kmax_for(nb: int, k: int | None, flags: int) -> int:
    if k is None:
        return nb
    nforced = 2 if (flags & KEEP_SINK) and nb > 1 else 1
    return min(nb, k + nforced)


def select(probs, shape: Shape, *, block: int, k: int | None = None, mass: float | None = None,
           flags: int = 0, kmax: int | None = None, counts=None, idx=None, stream=None):
    """sfa_select: returns (counts [B,Hq,nb] int32, idx [B,Hq,nb,kmax] int32)."""
    lib = load()
    _cuda(probs, "probs")
    if (k is None) == (mass is None):
        raise ValueError("give exactly one of k / mass")
    nb = shape.seq_len // block
    kmax = kmax_for(nb, k, flags) if kmax is None else kmax
    if counts is None:
        counts = torch.empty((shape.batch, shape.heads_q, nb), dtype=torch.int32, device=probs.device)
    if idx is None:
        idx = torch.empty((shape.batch, shape.heads_q, nb, kmax), dtype=torch.int32, device=probs.device)
    _expect(probs, "probs", (shape.batch, shape.heads_q, nb, nb), torch.float32)
    _expect(counts, "counts", (shape.batch, shape.heads_q, nb), torch.int32, probs.device)
    _expect(idx, "idx", (shape.batch, shape.heads_q, nb, kmax), torch.int32, probs.device)
    _check(lib.sfa_select(ctypes.byref(shape), block, _ptr(probs), -1 if k is None else int(k),
                          0.0 if mass is None else float(mass), flags, _ptr(counts), _ptr(idx), kmax,
                          _stream(stream)), "sfa_select")
    return counts, idx


def _check_attn_buffers(Q, K, V, counts, idx, O, lse, status, block):
    dev = Q.device
    B, Hq, L, _ = Q.shape
    nb = L // block if block > 0 else 0
    _expect(V, "V", K.shape, K.dtype, dev)
    _expect(counts, "counts", (B, Hq, nb), torch.int32, dev)
    _expect(idx, "idx", (B, Hq, nb, idx.shape[-1]), torch.int32, dev)
    _expect(O, "O", Q.shape, Q.dtype, dev)
    _expect(lse, "lse", (B, Hq, L), torch.float32, dev)
    _status(status)


def block_sparse_attn(Q, K, V, counts, idx, *, block: int, causal: bool = True, scale: float = 0.0,
                      O=None, lse=None, status=None, stream=None):
    """sfa_block_sparse_attn: returns O (and writes lse / status when given)."""
    lib = load()
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (counts, "counts"), (idx, "idx")):
        _cuda(t, n)
    shape = make_shape(Q, K)
    if V.shape != K.shape or V.dtype != K.dtype:
        raise ValueError("V must match K")
    O = torch.empty_like(Q) if O is None else O
    _check_attn_buffers(Q, K, V, counts, idx, O, lse, status, block)
    _check(lib.sfa_block_sparse_attn(ctypes.byref(shape), block, _ptr(Q), _ptr(K), _ptr(V), _ptr(counts),
                                     _ptr(idx), idx.shape[-1], 1 if causal else 0, float(scale), _ptr(O),
                                     _ptr(lse), _ptr(status), _stream(stream)), "sfa_block_sparse_attn")
    return O


def block_sparse_attn_rope(Q, cos, sin, K_rot, V, counts, idx, *, block: int, causal: bool = True,
                           scale: float = 0.0, O=None, lse=None, status=None, stream=None):
    """sfa_block_sparse_attn_rope: Q pre-RoPE (rotated on load with the cos/sin tables); returns O."""
    lib = load()
    for t, n in ((Q, "Q"), (cos, "cos"), (sin, "sin"), (K_rot, "K_rot"), (V, "V"), (counts, "counts"),
                 (idx, "idx")):
        _cuda(t, n)
    shape = make_shape(Q, K_rot)
    if V.shape != K_rot.shape or V.dtype != K_rot.dtype:
        raise ValueError("V must match K_rot")
    O = torch.empty_like(Q) if O is None else O
    _expect(cos, "cos", (Q.shape[2], Q.shape[-1] // 2), torch.float32, Q.device)
    _expect(sin, "sin", (Q.shape[2], Q.shape[-1] // 2), torch.float32, Q.device)
    _check_attn_buffers(Q, K_rot, V, counts, idx, O, lse, status, block)
    rope = Rope(cos.data_ptr(), sin.data_ptr(), 1)
    _check(lib.sfa_block_sparse_attn_rope(ctypes.byref(shape), block, _ptr(Q), ctypes.byref(rope), _ptr(K_rot),
                                          _ptr(V), _ptr(counts), _ptr(idx), idx.shape[-1], 1 if causal else 0,
                                          float(scale), _ptr(O), _ptr(lse), _ptr(status), _stream(stream)),
           "sfa_block_sparse_attn_rope")
    return O


class PrismAttention:
    """The whole path for one layer shape: estimate -> select -> exact sparse attention.

    Buffers (rotated Q/K, probabilities, workspace, index lists, output) are
    allocated once here; ``__call__`` only launches the library's kernels.
    With ``fused=True`` the estimate and the selection run as one call
    (sfa_block_scores_select) and the block probabilities are not stored.
    With ``rope_on_load=True`` the rotated Q is not stored: the attention
    (sfa_block_sparse_attn_rope) rotates Q tiles as it loads them."""

    def __init__(self, *, batch, heads_q, heads_kv, seq_len, head_dim, dtype, block, rope_base, band_split,
                 k=None, mass=None, flags=0, causal=True, device="cuda", with_lse=False, fused=False,
                 rope_on_load=False):
        tdt = torch.bfloat16 if dtype in ("bf16", torch.bfloat16) else torch.float32
        self.block, self.band_split, self.k, self.mass, self.flags, self.causal = (
            block, band_split, k, mass, flags, causal)
        self.fused = fused
        self.rope_on_load = rope_on_load
        self.shape = Shape(batch, heads_q, heads_kv, seq_len, head_dim, BF16 if tdt == torch.bfloat16 else F32)
        nb = seq_len // block
        self.nb = nb
        self.kmax = kmax_for(nb, k, flags)
        dev = torch.device(device)
        self.cos, self.sin = rope_table(rope_base, seq_len, head_dim, device=dev)
        self.Q_rot = None if rope_on_load else torch.empty((batch, heads_q, seq_len, head_dim), dtype=tdt,
                                                           device=dev)
        self.K_rot = torch.empty((batch, heads_kv, seq_len, head_dim), dtype=tdt, device=dev)
        self.probs = None if fused else torch.empty((batch, heads_q, nb, nb), dtype=torch.float32, device=dev)
        self.workspace = torch.empty(workspace_bytes(self.shape, block), dtype=torch.uint8, device=dev)
        self.counts = torch.empty((batch, heads_q, nb), dtype=torch.int32, device=dev)
        self.idx = torch.empty((batch, heads_q, nb, self.kmax), dtype=torch.int32, device=dev)
        self.O = torch.empty((batch, heads_q, seq_len, head_dim), dtype=tdt, device=dev)
        self.lse = torch.empty((batch, heads_q, seq_len), dtype=torch.float32, device=dev) if with_lse else None
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def scores(self, Q, K, stream=None):
        block_scores(Q, K, self.cos, self.sin, band_split=self.band_split, block=self.block, flags=self.flags,
                     Q_rot=self.Q_rot, K_rot=self.K_rot, probs=self.probs, workspace=self.workspace,
                     store_q_rot=not self.rope_on_load, stream=stream)

    def scores_select(self, Q, K, stream=None):
        block_scores_select(Q, K, self.cos, self.sin, band_split=self.band_split, block=self.block, k=self.k,
                            mass=self.mass, flags=self.flags, Q_rot=self.Q_rot, K_rot=self.K_rot,
                            probs=self.probs, kmax=self.kmax, counts=self.counts, idx=self.idx,
                            workspace=self.workspace, store_q_rot=not self.rope_on_load, stream=stream)

    def select(self, stream=None):
        select(self.probs, self.shape, block=self.block, k=self.k, mass=self.mass, flags=self.flags,
               kmax=self.kmax, counts=self.counts, idx=self.idx, stream=stream)

    def attend(self, V, Q=None, stream=None):
        """Attention over the selection; ``Q`` (pre-RoPE) is needed only with rope_on_load."""
        if self.rope_on_load:
            if Q is None:
                raise ValueError("rope_on_load: attend() needs the pre-RoPE Q")
            block_sparse_attn_rope(Q, self.cos, self.sin, self.K_rot, V, self.counts, self.idx, block=self.block,
                                   causal=self.causal, O=self.O, lse=self.lse, status=self.status, stream=stream)
        else:
            block_sparse_attn(self.Q_rot, self.K_rot, V, self.counts, self.idx, block=self.block,
                              causal=self.causal, O=self.O, lse=self.lse, status=self.status, stream=stream)

    def __call__(self, Q, K, V, stream=None):
        if self.fused:
            self.scores_select(Q, K, stream)
        else:
            self.scores(Q, K, stream)
            self.select(stream)
        self.attend(V, Q, stream)
        return self.O

    def run_host(self, Q_host, K_host, V_host, O_host, dev_in=None, stream=None):
        """End to end from pinned host tensors: H2D copies, the path, D2H copy of O, all on one
        stream (each step's copies serialise with its kernels; HostPipeline overlaps them)."""
        if dev_in is None:
            dev_in = tuple(torch.empty(t.shape, dtype=t.dtype, device=self.O.device) for t in (Q_host, K_host, V_host))
        for d, h in zip(dev_in, (Q_host, K_host, V_host)):
            d.copy_(h, non_blocking=True)
        self(*dev_in, stream=stream)
        O_host.copy_(self.O, non_blocking=True)
        return O_host


class HostPipeline:
    """Layers fed from and returned to pinned host memory, with the copies overlapped.

    Step n's inputs go host -> device on an upload stream and its output device -> host on a
    download stream, while step n - 1's path runs on the compute stream: device inputs and
    outputs are double-buffered and events order each buffer's reuse (an upload waits until the
    path of the step two back has read that input buffer; a path waits until the download of the
    step two back has read that output buffer).  The library's kernels are the ones PrismAttention
    launches; only the copies and events are added here."""

    def __init__(self, model: PrismAttention, like_q, like_k, like_v):
        dev = model.O.device
        self.model = model
        self.dev_in = [tuple(torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (like_q, like_k, like_v))
                       for _ in range(2)]
        self.dev_out = [model.O, torch.empty_like(model.O)]
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        self.in_ready, self.in_free, self.out_ready, self.out_free = ev(), ev(), ev(), ev()
        self.n = 0

    def submit(self, Q_host, K_host, V_host, O_host, stream=None):
        """Enqueue one step; O_host is written once the download stream reaches it."""
        comp = torch.cuda.current_stream(self.model.O.device) if stream is None else stream
        s = self.n % 2
        if self.n >= 2:
            self.up.wait_event(self.in_free[s])
        with torch.cuda.stream(self.up):
            for d, h in zip(self.dev_in[s], (Q_host, K_host, V_host)):
                d.copy_(h, non_blocking=True)
            self.in_ready[s].record(self.up)
        comp.wait_event(self.in_ready[s])
        if self.n >= 2:
            comp.wait_event(self.out_free[s])
        self.model.O = self.dev_out[s]
        with torch.cuda.stream(comp):
            self.model(*self.dev_in[s], stream=comp)
            self.in_free[s].record(comp)
            self.out_ready[s].record(comp)
        self.down.wait_event(self.out_ready[s])
        with torch.cuda.stream(self.down):
            O_host.copy_(self.dev_out[s], non_blocking=True)
            self.out_free[s].record(self.down)
        self.n += 1
        return O_host

    def drain(self, stream=None):
        """Make ``stream`` (default: the current one) wait for every copy submitted so far."""
        comp = torch.cuda.current_stream(self.model.O.device) if stream is None else stream
        comp.wait_stream(self.up)
        comp.wait_stream(self.down)


# ---------------------------------------------------------------------------
# Decode step (token importance on dominant rotary pairs -> top-k -> attention)
# ---------------------------------------------------------------------------
def _fc_host(fc) -> tuple:
    """fc [Hkv, nfc] (any int array-like) -> (ctypes int32 array, nfc)."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(fc, dtype=np.int32))
    if a.ndim != 2:
        raise ValueError("fc must be [heads_kv, nfc]")
    return (ctypes.c_int * a.size)(*a.reshape(-1).tolist()), a.shape[1]


def decode_shape(q, K_cache) -> Shape:
    B, Hq, d = q.shape
    return Shape(B, Hq, K_cache.shape[1], K_cache.shape[2], d, _dtype_code(q))


def decode_fc_gather(K_cache, fc, *, K_fc=None, pos0: int = 0, npos: int | None = None, stream=None):
    """sfa_decode_fc_gather: returns K_fc [B, Hkv, L, 2 nfc]."""
    lib = load()
    _cuda(K_cache, "K_cache")
    B, Hkv, L, d = K_cache.shape
    fch, nfc = _fc_host(fc)
    shape = Shape(B, Hkv, Hkv, L, d, _dtype_code(K_cache))
    if K_fc is None:
        K_fc = torch.empty((B, Hkv, L, 2 * nfc), dtype=K_cache.dtype, device=K_cache.device)
    _expect(K_fc, "K_fc", (B, Hkv, L, 2 * nfc), K_cache.dtype, K_cache.device)
    npos = L - pos0 if npos is None else npos
    _check(lib.sfa_decode_fc_gather(ctypes.byref(shape), _ptr(K_cache), fch, nfc, pos0, npos, _ptr(K_fc),
                                    _stream(stream)), "sfa_decode_fc_gather")
    return K_fc


def decode_select(q, K_fc, fc, L: int, *, k: int, idx=None, workspace=None, status=None, stream=None):
    """sfa_decode_select: returns idx [B, Hq, k] int32 (ascending, -1 padded)."""
    lib = load()
    _cuda(q, "q"); _cuda(K_fc, "K_fc")
    B, Hq, d = q.shape
    fch, nfc = _fc_host(fc)
    shape = Shape(B, Hq, K_fc.shape[1], L, d, _dtype_code(q))
    if idx is None:
        idx = torch.empty((B, Hq, k), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(lib.sfa_decode_workspace(ctypes.byref(shape), k), 256), dtype=torch.uint8,
                                device=q.device)
    _expect(K_fc, "K_fc", (B, K_fc.shape[1], L, 2 * nfc), q.dtype, q.device)
    _expect(idx, "idx", (B, Hq, k), torch.int32, q.device)
    _workspace(workspace)
    _status(status)
    _check(lib.sfa_decode_select(ctypes.byref(shape), _ptr(q), _ptr(K_fc), fch, nfc, k, _ptr(idx),
                                 _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
           "sfa_decode_select")
    return idx


def decode_attn(q, K_cache, V_cache, idx, *, scale: float = 0.0, o=None, lse=None, status=None, stream=None):
    """sfa_decode_attn: returns o [B, Hq, d]."""
    lib = load()
    for t, n in ((q, "q"), (K_cache, "K_cache"), (V_cache, "V_cache"), (idx, "idx")):
        _cuda(t, n)
    shape = decode_shape(q, K_cache)
    o = torch.empty_like(q) if o is None else o
    B, Hq, d = q.shape
    if K_cache.dim() != 4 or K_cache.shape[0] != B or K_cache.shape[3] != d:
        raise ValueError("K_cache must be [B, Hkv, L, d] matching q [B, Hq, d]")
    _expect(V_cache, "V_cache", K_cache.shape, K_cache.dtype, q.device)
    _expect(idx, "idx", (B, Hq, idx.shape[-1]), torch.int32, q.device)
    _expect(o, "o", q.shape, q.dtype, q.device)
    _expect(lse, "lse", (B, Hq), torch.float32, q.device)
    _status(status)
    _check(lib.sfa_decode_attn(ctypes.byref(shape), _ptr(q), _ptr(K_cache), _ptr(V_cache), _ptr(idx),
                               idx.shape[-1], float(scale), _ptr(o), _ptr(lse), _ptr(status), _stream(stream)),
           "sfa_decode_attn")
    return o


class FasaDecode:
    """One decode step for a fixed cache shape: TIP on the compact dominant-pair keys, top-k,
    focused attention.  ``fc`` [Hkv, nfc] are the dominant pairs (an input: the offline
    calibration that finds them is not part of this library).  Buffers are allocated once;
    ``refresh_keys`` (re)builds the compact key copy for a position range, ``__call__`` runs
    the step's three kernels."""

    def __init__(self, *, batch, heads_q, heads_kv, seq_len, head_dim, fc, k, device="cuda", with_lse=True):
        self.fc = fc
        self.k = k
        self.shape = Shape(batch, heads_q, heads_kv, seq_len, head_dim, BF16)
        dev = torch.device(device)
        _, nfc = _fc_host(fc)
        self.K_fc = torch.empty((batch, heads_kv, seq_len, 2 * nfc), dtype=torch.bfloat16, device=dev)
        ws = load().sfa_decode_workspace(ctypes.byref(self.shape), k)
        if ws == 0:
            raise SfaError(1, "sfa_decode_workspace")
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.idx = torch.empty((batch, heads_q, k), dtype=torch.int32, device=dev)
        self.o = torch.empty((batch, heads_q, head_dim), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((batch, heads_q), dtype=torch.float32, device=dev) if with_lse else None
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def refresh_keys(self, K_cache, pos0=0, npos=None, stream=None):
        decode_fc_gather(K_cache, self.fc, K_fc=self.K_fc, pos0=pos0, npos=npos, stream=stream)

    def select(self, q, stream=None):
        decode_select(q, self.K_fc, self.fc, self.shape.seq_len, k=self.k, idx=self.idx, workspace=self.workspace,
                      status=self.status, stream=stream)

    def attend(self, q, K_cache, V_cache, stream=None):
        decode_attn(q, K_cache, V_cache, self.idx, o=self.o, lse=self.lse, status=self.status, stream=stream)

    def __call__(self, q, K_cache, V_cache, stream=None):
        self.select(q, stream)
        self.attend(q, K_cache, V_cache, stream)
        return self.o

    def step(self, q, K_cache, V_cache, pos: int):
        """One decode step for the token at position ``pos`` (its compact key row, select, attend)
        replayed as a CUDA graph: captured on the first call for these buffers and this position,
        replayed on later calls (new values in the same q / cache tensors are picked up; the
        kernels, their arguments and the buffers are fixed at capture).  Runs on the current
        stream; returns ``self.o``."""
        key = (q.data_ptr(), K_cache.data_ptr(), V_cache.data_ptr(), int(pos))
        if getattr(self, "_graph_key", None) != key:
            side = torch.cuda.Stream(q.device)
            side.wait_stream(torch.cuda.current_stream(q.device))
            with torch.cuda.stream(side):  # one eager step before capture
                self.refresh_keys(K_cache, pos0=pos, npos=1)
                self(q, K_cache, V_cache)
            torch.cuda.current_stream(q.device).wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                self.refresh_keys(K_cache, pos0=pos, npos=1)
                self(q, K_cache, V_cache)
            self._graph, self._graph_key = graph, key
        self._graph.replay()
        return self.o


def selftest_bounded_wait(limit_ms: int, complete: bool, device="cuda", stream=None) -> int:
    """sfa_selftest_bounded_wait: returns the device status word (0 or SFA_ERR_TIMEOUT)."""
    lib = load()
    status = torch.full((1,), -1, dtype=torch.int32, device=device)
    _status(status)
    _check(lib.sfa_selftest_bounded_wait(_ptr(status), int(limit_ms), 1 if complete else 0, _stream(stream)),
           "sfa_selftest_bounded_wait")
    return int(status.item())
