"""B200 (sm_100a) LSH attention forward pass: Python binding of liblsh_attn.so.

The functions here carry the names of the C ABI in ``include/lsh_attn.h`` and
only marshal arguments: they check dtype/device/contiguity, allocate output
tensors with torch, and pass raw pointers plus the current CUDA stream to the
library.  Every step of the computation runs in the library's CUDA kernels.
There is no fallback: if the shared library is missing or no GPU is present,
the calls raise.

Build the library first:  python -m lsh_bucketed_sparse_b200.build
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

__all__ = [
    "LshError", "Shape", "lib", "make_shape", "lsh_attn_hash", "lsh_attn_sort",
    "lsh_attn_sort_workspace_size",
    "lsh_attn_chunked_fwd", "lsh_attn_chunked_fwd_ex", "lsh_attn_combine", "lsh_attn_forward",
    "lsh_attn_forward_workspace_size", "lsh_attn_forward_host",
    "lsh_attn_forward_host_device_bytes", "lsh_attn_device_check", "lsh_attn_forward_noalloc",
    "lsh_attn_backward", "lsh_attn_backward_workspace_size", "lsh_attn_kernel_launches",
    "LIB_PATH", "HEADER_PATH", "NOALLOC_SCRATCH_BYTES",
    "F32", "BF16", "FLAG_PORTABLE", "FLAG_DEDUP", "FLAG_BUCKET_MASK", "FLAG_KMEANS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "liblsh_attn.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "lsh_attn.h")

F32, BF16 = 0, 1
FLAG_PORTABLE = 1
FLAG_DEDUP = 2
FLAG_BUCKET_MASK = 4
FLAG_KMEANS = 8
NOALLOC_SCRATCH_BYTES = 64 << 20  # LSH_ATTN_NOALLOC_SCRATCH_BYTES
STATUS = {0: "LSH_OK", 1: "LSH_ERR_INVALID_ARG", 2: "LSH_ERR_UNSUPPORTED",
          3: "LSH_ERR_WORKSPACE", 4: "LSH_ERR_CUDA", 5: "LSH_ERR_DEVICE_TIMEOUT"}


class LshError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("seq_len", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("n_hashes", ctypes.c_int32), ("n_buckets", ctypes.c_int32),
                ("chunk_len", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


_lib = None
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_SHP = ctypes.POINTER(Shape)
_SIGS = {
    "lsh_attn_hash": [_SHP, _P, _P, _P, _P, _P],
    "lsh_attn_sort_workspace_size": [_SHP, ctypes.POINTER(_SZ)],
    "lsh_attn_sort": [_SHP, _P, _P, _P, _P, _P, _SZ, _P],
    "lsh_attn_chunked_fwd": [_SHP, _P, _P, _P, _P, _P, _P, _P],
    "lsh_attn_chunked_fwd_ex": [_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "lsh_attn_combine": [_SHP, _P, _P, _P, _P, _P],
    "lsh_attn_forward_workspace_size": [_SHP, ctypes.POINTER(_SZ)],
    "lsh_attn_forward": [_SHP, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "lsh_attn_forward_host_device_bytes": [_SHP, ctypes.POINTER(_SZ)],
    "lsh_attn_forward_host": [_SHP, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "lsh_attn_forward_noalloc": [_SHP, _P, _P, _P, _P, _P, _P],
    "lsh_attn_backward_workspace_size": [_SHP, ctypes.POINTER(_SZ)],
    "lsh_attn_backward": [_SHP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "lsh_attn_status_string": [ctypes.c_int],
    "lsh_attn_last_error": [],
    "lsh_attn_device_check": [_P],
    "lsh_attn_version": [],
    "lsh_attn_kernel_launches": [],
    "lsh_attn_test_hash_first_wait": [ctypes.c_ulonglong],
}


def lib() -> ctypes.CDLL:
    """Load liblsh_attn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m lsh_bucketed_sparse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.lsh_attn_status_string.restype = ctypes.c_char_p
        L.lsh_attn_last_error.restype = ctypes.c_char_p
        L.lsh_attn_kernel_launches.restype = ctypes.c_ulonglong
        L.lsh_attn_test_hash_first_wait.restype = ctypes.c_ulonglong
        _lib = L
    return _lib


def declared_symbols(header: str = HEADER_PATH):
    """Function names the public header declares (LSH_ATTN_API ... name()."""
    with open(header) as f:
        text = f.read()
    return re.findall(r"LSH_ATTN_API\s+[\w\s\*]+?\b(lsh_attn_\w+)\s*\(", text)


def _check(status: int):
    if status != 0:
        raise LshError(status, lib().lsh_attn_last_error().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return F32
    if t == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t}: use float32 or bfloat16")


def make_shape(batch, heads, seq_len, d_k, n_hashes, n_buckets, chunk_len, causal,
               dtype=torch.bfloat16, portable=False, dedup=False, bucket_mask=False,
               kmeans=False) -> Shape:
    return Shape(batch, heads, seq_len, d_k, n_hashes, n_buckets, chunk_len, int(bool(causal)),
                 dtype if isinstance(dtype, int) else _dtype_code(dtype),
                 (FLAG_PORTABLE if portable else 0) | (FLAG_DEDUP if dedup else 0)
                 | (FLAG_BUCKET_MASK if bucket_mask else 0) | (FLAG_KMEANS if kmeans else 0))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, name: str, dtype=None, shape=None, like=None):
    """Checks a tensor argument before its pointer reaches the library, which
    sees only pointers and so cannot check extents: a CUDA tensor, contiguous,
    of ``dtype`` and ``shape`` when given, on ``like``'s device when given."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if like is not None and t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, expected {like.device}")
    return t


def _host(t: torch.Tensor, name: str, dtype, shape):
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _qk(qk):
    _cuda(qk, "qk")
    if qk.dim() != 4:
        raise ValueError(f"qk must be [B, H, L, d], got shape {tuple(qk.shape)}")
    return qk.shape


def _rot_shape(n_hashes, d, n_buckets, kmeans):
    """rotations [n_h, d, n_b/2] (the random rotations), or the centroids
    [n_h, d, n_b] of the routing-style assignment."""
    return (n_hashes, d, n_buckets if kmeans else n_buckets // 2)


def _rotations(rotations, qk, n_hashes, n_buckets, kmeans):
    B, H, L, d = qk.shape
    if n_buckets == 1 and not kmeans:
        if rotations is not None:
            raise ValueError("rotations must be None when n_buckets == 1")
        return
    if rotations is None:
        raise ValueError("rotations is required when n_buckets > 1")
    _cuda(rotations, "rotations", qk.dtype, _rot_shape(n_hashes, d, n_buckets, kmeans), qk)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _shape_of(qk, n_hashes, n_buckets, chunk_len, causal, portable, dedup=False,
              bucket_mask=False, kmeans=False):
    B, H, L, d = qk.shape
    return make_shape(B, H, L, d, n_hashes, n_buckets, chunk_len, causal, qk.dtype, portable,
                      dedup, bucket_mask, kmeans)


# --------------------------------------------------------------------------
def lsh_attn_hash(qk, rotations, n_buckets, n_hashes=None, *, portable=False, kmeans=False,
                  stream=None):
    """Stage 1.  qk [B,H,L,d]; rotations [n_h,d,n_b/2] (None when n_b == 1).
    Returns (buckets int16 [B,H,n_h,L], inv_norm float32 [B,H,L])."""
    B, H, L, d = _qk(qk)
    if rotations is not None and rotations.dim() == 3:
        n_hashes = rotations.shape[0]
    if n_hashes is None:
        n_hashes = 1
    _rotations(rotations, qk, n_hashes, n_buckets, kmeans)
    shp = _shape_of(qk, n_hashes, n_buckets, 1, False, portable, kmeans=kmeans)
    buckets = torch.empty(B, H, n_hashes, L, dtype=torch.int16, device=qk.device)
    inv_norm = torch.empty(B, H, L, dtype=torch.float32, device=qk.device)
    _check(lib().lsh_attn_hash(ctypes.byref(shp), _ptr(qk), _ptr(rotations), _ptr(buckets),
                               _ptr(inv_norm), _stream(stream)))
    return buckets, inv_norm


def lsh_attn_sort(buckets, n_buckets, *, want_undo=True, want_counts=False, stream=None):
    """Stage 2.  buckets int16 [B,H,n_h,L].  Returns (perm, undo, counts); undo and
    counts are None unless asked for."""
    _cuda(buckets, "buckets", torch.int16)
    if buckets.dim() != 4:
        raise ValueError(f"buckets must be [B, H, n_h, L], got shape {tuple(buckets.shape)}")
    B, H, n_h, L = buckets.shape
    shp = make_shape(B, H, L, 8, n_h, n_buckets, 1, False, F32)
    perm = torch.empty(B, H, n_h, L, dtype=torch.int32, device=buckets.device)
    undo = torch.empty_like(perm) if want_undo else None
    counts = torch.empty(B, H, n_h, n_buckets, dtype=torch.int32, device=buckets.device) \
        if want_counts else None
    ws = torch.empty(lsh_attn_sort_workspace_size(shp), dtype=torch.uint8, device=buckets.device)
    _check(lib().lsh_attn_sort(ctypes.byref(shp), _ptr(buckets), _ptr(perm), _ptr(undo),
                               _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)))
    return perm, undo, counts


def lsh_attn_sort_workspace_size(shape: Shape) -> int:
    """Bytes of workspace lsh_attn_sort needs for `shape` (per-tile counts)."""
    n = _SZ()
    _check(lib().lsh_attn_sort_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def _stage3_args(qk, v, inv_norm, perm):
    """qk and v [B,H,L,d], inv_norm [B,H,L], perm [B,H,n_h,L]; returns n_h."""
    B, H, L, d = _qk(qk)
    _cuda(v, "v", qk.dtype, qk.shape, qk)
    _cuda(inv_norm, "inv_norm", torch.float32, (B, H, L), qk)
    _cuda(perm, "perm", torch.int32, None, qk)
    if perm.dim() != 4 or (perm.shape[0], perm.shape[1], perm.shape[3]) != (B, H, L):
        raise ValueError(f"perm must be [{B}, {H}, n_h, {L}], got shape {tuple(perm.shape)}")
    return perm.shape[2]


def lsh_attn_chunked_fwd(qk, v, inv_norm, perm, chunk_len, causal, *, n_buckets=2,
                         portable=False, stream=None):
    """Stage 3.  Returns (o_rounds [B,H,n_h,L,d] in qk's dtype, lse_rounds f32 [B,H,n_h,L])."""
    n_h = _stage3_args(qk, v, inv_norm, perm)
    B, H, L, d = qk.shape
    shp = _shape_of(qk, n_h, n_buckets, chunk_len, causal, portable)
    o_r = torch.empty(B, H, n_h, L, qk.shape[-1], dtype=qk.dtype, device=qk.device)
    lse_r = torch.empty(B, H, n_h, L, dtype=torch.float32, device=qk.device)
    _check(lib().lsh_attn_chunked_fwd(ctypes.byref(shp), _ptr(qk), _ptr(v), _ptr(inv_norm),
                                      _ptr(perm), _ptr(o_r), _ptr(lse_r), _stream(stream)))
    return o_r, lse_r


def lsh_attn_chunked_fwd_ex(qk, v, inv_norm, perm, chunk_len, causal, *, undo=None,
                            buckets=None, n_buckets=2, stream=None):
    """Stage 3 for the variants: the duplicate-count correction when ``undo``
    (every round's [B,H,n_h,L] int32, from lsh_attn_sort) is given, the
    bucket-equality mask when ``buckets`` ([B,H,n_h,L] int16) is given.
    Returns (o_rounds, lse_rounds)."""
    n_h = _stage3_args(qk, v, inv_norm, perm)
    B, H, L, d = qk.shape
    if undo is not None:
        _cuda(undo, "undo", torch.int32, perm.shape, qk)
    if buckets is not None:
        _cuda(buckets, "buckets", torch.int16, perm.shape, qk)
    shp = _shape_of(qk, n_h, n_buckets, chunk_len, causal, False, undo is not None,
                    buckets is not None)
    o_r = torch.empty(B, H, n_h, L, qk.shape[-1], dtype=qk.dtype, device=qk.device)
    lse_r = torch.empty(B, H, n_h, L, dtype=torch.float32, device=qk.device)
    _check(lib().lsh_attn_chunked_fwd_ex(ctypes.byref(shp), _ptr(qk), _ptr(v), _ptr(inv_norm),
                                         _ptr(perm), _ptr(undo), _ptr(buckets), _ptr(o_r),
                                         _ptr(lse_r), _stream(stream)))
    return o_r, lse_r


def lsh_attn_combine(o_rounds, lse_rounds, *, stream=None):
    """Stage 4.  Returns (out [B,H,L,d], lse f32 [B,H,L])."""
    _cuda(o_rounds, "o_rounds")
    if o_rounds.dim() != 5:
        raise ValueError(f"o_rounds must be [B, H, n_h, L, d], got shape {tuple(o_rounds.shape)}")
    B, H, n_h, L, d = o_rounds.shape
    _cuda(lse_rounds, "lse_rounds", torch.float32, (B, H, n_h, L), o_rounds)
    shp = make_shape(B, H, L, d, n_h, 2, 1, False, o_rounds.dtype)
    out = torch.empty(B, H, L, d, dtype=o_rounds.dtype, device=o_rounds.device)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=o_rounds.device)
    _check(lib().lsh_attn_combine(ctypes.byref(shp), _ptr(o_rounds), _ptr(lse_rounds), _ptr(out),
                                  _ptr(lse), _stream(stream)))
    return out, lse


def _outputs(qk, out, lse):
    """out [B,H,L,d] in qk's dtype and lse f32 [B,H,L]: checked, or allocated."""
    B, H, L, d = qk.shape
    if out is None:
        out = torch.empty_like(qk)
    if lse is None:
        lse = torch.empty(B, H, L, dtype=torch.float32, device=qk.device)
    _cuda(out, "out", qk.dtype, qk.shape, qk)
    _cuda(lse, "lse", torch.float32, (B, H, L), qk)
    return out, lse


def lsh_attn_forward_workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().lsh_attn_forward_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def lsh_attn_forward(qk, v, rotations, n_hashes, n_buckets, chunk_len, causal, *,
                     workspace=None, out=None, lse=None, portable=False, dedup=False,
                     bucket_mask=False, kmeans=False, stream=None):
    """The fused pass.  Returns (out [B,H,L,d], lse f32 [B,H,L]).  ``workspace`` (a
    uint8 CUDA tensor) can be passed in to avoid an allocation per call."""
    B, H, L, d = _qk(qk)
    _cuda(v, "v", qk.dtype, qk.shape, qk)
    _rotations(rotations, qk, n_hashes, n_buckets, kmeans)
    shp = _shape_of(qk, n_hashes, n_buckets, chunk_len, causal, portable, dedup, bucket_mask,
                    kmeans)
    need = lsh_attn_forward_workspace_size(shp)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=qk.device)
    _cuda(workspace, "workspace", None, None, qk)
    out, lse = _outputs(qk, out, lse)
    _check(lib().lsh_attn_forward(ctypes.byref(shp), _ptr(qk), _ptr(v), _ptr(rotations),
                                  _ptr(out), _ptr(lse), _ptr(workspace),
                                  ctypes.c_size_t(workspace.numel()), _stream(stream)))
    return out, lse


def lsh_attn_forward_host_device_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().lsh_attn_forward_host_device_bytes(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def lsh_attn_forward_host(shape: Shape, qk_host, v_host, rot_host, out_host, lse_host,
                          device_buffer, *, stream=None):
    """Forward pass from host tensors (ideally pinned): enqueues the copies in,
    the pass and the copies out on ``stream``; the caller synchronises."""
    dt = torch.float32 if shape.dtype == F32 else torch.bfloat16
    x_shape = (shape.batch, shape.heads, shape.seq_len, shape.d_k)
    for name, t in (("qk_host", qk_host), ("v_host", v_host), ("out_host", out_host)):
        _host(t, name, dt, x_shape)
    _host(lse_host, "lse_host", torch.float32, x_shape[:3])
    kmeans = bool(shape.flags & FLAG_KMEANS)
    if shape.n_buckets > 1 or kmeans:
        if rot_host is None:
            raise ValueError("rot_host is required when n_buckets > 1")
        _host(rot_host, "rot_host", dt,
              _rot_shape(shape.n_hashes, shape.d_k, shape.n_buckets, kmeans))
    elif rot_host is not None:
        raise ValueError("rot_host must be None when n_buckets == 1")
    _cuda(device_buffer, "device_buffer")
    _check(lib().lsh_attn_forward_host(
        ctypes.byref(shape), _ptr(qk_host), _ptr(v_host), _ptr(rot_host), _ptr(out_host),
        _ptr(lse_host), _ptr(device_buffer), ctypes.c_size_t(device_buffer.numel()),
        _stream(stream)))


def lsh_attn_forward_noalloc(qk, v, rotations, n_hashes, n_buckets, chunk_len, causal, *,
                             out=None, lse=None, portable=False, stream=None):
    """The fused pass with no workspace and no device allocation inside the
    library: for callers that are handed only input and output buffers (a
    plugin whose host framework owns all device memory) or that must not call
    cudaMalloc on a latency-critical path.  The intermediates live in a
    64 MiB scratch array inside the library, shared by every call on the
    device, so calls must not overlap on the GPU; larger problems raise
    LshError(LSH_ERR_WORKSPACE).  (This Python wrapper still allocates ``out``
    and ``lse`` with torch when they are not passed in.)"""
    B, H, L, d = _qk(qk)
    _cuda(v, "v", qk.dtype, qk.shape, qk)
    _rotations(rotations, qk, n_hashes, n_buckets, False)
    shp = _shape_of(qk, n_hashes, n_buckets, chunk_len, causal, portable)
    out, lse = _outputs(qk, out, lse)
    _check(lib().lsh_attn_forward_noalloc(ctypes.byref(shp), _ptr(qk), _ptr(v), _ptr(rotations),
                                          _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def lsh_attn_kernel_launches() -> int:
    """Kernels the library has launched in this process so far (host count)."""
    return int(lib().lsh_attn_kernel_launches())


def lsh_attn_device_check(stream=None):
    """Synchronise the stream and raise if a kernel's bounded wait ran out."""
    _check(lib().lsh_attn_device_check(_stream(stream)))


def lsh_attn_backward_workspace_size(shape: Shape) -> int:
    n = _SZ()
    _check(lib().lsh_attn_backward_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def lsh_attn_backward(qk, v, inv_norm, perm, out, lse, dout, chunk_len, causal, *,
                      n_buckets=2, workspace=None, stream=None):
    """Gradients of out w.r.t. qk and v with the buckets and sort held fixed.
    perm [B,H,n_h,L] and inv_norm from stages 1-2, out and lse from the
    forward.  Returns (dqk, dv), float32 [B,H,L,d]."""
    n_h = _stage3_args(qk, v, inv_norm, perm)
    B, H, L, d = qk.shape
    _cuda(out, "out", qk.dtype, qk.shape, qk)
    _cuda(lse, "lse", torch.float32, (B, H, L), qk)
    _cuda(dout, "dout", qk.dtype, qk.shape, qk)
    shp = _shape_of(qk, n_h, n_buckets, chunk_len, causal, False)
    need = lsh_attn_backward_workspace_size(shp)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=qk.device)
    _cuda(workspace, "workspace", None, None, qk)
    dqk = torch.empty(qk.shape, dtype=torch.float32, device=qk.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=qk.device)
    _check(lib().lsh_attn_backward(ctypes.byref(shp), _ptr(qk), _ptr(v), _ptr(inv_norm),
                                   _ptr(perm), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dqk),
                                   _ptr(dv), _ptr(workspace), _SZ(workspace.numel()),
                                   _stream(stream)))
    return dqk, dv
