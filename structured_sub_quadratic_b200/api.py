"""Python binding of the MonarchAttention C ABI (``include/monarch_attn.h``).

Argument marshalling only: torch tensors are passed to the library as raw
device pointers plus sizes, on the caller's current CUDA stream.  Every step
of the forward pass runs in the library's CUDA kernels; there is no fallback,
and a missing library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from ._build import LIB_PATH

MONARCH_OK = 0
MONARCH_ERR_INVALID_ARG = -1
MONARCH_ERR_UNSUPPORTED = -2
MONARCH_ERR_CUDA = -3
MONARCH_ERR_DEVICE_TIMEOUT = -4
MONARCH_ERR_NO_MEMORY = -5
MONARCH_ERR_SCRATCH_LIMIT = -6
DTYPE_BF16 = 0
DTYPE_F32 = 1
LAYOUTS = {"fh,w": 0, "w,fh": 1, "f,hw": 2, "hw,f": 3, "fw,h": 4, "h,fw": 5}

# Every symbol the header declares, with its ctypes signature.
_I, _P, _Z = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
_SIZES = [_I] * 8  # B, H, b1, b2, d, T, c1, c2
SIGNATURES = {
    "monarch_attn_fwd": (_I, [_P, _P, _P, _P, *_SIZES, _P]),
    "monarch_attn_fwd_f32": (_I, [_P, _P, _P, _P, *_SIZES, _P]),
    "monarch_attn_fwd_host": (_I, [_I, _P, _P, _P, _P, *_SIZES, _P]),
    "monarch_attn_fwd_noalloc": (_I, [_P, _P, _P, _P, *_SIZES, _P]),
    "monarch_attn_fwd_video": (_I, [_I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                    _I, _P]),
    "monarch_attn_fwd_padded": (_I, [_I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                     _I, _P]),
    "monarch_attn_bwd": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, *_SIZES, _P]),
    "monarch_attn_workspace_bytes": (_Z, [*_SIZES, _I]),
    "monarch_attn_release_workspace": (None, []),
    "monarch_attn_check": (_I, [_P]),
    "monarch_attn_strerror": (ctypes.c_char_p, [_I]),
    "monarch_attn_last_launches": (_I, []),
    "monarch_attn_version": (_I, []),
    "monarch_attn_selftest_timeout": (_I, [ctypes.c_ulonglong, _P]),
    "monarch_attn_timing_enable": (_I, [_I]),
    "monarch_attn_timing_read": (_I, [_I, ctypes.c_char_p, _I,
                                      ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_long)]),
}


class MonarchError(RuntimeError):
    def __init__(self, status: int, text: str):
        super().__init__(f"monarch_attn status {status}: {text}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the shared library and bind every declared symbol (raises if absent)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m structured_sub_quadratic_b200._build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int):
    if status != MONARCH_OK:
        raise MonarchError(status, load_library().monarch_attn_strerror(status).decode())


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dims(q, b1, b2):
    if q.dim() != 4:
        raise ValueError("expected (B, H, N, d) tensors")
    B, H, N, d = q.shape
    if N != b1 * b2:
        raise ValueError(f"N={N} != b1*b2={b1 * b2}")
    return B, H, d


def monarch_attn_fwd(q, k, v, b1, b2, T, c1=1, c2=1, out=None, stream=None):
    """MonarchAttention forward on device tensors (B, H, N, d), N = b1*b2.

    bf16 tensors go to ``monarch_attn_fwd`` and fp32 to
    ``monarch_attn_fwd_f32``.  Returns ``out`` (allocated if not given).
    """
    lib = load_library()
    B, H, d = _dims(q, b1, b2)
    for t in (q, k, v):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    if out is None:
        out = torch.empty_like(q)
    if q.dtype == torch.bfloat16:
        fn = lib.monarch_attn_fwd
    elif q.dtype == torch.float32:
        fn = lib.monarch_attn_fwd_f32
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _check(fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
              B, H, b1, b2, d, T, c1, c2, _stream_ptr(stream)))
    return out


def monarch_attn_fwd_noalloc(q, k, v, b1, b2, T, c1=1, c2=1, out=None, stream=None):
    """bf16 forward pass that allocates no device memory inside the library.

    For callers that cannot allocate when they call (a real-time frame loop
    that must not stall on cudaMalloc/cudaFree, or a host that reserves all
    device memory for its own pool).  It runs the kernels of
    ``monarch_attn_fwd`` and returns bit-identical results.  Scratch is a
    static 64 MiB device array shared by all calls on a device, committed at
    the first call on that device (make it at initialisation); calls that
    overlap on the GPU race on it, so keep them on one stream.  Pass ``out``
    to avoid the one allocation this wrapper would otherwise make through
    torch.
    """
    lib = load_library()
    B, H, d = _dims(q, b1, b2)
    for t in (q, k, v):
        if t.shape != q.shape or t.dtype != torch.bfloat16 or not t.is_cuda \
                or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors of one shape")
    if out is None:
        out = torch.empty_like(q)
    _check(lib.monarch_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        out.data_ptr(), B, H, b1, b2, d, T, c1, c2,
                                        _stream_ptr(stream)))
    return out


def monarch_attn_fwd_padded(q, k, v, b1, b2, T, c1=1, c2=1, pad_front=True, out=None,
                            stream=None):
    """Forward pass on (B, H, n_real, d) tensors with n_real <= b1*b2: the
    sequence is padded to the b1*b2 grid with the pad tokens before the real
    ones (``pad_front``, pre-padding) or after them; the objective covers the
    real tokens only.  Returns ``out`` (B, H, n_real, d)."""
    lib = load_library()
    if q.dim() != 4:
        raise ValueError("expected (B, H, n_real, d) tensors")
    B, H, n_real, d = q.shape
    for t in (q, k, v):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(q.dtype)
    if dtype is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if out is None:
        out = torch.empty_like(q)
    _check(lib.monarch_attn_fwd_padded(dtype, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       out.data_ptr(), B, H, n_real, b1, b2,
                                       1 if pad_front else 0, d, T, c1, c2, _stream_ptr(stream)))
    return out


def monarch_attn_bwd(q, k, v, dout, b1, b2, T=1, c1=1, c2=1, stream=None):
    """Gradients (dq, dk, dv) of sum(O * dout) for the T = 1 forward pass on
    device tensors (B, H, N, d), N = b1*b2, bf16 or fp32."""
    lib = load_library()
    B, H, d = _dims(q, b1, b2)
    for t in (q, k, v, dout):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v, dout must be contiguous CUDA tensors of one shape and dtype")
    dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(q.dtype)
    if dtype is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    _check(lib.monarch_attn_bwd(dtype, q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, b1, b2, d, T,
                                c1, c2, _stream_ptr(stream)))
    return dq, dk, dv


def video_blocks(f, h, w, layout):
    """(b1, b2) of an aligned layout name such as "w,fh" (see LAYOUTS)."""
    size = {"f": f, "h": h, "w": w}
    rows, cols = layout.split(",")
    b1 = 1
    for a in rows:
        b1 *= size[a]
    b2 = 1
    for a in cols:
        b2 *= size[a]
    return b1, b2


def monarch_attn_fwd_video(q, k, v, f, h, w, layout, T, c1=1, c2=1, out=None, stream=None):
    """Forward pass on a video latent (B, H, f*h*w, d) in raster token order,
    with the Monarch blocks aligned to ``layout`` (a key of LAYOUTS)."""
    lib = load_library()
    if layout not in LAYOUTS:
        raise ValueError(f"unknown layout {layout!r}; expected one of {sorted(LAYOUTS)}")
    if q.dim() != 4 or q.shape[2] != f * h * w:
        raise ValueError("expected (B, H, f*h*w, d) tensors")
    B, H, _, d = q.shape
    for t in (q, k, v):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(q.dtype)
    if dtype is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if out is None:
        out = torch.empty_like(q)
    _check(lib.monarch_attn_fwd_video(dtype, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                      out.data_ptr(), B, H, f, h, w, LAYOUTS[layout], d, T, c1,
                                      c2, _stream_ptr(stream)))
    return out


def monarch_attn_fwd_host(q, k, v, out, b1, b2, T, c1=1, c2=1, stream=None):
    """Forward pass on HOST tensors (pinned for full bandwidth); synchronous."""
    lib = load_library()
    B, H, d = _dims(q, b1, b2)
    for t in (q, k, v, out):
        if t.is_cuda or not t.is_contiguous() or t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("host tensors must be contiguous CPU tensors of one shape and dtype")
    dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}[q.dtype]
    _check(lib.monarch_attn_fwd_host(dtype, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                     out.data_ptr(), B, H, b1, b2, d, T, c1, c2,
                                     _stream_ptr(stream)))
    return out


def workspace_bytes(B, H, b1, b2, d, T, c1=1, c2=1, dtype=torch.bfloat16):
    code = DTYPE_BF16 if dtype == torch.bfloat16 else DTYPE_F32
    return load_library().monarch_attn_workspace_bytes(B, H, b1, b2, d, T, c1, c2, code)


def release_workspace():
    load_library().monarch_attn_release_workspace()


def check(stream=None):
    _check(load_library().monarch_attn_check(_stream_ptr(stream)))


def last_launches() -> int:
    return load_library().monarch_attn_last_launches()


def timing_enable(enable: bool) -> bool:
    """Turn per-kernel CUDA-event timing on or off; returns the old setting."""
    return bool(load_library().monarch_attn_timing_enable(1 if enable else 0))


def timing_read(max_kernels: int = 32):
    """{kernel name: (total ms, launches)} since the previous read."""
    lib = load_library()
    name_len = 64
    names = ctypes.create_string_buffer(max_kernels * name_len)
    ms = (ctypes.c_double * max_kernels)()
    cnt = (ctypes.c_long * max_kernels)()
    n = lib.monarch_attn_timing_read(max_kernels, names, name_len, ms, cnt)
    if n < 0:
        _check(n)
    out = {}
    for s in range(min(n, max_kernels)):
        raw = names.raw[s * name_len:(s + 1) * name_len]
        out[raw.split(b"\0", 1)[0].decode()] = (ms[s], cnt[s])
    return out


def selftest_timeout(limit_ns: int, stream=None):
    """Launch the bounded-wait self-test (see the header); check() then reports it."""
    _check(load_library().monarch_attn_selftest_timeout(limit_ns, _stream_ptr(stream)))
