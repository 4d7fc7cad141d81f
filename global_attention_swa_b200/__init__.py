"""Python binding of the MiMo-V2-Flash hybrid attention library (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libmimo_attn.so`` (C ABI in ``include/mimo_attn.h``).  PyTorch is
used for device memory and the current stream.  There is no fallback: if the
library cannot be loaded, importing this package raises.

Entry points (same names as the C ABI):

* ``mimo_attn_prefill(q, k, v, sinks, window, cu_seqlens, max_seqlen, ...)``
* ``mimo_attn_decode(q, k_cache, v_cache, seqlens, window, sinks, ...)``
* ``mimo_attn_decode_workspace_size(...)``, ``mimo_attn_device_status(...)``
"""

from __future__ import annotations

import contextlib
import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
#: MIMO_ATTN_CHECKED=1 in the environment loads the bounds-checked build
#: (libmimo_attn_checked.so: every kernel checks its row indices, see the header)
CHECKED = os.environ.get("MIMO_ATTN_CHECKED", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libmimo_attn_checked.so" if CHECKED else "libmimo_attn.so")

MIMO_OK = 0
MIMO_ERR_INVALID_ARG = 1
MIMO_ERR_UNSUPPORTED = 2
MIMO_ERR_CUDA = 3
MIMO_ERR_WORKSPACE = 4
MIMO_ERR_TIMEOUT = 5
MIMO_ERR_BOUNDS = 6
MIMO_DTYPE_BF16 = 0
MIMO_DTYPE_F32 = 1

#: entry points declared in include/mimo_attn.h
EXPORTED = (
    "mimo_attn_prefill",
    "mimo_attn_decode_workspace_size",
    "mimo_attn_decode",
    "mimo_attn_last_error",
    "mimo_attn_device_status",
    "mimo_attn_set_device_status",
    "mimo_attn_decode_noalloc",
    "mimo_attn_decode_fp8_workspace_size",
    "mimo_attn_decode_fp8",
    "mimo_attn_rope_append",
    "mimo_attn_decode_merge",
    "mimo_attn_prefill_backward_workspace_size",
    "mimo_attn_prefill_backward",
    "mimo_attn_wait_selftest",
    "mimo_attn_is_checked_build",
    "mimo_attn_checked_site",
    "mimo_attn_checked_selftest",
)


class MimoAttnError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"mimo_attn status {status}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [
        ("num_heads_q", ctypes.c_int),
        ("num_heads_kv", ctypes.c_int),
        ("head_dim_qk", ctypes.c_int),
        ("head_dim_v", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
        ("v_scale", ctypes.c_float),
        ("out_dtype", ctypes.c_int),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with global_attention_swa_b200._build.build("
            f"{'checked=True' if CHECKED else ''})")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    dp = ctypes.POINTER(Dims)
    lib.mimo_attn_prefill.argtypes = [dp, vp, vp, vp, vp, i32, vp, i32, i32, i32, vp, vp, vp]
    lib.mimo_attn_prefill.restype = i32
    lib.mimo_attn_decode_workspace_size.argtypes = [dp, i32, i32, i32]
    lib.mimo_attn_decode_workspace_size.restype = sz
    lib.mimo_attn_decode.argtypes = [dp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, sz, vp]
    lib.mimo_attn_decode.restype = i32
    lib.mimo_attn_last_error.argtypes = []
    lib.mimo_attn_last_error.restype = ctypes.c_char_p
    lib.mimo_attn_device_status.argtypes = [vp]
    lib.mimo_attn_device_status.restype = i32
    lib.mimo_attn_set_device_status.argtypes = [i32, vp]
    lib.mimo_attn_set_device_status.restype = i32
    lib.mimo_attn_decode_fp8_workspace_size.argtypes = [dp, i32, i32, i32]
    lib.mimo_attn_decode_fp8_workspace_size.restype = sz
    lib.mimo_attn_decode_fp8.argtypes = [dp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp,
                                         sz, vp]
    lib.mimo_attn_decode_fp8.restype = i32
    lib.mimo_attn_rope_append.argtypes = [dp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                          ctypes.c_float, i32, vp]
    lib.mimo_attn_rope_append.restype = i32
    lib.mimo_attn_decode_merge.argtypes = [dp, vp, vp, i32, i32, vp, vp, vp, vp]
    lib.mimo_attn_decode_merge.restype = i32
    lib.mimo_attn_prefill_backward_workspace_size.argtypes = [dp, i32]
    lib.mimo_attn_prefill_backward_workspace_size.restype = sz
    lib.mimo_attn_prefill_backward.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32,
                                               vp, vp, vp, vp, vp, sz, vp]
    lib.mimo_attn_prefill_backward.restype = i32
    lib.mimo_attn_wait_selftest.argtypes = [vp]
    lib.mimo_attn_wait_selftest.restype = i32
    lib.mimo_attn_is_checked_build.argtypes = []
    lib.mimo_attn_is_checked_build.restype = i32
    lib.mimo_attn_checked_site.argtypes = [vp]
    lib.mimo_attn_checked_site.restype = i32
    lib.mimo_attn_checked_selftest.argtypes = [vp]
    lib.mimo_attn_checked_selftest.restype = i32
    return lib


lib = _load()

if hasattr(lib, "mimo_attn_decode_noalloc"):
    lib.mimo_attn_decode_noalloc.argtypes = [ctypes.POINTER(Dims)] + [ctypes.c_void_p] * 4 + [
        ctypes.c_int, ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 4
    lib.mimo_attn_decode_noalloc.restype = ctypes.c_int


def _check(status):
    if status != MIMO_OK:
        raise MimoAttnError(status, lib.mimo_attn_last_error().decode())


_BF16, _F32, _I32 = torch.bfloat16, torch.float32, torch.int32
_OUT = (torch.bfloat16, torch.float32)


def _ptr(t, name="tensor", dtype=None):
    """Device address of a contiguous CUDA tensor (None for None).  The C ABI takes
    plain pointers, so a host tensor, a strided view or another dtype would be
    read as garbage: each is refused here."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    return ctypes.c_void_p(t.data_ptr())


def _shape(t, shape, name):
    """Refuse a tensor whose shape disagrees with the sizes the call derives from
    its other arguments (the library would read or write past its end)."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _same_device(dev, **tensors):
    """Refuse tensors that live on another device than the call's (the library
    launches on the current device and would dereference another GPU's memory)."""
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, but the call runs on {dev}")


@contextlib.contextmanager
def _on_device(dev):
    """Make the tensors' device current for the call (launches, device queries)."""
    if dev.type == "cuda":
        with torch.cuda.device(dev):
            yield
    else:  # host tensors never reach the library: _ptr refuses them
        yield


def _stream(stream, dev):
    """The stream to launch on: the caller's (which must belong to dev) or dev's
    current stream."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif stream.device != dev:
        raise ValueError(f"stream belongs to {stream.device}, but the call runs on {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def make_dims(hq, hkv, dqk=192, dv=128, softmax_scale=None, v_scale=1.0, out_dtype=torch.bfloat16):
    return Dims(hq, hkv, dqk, dv,
                0.0 if softmax_scale is None else float(softmax_scale),
                float(v_scale),
                MIMO_DTYPE_F32 if out_dtype == torch.float32 else MIMO_DTYPE_BF16)


def mimo_attn_prefill(q, k, v, sinks, window, cu_seqlens, max_seqlen, out=None, lse=None,
                      out_dtype=torch.bfloat16, softmax_scale=None, v_scale=1.0,
                      return_lse=True, stream=None):
    """Packed varlen prefill.  q [Nt,Hq,192], k [Nt,Hkv,192], v [Nt,Hkv,128] bf16 (CUDA).

    Returns (out [Nt,Hq,128], lse [Hq,Nt] fp32 or None).
    """
    nt, hq, dqk = q.shape
    hkv, dv = k.shape[1], v.shape[2]
    _shape(k, (nt, hkv, dqk), "k")
    _shape(v, (nt, hkv, dv), "v")
    _shape(sinks, (hq,), "sinks")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be 1-D with num_seqs + 1 entries")
    _shape(out, (nt, hq, dv), "out")
    _shape(lse, (hq, nt), "lse")
    if out is None:
        out = torch.empty((nt, hq, dv), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((hq, nt), dtype=torch.float32, device=q.device)
    dev = q.device
    _same_device(dev, k=k, v=v, sinks=sinks, cu_seqlens=cu_seqlens, out=out, lse=lse)
    dims = make_dims(hq, hkv, dqk, dv, softmax_scale, v_scale, out.dtype)
    with _on_device(dev):
        _check(lib.mimo_attn_prefill(ctypes.byref(dims), _ptr(q, "q", _BF16), _ptr(k, "k", _BF16),
                                     _ptr(v, "v", _BF16), _ptr(sinks, "sinks", _F32), int(window),
                                     _ptr(cu_seqlens, "cu_seqlens", _I32), int(cu_seqlens.numel() - 1),
                                     nt, int(max_seqlen), _ptr(out, "out", _OUT),
                                     _ptr(lse, "lse", _F32), _stream(stream, dev)))
    return out, lse


def _decode_shapes(q, k_cache, v_cache, seqlens, sinks, out, lse):
    B, hq, dqk = q.shape
    if k_cache.dim() != 4 or v_cache.dim() != 4:
        raise ValueError("caches must be [batch, capacity, Hkv, D]")
    C, hkv = k_cache.shape[1], k_cache.shape[2]
    _shape(k_cache, (B, C, hkv, dqk), "k_cache")
    _shape(v_cache, (B, C, hkv, v_cache.shape[3]), "v_cache")
    _shape(seqlens, (B,), "seqlens")
    _shape(sinks, (hq,), "sinks")
    _shape(out, (B, hq, v_cache.shape[3]), "out")
    _shape(lse, (B, hq), "lse")


def mimo_attn_decode_workspace_size(hq, hkv, batch, capacity, window, dqk=192, dv=128):
    dims = make_dims(hq, hkv, dqk, dv)
    return int(lib.mimo_attn_decode_workspace_size(ctypes.byref(dims), batch, capacity, window))


def mimo_attn_decode(q, k_cache, v_cache, seqlens, window, sinks, out=None, lse=None,
                     workspace=None, out_dtype=torch.bfloat16, softmax_scale=None, v_scale=1.0,
                     return_lse=True, stream=None):
    """One decode step.  q [B,Hq,192]; caches [B,C,Hkv,192/128] bf16; seqlens [B] int32.

    Returns (out [B,Hq,128], lse [B,Hq] fp32 or None).
    """
    B, hq, dqk = q.shape
    C, hkv = k_cache.shape[1], k_cache.shape[2]
    dv = v_cache.shape[3]
    _decode_shapes(q, k_cache, v_cache, seqlens, sinks, out, lse)
    if out is None:
        out = torch.empty((B, hq, dv), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    dev = q.device
    dims = make_dims(hq, hkv, dqk, dv, softmax_scale, v_scale, out.dtype)
    need = int(lib.mimo_attn_decode_workspace_size(ctypes.byref(dims), B, C, int(window)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _same_device(dev, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens, sinks=sinks, out=out,
                 lse=lse, workspace=workspace)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on_device(dev):
        _check(lib.mimo_attn_decode(ctypes.byref(dims), _ptr(q, "q", _BF16),
                                    _ptr(k_cache, "k_cache", _BF16), _ptr(v_cache, "v_cache", _BF16),
                                    _ptr(seqlens, "seqlens", _I32), B, C, int(window),
                                    _ptr(sinks, "sinks", _F32), _ptr(out, "out", _OUT),
                                    _ptr(lse, "lse", _F32), _ptr(workspace, "workspace"), wbytes,
                                    _stream(stream, dev)))
    return out, lse


def mimo_attn_decode_fp8(q, k_cache, v_cache, k_scale, v_scale_kv, seqlens, window, sinks,
                         out=None, lse=None, workspace=None, out_dtype=torch.bfloat16,
                         softmax_scale=None, v_scale=1.0, return_lse=True, stream=None):
    """One decode step against e4m3 caches.  q [B,Hq,192] bf16; caches [B,C,Hkv,192/128]
    as torch.float8_e4m3fn or uint8 codes; k_scale / v_scale_kv [Hkv] fp32.

    Returns (out [B,Hq,128], lse [B,Hq] fp32 or None).
    """
    B, hq, dqk = q.shape
    C, hkv = k_cache.shape[1], k_cache.shape[2]
    dv = v_cache.shape[3]
    if k_cache.element_size() != 1 or v_cache.element_size() != 1:
        raise TypeError("FP8 caches hold one byte per element")
    _decode_shapes(q, k_cache, v_cache, seqlens, sinks, out, lse)
    _shape(k_scale, (hkv,), "k_scale")
    _shape(v_scale_kv, (hkv,), "v_scale_kv")
    if out is None:
        out = torch.empty((B, hq, dv), dtype=out_dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    dev = q.device
    dims = make_dims(hq, hkv, dqk, dv, softmax_scale, v_scale, out.dtype)
    need = int(lib.mimo_attn_decode_fp8_workspace_size(ctypes.byref(dims), B, C, int(window)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _same_device(dev, k_cache=k_cache, v_cache=v_cache, k_scale=k_scale, v_scale_kv=v_scale_kv,
                 seqlens=seqlens, sinks=sinks, out=out, lse=lse, workspace=workspace)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on_device(dev):
        _check(lib.mimo_attn_decode_fp8(ctypes.byref(dims), _ptr(q, "q", _BF16),
                                        _ptr(k_cache, "k_cache"), _ptr(v_cache, "v_cache"),
                                        _ptr(k_scale, "k_scale", _F32),
                                        _ptr(v_scale_kv, "v_scale_kv", _F32),
                                        _ptr(seqlens, "seqlens", _I32), B, C, int(window),
                                        _ptr(sinks, "sinks", _F32), _ptr(out, "out", _OUT),
                                        _ptr(lse, "lse", _F32), _ptr(workspace, "workspace"), wbytes,
                                        _stream(stream, dev)))
    return out, lse


def mimo_attn_rope_append(q, k_new, v_new, k_cache, v_cache, seqlens, window, rope_theta,
                          rotary_dim=None, stream=None):
    """Rotate the new token's q (in place) and k, and write k, v into the cache slot of
    position seqlens - 1 (see include/mimo_attn.h).  Returns q."""
    B, hq, dqk = q.shape
    C, hkv = k_cache.shape[1], k_cache.shape[2]
    _decode_shapes(q, k_cache, v_cache, seqlens, None, None, None)
    _shape(k_new, (B, hkv, dqk), "k_new")
    _shape(v_new, (B, hkv, v_cache.shape[3]), "v_new")
    dev = q.device
    _same_device(dev, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens)
    dims = make_dims(hq, hkv, dqk, v_cache.shape[3])
    rd = dqk if rotary_dim is None else int(rotary_dim)
    with _on_device(dev):
        _check(lib.mimo_attn_rope_append(ctypes.byref(dims), _ptr(q, "q", _BF16),
                                         _ptr(k_new, "k_new", _BF16), _ptr(v_new, "v_new", _BF16),
                                         _ptr(k_cache, "k_cache", _BF16),
                                         _ptr(v_cache, "v_cache", _BF16),
                                         _ptr(seqlens, "seqlens", _I32), B, C, int(window),
                                         float(rope_theta), rd, _stream(stream, dev)))
    return q


def mimo_attn_decode_merge(part_out, part_lse, sinks, out=None, lse=None,
                           out_dtype=torch.bfloat16, v_scale=1.0, return_lse=True, stream=None):
    """Merge per-part decode results (part_out [R,B,Hq,128] fp32, part_lse [R,B,Hq] fp32)
    with the sink.  Returns (out [B,Hq,128], lse [B,Hq] or None)."""
    R, B, hq, dv = part_out.shape
    _shape(part_lse, (R, B, hq), "part_lse")
    _shape(sinks, (hq,), "sinks")
    _shape(out, (B, hq, dv), "out")
    _shape(lse, (B, hq), "lse")
    if out is None:
        out = torch.empty((B, hq, dv), dtype=out_dtype, device=part_out.device)
    if lse is None and return_lse:
        lse = torch.empty((B, hq), dtype=torch.float32, device=part_out.device)
    dev = part_out.device
    _same_device(dev, part_lse=part_lse, sinks=sinks, out=out, lse=lse)
    dims = make_dims(hq, 1, 192, dv, None, v_scale, out.dtype)
    with _on_device(dev):
        _check(lib.mimo_attn_decode_merge(ctypes.byref(dims), _ptr(part_out, "part_out", _F32),
                                          _ptr(part_lse, "part_lse", _F32), R, B,
                                          _ptr(sinks, "sinks", _F32), _ptr(out, "out", _OUT),
                                          _ptr(lse, "lse", _F32), _stream(stream, dev)))
    return out, lse


def mimo_attn_prefill_backward(q, k, v, out, lse, dout, sinks, window, cu_seqlens, max_seqlen,
                               softmax_scale=None, v_scale=1.0, stream=None):
    """Gradients of mimo_attn_prefill: returns (dq, dk, dv [fp32], dsinks [Hq] fp32 or None).

    ``out`` and ``lse`` are the forward's results; ``dout`` has out's dtype.
    """
    nt, hq, dqk = q.shape
    hkv, dv_dim = k.shape[1], v.shape[2]
    _shape(k, (nt, hkv, dqk), "k")
    _shape(v, (nt, hkv, dv_dim), "v")
    _shape(out, (nt, hq, dv_dim), "out")
    _shape(lse, (hq, nt), "lse")
    _shape(dout, (nt, hq, dv_dim), "dout")
    _shape(sinks, (hq,), "sinks")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be 1-D with num_seqs + 1 entries")
    dq = torch.empty((nt, hq, dqk), dtype=torch.float32, device=q.device)
    dk = torch.empty((nt, hkv, dqk), dtype=torch.float32, device=q.device)
    dv = torch.empty((nt, hkv, dv_dim), dtype=torch.float32, device=q.device)
    ds = None if sinks is None else torch.empty(hq, dtype=torch.float32, device=q.device)
    dev = q.device
    _same_device(dev, k=k, v=v, out=out, lse=lse, dout=dout, sinks=sinks, cu_seqlens=cu_seqlens)
    dims = make_dims(hq, hkv, dqk, dv_dim, softmax_scale, v_scale, out.dtype)
    need = int(lib.mimo_attn_prefill_backward_workspace_size(ctypes.byref(dims), nt))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    with _on_device(dev):
        _check(lib.mimo_attn_prefill_backward(ctypes.byref(dims), _ptr(q, "q", _BF16),
                                              _ptr(k, "k", _BF16), _ptr(v, "v", _BF16),
                                              _ptr(out, "out", _OUT), _ptr(lse, "lse", _F32),
                                              _ptr(dout, "dout", out.dtype),
                                              _ptr(sinks, "sinks", _F32), int(window),
                                              _ptr(cu_seqlens, "cu_seqlens", _I32),
                                              cu_seqlens.numel() - 1, nt, int(max_seqlen), _ptr(dq),
                                              _ptr(dk), _ptr(dv), _ptr(ds), _ptr(ws), ws.numel(),
                                              _stream(stream, dev)))
    return dq, dk, dv, ds


def _current_device():
    return torch.device("cuda", torch.cuda.current_device())


def mimo_attn_device_status(stream=None, device=None):
    """Synchronise the stream (default: the current stream of ``device``, itself
    defaulting to the current device); raise if a kernel recorded a device-side
    error on that device."""
    dev = torch.device(device) if device is not None else (
        stream.device if stream is not None else _current_device())
    with _on_device(dev):
        _check(lib.mimo_attn_device_status(_stream(stream, dev)))


def mimo_attn_set_device_status(code, stream=None, device=None):
    """Pre-load the device status word (test hook for the failure path; see
    include/mimo_attn.h)."""
    dev = torch.device(device) if device is not None else (
        stream.device if stream is not None else _current_device())
    with _on_device(dev):
        _check(lib.mimo_attn_set_device_status(int(code), _stream(stream, dev)))


def mimo_attn_wait_selftest(stream=None, device=None):
    """Failure-path test hook: a kernel whose wait runs out after its bound
    (about 1 s) and records MIMO_ERR_TIMEOUT (see include/mimo_attn.h)."""
    dev = torch.device(device) if device is not None else (
        stream.device if stream is not None else _current_device())
    with _on_device(dev):
        _check(lib.mimo_attn_wait_selftest(_stream(stream, dev)))


def mimo_attn_is_checked_build():
    """True when the loaded library is the bounds-checked build."""
    return bool(lib.mimo_attn_is_checked_build())


def mimo_attn_checked_site(stream=None, device=None):
    """Synchronise the stream; return (and clear) the first site at which the
    checked build caught a row index outside its buffer, 0 if none; raise if a
    CUDA call failed."""
    dev = torch.device(device) if device is not None else (
        stream.device if stream is not None else _current_device())
    with _on_device(dev):
        site = int(lib.mimo_attn_checked_site(_stream(stream, dev)))
    if site < 0:
        raise MimoAttnError(MIMO_ERR_CUDA, lib.mimo_attn_last_error().decode())
    return site


def mimo_attn_checked_selftest(stream=None, device=None):
    """Checked build only: launch the one-thread kernel whose row check fails
    without touching memory (see include/mimo_attn.h)."""
    dev = torch.device(device) if device is not None else (
        stream.device if stream is not None else _current_device())
    with _on_device(dev):
        _check(lib.mimo_attn_checked_selftest(_stream(stream, dev)))


def default_scale(dqk=192):
    return 1.0 / math.sqrt(dqk)


def mimo_attn_decode_noalloc(q, k_cache, v_cache, seqlens, window, sinks, out, lse=None,
                             softmax_scale=None, v_scale=1.0, stream=None):
    """Decode through the entry point that allocates nothing (see include/mimo_attn.h).

    The caller passes preallocated ``out`` [B,Hq,128] and optional ``lse`` [B,Hq].
    """
    B, hq, dqk = q.shape
    C, hkv = k_cache.shape[1], k_cache.shape[2]
    _decode_shapes(q, k_cache, v_cache, seqlens, sinks, out, lse)
    dev = q.device
    _same_device(dev, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens, sinks=sinks, out=out,
                 lse=lse)
    dims = make_dims(hq, hkv, dqk, v_cache.shape[3], softmax_scale, v_scale, out.dtype)
    with _on_device(dev):
        _check(lib.mimo_attn_decode_noalloc(ctypes.byref(dims), _ptr(q, "q", _BF16),
                                            _ptr(k_cache, "k_cache", _BF16),
                                            _ptr(v_cache, "v_cache", _BF16),
                                            _ptr(seqlens, "seqlens", _I32), B, C, int(window),
                                            _ptr(sinks, "sinks", _F32), _ptr(out, "out", _OUT),
                                            _ptr(lse, "lse", _F32), _stream(stream, dev)))
    return out, lse
