"""ctypes binding over the C ABI in ``include/monarch_attn.h``.

Argument marshalling only: every step of the operator runs in the CUDA
library.  Tensors are PyTorch tensors purely as device memory; the stream is
PyTorch's current stream unless one is given.  There is no fallback: if the
library is missing or the call fails, this raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

FACT_FRAME = 0
FACT_TILED = 1
FACT_ROW = 2
DTYPE_F32 = 0
DTYPE_BF16 = 1
DTYPE_F16 = 2

STATUS_NAMES = {0: "MONARCH_OK", 1: "MONARCH_ERR_INVALID_ARG", 2: "MONARCH_ERR_UNSUPPORTED",
                3: "MONARCH_ERR_LAUNCH", 4: "MONARCH_ERR_TIMEOUT", 5: "MONARCH_ERR_CUDA"}

_lib = None


class MonarchError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({strerror(status)})")


def lib_path() -> str:
    return _build.LIB


def load_library(path: str | None = None):
    """Load libmonarch_attn.so (built in-tree by ``build.build()``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or _build.LIB
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.monarch_attn_fwd.argtypes = [vp, vp, vp, vp] + [i] * 10 + [vp]
    lib.monarch_attn_fwd.restype = i
    lib.monarch_attn_fwd_profiled.argtypes = ([vp, vp, vp, vp] + [i] * 10 +
                                              [vp, ctypes.POINTER(vp), i, ctypes.POINTER(i)])
    lib.monarch_attn_fwd_profiled.restype = i
    lib.monarch_attn_fwd_host.argtypes = [vp] * 8 + [i] * 10 + [vp]
    lib.monarch_attn_fwd_host_pipelined.argtypes = [vp] * 8 + [i] * 11 + [vp]
    lib.monarch_attn_fwd_host_pipelined.restype = i
    lib.monarch_attn_fwd_host.restype = i
    lib.monarch_attn_strerror.argtypes = [i]
    lib.monarch_attn_strerror.restype = ctypes.c_char_p
    lib.monarch_attn_device_status.argtypes = [vp, i]
    lib.monarch_attn_device_status.restype = i
    lib.monarch_attn_selftest_timeout.argtypes = [ctypes.c_longlong, vp]
    lib.monarch_attn_selftest_timeout.restype = i
    ll = ctypes.c_longlong
    sz = ctypes.c_size_t
    lib.monarch_attn_bwd.argtypes = [vp] * 8 + [sz] + [i] * 10 + [vp]
    lib.monarch_attn_bwd.restype = i
    lib.monarch_attn_bwd_profiled.argtypes = ([vp] * 8 + [sz] + [i] * 10 + [vp] +
                                              [ctypes.POINTER(vp), i, ctypes.POINTER(i)])
    lib.monarch_attn_bwd_profiled.restype = i
    lib.monarch_attn_bwd_workspace_size.argtypes = [i] * 7
    lib.monarch_attn_bwd_workspace_size.restype = sz
    lib.monarch_attn_fwd_strided.argtypes = [vp, vp, vp, vp] + [i] * 10 + [ll, ll, ll, vp]
    lib.monarch_attn_fwd_strided.restype = i
    lib.monarch_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp] + [i] * 9 + [vp]
    lib.monarch_attn_fwd_noalloc.restype = i
    lib.monarch_attn_fwd_chunk.argtypes = [vp] * 7 + [i] * 11 + [vp]
    lib.monarch_attn_fwd_chunk.restype = i
    lib.monarch_attn_fwd_chunk_profiled.argtypes = ([vp] * 7 + [i] * 11 +
                                                    [vp, ctypes.POINTER(vp), i, ctypes.POINTER(i)])
    lib.monarch_attn_fwd_chunk_profiled.restype = i
    lib.monarch_attn_version.argtypes = []
    lib.monarch_attn_version.restype = i
    if path == _build.LIB:
        _lib = lib
    return lib


def monarch_attn_strerror(status: int) -> str:
    """Text of a library status code."""
    return load_library().monarch_attn_strerror(int(status)).decode()


def monarch_attn_version() -> int:
    """Library version number."""
    return int(load_library().monarch_attn_version())


strerror = monarch_attn_strerror


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float16:
        return DTYPE_F16
    if t.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16, float16 or float32")


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def monarch_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, T: int, H: int, W: int,
                     factorisation: int = FACT_FRAME, tile_h: int = 0, tile_w: int = 0,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out = P^T B2 P B1 V for q, k, v of shape [B, heads, T*H*W, d] on a CUDA device.

    Queued on ``stream`` (default: PyTorch's current stream); returns ``out``.
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, heads, N, d]")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, heads, N, d] shape")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype")
    B, heads, N, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous() or not out.is_cuda:
        raise ValueError("out must be a contiguous CUDA tensor shaped and typed like q")
    if N != T * H * W:
        raise ValueError(f"N={N} does not equal T*H*W={T * H * W}")
    st = load_library().monarch_attn_fwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, heads, T, H, W, d,
        int(factorisation), int(tile_h), int(tile_w), _dtype_code(q), _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd")
    return out


def monarch_attn_fwd_strided(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                             T: int, H: int, W: int, factorisation: int = FACT_FRAME, tile_h: int = 0,
                             tile_w: int = 0, stream=None) -> torch.Tensor:
    """monarch_attn_fwd on [B, heads, N, d] views with any batch/head/token
    strides (feature stride 1), e.g. ``x.permute(0, 2, 1, 3)`` of a [B, N, heads, d]
    tensor.  q, k, v and out must share one shape, dtype and stride set.
    """
    ts = (q, k, v, out)
    if not all(t.is_cuda for t in ts):
        raise ValueError("q, k, v, out must be CUDA tensors")
    if q.dim() != 4 or any(t.shape != q.shape or t.dtype != q.dtype for t in ts):
        raise ValueError("q, k, v, out must share one [B, heads, N, d] shape and dtype")
    if any(t.stride() != q.stride() for t in ts) or q.stride(3) != 1:
        raise ValueError("q, k, v, out must share strides, with unit feature stride")
    B, heads, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"N={N} does not equal T*H*W={T * H * W}")
    sb, sh, sn, _ = q.stride()
    st = load_library().monarch_attn_fwd_strided(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, heads, T, H, W, d,
        int(factorisation), int(tile_h), int(tile_w), _dtype_code(q), sb, sh, sn, _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_strided")
    return out


def monarch_attn_bwd_workspace_size(B: int, heads: int, T: int, H: int, W: int, d: int, dtype: int) -> int:
    """Workspace bytes monarch_attn_bwd needs for these sizes and dtype code (0 if unsupported)."""
    return int(load_library().monarch_attn_bwd_workspace_size(B, heads, T, H, W, d, int(dtype)))


def monarch_attn_bwd_workspace(q, T: int, H: int, W: int) -> torch.Tensor:
    """A workspace for monarch_attn_bwd on tensors shaped and typed like q."""
    B, heads, N, d = q.shape
    need = monarch_attn_bwd_workspace_size(B, heads, T, H, W, d, _dtype_code(q))
    return torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)


def monarch_attn_bwd(q, k, v, dout, T: int, H: int, W: int, factorisation: int = FACT_FRAME,
                     tile_h: int = 0, tile_w: int = 0, stream=None, out=None, workspace=None):
    """Gradients (dq, dk, dv) of monarch_attn_fwd for an upstream gradient dout;
    [B, heads, N, d] contiguous CUDA tensors of one dtype (bf16 and fp16 on
    tensor cores, fp32 on CUDA cores).  ``out`` = (dq, dk, dv) and
    ``workspace`` (monarch_attn_bwd_workspace) may be given to reuse buffers;
    otherwise they are allocated here with PyTorch.  Every step runs in the
    library's kernels.
    """
    ts = (q, k, v, dout)
    if not all(t.is_cuda and t.is_contiguous() for t in ts):
        raise ValueError("q, k, v, dout must be contiguous CUDA tensors")
    if q.dim() != 4 or any(t.shape != q.shape or t.dtype != q.dtype for t in ts):
        raise ValueError("q, k, v, dout must share one [B, heads, N, d] shape and dtype")
    B, heads, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"N={N} does not equal T*H*W={T * H * W}")
    if any(t.device != q.device for t in ts):
        raise ValueError("q, k, v, dout must be on one device")
    lib = load_library()
    code = _dtype_code(q)
    if workspace is None:
        ws = monarch_attn_bwd_workspace(q, T, H, W)
    else:
        ws = workspace
        if not (ws.is_cuda and ws.device == q.device and ws.is_contiguous()):
            raise ValueError("workspace must be a contiguous CUDA tensor on q's device")
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    else:
        dq, dk, dv = out
        if any(t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous() or not t.is_cuda
               or t.device != q.device for t in (dq, dk, dv)):
            raise ValueError("out must be three contiguous CUDA tensors on q's device, shaped and typed like q")
    ws_bytes = ws.numel() * ws.element_size()
    st = lib.monarch_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                              dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws_bytes, B, heads, T, H, W,
                              d, int(factorisation), int(tile_h), int(tile_w), code, _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_bwd")
    return dq, dk, dv


def monarch_attn_fwd_chunk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, k_cache, y1_cache,
                           T_old: int, T_new: int, H: int, W: int, factorisation: int = FACT_FRAME,
                           tile_h: int = 0, tile_w: int = 0, out=None, y1_new=None, stream=None):
    """One autoregressive chunk: the forward of T_new new frames (q, k, v of shape
    [B, heads, T_new*H*W, d]) with T_old context frames given by their keys and
    stage-1 outputs (k_cache, y1_cache of shape [B, heads, T_old*H*W, d]; None
    when T_old = 0).  Returns (out, y1_new); y1_new is the new frames' stage-1
    output, to append to y1_cache for the next chunk.
    """
    ts = [q, k, v] + ([k_cache, y1_cache] if T_old > 0 else [])
    if not all(t is not None and t.is_cuda and t.is_contiguous() for t in ts):
        raise ValueError("q, k, v and the context must be contiguous CUDA tensors")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or any(t.dtype != q.dtype for t in ts):
        raise ValueError("q, k, v must share one [B, heads, N, d] shape and dtype")
    B, heads, N, d = q.shape
    if N != T_new * H * W:
        raise ValueError(f"N={N} does not equal T_new*H*W={T_new * H * W}")
    if T_old > 0 and (k_cache.shape != (B, heads, T_old * H * W, d) or y1_cache.shape != k_cache.shape):
        raise ValueError("k_cache and y1_cache must be [B, heads, T_old*H*W, d]")
    out = torch.empty_like(q) if out is None else out
    y1_new = torch.empty_like(q) if y1_new is None else y1_new
    for t in (out, y1_new):
        if t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("out and y1_new must be contiguous CUDA tensors shaped and typed like q")
    kc = k_cache.data_ptr() if T_old > 0 else None
    yc = y1_cache.data_ptr() if T_old > 0 else None
    st = load_library().monarch_attn_fwd_chunk(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), kc, yc, out.data_ptr(), y1_new.data_ptr(), B, heads,
        int(T_old), int(T_new), H, W, d, int(factorisation), int(tile_h), int(tile_w), _dtype_code(q),
        _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_chunk")
    return out, y1_new


def monarch_attn_fwd_chunk_profiled(q, k, v, k_cache, y1_cache, out, y1_new, T_old, T_new, H, W, events,
                                    factorisation=FACT_FRAME, tile_h=0, tile_w=0, stream=None) -> int:
    """monarch_attn_fwd_chunk into given ``out`` / ``y1_new``, recording ``events``
    (torch.cuda.Event list) around each kernel launch.  Returns the number of
    kernel launches queued."""
    B, heads, N, d = q.shape
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    n = ctypes.c_int(0)
    kc = k_cache.data_ptr() if T_old > 0 else None
    yc = y1_cache.data_ptr() if T_old > 0 else None
    st = load_library().monarch_attn_fwd_chunk_profiled(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), kc, yc, out.data_ptr(), y1_new.data_ptr(), B, heads,
        int(T_old), int(T_new), H, W, d, int(factorisation), int(tile_h), int(tile_w), _dtype_code(q),
        _stream_ptr(stream), arr, len(events), ctypes.byref(n))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_chunk_profiled")
    return n.value


def monarch_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                             T: int, H: int, W: int, factorisation: int = FACT_FRAME, tile_h: int = 0,
                             tile_w: int = 0, stream=None) -> torch.Tensor:
    """bf16 monarch_attn_fwd through the entry point that allocates no device
    memory (static per-device counters; calls on one device must not overlap).
    ``out`` is required, since this path allocates nothing.
    """
    ts = (q, k, v, out)
    if not all(t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16 for t in ts):
        raise ValueError("q, k, v, out must be contiguous bf16 CUDA tensors")
    if q.dim() != 4 or any(t.shape != q.shape for t in ts):
        raise ValueError("q, k, v, out must share one [B, heads, N, d] shape")
    B, heads, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"N={N} does not equal T*H*W={T * H * W}")
    st = load_library().monarch_attn_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, heads, T, H, W, d,
        int(factorisation), int(tile_h), int(tile_w), _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_noalloc")
    return out


def monarch_attn_fwd_profiled(q, k, v, out, T, H, W, events, factorisation=FACT_FRAME, tile_h=0,
                              tile_w=0, stream=None) -> int:
    """monarch_attn_fwd recording ``events`` (torch.cuda.Event list) around each
    kernel launch: events[0] before the first, events[i+1] after launch i.
    Returns the number of kernel launches queued."""
    B, heads, N, d = q.shape
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    n = ctypes.c_int(0)
    st = load_library().monarch_attn_fwd_profiled(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, heads, T, H, W, d,
        int(factorisation), int(tile_h), int(tile_w), _dtype_code(q), _stream_ptr(stream),
        arr, len(events), ctypes.byref(n))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_profiled")
    return n.value


def monarch_attn_fwd_host(h_q, h_k, h_v, h_out, d_q, d_k, d_v, d_out, T, H, W,
                          factorisation=FACT_FRAME, tile_h=0, tile_w=0, stream=None):
    """Host-buffer variant: copies in, computes on the device buffers, copies out, syncs."""
    B, heads, N, d = h_q.shape
    st = load_library().monarch_attn_fwd_host(
        h_q.data_ptr(), h_k.data_ptr(), h_v.data_ptr(), h_out.data_ptr(),
        d_q.data_ptr(), d_k.data_ptr(), d_v.data_ptr(), d_out.data_ptr(),
        B, heads, T, H, W, d, int(factorisation), int(tile_h), int(tile_w),
        _dtype_code(h_q), _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_host")
    return h_out


def monarch_attn_fwd_host_pipelined(h_q, h_k, h_v, h_out, d_q, d_k, d_v, d_out, T, H, W,
                                    factorisation=FACT_FRAME, tile_h=0, tile_w=0, nchunks=4,
                                    stream=None) -> None:
    """monarch_attn_fwd_host with uploads, computation and downloads overlapped
    over `nchunks` chunks of batch-heads (pinned host tensors for overlap)."""
    B, heads, N, d = h_q.shape
    st = load_library().monarch_attn_fwd_host_pipelined(
        h_q.data_ptr(), h_k.data_ptr(), h_v.data_ptr(), h_out.data_ptr(), d_q.data_ptr(), d_k.data_ptr(),
        d_v.data_ptr(), d_out.data_ptr(), B, heads, T, H, W, d, int(factorisation), int(tile_h),
        int(tile_w), _dtype_code(h_q), int(nchunks), _stream_ptr(stream))
    if st != 0:
        raise MonarchError(st, "monarch_attn_fwd_host_pipelined")


def monarch_attn_device_status(stream=None, reset: bool = True) -> int:
    """Status word of the library's device-side waits (0 = none timed out); synchronises the stream."""
    return int(load_library().monarch_attn_device_status(_stream_ptr(stream), 1 if reset else 0))


def monarch_attn_selftest_timeout(limit_cycles: int, stream=None) -> int:
    """Runs one bounded wait that nothing completes; returns the resulting status (4 = timed out)."""
    return int(load_library().monarch_attn_selftest_timeout(int(limit_cycles), _stream_ptr(stream)))


def last_device_error(reset: bool = True, stream=None) -> int:
    return monarch_attn_device_status(stream, reset)


selftest_timeout = monarch_attn_selftest_timeout


def monarch_attn_bwd_profiled(q, k, v, dout, dq, dk, dv, workspace, T, H, W, events,
                              factorisation=FACT_FRAME, tile_h=0, tile_w=0, stream=None) -> int:
    """monarch_attn_bwd into given buffers, recording ``events`` (torch.cuda.Event
    list) around its phases (see include/monarch_attn.h).  Returns the number
    of phases recorded."""
    B, heads, N, d = q.shape
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    n = ctypes.c_int(0)
    st = load_library().monarch_attn_bwd_profiled(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), B, heads, T, H, W, d,
        int(factorisation), int(tile_h), int(tile_w), _dtype_code(q), _stream_ptr(stream), arr, len(events),
        ctypes.byref(n))
    if st != 0:
        raise MonarchError(st, "monarch_attn_bwd_profiled")
    return n.value
