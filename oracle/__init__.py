"""fp64 CPU oracle for the Monarch attention forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never imports, links or executes anything here, and nothing
here imports the product path.

The arithmetic lives in ``monarch_oracle.c`` (plain double-precision loops,
OpenMP over independent blocks).  This module only compiles it with gcc and
marshals numpy arrays through ctypes.

Definition followed: MonarchRT: Efficient Attention for Real-Time Video
Generation (gist.science/nl/paper/2602.12271, "Methodologie": permutation and
block-diagonal factors; gist.science/zh/paper/2602.12271, section 2.2: blocks
aligned with the (f, h, w) axes, tiled Monarch).  ``out = P^T B2 P B1 V`` with
each diagonal block a dense softmax attention, scale 1/sqrt(d).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

FACT_FRAME = 0
FACT_TILED = 1
FACT_ROW = 2  # the (f*h, w) split: stage-1 blocks are the W tokens of one (frame, row)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "monarch_oracle.c")
_LIB = os.path.join(_HERE, "libmonarch_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmonarch_oracle.so`` with gcc."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _configure(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.oracle_monarch_fwd.argtypes = [dp, dp, dp, dp] + [i] * 9
    lib.oracle_monarch_stage1.argtypes = [dp, dp, dp, dp] + [i] * 9
    lib.oracle_monarch_stage2.argtypes = [dp, dp, dp, dp] + [i] * 6
    lib.oracle_monarch_fwd_groups.argtypes = (
        [dp, dp, dp] + [i] * 9 + [ctypes.POINTER(ctypes.c_long), i, dp])
    lib.oracle_monarch_bwd.argtypes = [dp] * 7 + [i] * 9
    lib.oracle_monarch_fwd_chunk.argtypes = [dp] * 7 + [i] * 10
    for f in (lib.oracle_monarch_fwd, lib.oracle_monarch_stage1,
              lib.oracle_monarch_stage2, lib.oracle_monarch_fwd_groups,
              lib.oracle_monarch_bwd, lib.oracle_monarch_fwd_chunk, lib.oracle_num_threads):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


def use_library(path):
    """Point this module at another build of the oracle source (used by the
    mutation tests, which compile deliberately broken copies); returns the
    previous library so the caller can restore it."""
    global _lib
    with _lock:
        prev = _lib
        _lib = _configure(ctypes.CDLL(path)) if path else None
    return prev


def restore_library(prev):
    global _lib
    with _lock:
        _lib = prev


def num_threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def _dims(q, T, H, W):
    if q.ndim != 4:
        raise ValueError("expected [B, heads, N, d]")
    B, heads, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"N={N} != T*H*W={T * H * W}")
    return B, heads, d


def monarch_fwd(q, k, v, T, H, W, fact=FACT_FRAME, tile_h=0, tile_w=0) -> np.ndarray:
    """out = P^T B2 P B1 V for [B, heads, T*H*W, d] inputs, in float64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, heads, d = _dims(q, T, H, W)
    out = np.empty_like(q)
    _check(_load().oracle_monarch_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                      B, heads, T, H, W, d, fact, tile_h, tile_w), "fwd")
    return out


def monarch_bwd(q, k, v, dout, T, H, W, fact=FACT_FRAME, tile_h=0, tile_w=0):
    """Gradients (dq, dk, dv) of out = P^T B2 P B1 V for an upstream gradient
    dout, all [B, heads, T*H*W, d], in float64."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, heads, d = _dims(q, T, H, W)
    if dout.shape != q.shape:
        raise ValueError("dout must be shaped like q")
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _check(_load().oracle_monarch_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                      _ptr(dv), B, heads, T, H, W, d, fact, tile_h, tile_w), "bwd")
    return dq, dk, dv


def monarch_fwd_chunk(q, k, v, k_cache, y1_cache, T_old, T_new, H, W, fact=FACT_FRAME, tile_h=0,
                      tile_w=0):
    """Forward of a chunk of T_new new frames with T_old earlier frames as
    context (their keys k_cache and stage-1 outputs y1_cache, [B, heads,
    T_old*H*W, d]; None when T_old = 0).  Returns (out, y1_new) for the new
    frames, float64."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, heads, d = _dims(q, T_new, H, W)
    out, y1 = np.empty_like(q), np.empty_like(q)
    if T_old > 0:
        kc, yc = _as_f64(k_cache), _as_f64(y1_cache)
        if kc.shape != (B, heads, T_old * H * W, d) or yc.shape != kc.shape:
            raise ValueError("k_cache and y1_cache must be [B, heads, T_old*H*W, d]")
        pk, py = _ptr(kc), _ptr(yc)
    else:
        pk = py = None
    _check(_load().oracle_monarch_fwd_chunk(_ptr(q), _ptr(k), _ptr(v), pk, py, _ptr(out), _ptr(y1), B, heads,
                                            T_old, T_new, H, W, d, fact, tile_h, tile_w), "fwd_chunk")
    return out, y1


def monarch_stage1(q, k, v, T, H, W, fact=FACT_FRAME, tile_h=0, tile_w=0) -> np.ndarray:
    """Stage-1 output Y1 = B1 V only (block-local attention)."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, heads, d = _dims(q, T, H, W)
    y1 = np.empty_like(q)
    _check(_load().oracle_monarch_stage1(_ptr(q), _ptr(k), _ptr(v), _ptr(y1),
                                         B, heads, T, H, W, d, fact, tile_h, tile_w), "stage1")
    return y1


def monarch_stage2(q, k, y1, T, H, W) -> np.ndarray:
    """Stage-2 output P^T B2 P Y1 (attention across frames per position)."""
    q, k, y1 = _as_f64(q), _as_f64(k), _as_f64(y1)
    B, heads, d = _dims(q, T, H, W)
    out = np.empty_like(q)
    _check(_load().oracle_monarch_stage2(_ptr(q), _ptr(k), _ptr(y1), _ptr(out),
                                         B, heads, T, H, W, d), "stage2")
    return out


def monarch_fwd_groups(q, k, v, T, H, W, groups, fact=FACT_FRAME, tile_h=0,
                       tile_w=0) -> np.ndarray:
    """Exact output rows for the listed (bh, pos) stage-2 groups.

    Returns float64 [len(groups), T, d]; row t of group g is the output token
    n = t*H*W + pos of batch-head bh.
    """
    if q.ndim != 4:
        raise ValueError("expected [B, heads, N, d]")
    B, heads, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"N={N} != T*H*W={T * H * W}")
    g = np.asarray(groups, dtype=np.int64).reshape(-1, 2).copy()
    # Convert only the batch-heads the groups touch (large workloads).
    used = sorted(set(int(x) for x in g[:, 0]))
    remap = {bh: i for i, bh in enumerate(used)}

    def pick(x):
        if hasattr(x, "detach"):
            x = x.detach().reshape(B * heads, N, d)
            return np.ascontiguousarray(
                np.stack([x[bh].to("cpu").double().numpy() for bh in used])[None])
        x = np.asarray(x).reshape(B * heads, N, d)
        return np.ascontiguousarray(x[used][None], dtype=np.float64)

    qs, ks, vs = pick(q), pick(k), pick(v)
    g[:, 0] = [remap[int(x)] for x in g[:, 0]]
    g = np.ascontiguousarray(g)
    out = np.empty((g.shape[0], T, d), dtype=np.float64)
    _check(_load().oracle_monarch_fwd_groups(
        _ptr(qs), _ptr(ks), _ptr(vs), 1, len(used), T, H, W, d, fact, tile_h, tile_w,
        g.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), int(g.shape[0]), _ptr(out)), "groups")
    return out
