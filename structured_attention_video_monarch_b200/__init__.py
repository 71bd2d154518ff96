"""B200-native Monarch attention forward (MonarchRT).

    out = P^T B2 P B1 V

over a video token grid N = T*H*W: stage 1 is softmax attention inside each
frame (or spatial tile of a frame, or frame row for the (f*h, w) split),
stage 2 is softmax attention across frames at each spatial position (or down
each column), applied to stage 1's output.  Also: one autoregressive chunk of
new frames against cached keys and stage-1 outputs (``monarch_attn_fwd_chunk``)
and gradients (``monarch_attn_bwd``: bf16/fp16 on tensor cores, fp32 on CUDA
cores).  Every step runs in
hand-written sm_100a CUDA kernels behind a C ABI (``include/monarch_attn.h``);
this package is the thin ctypes binding over it.

The binding is imported lazily so that ``workloads`` (seeded inputs) can be
used without loading the CUDA library.
"""

__all__ = [
    "monarch_attn_fwd", "monarch_attn_fwd_host", "monarch_attn_fwd_chunk", "monarch_attn_bwd",
    "monarch_attn_bwd_workspace", "monarch_attn_fwd_noalloc", "MonarchError", "lib_path",
    "FACT_FRAME", "FACT_TILED", "FACT_ROW", "DTYPE_F32", "DTYPE_BF16", "DTYPE_F16",
]

FACT_FRAME = 0
FACT_TILED = 1
FACT_ROW = 2
DTYPE_F32 = 0
DTYPE_BF16 = 1
DTYPE_F16 = 2


def __getattr__(name):
    if name in ("monarch_attn_fwd", "monarch_attn_fwd_host", "monarch_attn_fwd_chunk", "monarch_attn_bwd",
                "monarch_attn_bwd_workspace", "monarch_attn_fwd_noalloc", "MonarchError", "lib_path",
                "load_library", "strerror", "last_device_error"):
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
