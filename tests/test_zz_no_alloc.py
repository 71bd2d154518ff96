"""GPU: monarch_attn_fwd_noalloc (static per-device counters, no cudaMalloc)
against monarch_attn_fwd on the same inputs, through the C ABI.

The file name sorts last so the entry point is also exercised after every
other GPU test has run in the same process; it passes on its own as well.
Tolerance is the bf16 parity bar (max-abs <= 2e-2, relative L2 <= 1e-2).
"""
import ctypes

import numpy as np
import pytest
import torch

from structured_attention_video_monarch_b200 import binding, workloads

pytestmark = pytest.mark.gpu

BF16_ATOL = 2e-2
BF16_RL2 = 1e-2
MAX_BH = 4096  # MONARCH_NOALLOC_MAX_BH in the header

CASES = [
    # name, B, heads, T, H, W, d, fact, tile_h, tile_w
    ("chunk_frame_d128", 1, 12, 3, 30, 52, 128, 0, 0, 0),
    ("tiled_d128", 2, 3, 5, 10, 26, 128, 1, 5, 13),
    ("frame_d64_ragged", 3, 2, 7, 9, 17, 64, 0, 0, 0),
]


def _inputs(B, heads, T, H, W, d, seed):
    q, k, v = workloads.random_inputs(B, heads, T, H, W, d, torch.bfloat16, seed)
    dev = torch.device("cuda:0")
    return tuple(x.to(dev) for x in (q, k, v))


def _close(got: torch.Tensor, ref: torch.Tensor):
    g, r = got.double().cpu().numpy(), ref.double().cpu().numpy()
    assert np.isfinite(g).all(), "non-finite output (unwritten element)"
    err = np.abs(g - r).max()
    rl2 = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert err <= BF16_ATOL, f"max-abs {err:.3e}"
    assert rl2 <= BF16_RL2, f"rel-L2 {rl2:.3e}"


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_fwd_on_two_calls_in_a_row(case):
    _, B, heads, T, H, W, d, fact, th, tw = case
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q, k, v = _inputs(B, heads, T, H, W, d, seed=11)
    ref = torch.full_like(q, float("nan"))
    binding.monarch_attn_fwd(q, k, v, T, H, W, fact, th, tw, out=ref)
    outs = []
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        binding.monarch_attn_fwd_noalloc(q, k, v, out, T, H, W, fact, th, tw)
        outs.append(out)
    torch.cuda.synchronize()
    assert binding.last_device_error() == 0
    for out in outs:
        _close(out, ref)


def test_noalloc_counters_reset_between_shapes():
    # A call over many batch-heads, then one over few, then many again: the
    # counters each call leaves behind must not leak into the next call.
    shapes = [(4, 16, 4, 8, 16, 128), (1, 1, 4, 8, 16, 128), (4, 16, 4, 8, 16, 128)]
    for i, (B, heads, T, H, W, d) in enumerate(shapes):
        q, k, v = _inputs(B, heads, T, H, W, d, seed=100 + i)
        ref = torch.full_like(q, float("nan"))
        binding.monarch_attn_fwd(q, k, v, T, H, W, out=ref)
        out = torch.full_like(q, float("nan"))
        binding.monarch_attn_fwd_noalloc(q, k, v, out, T, H, W)
        torch.cuda.synchronize()
        assert binding.last_device_error() == 0
        _close(out, ref)


def test_noalloc_rejects_more_batch_heads_than_its_scratch():
    lib = binding.load_library()
    B, heads, T, H, W, d = 1, MAX_BH + 1, 1, 1, 1, 64
    q, k, v = _inputs(B, heads, T, H, W, d, seed=5)
    out = torch.zeros_like(q)
    st = lib.monarch_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      B, heads, T, H, W, d, 0, 0, 0,
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 2  # MONARCH_ERR_UNSUPPORTED, nothing queued
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0
