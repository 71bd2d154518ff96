"""GPU: the fp32 backward (monarch_attn_bwd, through the C ABI) against the
fp64 gradient oracle.

Tolerance: max-abs <= 1e-4.  Every gradient element is a sum over a block
(at most a few hundred terms here) of products of O(1) factors, accumulated in
fp32 (and, for dK and dV, by atomic adds in a varying order): the rounding
error stays below m * 2^-24 * |term| ~ 2.4e-5 for m = 400, and the 1e-4 bound
leaves a factor-4 margin.  Inputs are scaled by d^-1/4 as in the fp32
forward tests.
"""
import numpy as np
import pytest
import torch

import oracle
from structured_attention_video_monarch_b200 import binding, workloads

pytestmark = pytest.mark.gpu

ATOL = 1e-4

CASES = [
    # B, heads, T, H, W, d, fact, tile_h, tile_w
    (1, 2, 3, 5, 7, 128, 0, 0, 0),      # m = 35
    (1, 1, 2, 8, 16, 64, 0, 0, 0),      # m = 128
    (2, 1, 4, 20, 20, 128, 0, 0, 0),    # m = 400
    (1, 2, 3, 8, 12, 64, 1, 4, 3),      # tiles of 12 tokens
    (1, 1, 1, 9, 9, 128, 0, 0, 0),      # T = 1
    (1, 1, 21, 2, 3, 64, 0, 0, 0),      # T = 21, m = 6
]


@pytest.mark.parametrize("B,heads,T,H,W,d,fact,th,tw", CASES)
def test_backward_matches_oracle(B, heads, T, H, W, d, fact, th, tw):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    dev = torch.device("cuda:0")
    q, k, v = workloads.random_inputs(B, heads, T, H, W, d, dtype=torch.float32, seed=T * 100 + H,
                                      scale=d ** -0.25)
    g = torch.Generator().manual_seed(5)
    do = torch.randn(q.shape, generator=g)
    dq, dk, dv = binding.monarch_attn_bwd(*(x.to(dev) for x in (q, k, v, do)), T, H, W, fact, th, tw)
    torch.cuda.synchronize()
    ref = oracle.monarch_bwd(q, k, v, do, T, H, W, fact, th, tw)
    for name, got, want in zip("qkv", (dq, dk, dv), ref):
        got = got.cpu().double().numpy()
        assert np.isfinite(got).all(), f"non-finite d{name}"
        err = np.abs(got - want).max()
        assert err <= ATOL, f"d{name}: max-abs {err:.3e}"


def test_backward_fp32_rejects_row_split():
    """The (f*h, w) split has gradients on the tensor-core path only."""
    dev = torch.device("cuda:0")
    x = torch.zeros(1, 1, 2 * 4 * 4, 128, dtype=torch.float32, device=dev)
    with pytest.raises(binding.MonarchError):
        binding.monarch_attn_bwd(x, x, x, x, 2, 4, 4, factorisation=2)


# m = 1560 (one 30 x 52 frame, the chunk workload's block): the stage-1
# backward needs more than 48 KB of dynamic shared memory there.  The same
# rounding argument as above gives m * 2^-24 * |term| ~ 9.3e-5 per gradient
# element; the bound keeps the factor-4 margin.
ATOL_M1560 = 4e-4


def test_backward_frame_1560_reusing_buffers():
    dev = torch.device("cuda:0")
    B, heads, T, H, W, d = 1, 1, 2, 30, 52, 128
    q, k, v = workloads.random_inputs(B, heads, T, H, W, d, dtype=torch.float32, seed=1560, scale=d ** -0.25)
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(6))
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    out = tuple(torch.full_like(qd, float("nan")) for _ in range(3))
    ws = binding.monarch_attn_bwd_workspace(qd, T, H, W)
    ref = oracle.monarch_bwd(q, k, v, do, T, H, W)
    for _ in range(2):  # the second call reuses (and overwrites) the same buffers
        got = binding.monarch_attn_bwd(qd, kd, vd, dod, T, H, W, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert all(g is o for g, o in zip(got, out))
        for name, g, want in zip("qkv", got, ref):
            g = g.cpu().double().numpy()
            assert np.isfinite(g).all(), f"non-finite d{name}"
            err = np.abs(g - want).max()
            assert err <= ATOL_M1560, f"d{name}: max-abs {err:.3e}"


def test_backward_rejects_bad_buffers():
    dev = torch.device("cuda:0")
    T, H, W = 2, 4, 4
    x = torch.zeros(1, 1, T * H * W, 64, device=dev)
    ws = binding.monarch_attn_bwd_workspace(x, T, H, W)
    good = tuple(torch.empty_like(x) for _ in range(3))
    with pytest.raises(ValueError):  # a workspace in host memory
        binding.monarch_attn_bwd(x, x, x, x, T, H, W, workspace=ws.cpu())
    with pytest.raises(ValueError):  # a non-contiguous workspace
        binding.monarch_attn_bwd(x, x, x, x, T, H, W, workspace=ws[::2])
    with pytest.raises(ValueError):  # a mis-shaped gradient buffer
        binding.monarch_attn_bwd(x, x, x, x, T, H, W, out=(good[0], good[1], torch.empty(1, 1, 8, 64, device=dev)))
    with pytest.raises(ValueError):  # a gradient buffer in host memory
        binding.monarch_attn_bwd(x, x, x, x, T, H, W, out=(good[0], good[1], good[2].cpu()))
    with pytest.raises(binding.MonarchError):  # a workspace too small (its size is passed in bytes)
        binding.monarch_attn_bwd(x, x, x, x, T, H, W, workspace=ws[: ws.numel() // 2])
