"""GPU: bf16 / fp16 gradients on tensor cores (monarch_attn_bwd through the C
ABI) against the fp64 gradient oracle, element by element.

Bound, per gradient: relative L2 <= 1e-2 and max-abs <= 3e-2.  The kernels
hold Y1, O, P, dS and dY1 in the 16-bit type and accumulate in fp32; a
tile-level model of that arithmetic (each 16-bit rounding placed where the
kernels store) against the same oracle reaches a relative L2 of about 3.4e-3
and a max-abs of about 1e-2 on frame, tiled and (f*h, w) shapes with
unit-variance inputs, so the bounds keep a factor of about 3.
"""
import numpy as np
import pytest
import torch

import oracle
from structured_attention_video_monarch_b200 import binding

pytestmark = pytest.mark.gpu

RL2 = 1e-2
ATOL = 3e-2

CASES = [
    # B, heads, T, H, W, d, fact, tile_h, tile_w
    (1, 2, 3, 6, 20, 128, 0, 0, 0),     # m = 120: one ragged tile
    (1, 1, 4, 10, 26, 64, 0, 0, 0),     # m = 260: three tiles
    (1, 1, 2, 16, 16, 128, 0, 0, 0),    # m = 256: two full tiles
    (2, 1, 21, 4, 5, 128, 0, 0, 0),     # T = 21: stacked stage-2 tiles of 6 positions
    (1, 1, 1, 9, 13, 128, 0, 0, 0),     # T = 1: stage 2 is the identity
    (1, 1, 128, 1, 2, 64, 0, 0, 0),     # T = 128, m = 2: one position per stage-2 tile
    (1, 2, 3, 8, 24, 128, 1, 4, 8),     # tiled, 32-token tiles
    (1, 1, 2, 10, 26, 64, 1, 10, 13),   # tiled, 130-token tiles (two query tiles)
    (1, 2, 3, 4, 20, 128, 2, 0, 0),     # (f*h, w): rows of 20, columns of 12
    (1, 1, 9, 30, 3, 64, 2, 0, 0),      # (f*h, w): columns of 270 (three tiles)
]


def _grads(q, k, v, do, T, H, W, fact, th, tw, **kw):
    dev = torch.device("cuda:0")
    out = binding.monarch_attn_bwd(*(x.to(dev) for x in (q, k, v, do)), T, H, W, fact, th, tw, **kw)
    torch.cuda.synchronize()
    assert binding.last_device_error() == 0
    return out


def _check(got, want):
    for name, g, ref in zip(("dq", "dk", "dv"), got, want):
        g = g.double().cpu().numpy()
        assert np.isfinite(g).all(), f"non-finite {name}"
        rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        err = np.abs(g - ref).max()
        assert rel <= RL2, f"{name}: relative L2 {rel:.3g} (max-abs {err:.3g})"
        assert err <= ATOL, f"{name}: max-abs {err:.3g} (relative L2 {rel:.3g})"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "f16"])
@pytest.mark.parametrize("B,heads,T,H,W,d,fact,th,tw", CASES)
def test_tc_gradients_match_oracle(B, heads, T, H, W, d, fact, th, tw, dtype):
    g = torch.Generator().manual_seed(T * 100 + W)
    q, k, v, do = (torch.randn(B, heads, T * H * W, d, generator=g).to(dtype) for _ in range(4))
    got = _grads(q, k, v, do, T, H, W, fact, th, tw)
    _check(got, oracle.monarch_bwd(q, k, v, do, T, H, W, fact, th, tw))


def test_tc_gradients_chunk_shape():
    """The chunk workload's shape (frames of 30 x 52 = 1560 tokens, 13 query
    tiles per block), two heads, with caller buffers reused over two calls."""
    B, heads, T, H, W, d = 1, 2, 3, 30, 52, 128
    g = torch.Generator().manual_seed(4680)
    q, k, v, do = (torch.randn(B, heads, T * H * W, d, generator=g).to(torch.bfloat16) for _ in range(4))
    dev = torch.device("cuda:0")
    qd = q.to(dev)
    ws = binding.monarch_attn_bwd_workspace(qd, T, H, W)
    out = tuple(torch.full_like(qd, float("nan")) for _ in range(3))
    want = oracle.monarch_bwd(q, k, v, do, T, H, W)
    first = None
    for _ in range(2):
        got = _grads(q, k, v, do, T, H, W, 0, 0, 0, out=out, workspace=ws)
        _check(got, want)
        cur = [x.clone() for x in got]
        if first is not None:  # one owning CTA per gradient row: deterministic
            assert all(torch.equal(a, b) for a, b in zip(first, cur))
        first = cur


def test_tc_gradients_rejections():
    dev = torch.device("cuda:0")
    x = torch.zeros(1, 1, 129 * 2, 128, dtype=torch.bfloat16, device=dev)
    with pytest.raises(binding.MonarchError):  # T > 128 (frame split)
        binding.monarch_attn_bwd(x, x, x, x, 129, 1, 2)
    y = torch.zeros(1, 1, 2 * 4 * 4, 128, dtype=torch.bfloat16, device=dev)
    ws = binding.monarch_attn_bwd_workspace(y, 2, 4, 4)
    with pytest.raises(binding.MonarchError):  # workspace too small
        binding.monarch_attn_bwd(y, y, y, y, 2, 4, 4, workspace=ws[:-16])
