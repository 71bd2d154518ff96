"""Autoregressive chunk forward (monarch_attn_fwd_chunk) against the fp64
oracle's chunk form, element by element, through the C ABI.

The chunk runs the forward's stage-1 kernel on the new frames (tensor cores
for bf16/fp16, CUDA cores for fp32) and a CUDA-core stage 2 over the context
and the new frames.  Bounds are the forward's: Y1 is held in the input dtype
in both the output y1_new and the context.
"""
import numpy as np
import pytest
import torch

import oracle
from structured_attention_video_monarch_b200 import binding

pytestmark = pytest.mark.gpu

TOL = {  # dtype: (max-abs, relative L2)
    torch.float32: (1e-5, None),
    torch.bfloat16: (2e-2, 1e-2),
    torch.float16: (1e-2, 4e-3),
}

CASES = [
    # B, heads, T_old, T_new, H, W, d, fact, tile_h, tile_w
    (1, 2, 4, 3, 6, 20, 128, 0, 0, 0),      # m = 120: one ragged query tile
    (2, 1, 6, 3, 8, 25, 64, 0, 0, 0),       # m = 200: two tiles, 9 keys (ragged vs 4-key steps)
    (1, 1, 0, 3, 6, 20, 128, 0, 0, 0),      # no context
    (1, 2, 7, 1, 5, 30, 128, 0, 0, 0),      # one new frame
    (1, 1, 3, 6, 4, 34, 128, 0, 0, 0),      # six new frames: two query passes of 4
    (1, 2, 5, 3, 8, 24, 128, 1, 4, 8),      # tiled, 32-token tiles
    (1, 1, 2, 2, 10, 40, 64, 1, 5, 20),     # tiled, 100-token tiles
]


def _inputs(B, heads, T_old, T_new, H, W, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    n_new, n_old = T_new * H * W, T_old * H * W
    scale = d ** -0.25 if dtype == torch.float32 else 1.0
    q, k, v = (torch.randn(B, heads, n_new, d, generator=g) * scale for _ in range(3))
    kc = torch.randn(B, heads, n_old, d, generator=g) * scale
    yc = torch.randn(B, heads, n_old, d, generator=g)
    return [t.to(dtype) for t in (q, k, v, kc, yc)]


def _check(got, want, dtype, what):
    got = got.double().cpu().numpy()
    atol, rl2 = TOL[dtype]
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want).max()
    assert err <= atol, f"{what}: max-abs {err:.3g} > {atol}"
    if rl2 is not None:
        rel = np.linalg.norm(got - want) / np.linalg.norm(want)
        assert rel <= rl2, f"{what}: relative L2 {rel:.3g} > {rl2}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32], ids=["bf16", "f16", "f32"])
@pytest.mark.parametrize("B,heads,T_old,T_new,H,W,d,fact,th,tw", CASES)
def test_chunk_matches_oracle(B, heads, T_old, T_new, H, W, d, fact, th, tw, dtype):
    q, k, v, kc, yc = _inputs(B, heads, T_old, T_new, H, W, d, dtype, seed=T_old * 31 + W)
    dev = [t.cuda() for t in (q, k, v, kc, yc)]
    out = torch.full_like(dev[0], float("nan"))
    y1 = torch.full_like(dev[0], float("nan"))
    binding.monarch_attn_fwd_chunk(*dev[:3], dev[3] if T_old else None, dev[4] if T_old else None, T_old,
                                   T_new, H, W, fact, th, tw, out=out, y1_new=y1)
    torch.cuda.synchronize()
    f64 = [t.double().numpy() for t in (q, k, v, kc, yc)]
    want_out, want_y1 = oracle.monarch_fwd_chunk(*f64, T_old, T_new, H, W, fact, th, tw)
    _check(y1, want_y1, dtype, "y1_new")
    _check(out, want_out, dtype, "out")


def test_last_chunk_matches_full_forward_bf16():
    # a 9-frame clip: the forward of all 9 frames, and the chunk of the last 3
    # with the first 6 frames' keys and (device-computed) stage-1 outputs as context
    B, heads, H, W, d, T_old, T_new = 1, 2, 6, 20, 128, 6, 3
    T = T_old + T_new
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(B, heads, T * H * W, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    full = binding.monarch_attn_fwd(q, k, v, T, H, W)
    n_old = T_old * H * W
    _, y1_old = binding.monarch_attn_fwd_chunk(q[:, :, :n_old].contiguous(), k[:, :, :n_old].contiguous(),
                                               v[:, :, :n_old].contiguous(), None, None, 0, T_old, H, W)
    out, _ = binding.monarch_attn_fwd_chunk(q[:, :, n_old:].contiguous(), k[:, :, n_old:].contiguous(),
                                            v[:, :, n_old:].contiguous(), k[:, :, :n_old].contiguous(),
                                            y1_old, T_old, T_new, H, W)
    torch.cuda.synchronize()
    diff = (out.float() - full[:, :, n_old:].float()).abs().max().item()
    # two bf16 paths over the same bf16 Y1 differ only in the stage-2 rounding
    # (bf16 P in the tensor-core stage 2): a few bf16 ulps of |out| <= ~3
    assert diff <= 2e-2, diff


def test_chunk_workload_full_size_sampled_heads():
    # the chunk shape at full size (12 heads, 30 x 52 grid, d 128) as the last
    # 3 frames of a 21-frame clip; the oracle checks two heads in full
    B, heads, T_old, T_new, H, W, d = 1, 12, 18, 3, 30, 52, 128
    q, k, v, kc, yc = _inputs(B, heads, T_old, T_new, H, W, d, torch.bfloat16, seed=77)
    dev = [t.cuda() for t in (q, k, v, kc, yc)]
    out, y1 = binding.monarch_attn_fwd_chunk(*dev, T_old, T_new, H, W)
    torch.cuda.synchronize()
    for h in (0, 11):
        f64 = [t[:, h:h + 1].double().numpy() for t in (q, k, v, kc, yc)]
        want_out, want_y1 = oracle.monarch_fwd_chunk(*f64, T_old, T_new, H, W)
        _check(y1[:, h:h + 1], want_y1, torch.bfloat16, f"y1_new head {h}")
        _check(out[:, h:h + 1], want_out, torch.bfloat16, f"out head {h}")
    assert torch.isfinite(out.float()).all()


def test_chunk_repeat_is_deterministic():
    q, k, v, kc, yc = (t.cuda() for t in _inputs(1, 2, 5, 3, 8, 24, 128, torch.bfloat16, seed=3))
    a, ya = binding.monarch_attn_fwd_chunk(q, k, v, kc, yc, 5, 3, 8, 24)
    b, yb = binding.monarch_attn_fwd_chunk(q, k, v, kc, yc, 5, 3, 8, 24)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(ya, yb)
