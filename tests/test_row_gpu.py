"""The (f*h, w) split (MONARCH_FACT_ROW) through the C ABI against the fp64
oracle's FACT_ROW forward, element by element.

The split runs as two stage-1 passes of the forward's kernels over virtual
shapes: rows of W tokens (a frame split of T*H one-row frames), then columns
of T*H tokens (a tiled split of one (T*H) x W frame with 1-wide tiles) with
the rows' output as values.  Bounds are the forward's.
"""
import numpy as np
import pytest
import torch

import oracle
from structured_attention_video_monarch_b200 import binding

pytestmark = pytest.mark.gpu

ROW = 2
TOL = {  # dtype: (max-abs, relative L2)
    torch.float32: (1e-5, None),
    torch.bfloat16: (2e-2, 1e-2),
    torch.float16: (1e-2, 4e-3),
}

CASES = [
    # B, heads, T, H, W, d
    (1, 2, 3, 4, 20, 128),    # rows of 20 tokens, columns of 12
    (2, 1, 2, 5, 40, 64),
    (1, 1, 4, 40, 8, 128),    # columns of 160 tokens: two key tiles, ragged
    (1, 1, 1, 1, 200, 128),   # one row of 200 tokens (two tiles); columns of one token
    (1, 1, 9, 30, 3, 64),     # columns of 270 tokens (three tiles); rows of 3
    (1, 2, 3, 1, 30, 128),    # H = 1: the frame split's blocks and groups
    (1, 1, 130, 1, 16, 128),  # more than 128 frames (allowed for this split)
    (1, 1, 7, 1, 40, 128),    # 7 frame rows (prime count): rows of 40 stay unpacked
    (1, 2, 6, 5, 52, 128),    # rows of 52 packed two to a query tile (the full clip's width)
]


def _inputs(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    scale = shape[-1] ** -0.25 if dtype == torch.float32 else 1.0
    return [(torch.randn(*shape, generator=g) * scale).to(dtype) for _ in range(3)]


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
@pytest.mark.parametrize("B,heads,T,H,W,d", CASES)
def test_row_split_matches_oracle(B, heads, T, H, W, d, dtype):
    q, k, v = _inputs((B, heads, T * H * W, d), dtype, seed=T * 100 + H * 10 + W)
    out = torch.full(q.shape, float("nan"), dtype=dtype, device="cuda")
    binding.monarch_attn_fwd(q.cuda(), k.cuda(), v.cuda(), T, H, W, ROW, out=out)
    torch.cuda.synchronize()
    want = oracle.monarch_fwd(q.double().numpy(), k.double().numpy(), v.double().numpy(), T, H, W, ROW)
    _check(out, want, dtype, "out")


def test_row_split_full_clip_one_head_exact():
    # the full-clip grid (12 heads, 21 x 30 x 52, d 128); the oracle checks one head in full
    B, heads, T, H, W, d = 1, 12, 21, 30, 52, 128
    q, k, v = _inputs((B, heads, T * H * W, d), torch.bfloat16, seed=6)
    out = binding.monarch_attn_fwd(q.cuda(), k.cuda(), v.cuda(), T, H, W, ROW)
    torch.cuda.synchronize()
    h = 7
    want = oracle.monarch_fwd(*(x[:, h:h + 1].double().numpy() for x in (q, k, v)), T, H, W, ROW)
    _check(out[:, h:h + 1], want, torch.bfloat16, f"head {h}")
    assert torch.isfinite(out.float()).all()


def test_row_split_repeat_and_second_stream():
    q, k, v = (x.cuda() for x in _inputs((1, 2, 3 * 4 * 20, 128), torch.bfloat16, seed=9))
    a = binding.monarch_attn_fwd(q, k, v, 3, 4, 20, ROW)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = binding.monarch_attn_fwd(q, k, v, 3, 4, 20, ROW)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_row_split_profiled_events_bracket_each_pass():
    # events[0] before the rows pass, events[1] between the passes, events[2] after
    q, k, v = (x.cuda() for x in _inputs((1, 2, 3 * 4 * 20, 128), torch.bfloat16, seed=10))
    out = torch.empty_like(q)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in ev:
        e.record()
    n = binding.monarch_attn_fwd_profiled(q, k, v, out, 3, 4, 20, ev, ROW)
    torch.cuda.synchronize()
    assert n == 2
    assert ev[0].elapsed_time(ev[1]) > 0 and ev[1].elapsed_time(ev[2]) > 0
