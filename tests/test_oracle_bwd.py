"""Pins for the oracle's gradients (oracle_monarch_bwd), independent of it:

  * dV = M^T dO with M the explicit N x N Monarch matrix P^T B2 P B1 built
    from dense block softmaxes -> catches errors in the value gradient and in
    how stage 2's value gradient (dY1) feeds stage 1;
  * central finite differences of L = <dO, out> for sampled entries of q, k
    and v, on the frame and tiled splits -> catches a dropped softmax-Jacobian
    term, a missing scale, a lost stage-1 or stage-2 contribution to dQ/dK;
  * T = 1 and H = W = 1 reduce to dense attention, whose gradients come from
    the library's autograd (float64, CPU).
"""
import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import BRUTE_SHAPES, _explicit_factors, _rand


@pytest.mark.parametrize("T,H,W,d,fact,th,tw", BRUTE_SHAPES)
def test_value_gradient_is_monarch_transpose(T, H, W, d, fact, th, tw):
    N = T * H * W
    q, k, v, do = (_rand((1, 1, N, d), s) for s in (20, 21, 22, 23))
    B1, P, B2 = _explicit_factors(q[0, 0], k[0, 0], T, H, W, fact, th, tw)
    M = P.T @ B2 @ P @ B1
    _, _, dv = oracle.monarch_bwd(q, k, v, do, T, H, W, fact, th, tw)
    np.testing.assert_allclose(dv[0, 0], M.T @ do[0, 0], rtol=0, atol=1e-12)


FD_SHAPES = [
    # B, heads, T, H, W, d, fact, tile_h, tile_w
    (1, 2, 3, 2, 3, 4, 0, 0, 0),
    (2, 1, 2, 4, 4, 4, 1, 2, 2),
    (1, 1, 4, 3, 2, 6, 0, 0, 0),
]


@pytest.mark.parametrize("B,heads,T,H,W,d,fact,th,tw", FD_SHAPES)
def test_finite_differences(B, heads, T, H, W, d, fact, th, tw):
    N = T * H * W
    shape = (B, heads, N, d)
    q, k, v, do = (_rand(shape, s) for s in (30, 31, 32, 33))
    grads = dict(zip("qkv", oracle.monarch_bwd(q, k, v, do, T, H, W, fact, th, tw)))
    x = {"q": q, "k": k, "v": v}

    def loss():
        return float(np.sum(do * oracle.monarch_fwd(x["q"], x["k"], x["v"], T, H, W, fact, th, tw)))

    rng = np.random.default_rng(7)
    h = 1e-5
    for name in "qkv":
        for _ in range(12):
            idx = tuple(int(rng.integers(n)) for n in shape)
            keep = x[name][idx]
            x[name][idx] = keep + h
            up = loss()
            x[name][idx] = keep - h
            down = loss()
            x[name][idx] = keep
            fd = (up - down) / (2 * h)
            assert abs(fd - grads[name][idx]) < 1e-7 * max(1.0, abs(fd)), (name, idx, fd, grads[name][idx])


def _sdpa_grads(q, k, v, do):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).requires_grad_(True)
    tq, tk, tv = t(q), t(k), t(v)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(torch.from_numpy(np.ascontiguousarray(do)))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("H,W,d", [(3, 5, 8), (4, 4, 16)])
def test_single_frame_gradients_are_dense_attention_gradients(H, W, d):
    q, k, v, do = (_rand((1, 2, H * W, d), s) for s in (40, 41, 42, 43))
    got = oracle.monarch_bwd(q, k, v, do, 1, H, W)
    for a, b in zip(got, _sdpa_grads(q, k, v, do)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,d", [(5, 8), (7, 4)])
def test_single_position_gradients_are_dense_attention_gradients(T, d):
    # H = W = 1: stage 1 attends to the token itself (weight 1), stage 2 is
    # dense attention across the T frames
    q, k, v, do = (_rand((2, 1, T, d), s) for s in (50, 51, 52, 53))
    got = oracle.monarch_bwd(q, k, v, do, T, 1, 1)
    for a, b in zip(got, _sdpa_grads(q, k, v, do)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_rejects_mismatched_dout():
    q = _rand((1, 1, 8, 4), 1)
    with pytest.raises(ValueError):
        oracle.monarch_bwd(q, q, q, q[:, :, :4], 2, 2, 2)
