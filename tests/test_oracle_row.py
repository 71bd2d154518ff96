"""Pins for the oracle's (f*h, w) split (FACT_ROW), the aligned block choice
(b1, b2) = (f*h, w) that the pages give as their example (pt page,
"Alinhamento de Blocos"; zh page, section 2.2): the N tokens form a
(T*H) x W grid; stage-1 blocks are its rows (the W tokens of one frame row),
stage-2 groups its columns (the T*H tokens sharing a column w).

  * brute-force N x N product P^T B2 P B1 from explicit matrices, and the
    closed form M[x, y] = B2[x, kappa] B1[kappa, y], kappa = (row of y,
    column of x) -> any block, group or permutation error;
  * H = 1 makes it the frame split; W = 1 and T = H = 1 reduce it to dense
    attention (library SDPA);
  * relabelling of columns and of frame rows;
  * gradients: dV = M^T dO and finite differences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import _block_softmax, _rand, _sdpa

ROW = oracle.FACT_ROW


def _row_factors(q, k, T, H, W):
    N, d = q.shape
    s = 1.0 / math.sqrt(d)
    R = T * H  # grid rows
    B1 = np.zeros((N, N))
    for r in range(R):
        blk = list(range(r * W, (r + 1) * W))
        B1[np.ix_(blk, blk)] = _block_softmax(q[blk], k[blk], s)
    # P maps token n = r*W + c to c*R + r (column-major grid order)
    P = np.zeros((N, N))
    for r in range(R):
        for c in range(W):
            P[c * R + r, r * W + c] = 1.0
    qp, kp = P @ q, P @ k
    B2 = np.zeros((N, N))
    for c in range(W):
        g = list(range(c * R, (c + 1) * R))
        B2[np.ix_(g, g)] = _block_softmax(qp[g], kp[g], s)
    return B1, P, B2


@pytest.mark.parametrize("T,H,W,d", [(2, 3, 4, 4), (3, 2, 5, 8), (1, 4, 3, 6)])
def test_brute_force_effective_matrix(T, H, W, d):
    N = T * H * W
    q, k, v = (_rand((1, 1, N, d), s) for s in (60, 61, 62))
    B1, P, B2 = _row_factors(q[0, 0], k[0, 0], T, H, W)
    M = P.T @ B2 @ P @ B1
    out = oracle.monarch_fwd(q, k, v, T, H, W, ROW)[0, 0]
    np.testing.assert_allclose(out, M @ v[0, 0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(M.sum(axis=1), np.ones(N), rtol=0, atol=1e-14)
    assert (M > 0).all(), "aligned split: every (x, y) pair has exactly one path"
    B2o = P.T @ B2 @ P
    for x in range(N):
        for y in range(N):
            kappa = (y // W) * W + (x % W)
            assert abs(M[x, y] - B2o[x, kappa] * B1[kappa, y]) < 1e-15


def test_single_row_height_is_the_frame_split():
    T, H, W, d = 4, 1, 6, 8
    q, k, v = (_rand((2, 1, T * H * W, d), s) for s in (63, 64, 65))
    np.testing.assert_allclose(oracle.monarch_fwd(q, k, v, T, H, W, ROW),
                               oracle.monarch_fwd(q, k, v, T, H, W), rtol=0, atol=1e-14)


def test_single_column_is_dense_attention():
    T, H, d = 3, 4, 8  # W = 1: stage 1 is the identity, stage 2 spans all tokens
    q, k, v = (_rand((1, 2, T * H, d), s) for s in (66, 67, 68))
    np.testing.assert_allclose(oracle.monarch_fwd(q, k, v, T, H, 1, ROW), _sdpa(q, k, v), rtol=0,
                               atol=1e-13)


def test_single_row_is_dense_attention():
    W, d = 9, 8  # T = H = 1: stage 1 spans all tokens, stage 2 groups are single tokens
    q, k, v = (_rand((1, 2, W, d), s) for s in (69, 70, 71))
    np.testing.assert_allclose(oracle.monarch_fwd(q, k, v, 1, 1, W, ROW), _sdpa(q, k, v), rtol=0,
                               atol=1e-13)


def test_relabel_columns_and_rows():
    T, H, W, d = 2, 3, 5, 4
    R = T * H
    q, k, v = (_rand((1, 1, R * W, d), s) for s in (72, 73, 74))
    out = oracle.monarch_fwd(q, k, v, T, H, W, ROW)
    rng = np.random.default_rng(3)
    cp, rp = rng.permutation(W), rng.permutation(R)

    def perm(x):
        g = x.reshape(1, 1, R, W, d)
        return g[:, :, rp][:, :, :, cp].reshape(x.shape)

    np.testing.assert_allclose(oracle.monarch_fwd(perm(q), perm(k), perm(v), T, H, W, ROW), perm(out),
                               rtol=0, atol=1e-13)


def test_value_gradient_is_monarch_transpose():
    T, H, W, d = 2, 3, 4, 4
    N = T * H * W
    q, k, v, do = (_rand((1, 1, N, d), s) for s in (75, 76, 77, 78))
    B1, P, B2 = _row_factors(q[0, 0], k[0, 0], T, H, W)
    M = P.T @ B2 @ P @ B1
    _, _, dv = oracle.monarch_bwd(q, k, v, do, T, H, W, ROW)
    np.testing.assert_allclose(dv[0, 0], M.T @ do[0, 0], rtol=0, atol=1e-12)


def test_finite_differences():
    T, H, W, d = 2, 2, 3, 4
    shape = (1, 2, T * H * W, d)
    q, k, v, do = (_rand(shape, s) for s in (80, 81, 82, 83))
    grads = dict(zip("qkv", oracle.monarch_bwd(q, k, v, do, T, H, W, ROW)))
    x = {"q": q, "k": k, "v": v}
    loss = lambda: float(np.sum(do * oracle.monarch_fwd(x["q"], x["k"], x["v"], T, H, W, ROW)))
    rng = np.random.default_rng(9)
    h = 1e-5
    for name in "qkv":
        for _ in range(10):
            idx = tuple(int(rng.integers(n)) for n in shape)
            keep = x[name][idx]
            x[name][idx] = keep + h
            up = loss()
            x[name][idx] = keep - h
            down = loss()
            x[name][idx] = keep
            fd = (up - down) / (2 * h)
            assert abs(fd - grads[name][idx]) < 1e-7 * max(1.0, abs(fd)), (name, idx, fd, grads[name][idx])


def test_sampled_group_mode_refuses_the_row_split():
    q = _rand((1, 1, 12, 4), 1)
    with pytest.raises(ValueError):
        oracle.monarch_fwd_groups(q, q, q, 2, 2, 3, [(0, 0)], ROW)


@pytest.mark.parametrize("T,H,W", [(2, 3, 5), (3, 4, 2), (1, 6, 7)])
def test_row_split_is_the_frame_split_of_the_row_grid(T, H, W):
    # the (f*h, w) split of a T x H x W grid is the frame split of a (T*H) x 1 x W
    # grid: its blocks (frame rows) are those frames, its groups (columns) those positions
    d = 6
    q, k, v = (_rand((1, 2, T * H * W, d), s) for s in (91, 92, 93))
    np.testing.assert_allclose(oracle.monarch_fwd(q, k, v, T, H, W, oracle.FACT_ROW),
                               oracle.monarch_fwd(q, k, v, T * H, 1, W, oracle.FACT_FRAME), rtol=0, atol=1e-14)
    g = _rand((1, 2, T * H * W, d), 94)
    for a, b in zip(oracle.monarch_bwd(q, k, v, g, T, H, W, oracle.FACT_ROW),
                    oracle.monarch_bwd(q, k, v, g, T * H, 1, W, oracle.FACT_FRAME)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
