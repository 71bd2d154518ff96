"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics,
independent of the oracle's own code.

Which pin catches which plausible mistake:
  * hand-derived golden cases -> wrong stage order, wrong grouping, wrong
    scale, dropped normalisation, tile geometry;
  * single frame (T=1) == library SDPA -> stage-1 attention itself;
  * single position (H=W=1) == library SDPA over frames -> stage-2 attention;
  * brute-force N x N product P^T B2 P B1 built from explicit matrices ->
    any index/permutation error, transposed operand, values of the wrong stage;
  * row-stochastic / positivity / closed form M[x,y] = B2[x,kappa] B1[kappa,y];
  * relabelling (frame permutation, spatial permutation, H<->W transpose);
  * Q=K=0 closed form (global or tile mean of V), V constant, key shift;
  * second independent numpy restatement on the small workloads.
(MonarchRT: Efficient Attention for Real-Time Video Generation,
gist.science/nl/paper/2602.12271 "Methodologie"; gist.science/zh/paper/2602.12271
section 2.2, block alignment and tiled Monarch.)
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from structured_attention_video_monarch_b200 import workloads
from numpy_monarch import monarch_fwd_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _val(x):
    if isinstance(x, str):
        if x == "ln2":
            return math.log(2.0)
        if x == "ln3":
            return math.log(3.0)
        return float(Fraction(x))
    return float(x)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v):
    """Textbook attention from the library (float64, CPU), scale 1/sqrt(d)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy()


# ---------------------------------------------------------------- golden

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_derived_golden(case):
    T, H, W, d = case["T"], case["H"], case["W"], case["d"]
    N = T * H * W
    arr = lambda key: np.array([[_val(x) for x in row] for row in case[key]]).reshape(1, 1, N, d)
    out = oracle.monarch_fwd(arr("q"), arr("k"), arr("v"), T, H, W,
                             case["fact"], case["tile_h"], case["tile_w"])
    np.testing.assert_allclose(out, arr("expected"), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- library special cases

@pytest.mark.parametrize("H,W,d", [(4, 5, 8), (3, 7, 16), (1, 9, 4)])
def test_single_frame_is_dense_attention(H, W, d):
    """T = 1: one stage-1 block holds every token and stage 2 is the identity."""
    q, k, v = (_rand((2, 3, H * W, d), s) for s in (1, 2, 3))
    out = oracle.monarch_fwd(q, k, v, 1, H, W)
    np.testing.assert_allclose(out, _sdpa(q, k, v), rtol=0, atol=1e-13)


@pytest.mark.parametrize("T,d", [(5, 8), (21, 4), (2, 16)])
def test_single_position_is_dense_attention_across_frames(T, d):
    """H = W = 1: stage-1 blocks are single tokens (identity); stage 2 attends over all T."""
    q, k, v = (_rand((1, 2, T, d), s) for s in (4, 5, 6))
    out = oracle.monarch_fwd(q, k, v, T, 1, 1)
    np.testing.assert_allclose(out, _sdpa(q, k, v), rtol=0, atol=1e-13)


def test_stage1_alone_is_blockwise_sdpa():
    T, H, W, d = 3, 2, 5, 8
    q, k, v = (_rand((1, 2, T * H * W, d), s) for s in (7, 8, 9))
    y1 = oracle.monarch_stage1(q, k, v, T, H, W)
    m = H * W
    for t in range(T):
        sl = slice(t * m, (t + 1) * m)
        np.testing.assert_allclose(y1[:, :, sl], _sdpa(q[:, :, sl], k[:, :, sl], v[:, :, sl]),
                                   rtol=0, atol=1e-13)


# ---------------------------------------------------------------- brute force matrices

def _block_softmax(qs, ks, scale):
    return torch.softmax(torch.from_numpy(qs @ ks.T * scale), dim=-1).numpy()


def _explicit_factors(q, k, T, H, W, fact, tile_h, tile_w):
    """Explicit N x N matrices B1, P, B2 for one (batch, head)."""
    N, d = q.shape
    s = 1.0 / math.sqrt(d)
    HW = H * W
    # stage-1 blocks as token lists
    blocks = []
    for t in range(T):
        if fact == 0:
            blocks.append([t * HW + i for i in range(HW)])
        else:
            for ti in range(H // tile_h):
                for tj in range(W // tile_w):
                    blocks.append([t * HW + (ti * tile_h + a) * W + tj * tile_w + b
                                   for a in range(tile_h) for b in range(tile_w)])
    B1 = np.zeros((N, N))
    for blk in blocks:
        B1[np.ix_(blk, blk)] = _block_softmax(q[blk], k[blk], s)
    # P maps token n = t*HW + pos to permuted index pos*T + t
    P = np.zeros((N, N))
    for t in range(T):
        for pos in range(HW):
            P[pos * T + t, t * HW + pos] = 1.0
    qp, kp = P @ q, P @ k
    B2 = np.zeros((N, N))
    for pos in range(HW):
        g = list(range(pos * T, (pos + 1) * T))
        B2[np.ix_(g, g)] = _block_softmax(qp[g], kp[g], s)
    return B1, P, B2


BRUTE_SHAPES = [
    (3, 2, 3, 4, 0, 0, 0),
    (2, 4, 4, 8, 1, 2, 2),
    (4, 3, 4, 6, 1, 3, 2),
    (5, 4, 4, 8, 0, 0, 0),
]


@pytest.mark.parametrize("T,H,W,d,fact,th,tw", BRUTE_SHAPES)
def test_brute_force_effective_matrix(T, H, W, d, fact, th, tw):
    N = T * H * W
    q, k, v = (_rand((1, 1, N, d), s) for s in (10, 11, 12))
    B1, P, B2 = _explicit_factors(q[0, 0], k[0, 0], T, H, W, fact, th, tw)
    M = P.T @ B2 @ P @ B1
    out = oracle.monarch_fwd(q, k, v, T, H, W, fact, th, tw)[0, 0]
    np.testing.assert_allclose(out, M @ v[0, 0], rtol=0, atol=1e-13)
    # row-stochastic with positive entries exactly where a path exists
    np.testing.assert_allclose(M.sum(axis=1), np.ones(N), rtol=0, atol=1e-14)
    assert (M >= 0).all()
    if fact == 0:
        assert (M > 0).all(), "frame split: every (x, y) pair has exactly one path"
        # closed form: M[x,y] = B2[x, kappa] B1[kappa, y], kappa = (t_y, h_x, w_x)
        HW = H * W
        B2o = P.T @ B2 @ P  # B2 in original token order
        for x in range(N):
            for y in range(0, N, 3):
                kappa = (y // HW) * HW + (x % HW)
                assert abs(M[x, y] - B2o[x, kappa] * B1[kappa, y]) < 1e-15
    else:
        HW = H * W
        tile_of = lambda n: (((n % HW) // W) // th, ((n % HW) % W) // tw)
        for x in range(N):
            for y in range(N):
                assert (M[x, y] > 0) == (tile_of(x) == tile_of(y))


# ---------------------------------------------------------------- relabelling

def _grid(x, T, H, W):
    return x.reshape(x.shape[0], x.shape[1], T, H, W, x.shape[-1])


@pytest.mark.parametrize("fact,th,tw", [(0, 0, 0), (1, 2, 3)])
def test_transpose_h_w(fact, th, tw):
    T, H, W, d = 3, 4, 6, 8
    q, k, v = (_rand((1, 2, T * H * W, d), s) for s in (13, 14, 15))
    out = oracle.monarch_fwd(q, k, v, T, H, W, fact, th, tw)
    tr = lambda x: _grid(x, T, H, W).transpose(0, 1, 2, 4, 3, 5).reshape(x.shape)
    out_t = oracle.monarch_fwd(tr(q), tr(k), tr(v), T, W, H, fact, tw, th)
    np.testing.assert_allclose(out_t, tr(out), rtol=0, atol=1e-13)


def test_permute_frames_and_positions():
    T, H, W, d = 4, 3, 5, 8
    q, k, v = (_rand((2, 1, T * H * W, d), s) for s in (16, 17, 18))
    out = oracle.monarch_fwd(q, k, v, T, H, W)
    rng = np.random.default_rng(19)
    fp, pp = rng.permutation(T), rng.permutation(H * W)

    def perm(x):
        g = x.reshape(x.shape[0], x.shape[1], T, H * W, d)
        return g[:, :, fp][:, :, :, pp].reshape(x.shape)

    out_p = oracle.monarch_fwd(perm(q), perm(k), perm(v), T, H, W)
    np.testing.assert_allclose(out_p, perm(out), rtol=0, atol=1e-13)


def test_permute_tiles():
    T, H, W, d, th, tw = 2, 4, 6, 4, 2, 3
    q, k, v = (_rand((1, 1, T * H * W, d), s) for s in (20, 21, 22))
    out = oracle.monarch_fwd(q, k, v, T, H, W, 1, th, tw)
    # swap the two tile rows and reverse frames
    def perm(x):
        g = _grid(x, T, H, W)[:, :, ::-1]
        g = np.concatenate([g[:, :, :, th:], g[:, :, :, :th]], axis=3)
        return np.ascontiguousarray(g).reshape(x.shape)
    out_p = oracle.monarch_fwd(perm(q), perm(k), perm(v), T, H, W, 1, th, tw)
    np.testing.assert_allclose(out_p, perm(out), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- closed forms

def test_zero_qk_gives_global_mean():
    T, H, W, d = 3, 4, 5, 6
    v = _rand((2, 2, T * H * W, d), 23)
    z = np.zeros_like(v)
    out = oracle.monarch_fwd(z, z, v, T, H, W)
    mean = v.mean(axis=2, keepdims=True)
    np.testing.assert_allclose(out, np.broadcast_to(mean, v.shape), rtol=0, atol=1e-13)


def test_zero_qk_tiled_gives_tile_mean():
    T, H, W, d, th, tw = 3, 4, 6, 5, 2, 3
    v = _rand((1, 2, T * H * W, d), 24)
    z = np.zeros_like(v)
    out = _grid(oracle.monarch_fwd(z, z, v, T, H, W, 1, th, tw), T, H, W)
    g = _grid(v, T, H, W)
    for i in range(H // th):
        for j in range(W // tw):
            blk = g[:, :, :, i * th:(i + 1) * th, j * tw:(j + 1) * tw]
            mean = blk.mean(axis=(2, 3, 4))
            got = out[:, :, :, i * th:(i + 1) * th, j * tw:(j + 1) * tw]
            np.testing.assert_allclose(got, np.broadcast_to(mean[:, :, None, None, None], got.shape),
                                       rtol=0, atol=1e-13)


def test_constant_values_pass_through():
    T, H, W, d = 3, 3, 4, 8
    q, k = _rand((1, 2, T * H * W, d), 25), _rand((1, 2, T * H * W, d), 26)
    c = np.linspace(-2, 3, d)
    v = np.broadcast_to(c, q.shape).copy()
    for fact, th, tw in ((0, 0, 0), (1, 3, 2)):
        out = oracle.monarch_fwd(q, k, v, T, H, W, fact, th, tw)
        np.testing.assert_allclose(out, v, rtol=0, atol=1e-13)


def test_key_shift_invariance():
    T, H, W, d = 4, 3, 3, 8
    q, k, v = (_rand((1, 2, T * H * W, d), s) for s in (27, 28, 29))
    shift = _rand((d,), 30)
    base = oracle.monarch_fwd(q, k, v, T, H, W)
    np.testing.assert_allclose(oracle.monarch_fwd(q, k + shift, v, T, H, W), base,
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------- sampled-group mode

@pytest.mark.parametrize("fact,th,tw", [(0, 0, 0), (1, 2, 5)])
def test_group_mode_matches_full(fact, th, tw):
    T, H, W, d = 5, 4, 10, 8
    q, k, v = (_rand((2, 2, T * H * W, d), s) for s in (31, 32, 33))
    full = oracle.monarch_fwd(q, k, v, T, H, W, fact, th, tw).reshape(4, T, H * W, d)
    groups = [(0, 0), (3, 39), (1, 17), (2, 5)]
    rows = oracle.monarch_fwd_groups(q, k, v, T, H, W, groups, fact, th, tw)
    for g, (bh, pos) in enumerate(groups):
        np.testing.assert_allclose(rows[g], full[bh, :, pos], rtol=0, atol=0)


# ---------------------------------------------------------------- independent restatement

@pytest.mark.parametrize("shape", [
    (2, 3, 4, 5, 8, 0, 0, 0),
    (1, 2, 6, 4, 6, 1, 2, 3),
    (1, 1, 7, 2, 3, 1, 2, 1),
])
def test_numpy_restatement_small(shape):
    B, Hd, T, H, W, fact, th, tw = shape
    d = 8
    q, k, v = (_rand((B, Hd, T * H * W, d), s) for s in (34, 35, 36))
    np.testing.assert_allclose(oracle.monarch_fwd(q, k, v, T, H, W, fact, th, tw),
                               monarch_fwd_np(q, k, v, T, H, W, fact, th, tw),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("name,heads", [("tiny_fp32", None), ("chunk_bf16", 2)])
def test_numpy_restatement_workloads(name, heads):
    wl = workloads.BY_NAME[name]
    q, k, v = workloads.generate(wl, heads=heads)
    a = oracle.monarch_fwd(q, k, v, wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w)
    b = monarch_fwd_np(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                       wl.T, wl.H, wl.W, wl.fact, wl.tile_h, wl.tile_w)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_rejects_bad_tiles():
    q = np.zeros((1, 1, 2 * 4 * 6, 4))
    with pytest.raises(ValueError):
        oracle.monarch_fwd(q, q, q, 2, 4, 6, 1, 3, 3)
