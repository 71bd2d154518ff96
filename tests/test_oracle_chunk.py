"""Pins for the oracle's autoregressive chunk form (oracle_monarch_fwd_chunk):
a chunk of new frames with the earlier frames' keys and stage-1 outputs as
context.

  * the last chunk equals the full forward's rows for its frames, with the
    context computed by the full forward's stage 1 (frame and tiled splits)
    -> catches misplaced cache rows, a missing context frame, values taken
    from V instead of Y1;
  * no context (T_old = 0) is the plain forward over the chunk;
  * the chunk's own stage-1 output is the stage-1 output of those frames.
"""
import numpy as np
import pytest

import oracle
from test_oracle_pins import _rand

CASES = [
    # B, heads, T_old, T_new, H, W, d, fact, tile_h, tile_w
    (1, 2, 4, 2, 3, 4, 8, 0, 0, 0),
    (2, 1, 1, 3, 2, 5, 4, 0, 0, 0),
    (1, 1, 3, 1, 4, 4, 6, 1, 2, 2),
]


def _split(x, T_old, HW):
    return x[:, :, :T_old * HW], x[:, :, T_old * HW:]


@pytest.mark.parametrize("B,heads,T_old,T_new,H,W,d,fact,th,tw", CASES)
def test_last_chunk_equals_full_forward_rows(B, heads, T_old, T_new, H, W, d, fact, th, tw):
    T, HW = T_old + T_new, H * W
    q, k, v = (_rand((B, heads, T * HW, d), s) for s in (90, 91, 92))
    full = oracle.monarch_fwd(q, k, v, T, H, W, fact, th, tw)
    y1_all = oracle.monarch_stage1(q, k, v, T, H, W, fact, th, tw)
    k_old, k_new = _split(k, T_old, HW)
    y1_old, y1_tail = _split(y1_all, T_old, HW)
    out, y1_new = oracle.monarch_fwd_chunk(_split(q, T_old, HW)[1], k_new, _split(v, T_old, HW)[1], k_old,
                                           y1_old, T_old, T_new, H, W, fact, th, tw)
    np.testing.assert_allclose(out, full[:, :, T_old * HW:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(y1_new, y1_tail, rtol=0, atol=1e-14)


def test_no_context_is_the_plain_forward():
    B, heads, T, H, W, d = 1, 2, 3, 3, 4, 8
    q, k, v = (_rand((B, heads, T * H * W, d), s) for s in (93, 94, 95))
    out, y1 = oracle.monarch_fwd_chunk(q, k, v, None, None, 0, T, H, W)
    np.testing.assert_allclose(out, oracle.monarch_fwd(q, k, v, T, H, W), rtol=0, atol=1e-14)
    np.testing.assert_allclose(y1, oracle.monarch_stage1(q, k, v, T, H, W), rtol=0, atol=1e-14)


def test_rejects_the_row_split_and_bad_context():
    q = _rand((1, 1, 2 * 2 * 3, 4), 1)
    with pytest.raises(ValueError):
        oracle.monarch_fwd_chunk(q, q, q, None, None, 0, 2, 2, 3, oracle.FACT_ROW)
    with pytest.raises(ValueError):
        oracle.monarch_fwd_chunk(q, q, q, q[:, :, :6], q, 1, 2, 2, 3)


def test_chunk_workload_context_and_counts():
    from structured_attention_video_monarch_b200 import workloads
    wl = workloads.BY_NAME["chunk_ar_bf16"]
    assert (wl.T, wl.T_ctx, wl.H, wl.W, wl.heads, wl.d) == (3, 18, 30, 52, 12, 128)
    kc, yc = workloads.generate_context(wl, heads=1)
    assert kc.shape == yc.shape == (1, 1, 18 * 30 * 52, 128)
    kc2, _ = workloads.generate_context(wl, heads=1)
    assert (kc.float() == kc2.float()).all()  # seeded
    # per query: m stage-1 keys and T_ctx + T stage-2 keys, 4*d flops each
    assert wl.flops == 4.0 * wl.N * (wl.H * wl.W + 21) * wl.d * wl.heads
    # read Q, K, V and the context's K and Y1; write out and the new Y1
    assert wl.io_bytes == (5 * wl.N + 2 * 18 * 30 * 52) * wl.heads * wl.d * 2
