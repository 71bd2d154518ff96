"""Second, independently written fp64 restatement of the Monarch attention
forward, vectorised with numpy.  Test-only: used to cross-check the C oracle.

Where the C oracle walks token lists with loops, this version applies the
permutation P as an explicit reshape/transpose of the token axis:
  [T, H, W] --(stage-1 blocks)--> attention over each frame's (or tile's) tokens
  P: move the frame axis next to the feature axis -> groups [H*W, T]
  stage-2 attention over each group, then P^T moves the axes back.
(MonarchRT: Efficient Attention for Real-Time Video Generation,
gist.science/nl/paper/2602.12271, "Methodologie".)
"""
import numpy as np


def _softmax_attn(q, k, v, scale):
    """Batched softmax attention over the second-to-last axis."""
    logits = np.einsum("...id,...jd->...ij", q, k) * scale
    logits -= logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    w /= w.sum(axis=-1, keepdims=True)
    return np.einsum("...ij,...jd->...id", w, v)


def monarch_fwd_np(q, k, v, T, H, W, fact=0, tile_h=0, tile_w=0):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hd, N, d = q.shape
    s = 1.0 / np.sqrt(d)
    grid = (B, Hd, T, H, W, d)
    qg, kg, vg = q.reshape(grid), k.reshape(grid), v.reshape(grid)
    if fact == 0:
        # stage-1 blocks: one frame each, H*W tokens
        blk = lambda x: x.reshape(B, Hd, T, H * W, d)
        y1 = _softmax_attn(blk(qg), blk(kg), blk(vg), s).reshape(grid)
    else:
        th, tw = H // tile_h, W // tile_w
        # [B, Hd, T, th, tile_h, tw, tile_w, d] -> [B, Hd, T, th, tw, tile_h*tile_w, d]
        def blk(x):
            x = x.reshape(B, Hd, T, th, tile_h, tw, tile_w, d)
            return x.transpose(0, 1, 2, 3, 5, 4, 6, 7).reshape(B, Hd, T, th, tw, tile_h * tile_w, d)
        y = _softmax_attn(blk(qg), blk(kg), blk(vg), s)
        y1 = (y.reshape(B, Hd, T, th, tw, tile_h, tile_w, d)
               .transpose(0, 1, 2, 3, 5, 4, 6, 7).reshape(grid))
    # P: frames become the in-group axis; groups are spatial positions
    perm = lambda x: x.reshape(B, Hd, T, H * W, d).transpose(0, 1, 3, 2, 4)
    o = _softmax_attn(perm(qg), perm(kg), perm(y1), s)          # [B, Hd, HW, T, d]
    return o.transpose(0, 1, 3, 2, 4).reshape(B, Hd, N, d)     # P^T
