"""GPU: the library's own device buffers stay bounded and correctly ordered.

The bf16 / fp16 path draws its per-batch-head completion counters from a
fixed pool of slots per device, and the (f*h, w) split its Y1 scratch from one
buffer per device; a stream that takes over a slot or the scratch waits for
the previous user's last launch on the device (an event), not on the host.
These tests call through the C ABI on many short-lived streams and check that
device memory does not grow with the number of streams and that every result
equals the one computed on the default stream.
"""
import ctypes

import pytest
import torch

from structured_attention_video_monarch_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _rt():
    from cuda.bindings import runtime as rt
    return rt


def _new_stream():
    rt = _rt()
    err, s = rt.cudaStreamCreateWithFlags(rt.cudaStreamNonBlocking)
    assert int(err) == 0
    return s


def _handle(s) -> int:
    return int(s)


def _destroy(s):
    rt = _rt()
    assert int(rt.cudaStreamSynchronize(s)[0]) == 0
    assert int(rt.cudaStreamDestroy(s)[0]) == 0


def _call(lib, q, k, v, out, T, H, W, fact, th, tw, stream_handle):
    B, heads, N, d = q.shape
    st = lib.monarch_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, heads, T, H, W, d,
                              fact, th, tw, binding.DTYPE_BF16, ctypes.c_void_p(stream_handle))
    assert st == 0, binding.strerror(st)


@pytest.mark.parametrize("fact,T,H,W,th,tw", [(0, 3, 12, 20, 0, 0), (2, 3, 6, 40, 0, 0)], ids=["frame", "row"])
def test_many_fresh_streams_bounded_memory(fact, T, H, W, th, tw):
    dev = torch.device("cuda:0")
    lib = binding.load_library()
    q, k, v = (x.to(dev) for x in workloads.random_inputs(2, 3, T, H, W, 128, seed=11))
    ref = binding.monarch_attn_fwd(q, k, v, T, H, W, fact, th, tw)
    outs = [torch.full_like(q, float("nan")) for _ in range(8)]
    torch.cuda.synchronize()
    # first calls on a few streams: the pools exist after these
    for i in range(2):
        s = _new_stream()
        _call(lib, q, k, v, outs[i], T, H, W, fact, th, tw, _handle(s))
        _destroy(s)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for i in range(80):  # more streams than the counter pool has slots
        s = _new_stream()
        o = outs[i % len(outs)]
        o.fill_(float("nan"))
        torch.cuda.synchronize()
        _call(lib, q, k, v, o, T, H, W, fact, th, tw, _handle(s))
        _destroy(s)
        assert torch.equal(o, ref), f"stream {i}"
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free0 - free1 <= 2 * 2**20, f"device memory grew by {(free0 - free1) / 2**20:.1f} MiB"
    assert binding.last_device_error() == 0


def test_interleaved_streams_share_pools_in_order():
    """Two long-lived streams queue calls back to back without host syncs; the
    row split shares one Y1 scratch between them, so the second stream must be
    ordered after the first one's launches."""
    dev = torch.device("cuda:0")
    lib = binding.load_library()
    T, H, W = 4, 6, 40
    q, k, v = (x.to(dev) for x in workloads.random_inputs(1, 4, T, H, W, 128, seed=12))
    q2, k2, v2 = (x.to(dev) for x in workloads.random_inputs(1, 4, T, H, W, 128, seed=13))
    ref = binding.monarch_attn_fwd(q, k, v, T, H, W, 2)
    ref2 = binding.monarch_attn_fwd(q2, k2, v2, T, H, W, 2)
    torch.cuda.synchronize()
    s1, s2 = _new_stream(), _new_stream()
    outs = []
    for i in range(6):
        a, b = torch.full_like(q, float("nan")), torch.full_like(q, float("nan"))
        torch.cuda.synchronize()
        _call(lib, q, k, v, a, T, H, W, 2, 0, 0, _handle(s1))
        _call(lib, q2, k2, v2, b, T, H, W, 2, 0, 0, _handle(s2))
        outs.append((a, b))
    _destroy(s1)
    _destroy(s2)
    torch.cuda.synchronize()
    for a, b in outs:
        assert torch.equal(a, ref) and torch.equal(b, ref2)


def test_counter_pool_grows_for_many_batch_heads():
    """More batch-heads than the counter pool's first slot size (4096 plus the
    unit-claim counter): the pool is reallocated larger, earlier slots retired,
    and the result still matches the oracle."""
    import oracle
    dev = torch.device("cuda:0")
    B, heads, T, H, W, d = 2, 2500, 2, 1, 3, 64
    q, k, v = workloads.random_inputs(B, heads, T, H, W, d, seed=21)
    got = binding.monarch_attn_fwd(*(x.to(dev) for x in (q, k, v)), T, H, W)
    torch.cuda.synchronize()
    assert binding.last_device_error() == 0
    ref = oracle.monarch_fwd(q, k, v, T, H, W)
    err = (got.cpu().double() - torch.from_numpy(ref)).abs().max().item()
    assert err <= 2e-2
