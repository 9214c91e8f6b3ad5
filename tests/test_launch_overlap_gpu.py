"""Launch overlap (programmatic dependent launch) keeps stream order.

Every kernel of the library may start its prologue while the previous kernel
on the stream finishes, and touches global memory only after that kernel has
completed.  These tests chain calls whose inputs are the previous call's
outputs (O of one forward is the Q of the next, the backward reads the
forward's O and lse) on one stream, directly and replayed from a captured CUDA
graph, and compare every result with the same chain run with a device
synchronisation between the calls.
"""

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
from exact_attention_120_b200.workloads import make_qkv
from fa_helpers import to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _chain(q, k, v, steps, causal, sync):
    outs = []
    x = q
    for _ in range(steps):
        o, lse = fa.attention_forward(x, k, v, causal=causal)
        if sync:
            torch.cuda.synchronize()
        outs.append((o, lse))
        x = o
    return outs


@pytest.mark.parametrize("shape", [(1, 1, 128, 64), (4, 8, 1024, 64), (2, 4, 2048, 128)])
def test_chained_forwards_match_synchronised_chain(shape):
    B, H, N, d = shape
    q, k, v = (t.to(DEV) for t in make_qkv(B, H, N, d, seed=N + d))
    ref = _chain(q, k, v, 4, True, sync=True)
    got = _chain(q, k, v, 4, True, sync=False)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    for (o1, l1), (o2, l2) in zip(got, ref):
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_forward_then_backward_back_to_back():
    B, H, N, d = 2, 4, 700, 128
    q, k, v = (t.to(DEV) for t in make_qkv(B, H, N, d, seed=5))
    g = torch.Generator().manual_seed(6)
    do = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).to(DEV)
    o, lse = fa.attention_forward(q, k, v, causal=True)
    got = fa.attention_backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    o2, lse2 = fa.attention_forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    ref = fa.attention_backward(q, k, v, o2, lse2, do, causal=True)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_graph_replay_of_a_chain():
    B, H, N, d = 4, 8, 1024, 64
    q, k, v = (t.to(DEV) for t in make_qkv(B, H, N, d, seed=9))
    ref = _chain(q, k, v, 3, False, sync=True)
    o_bufs = [torch.empty_like(q) for _ in range(3)]
    l_bufs = [torch.empty((B, H, N), device=DEV) for _ in range(3)]
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        fa.attention_forward(q, k, v, out=o_bufs[0], lse=l_bufs[0])  # set-up outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        x = q
        for i in range(3):
            fa.attention_forward(x, k, v, out=o_bufs[i], lse=l_bufs[i])
            x = o_bufs[i]
    for buf in o_bufs:
        buf.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    for (o_ref, l_ref), o, l in zip(ref, o_bufs, l_bufs):
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
    assert np.isfinite(to_np64(o_bufs[-1])).all()
