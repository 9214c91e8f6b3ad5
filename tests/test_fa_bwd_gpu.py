"""GPU parity of the backward pass (fa_bwd) against the float64 gradient
oracle, on the forward's own bf16 O and lse.

Tolerance: every element of dQ, dK, dV within 2^-6 (1.6 %) of the largest
magnitude of that gradient.  The kernel rounds P and dS to bf16 (relative
2^-9) before the MMAs that consume them, accumulates in fp32 and rounds the
outputs to bf16 (2^-9); D is formed from the bf16 O.  Those errors stay
near 2^-8 of the gradient's scale, and 2^-6 leaves headroom for the sums over
long rows."""

import math

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from exact_attention_120_b200.workloads import WORKLOADS, make_inputs, make_qkv
from fa_helpers import oracle_per_head, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
REL = 2.0 ** -6


def _case(B, H, Nq, Nk, d, seed):
    q, _, _ = make_qkv(B, H, Nq, d, seed)
    _, k, v = make_qkv(B, H, Nk, d, seed + 1)
    g = torch.Generator().manual_seed(seed + 2)
    do = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16)
    return q, k, v, do


def _check(q, k, v, do, causal, mask=None, report=None):
    d = q.shape[-1]
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    md = None if mask is None else mask.to(DEV)
    o, lse = fa.attention_forward(qd, kd, vd, causal=causal, block_mask=md)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, o, lse, dod, causal=causal, block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    ref = oracle.attention_bwd_ref(to_np64(q), to_np64(k), to_np64(v), to_np64(do), 1 / math.sqrt(d),
                                   causal=causal, block_mask=None if mask is None else mask.numpy())
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        got = to_np64(got)
        assert np.all(np.isfinite(got)), name
        err = np.max(np.abs(got - want))
        scale = max(np.max(np.abs(want)), 1e-6)
        if report is not None:
            report.append((name, err, scale))
        assert err <= REL * scale, f"{name}: max|d| {err:.3e} > {REL} x {scale:.3e}"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [128, 300, 513])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_shapes(d, N, causal):
    _check(*_case(2, 2, N, N, d, seed=N + d), causal)


@pytest.mark.parametrize("nq,nk", [(200, 700), (640, 300), (1, 1000)])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_qk_lengths(nq, nk, causal):
    _check(*_case(1, 2, nq, nk, 64, seed=nq + nk), causal)


def test_bwd_block_sparse():
    B, H, N, d = 2, 2, 700, 128
    q, k, v, do = _case(B, H, N, N, d, seed=31)
    g = torch.Generator().manual_seed(32)
    nb = (N + 127) // 128
    mask = (torch.rand((B, H, nb, nb), generator=g) < 0.4).to(torch.uint8)
    mask |= torch.eye(nb, dtype=torch.uint8)
    for causal in (False, True):
        _check(q, k, v, do, causal, mask)


def test_bwd_longer_sequence():
    _check(*_case(1, 4, 2048, 2048, 128, seed=41), True)


def test_bwd_long_full_shape_two_heads_every_row():
    # The backward in the configuration bench.py --pass bwd times: the long
    # full-attention workload (B=1, H=16, N=16384, d=128, Q/K std 3) with the
    # bench's seeded dO, on all 16 heads.  Heads 0 and 15 are compared with the
    # float64 gradient oracle on every row of dQ, dK and dV.
    w = WORKLOADS["long_full"]
    q, k, v, _ = make_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 7)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    o, lse = fa.attention_forward(qd, kd, vd)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, o, lse, dod)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    heads = [(0, 0), (0, w.H - 1)]
    got = [tuple(to_np64(t[b, h]) for t in (dq, dk, dv)) for b, h in heads]
    del qd, kd, vd, dod, o, lse, dq, dk, dv

    def one(b, h):
        sl = lambda t: to_np64(t[b:b + 1, h:h + 1])  # noqa: E731
        return oracle.attention_bwd_ref(sl(q), sl(k), sl(v), sl(do), w.scale)

    refs = oracle_per_head(one, heads)
    for (b, h), g3, r3 in zip(heads, got, refs):
        for name, gt, want in zip(("dq", "dk", "dv"), g3, r3):
            want = want[0, 0]
            assert np.all(np.isfinite(gt)), (name, h)
            err = np.max(np.abs(gt - want))
            scale = max(np.max(np.abs(want)), 1e-6)
            assert err <= REL * scale, f"head {h} {name}: max|d| {err:.3e} > {REL} x {scale:.3e}"


@pytest.mark.parametrize("name", ["mid_causal", "sparse"])
def test_bwd_bench_shapes_two_heads_every_row(name):
    # The backward of the causal and block-sparse workloads in the
    # configuration bench.py --pass bwd --workload NAME times (all heads, the
    # bench's seeded dO); two heads compared on every row of dQ, dK and dV.
    w = WORKLOADS[name]
    q, k, v, mask = make_inputs(w)
    g = torch.Generator().manual_seed(w.seed + 7)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    md = None if mask is None else mask.to(DEV)
    o, lse = fa.attention_forward(qd, kd, vd, causal=w.causal, block_mask=md)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, o, lse, dod, causal=w.causal, block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    got = [tuple(to_np64(t[b, h]) for t in (dq, dk, dv)) for b, h in heads]

    def one(b, h):
        sl = lambda t: to_np64(t[b:b + 1, h:h + 1])  # noqa: E731
        bm = None if mask is None else mask[b:b + 1, h:h + 1].numpy()
        return oracle.attention_bwd_ref(sl(q), sl(k), sl(v), sl(do), w.scale, causal=w.causal, block_mask=bm)

    refs = oracle_per_head(one, heads)
    for (b, h), g3, r3 in zip(heads, got, refs):
        for gname, gt, want in zip(("dq", "dk", "dv"), g3, r3):
            want = want[0, 0]
            assert np.all(np.isfinite(gt)), (gname, b, h)
            err = np.max(np.abs(gt - want))
            scale = max(np.max(np.abs(want)), 1e-6)
            assert err <= REL * scale, f"({b},{h}) {gname}: max|d| {err:.3e} > {REL} x {scale:.3e}"
