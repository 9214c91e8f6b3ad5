"""GPU parity of the 8-bit forward (fa_fwd_fp8) against the float64 oracle on
the real values the E4M3 codes stand for.

Bar, derived from the arithmetic: the kernel rounds P to e4m3 (relative
error u = 2^-4) and normalises by the sum of those same rounded values, so
each O row is an exact weighted mean of V rows with weights perturbed by at
most u relative.  That moves O_it by at most u / (1 - u) times the weighted
spread of V (oracle.weighted_spread).  On top: the bf16 output rounding
(2^-9 |O|, taken as 2^-8 |O|) and an absolute 2^-9 max|V| for P values
that fall into e4m3's subnormal range, where the relative bound does not
hold.  lse: the row sum is off by at most u relative, |dlse| <= ln(1 + u).
"""

import math

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from exact_attention_120_b200.workloads import make_block_mask, make_qkv_fp8
from fa_helpers import oracle_per_head, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
U = 2.0 ** -4


def _check(B, H, N, causal, seed, Nk=None, mask=None, qk_std=1.0, report=None):
    d = 128
    Nk = N if Nk is None else Nk
    (q8, k8, v8), (qd, kd, vd) = make_qkv_fp8(B, H, N, d, seed, qk_std=qk_std, Nk=Nk)
    md = None if mask is None else mask.to(DEV)
    o, lse = fa.attention_forward_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), qd, kd, vd, causal=causal,
                                      block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    o, lse = to_np64(o), to_np64(lse)
    scale = 1.0 / math.sqrt(d)
    mnp = None if mask is None else mask.numpy()
    qf = oracle.e4m3_decode(q8.numpy()) * qd
    kf = oracle.e4m3_decode(k8.numpy()) * kd
    vf = oracle.e4m3_decode(v8.numpy()) * vd
    o_ref, lse_ref = oracle.attention_ref(qf, kf, vf, scale, causal=causal, block_mask=mnp)
    spread = oracle.weighted_spread(qf, kf, vf, scale, causal=causal, block_mask=mnp)
    bound = U / (1 - U) * spread + 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -9 * np.max(np.abs(vf))
    assert np.all(np.isfinite(o))
    excess = np.abs(o - o_ref) - bound
    assert np.max(excess) <= 0, f"O outside the bound by {np.max(excess):.3e}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    dl = np.max(np.abs(lse[fin] - lse_ref[fin])) if fin.any() else 0.0
    assert dl <= math.log1p(U), f"max|dlse| = {dl:.3e}"
    if report is not None:
        report.append((np.max(np.abs(o - o_ref)), np.sqrt(np.mean((o - o_ref) ** 2)), dl))


@pytest.mark.parametrize("N", [1, 127, 128, 300, 513])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_shapes(N, causal):
    _check(2, 2, N, causal, seed=N)


@pytest.mark.parametrize("nq,nk", [(200, 700), (640, 300), (1, 1000)])
def test_fp8_qk_lengths(nq, nk):
    _check(1, 2, nq, True, seed=nq + nk, Nk=nk)


def test_fp8_block_sparse():
    N = 700
    mask = make_block_mask(2, 2, N, 0.4, 3)
    _check(2, 2, N, True, seed=8, mask=mask)
    _check(2, 2, N, False, seed=9, mask=mask)


def test_fp8_wide_scores():
    # Q, K std 3: nearly one-hot rows, many P values in e4m3's subnormal range.
    _check(1, 2, 1024, False, seed=12, qk_std=3.0)


def test_fp8_long_workload_every_row():
    # The inputs bench.py --pass fp8 times (the long workload: B=1, H=16,
    # N=16384, d=128, Q/K std 3, seed 3), every row of every head against the
    # bound above.  The oracle and the weighted spread run per head in chunks
    # of 1024 complete query rows (full attention, so a row's result needs
    # only its own row of scores), one thread-pool task per head.
    B, H, N, d = 1, 16, 16384, 128
    (q8, k8, v8), (qd, kd, vd) = make_qkv_fp8(B, H, N, d, 3, qk_std=3.0, v_std=1.0)
    o, lse = fa.attention_forward_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), qd, kd, vd)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    o, lse = to_np64(o), to_np64(lse)
    qf = oracle.e4m3_decode(q8.numpy()) * qd
    kf = oracle.e4m3_decode(k8.numpy()) * kd
    vf = oracle.e4m3_decode(v8.numpy()) * vd
    vmax = float(np.max(np.abs(vf)))
    scale = 1.0 / math.sqrt(d)

    def one(b, h):
        worst_o, worst_l = -np.inf, 0.0
        for r0 in range(0, N, 1024):
            sl = (slice(b, b + 1), slice(h, h + 1), slice(r0, r0 + 1024))
            qs, ks, vs = qf[sl], kf[b:b + 1, h:h + 1], vf[b:b + 1, h:h + 1]
            o_ref, lse_ref = oracle.attention_ref(qs, ks, vs, scale)
            spread = oracle.weighted_spread(qs, ks, vs, scale)
            bound = U / (1 - U) * spread + 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -9 * vmax
            worst_o = max(worst_o, float(np.max(np.abs(o[sl] - o_ref) - bound)))
            worst_l = max(worst_l, float(np.max(np.abs(lse[sl] - lse_ref))))
        return worst_o, worst_l

    res = oracle_per_head(one, [(0, h) for h in range(H)])
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    worst_o = max(r[0] for r in res)
    worst_l = max(r[1] for r in res)
    assert worst_o <= 0, f"O outside the bound by {worst_o:.3e}"
    assert worst_l <= math.log1p(U), f"max|dlse| = {worst_l:.3e}"


def test_fp8_argument_errors():
    q = torch.zeros((1, 1, 128, 128), dtype=torch.uint8, device=DEV)
    o = torch.empty((1, 1, 128, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, 1, 128), dtype=torch.float32, device=DEV)
    lib = fa.load_library()
    base = [q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 1, 128, 128,
            128, 0.1, 0, None, 1.0, 1.0, 1.0, None]
    for i, val in {13: 0.0, 14: -1.0, 15: float("inf")}.items():
        a = list(base)
        a[i] = val
        assert lib.fa_fwd_fp8(*a) == fa.FA_ERR_INVALID_ARGUMENT, i
    a = list(base)
    a[9] = 64
    assert lib.fa_fwd_fp8(*a) == fa.FA_ERR_UNSUPPORTED
