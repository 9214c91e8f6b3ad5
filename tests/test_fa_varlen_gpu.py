"""GPU parity of variable-length batches (fa_fwd_varlen) against the float64
oracle, element by element, at the forward's bar (max|dO| <= 2e-2,
max|dlse| <= 1e-2, absolute)."""

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from exact_attention_120_b200.workloads import VARLEN_WORKLOADS, make_varlen, make_varlen_inputs
from fa_helpers import TOL_LSE, TOL_O, assert_lse_close, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _run(q, k, v, cu_q, cu_k, causal, max_q=None):
    lq = (cu_q[1:] - cu_q[:-1]).tolist()
    max_q = max(max(lq), 1) if max_q is None else max_q
    o, lse = fa.attention_forward_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV), cu_k.to(DEV),
                                         max_q, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    return to_np64(o), to_np64(lse)


def _check(lq, lk, d, causal, seed, H=2):
    q, k, v, cu_q, cu_k = make_varlen(lq, lk, H, d, seed)
    o, lse = _run(q, k, v, cu_q, cu_k, causal)
    scale = 1.0 / np.sqrt(d)
    o_ref, lse_ref = oracle.attention_varlen_ref(to_np64(q), to_np64(k), to_np64(v), cu_q.tolist(),
                                                 cu_k.tolist(), scale, causal=causal)
    assert np.all(np.isfinite(o))
    err = np.max(np.abs(o - o_ref)) if o.size else 0.0
    assert err <= TOL_O, f"max|dO| = {err:.3e}"
    assert_lse_close(lse, lse_ref, TOL_LSE)


MIXES = [
    ([1, 127, 128, 129, 300, 513], None),
    ([200, 5, 0, 640, 1], [700, 300, 10, 128, 1]),   # nq != nk, an empty query sequence
    ([64, 300], [0, 257]),                            # a sequence without keys
    ([1000], [1000]),
    ([17, 256, 255, 1, 384], [1024, 3, 255, 900, 128]),
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mix", range(len(MIXES)))
def test_varlen_mixes(d, causal, mix):
    lq, lk = MIXES[mix]
    _check(lq, lq if lk is None else lk, d, causal, seed=10 * mix + d)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_dense_bitwise(causal):
    # Equal lengths that are whole tiles: the packed layout must give exactly
    # the dense kernel's bits (same tiles, same order of operations).
    B, H, N, d = 3, 4, 384, 128
    q, k, v, cu_q, cu_k = make_varlen([N] * B, [N] * B, H, d, seed=7)
    o, lse = _run(q, k, v, cu_q, cu_k, causal)
    to_dense = lambda t: t.view(B, N, H, d).permute(0, 2, 1, 3).contiguous().to(DEV)  # noqa: E731
    od, ld = fa.attention_forward(to_dense(q), to_dense(k), to_dense(v), causal=causal)
    torch.cuda.synchronize()
    od = to_np64(od).transpose(0, 2, 1, 3).reshape(B * N, H, d)
    ld = to_np64(ld).transpose(1, 0, 2).reshape(H, B * N)
    assert np.array_equal(o, od)
    assert np.array_equal(lse, ld)


def test_varlen_workload_full_size():
    # The benchmark's length mix (32 sequences, 128..8192 tokens, H=16, d=128,
    # causal), compared on every row of every sequence for two heads.
    w = VARLEN_WORKLOADS["varlen_mix"]
    lens, q, k, v, cu_q, cu_k = make_varlen_inputs(w)
    o, lse = _run(q, k, v, cu_q, cu_k, w.causal)
    for h in (0, w.H - 1):
        qh, kh, vh = (to_np64(t[:, h:h + 1]) for t in (q, k, v))
        o_ref, lse_ref = oracle.attention_varlen_ref(qh, kh, vh, cu_q.tolist(), cu_k.tolist(), w.scale,
                                                     causal=w.causal)
        err = np.max(np.abs(o[:, h:h + 1] - o_ref))
        assert err <= TOL_O, f"head {h}: max|dO| = {err:.3e}"
        assert_lse_close(lse[h:h + 1], lse_ref, TOL_LSE)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_more_sequences_than_one_launch(causal):
    # 4396 short sequences (0 to 300 tokens, empty ones among them): more
    # than the 4096 one launch deals, so the call takes two launches, the
    # second starting 4096 entries into the offsets.
    g = torch.Generator().manual_seed(31)
    lq = torch.randint(0, 301, (4396,), generator=g)
    lq[::97] = 0
    lq = lq.tolist()
    _check(lq, lq, 64, causal, seed=33, H=1)


def test_varlen_heads_split_into_l2_groups():
    # A causal sequence long enough that the K/V of all 16 heads exceed the
    # L2 share of one head group (15 heads of 6200 keys fit, the 16th starts a
    # group of one), next to short and empty sequences.
    _check([6200, 150, 0, 700], [6200, 150, 0, 700], 128, True, seed=35, H=16)


def test_varlen_understated_max_length():
    # max_seqlen_q only sizes the launch: a bound below the real lengths still
    # gives every row of every sequence.
    lq = [300, 1000, 1]
    q, k, v, cu_q, cu_k = make_varlen(lq, lq, 2, 64, 37)
    o, lse = _run(q, k, v, cu_q, cu_k, True, max_q=130)
    o_ref, lse_ref = oracle.attention_varlen_ref(to_np64(q), to_np64(k), to_np64(v), cu_q.tolist(),
                                                 cu_k.tolist(), 0.125, causal=True)
    assert np.max(np.abs(o - o_ref)) <= TOL_O
    assert_lse_close(lse, lse_ref, TOL_LSE)


def test_varlen_argument_errors():
    q = torch.zeros((8, 2, 64), dtype=torch.bfloat16, device=DEV)
    cu = torch.tensor([0, 8], dtype=torch.int32, device=DEV)
    lib = fa.load_library()
    o = torch.empty_like(q)
    lse = torch.empty((2, 8), dtype=torch.float32, device=DEV)
    args = [q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(), cu.data_ptr(),
            cu.data_ptr(), 1, 2, 8, 8, 8, 64, 0.125, 0, None]
    bad = {7: 0, 9: 0, 11: 0, 13: -1.0, 14: 2}  # B, total_q, max_seqlen_q, scale, causal
    for i, val in bad.items():
        a = list(args)
        a[i] = val
        assert lib.fa_fwd_varlen(*a) == fa.FA_ERR_INVALID_ARGUMENT, i
    a = list(args)
    a[12] = 96
    assert lib.fa_fwd_varlen(*a) == fa.FA_ERR_UNSUPPORTED
    a = list(args)
    cu_host = cu.cpu()
    a[5] = cu_host.data_ptr()  # host offsets
    assert lib.fa_fwd_varlen(*a) == fa.FA_ERR_INVALID_ARGUMENT
    a = list(args)
    a[3] = q.data_ptr()  # o aliases q
    assert lib.fa_fwd_varlen(*a) == fa.FA_ERR_INVALID_ARGUMENT
