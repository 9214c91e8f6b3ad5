"""Pins for the gradient oracle (no GPU): central finite differences of the
(pinned) forward oracle, PyTorch float64 autograd through SDPA, closed forms
and invariants of the softmax gradient."""

import math

import numpy as np
import pytest
import torch

import oracle


def _r(seed):
    return np.random.default_rng(seed)


def _case(B, H, Nq, Nk, d, seed, std=1.0):
    r = _r(seed)
    return (r.normal(size=(B, H, Nq, d)) * std, r.normal(size=(B, H, Nk, d)) * std,
            r.normal(size=(B, H, Nk, d)), r.normal(size=(B, H, Nq, d)))


def _mode(mode, B, H, Nq, Nk, block, seed=3):
    causal = mode in ("causal", "sparse_causal")
    mask = None
    if mode.startswith("sparse"):
        r = _r(seed)
        m = r.random((H, -(-Nq // block), -(-Nk // block))) < 0.6
        mask = np.broadcast_to(m[None], (B, H) + m.shape[1:]).astype(np.uint8)
    return causal, mask


MODES = ["full", "causal", "sparse", "sparse_causal"]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("nq,nk", [(5, 5), (3, 6), (6, 4)])
def test_gradients_match_finite_differences(mode, nq, nk):
    B, H, d, block, scale = 1, 2, 3, 2, 0.7
    q, k, v, do = _case(B, H, nq, nk, d, nq * 7 + nk)
    causal, mask = _mode(mode, B, H, nq, nk, block)
    dq, dk, dv = oracle.attention_bwd_ref(q, k, v, do, scale, causal, mask, block)

    def loss(q_, k_, v_):
        o, _ = oracle.attention_ref(q_, k_, v_, scale, causal=causal, block_mask=mask, block=block)
        return float(np.sum(o * do))

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-7, err_msg=name)


@pytest.mark.parametrize("row_chunk", [1024, 5])
@pytest.mark.parametrize("nq,nk,causal", [(16, 16, False), (16, 16, True), (8, 20, True),
                                          (20, 9, False)])
def test_gradients_match_torch_autograd(nq, nk, causal, row_chunk):
    # row_chunk = 5 cuts the query rows into ragged chunks, so dK and dV are
    # summed over several chunks.
    from torch.nn.attention.bias import causal_lower_right

    B, H, d, scale = 2, 2, 8, 0.35
    q, k, v, do = _case(B, H, nq, nk, d, nq + nk)
    dq, dk, dv = oracle.attention_bwd_ref(q, k, v, do, scale, causal, row_chunk=row_chunk)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    mask = causal_lower_right(nq, nk) if causal else None
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_constant_values_give_no_query_key_gradient():
    # O = c whatever the softmax is, so dQ = dK = 0 and dV_j = sum_i P_ij dO_i
    B, H, nq, nk, d = 1, 2, 7, 9, 4
    q, k, _, do = _case(B, H, nq, nk, d, 5, std=2.0)
    v = np.broadcast_to(np.array([0.5, -1.0, 2.0, 3.0]), (B, H, nk, d)).copy()
    dq, dk, dv = oracle.attention_bwd_ref(q, k, v, do, 0.5, causal=True)
    assert np.max(np.abs(dq)) < 1e-12 and np.max(np.abs(dk)) < 1e-12
    # dV summed over keys = sum of dO over the rows that see at least one key
    np.testing.assert_allclose(dv.sum(axis=2), do[:, :, :].sum(axis=2), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", MODES)
def test_softmax_gradient_rows_sum_to_zero(mode):
    # sum_j dS_ij = 0 for every row, hence sum_j dK_j = 0
    B, H, nq, nk, d, block = 2, 2, 12, 10, 5, 4
    q, k, v, do = _case(B, H, nq, nk, d, 9)
    causal, mask = _mode(mode, B, H, nq, nk, block)
    _, dk, _ = oracle.attention_bwd_ref(q, k, v, do, 0.9, causal, mask, block)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)


def test_invisible_keys_get_no_gradient():
    B, H, nq, nk, d, block = 1, 1, 4, 8, 3, 4
    q, k, v, do = _case(B, H, nq, nk, d, 11)
    mask = np.ones((1, 1, 1, 2), np.uint8)
    mask[0, 0, 0, 1] = 0  # keys 4..7 are masked for every query
    dq, dk, dv = oracle.attention_bwd_ref(q, k, v, do, 1.0, False, mask, block)
    assert not dk[:, :, 4:].any() and not dv[:, :, 4:].any()
    assert np.abs(dk[:, :, :4]).sum() > 0


@pytest.mark.parametrize("causal", [False, True])
def test_delta_equals_probability_weighted_dp(causal):
    # D_i = dO_i . O_i must equal sum_j P_ij (dO_i . v_j), with P taken from
    # the pure-Python brute force's logsumexp (P_ij = exp(s_ij - lse_i)) and
    # every sum formed with math.fsum: a second route to D that never forms O.
    B, H, nq, nk, d, scale = 1, 2, 5, 7, 3, 0.8
    q, k, v, do = _case(B, H, nq, nk, d, 21)
    o, lse = oracle.attention_brute(q.tolist(), k.tolist(), v.tolist(), scale, causal=causal)
    o, lse = np.array(o), np.array(lse)
    got = oracle.softmax_delta(o, do)
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                terms = []
                for j in range(nk):
                    if causal and j > i + (nk - nq):
                        continue
                    s_ij = scale * math.fsum(q[b, h, i, t] * k[b, h, j, t] for t in range(d))
                    dp_ij = math.fsum(do[b, h, i, t] * v[b, h, j, t] for t in range(d))
                    terms.append(math.exp(s_ij - lse[b, h, i]) * dp_ij)
                assert abs(got[b, h, i] - math.fsum(terms)) <= 1e-12 * (1 + abs(got[b, h, i]))


# Plausible mistakes planted in a copy of the gradient oracle (on the CPU): a
# dropped or sign-flipped row term, a missing scale, a swapped operand, the
# mask left out.  Each must make at least one pin above fail.
PLANTED = {
    "drop_delta": ("attention_bwd_ref", "ds = p * (dp - dd[:, None])", "ds = p * dp"),
    "delta_sign": ("attention_bwd_ref", "ds = p * (dp - dd[:, None])", "ds = p * (dp + dd[:, None])"),
    "dq_no_scale": ("attention_bwd_ref", "dq[b, h, rows] = scale * (ds @ k[b, h])",
                    "dq[b, h, rows] = ds @ k[b, h]"),
    "dq_uses_v": ("attention_bwd_ref", "dq[b, h, rows] = scale * (ds @ k[b, h])",
                  "dq[b, h, rows] = scale * (ds @ v[b, h])"),
    "dv_uses_o": ("attention_bwd_ref", "dv[b, h] += p.T @ doc", "dv[b, h] += p.T @ o"),
    "delta_from_q": ("attention_bwd_ref", "dd = softmax_delta(o, doc)", "dd = softmax_delta(qc, doc)"),
    "dk_uses_do": ("attention_bwd_ref", "dk[b, h] += scale * (ds.T @ qc)",
                   "dk[b, h] += scale * (ds.T @ doc)"),
    "mask_ignored": ("attention_bwd_ref", "s = np.where(vis, s, -np.inf)", "s = s"),
    "dk_last_chunk_only": ("attention_bwd_ref", "dk[b, h] += scale * (ds.T @ qc)",
                           "dk[b, h] = scale * (ds.T @ qc)"),
    "delta_squares_o": ("softmax_delta", "np.sum(_as64(o) * _as64(do), axis=-1)",
                        "np.sum(_as64(o) * _as64(o), axis=-1)"),
    "delta_negated": ("softmax_delta", "np.sum(_as64(o) * _as64(do), axis=-1)",
                      "-np.sum(_as64(o) * _as64(do), axis=-1)"),
}


def _bwd_mutant(func, old, new, monkeypatch):
    """Plant `new` in place of `old` in a copy of oracle.backward's `func`;
    the copied attention_bwd_ref calls the mutated helpers."""
    import inspect

    from oracle import backward as bwd_mod

    ns = dict(vars(bwd_mod))
    src = inspect.getsource(getattr(bwd_mod, func))
    assert src.count(old) == 1, old
    exec(compile(src.replace(old, new), bwd_mod.__file__, "exec"), ns)
    if func != "attention_bwd_ref":
        exec(compile(inspect.getsource(bwd_mod.attention_bwd_ref), bwd_mod.__file__, "exec"), ns)
        monkeypatch.setattr(oracle, func, ns[func])
    monkeypatch.setattr(oracle, "attention_bwd_ref", ns["attention_bwd_ref"])


@pytest.mark.parametrize("kind", sorted(PLANTED))
def test_planted_gradient_mistakes_are_caught(kind, monkeypatch):
    _bwd_mutant(*PLANTED[kind], monkeypatch)
    pins = [lambda: test_gradients_match_finite_differences("sparse_causal", 3, 6),
            lambda: test_gradients_match_finite_differences("full", 5, 5),
            lambda: test_gradients_match_torch_autograd(8, 20, True, 1024),
            lambda: test_gradients_match_torch_autograd(20, 9, False, 5),
            test_constant_values_give_no_query_key_gradient,
            lambda: test_softmax_gradient_rows_sum_to_zero("causal"),
            test_invisible_keys_get_no_gradient,
            lambda: test_delta_equals_probability_weighted_dp(True)]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught the planted mistake {kind!r}"
