"""Pins for the CPU oracle (no GPU).

The oracle is trusted only because these tests tie it to things other than
itself:

* the worked online-softmax example on the vector read as 2, 1, 3 (wmrh.cn
  article, "2.1 Online Softmax"), checked against closed forms derived by hand;
* shift invariance of softmax ("理解 Flash Attention" article, "瓦片注意力计算");
* the concatenated-softmax merge rule (same section), against the unsplit row;
* closed forms of attention: constant V rows, Q = 0 (averages over the visible
  keys), the first causal row, a shift of every key by one vector;
* normalisation of the softmax weights;
* an independent pure-Python brute force on tiny shapes (all mask modes);
* PyTorch's float64 ``scaled_dot_product_attention`` on the CPU (a library
  routine the dense and masked cases reduce to);
* the pages' one-pass tiled algorithm, which must reach the definition.

``test_planted_mistakes_are_caught`` plants plausible mistakes in a copy of the
oracle (on the CPU) and checks that some pin fails for each.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as ar_mod
from oracle.softmax import partial_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "online_softmax_example.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(a):
    """Round a float array to bfloat16 values (held in float64)."""
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).double().numpy()


# ---------------------------------------------------------------- softmax ---

def test_worked_example_online_softmax():
    g = json.load(open(GOLDEN))
    x = g["input"]
    a, m, d, trace = oracle.online_softmax_2pass(x)
    # Closed forms, dividing numerator and denominator by e^3 (by hand):
    e1, e2 = math.exp(-1.0), math.exp(-2.0)
    expect_d = [1.0, 1.0 + e1, 1.0 + e1 + e2]
    for step, (mi, di) in enumerate(trace):
        assert mi == g["running_max"][step]
        assert di == pytest.approx(expect_d[step], rel=1e-15, abs=0)
    changed = [trace[0][0] != -math.inf] + [trace[i][0] != trace[i - 1][0] for i in range(1, 3)]
    assert changed[1:] == g["max_changes_at_step"][1:]
    den = 1.0 + e1 + e2
    expect_a = [e1 / den, e2 / den, 1.0 / den]
    np.testing.assert_allclose(a, expect_a, rtol=1e-15, atol=0)
    assert m == 3.0 and d == pytest.approx(den, rel=1e-15)
    # The page's claim: the online result equals the 3-pass safe softmax.
    a3, m3, d3 = oracle.safe_softmax_3pass(x)
    np.testing.assert_allclose(a, a3, rtol=1e-15, atol=0)
    assert m3 == m and d3 == pytest.approx(d, rel=1e-15)
    # logsumexp of the example: 3 + ln(1 + e^-1 + e^-2)
    assert m3 + math.log(d3) == pytest.approx(3.0 + math.log(den), rel=1e-15)


@pytest.mark.parametrize("n", [1, 2, 7, 100])
def test_online_equals_three_pass(n):
    x = _rng(n).normal(size=n) * 5
    a2, m2, d2, _ = oracle.online_softmax_2pass(x)
    a3, m3, d3 = oracle.safe_softmax_3pass(x)
    assert m2 == m3
    np.testing.assert_allclose(d2, d3, rtol=1e-13)
    np.testing.assert_allclose(a2, a3, rtol=1e-13, atol=1e-300)
    assert math.isclose(float(np.sum(a3)), 1.0, rel_tol=1e-14)


def test_shift_invariance_of_softmax():
    x = _rng(1).normal(size=50) * 4
    a, _, _ = oracle.safe_softmax_3pass(x)
    for c in (-7.25, 3.0, 1000.0):
        a_c, _, _ = oracle.safe_softmax_3pass(x + c)
        np.testing.assert_allclose(a_c, a, rtol=1e-13, atol=1e-300)
    # Large inputs do not overflow (the reason for the shift).
    a_big, m_big, _ = oracle.safe_softmax_3pass(np.array([1000.0, 999.0, 1001.0]))
    e1, e2 = math.exp(-1.0), math.exp(-2.0)
    np.testing.assert_allclose(a_big, np.array([e1, e2, 1.0]) / (1 + e1 + e2), rtol=1e-14)


def test_all_masked_softmax_is_zero():
    a, m, d = oracle.safe_softmax_3pass([-math.inf] * 3)
    assert m == -math.inf and d == 0 and not a.any()
    a, m, d, _ = oracle.online_softmax_2pass([-math.inf, -math.inf])
    assert m == -math.inf and d == 0 and not a.any()


@pytest.mark.parametrize("seed", range(5))
def test_merge_rule_equals_unsplit(seed):
    r = _rng(seed)
    n, dv = 37, 5
    s = r.normal(size=n) * 3
    s[r.random(n) < 0.2] = -math.inf
    v = r.normal(size=(n, dv))
    cut = int(r.integers(0, n + 1))
    merged = oracle.merge_partials(partial_state(s[:cut], v[:cut]), partial_state(s[cut:], v[cut:]))
    whole = partial_state(s, v)
    assert merged[0] == whole[0]
    np.testing.assert_allclose(merged[1], whole[1], rtol=1e-13)
    np.testing.assert_allclose(merged[2], whole[2], rtol=1e-12, atol=1e-13)
    # normalised output equals softmax(s) @ v computed by the 3-pass definition
    a, _, _ = oracle.safe_softmax_3pass(s)
    np.testing.assert_allclose(merged[2] / merged[1], a @ v, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------- attention pins -------

def _inputs(B, H, N, d, seed, std=1.0):
    r = _rng(seed)
    q = _bf16(r.normal(size=(B, H, N, d)) * std)
    k = _bf16(r.normal(size=(B, H, N, d)) * std)
    v = _bf16(r.normal(size=(B, H, N, d)))
    return q, k, v


def _mask(B, H, N, block, p, seed):
    nb = -(-N // block)
    r = _rng(seed)
    m = (r.random((H, nb, nb)) < p) | np.eye(nb, dtype=bool)[None]
    return np.broadcast_to(m[None], (B, H, nb, nb)).astype(np.uint8)


MODES = ["full", "causal", "sparse", "sparse_causal"]


def _mode_args(mode, B, H, N, block, seed=9):
    causal = mode in ("causal", "sparse_causal")
    mask = _mask(B, H, N, block, 0.4, seed) if mode.startswith("sparse") else None
    return causal, mask


def _vis_count(N, causal, mask_bh, block):
    return oracle.visible_mask(N, N, causal, mask_bh, block).sum(axis=1)


def pin_constant_v(attn, mode):
    B, H, N, d, block = 2, 2, 19, 4, 4
    q, k, _ = _inputs(B, H, N, d, 1, std=2.0)
    c = np.array([0.5, -1.25, 3.0, 7.0])
    v = np.broadcast_to(c, (B, H, N, d)).copy()
    causal, mask = _mode_args(mode, B, H, N, block)
    o, lse = attn(q, k, v, 0.7, causal=causal, block_mask=mask, block=block)
    for b in range(B):
        for h in range(H):
            cnt = _vis_count(N, causal, None if mask is None else mask[b, h], block)
            for i in range(N):
                if cnt[i]:
                    np.testing.assert_allclose(o[b, h, i], c, rtol=1e-13)


def pin_zero_q(attn, mode):
    """Q = 0: every visible score is 0, so O_i is the plain mean of the visible
    V rows and lse_i = ln(number of visible keys)."""
    B, H, N, d, block = 2, 3, 23, 3, 4
    _, k, v = _inputs(B, H, N, d, 2)
    q = np.zeros_like(k)
    causal, mask = _mode_args(mode, B, H, N, block)
    o, lse = attn(q, k, v, 1.3, causal=causal, block_mask=mask, block=block)
    for b in range(B):
        for h in range(H):
            vis = oracle.visible_mask(N, N, causal, None if mask is None else mask[b, h], block)
            for i in range(N):
                js = np.nonzero(vis[i])[0]
                if js.size == 0:
                    assert lse[b, h, i] == -math.inf and not o[b, h, i].any()
                    continue
                mean = sum(v[b, h, j] for j in js) / js.size
                np.testing.assert_allclose(o[b, h, i], mean, rtol=1e-12, atol=1e-14)
                assert lse[b, h, i] == pytest.approx(math.log(js.size), rel=1e-13, abs=1e-14)


def pin_first_causal_row(attn):
    B, H, N, d = 1, 2, 9, 5
    q, k, v = _inputs(B, H, N, d, 3)
    scale = 0.45
    o, lse = attn(q, k, v, scale, causal=True, block_mask=None, block=4)
    for h in range(H):
        np.testing.assert_allclose(o[0, h, 0], v[0, h, 0], rtol=1e-14)
        s00 = scale * math.fsum(q[0, h, 0, t] * k[0, h, 0, t] for t in range(d))
        assert lse[0, h, 0] == pytest.approx(s00, rel=1e-13)


def pin_key_shift(attn, mode):
    """Adding one vector u to every key adds scale*q_i.u to every score of row
    i: O is unchanged and lse_i grows by exactly that amount."""
    B, H, N, d, block = 1, 2, 17, 6, 4
    q, k, v = _inputs(B, H, N, d, 4)
    u = _rng(44).normal(size=d)
    scale = 0.8
    causal, mask = _mode_args(mode, B, H, N, block)
    o1, l1 = attn(q, k, v, scale, causal=causal, block_mask=mask, block=block)
    o2, l2 = attn(q, k + u, v, scale, causal=causal, block_mask=mask, block=block)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-12)
    fin = np.isfinite(l1)
    shift = scale * np.einsum("bhnd,d->bhn", q, u)
    np.testing.assert_allclose(l2[fin], (l1 + shift)[fin], rtol=1e-12, atol=1e-12)


def pin_normalisation(attn, mode):
    B, H, N, d, block = 1, 2, 21, 4, 4
    q, k, v = _inputs(B, H, N, d, 5, std=2.0)
    scale = 0.6
    causal, mask = _mode_args(mode, B, H, N, block)
    _, lse = attn(q, k, v, scale, causal=causal, block_mask=mask, block=block)
    for h in range(H):
        vis = oracle.visible_mask(N, N, causal, None if mask is None else mask[0, h], block)
        for i in range(N):
            js = np.nonzero(vis[i])[0]
            if js.size:
                tot = math.fsum(math.exp(scale * float(q[0, h, i] @ k[0, h, j]) - lse[0, h, i]) for j in js)
                assert tot == pytest.approx(1.0, rel=1e-12)


def pin_brute(attn, mode):
    for (B, H, N, d, block) in [(1, 1, 1, 1, 1), (1, 2, 3, 2, 2), (2, 1, 5, 4, 2), (1, 1, 8, 3, 2)]:
        q, k, v = _inputs(B, H, N, d, N + d, std=1.5)
        causal, mask = _mode_args(mode, B, H, N, block, seed=N)
        o, lse = attn(q, k, v, 0.9, causal=causal, block_mask=mask, block=block)
        ob, lb = oracle.attention_brute(q.tolist(), k.tolist(), v.tolist(), 0.9, causal=causal,
                                        block_mask=None if mask is None else mask.tolist(), block=block)
        np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, np.array(lb), rtol=1e-12, atol=1e-13)


def pin_sdpa(attn, mode):
    """PyTorch's float64 CPU scaled_dot_product_attention computes the same
    definition (masked keys excluded through a boolean mask)."""
    B, H, N, d, block = 2, 2, 40, 8, 8
    q, k, v = _inputs(B, H, N, d, 6, std=1.5)
    scale = 0.3
    causal, mask = _mode_args(mode, B, H, N, block)
    o, _ = attn(q, k, v, scale, causal=causal, block_mask=mask, block=block)
    vis = np.stack([np.stack([oracle.visible_mask(N, N, causal, None if mask is None else mask[b, h], block)
                              for h in range(H)]) for b in range(B)])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(vis), scale=scale).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def _oracle_attn(q, k, v, scale, causal=False, block_mask=None, block=128):
    return oracle.attention_ref(q, k, v, scale, causal=causal, block_mask=block_mask, block=block)


@pytest.mark.parametrize("mode", MODES)
def test_constant_v(mode):
    pin_constant_v(_oracle_attn, mode)


@pytest.mark.parametrize("mode", MODES)
def test_zero_q_means(mode):
    pin_zero_q(_oracle_attn, mode)


def test_first_causal_row():
    pin_first_causal_row(_oracle_attn)


@pytest.mark.parametrize("mode", MODES)
def test_key_shift(mode):
    pin_key_shift(_oracle_attn, mode)


@pytest.mark.parametrize("mode", MODES)
def test_normalisation(mode):
    pin_normalisation(_oracle_attn, mode)


@pytest.mark.parametrize("mode", MODES)
def test_brute_force_tiny(mode):
    pin_brute(_oracle_attn, mode)


@pytest.mark.parametrize("mode", MODES)
def test_sdpa_float64(mode):
    pin_sdpa(_oracle_attn, mode)


def test_row_chunking_is_invisible():
    q, k, v = _inputs(1, 2, 50, 4, 7)
    a = oracle.attention_ref(q, k, v, 0.5, causal=True, row_chunk=7)
    b = oracle.attention_ref(q, k, v, 0.5, causal=True, row_chunk=1024)
    # BLAS may block the products differently per chunk shape: last-ulp only
    np.testing.assert_allclose(a[0], b[0], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-14, atol=1e-15)


def test_sampled_rows_match_full():
    B, H, N, d, block = 2, 2, 33, 4, 8
    q, k, v = _inputs(B, H, N, d, 8)
    mask = _mask(B, H, N, block, 0.5, 3)
    o, lse = oracle.attention_ref(q, k, v, 0.5, causal=True, block_mask=mask, block=block)
    sample = [(1, 0, 0), (0, 1, 32), (1, 1, 17), (0, 0, 8)]
    so, sl = oracle.attention_ref_rows(q, k, v, 0.5, sample, causal=True, block_mask=mask, block=block)
    for n, (b, h, i) in enumerate(sample):
        np.testing.assert_allclose(so[n], o[b, h, i], rtol=1e-14, atol=1e-15)
        assert sl[n] == pytest.approx(lse[b, h, i], rel=1e-14)


def test_empty_rows():
    B, H, N, d, block = 1, 1, 8, 2, 2
    q, k, v = _inputs(B, H, N, d, 9)
    mask = np.ones((1, 1, 4, 4), dtype=np.uint8)
    mask[0, 0, 1, :] = 0  # query rows 2 and 3 see nothing
    o, lse = oracle.attention_ref(q, k, v, 1.0, block_mask=mask, block=block)
    assert np.all(lse[0, 0, 2:4] == -math.inf) and not o[0, 0, 2:4].any()
    assert np.all(np.isfinite(lse[0, 0, [0, 1, 4, 5, 6, 7]]))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("bm,bn", [(4, 4), (3, 5), (8, 2)])
def test_tiled_algorithm_reaches_definition(mode, bm, bn):
    B, H, N, d, block = 1, 2, 19, 4, 4
    q, k, v = _inputs(B, H, N, d, 10, std=3.0)
    causal, mask = _mode_args(mode, B, H, N, block)
    o1, l1 = oracle.attention_ref(q, k, v, 0.7, causal=causal, block_mask=mask, block=block)
    o2, l2 = oracle.attention_tiled_online(q, k, v, 0.7, causal=causal, block_mask=mask,
                                           block=block, bm=bm, bn=bn)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=1e-13, atol=1e-13)


# ------------------------------------------------- planted mistakes ---------

def _mutant(kind):
    """A copy of the oracle with one plausible mistake planted (CPU only)."""
    def rows_of_head(qh, kh, vh, scale, causal, bm_bh, block, rows):
        n_q, n_k = qh.shape[0], kh.shape[0]
        if kind == "no_scale":
            s = qh[rows] @ kh.T
        elif kind == "k_for_v":
            s = scale * (qh[rows] @ kh.T)
        else:
            s = scale * (qh[rows] @ kh.T)
        c = causal
        vis = ar_mod.visible_mask(n_q, n_k, c, bm_bh, block, rows)
        if kind == "causal_strict" and causal:
            vis &= np.arange(n_k)[None, :] < np.asarray(rows)[:, None]
        if kind == "mask_transposed" and bm_bh is not None:
            vis = ar_mod.visible_mask(n_q, n_k, c, np.asarray(bm_bh).T, block, rows)
        if kind == "mask_after_softmax":
            p, m, d = ar_mod._softmax_rows_3pass(s)
            p = np.where(vis, p, 0.0)
        else:
            s = np.where(vis, s, -np.inf)
            p, m, d = ar_mod._softmax_rows_3pass(s)
        o = p @ (kh if kind == "k_for_v" else vh)
        if kind == "lse_no_max":
            m = np.zeros_like(m)
        with np.errstate(divide="ignore"):
            lse = np.where(d > 0, m + np.log(np.where(d > 0, d, 1.0)), -np.inf)
        return o, lse
    return rows_of_head


@pytest.mark.parametrize("kind", ["no_scale", "k_for_v", "causal_strict", "mask_transposed",
                                  "mask_after_softmax", "lse_no_max"])
def test_planted_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(ar_mod, "_rows_of_head", _mutant(kind))
    pins = [lambda: pin_constant_v(_oracle_attn, "sparse_causal")]
    for mode in MODES:
        pins += [lambda m=mode: pin_zero_q(_oracle_attn, m),
                 lambda m=mode: pin_key_shift(_oracle_attn, m),
                 lambda m=mode: pin_brute(_oracle_attn, m),
                 lambda m=mode: pin_normalisation(_oracle_attn, m)]
    pins.append(lambda: pin_first_causal_row(_oracle_attn))
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught the planted mistake {kind!r}"


# ------------------------------------------ different query / key lengths ---

def _inputs_qk(B, H, Nq, Nk, d, seed, std=1.0):
    r = _rng(seed)
    q = _bf16(r.normal(size=(B, H, Nq, d)) * std)
    k = _bf16(r.normal(size=(B, H, Nk, d)) * std)
    v = _bf16(r.normal(size=(B, H, Nk, d)))
    return q, k, v


def _mask_qk(B, H, Nq, Nk, block, p, seed):
    r = _rng(seed)
    m = r.random((H, -(-Nq // block), -(-Nk // block))) < p
    return np.broadcast_to(m[None], (B, H) + m.shape[1:]).astype(np.uint8)


@pytest.mark.parametrize("nq,nk", [(1, 5), (3, 8), (8, 3), (6, 6), (2, 7)])
@pytest.mark.parametrize("mode", MODES)
def test_qk_lengths_brute_force(nq, nk, mode):
    B, H, d, block = 1, 2, 3, 2
    q, k, v = _inputs_qk(B, H, nq, nk, d, nq * 10 + nk, std=1.5)
    causal = mode in ("causal", "sparse_causal")
    mask = _mask_qk(B, H, nq, nk, block, 0.6, nq + nk) if mode.startswith("sparse") else None
    o, lse = oracle.attention_ref(q, k, v, 0.8, causal=causal, block_mask=mask, block=block)
    ob, lb = oracle.attention_brute(q.tolist(), k.tolist(), v.tolist(), 0.8, causal=causal,
                                    block_mask=None if mask is None else mask.tolist(), block=block)
    np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(lb), rtol=1e-12, atol=1e-13)
    o2, l2 = oracle.attention_tiled_online(q, k, v, 0.8, causal=causal, block_mask=mask, block=block,
                                           bm=3, bn=2)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, lse, rtol=1e-12, atol=1e-13)


# With nq > nk the library warns that fully masked rows come out NaN; those
# rows are excluded from the comparison below.
@pytest.mark.filterwarnings("ignore:Lower right causal bias will produce NaNs")
@pytest.mark.parametrize("nq,nk", [(5, 40), (40, 40), (33, 17)])
def test_qk_causal_matches_lower_right_sdpa(nq, nk):
    """PyTorch's lower-right causal bias is the same bottom-right alignment."""
    from torch.nn.attention.bias import causal_lower_right

    B, H, d = 2, 2, 8
    q, k, v = _inputs_qk(B, H, nq, nk, d, 31)
    o, lse = oracle.attention_ref(q, k, v, 0.4, causal=True)
    if nq > nk:
        # the first nq - nk rows see no key at all
        assert np.all(lse[:, :, : nq - nk] == -math.inf) and not o[:, :, : nq - nk].any()
        rows = slice(nq - nk, nq)
    else:
        rows = slice(0, nq)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=causal_lower_right(nq, nk), scale=0.4).numpy()
    np.testing.assert_allclose(o[:, :, rows], ref[:, :, rows], rtol=1e-11, atol=1e-12)


def test_decode_row_sees_every_key():
    B, H, nk, d = 1, 3, 50, 4
    q, k, v = _inputs_qk(B, H, 1, nk, d, 41)
    oc, lc = oracle.attention_ref(q, k, v, 0.6, causal=True)
    of, lf = oracle.attention_ref(q, k, v, 0.6, causal=False)
    np.testing.assert_array_equal(oc, of)
    np.testing.assert_array_equal(lc, lf)
