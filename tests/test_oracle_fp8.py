"""Pins for the 8-bit oracle (no GPU).

* e4m3_decode against the format's closed-form values and, for all 256
  codes, against PyTorch's float8_e4m3fn conversion (a library routine).
* attention_fp8_ref against the pure-Python brute force on the decoded,
  descaled values.
* weighted_spread: zero for constant V; for Q = 0 (uniform weights) the
  plain standard deviation of the visible V rows; brute force on tiny shapes.
* The rounding bound the GPU test relies on: weights perturbed by relative
  errors |e| <= u move O by at most u / (1 - u) times the spread.
"""

import math

import numpy as np
import pytest
import torch

import oracle


def test_e4m3_closed_forms():
    d = oracle.e4m3_decode
    assert d(0x00) == 0.0 and math.copysign(1.0, d(0x80)) == -1.0
    assert d(0x38) == 1.0 and d(0xB8) == -1.0
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert d(0x08) == 2.0 ** -6           # smallest normal
    assert d(0x01) == 2.0 ** -9           # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9       # largest subnormal
    assert d(0x39) == 1.125               # one mantissa step above 1
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ours[~nan], ref[~nan])


def _codes(shape, seed):
    r = np.random.default_rng(seed)
    c = r.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38  # no NaN codes
    c[(c & 0x78) >= 0x50] &= 0x3F  # keep magnitudes moderate
    return c


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_attention_matches_brute(causal):
    q8, k8, v8 = _codes((1, 2, 5, 3), 1), _codes((1, 2, 6, 3), 2), _codes((1, 2, 6, 3), 3)
    qd, kd, vd, scale = 0.25, 0.5, 2.0, 0.7
    o, lse = oracle.attention_fp8_ref(q8, k8, v8, qd, kd, vd, scale, causal=causal)
    dq = (oracle.e4m3_decode(q8) * qd).tolist()
    dk = (oracle.e4m3_decode(k8) * kd).tolist()
    dv = (oracle.e4m3_decode(v8) * vd).tolist()
    ob, lb = oracle.attention_brute(dq, dk, dv, scale, causal=causal)
    np.testing.assert_allclose(o, np.array(ob), rtol=0, atol=1e-12)
    lb = np.array(lb)
    fin = np.isfinite(lb)
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


def test_spread_constant_v_is_zero():
    r = np.random.default_rng(4)
    q, k = r.normal(size=(1, 2, 7, 4)), r.normal(size=(1, 2, 9, 4))
    v = np.broadcast_to(r.normal(size=(1, 2, 1, 4)), (1, 2, 9, 4)).copy()
    assert np.max(oracle.weighted_spread(q, k, v, 0.5, causal=True)) < 1e-7


@pytest.mark.parametrize("causal", [False, True])
def test_spread_uniform_weights_is_plain_std(causal):
    r = np.random.default_rng(5)
    n, d = 8, 3
    q, k, v = np.zeros((1, 1, n, d)), r.normal(size=(1, 1, n, d)), r.normal(size=(1, 1, n, d))
    sp = oracle.weighted_spread(q, k, v, 1.0, causal=causal)
    for i in range(n):
        rows = v[0, 0, : i + 1] if causal else v[0, 0]
        np.testing.assert_allclose(sp[0, 0, i], np.std(rows, axis=0), rtol=1e-9, atol=1e-12)


def test_spread_brute_force():
    r = np.random.default_rng(6)
    q, k, v = r.normal(size=(1, 1, 3, 2)), r.normal(size=(1, 1, 4, 2)), r.normal(size=(1, 1, 4, 2))
    sp = oracle.weighted_spread(q, k, v, 0.9)
    for i in range(3):
        s = [0.9 * math.fsum(q[0, 0, i, t] * k[0, 0, j, t] for t in range(2)) for j in range(4)]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        w = [x / math.fsum(e) for x in e]
        for t in range(2):
            o = math.fsum(w[j] * v[0, 0, j, t] for j in range(4))
            want = math.sqrt(math.fsum(w[j] * (v[0, 0, j, t] - o) ** 2 for j in range(4)))
            assert abs(sp[0, 0, i, t] - want) < 1e-12


@pytest.mark.parametrize("seed", range(5))
def test_rounding_bound_holds(seed):
    r = np.random.default_rng(seed)
    u = 2.0 ** -4
    q, k, v = r.normal(size=(1, 1, 16, 8)) * 2, r.normal(size=(1, 1, 40, 8)) * 2, r.normal(size=(1, 1, 40, 8))
    o, _ = oracle.attention_ref(q, k, v, 0.35)
    sp = oracle.weighted_spread(q, k, v, 0.35)
    s = 0.35 * q[0, 0] @ k[0, 0].T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    for _ in range(20):
        e = r.uniform(-u, u, size=p.shape)
        e[:, ::3] = np.sign(e[:, ::3]) * u  # extremes too
        pt = p * (1 + e)
        o2 = (pt @ v[0, 0]) / pt.sum(axis=1, keepdims=True)
        assert np.all(np.abs(o2 - o[0, 0]) <= u / (1 - u) * sp[0, 0] + 1e-12)


# Plausible mistakes planted in a copy of the 8-bit oracle (on the CPU); each
# must make at least one pin above fail.
PLANTED = {
    "bias_8": ("np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)"),
    "subnormal_exp": ("(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7"),
    "subnormal_implicit_one": ("sub = sign * (m / 8.0)", "sub = sign * (1.0 + m / 8.0)"),
    "mantissa_16ths": ("(1.0 + m / 8.0) * np.exp2", "(1.0 + m / 16.0) * np.exp2"),
    "nan_as_max": ("np.where((c & 0x7F) == 0x7F, np.nan, out)", "out"),
    "v_takes_k_scale": ("e4m3_decode(v8) * float(v_descale)", "e4m3_decode(v8) * float(k_descale)"),
    "q_unscaled": ("e4m3_decode(q8) * float(q_descale)", "e4m3_decode(q8)"),
}


def _fp8_mutant(kind, monkeypatch):
    import inspect

    from oracle import fp8 as fp8_mod

    old, new = PLANTED[kind]
    for name in ("e4m3_decode", "attention_fp8_ref"):
        src = inspect.getsource(getattr(fp8_mod, name))
        if old in src:
            ns = dict(vars(fp8_mod))
            exec(compile(src.replace(old, new), fp8_mod.__file__, "exec"), ns)
            monkeypatch.setattr(oracle, name, ns[name])
            return
    raise AssertionError(f"{old!r} not found")


@pytest.mark.parametrize("kind", sorted(PLANTED))
def test_planted_fp8_mistakes_are_caught(kind, monkeypatch):
    _fp8_mutant(kind, monkeypatch)
    pins = [test_e4m3_closed_forms, test_e4m3_all_codes_match_torch,
            lambda: test_fp8_attention_matches_brute(True)]
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0, f"no pin caught the planted mistake {kind!r}"
