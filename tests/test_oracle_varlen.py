"""Pins for the variable-length oracle (no GPU).

* Each sequence against the pure-Python brute force (nested loops,
  math.fsum), on tiny ragged batches with empty sequences, queries without
  keys and more queries than keys, full and causal.
* Sequences are independent: changing one sequence's tokens leaves every
  other sequence's outputs bit-identical.
* Planted mistakes fail a pin: attending across sequence boundaries, and
  mutants planted in a copy of the oracle (keys of the wrong sequence, the
  query offsets used for the keys, values not offset, heads reversed in O or
  in lse).
"""

import math

import numpy as np
import pytest

import oracle


def _batch(lq, lk, H, d, seed):
    r = np.random.default_rng(seed)
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(np.int64)
    q = r.normal(size=(int(cu_q[-1]), H, d))
    k = r.normal(size=(int(cu_k[-1]), H, d))
    v = r.normal(size=(int(cu_k[-1]), H, d))
    return q, k, v, cu_q, cu_k


def _brute_varlen(q, k, v, cu_q, cu_k, scale, causal):
    Tq, H, d = q.shape
    o = np.zeros((Tq, H, d))
    lse = np.full((H, Tq), -math.inf)
    for b in range(len(cu_q) - 1):
        qa, qb, ka, kb = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if qb == qa:
            continue
        for h in range(H):
            qs = [[[q[i, h].tolist() for i in range(qa, qb)]]]
            ks = [[[k[j, h].tolist() for j in range(ka, kb)]]]
            vs = [[[v[j, h].tolist() for j in range(ka, kb)]]]
            if kb == ka:
                continue
            ob, lb = oracle.attention_brute(qs, ks, vs, scale, causal=causal)
            o[qa:qb, h] = np.array(ob[0][0])
            lse[h, qa:qb] = np.array(lb[0][0])
    return o, lse


CASES = [
    ([3, 5, 1], [3, 5, 1]),
    ([4, 0, 6, 2], [2, 3, 6, 5]),   # empty query sequence, nq > nk and nq < nk
    ([2, 3], [0, 4]),               # a sequence without keys
    ([7], [9]),
]


@pytest.mark.parametrize("lq,lk", CASES)
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_matches_brute_force(lq, lk, causal):
    q, k, v, cu_q, cu_k = _batch(lq, lk, H=2, d=3, seed=len(lq) + sum(lk))
    o, lse = oracle.attention_varlen_ref(q, k, v, cu_q, cu_k, 0.6, causal=causal)
    ob, lb = _brute_varlen(q, k, v, cu_q, cu_k, 0.6, causal)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)
    assert lse.shape == (2, q.shape[0])


def test_sequences_are_independent():
    lq, lk = [5, 4, 6], [6, 3, 7]
    q, k, v, cu_q, cu_k = _batch(lq, lk, H=2, d=4, seed=11)
    o1, l1 = oracle.attention_varlen_ref(q, k, v, cu_q, cu_k, 0.5, causal=True)
    k2, v2 = k.copy(), v.copy()
    k2[cu_k[1]:cu_k[2]] += 3.0
    v2[cu_k[1]:cu_k[2]] *= -2.0
    o2, l2 = oracle.attention_varlen_ref(q, k2, v2, cu_q, cu_k, 0.5, causal=True)
    for b in (0, 2):
        sl = slice(int(cu_q[b]), int(cu_q[b + 1]))
        assert np.array_equal(o1[sl], o2[sl]) and np.array_equal(l1[:, sl], l2[:, sl])
    sl = slice(int(cu_q[1]), int(cu_q[2]))
    assert not np.allclose(o1[sl], o2[sl])


def test_planted_cross_sequence_mistake_is_caught():
    lq, lk = [3, 4], [3, 4]
    q, k, v, cu_q, cu_k = _batch(lq, lk, H=1, d=3, seed=5)
    # Mutant: the whole packed stream treated as one sequence.
    mo, _ = oracle.attention_varlen_ref(q, k, v, [0, 7], [0, 7], 0.6, causal=False)
    ob, _ = _brute_varlen(q, k, v, cu_q, cu_k, 0.6, False)
    assert np.max(np.abs(mo - ob)) > 1e-3


def test_bad_offsets_rejected():
    q, k, v, cu_q, cu_k = _batch([2, 2], [2, 2], H=1, d=2, seed=1)
    with pytest.raises(ValueError):
        oracle.attention_varlen_ref(q, k, v, [0, 3, 2], cu_k, 1.0)
    with pytest.raises(ValueError):
        oracle.attention_varlen_ref(q, k, v, [0, 2, 5], cu_k, 1.0)


PLANTED = {
    "keys_of_previous_sequence": ("ka, kb = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]",
                                  "ka, kb = cu_q[b], cu_q[b + 1], cu_k[max(b - 1, 0)], cu_k[max(b, 1)]"),
    "query_offsets_for_keys": ("ks = k[ka:kb]", "ks = k[qa:qa + (kb - ka)]"),
    "values_from_the_start": ("vs = v[ka:kb]", "vs = v[:kb - ka]"),
    "heads_reversed": ("o[qa:qb] = ob[0].transpose(1, 0, 2)",
                       "o[qa:qb] = ob[0][::-1].transpose(1, 0, 2)"),
    "lse_heads_reversed": ("lse[:, qa:qb] = lb[0]", "lse[:, qa:qb] = lb[0][::-1]"),
}


@pytest.mark.parametrize("kind", sorted(PLANTED))
def test_planted_varlen_mistakes_are_caught(kind, monkeypatch):
    import inspect

    from oracle import varlen as varlen_mod

    old, new = PLANTED[kind]
    src = inspect.getsource(varlen_mod.attention_varlen_ref)
    assert src.count(old) == 1, old
    ns = dict(vars(varlen_mod))
    exec(compile(src.replace(old, new), varlen_mod.__file__, "exec"), ns)
    monkeypatch.setattr(oracle, "attention_varlen_ref", ns["attention_varlen_ref"])
    failed = 0
    for lq, lk in CASES:
        for causal in (False, True):
            try:
                test_varlen_matches_brute_force(lq, lk, causal)
            except (AssertionError, ValueError):
                failed += 1
    assert failed > 0, f"no pin caught the planted mistake {kind!r}"
