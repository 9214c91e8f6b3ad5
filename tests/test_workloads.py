"""The seeded input generators (no GPU): determinism, value ranges and the
useful-FLOP counts the bench divides by.

The FLOP counts are checked against a brute-force count of visible (query,
key) pairs from the oracle's visibility mask, so a wrong causal or sparse
credit in the benchmark would show here."""

import math

import numpy as np
import torch

import oracle
from exact_attention_120_b200 import workloads as wl


def test_generators_are_deterministic():
    a = wl.make_qkv(1, 2, 64, 64, seed=5, qk_std=3.0)
    b = wl.make_qkv(1, 2, 64, 64, seed=5, qk_std=3.0)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and torch.equal(x, y)
    c = wl.make_qkv(1, 2, 64, 64, seed=6)
    assert not torch.equal(a[0], c[0])
    assert wl.varlen_lengths(8, 128, 8192, 3) == wl.varlen_lengths(8, 128, 8192, 3)


def test_block_mask_keeps_the_diagonal_and_repeats_over_batch():
    m = wl.make_block_mask(3, 2, 1000, 0.25, seed=4)
    nb = math.ceil(1000 / 128)
    assert m.shape == (3, 2, nb, nb) and m.dtype == torch.uint8
    for h in range(2):
        assert torch.all(torch.diagonal(m[0, h]) == 1)
        assert torch.equal(m[0, h], m[2, h])
    assert 0.1 < float(m.float().mean()) < 0.6


def test_fp8_codes_are_finite_e4m3_with_saturating_scale():
    (q8, k8, v8), scales = wl.make_qkv_fp8(1, 2, 256, 128, seed=1, qk_std=3.0)
    for t, s in zip((q8, k8, v8), scales):
        codes = t.numpy()
        assert t.dtype == torch.uint8 and s > 0
        assert not np.any((codes & 0x7F) == 0x7F)          # no NaN codes
        vals = oracle.e4m3_decode(codes)
        assert np.max(np.abs(vals)) == 448.0               # the largest magnitude maps to 448


def test_varlen_offsets_and_lengths():
    lens = wl.varlen_lengths(32, 128, 8192, 5)
    assert all(128 <= n <= 8192 for n in lens)
    q, k, v, cu_q, cu_k = wl.make_varlen(lens, lens, 2, 64, seed=1)
    assert cu_q.dtype == torch.int32 and cu_q[0] == 0 and int(cu_q[-1]) == q.shape[0] == sum(lens)
    assert torch.all(cu_q[1:] >= cu_q[:-1]) and torch.equal(cu_q, cu_k)
    assert q.shape == (sum(lens), 2, 64) and v.shape == k.shape


def test_useful_flops_match_visible_pairs():
    B, H, N, d = 1, 2, 300, 64
    assert wl.useful_flops(B, H, N, d) == 4.0 * B * H * N * N * d
    # Causal credit is exactly half of full (the formula's convention); the
    # exact visible count is N(N+1)/2, within 1/N of it.
    vis = oracle.visible_mask(N, N, True).sum()
    assert abs(wl.useful_flops(B, H, N, d, causal=True) / (4.0 * B * H * d) - vis) / vis < 1.0 / N + 1e-12
    m = wl.make_block_mask(B, H, N, 0.3, seed=2)
    vis_sparse = sum(oracle.visible_mask(N, N, False, m[0, h].numpy()).sum() for h in range(H))
    # Block density times N^2: exact when N is a multiple of 128, close otherwise.
    credit = wl.useful_flops(B, H, N, d, block_mask=m) / (4.0 * d)
    assert abs(credit - vis_sparse) / vis_sparse < 0.35


def test_varlen_flops_count_visible_pairs_exactly():
    lq, lk = [5, 130, 1, 64], [7, 100, 3, 64]
    for causal in (False, True):
        want = sum(oracle.visible_mask(nq, nk, causal).sum() for nq, nk in zip(lq, lk))
        assert wl.varlen_flops(lq, lk, 3, 64, causal) == 4.0 * 64 * 3 * want
