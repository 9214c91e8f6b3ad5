"""Shared helpers for the GPU tests: run the CUDA path through the C ABI and
compare with the float64 oracle on the same seeded bf16 inputs."""

import math

import numpy as np
import torch

import oracle
from exact_attention_120_b200 import attention_forward
from exact_attention_120_b200.workloads import make_block_mask, make_qkv

# Parity bar: absolute, over every compared element, against the fp64 oracle.
TOL_O = 2e-2
TOL_LSE = 1e-2


def to_np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def run_cuda(q, k, v, causal=False, mask=None, scale=None):
    """CPU bf16 tensors in, (O float64 numpy, lse float64 numpy) out."""
    dev = torch.device("cuda", 0)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    md = None if mask is None else mask.to(dev)
    o, lse = attention_forward(qd, kd, vd, causal=causal, block_mask=md, scale=scale)
    torch.cuda.synchronize()
    return to_np64(o), to_np64(lse)


def make_case(B, H, N, d, seed, causal=False, sparse_p=None, qk_std=1.0, mask_seed=None):
    q, k, v = make_qkv(B, H, N, d, seed, qk_std=qk_std)
    mask = None
    if sparse_p is not None:
        mask = make_block_mask(B, H, N, sparse_p, seed if mask_seed is None else mask_seed)
    return q, k, v, mask


def assert_lse_close(got, ref, tol=TOL_LSE):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "lse: finiteness differs from the oracle"
    assert np.all(got[~fin] == ref[~fin]), "lse: empty rows must be -inf"
    if fin.any():
        err = np.max(np.abs(got[fin] - ref[fin]))
        assert err <= tol, f"max|dlse| = {err:.3e} > {tol}"


def assert_parity(o, lse, o_ref, lse_ref, tol_o=TOL_O, tol_lse=TOL_LSE):
    assert np.all(np.isfinite(o)), "O has non-finite values"
    err = np.max(np.abs(o - o_ref)) if o.size else 0.0
    assert err <= tol_o, f"max|dO| = {err:.3e} > {tol_o}"
    assert_lse_close(lse, lse_ref, tol_lse)
    return err


def full_parity(q, k, v, causal=False, mask=None, scale=None):
    d = q.shape[-1]
    s = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = run_cuda(q, k, v, causal, mask, scale)
    o_ref, lse_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), s, causal=causal,
                                          block_mask=None if mask is None else mask.numpy())
    return assert_parity(o, lse, o_ref, lse_ref)


def sample_rows(B, H, N, count, seed, per_tile=True):
    """(b, h, i) samples: first and last rows, tile edges, one random row in
    every (b, h, 128-row query tile) when `per_tile`, and random rows up to
    `count` extra."""
    r = np.random.default_rng(seed)
    rows = {(0, 0, 0), (B - 1, H - 1, N - 1), (0, H - 1, min(N - 1, 127)),
            (B - 1, 0, min(N - 1, 128)), (0, 0, N // 2)}
    if per_tile:
        for b in range(B):
            for h in range(H):
                for t0 in range(0, N, 128):
                    rows.add((b, h, int(r.integers(t0, min(N, t0 + 128)))))
    target = len(rows) + count
    while len(rows) < target:
        rows.add((int(r.integers(B)), int(r.integers(H)), int(r.integers(N))))
    return sorted(rows)
