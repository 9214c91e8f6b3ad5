"""Shared helpers for the GPU tests: run the CUDA path through the C ABI and
compare with the float64 oracle on the same seeded bf16 inputs."""

import math
import os
from concurrent.futures import ThreadPoolExecutor

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


def host_cores():
    """Cores this process may run on (the affinity mask; a container may
    see far more cores in os.cpu_count() than it is allowed to use)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except (AttributeError, OSError):
        return max(1, os.cpu_count() or 1)


def _pool_size():
    return min(16, host_cores())


def oracle_per_head(fn, heads):
    """Run `fn(b, h)` for every (b, h) in `heads` on a thread pool (NumPy
    releases the GIL in its array loops and BLAS calls, so the heads run side
    by side), the host's cores shared out between the tasks as BLAS threads.
    Returns the results in order."""
    from threadpoolctl import threadpool_limits

    workers = min(_pool_size(), len(heads))
    with threadpool_limits(max(1, host_cores() // workers)), ThreadPoolExecutor(workers) as ex:
        return list(ex.map(lambda bh: fn(*bh), heads))


def oracle_full(q, k, v, scale, causal=False, mask=None):
    """The float64 oracle on every row of every head (numpy inputs), one
    thread-pool task per head.  Same function, same arithmetic as calling
    oracle.attention_ref on the whole batch."""
    B, H, N, _ = q.shape
    heads = [(b, h) for b in range(B) for h in range(H)]

    def one(b, h):
        bm = None if mask is None else mask[b:b + 1, h:h + 1]
        return oracle.attention_ref(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                                    scale, causal=causal, block_mask=bm)

    res = oracle_per_head(one, heads)
    o = np.empty((B, H, N, v.shape[-1]))
    lse = np.empty((B, H, N))
    for (b, h), (oh, lh) in zip(heads, res):
        o[b, h], lse[b, h] = oh[0, 0], lh[0, 0]
    return o, lse
