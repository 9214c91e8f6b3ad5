"""GPU parity of the split-key forward (fa_fwd_splitkv + merge kernel) against
the float64 oracle: decoding against long caches, long causal sequences cut
into slices, block-sparse masks, and argument errors."""

import math

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from exact_attention_120_b200.workloads import make_qkv
from fa_helpers import assert_parity, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _case(B, H, Nq, Nk, d, seed, std=1.0):
    q, _, _ = make_qkv(B, H, Nq, d, seed, qk_std=std)
    _, k, v = make_qkv(B, H, Nk, d, seed + 1, qk_std=std)
    return q, k, v


def _run(q, k, v, causal, splits, mask=None):
    o, lse = fa.attention_forward_splitkv(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal,
                                          block_mask=None if mask is None else mask.to(DEV),
                                          num_splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    return to_np64(o), to_np64(lse)


def _ref(q, k, v, causal, mask=None):
    d = q.shape[-1]
    return oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1 / math.sqrt(d), causal=causal,
                                block_mask=None if mask is None else mask.numpy())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("splits", [2, 7, 32, None])
@pytest.mark.parametrize("causal", [False, True])
def test_decode_splits(d, splits, causal):
    q, k, v = _case(2, 4, 1, 8192 + 77, d, seed=splits or 5, std=2.0)
    o, lse = _run(q, k, v, causal, splits)
    assert_parity(o, lse, *_ref(q, k, v, causal))


@pytest.mark.parametrize("splits", [2, 3, 16])
def test_long_causal_splits(splits):
    q, k, v = _case(1, 2, 1000, 1000, 128, seed=splits)
    o, lse = _run(q, k, v, True, splits)
    assert_parity(o, lse, *_ref(q, k, v, True))


def test_empty_slices_and_rows():
    # Nq > Nk causal: early rows see nothing; many slices see nothing for many rows
    q, k, v = _case(1, 2, 500, 300, 64, seed=3)
    o, lse = _run(q, k, v, True, 3)
    assert np.all(np.isneginf(lse[:, :, :200])) and not o[:, :, :200].any()
    assert_parity(o, lse, *_ref(q, k, v, True))


def test_block_sparse_splits():
    B, H, nq, nk, d = 2, 2, 200, 2000, 64
    q, k, v = _case(B, H, nq, nk, d, seed=4)
    g = torch.Generator().manual_seed(8)
    mask = (torch.rand((B, H, 2, 16), generator=g) < 0.3).to(torch.uint8)
    o, lse = _run(q, k, v, False, 5, mask)
    assert_parity(o, lse, *_ref(q, k, v, False, mask))


def test_split_matches_unsplit():
    q, k, v = _case(1, 8, 64, 4096, 128, seed=6)
    o1, l1 = _run(q, k, v, False, 1)
    o8, l8 = _run(q, k, v, False, 8)
    assert np.max(np.abs(o1 - o8)) <= 2e-2 and np.max(np.abs(l1 - l8)) <= 1e-3


def test_workspace_errors():
    q, k, v = _case(1, 1, 1, 1024, 64, seed=7)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty((1, 1, 1), device=DEV)
    need = fa.fa_fwd_splitkv_workspace_bytes(1, 1, 1, 1024, 64, 4)
    assert need == 4 * 1 * 65 * 4
    small = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    args = (qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 1, 1, 1024,
            64, 0.125, 0, None)
    assert fa.fa_fwd_splitkv(*args, 4, small.data_ptr(), need - 16, s) == fa.FA_ERR_INVALID_ARGUMENT
    assert fa.fa_fwd_splitkv(*args, 4, None, 0, s) == fa.FA_ERR_INVALID_ARGUMENT
    assert fa.fa_fwd_splitkv(*args, 0, None, 0, s) == fa.FA_ERR_INVALID_ARGUMENT
    assert fa.fa_fwd_splitkv(*args, 1, None, 0, s) == fa.FA_OK  # one slice: no workspace
    torch.cuda.synchronize()
