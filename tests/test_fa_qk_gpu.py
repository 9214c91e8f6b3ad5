"""GPU parity for different query and key lengths (fa_fwd_qk): cross-attention
and decoding against a key/value cache, causal diagonal aligned to the last
key, against the float64 oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_120_b200 import FA_OK, fa_device_status
from exact_attention_120_b200.workloads import make_qkv
from fa_helpers import assert_parity, run_cuda, to_np64

pytestmark = pytest.mark.gpu


def _qk_case(B, H, Nq, Nk, d, seed, std=1.0):
    q, _, _ = make_qkv(B, H, Nq, d, seed, qk_std=std)
    _, k, v = make_qkv(B, H, Nk, d, seed + 1, qk_std=std)
    return q, k, v


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("nq,nk", [(1, 1000), (7, 300), (128, 1024), (200, 129), (300, 700),
                                   (513, 256), (1000, 1000)])
@pytest.mark.parametrize("causal", [False, True])
def test_qk_lengths(d, nq, nk, causal):
    q, k, v = _qk_case(2, 2, nq, nk, d, seed=nq + 3 * nk + d)
    o, lse = run_cuda(q, k, v, causal)
    o_ref, l_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1 / math.sqrt(d),
                                        causal=causal)
    assert_parity(o, lse, o_ref, l_ref)
    assert fa_device_status(None) == FA_OK


@pytest.mark.parametrize("causal", [False, True])
def test_qk_block_sparse(causal):
    B, H, nq, nk, d = 2, 2, 300, 900, 64
    q, k, v = _qk_case(B, H, nq, nk, d, seed=5)
    g = torch.Generator().manual_seed(6)
    mask = (torch.rand((B, H, 3, 8), generator=g) < 0.4).to(torch.uint8)
    o, lse = run_cuda(q, k, v, causal, mask)
    o_ref, l_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1 / 8, causal=causal,
                                        block_mask=mask.numpy())
    assert_parity(o, lse, o_ref, l_ref)


def test_more_queries_than_keys_causal_empty_rows():
    q, k, v = _qk_case(1, 2, 400, 150, 128, seed=9)
    o, lse = run_cuda(q, k, v, True)
    assert np.all(np.isneginf(lse[:, :, :250])) and not o[:, :, :250].any()
    o_ref, l_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1 / math.sqrt(128),
                                        causal=True)
    assert_parity(o, lse, o_ref, l_ref)


def test_decode_long_cache():
    # one new query per sequence against a 16k-key cache
    q, k, v = _qk_case(4, 8, 1, 16384, 128, seed=10, std=2.0)
    o, lse = run_cuda(q, k, v, True)
    o_ref, l_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1 / math.sqrt(128),
                                        causal=True)
    assert_parity(o, lse, o_ref, l_ref)
