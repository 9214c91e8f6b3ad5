"""GPU parity of the sm_100a kernel against the float64 oracle, through the C ABI.

Bar: max|dO| <= 2e-2 and max|dlse| <= 1e-2 (absolute, every compared element),
inputs bf16 drawn by the seeded generators shared with bench.py.  Small and
ragged shapes, and the full-size workloads in the launch configuration
bench.py times, are compared element by element on every row.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_120_b200 import (FA_OK, attention_forward, fa_device_status, fa_fwd,
                                      fa_fwd_stream)
from exact_attention_120_b200.workloads import WORKLOADS, make_block_mask, make_inputs, make_qkv
from fa_helpers import assert_parity, full_parity, make_case, oracle_full, run_cuda, to_np64

pytestmark = pytest.mark.gpu


def _status_ok():
    assert fa_device_status(None) == FA_OK


# ------------------------------------------------------- small, exhaustive --

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 256, 300, 513])
@pytest.mark.parametrize("mode", ["full", "causal"])
def test_shapes_dense(d, N, mode):
    q, k, v, _ = make_case(2, 3, N, d, seed=N * 7 + d)
    full_parity(q, k, v, causal=(mode == "causal"))
    _status_ok()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [200, 640, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_shapes_block_sparse(d, N, causal):
    q, k, v, mask = make_case(2, 2, N, d, seed=N + d, sparse_p=0.3)
    full_parity(q, k, v, causal=causal, mask=mask)
    _status_ok()


def test_wide_score_range_rescales():
    # std 3 inputs: the running max moves by many units of 2^8 across tiles.
    q, k, v, _ = make_case(1, 4, 1024, 128, seed=11, qk_std=3.0)
    full_parity(q, k, v)


@pytest.mark.parametrize("d", [64, 128])
def test_increasing_scores_force_rescale_every_tile(d):
    # Key norms grow along the sequence, so every new tile raises the max.
    B, H, N = 1, 2, 1024
    q, k, v, _ = make_case(B, H, N, d, seed=12)
    ramp = torch.linspace(0.2, 6.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float().abs() + 0.5).to(torch.bfloat16)
    k = k.float().abs().to(torch.bfloat16)
    full_parity(q, k, v)


@pytest.mark.parametrize("jump", [31.0, 80.0])
@pytest.mark.parametrize("causal", [False, True])
def test_row_max_jump_within_a_unit(jump, causal):
    # Keys of tile 3 score `jump` (log2 units) above everything before them:
    # 31 moves the reference after the tile (its P reaches 2^31), 80 exceeds
    # what one tile may absorb against the old reference and is redone.
    B, H, N, d = 1, 2, 896, 128
    q, k, v, _ = make_case(B, H, N, d, seed=21)
    scale = 1 / math.sqrt(d)
    q = torch.full((B, H, N, d), 8.0).to(torch.bfloat16)
    k = (k.float() * 0.1).to(torch.bfloat16)
    kval = jump / (math.log2(math.e) * scale * 8.0 * d)
    k[:, :, 3 * 128:3 * 128 + 5] = kval
    full_parity(q, k, v, causal=causal)


def test_empty_rows_and_empty_tiles():
    B, H, N, d = 1, 2, 600, 64
    q, k, v, mask = make_case(B, H, N, d, seed=13, sparse_p=0.5)
    mask[0, 0, 2, :] = 0          # query tile 2 of head 0 sees nothing
    mask[0, 1, 1, :] = 0
    mask[0, 1, 1, 3] = 1          # with causal, tile 1 of head 1 sees nothing
    for causal in (False, True):
        o, lse = run_cuda(q, k, v, causal, mask)
        o_ref, lse_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1 / 8,
                                              causal=causal, block_mask=mask.numpy())
        assert np.all(np.isneginf(lse[0, 0, 256:384]))
        assert not o[0, 0, 256:384].any()
        assert_parity(o, lse, o_ref, lse_ref)


def test_non_default_scale():
    q, k, v, _ = make_case(1, 2, 300, 64, seed=14)
    full_parity(q, k, v, causal=True, scale=0.37)


# ------------------------------------------- the five workloads ----------

def test_tiny_full():
    q, k, v, _ = make_inputs(WORKLOADS["tiny"])
    full_parity(q, k, v)


@pytest.mark.parametrize("name", ["small", "small_causal"])
def test_small_full_compare(name):
    w = WORKLOADS[name]
    q, k, v, _ = make_inputs(w)
    full_parity(q, k, v, causal=w.causal)


@pytest.mark.parametrize("name", ["mid_causal", "long_full", "sparse"])
def test_full_size_every_row(name):
    # The full-size workloads in the launch configuration bench.py times,
    # compared with the float64 oracle on every element of O and lse.
    w = WORKLOADS[name]
    q, k, v, mask = make_inputs(w)
    o, lse = run_cuda(q, k, v, w.causal, mask)
    _status_ok()
    o_ref, lse_ref = oracle_full(to_np64(q), to_np64(k), to_np64(v), w.scale, causal=w.causal,
                                 mask=None if mask is None else mask.numpy())
    assert_parity(o, lse, o_ref, lse_ref)


def test_legacy_default_stream_entry():
    # fa_fwd itself: the entry point without a stream argument launches on the
    # legacy default stream; torch.cuda.synchronize waits for the device.
    w = WORKLOADS["mid_causal"]
    B, H = 1, 3
    q, k, v = make_qkv(B, H, 1000, 128, seed=23)
    dev = torch.device("cuda", 0)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    torch.cuda.synchronize()
    for causal, mask in ((0, None), (1, None), (0, make_block_mask(B, H, 1000, 0.4, 5))):
        o = torch.full_like(qd, float("nan"))
        lse = torch.full((B, H, 1000), float("nan"), device=dev)
        md = None if mask is None else mask.to(dev)
        torch.cuda.synchronize()
        st = fa_fwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                    B, H, 1000, 128, w.scale, causal, None if md is None else md.data_ptr())
        assert st == FA_OK
        torch.cuda.synchronize()
        o_ref, lse_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), w.scale,
                                              causal=bool(causal),
                                              block_mask=None if mask is None else mask.numpy())
        assert_parity(to_np64(o), to_np64(lse), o_ref, lse_ref)
    _status_ok()


# ------------------------------------------------------ invariants --------

def test_constant_v_rows():
    B, H, N, d = 1, 2, 700, 128
    q, k, _, _ = make_case(B, H, N, d, seed=15, qk_std=2.0)
    c = torch.randn(d).to(torch.bfloat16)
    v = c.view(1, 1, 1, d).expand(B, H, N, d).contiguous()
    for causal in (False, True):
        o, _ = run_cuda(q, k, v, causal)
        assert np.max(np.abs(o - to_np64(c))) <= 2e-2


def test_zero_q_gives_means():
    B, H, N, d = 1, 1, 384, 64
    _, k, v, _ = make_case(B, H, N, d, seed=16)
    q = torch.zeros_like(k)
    o, lse = run_cuda(q, k, v, True)
    vv = to_np64(v)[0, 0]
    means = np.cumsum(vv, axis=0) / np.arange(1, N + 1)[:, None]
    assert np.max(np.abs(o[0, 0] - means)) <= 2e-2
    assert np.max(np.abs(lse[0, 0] - np.log(np.arange(1, N + 1)))) <= 1e-2


def test_query_permutation_permutes_rows():
    B, H, N, d = 1, 2, 256, 64
    q, k, v, _ = make_case(B, H, N, d, seed=17)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(3))
    o1, l1 = run_cuda(q, k, v)
    o2, l2 = run_cuda(q[:, :, perm].contiguous(), k, v)
    assert np.array_equal(o2, o1[:, :, perm.numpy()])
    assert np.array_equal(l2, l1[:, :, perm.numpy()])


def test_deterministic():
    q, k, v, mask = make_case(2, 2, 1000, 128, seed=18, sparse_p=0.4)
    a = run_cuda(q, k, v, True, mask)
    b = run_cuda(q, k, v, True, mask)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------------------------------------ memory safety (canaries) ------

def test_outputs_fully_written_and_bounds_kept():
    B, H, N, d = 2, 3, 333, 128
    q, k, v, _ = make_case(B, H, N, d, seed=19)
    dev = torch.device("cuda", 0)
    pad = 4096
    o_buf = torch.full((pad + B * H * N * d + pad,), float("nan"), dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((pad + B * H * N + pad,), float("nan"), dtype=torch.float32, device=dev)
    o_buf[:pad] = 7.0
    o_buf[-pad:] = 7.0
    l_buf[:pad] = 7.0
    l_buf[-pad:] = 7.0
    o = o_buf[pad:pad + B * H * N * d].view(B, H, N, d)
    lse = l_buf[pad:pad + B * H * N].view(B, H, N)
    attention_forward(q.to(dev), k.to(dev), v.to(dev), out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(o_buf[:pad] == 7.0) and torch.all(o_buf[-pad:] == 7.0)
    assert torch.all(l_buf[:pad] == 7.0) and torch.all(l_buf[-pad:] == 7.0)
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()


# --------------------------------------------------- argument errors ------

def test_errors_launch_nothing():
    dev = torch.device("cuda", 0)
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device=dev)
    o = torch.full_like(q, 3.0)
    lse = torch.full((1, 1, 128), 3.0, device=dev)
    p = q.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    cases = [
        ((0, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 128, 64, 0.1, 0, None), 1),
        ((p, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 128, 96, 0.1, 0, None), 2),
        ((p, p, p, o.data_ptr(), lse.data_ptr(), 0, 1, 128, 64, 0.1, 0, None), 1),
        ((p, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 128, 64, float("nan"), 0, None), 1),
        ((p, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 128, 64, -1.0, 0, None), 1),
        ((p, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 128, 64, 0.1, 2, None), 1),
        ((p + 2, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 64, 64, 0.1, 0, None), 1),
        ((p, p, p, p, lse.data_ptr(), 1, 1, 128, 64, 0.1, 0, None), 1),
    ]
    host = torch.zeros(128 * 64, dtype=torch.bfloat16)
    cases.append(((host.data_ptr(), p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 128, 64, 0.1, 0, None), 1))
    for args, want in cases:
        assert fa_fwd_stream(*args, s) == want, args
    torch.cuda.synchronize()
    assert torch.all(o == 3.0) and torch.all(lse == 3.0)
    _status_ok()
