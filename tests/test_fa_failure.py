"""Failure detection on the GPU without a GPU fault.

The kernel bounds every barrier wait.  The test entry point
fa_testing_fwd_starved launches it with the TMA producer issuing nothing and a
2 ms wait limit: the MMA issuer's first wait cannot complete, so the kernel
must take its timeout path.  It records FA_ERR_DEVICE_TIMEOUT, stops every
role, drains and frees tensor memory, and exits, leaving the context usable.
No trap, fault or hang is involved."""

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from fa_helpers import assert_parity, make_case, to_np64

pytestmark = pytest.mark.gpu


def _buffers(B, H, N, d):
    dev = torch.device("cuda", 0)
    q, k, v, _ = make_case(B, H, N, d, seed=21)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device=dev)
    return (q, k, v), (qd, kd, vd, o, lse)


@pytest.mark.parametrize("d", [64, 128])
def test_wait_timeout_is_reported_and_context_survives(d):
    B, H, N = 1, 2, 256
    (q, k, v), (qd, kd, vd, o, lse) = _buffers(B, H, N, d)
    lib = fa.load_library()
    s = torch.cuda.current_stream().cuda_stream
    assert fa.fa_device_status(s) == fa.FA_OK
    st = lib.fa_testing_fwd_starved(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                                    lse.data_ptr(), B, H, N, d, 1.0 / d ** 0.5, 0, None, s,
                                    2_000_000)
    assert st == fa.FA_OK
    torch.cuda.synchronize()  # no CUDA error: the kernel returned normally
    assert fa.fa_device_status(s) == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.fa_device_status(s) == fa.FA_OK  # reading clears it
    # The context is intact: a normal call right after is exact.
    fa.attention_forward(qd, kd, vd, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_device_status(s) == fa.FA_OK
    o_ref, l_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1.0 / d ** 0.5)
    assert_parity(to_np64(o), to_np64(lse), o_ref, l_ref)


def test_starved_entry_rejects_bad_limits():
    lib = fa.load_library()
    (_, _, _), (qd, kd, vd, o, lse) = _buffers(1, 1, 128, 64)
    args = (qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 1, 128,
            64, 0.125, 0, None, torch.cuda.current_stream().cuda_stream)
    assert lib.fa_testing_fwd_starved(*args, 0) == fa.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_testing_fwd_starved(*args, 5_000_000_000) == fa.FA_ERR_INVALID_ARGUMENT
