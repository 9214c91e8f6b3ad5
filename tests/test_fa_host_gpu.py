"""GPU tests of the host-buffer forward (fa_fwd_host): the chunked, overlapped
copies must give exactly the device entry point's results, and those agree
with the float64 oracle at the forward's bar (max|dO| <= 2e-2,
max|dlse| <= 1e-2)."""

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from exact_attention_120_b200.workloads import make_block_mask, make_qkv
from fa_helpers import assert_parity, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

# (B, H, N, d, causal, sparse_p): B*H of 1, of fewer heads than chunks, of
# more (an uneven last chunk), with and without masks.
CASES = [
    (1, 1, 128, 64, False, None),
    (2, 3, 300, 64, True, None),
    (1, 16, 1024, 128, True, None),
    (3, 5, 257, 128, False, 0.4),
    (2, 9, 640, 64, False, None),
]


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("case", range(len(CASES)))
def test_host_entry_equals_device_entry_bitwise(case):
    B, H, N, d, causal, sp = CASES[case]
    q, k, v = make_qkv(B, H, N, d, seed=40 + case)
    mask = None if sp is None else make_block_mask(B, H, N, sp, 41 + case).to(DEV)
    o_ref, l_ref = fa.attention_forward(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, block_mask=mask)
    torch.cuda.synchronize()
    bufs = tuple(torch.full_like(t, float("nan")) for t in (q.to(DEV), k.to(DEV), v.to(DEV), o_ref, l_ref))
    o, lse = fa.attention_forward_host(_pinned(q), _pinned(k), _pinned(v), causal=causal, block_mask=mask,
                                       device_buffers=bufs)
    assert fa.fa_device_status(None) == fa.FA_OK
    assert torch.equal(o, o_ref.cpu())
    assert torch.equal(lse, l_ref.cpu())
    # the device buffers hold the inputs and the results afterwards
    assert torch.equal(bufs[0].cpu(), q) and torch.equal(bufs[2].cpu(), v)
    assert torch.equal(bufs[3], o_ref) and torch.equal(bufs[4], l_ref)


def test_host_entry_against_oracle():
    B, H, N, d = 2, 5, 389, 128
    q, k, v = make_qkv(B, H, N, d, seed=47)
    o, lse = fa.attention_forward_host(_pinned(q), _pinned(k), _pinned(v), causal=True)
    o_ref, lse_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1.0 / np.sqrt(d), causal=True)
    assert_parity(to_np64(o), to_np64(lse), o_ref, lse_ref)


def test_host_entry_pageable_memory():
    # Pageable host tensors: the copies do not overlap, the results are the same.
    B, H, N, d = 1, 4, 512, 64
    q, k, v = make_qkv(B, H, N, d, seed=48)
    o_ref, l_ref = fa.attention_forward(q.to(DEV), k.to(DEV), v.to(DEV))
    out = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    lse = torch.empty((B, H, N), dtype=torch.float32)
    o, l_ = fa.attention_forward_host(q, k, v, out=out, lse=lse)
    assert o is out and l_ is lse
    assert torch.equal(out, o_ref.cpu()) and torch.equal(lse, l_ref.cpu())


def test_host_entry_back_to_back_on_one_stream():
    # Two calls through the same device buffers with no synchronisation in
    # between: the second call's copies in wait for the first call's copies
    # out, so each call returns its own results.
    B, H, N, d = 2, 8, 768, 128
    q1, k1, v1 = make_qkv(B, H, N, d, seed=49)
    q2, k2, v2 = make_qkv(B, H, N, d, seed=50)
    bufs = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=DEV) for _ in range(4))
    bufs = tuple(bufs) + (torch.empty((B, H, N), dtype=torch.float32, device=DEV),)
    # The host inputs must outlive the copies: hold them until the stream is done.
    h1 = [_pinned(t) for t in (q1, k1, v1)]
    h2 = [_pinned(t) for t in (q2, k2, v2)]
    o1, l1 = fa.attention_forward_host(*h1, device_buffers=bufs, synchronize=False)
    o2, l2 = fa.attention_forward_host(*h2, device_buffers=bufs, synchronize=False)
    torch.cuda.synchronize()
    for (q, k, v), o, l_ in (((q1, k1, v1), o1, l1), ((q2, k2, v2), o2, l2)):
        o_ref, l_ref = fa.attention_forward(q.to(DEV), k.to(DEV), v.to(DEV))
        assert torch.equal(o, o_ref.cpu()) and torch.equal(l_, l_ref.cpu())


def test_host_entry_rejects_swapped_memory_kinds():
    B, H, N, d = 1, 2, 128, 64
    qd = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device=DEV)
    od = torch.zeros_like(qd)
    ld = torch.zeros((B, H, N), dtype=torch.float32, device=DEV)
    qh = torch.zeros((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    oh = torch.zeros_like(qh).pin_memory()
    lh = torch.zeros((B, H, N), dtype=torch.float32).pin_memory()
    lib = fa.load_library()
    s = torch.cuda.current_stream().cuda_stream
    args = [qh.data_ptr()] * 3 + [oh.data_ptr(), lh.data_ptr()]
    dargs = [qd.data_ptr()] * 3 + [od.data_ptr(), ld.data_ptr()]
    tail = [B, H, N, d, 0.125, 0, None, s]
    assert lib.fa_fwd_host(*args, *dargs, *tail) == fa.FA_OK
    torch.cuda.synchronize()
    # a device pointer where host memory belongs, and the reverse
    assert lib.fa_fwd_host(qd.data_ptr(), *args[1:], *dargs, *tail) == fa.FA_ERR_INVALID_ARGUMENT
    assert lib.fa_fwd_host(*args, qh.data_ptr(), *dargs[1:], *tail) == fa.FA_ERR_INVALID_ARGUMENT


def test_host_entry_from_two_threads_on_two_streams():
    # Two host threads call at once, each with its own buffers and stream: the
    # calls share the library's copy streams (one call's enqueue is kept whole)
    # and each must return its own results.
    import threading

    B, H, N, d = 1, 6, 1024, 64
    jobs = []
    for seed in (51, 52):
        q, k, v = make_qkv(B, H, N, d, seed=seed)
        bufs = tuple(torch.empty((B, H, N, d), dtype=torch.bfloat16, device=DEV) for _ in range(4)) + (
            torch.empty((B, H, N), dtype=torch.float32, device=DEV),)
        out = (_pinned(torch.empty((B, H, N, d), dtype=torch.bfloat16)),
               _pinned(torch.empty((B, H, N), dtype=torch.float32)))
        jobs.append(dict(qkv=(q, k, v), host=[_pinned(t) for t in (q, k, v)], bufs=bufs,
                         stream=torch.cuda.Stream(DEV), out=out))

    def run(job):
        with torch.cuda.device(DEV):
            for _ in range(3):
                fa.attention_forward_host(*job["host"], out=job["out"][0], lse=job["out"][1],
                                          device_buffers=job["bufs"], stream=job["stream"].cuda_stream,
                                          synchronize=False)
            job["stream"].synchronize()

    threads = [threading.Thread(target=run, args=(j,)) for j in jobs]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    for job in jobs:
        q, k, v = job["qkv"]
        o_ref, l_ref = fa.attention_forward(q.to(DEV), k.to(DEV), v.to(DEV))
        o, l_ = job["out"]
        assert torch.equal(o, o_ref.cpu()) and torch.equal(l_, l_ref.cpu())
