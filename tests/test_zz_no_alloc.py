"""fa_fwd_splitkv_noalloc: the split-key forward pass without a caller workspace.

Some callers cannot allocate device memory at the moment they call the
library. Examples: plugin code inside a host framework that owns every
allocation; latency-critical paths that must not pay for cudaMalloc; code
running while allocation is not allowed. For them the library keeps the
partial results of the split-key pass in one fixed array of its own device
memory (FA_NOALLOC_SCRATCH_BYTES), so the call allocates nothing.

The tests call the entry point through the C ABI:

* twice in a row, on different shapes and inputs; each result is compared
  with the workspace-taking fa_fwd_splitkv on the same inputs and with the
  float64 oracle, within the parity tolerances of the other GPU tests;
* after a first call, further calls leave torch's allocator statistics and
  the device's free memory unchanged;
* a problem whose partial results fill the array to within 1 KiB runs and
  matches; one query row more is refused before any launch.

This file is collected last. It passes alone in a fresh process and after
every other test.
"""

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
import oracle
from exact_attention_120_b200.workloads import make_qkv
from fa_helpers import TOL_LSE, TOL_O, assert_parity, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
SCRATCH_BYTES = 16 << 20  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def _inputs(B, H, Nq, Nk, d, seed):
    q, _, _ = make_qkv(B, H, Nq, d, seed, qk_std=2.0)
    _, k, v = make_qkv(B, H, Nk, d, seed + 1, qk_std=2.0)
    return q, k, v


def _noalloc(lib, q, k, v, causal, splits, o=None, lse=None):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if o is None:
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, Nq), float("nan"), device=DEV)
    st = lib.fa_fwd_splitkv_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                    lse.data_ptr(), B, H, Nq, Nk, d, 1.0 / d ** 0.5, int(causal),
                                    None, splits, torch.cuda.current_stream().cuda_stream)
    return st, o, lse


def _with_workspace(q, k, v, causal, splits):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    need = fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, splits)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=DEV)
    return fa.attention_forward_splitkv(q, k, v, causal=causal, num_splits=splits, workspace=ws)


def _check(lib, shape, seed):
    B, H, Nq, Nk, d, causal, splits = shape
    assert fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, splits) <= SCRATCH_BYTES
    q, k, v = _inputs(B, H, Nq, Nk, d, seed)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    st, o, lse = _noalloc(lib, qd, kd, vd, causal, splits)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    o_ws, lse_ws = _with_workspace(qd, kd, vd, causal, splits)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    o, lse, o_ws, lse_ws = to_np64(o), to_np64(lse), to_np64(o_ws), to_np64(lse_ws)
    # against the entry point that takes a workspace ...
    assert_parity(o, lse, o_ws, lse_ws, TOL_O, TOL_LSE)
    # ... and against the float64 oracle
    o_ref, lse_ref = oracle.attention_ref(to_np64(q), to_np64(k), to_np64(v), 1.0 / d ** 0.5,
                                          causal=causal)
    assert_parity(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("shapes", [
    # (B, H, Nq, Nk, d, causal, splits): decode against a cache, then a
    # prefill-sized problem with a different head dim, back to back
    [(2, 4, 1, 4096 + 33, 128, True, 8), (1, 2, 300, 1000, 64, False, 3)],
])
def test_noalloc_matches_workspace_entry_and_oracle_on_two_calls(shapes):
    lib = fa.load_library()
    for i, shape in enumerate(shapes):
        _check(lib, shape, seed=100 + i)


def test_noalloc_calls_allocate_nothing():
    lib = fa.load_library()
    B, H, Nq, Nk, d = 2, 4, 1, 4096 + 33, 128
    q, k, v = (t.to(DEV) for t in _inputs(B, H, Nq, Nk, d, seed=5))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), device=DEV)
    st, _, _ = _noalloc(lib, q, k, v, True, 8, o, lse)  # the first call may set up the device
    assert st == fa.FA_OK
    torch.cuda.synchronize()
    stats0 = torch.cuda.memory_stats(DEV)
    free0, _ = torch.cuda.mem_get_info(DEV)
    for splits in (8, 3):
        st, _, _ = _noalloc(lib, q, k, v, True, splits, o, lse)
        assert st == fa.FA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(DEV)
    stats1 = torch.cuda.memory_stats(DEV)
    assert free1 == free0, (free0, free1)
    for key in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current",
                "allocated_bytes.all.current"):
        assert stats1.get(key) == stats0.get(key), key
    assert fa.fa_device_status(None) == fa.FA_OK


def test_noalloc_at_the_limit_runs_and_one_row_more_is_refused():
    lib = fa.load_library()
    # 2 slices x 16256 rows x (128 + 1) floats = 16 MiB - 1 KiB
    B, H, Nq, Nk, d, splits = 1, 1, 16256, 256, 128, 2
    assert SCRATCH_BYTES - 1024 == fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, splits)
    _check(lib, (B, H, Nq, Nk, d, False, splits), seed=9)
    Nq += 1
    assert fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, splits) > SCRATCH_BYTES
    q, k, v = (t.to(DEV) for t in _inputs(B, H, Nq, Nk, d, seed=7))
    st, o, lse = _noalloc(lib, q, k, v, False, splits)
    assert st == fa.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.isnan(o).all() and torch.isnan(lse).all()  # nothing was launched
    assert fa.fa_device_status(None) == fa.FA_OK
