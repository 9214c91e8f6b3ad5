"""fa_fwd_splitkv_noalloc: the split-key forward pass without a caller workspace.

Some callers cannot allocate device memory at the moment they call the
library. Examples: plugin code inside a host framework that owns every
allocation; latency-critical paths that must not pay for cudaMalloc; code
running while allocation is not allowed. For them the library keeps the
partial results of the split-key pass in one fixed array of its own device
memory (FA_NOALLOC_SCRATCH_BYTES), so the call allocates nothing.

The test calls the entry point through the C ABI twice in a row, on different
shapes and inputs. Each result is compared with the workspace-taking
fa_fwd_splitkv on the same inputs, within the parity tolerances of the other
GPU tests. A problem too large for the array must be refused before any
launch. This file is collected last. It passes alone in a fresh process and
after every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import exact_attention_120_b200 as fa
from exact_attention_120_b200.workloads import make_qkv
from fa_helpers import TOL_LSE, TOL_O, to_np64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
SCRATCH_BYTES = 16 << 20  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def _inputs(B, H, Nq, Nk, d, seed):
    q, _, _ = make_qkv(B, H, Nq, d, seed, qk_std=2.0)
    _, k, v = make_qkv(B, H, Nk, d, seed + 1, qk_std=2.0)
    return q.to(DEV), k.to(DEV), v.to(DEV)


def _noalloc(lib, q, k, v, causal, splits):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
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


@pytest.mark.parametrize("shape", [
    # (B, H, Nq, Nk, d, causal, splits): decode against a cache, then a
    # prefill-sized problem with a different head dim, back to back
    [(2, 4, 1, 4096 + 33, 128, True, 8), (1, 2, 300, 1000, 64, False, 3)],
])
def test_noalloc_matches_workspace_entry_on_two_calls(shape):
    lib = fa.load_library()
    for i, (B, H, Nq, Nk, d, causal, splits) in enumerate(shape):
        assert fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, splits) <= SCRATCH_BYTES
        q, k, v = _inputs(B, H, Nq, Nk, d, seed=100 + i)
        st, o, lse = _noalloc(lib, q, k, v, causal, splits)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        o_ref, lse_ref = _with_workspace(q, k, v, causal, splits)
        torch.cuda.synchronize()
        assert fa.fa_device_status(None) == fa.FA_OK
        o, lse, o_ref, lse_ref = to_np64(o), to_np64(lse), to_np64(o_ref), to_np64(lse_ref)
        assert np.all(np.isfinite(o))
        assert np.max(np.abs(o - o_ref)) <= TOL_O
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lse), fin)
        assert np.max(np.abs(lse[fin] - lse_ref[fin])) <= TOL_LSE


def test_noalloc_refuses_problems_beyond_its_array():
    lib = fa.load_library()
    B, H, Nq, Nk, d, splits = 1, 1, 65536, 256, 128, 2
    need = fa.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, splits)
    assert need > SCRATCH_BYTES
    q, k, v = _inputs(B, H, Nq, Nk, d, seed=7)
    st, _, _ = _noalloc(lib, q, k, v, False, splits)
    assert st == fa.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
