"""Oracle for variable-length batches, in float64 (test infrastructure).

Test infrastructure only: imported by the tests, never by the CUDA path.

A variable-length batch is B independent attention problems stored back to
back without padding (token-major [T, H, d], the layout of packed token
streams).  Sequence b owns query rows cu_q[b]:cu_q[b+1] and key rows
cu_k[b]:cu_k[b+1]; its queries see only its own keys.  Each sequence is the
attention of ``attention_ref`` ([UF] "什么是注意力": softmax(scale Q K^T) V per
head) with the same causal rule (diagonal aligned to the last key, key j
visible to query i iff j <= i + (nk - nq)).  The pages treat one sequence;
batching unequal lengths is the plainest extension: nothing couples two
sequences.  lse is returned head-major, [H, T].
"""

from __future__ import annotations

import numpy as np

from .attention import _as64, attention_ref


def attention_varlen_ref(q, k, v, cu_q, cu_k, scale, causal=False):
    """q: [Tq, H, d]; k, v: [Tk, H, d]; cu_q, cu_k: B+1 offsets.
    Returns (O [Tq, H, d], lse [H, Tq]) in float64."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    if len(cu_q) != len(cu_k) or cu_q[0] != 0 or cu_k[0] != 0:
        raise ValueError("cu_q and cu_k need B+1 offsets starting at 0")
    if cu_q[-1] != q.shape[0] or cu_k[-1] != k.shape[0]:
        raise ValueError("the last offsets must equal the token counts")
    if any(b < a for a, b in zip(cu_q, cu_q[1:])) or any(b < a for a, b in zip(cu_k, cu_k[1:])):
        raise ValueError("offsets must not decrease")
    Tq, H, d = q.shape
    o = np.zeros((Tq, H, v.shape[2]))
    lse = np.full((H, Tq), -np.inf)
    for b in range(len(cu_q) - 1):
        qa, qb, ka, kb = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if qb == qa:
            continue
        if kb == ka:  # no key at all: every row is empty
            continue
        # [n, H, d] -> [1, H, n, d]
        qs = q[qa:qb].transpose(1, 0, 2)[None]
        ks = k[ka:kb].transpose(1, 0, 2)[None]
        vs = v[ka:kb].transpose(1, 0, 2)[None]
        ob, lb = attention_ref(qs, ks, vs, scale, causal=causal)
        o[qa:qb] = ob[0].transpose(1, 0, 2)
        lse[:, qa:qb] = lb[0]
    return o, lse
