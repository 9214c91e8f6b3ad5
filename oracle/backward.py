"""Oracle for the gradients of masked attention, in float64 (test infrastructure).

Test infrastructure only: imported by the tests, never by the CUDA path.

The pages say only that the score matrix is not stored but recomputed in the
backward pass, so memory stays O(n) ([UF] "瓦片注意力计算": the matrix is
needed for backpropagation and is recomputed there instead of kept).  The
gradients themselves are the plain chain rule through the definition of
attention used by ``attention_ref`` (for one (b, h), query rows i, keys j):

    S_ij = scale * q_i . k_j     (-inf where key j is not visible to query i)
    P_ij = exp(S_ij - lse_i)     (the softmax, from the forward's logsumexp)
    O_i  = sum_j P_ij v_j

Given the upstream gradient dO:

    dV_j  = sum_i P_ij dO_i
    dP_ij = dO_i . v_j
    D_i   = sum_j P_ij dP_ij = dO_i . O_i          (``softmax_delta``)
    dS_ij = P_ij (dP_ij - D_i)
    dQ_i  = scale * sum_j dS_ij k_j
    dK_j  = scale * sum_i dS_ij q_i

A row with no visible key (lse = -inf) has P = 0 and contributes nothing.
"""

from __future__ import annotations

import numpy as np

from .attention import MASK_BLOCK, _as64, visible_mask


def softmax_delta(o, do):
    """D_i = dO_i . O_i per query row (the row term of dS), float64.

    o, do: [..., rows, d]; returns [..., rows].  Equal to sum_j P_ij dP_ij
    because O_i = sum_j P_ij v_j and dP_ij = dO_i . v_j.
    """
    return np.sum(_as64(o) * _as64(do), axis=-1)


def attention_bwd_ref(q, k, v, do, scale, causal=False, block_mask=None, block=MASK_BLOCK,
                      row_chunk=1024):
    """dQ, dK, dV (float64) of attention at (q, k, v) for the upstream dO.

    q, do: [B, H, Nq, d]; k, v: [B, H, Nk, d]; masks as in ``attention_ref``.
    The softmax is formed from the definition (not from a supplied lse).
    Query rows are taken ``row_chunk`` at a time, each chunk holding complete
    rows of S: dQ of a row needs only its own row, and dK, dV are the sums
    over query rows written above, added up chunk by chunk.
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            bm = None if block_mask is None else np.asarray(block_mask)[b, h]
            for r0 in range(0, Nq, row_chunk):
                rows = np.arange(r0, min(Nq, r0 + row_chunk))
                qc, doc = q[b, h, rows], do[b, h, rows]
                s = scale * (qc @ k[b, h].T)
                vis = visible_mask(Nq, Nk, causal, bm, block, rows)
                s = np.where(vis, s, -np.inf)
                m = np.max(s, axis=1)
                empty = ~np.isfinite(m)
                e = np.exp(s - np.where(empty, 0.0, m)[:, None])
                den = np.sum(e, axis=1)
                p = e / np.where(empty, 1.0, den)[:, None]
                p[empty] = 0.0
                o = p @ v[b, h]
                dv[b, h] += p.T @ doc
                dp = doc @ v[b, h].T
                dd = softmax_delta(o, doc)
                ds = p * (dp - dd[:, None])
                dq[b, h, rows] = scale * (ds @ k[b, h])
                dk[b, h] += scale * (ds.T @ qc)
    return dq, dk, dv
