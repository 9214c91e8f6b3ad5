"""Oracle for masked scaled-dot-product attention, in float64 (test infrastructure).

Test infrastructure only: imported by the tests and by bench.py's CPU-baseline
arm, never by the CUDA path (which shares no code with this file).

What is computed, and where it is stated
---------------------------------------
The method on the pages is *exact* attention ([WM] intro: it gives up no
accuracy; [WM] "2.1 Online Softmax": the online result is identical to safe
softmax).  So the oracle is the definition itself, not the tiled algorithm:

    S   = scale * Q K^T                          ([UF] "什么是注意力": softmax(QK^T/sqrt(d)) V;
                                                  the caller passes ``scale``)
    S_ij = -inf for keys j not visible to query i (causal: j <= i; block mask:
                                                  the 128x128 block (i//128, j//128) is kept)
    P   = safe softmax of each row of S           ([AY] "(Safe) Softmax", three passes)
    O   = P V,   lse_i = m_i + ln d_i             (natural log of sum_j exp(S_ij))

Readings where the pages are silent: ``lse`` is the natural-log logsumexp of
the *scaled* scores; a query row with no visible key has O = 0 and
lse = -inf; the causal rule is "key j visible to query i iff j <= i" with equal
query and key lengths; a masked block contributes nothing (its scores are -inf
before the softmax, not zero after it).

Inputs are converted exactly to float64 (bf16 and fp32 values are exactly
representable), so the oracle sees the very values the GPU reads.

``attention_tiled_online`` writes the pages' one-pass tiled algorithm in
float64 ([AY] "FlashAttention"; [WM] "2.2 把 Online Softmax 嵌入注意力": fix one
Q block, stream every K/V block, keep per-row m, l and an un-normalised output
that is corrected whenever the running max grows; [UF] "算法概述": one job per
Q block).  It exists so the tests can show that the algorithm reaches the
definition; the GPU parity tests compare against ``attention_ref``.
"""

from __future__ import annotations

import math

import numpy as np

from .softmax import merge_partials, partial_state

MASK_BLOCK = 128  # block size of the block-sparse mask (configs use 128x128 blocks)


def _as64(a):
    return np.asarray(a, dtype=np.float64)


def visible_mask(n_q, n_k, causal, block_mask_bh=None, block=MASK_BLOCK, rows=None):
    """Boolean [len(rows), n_k] visibility of keys for the given query rows.

    causal: key j visible to query i iff j <= i + (n_k - n_q), i.e. the
    diagonal is aligned to the last key (for n_q = n_k: j <= i; with fewer
    queries than keys the queries are the latest positions of the sequence).
    block_mask_bh: [ceil(n_q/block), ceil(n_k/block)] array, nonzero = the
    block of (query block, key block) is kept.  Both rules intersect.
    """
    if rows is None:
        rows = np.arange(n_q)
    rows = np.asarray(rows)
    cols = np.arange(n_k)
    vis = np.ones((rows.size, n_k), dtype=bool)
    if causal:
        vis &= cols[None, :] <= rows[:, None] + (n_k - n_q)
    if block_mask_bh is not None:
        bm = np.asarray(block_mask_bh) != 0
        vis &= bm[(rows // block)[:, None], (cols // block)[None, :]]
    return vis


def _softmax_rows_3pass(s):
    """Row-wise safe softmax of a [r, n] score block with -inf masks.

    Pass 1: m = row max.  Pass 2: d = sum exp(s - m).  Pass 3: p = exp(s - m)/d.
    Rows with no finite score give p = 0, m = -inf, d = 0.
    """
    m = np.max(s, axis=1)  # pass 1
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe[:, None])  # exp(-inf) = 0 for masked keys
    d = np.sum(e, axis=1)  # pass 2
    d_safe = np.where(empty, 1.0, d)
    p = e / d_safe[:, None]  # pass 3
    p[empty] = 0.0
    return p, m, np.where(empty, 0.0, d)


def _rows_of_head(qh, kh, vh, scale, causal, bm_bh, block, rows):
    """O and lse for the listed query rows of one (b, h), by the definition."""
    n_q, n_k = qh.shape[0], kh.shape[0]
    s = scale * (qh[rows] @ kh.T)  # S = scale * Q K^T for these rows
    vis = visible_mask(n_q, n_k, causal, bm_bh, block, rows)
    s = np.where(vis, s, -np.inf)
    p, m, d = _softmax_rows_3pass(s)
    o = p @ vh
    with np.errstate(divide="ignore"):
        lse = np.where(d > 0, m + np.log(np.where(d > 0, d, 1.0)), -np.inf)
    return o, lse


def attention_ref(q, k, v, scale, causal=False, block_mask=None, block=MASK_BLOCK, row_chunk=1024):
    """Full oracle: O [B,H,Nq,d] and lse [B,H,Nq], both float64.

    q: [B, H, Nq, d]; k, v: [B, H, Nk, d] (converted exactly to float64).
    block_mask: None or [B, H, ceil(Nq/block), ceil(Nk/block)], nonzero = keep.
    Rows are processed ``row_chunk`` at a time; each chunk holds complete
    rows of S, so the result is the definition, never an online update.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, N, d = q.shape  # N query rows; k and v may hold a different number of keys
    o = np.zeros((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            bm = None if block_mask is None else np.asarray(block_mask)[b, h]
            for r0 in range(0, N, row_chunk):
                rows = np.arange(r0, min(N, r0 + row_chunk))
                o[b, h, rows], lse[b, h, rows] = _rows_of_head(
                    q[b, h], k[b, h], v[b, h], scale, causal, bm, block, rows)
    return o, lse


def attention_ref_rows(q, k, v, scale, sample, causal=False, block_mask=None, block=MASK_BLOCK):
    """Oracle for sampled query rows of a large problem.

    sample: iterable of (b, h, i).  Returns (o [len, d], lse [len]) in the
    order given.  Same arithmetic as ``attention_ref``, restricted to rows.
    """
    sample = list(sample)
    out_o = np.zeros((len(sample), np.shape(v)[-1]), dtype=np.float64)
    out_l = np.zeros(len(sample), dtype=np.float64)
    groups = {}
    for idx, (b, h, i) in enumerate(sample):
        groups.setdefault((int(b), int(h)), []).append((idx, int(i)))
    for (b, h), items in groups.items():
        rows = np.array([i for _, i in items])
        bm = None if block_mask is None else np.asarray(block_mask)[b, h]
        o, l = _rows_of_head(_as64(q[b, h]), _as64(k[b, h]), _as64(v[b, h]),
                             scale, causal, bm, block, rows)
        for n, (idx, _) in enumerate(items):
            out_o[idx] = o[n]
            out_l[idx] = l[n]
    return out_o, out_l


def attention_tiled_online(q, k, v, scale, causal=False, block_mask=None, block=MASK_BLOCK,
                           bm=128, bn=128):
    """The one-pass tiled algorithm, in float64, in the pages' order.

    For each Q block of ``bm`` rows: start from (m, l, acc) = (-inf, 0, 0) per
    row; for each K/V block of ``bn`` keys compute that block's scores, its
    per-row state, and fold it into the running state with the concatenated-
    softmax rule (which is the "correct O with the new max" step of the
    pages).  At the end O = acc / l and lse = m + ln l.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, N, d = q.shape
    Nk = k.shape[2]
    dv = v.shape[-1]
    o = np.zeros((B, H, N, dv))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            bmask = None if block_mask is None else np.asarray(block_mask)[b, h]
            for q0 in range(0, N, bm):
                rows = np.arange(q0, min(N, q0 + bm))
                state = [(-math.inf, 0.0, np.zeros(dv)) for _ in rows]
                for k0 in range(0, Nk, bn):
                    cols = np.arange(k0, min(Nk, k0 + bn))
                    s = scale * (q[b, h, rows] @ k[b, h, cols].T)
                    vis = visible_mask(N, Nk, causal, bmask, block, rows)[:, cols]
                    s = np.where(vis, s, -np.inf)
                    for r in range(rows.size):
                        state[r] = merge_partials(state[r], partial_state(s[r], v[b, h, cols]))
                for r, i in enumerate(rows):
                    m, l, acc = state[r]
                    if l > 0:
                        o[b, h, i] = acc / l
                        lse[b, h, i] = m + math.log(l)
                    else:
                        lse[b, h, i] = -math.inf
    return o, lse
