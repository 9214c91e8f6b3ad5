"""Oracle for the 8-bit (FP8 E4M3) forward pass, in float64 (test infrastructure).

Test infrastructure only: imported by the tests, never by the CUDA path.

The wmrh.cn article on FlashAttention (section "FlashAttention 的局限和后续发展")
names low-precision FP8 as the direction after FlashAttention-2.  What is
computed is still exact attention, of the real values the 8-bit codes stand
for: q = q_descale * decode(q8), and likewise k and v.  So the oracle is
``attention_ref`` on the decoded, descaled inputs.

``e4m3_decode`` writes out the OCP 8-bit floating-point format E4M3 (the
"fn" variant: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
no infinities, S.1111.111 = NaN, largest finite 448, subnormals down to
2^-9).  It is the format's definition, not a library conversion.

``weighted_spread`` gives, per query row i and output column t, the standard
deviation of V under the attention weights, sqrt(sum_j w_ij (v_jt - O_it)^2).
When every weight w_j is perturbed to w_j (1 + e_j) / sum_k w_k (1 + e_k) with
|e_j| <= u (rounding the weights' numerators to a u-precision format and
normalising by their rounded sum), O moves by at most u / (1 - u) times this
spread (Cauchy-Schwarz on sum_j w_j e_j (v_j - O)).  The tests use it to
bound the effect of rounding P to e4m3 (u = 2^-4).
"""

from __future__ import annotations

import math

import numpy as np

from .attention import MASK_BLOCK, _as64, attention_ref, visible_mask


def e4m3_decode(codes):
    """uint8 codes -> float64 values of OCP E4M3 (fn variant)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = sign * (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = sign * (m / 8.0) * 2.0 ** -6
    out = np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def attention_fp8_ref(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal=False,
                      block_mask=None, block=MASK_BLOCK):
    """O, lse (float64) of attention on the real values the codes stand for."""
    q = e4m3_decode(q8) * float(q_descale)
    k = e4m3_decode(k8) * float(k_descale)
    v = e4m3_decode(v8) * float(v_descale)
    return attention_ref(q, k, v, scale, causal=causal, block_mask=block_mask, block=block)


def weighted_spread(q, k, v, scale, causal=False, block_mask=None, block=MASK_BLOCK):
    """sqrt(sum_j w_ij (v_jt - O_it)^2) per (b, h, i, t), float64; 0 for empty rows."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, Nq, _ = q.shape
    Nk = k.shape[2]
    out = np.zeros((B, H, Nq, v.shape[-1]))
    for b in range(B):
        for h in range(H):
            bm = None if block_mask is None else np.asarray(block_mask)[b, h]
            s = scale * (q[b, h] @ k[b, h].T)
            s = np.where(visible_mask(Nq, Nk, causal, bm, block), s, -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            empty = ~np.isfinite(m[:, 0])
            w = np.exp(s - np.where(np.isfinite(m), m, 0.0))
            w = w / np.where(empty, 1.0, w.sum(axis=1))[:, None]
            w[empty] = 0.0
            o = w @ v[b, h]
            var = w @ (v[b, h] ** 2) - o ** 2
            out[b, h] = np.sqrt(np.maximum(var, 0.0))
    return out


E4M3_MAX = 448.0
E4M3_MIN_SUBNORMAL = math.ldexp(1.0, -9)
