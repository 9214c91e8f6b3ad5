"""Pure-Python brute-force attention for tiny shapes (test infrastructure).

Test infrastructure only.  Written independently of ``attention_ref``: nested
loops, ``math.exp`` and ``math.fsum`` (exactly rounded sums), no NumPy
arithmetic.  It computes, for every query row i of every (b, h),

    s_ij = scale * sum_t q_it k_jt              for visible keys j
    w_ij = exp(s_ij - max_j s_ij)
    O_i  = sum_j w_ij v_j / sum_j w_ij,   lse_i = max_j s_ij + ln(sum_j w_ij)

with visibility j <= i + (Nk - N) when causal (N queries, Nk keys: the
diagonal is aligned to the last key) and the 128x128 (or ``block``-sized) block
(i // block, j // block) kept when a block mask is given -- the definition of
attention in [UF] "什么是注意力" with the safe softmax of [AY] "(Safe) Softmax".
A row with no visible key gives O_i = 0 and lse_i = -inf.
"""

from __future__ import annotations

import math


def attention_brute(q, k, v, scale, causal=False, block_mask=None, block=128):
    """q: nested lists [B][H][N][d]; k, v: [B][H][Nk][d].  Returns (O, lse) as lists."""
    B, H, N = len(q), len(q[0]), len(q[0][0])
    Nk = len(k[0][0])
    out_o, out_l = [], []
    for b in range(B):
        ob, lb = [], []
        for h in range(H):
            oh, lh = [], []
            for i in range(N):
                keys = []
                for j in range(Nk):
                    if causal and j - (Nk - N) > i:  # diagonal aligned to the last key
                        continue
                    if block_mask is not None and not block_mask[b][h][i // block][j // block]:
                        continue
                    keys.append(j)
                dv = len(v[b][h][0])
                if not keys:
                    oh.append([0.0] * dv)
                    lh.append(-math.inf)
                    continue
                s = {}
                for j in keys:
                    s[j] = scale * math.fsum(float(q[b][h][i][t]) * float(k[b][h][j][t])
                                             for t in range(len(q[b][h][i])))
                mx = max(s.values())
                w = {j: math.exp(s[j] - mx) for j in keys}
                den = math.fsum(w.values())
                oh.append([math.fsum(w[j] * float(v[b][h][j][t]) for j in keys) / den
                           for t in range(dv)])
                lh.append(mx + math.log(den))
            ob.append(oh)
            lb.append(lh)
        out_o.append(ob)
        out_l.append(lb)
    return out_o, out_l
