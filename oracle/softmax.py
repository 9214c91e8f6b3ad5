"""Softmax building blocks of the oracle, in float64 (test infrastructure).

Test infrastructure only: imported by the tests and by bench.py's CPU-baseline
arm, never by the CUDA path.

Each function follows the page that states it:

* ``safe_softmax_3pass``   -- [AY] "(Safe) Softmax": one pass for the maximum
  m_N, one for the denominator d_N = sum_j exp(x_j - m_N), one for the outputs
  a_i = exp(x_i - m_N) / d_N.  This is the plain definition of softmax made
  overflow-free by the shift invariance that [UF] "瓦片注意力计算" states.
* ``online_softmax_2pass`` -- [AY] "从3-pass到2-pass" and [WM] "2.1 Online
  Softmax": the running maximum m_i = max(m_{i-1}, x_i) and the running
  denominator d'_i = d'_{i-1} * exp(m_{i-1} - m_i) + exp(x_i - m_i), so that
  d'_N = d_N; a second pass then forms the outputs.  The page's printed
  correction factor is garbled in extraction; the factor exp(m_{i-1} - m_i) is
  the only one for which the page's own claim d'_N = d_N holds, and it is the
  reading taken here.
* ``merge_partials``       -- [UF] "瓦片注意力计算": the softmax denominator of
  a concatenation [x1, x2] from the two parts' maxima and denominators,
  m = max(m(x1), m(x2)), l = exp(m(x1) - m) l(x1) + exp(m(x2) - m) l(x2);
  because P V is linear the same rescaling carries the un-normalised output
  accumulators.

A row with no finite entry (every key masked) has m = -inf and d = 0; its
softmax is defined here as all zeros (the pages never reach that case).
"""

from __future__ import annotations

import math

import numpy as np


def safe_softmax_3pass(x):
    """Return (a, m_N, d_N) for a 1-D vector x, in float64.

    Pass 1: m_N = max_j x_j.  Pass 2: d_N = sum_j exp(x_j - m_N).
    Pass 3: a_i = exp(x_i - m_N) / d_N.  ([AY] "(Safe) Softmax".)
    """
    x = np.asarray(x, dtype=np.float64)
    m = -math.inf
    for xj in x:  # pass 1
        if xj > m:
            m = float(xj)
    if m == -math.inf:
        return np.zeros_like(x), m, 0.0
    d = float(np.sum(np.exp(x - m)))  # pass 2
    a = np.exp(x - m) / d  # pass 3
    return a, m, d


def online_softmax_2pass(x):
    """Return (a, m_N, d'_N, trace) for a 1-D vector x, in float64.

    Pass 1 walks x once, keeping the running max m_i and the running
    denominator d'_i = d'_{i-1} * exp(m_{i-1} - m_i) + exp(x_i - m_i)
    ([AY] "从3-pass到2-pass"; [WM] "2.1 Online Softmax").  ``trace`` lists the
    state (m_i, d'_i) after each element, as in the page's worked example.
    Pass 2 forms a_i = exp(x_i - m_N) / d'_N.
    """
    x = np.asarray(x, dtype=np.float64)
    m_prev, d_prev = -math.inf, 0.0
    trace = []
    for xi in x:
        m_i = max(m_prev, float(xi))
        if m_i == -math.inf:  # nothing finite seen yet
            d_i = 0.0
        else:
            rescale = math.exp(m_prev - m_i) if m_prev != -math.inf else 0.0
            d_i = d_prev * rescale + math.exp(float(xi) - m_i)
        trace.append((m_i, d_i))
        m_prev, d_prev = m_i, d_i
    if m_prev == -math.inf:
        return np.zeros_like(x), m_prev, 0.0, trace
    a = np.exp(x - m_prev) / d_prev
    return a, m_prev, d_prev, trace


def partial_state(s, v):
    """Un-normalised softmax state of one block of keys for one query row.

    s: scores of the block, shape [n] (masked keys as -inf); v: values [n, d].
    Returns (m, l, acc) with m = max s, l = sum exp(s - m),
    acc = sum_j exp(s_j - m) v_j.  An all-masked block gives (-inf, 0, 0).
    """
    s = np.asarray(s, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    m = float(np.max(s)) if s.size else -math.inf
    if m == -math.inf:
        return m, 0.0, np.zeros(v.shape[1:], dtype=np.float64)
    w = np.exp(s - m)
    return m, float(np.sum(w)), w @ v


def merge_partials(p1, p2):
    """Concatenated-softmax rule of [UF] "瓦片注意力计算".

    (m1, l1, acc1) and (m2, l2, acc2) are the states of two disjoint key sets;
    the state of their union is m = max(m1, m2),
    l = exp(m1 - m) l1 + exp(m2 - m) l2, acc = exp(m1 - m) acc1 + exp(m2 - m) acc2.
    """
    m1, l1, a1 = p1
    m2, l2, a2 = p2
    m = max(m1, m2)
    if m == -math.inf:
        return m, 0.0, np.zeros_like(np.asarray(a1, dtype=np.float64))
    f1 = math.exp(m1 - m) if m1 != -math.inf else 0.0
    f2 = math.exp(m2 - m) if m2 != -math.inf else 0.0
    return m, f1 * l1 + f2 * l2, f1 * np.asarray(a1) + f2 * np.asarray(a2)
