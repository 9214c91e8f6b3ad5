"""The FMA-pipe exp2 of the kernel: its constants are the committed fit, and
the operation sequence it runs (emulated in NumPy float32) stays within a
relative error far below bf16 rounding over the argument range used."""

import os
import re

import numpy as np

from exact_attention_120_b200 import exp2_poly_fit as fitmod

KERNEL = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "exact_attention_120_b200", "csrc", "fa_fwd_kernel.cuh")


def _kernel_constants():
    text = open(KERNEL).read()
    out = {}
    for name in ("kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3", "kExp2Clamp", "kExp2Round"):
        m = re.search(name + r"\s*=\s*([-+0-9.eE]+)f", text)
        assert m, name
        out[name] = float(m.group(1))
    return out


def test_kernel_constants_match_fit():
    coef, rel = fitmod.fit()
    k = _kernel_constants()
    for i in range(4):
        assert np.float32(k[f"kExp2C{i}"]) == np.float32(coef[i])
    assert rel < 1e-4
    assert k["kExp2Clamp"] == fitmod.CLAMP
    assert k["kExp2Round"] == 1.5 * 2 ** 23


def test_emulated_sequence_error():
    x = np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32)
    y = fitmod.exp2_emulated(x)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4  # bf16 keeps 2^-9 ~ 2e-3


def test_integers_and_masked_arguments():
    y = fitmod.exp2_emulated(np.array([0.0, 1.0, -3.0, 8.0], np.float32))
    np.testing.assert_allclose(y, [1.0, 2.0, 0.125, 256.0], rtol=1e-4)
    tiny = fitmod.exp2_emulated(np.array([-np.inf, -1e30, -200.0], np.float32))
    assert np.all(np.isfinite(tiny)) and np.all(tiny > 0) and np.all(tiny < 1e-37)
