"""Seeded synthetic inputs for the attention forward pass.

This module only draws random numbers; it holds none of the method's
arithmetic.  The tests feed the same tensors to the CUDA path and to the CPU
oracle, and ``bench.py`` times the CUDA path on them.

Every tensor is drawn on the CPU with ``torch.Generator`` in float32 from
N(0, 1), multiplied by its standard deviation, then rounded to bfloat16
(round-to-nearest-even), in the order q, k, v.  Layout is [B, H, N, d],
contiguous, d fastest.

The workload shapes follow the pages' description of the problem: sequence
lengths from 128 to 16k, head dim 64 and 128, full, causal and block-sparse
attention.  "N(0,3)" for the long workload is read as standard deviation 3
(it is meant to widen the score range so the running max is rescaled often;
std 3 gives score std ~9 at scale 1/sqrt(d), variance 3 only ~3).
"""

from __future__ import annotations

import itertools
import math
from dataclasses import dataclass, field

import torch

MASK_BLOCK = 128


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool = False
    seed: int = 0
    qk_std: float = 1.0
    v_std: float = 1.0
    sparse_p: float | None = None  # keep probability of off-diagonal blocks
    mask_seed: int | None = None
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> str:
        parts = [f"B={self.B},H={self.H},N={self.N},d={self.d}"]
        parts.append("causal" if self.causal else "full")
        if self.sparse_p is not None:
            parts.append(f"block-sparse 128x128 diag+p={self.sparse_p}")
        if self.qk_std != 1.0:
            parts.append(f"Q,K std {self.qk_std}")
        return " ".join(parts)


# The five workloads: tiny full, small (full and causal), mid causal,
# long full with a wide score range, block-sparse.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 64, seed=0),
    "small": Workload("small", 4, 8, 1024, 64, seed=1),
    "small_causal": Workload("small_causal", 4, 8, 1024, 64, causal=True, seed=1),
    "mid_causal": Workload("mid_causal", 2, 16, 4096, 128, causal=True, seed=2),
    "long_full": Workload("long_full", 1, 16, 16384, 128, seed=3, qk_std=3.0),
    "sparse": Workload("sparse", 2, 16, 8192, 64, seed=4, sparse_p=0.25, mask_seed=4),
}


def make_qkv(B, H, N, d, seed, qk_std=1.0, v_std=1.0):
    """q, k, v as contiguous CPU bfloat16 tensors [B, H, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shape = (B, H, N, d)
    q = (torch.randn(shape, generator=g, dtype=torch.float32) * qk_std).to(torch.bfloat16)
    k = (torch.randn(shape, generator=g, dtype=torch.float32) * qk_std).to(torch.bfloat16)
    v = (torch.randn(shape, generator=g, dtype=torch.float32) * v_std).to(torch.bfloat16)
    return q, k, v


def make_block_mask(B, H, N, p, seed, block=MASK_BLOCK):
    """uint8 [B, H, nb, nb] block mask, nb = ceil(N / block), 1 = keep.

    One mask per head (diagonal blocks always kept, off-diagonal blocks kept
    independently with probability p), the same for every batch index.
    """
    nb = (N + block - 1) // block
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    keep = torch.rand((H, nb, nb), generator=g) < p
    keep |= torch.eye(nb, dtype=torch.bool).unsqueeze(0)
    return keep.to(torch.uint8).unsqueeze(0).expand(B, H, nb, nb).contiguous()


def make_inputs(w: Workload):
    """(q, k, v, block_mask or None) on the CPU for a workload."""
    q, k, v = make_qkv(w.B, w.H, w.N, w.d, w.seed, w.qk_std, w.v_std)
    mask = None
    if w.sparse_p is not None:
        mask = make_block_mask(w.B, w.H, w.N, w.sparse_p, w.mask_seed)
    return q, k, v, mask


def useful_flops(B, H, N, d, causal=False, block_mask=None):
    """FLOPs credited to one forward pass: 4*B*H*N^2*d, halved when causal,
    times the kept-block fraction when a block mask is given."""
    f = 4.0 * B * H * N * N * d
    if causal:
        f *= 0.5
    if block_mask is not None:
        f *= float(block_mask.to(torch.float64).mean())
    return f


def algorithmic_bytes(B, H, N, d):
    """HBM bytes of one forward pass if every tensor moves once:
    bf16 Q, K, V read and O written (8*N*d per head) plus fp32 lse (4*N)."""
    return float(B * H * (8 * N * d + 4 * N))


# ---------------------------------------------------------------- varlen ---
# Variable-length batches: sequences packed token-major ([T, H, d]) with int32
# offsets cu = [0, n_0, n_0 + n_1, ...].  The length mix is log-uniform, the
# shape of a batch of documents or prompts of very different sizes.


@dataclass(frozen=True)
class VarlenWorkload:
    name: str
    B: int          # sequences
    H: int
    d: int
    min_len: int
    max_len: int
    causal: bool = True
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> str:
        return (f"B={self.B} sequences, lengths log-uniform in [{self.min_len},{self.max_len}], "
                f"H={self.H}, d={self.d}, {'causal' if self.causal else 'full'}")


VARLEN_WORKLOADS = {
    "varlen_mix": VarlenWorkload("varlen_mix", 32, 16, 128, 128, 8192, causal=True, seed=5),
}


def varlen_lengths(B, lo, hi, seed):
    """B integer lengths, log-uniform in [lo, hi]."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    u = torch.rand(B, generator=g, dtype=torch.float64)
    n = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))
    return [int(x) for x in n.round().clamp(lo, hi).tolist()]


def make_varlen(lengths_q, lengths_k, H, d, seed, qk_std=1.0):
    """Packed bf16 q [Tq, H, d], k, v [Tk, H, d] and int32 offsets cu_q, cu_k
    (CPU), drawn like make_qkv in the order q, k, v."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    Tq, Tk = int(sum(lengths_q)), int(sum(lengths_k))
    q = (torch.randn((Tq, H, d), generator=g) * qk_std).to(torch.bfloat16)
    k = (torch.randn((Tk, H, d), generator=g) * qk_std).to(torch.bfloat16)
    v = torch.randn((Tk, H, d), generator=g).to(torch.bfloat16)
    cu = lambda ls: torch.tensor([0] + list(itertools.accumulate(ls)), dtype=torch.int32)  # noqa: E731
    return q, k, v, cu(lengths_q), cu(lengths_k)


def make_varlen_inputs(w: VarlenWorkload):
    lens = varlen_lengths(w.B, w.min_len, w.max_len, w.seed)
    return (lens,) + make_varlen(lens, lens, w.H, w.d, w.seed + 1)


def varlen_flops(lengths_q, lengths_k, H, d, causal):
    """Useful FLOPs: 4 d per visible (query, key) pair, per head (causal: key
    j visible to query i iff j <= i + nk - nq)."""
    f = 0.0
    for nq, nk in zip(lengths_q, lengths_k):
        if causal:
            off = nk - nq
            # sum over i of clamp(i + off + 1, 0, nk)
            vis = sum(min(max(i + off + 1, 0), nk) for i in range(nq))
        else:
            vis = nq * nk
        f += 4.0 * d * H * vis
    return f


# ------------------------------------------------------------------ fp8 ---
# 8-bit inputs: the same float32 draws as make_qkv, each tensor quantised to
# OCP E4M3 with one scale per tensor (amax / 448, so the largest magnitude
# maps to the format's largest finite value), rounding by PyTorch's
# float8_e4m3fn conversion.  Quantisation is the caller's step, not part of
# the attention being computed.


def make_qkv_fp8(B, H, N, d, seed, qk_std=1.0, v_std=1.0, Nk=None):
    """(q8, k8, v8) uint8 codes [B, H, N(k), d] on the CPU and their
    dequantisation scales (q_descale, k_descale, v_descale)."""
    Nk = N if Nk is None else Nk
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    xs = [torch.randn((B, H, N, d), generator=g) * qk_std,
          torch.randn((B, H, Nk, d), generator=g) * qk_std,
          torch.randn((B, H, Nk, d), generator=g) * v_std]
    codes, scales = [], []
    for x in xs:
        s = float(x.abs().max()) / 448.0
        codes.append((x / s).to(torch.float8_e4m3fn).view(torch.uint8).contiguous())
        scales.append(s)
    return tuple(codes), tuple(scales)
