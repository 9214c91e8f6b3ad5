#!/usr/bin/env python
"""Benchmark of the fused attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--pass fwd|bwd]

One step = one fa_fwd launch over one batch of the workload (default: the
long full-attention workload B=1, H=16, N=16384, d=128, Q/K std 3 -- the
d=128, N>=4096 full-attention case the throughput target is stated on).
Inputs are seeded and synthetic, resident in HBM when the timed region starts,
and larger than L2 (Q, K, V, O = 256 MB per step), so no L2 flush is needed.

Rank 0 prints ONE JSON line.  ``value`` is the whole-job TFLOP/s (useful
FLOPs 4*B*H*N^2*d, halved when causal, times the kept-block fraction when
block-sparse), timed with CUDA events on the launching stream, max over
ranks.  ``e2e`` times the same metric through the public API with pinned host
buffers, copies included.  ``roofline`` relates the kernel to the measured
dense-bf16 tensor peak.  ``cpu_baseline`` times the float64 CPU oracle on a
bounded sample of the same workload.  ``--impl reference`` times that oracle
alone as the reference arm.

``--pass bwd`` times fa_bwd (dQ, dK, dV from the forward's O and lse) on the
same workload instead, credited with 2.5x the forward's FLOPs.  ``--pass
varlen`` times fa_fwd_varlen on varlen_mix (32 causal sequences of 128 to 8192
tokens packed without padding, H=16, d=128).  ``--pass fp8`` times fa_fwd_fp8
on the workload's shape with Q, K, V quantised to E4M3.

Multi-GPU (launched by torchrun): ranks share nothing on the data path; each
rank runs the full workload shape on its own batch slice (weak scaling).
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_attention_120_b200 import sharding  # noqa: E402
from exact_attention_120_b200.workloads import (VARLEN_WORKLOADS, WORKLOADS, algorithmic_bytes,  # noqa: E402
                                                make_inputs, make_qkv_fp8, make_varlen_inputs,
                                                useful_flops, varlen_flops)

METRIC = "fused attention fwd TFLOP/s (bf16, causal & full) and % of dense BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAK_TFLOPS = 1590.0
KERNEL_SOURCES = ("exact_attention_120_b200/csrc/fa_fwd_kernel.cuh",
                  "exact_attention_120_b200/csrc/ptx.cuh",
                  "exact_attention_120_b200/csrc/fa_api.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")

THROTTLE_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), \
            "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_PEAK_TFLOPS, 1400.0, "fallback"


def kernel_hash(sources=KERNEL_SOURCES) -> str:
    """Hash of the kernel sources' code: comments and whitespace are dropped,
    so a comment edit keeps the recorded counters while any code change
    invalidates them."""
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_traffic(workload: str, pass_: str = "fwd", khash: str | None = None):
    """DRAM bytes per launch from the committed ncu summary, only if it was
    taken on the current kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(workload if pass_ == "fwd" else f"{pass_}:{workload}")
    if not entry or entry.get("kernel_hash") != (khash or kernel_hash()):
        return None
    return float(entry["dram_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    def __init__(self, torch_device, period_s=0.02):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml

            pynvml.nvmlInit()
            props = __import__("torch").cuda.get_device_properties(torch_device)
            bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                        props.pci_device_id)
            try:
                self._handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except pynvml.NVMLError:
                self._handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: clocks reported as unknown
            self._handle = None

    def _run(self):
        nv = self._nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self._handle))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        names = sorted(n for bit, n in THROTTLE_BITS.items() if self.reasons & bit and n != "gpu_idle")
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(w, q, k, v, mask, rows_per_chunk, budget_s=None, max_chunks=None, start=0,
                  keep=None):
    """Time the float64 oracle on successive chunks of query rows of the
    workload (head-major order), until `budget_s` seconds or `max_chunks`.
    Returns (useful_flops, seconds, rows).  With a list `keep`, appends each
    chunk's (sample, o, lse) to it."""
    import numpy as np

    import oracle

    total_rows = w.B * w.H * w.N
    flops = 0.0
    rows_done = 0
    t_total = 0.0
    chunk = 0
    while True:
        r0 = (start + chunk * rows_per_chunk) % total_rows
        idx = [(r0 + i) % total_rows for i in range(rows_per_chunk)]
        sample = [(i // (w.H * w.N), (i // w.N) % w.H, i % w.N) for i in idx]
        t0 = time.perf_counter()
        ref = oracle.attention_ref_rows(q, k, v, w.scale, sample, causal=w.causal,
                                        block_mask=None if mask is None else mask)
        t_total += time.perf_counter() - t0
        if keep is not None:
            keep.append((sample, ref[0], ref[1]))
        for (b, h, i) in sample:
            vis = oracle.visible_mask(w.N, w.N, w.causal,
                                      None if mask is None else mask[b, h], rows=np.array([i]))
            flops += 4.0 * w.d * float(vis.sum())
        rows_done += len(sample)
        chunk += 1
        if (budget_s is not None and t_total >= budget_s) or (max_chunks is not None and chunk >= max_chunks):
            break
    return flops, t_total, rows_done


def numpy_inputs(q, k, v, mask):
    import torch

    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731  exact bf16 -> fp64
    return f(q), f(k), f(v), (None if mask is None else mask.numpy())


def run_reference(args, info):
    """Reference arm: the float64 CPU oracle as it stands, on host cores."""
    if not info.is_root:
        return 0
    w = WORKLOADS[args.workload]
    q, k, v, mask = make_inputs(w)
    qn, kn, vn, mn = numpy_inputs(q, k, v, mask)
    rows = args.reference_rows
    cores = blas_threads()
    oracle_sample(w, qn, kn, vn, mn, rows, max_chunks=max(1, args.warmup))  # warm-up
    step_s, step_f = [], []
    for s in range(args.steps):
        f, t, _ = oracle_sample(w, qn, kn, vn, mn, rows, max_chunks=1, start=(s + 1) * rows * 7)
        step_f.append(f)
        step_s.append(t)
    value = sum(step_f) / sum(step_s) / 1e12
    sample = (f"{rows} query rows per step (complete rows of S over all N={w.N} keys), "
              f"head-major order; float64 NumPy/BLAS oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": info.world_size,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(step_s) / len(step_s),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, info.world_size),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(info, line)
    return 0


def workload_config(w, world):
    return {"workload": f"{w.name}: {w.describe()}, scale 1/sqrt(d), seed {w.seed}",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "block_sparse": w.sparse_p is not None, "global_batch": w.B * world, "seq_len": w.N,
            "parallelism": "replicas" if world == 1 else f"dp{world} (independent batch slices)",
            "l2": "inputs larger than L2 (Q, K, V, O = %d MB per step); no flush"
                  % (algorithmic_bytes(w.B, w.H, w.N, w.d) // 2**20)}


def bwd_oracle_sample(w, q, k, v, mask, n_max=2048):
    """Time the float64 gradient oracle on head (0, 0) of the workload cut to
    its first n_max queries and keys.  Returns (credited_flops, seconds, n)."""
    import numpy as np
    import torch

    import oracle

    n = min(w.N, n_max)
    f = lambda t: t[0:1, 0:1, :n].to(torch.float64).numpy()  # noqa: E731
    g = torch.Generator().manual_seed(w.seed + 7)
    do = torch.randn((1, 1, n, w.d), generator=g).to(torch.bfloat16)
    bm = None
    if mask is not None:
        nb = (n + 127) // 128
        bm = np.ascontiguousarray(mask[0:1, 0:1, :nb, :nb].numpy())
    t0 = time.perf_counter()
    oracle.attention_bwd_ref(f(q), f(k), f(v), f(do), w.scale, causal=w.causal, block_mask=bm)
    t = time.perf_counter() - t0
    flops = 2.5 * useful_flops(1, 1, n, w.d, w.causal, None if bm is None else torch.from_numpy(bm))
    return flops, t, n


class FwdJob:
    """One step = one fa_fwd launch (one forward pass over the workload)."""

    name = "fwd"
    e2e_entry = "attention_forward_host (fa_fwd_host: chunked copies overlapping the kernels)"
    metric = METRIC
    kernel_sources = KERNEL_SOURCES

    def __init__(self, fa, torch, w, q, k, v, mask, dev, stream):
        self.fa, self.w = fa, w
        self.flops = useful_flops(w.B, w.H, w.N, w.d, w.causal, mask)
        self.q, self.k, self.v, self.mask = q, k, v, mask
        self.qd, self.kd, self.vd = q.to(dev), k.to(dev), v.to(dev)
        self.md = None if mask is None else mask.to(dev)
        self.od = torch.empty_like(self.qd)
        self.ld = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        self.stream = stream
        self.ptrs = (self.qd.data_ptr(), self.kd.data_ptr(), self.vd.data_ptr(),
                     self.od.data_ptr(), self.ld.data_ptr())
        self.mptr = None if self.md is None else self.md.data_ptr()
        self.launches_per_step = fa.fa_launches_per_call()

    def launch(self):
        w, fa = self.w, self.fa
        st = fa.fa_fwd_stream(*self.ptrs, w.B, w.H, w.N, w.d, w.scale, int(w.causal), self.mptr,
                              self.stream.cuda_stream)
        if st != fa.FA_OK:
            raise fa.FaError(st, "fa_fwd_stream")

    def host_buffers(self):
        self.hin = [t.pin_memory() for t in (self.q, self.k, self.v)]
        self.hm = None if self.mask is None else self.mask.pin_memory()
        self.hout = [__import__("torch").empty(t.shape, dtype=t.dtype).pin_memory()
                     for t in (self.od, self.ld)]
        h2d = sum(t.numel() * t.element_size() for t in self.hin) + (0 if self.hm is None else self.hm.numel())
        d2h = sum(t.numel() * t.element_size() for t in self.hout)
        return h2d, d2h

    def e2e_step(self):
        # The host-buffer entry point: Q, K, V go in and O, lse come out chunk
        # by chunk of heads, the copies overlapping the kernels.
        if self.hm is not None:
            self.md.copy_(self.hm, non_blocking=True)
        w = self.w
        self.fa.attention_forward_host(*self.hin, causal=w.causal, block_mask=self.md, scale=w.scale,
                                       out=self.hout[0], lse=self.hout[1],
                                       device_buffers=(self.qd, self.kd, self.vd, self.od, self.ld),
                                       stream=self.stream.cuda_stream, synchronize=False)

    def algorithmic_bytes(self):
        w = self.w
        return algorithmic_bytes(w.B, w.H, w.N, w.d)

    def cpu_baseline(self, args):
        w = self.w
        qn, kn, vn, mn = numpy_inputs(self.q, self.k, self.v, self.mask)
        kept = []
        f, t, rows = oracle_sample(w, qn, kn, vn, mn, args.cpu_rows, budget_s=args.cpu_budget,
                                   keep=kept)
        self.parity = self._parity(kept)
        return {"value": f / t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"{rows} query rows of {w.name} (complete rows over all N={w.N} keys, "
                          f"head-major from row 0), {t:.1f} s of float64 NumPy/BLAS oracle"}

    def _parity(self, kept):
        """max |O - O_ref| and |lse - lse_ref| of the timed run's output on the
        rows the oracle computed (after the timed region, untimed)."""
        import numpy as np
        import torch

        o = self.od.to("cpu", torch.float64).numpy()
        lse = self.ld.to("cpu", torch.float64).numpy()
        e_o = e_l = 0.0
        n = 0
        for sample, o_ref, l_ref in kept:
            b, h, i = (np.array(x) for x in zip(*sample))
            e_o = max(e_o, float(np.max(np.abs(o[b, h, i] - o_ref))))
            fin = np.isfinite(l_ref)
            if fin.any():
                e_l = max(e_l, float(np.max(np.abs(lse[b, h, i][fin] - l_ref[fin]))))
            n += len(sample)
        return {"rows": n, "max_abs_dO": e_o, "max_abs_dlse": e_l, "bar": {"dO": 2e-2, "dlse": 1e-2},
                "within_bar": e_o <= 2e-2 and e_l <= 1e-2}


class BwdJob(FwdJob):
    """One step = one fa_bwd call (dQ kernel + dK/dV kernel) on the forward's
    O and lse, for a seeded upstream gradient dO.  Credited FLOPs: 2.5x the
    forward's (five products of the forward's size against its two)."""

    name = "bwd"
    e2e_entry = "attention_backward (whole-tensor copies in and out on the stream)"
    metric = "fused attention bwd TFLOP/s (bf16 dQ, dK, dV; 2.5x forward FLOPs) and % of dense BF16 peak"
    kernel_sources = ("exact_attention_120_b200/csrc/fa_bwd_kernel.cuh",
                      "exact_attention_120_b200/csrc/fa_fwd_kernel.cuh",  # shared helpers
                      "exact_attention_120_b200/csrc/ptx.cuh",
                      "exact_attention_120_b200/csrc/fa_api.cu")

    def __init__(self, fa, torch, w, q, k, v, mask, dev, stream):
        super().__init__(fa, torch, w, q, k, v, mask, dev, stream)
        self.flops *= 2.5
        g = torch.Generator().manual_seed(w.seed + 7)
        self.do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
        self.dod = self.do.to(dev)
        super().launch()  # O and lse of the forward, the backward's inputs
        torch.cuda.synchronize(dev)
        self.ho_lse = None
        self.dq, self.dk, self.dv = (torch.empty_like(t) for t in (self.qd, self.kd, self.vd))
        self.ws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.H, w.N), dtype=torch.uint8, device=dev)
        self.bptrs = (self.qd.data_ptr(), self.kd.data_ptr(), self.vd.data_ptr(), self.od.data_ptr(),
                      self.ld.data_ptr(), self.dod.data_ptr(), self.dq.data_ptr(), self.dk.data_ptr(),
                      self.dv.data_ptr())
        self.launches_per_step = 2

    def launch(self):
        w, fa = self.w, self.fa
        st = fa.fa_bwd(*self.bptrs, w.B, w.H, w.N, w.N, w.d, w.scale, int(w.causal), self.mptr,
                       self.ws.data_ptr(), self.ws.numel(), self.stream.cuda_stream)
        if st != fa.FA_OK:
            raise fa.FaError(st, "fa_bwd")

    def host_buffers(self):
        torch = __import__("torch")
        self.hin = [t.pin_memory() for t in (self.q, self.k, self.v)]
        self.hin += [self.od.cpu().pin_memory(), self.ld.cpu().pin_memory(), self.do.pin_memory()]
        self.hm = None if self.mask is None else self.mask.pin_memory()
        self.hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (self.dq, self.dk, self.dv)]
        h2d = sum(t.numel() * t.element_size() for t in self.hin) + (0 if self.hm is None else self.hm.numel())
        d2h = sum(t.numel() * t.element_size() for t in self.hout)
        return h2d, d2h

    def e2e_step(self):
        devs = (self.qd, self.kd, self.vd, self.od, self.ld, self.dod)
        for d, h in zip(devs, self.hin):
            d.copy_(h, non_blocking=True)
        if self.hm is not None:
            self.md.copy_(self.hm, non_blocking=True)
        w = self.w
        grads = self.fa.attention_backward(self.qd, self.kd, self.vd, self.od, self.ld, self.dod,
                                           causal=w.causal, block_mask=self.md, scale=w.scale,
                                           workspace=self.ws)
        for h, d in zip(self.hout, grads):
            h.copy_(d, non_blocking=True)

    def algorithmic_bytes(self):
        # Q, K, V, O, dO read, dQ, dK, dV written (bf16), lse read (fp32).
        w = self.w
        return float(w.B * w.H * (16 * w.N * w.d + 4 * w.N))

    def cpu_baseline(self, args):
        f, t, n = bwd_oracle_sample(self.w, self.q, self.k, self.v, self.mask)
        return {"value": f / t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"float64 gradient oracle on head (0,0) of {self.w.name} cut to its first "
                          f"{n} queries and keys, {t:.1f} s"}


class VarlenJob(FwdJob):
    """One step = one fa_fwd_varlen launch over a packed batch of sequences of
    mixed lengths (the varlen_mix workload)."""

    name = "varlen"
    e2e_entry = "attention_forward_varlen (whole-tensor copies in and out on the stream)"
    metric = "fused attention fwd TFLOP/s, variable-length batch (bf16) and % of dense BF16 peak"

    def __init__(self, fa, torch, w, dev, stream):
        self.fa, self.w, self.stream = fa, w, stream
        self.lens, q, k, v, cu_q, cu_k = make_varlen_inputs(w)
        self.flops = varlen_flops(self.lens, self.lens, w.H, w.d, w.causal)
        self.q, self.k, self.v, self.cu = q, k, v, cu_q
        self.qd, self.kd, self.vd = q.to(dev), k.to(dev), v.to(dev)
        self.cud = cu_q.to(dev)
        self.od = torch.empty_like(self.qd)
        self.ld = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=dev)
        self.max_q = max(self.lens)
        self.launches_per_step = 1
        self.mask = None

    def launch(self):
        w, fa = self.w, self.fa
        st = fa.fa_fwd_varlen(self.qd.data_ptr(), self.kd.data_ptr(), self.vd.data_ptr(),
                              self.od.data_ptr(), self.ld.data_ptr(), self.cud.data_ptr(),
                              self.cud.data_ptr(), w.B, w.H, self.qd.shape[0], self.kd.shape[0],
                              self.max_q, w.d, w.scale, int(w.causal), self.stream.cuda_stream)
        if st != fa.FA_OK:
            raise fa.FaError(st, "fa_fwd_varlen")

    def host_buffers(self):
        torch = __import__("torch")
        self.hin = [t.pin_memory() for t in (self.q, self.k, self.v, self.cu)]
        self.hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (self.od, self.ld)]
        h2d = sum(t.numel() * t.element_size() for t in self.hin)
        d2h = sum(t.numel() * t.element_size() for t in self.hout)
        return h2d, d2h

    def e2e_step(self):
        for d, h in zip((self.qd, self.kd, self.vd, self.cud), self.hin):
            d.copy_(h, non_blocking=True)
        w = self.w
        self.fa.attention_forward_varlen(self.qd, self.kd, self.vd, self.cud, self.cud, self.max_q,
                                         causal=w.causal, scale=w.scale, out=self.od, lse=self.ld)
        for h, d in zip(self.hout, (self.od, self.ld)):
            h.copy_(d, non_blocking=True)

    def algorithmic_bytes(self):
        w, T = self.w, self.qd.shape[0]
        return float(w.H * (8 * T * w.d + 4 * T))

    def cpu_baseline(self, args):
        import oracle

        # The oracle on whole sequences, shortest first, head 0, ~cpu_budget s.
        order = sorted(range(len(self.lens)), key=lambda b: self.lens[b])
        cu = self.cu.tolist()
        f64 = lambda t: t.to(__import__("torch").float64).numpy()  # noqa: E731
        flops, t_total, done = 0.0, 0.0, 0
        for b in order:
            sl = slice(cu[b], cu[b + 1])
            qs, ks, vs = f64(self.q[sl, 0:1]), f64(self.k[sl, 0:1]), f64(self.v[sl, 0:1])
            n = self.lens[b]
            t0 = time.perf_counter()
            oracle.attention_varlen_ref(qs, ks, vs, [0, n], [0, n], self.w.scale, causal=self.w.causal)
            t_total += time.perf_counter() - t0
            flops += varlen_flops([n], [n], 1, self.w.d, self.w.causal)
            done += 1
            if t_total >= args.cpu_budget:
                break
        return {"value": flops / t_total / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"float64 oracle on head 0 of the {done} shortest sequences of {self.w.name}, "
                          f"{t_total:.1f} s"}


class Fp8Job(FwdJob):
    """One step = one fa_fwd_fp8 launch: the workload's shape with Q, K, V
    quantised to E4M3 (one scale per tensor), O in bf16."""

    name = "fp8"
    e2e_entry = "attention_forward_fp8 (whole-tensor copies in and out on the stream)"
    metric = "fused attention fwd TFLOP/s, 8-bit E4M3 inputs, and % of dense FP8 peak"
    peak_ratio = 2.0  # dense fp8 / dense bf16, nominal (4.5 / 2.25 PFLOP/s)

    def __init__(self, fa, torch, w, dev, stream):
        if w.d != 128 or w.sparse_p is not None:
            raise SystemExit("--pass fp8 runs d=128 workloads without a block mask")
        self.fa, self.w, self.stream = fa, w, stream
        (q8, k8, v8), self.descales = make_qkv_fp8(w.B, w.H, w.N, w.d, w.seed, w.qk_std, w.v_std)
        self.flops = useful_flops(w.B, w.H, w.N, w.d, w.causal, None)
        self.q, self.k, self.v = q8, k8, v8
        self.qd, self.kd, self.vd = q8.to(dev), k8.to(dev), v8.to(dev)
        self.od = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
        self.ld = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        self.mask = None
        self.launches_per_step = 1

    def launch(self):
        w, fa = self.w, self.fa
        st = fa.fa_fwd_fp8(self.qd.data_ptr(), self.kd.data_ptr(), self.vd.data_ptr(),
                           self.od.data_ptr(), self.ld.data_ptr(), w.B, w.H, w.N, w.N, w.d, w.scale,
                           int(w.causal), None, *self.descales, self.stream.cuda_stream)
        if st != fa.FA_OK:
            raise fa.FaError(st, "fa_fwd_fp8")

    def host_buffers(self):
        torch = __import__("torch")
        self.hin = [t.pin_memory() for t in (self.q, self.k, self.v)]
        self.hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (self.od, self.ld)]
        return (sum(t.numel() * t.element_size() for t in self.hin),
                sum(t.numel() * t.element_size() for t in self.hout))

    def e2e_step(self):
        for d, h in zip((self.qd, self.kd, self.vd), self.hin):
            d.copy_(h, non_blocking=True)
        w = self.w
        self.fa.attention_forward_fp8(self.qd, self.kd, self.vd, *self.descales, causal=w.causal,
                                      scale=w.scale, out=self.od, lse=self.ld)
        for h, d in zip(self.hout, (self.od, self.ld)):
            h.copy_(d, non_blocking=True)

    def algorithmic_bytes(self):
        # 1-byte Q, K, V read, bf16 O and fp32 lse written.
        w = self.w
        return float(w.B * w.H * (5 * w.N * w.d + 4 * w.N))

    def cpu_baseline(self, args):
        import oracle

        torch = __import__("torch")
        w = self.w
        qd, kd, vd = self.descales
        f64 = lambda t, s: torch.from_numpy(oracle.e4m3_decode(t.numpy()) * s)  # noqa: E731
        qf, kf, vf = f64(self.q, qd), f64(self.k, kd), f64(self.v, vd)
        f, t, rows = oracle_sample(w, qf.numpy(), kf.numpy(), vf.numpy(), None, args.cpu_rows,
                                   budget_s=args.cpu_budget)
        return {"value": f / t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"{rows} query rows of {w.name} (E4M3 inputs decoded exactly), {t:.1f} s "
                          f"of float64 NumPy/BLAS oracle"}


def varlen_config(w, job, world):
    return {"workload": f"{w.name}: {w.describe()}, scale 1/sqrt(d), seed {w.seed}",
            "B": w.B, "H": w.H, "d": w.d, "causal": w.causal, "total_tokens": int(job.qd.shape[0]),
            "max_seqlen": job.max_q, "global_batch": w.B * world,
            "parallelism": "replicas" if world == 1 else f"dp{world} (independent batch slices)",
            "l2": "Q, K, V, O = %d MB per step, larger than L2; no flush"
                  % (job.algorithmic_bytes() // 2**20)}


class EventTimer:
    """CUDA events on the launching stream (and the clock sampler, if any,
    running from start to stop)."""

    def __init__(self, torch, stream, sampler=None):
        self.stream, self.sampler = stream, sampler
        self.e0 = torch.cuda.Event(enable_timing=True)
        self.e1 = torch.cuda.Event(enable_timing=True)

    def start(self):
        if self.sampler is not None:
            self.sampler.start()
        self.e0.record(self.stream)

    def stop(self):
        self.e1.record(self.stream)

    def elapsed_ms(self):  # after a synchronise
        if self.sampler is not None:
            self.sampler.stop()
        return self.e0.elapsed_time(self.e1)


def rank_workload(w, info):
    """The workload rank `info.rank` runs: the same shape, its own seed."""
    return dataclasses.replace(w, seed=sharding.rank_seed(w.seed, info.rank))


def emit(info, line, file=None):
    """Print the JSON line on rank 0 only; returns whether it printed."""
    if not info.is_root:
        return False
    print(json.dumps(line), file=file or sys.stdout, flush=True)
    return True


def run_ours(args, info):
    import torch

    import exact_attention_120_b200 as fa

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device (the kernel has no CPU path)")
    dev = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(dev)
    sharding.init_process_group(info, "nccl")
    fa.load_library()

    stream = torch.cuda.current_stream(dev)
    if args.pass_ == "fp8":
        w = WORKLOADS[args.workload]
        job = Fp8Job(fa, torch, rank_workload(w, info), dev, stream)
    elif args.pass_ == "varlen":
        w = VARLEN_WORKLOADS["varlen_mix"]
        job = VarlenJob(fa, torch, rank_workload(w, info), dev, stream)
    else:
        w = WORKLOADS[args.workload]
        q, k, v, mask = make_inputs(rank_workload(w, info))
        job = (BwdJob if args.pass_ == "bwd" else FwdJob)(fa, torch, w, q, k, v, mask, dev, stream)
    flops = job.flops

    for _ in range(args.warmup):
        job.launch()
    torch.cuda.synchronize(dev)
    st = fa.fa_device_status(stream.cuda_stream)
    if st != fa.FA_OK:
        raise fa.FaError(st, "device status after warm-up")

    # ---- device-timed region: K steps, inputs resident in HBM
    sampler = ClockSampler(dev)
    sync = lambda: torch.cuda.synchronize(dev)  # noqa: E731
    ms_step = sharding.timed_region(job.launch, args.steps, EventTimer(torch, stream, sampler), dev, sync)
    st = fa.fa_device_status(stream.cuda_stream)
    if st != fa.FA_OK:
        raise fa.FaError(st, "device status after timed region")

    # ---- per-step distribution (outside the timed region): one event pair per step
    per = []
    for _ in range(min(args.steps, 50)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        job.launch()
        b.record(stream)
        per.append((a, b))
    torch.cuda.synchronize(dev)
    per_ms = sorted(a.elapsed_time(b) for a, b in per)
    pct = lambda f: per_ms[min(len(per_ms) - 1, int(f * len(per_ms)))]  # noqa: E731

    # ---- host side of one call (argument checks, pointer queries, tensor-map
    # encoding, launch), the device work left running: median of 50 calls
    host_us = []
    for _ in range(50):
        t0 = time.perf_counter()
        job.launch()
        host_us.append(1e6 * (time.perf_counter() - t0))
    torch.cuda.synchronize(dev)

    # ---- end to end: pinned host inputs -> device -> public API -> host outputs
    h2d, d2h = job.host_buffers()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(min(3, args.warmup)):
        job.e2e_step()
    e2e_ms = sharding.timed_region(job.e2e_step, e2e_steps, EventTimer(torch, stream), dev, sync)

    clocks = sampler.summary()
    if info.world_size > 1:
        import torch.distributed as dist

        allc = [None] * info.world_size
        dist.all_gather_object(allc, clocks)
        clocks = dict(clocks)
        clocks["reasons"] = sorted({r for c in allc for r in c["reasons"]})
    sharding.destroy()
    if not info.is_root:
        return 0

    peak, peak_sus, peak_src = load_peaks()
    ratio = getattr(job, "peak_ratio", 1.0)
    peak, peak_sus = peak * ratio, peak_sus * ratio
    achieved = flops / (ms_step * 1e-3) / 1e12  # one call per step
    value = info.world_size * achieved
    cpu = None
    if info.world_size == 1 and not args.no_cpu_baseline:
        cpu = job.cpu_baseline(args)
    khash = kernel_hash(job.kernel_sources)
    line = {
        "metric": job.metric, "value": value, "unit": UNIT, "n_gpus": info.world_size,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if job.name == "fp8" else "bf16",
        "data": "synthetic (seeded N(0,1) draws, bf16)",
        "config": (varlen_config(w, job, info.world_size) if job.name == "varlen"
                   else workload_config(w, info.world_size)),
        "pct_of_dense_bf16_peak": 100.0 * achieved / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": load_traffic(w.name, job.name, khash),
                     "peak_kind": (f"{peak_src} burst dense bf16" if ratio == 1.0 else
                                   f"{peak_src} burst dense bf16 x {ratio:g} (nominal fp8/bf16 ratio)"),
                     "frac_of_sustained_peak": achieved / peak_sus,
                     "algorithmic_bytes": job.algorithmic_bytes(),
                     "flops_per_launch": flops},
        "e2e": {"value": info.world_size * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "entry": job.e2e_entry},
        "ms_per_step_percentiles": {"p10": pct(0.1), "p50": pct(0.5), "p90": pct(0.9),
                                    "steps": len(per_ms),
                                    "taken": "after the timed region, one event pair per launch"},
        "host_us_per_call": statistics.median(host_us),
        "gpu_launches": args.steps * job.launches_per_step,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "kernel_hash": khash,
        "device": {"name": torch.cuda.get_device_name(dev), "torch": torch.__version__,
                   "cuda": torch.version.cuda},
    }
    if getattr(job, "parity", None) is not None:
        line["parity_sample"] = job.parity
    if job.name == "bwd":
        line["config"]["pass"] = "backward (fa_bwd: dQ kernel then dK/dV kernel)"
    emit(info, line)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="long_full", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd", "varlen", "fp8"],
                    help="time the forward (default), the backward pass, the 8-bit forward, or the "
                         "forward on the variable-length batch varlen_mix (--workload is then ignored)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-rows", type=int, default=256, help="oracle rows per timed chunk")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--reference-rows", type=int, default=256, help="oracle rows per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    info = sharding.rank_info_from_env()
    if info.world_size != args.gpus:
        if info.world_size == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    if args.impl == "reference":
        if args.pass_ != "fwd":
            ap.error("--impl reference times the forward oracle only")
        return run_reference(args, info)
    return run_ours(args, info)


if __name__ == "__main__":
    sys.exit(main())
