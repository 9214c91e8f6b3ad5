"""B200 (sm_100a) fused exact attention: Python binding of the C ABI.

The binding only marshals arguments: every step of the forward and backward
passes runs in the CUDA kernels behind ``libfa_b200.so`` (see
``include/fa.h``).  PyTorch is used for device memory and streams.  There is
no CPU fallback: if the library is missing or the device is not an sm_100
GPU the calls raise.  The tensor-level functions check every tensor's dtype,
device, contiguity and shape before anything is launched (the C ABI takes raw
pointers and cannot).

Functions with the C names take raw device addresses:

* ``fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask)``
* ``fa_fwd_stream(..., stream)``
* ``fa_fwd_qk(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, stream)``
* ``fa_fwd_splitkv(..., num_splits, workspace, workspace_bytes, stream)`` with
  ``fa_fwd_splitkv_workspace_bytes`` and ``fa_fwd_splitkv_heuristic``
* ``fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, scale, causal,
  block_mask, workspace, workspace_bytes, stream)`` and ``fa_bwd_workspace_bytes``
* ``fa_fwd_varlen(...)``, ``fa_fwd_fp8(...)``
* ``fa_device_status(stream)``, ``fa_status_string(status)``

Tensor-level functions (allocate outputs with torch, launch on torch's current
stream): ``attention_forward``, ``attention_forward_splitkv``,
``attention_forward_varlen``, ``attention_forward_fp8`` and
``attention_backward``.
"""

from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "FaError", "library_path", "load_library", "fa_fwd", "fa_fwd_stream", "fa_fwd_qk",
    "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_bytes", "fa_fwd_splitkv_heuristic",
    "attention_forward_splitkv", "fa_bwd", "fa_bwd_workspace_bytes", "attention_backward",
    "fa_device_status", "fa_fwd_varlen", "attention_forward_varlen", "fa_fwd_fp8",
    "attention_forward_fp8", "fa_fwd_host", "attention_forward_host",
    "fa_status_string", "fa_launches_per_call", "attention_forward", "FA_OK",
    "FA_ERR_INVALID_ARGUMENT", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA", "FA_ERR_DEVICE_TIMEOUT",
    "MASK_BLOCK",
]

FA_OK = 0
FA_ERR_INVALID_ARGUMENT = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_CUDA = 3
FA_ERR_DEVICE_TIMEOUT = 4
MASK_BLOCK = 128

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB = None

# Exported symbols of the library, with their ctypes signatures.
_SIGNATURES = {
    "fa_fwd": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_void_p, ctypes.c_void_p]
               + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "fa_fwd_stream": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_void_p, ctypes.c_void_p]
                      + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                              ctypes.c_void_p]),
    "fa_fwd_host": (ctypes.c_int, [ctypes.c_void_p] * 10 + [ctypes.c_int] * 4
                    + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "fa_fwd_qk": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_void_p, ctypes.c_void_p]
                  + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "fa_fwd_splitkv": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_void_p, ctypes.c_void_p]
                       + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                               ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                               ctypes.c_void_p]),
    "fa_fwd_splitkv_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 6),
    "fa_fwd_splitkv_noalloc": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_void_p, ctypes.c_void_p]
                               + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                                       ctypes.c_int, ctypes.c_void_p]),
    "fa_fwd_splitkv_heuristic": (ctypes.c_int, [ctypes.c_int] * 4),
    "fa_fwd_fp8": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5
                   + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p] + [ctypes.c_float] * 3
                   + [ctypes.c_void_p]),
    "fa_fwd_varlen": (ctypes.c_int, [ctypes.c_void_p] * 7 + [ctypes.c_int] * 6
                      + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p]),
    "fa_bwd": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 5
               + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                  ctypes.c_void_p]),
    "fa_bwd_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 3),
    "fa_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "fa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fa_last_cuda_error": (ctypes.c_int, []),
    "fa_launches_per_call": (ctypes.c_int, []),
    "fa_testing_fwd_starved": (ctypes.c_int, [ctypes.c_void_p] * 3 + [ctypes.c_void_p, ctypes.c_void_p]
                               + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                                       ctypes.c_void_p, ctypes.c_ulonglong]),
}


class FaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = fa_status_string(status) if _LIB is not None else str(status)
        extra = ""
        if status == FA_ERR_CUDA and _LIB is not None:
            extra = f" (cuda error {_LIB.fa_last_cuda_error()})"
        super().__init__(f"{what}: {name}{extra}" if what else f"{name}{extra}")


def library_path() -> str:
    return os.path.join(_PKG, "libfa_b200.so")


def load_library():
    """Load ``libfa_b200.so`` (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise FileNotFoundError(
                f"{path} is missing: build it with `python -m exact_attention_120_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask) -> int:
    """C ``fa_fwd`` on raw device addresses (ints); returns the status code."""
    return load_library().fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask)


def fa_fwd_stream(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, stream) -> int:
    """C ``fa_fwd_stream`` on raw device addresses and a cudaStream_t (int)."""
    return load_library().fa_fwd_stream(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask,
                                        stream)


def fa_fwd_qk(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, stream) -> int:
    """C ``fa_fwd_qk`` (Nq query rows, Nk keys) on raw device addresses."""
    return load_library().fa_fwd_qk(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask,
                                    stream)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, num_splits,
                   workspace, workspace_bytes, stream) -> int:
    """C ``fa_fwd_splitkv`` on raw device addresses."""
    return load_library().fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal,
                                         block_mask, num_splits, workspace, workspace_bytes, stream)


def fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, num_splits) -> int:
    return load_library().fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, num_splits)


def fa_fwd_splitkv_heuristic(B, H, Nq, Nk) -> int:
    return load_library().fa_fwd_splitkv_heuristic(B, H, Nq, Nk)


def fa_device_status(stream=None) -> int:
    return load_library().fa_device_status(stream)


def fa_status_string(status: int) -> str:
    return load_library().fa_status_string(status).decode()


def fa_launches_per_call() -> int:
    return load_library().fa_launches_per_call()


def fa_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev, B, H, N,
                d, scale, causal, block_mask, stream) -> int:
    """C ``fa_fwd_host`` on raw host and device addresses and a cudaStream_t."""
    return load_library().fa_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev,
                                      o_dev, lse_dev, B, H, N, d, scale, causal, block_mask, stream)


def _check(t, name, dtype, shape, device=None):
    """Raise ValueError unless `t` is a contiguous CUDA tensor of `dtype` and
    `shape` (on `device` when given)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}")


def _check_qkv(q, k, v, dtype):
    """q [B, H, Nq, d], k and v [B, H, Nk, d] of `dtype` on one device."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, H, Nq, d] and k, v [B, H, Nk, d]")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    _check(q, "q", dtype, (B, H, Nq, d))
    _check(k, "k", dtype, (B, H, Nk, d), q.device)
    _check(v, "v", dtype, (B, H, Nk, d), q.device)
    return B, H, Nq, Nk, d


def _check_mask(block_mask, B, H, Nq, Nk, device):
    if block_mask is None:
        return None
    nbq = (Nq + MASK_BLOCK - 1) // MASK_BLOCK
    nbk = (Nk + MASK_BLOCK - 1) // MASK_BLOCK
    import torch

    _check(block_mask, "block_mask", torch.uint8, (B, H, nbq, nbk), device)
    return block_mask.data_ptr()


def attention_forward(q, k, v, causal=False, block_mask=None, scale=None, out=None, lse=None,
                      stream=None):
    """O, lse = attention(q, k, v) through the C ABI.

    q: CUDA bfloat16 [B, H, Nq, d]; k, v: CUDA bfloat16 [B, H, Nk, d]; all
    contiguous, d in {64, 128}.  Nq = Nk uses ``fa_fwd_stream``, otherwise
    ``fa_fwd_qk`` (causal diagonal aligned to the last key).
    block_mask: None or a CUDA uint8 tensor [B, H, ceil(Nq/128), ceil(Nk/128)].
    scale: defaults to 1/sqrt(d).  Returns (o bf16 [B,H,Nq,d], lse fp32 [B,H,Nq]).
    """
    import torch

    B, H, Nq, Nk, d = _check_qkv(q, k, v, torch.bfloat16)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, (B, H, Nq, d), q.device)
    _check(lse, "lse", torch.float32, (B, H, Nq), q.device)
    mask_ptr = _check_mask(block_mask, B, H, Nq, Nk, q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        if Nq == Nk:
            st = fa_fwd_stream(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, H, Nq, d, float(scale), int(bool(causal)),
                               mask_ptr, stream)
        else:
            st = fa_fwd_qk(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                           B, H, Nq, Nk, d, float(scale), int(bool(causal)), mask_ptr, stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd")
    return out, lse


def attention_forward_host(q, k, v, causal=False, block_mask=None, scale=None, out=None, lse=None,
                           device_buffers=None, stream=None, synchronize=True):
    """O, lse of host-resident inputs through ``fa_fwd_host``: the copies to and
    from the device overlap the computation, chunk by chunk of heads.

    q, k, v: CPU bfloat16 [B, H, N, d], contiguous (page-locked for the copies
    to overlap).  out / lse: CPU bf16 [B, H, N, d] / fp32 [B, H, N] to write
    (page-locked ones are allocated when None).  device_buffers: None or the
    CUDA tensors (q, k, v, o, lse) the data pass through (allocated on the
    current device when None).  block_mask: None or a CUDA uint8 tensor as for
    attention_forward.  With ``synchronize`` the call's stream (the device, for
    a raw stream handle) is synchronised before returning, so out and lse are
    ready; otherwise they are complete once the
    stream has passed this call, and q, k, v, out and lse must stay alive until
    then (the copies are not known to torch's pinned-memory cache, which would
    otherwise hand their memory to the next pinned tensor).  Returns (out, lse).
    """
    import torch

    if q.dim() != 4:
        raise ValueError("q must be [B, H, N, d]")
    B, H, N, d = q.shape
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must be a contiguous CPU bfloat16 tensor of shape {(B, H, N, d)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    for t, name, dt, shape in ((out, "out", torch.bfloat16, (B, H, N, d)),
                               (lse, "lse", torch.float32, (B, H, N))):
        if t.dtype != dt or t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be a contiguous CPU {dt} tensor of shape {shape}")
    dev = torch.device("cuda", torch.cuda.current_device()) if block_mask is None else block_mask.device
    if device_buffers is None:
        device_buffers = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N), dtype=torch.float32, device=dev))
    qd, kd, vd, od, ld = device_buffers
    dev = qd.device
    for t, name in ((qd, "q_dev"), (kd, "k_dev"), (vd, "v_dev"), (od, "o_dev")):
        _check(t, name, torch.bfloat16, (B, H, N, d), dev)
    _check(ld, "lse_dev", torch.float32, (B, H, N), dev)
    mask_ptr = _check_mask(block_mask, B, H, N, N, dev)
    torch_stream = torch.cuda.current_stream(dev) if stream is None else None
    if stream is None:
        stream = torch_stream.cuda_stream
    with torch.cuda.device(dev):
        st = fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                         qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), ld.data_ptr(),
                         B, H, N, d, float(scale), int(bool(causal)), mask_ptr, stream)
        if st != FA_OK:
            raise FaError(st, "fa_fwd_host")
        if synchronize:
            # The call's work ends on its stream: wait for that stream (for a raw
            # handle passed in, for the device).
            if torch_stream is not None:
                torch_stream.synchronize()
            else:
                torch.cuda.synchronize(dev)
    return out, lse


def attention_forward_splitkv(q, k, v, causal=False, block_mask=None, scale=None, num_splits=None,
                              workspace=None, out=None, lse=None, stream=None):
    """attention_forward with the keys cut into slices (fa_fwd_splitkv).

    num_splits: None picks fa_fwd_splitkv_heuristic.  workspace: a CUDA uint8
    tensor of at least fa_fwd_splitkv_workspace_bytes(...) bytes, or None to
    allocate one with torch.  Returns (o, lse).
    """
    import torch

    B, H, Nq, Nk, d = _check_qkv(q, k, v, torch.bfloat16)
    if num_splits is None:
        num_splits = fa_fwd_splitkv_heuristic(B, H, Nq, Nk)
    need = fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None and (not workspace.is_cuda or not workspace.is_contiguous()
                                  or workspace.device != q.device):
        raise ValueError("workspace must be a contiguous CUDA tensor on q's device")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, (B, H, Nq, d), q.device)
    _check(lse, "lse", torch.float32, (B, H, Nq), q.device)
    mask_ptr = _check_mask(block_mask, B, H, Nq, Nk, q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    ws_ptr = None if workspace is None else workspace.data_ptr()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        st = fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                            B, H, Nq, Nk, d, float(scale), int(bool(causal)), mask_ptr, num_splits,
                            ws_ptr, ws_bytes, stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv")
    return out, lse


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, scale, causal, block_mask, workspace,
           workspace_bytes, stream) -> int:
    return load_library().fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, scale, causal,
                                 block_mask, workspace, workspace_bytes, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q,
                  d, scale, causal, stream) -> int:
    return load_library().fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q,
                                        total_k, max_seqlen_q, d, scale, causal, stream)


def fa_fwd_fp8(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, q_descale, k_descale,
               v_descale, stream) -> int:
    return load_library().fa_fwd_fp8(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask,
                                     q_descale, k_descale, v_descale, stream)


def fa_bwd_workspace_bytes(B, H, Nq) -> int:
    return load_library().fa_bwd_workspace_bytes(B, H, Nq)


def attention_backward(q, k, v, o, lse, dout, causal=False, block_mask=None, scale=None,
                       workspace=None, stream=None):
    """dq, dk, dv of attention_forward through the C ABI (fa_bwd).

    q, o, dout: CUDA bf16 [B, H, Nq, d]; k, v: [B, H, Nk, d]; lse: fp32
    [B, H, Nq] from the forward; causal / block_mask / scale as in the forward.
    """
    import torch

    B, H, Nq, Nk, d = _check_qkv(q, k, v, torch.bfloat16)
    _check(o, "o", torch.bfloat16, (B, H, Nq, d), q.device)
    _check(dout, "dout", torch.bfloat16, (B, H, Nq, d), q.device)
    _check(lse, "lse", torch.float32, (B, H, Nq), q.device)
    mask_ptr = _check_mask(block_mask, B, H, Nq, Nk, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    need = fa_bwd_workspace_bytes(B, H, Nq)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous() or workspace.device != q.device:
        raise ValueError("workspace must be a contiguous CUDA tensor on q's device")
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        st = load_library().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, H, Nq, Nk, d, float(scale), int(bool(causal)),
                                   mask_ptr, workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), stream)
    if st != FA_OK:
        raise FaError(st, "fa_bwd")
    return dq, dk, dv


def attention_forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal=False,
                             scale=None, out=None, lse=None, stream=None):
    """O, lse of a variable-length batch through the C ABI (fa_fwd_varlen).

    q: CUDA bf16 [total_q, H, d]; k, v: [total_k, H, d] (packed tokens);
    cu_seqlens_q / cu_seqlens_k: CUDA int32 [B + 1] offsets; max_seqlen_q:
    the longest query sequence.  Returns O [total_q, H, d] and lse
    [H, total_q] (fp32).
    """
    import torch

    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("q must be [total_q, H, d] and k, v [total_k, H, d]")
    Tq, H, d = q.shape
    Tk = k.shape[0]
    _check(q, "q", torch.bfloat16, (Tq, H, d))
    _check(k, "k", torch.bfloat16, (Tk, H, d), q.device)
    _check(v, "v", torch.bfloat16, (Tk, H, d), q.device)
    if cu_seqlens_q.dim() != 1 or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q must hold B + 1 >= 2 offsets")
    B = cu_seqlens_q.numel() - 1
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, (B + 1,), q.device)
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, (B + 1,), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.bfloat16, (Tq, H, d), q.device)
    _check(lse, "lse", torch.float32, (H, Tq), q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        st = load_library().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                          lse.data_ptr(), cu_seqlens_q.data_ptr(),
                                          cu_seqlens_k.data_ptr(), B, H, Tq, Tk, int(max_seqlen_q), d,
                                          float(scale), int(bool(causal)), stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_varlen")
    return out, lse


def attention_forward_fp8(q8, k8, v8, q_descale, k_descale, v_descale, causal=False, block_mask=None,
                          scale=None, out=None, lse=None, stream=None):
    """O (bf16), lse of attention on 8-bit E4M3 inputs through the C ABI (fa_fwd_fp8).

    q8: CUDA uint8 or float8_e4m3fn [B, H, Nq, 128]; k8, v8: [B, H, Nk, 128];
    the codes stand for q_descale * q8 etc.  scale defaults to 1/sqrt(d).
    """
    import torch

    if q8.dim() != 4 or k8.dim() != 4:
        raise ValueError("q8 must be [B, H, Nq, d] and k8, v8 [B, H, Nk, d]")
    codes = (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8))
    B, H, Nq, d = q8.shape
    Nk = k8.shape[2]
    for t, name, shape in ((q8, "q8", (B, H, Nq, d)), (k8, "k8", (B, H, Nk, d)), (v8, "v8", (B, H, Nk, d))):
        if t.dtype not in codes:
            raise ValueError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn)")
        _check(t, name, t.dtype, shape, q8.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q8.device)
    _check(out, "out", torch.bfloat16, (B, H, Nq, d), q8.device)
    _check(lse, "lse", torch.float32, (B, H, Nq), q8.device)
    mask_ptr = _check_mask(block_mask, B, H, Nq, Nk, q8.device)
    if stream is None:
        stream = torch.cuda.current_stream(q8.device).cuda_stream
    with torch.cuda.device(q8.device):
        st = load_library().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                                       lse.data_ptr(), B, H, Nq, Nk, d, float(scale), int(bool(causal)),
                                       mask_ptr, float(q_descale), float(k_descale), float(v_descale),
                                       stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_fp8")
    return out, lse
