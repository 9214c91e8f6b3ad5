"""The C-ABI library builds, loads and exports every function include/fa.h
declares; argument checks that precede any CUDA call work without a GPU."""

import ctypes
import os
import re

import pytest

from exact_attention_120_b200 import build as build_mod
import exact_attention_120_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return fa.load_library()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"^\s*(?:FA_API\s+)?(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", text, flags=re.M))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"fa_fwd", "fa_fwd_stream", "fa_device_status", "fa_status_string"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARGUMENT"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_CUDA"), (4, "FA_ERR_DEVICE_TIMEOUT")]:
        assert fa.fa_status_string(code) == name
    assert fa.fa_status_string(99) == "FA_UNKNOWN_STATUS"
    assert fa.fa_launches_per_call() == 1


def test_argument_errors_before_any_cuda_call(lib):
    p = 1 << 20  # never dereferenced: every case fails validation first
    base = [p, p, p, p * 2, p * 3, 1, 1, 128, 64, 0.125, 0, None]

    def call(**kw):
        a = list(base)
        names = ["q", "k", "v", "o", "lse", "B", "H", "N", "d", "scale", "causal", "mask"]
        for key, val in kw.items():
            a[names.index(key)] = val
        return fa.fa_fwd(*a)

    assert call(q=None) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(lse=None) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(B=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(N=-5) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(scale=float("inf")) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(scale=0.0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(causal=3) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(d=256) == fa.FA_ERR_UNSUPPORTED
    assert call(q=p + 8) == fa.FA_ERR_INVALID_ARGUMENT  # not 16-byte aligned
    assert call(o=p) == fa.FA_ERR_INVALID_ARGUMENT      # o aliases q
    assert call(B=1 << 16, H=1 << 16) == fa.FA_ERR_UNSUPPORTED  # B*H beyond 32 bits
    # Overlap by address range, not only equal pointers (q, k, v are 16 KB
    # each here; o 16 KB, lse 512 B).
    assert call(o=p + 4096) == fa.FA_ERR_INVALID_ARGUMENT       # o inside q
    assert call(o=p * 3 - 4096) == fa.FA_ERR_INVALID_ARGUMENT   # o runs into lse
    assert call(lse=p + 256) == fa.FA_ERR_INVALID_ARGUMENT      # lse inside q
    assert call(lse=p * 2 + 16384 - 4) == fa.FA_ERR_INVALID_ARGUMENT  # last float of o
    assert call(mask=p * 3 + 16) == fa.FA_ERR_INVALID_ARGUMENT  # lse over the mask


def test_noalloc_argument_errors_before_any_cuda_call(lib):
    """fa_fwd_splitkv_noalloc checks its arguments, and its size limit, before
    any CUDA call (no device is needed to see these statuses)."""
    p = 1 << 24  # never dereferenced
    names = ["q", "k", "v", "o", "lse", "B", "H", "Nq", "Nk", "d", "scale", "causal", "mask",
             "splits", "stream"]
    base = [p, p * 2, p * 3, p * 4, p * 5, 1, 2, 64, 4096, 128, 0.1, 0, None, 4, None]

    def call(**kw):
        a = list(base)
        for key, val in kw.items():
            a[names.index(key)] = val
        return lib.fa_fwd_splitkv_noalloc(*a)

    for name in ("q", "k", "v", "o", "lse"):
        assert call(**{name: None}) == fa.FA_ERR_INVALID_ARGUMENT, name
    assert call(B=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(scale=float("nan")) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(causal=5) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(q=p + 4) == fa.FA_ERR_INVALID_ARGUMENT      # misaligned
    assert call(o=p * 2 + 64) == fa.FA_ERR_INVALID_ARGUMENT  # o inside k
    assert call(splits=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(splits=257) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    # a null pointer is an argument error even when the problem is too large
    assert call(q=None, Nq=1 << 20) == fa.FA_ERR_INVALID_ARGUMENT
    # beyond the array: 2 slices x 16257 rows x 129 floats > 16 MiB
    assert call(B=1, H=1, Nq=16257, Nk=256, splits=2) == fa.FA_ERR_UNSUPPORTED


def test_host_entry_argument_errors_before_any_cuda_call(lib):
    """fa_fwd_host checks pointers, sizes and overlaps before any CUDA call."""
    p = 1 << 24  # never dereferenced: every case fails validation first
    names = ["qh", "kh", "vh", "oh", "lh", "qd", "kd", "vd", "od", "ld", "B", "H", "N", "d", "scale",
             "causal", "mask", "stream"]
    # host buffers at 11p.., device buffers at p..; each tensor is 16 KB
    # (one head, N = 128, d = 64), lse 512 B
    base = [p * 11, p * 12, p * 13, p * 14, p * 15, p, p * 2, p * 3, p * 4, p * 5, 1, 1, 128, 64, 0.125,
            0, None, None]

    def call(**kw):
        a = list(base)
        for key, val in kw.items():
            a[names.index(key)] = val
        return lib.fa_fwd_host(*a)

    for name in ("qh", "kh", "vh", "oh", "lh", "qd", "kd", "vd", "od", "ld"):
        assert call(**{name: None}) == fa.FA_ERR_INVALID_ARGUMENT, name
    assert call(B=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(N=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(scale=-1.0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(causal=2) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(d=32) == fa.FA_ERR_UNSUPPORTED
    assert call(qd=p + 8) == fa.FA_ERR_INVALID_ARGUMENT          # device q misaligned
    assert call(od=p * 2 + 4096) == fa.FA_ERR_INVALID_ARGUMENT   # device o inside device k
    assert call(oh=p * 13 + 4096) == fa.FA_ERR_INVALID_ARGUMENT  # host o inside host v
    assert call(lh=p * 11 + 64) == fa.FA_ERR_INVALID_ARGUMENT    # host lse inside host q
    assert call(lh=p * 14 + 16384 - 4) == fa.FA_ERR_INVALID_ARGUMENT  # host lse on host o's end


def test_splitkv_workspace_size(lib):
    # [splits][rows][d] fp32 partial outputs + [splits][rows] fp32 lse
    assert fa.fa_fwd_splitkv_workspace_bytes(2, 4, 1, 16384, 128, 8) == 8 * 8 * 129 * 4
    # 3 key tiles in at most 3 slices, whatever is asked
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 1, 10, 300, 64, 100) == 3 * 10 * 65 * 4
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 1, 10, 300, 64, 1) == 0
    assert fa.fa_fwd_splitkv_workspace_bytes(1, 1, 10, 300, 64, 0) == 0


def test_every_public_name_exists():
    import exact_attention_120_b200 as fa

    missing = [n for n in fa.__all__ if not hasattr(fa, n)]
    assert not missing, missing


def test_backward_argument_errors_before_any_cuda_call(lib):
    p = 1 << 20  # never dereferenced: every case fails validation first
    names = ["q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv", "B", "H", "Nq", "Nk", "d", "scale",
             "causal", "mask", "ws", "ws_bytes", "stream"]
    base = [p, p * 2, p * 3, p * 4, p * 5, p * 6, p * 7, p * 8, p * 9, 1, 2, 300, 200, 64, 0.125, 0,
            None, p * 10, 4096, None]

    def call(**kw):
        a = list(base)
        for key, val in kw.items():
            a[names.index(key)] = val
        return fa.fa_bwd(*a)

    for name in ("q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv", "ws"):
        assert call(**{name: None}) == fa.FA_ERR_INVALID_ARGUMENT, name
    assert call(B=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(Nk=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(scale=float("nan")) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(causal=2) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(dk=p * 8 + 4) == fa.FA_ERR_INVALID_ARGUMENT   # not 16-byte aligned
    assert call(ws_bytes=100) == fa.FA_ERR_INVALID_ARGUMENT   # below 2*300*4 bytes of D
    assert call(dq=p) == fa.FA_ERR_INVALID_ARGUMENT           # dq aliases q
    assert call(dv=p * 8) == fa.FA_ERR_INVALID_ARGUMENT       # dv aliases dk
    # by address range: dk (51 KB) starting inside o, the workspace inside dq
    assert call(dk=p * 4 + 1024) == fa.FA_ERR_INVALID_ARGUMENT
    assert call(ws=p * 7 + 4096) == fa.FA_ERR_INVALID_ARGUMENT
    assert fa.fa_bwd_workspace_bytes(2, 3, 300) == 2 * 3 * 300 * 4
    assert fa.fa_bwd_workspace_bytes(1, 1, 5) == 32          # rounded up to 16 bytes
    assert fa.fa_bwd_workspace_bytes(0, 1, 5) == 0


def test_varlen_and_fp8_argument_errors_before_any_cuda_call(lib):
    p = 1 << 20
    # fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_seqlen_q, d, scale, causal, stream)
    vbase = [p, p * 2, p * 3, p * 4, p * 5, p * 6, p * 7, 2, 4, 100, 100, 60, 128, 0.1, 1, None]
    vnames = ["q", "k", "v", "o", "lse", "cu_q", "cu_k", "B", "H", "tq", "tk", "maxq", "d", "scale",
              "causal", "stream"]

    def vcall(**kw):
        a = list(vbase)
        for key, val in kw.items():
            a[vnames.index(key)] = val
        return fa.fa_fwd_varlen(*a)

    assert vcall(cu_q=None) == fa.FA_ERR_INVALID_ARGUMENT
    assert vcall(tq=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert vcall(maxq=0) == fa.FA_ERR_INVALID_ARGUMENT
    assert vcall(cu_k=p * 7 + 2) == fa.FA_ERR_INVALID_ARGUMENT  # offsets not 4-byte aligned
    assert vcall(o=p * 2) == fa.FA_ERR_INVALID_ARGUMENT         # o aliases k
    assert vcall(lse=p + 512) == fa.FA_ERR_INVALID_ARGUMENT     # lse inside q
    assert vcall(o=p * 6 - 64) == fa.FA_ERR_INVALID_ARGUMENT    # o runs into cu_seqlens_q
    assert vcall(d=32) == fa.FA_ERR_UNSUPPORTED
    # fa_fwd_fp8(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, mask, qd, kd, vd, stream)
    fbase = [p, p * 2, p * 3, p * 4, p * 5, 1, 1, 128, 128, 128, 0.1, 0, None, 1.0, 1.0, 1.0, None]
    fnames = ["q", "k", "v", "o", "lse", "B", "H", "Nq", "Nk", "d", "scale", "causal", "mask", "qd",
              "kd", "vd", "stream"]

    def fcall(**kw):
        a = list(fbase)
        for key, val in kw.items():
            a[fnames.index(key)] = val
        return fa.fa_fwd_fp8(*a)

    assert fcall(qd=0.0) == fa.FA_ERR_INVALID_ARGUMENT
    assert fcall(kd=float("inf")) == fa.FA_ERR_INVALID_ARGUMENT
    assert fcall(vd=-1.0) == fa.FA_ERR_INVALID_ARGUMENT
    assert fcall(d=64) == fa.FA_ERR_UNSUPPORTED                 # 8-bit inputs need d = 128
    assert fcall(v=None) == fa.FA_ERR_INVALID_ARGUMENT


def _c_prototypes():
    """Name -> (return type, [parameter types]) of every FA_API declaration."""
    protos = {}
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for ret, name, params in re.findall(r"FA_API\s+([\w\s\*]+?)\s*\b(fa_\w+)\s*\(([^)]*)\)\s*;",
                                            text):
            params = " ".join(params.split())
            types = [] if params in ("", "void") else \
                [re.sub(r"\s*\b\w+$", "", p.strip()) for p in params.split(",")]
            protos[name] = (" ".join(ret.split()), types)
    return protos


def _ctype_of(c_type):
    c_type = c_type.replace("const ", "").strip()
    if c_type.endswith("*"):
        return ctypes.c_char_p if c_type == "char*" else ctypes.c_void_p
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t,
            "unsigned long long": ctypes.c_ulonglong}[c_type]


def test_binding_signatures_match_the_headers():
    """Every ctypes signature the binding installs has the C prototype's
    parameter count and, position by position, the same kind of argument
    (pointer, int, float, size_t, 64-bit integer) and return type."""
    protos = _c_prototypes()
    assert set(protos) == _declared_functions()
    assert set(fa._SIGNATURES) == set(protos)
    for name, (ret, params) in protos.items():
        res, args = fa._SIGNATURES[name]
        assert res is _ctype_of(ret), (name, ret)
        assert len(args) == len(params), (name, len(args), len(params))
        for i, (got, want) in enumerate(zip(args, params)):
            assert got is _ctype_of(want), (name, i, want)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without the built library every entry point raises."""
    monkeypatch.setattr(fa, "_LIB", None)
    monkeypatch.setattr(fa, "library_path", lambda: str(tmp_path / "libfa_b200.so"))
    p = 1 << 20
    for call in (lambda: fa.fa_fwd(p, p, p, p, p, 1, 1, 128, 64, 0.125, 0, None),
                 lambda: fa.fa_bwd_workspace_bytes(1, 1, 128),
                 lambda: fa.fa_status_string(0),
                 fa.load_library):
        with pytest.raises(FileNotFoundError, match="build it"):
            call()
