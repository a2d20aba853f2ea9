"""The C ABI on the host: the library loads, exports every function
include/*.h declares, and validates configurations without touching a GPU."""
import ctypes
import glob
import os
import re

import pytest

from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import build as _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names |= set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(fldce_\w+)\s*\(", txt, flags=re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return B.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert len(declared) >= 10
    for name in sorted(declared):
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert declared == set(B.EXPORTS)


def test_exports_are_c_symbols():
    txt = open(B.LIB_PATH, "rb").read()
    for name in B.EXPORTS:
        assert name.encode() + b"\x00" in txt


def test_version(lib):
    assert B.fldce_version() == 100


@pytest.mark.parametrize("kw,code", [
    (dict(D=0), B.FLDCE_ERR_INVALID_ARG),
    (dict(V=0), B.FLDCE_ERR_INVALID_ARG),
    (dict(max_N=0), B.FLDCE_ERR_INVALID_ARG),
    (dict(chunk_N=-1), B.FLDCE_ERR_INVALID_ARG),
    (dict(label_smoothing=1.5), B.FLDCE_ERR_INVALID_ARG),
    (dict(label_smoothing=-0.1), B.FLDCE_ERR_INVALID_ARG),
    (dict(logit_scale=0.0), B.FLDCE_ERR_INVALID_ARG),
    (dict(logit_scale=float("inf")), B.FLDCE_ERR_INVALID_ARG),
    (dict(D=60), B.FLDCE_ERR_UNSUPPORTED),
    (dict(dtype=7), B.FLDCE_ERR_UNSUPPORTED),
    (dict(flags=0x20), B.FLDCE_ERR_UNSUPPORTED),
    (dict(dtype=1, flags=0x2), B.FLDCE_ERR_UNSUPPORTED),
])
def test_create_rejects(lib, kw, code):
    args = dict(dtype=B.FLDCE_BF16, D=64, V=100, max_N=10)
    args.update(kw)
    dtype, D, V, max_N = args.pop("dtype"), args.pop("D"), args.pop("V"), args.pop("max_N")
    with pytest.raises(B.FldceError) as e:
        B.fldce_create(dtype, D, V, max_N, **args)
    assert e.value.status == code


def test_null_arguments(lib):
    cfg = B.fldce_config(0, 0, 64, 100, 10, 0, 1.0, 0.0, -100)
    assert lib.fldce_create(None, ctypes.byref(cfg), None) == B.FLDCE_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert lib.fldce_create(ctypes.byref(h), None, None) == B.FLDCE_ERR_INVALID_ARG
    assert lib.fldce_workspace_size(None, 1, None) == B.FLDCE_ERR_INVALID_ARG
    assert lib.fldce_destroy(None) == B.FLDCE_OK
    assert lib.fldce_fwd_bwd(None, *([None] * 4), 1, 0.0, 1.0, *([None] * 7), 0, None,
                             None) == B.FLDCE_ERR_INVALID_ARG


def test_workspace_and_chunking(lib):
    h, ws = B.fldce_create(B.FLDCE_BF16, 2560, 151936, 8192)
    try:
        assert B.fldce_chunk_size(h) == 8192           # G of 2.5 GB fits one chunk
        assert ws == B.fldce_workspace_size(h, 8192)
        assert B.fldce_workspace_size(h, 100) < ws
        assert B.fldce_workspace_size(h, 0) > 0
        with pytest.raises(B.FldceError):
            B.fldce_workspace_size(h, 8193)
    finally:
        B.fldce_destroy(h)
    h, ws = B.fldce_create(B.FLDCE_BF16, 4096, 256000, 32768)
    try:
        c = B.fldce_chunk_size(h)
        assert c % 256 == 0 and c * 256000 * 2 <= 1 << 32 and c < 32768
        # chunked: G for one chunk plus the fp32 dW accumulator
        assert ws >= c * 256000 * 2 + 256000 * 4096 * 4
    finally:
        B.fldce_destroy(h)
    h, ws_fp32 = B.fldce_create(B.FLDCE_BF16, 4096, 256000, 32768, flags=B.FLDCE_FLAG_DW_FP32)
    try:
        assert ws_fp32 < 256000 * 4096 * 4 + ws_fp32 and ws_fp32 < ws  # no accumulator
    finally:
        B.fldce_destroy(h)
    h, _ = B.fldce_create(B.FLDCE_FP32, 64, 512, 64, chunk_N=16)
    try:
        assert B.fldce_chunk_size(h) == 16
    finally:
        B.fldce_destroy(h)


def test_accumulate_workspace(lib):
    # a bf16 dW accumulated into needs the fp32 accumulator even in one chunk;
    # an fp32 dW takes the reduce-adds directly and needs none
    D, V, N = 2560, 151936, 8192
    sizes = {}
    for name, flags in [("plain", 0), ("acc", B.FLDCE_FLAG_DW_ACCUMULATE),
                        ("fp32", B.FLDCE_FLAG_DW_FP32),
                        ("fp32_acc", B.FLDCE_FLAG_DW_FP32 | B.FLDCE_FLAG_DW_ACCUMULATE)]:
        h, ws = B.fldce_create(B.FLDCE_BF16, D, V, N, flags=flags)
        B.fldce_destroy(h)
        sizes[name] = ws
    assert sizes["acc"] >= sizes["plain"] + V * D * 4
    assert sizes["fp32_acc"] == sizes["fp32"] == sizes["plain"]


def test_profile_kinds(lib):
    names = [B.fldce_profile_kind_name(k) for k in range(B.FLDCE_PROF_KINDS)]
    assert names == ["count_targets", "lse_sweep", "merge", "g_sweep", "dh_gemm", "dw_gemm",
                     "finish", "convert", "db_colsum"]
    assert B.fldce_profile_kind_name(B.FLDCE_PROF_KINDS) is None


def test_strerror(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert B.fldce_strerror(code) and B.fldce_strerror(code) != "unknown status"
    assert B.fldce_strerror(-99) == "unknown status"


def test_fused_dh_flag_combinations(lib):
    # the fused sweep-2 + dH kernel is a bf16 tensor-core design and runs on
    # every token (no compaction); its workspace is that of the staged design
    h, ws_f = B.fldce_create(B.FLDCE_BF16, 2560, 151936, 8192, flags=B.FLDCE_FLAG_FUSED_DH)
    B.fldce_destroy(h)
    h, ws = B.fldce_create(B.FLDCE_BF16, 2560, 151936, 8192)
    B.fldce_destroy(h)
    assert ws_f == ws
    for dtype, flags in ((B.FLDCE_FP32, B.FLDCE_FLAG_FUSED_DH),
                         (B.FLDCE_BF16, B.FLDCE_FLAG_FUSED_DH | B.FLDCE_FLAG_SKIP_IGNORED)):
        with pytest.raises(B.FldceError) as e:
            B.fldce_create(dtype, 64, 512, 64, flags=flags)
        assert e.value.status == B.FLDCE_ERR_UNSUPPORTED
    h, _ = B.fldce_create(B.FLDCE_BF16, 64, 512, 64,
                          flags=B.FLDCE_FLAG_FUSED_DH | B.FLDCE_FLAG_DH_FP32)
    B.fldce_destroy(h)
