"""ctypes binding of libfldce.so, one Python function per C entry point.

Argument marshalling only: tensors become device pointers, streams become
cudaStream_t handles, non-zero status codes become ``FldceError``.  Every
step of the computation runs in the library's CUDA kernels; if the library
is missing or fails to load, every call raises -- there is no fallback.

``Plan`` is a convenience owner of a handle plus a torch-allocated workspace
(PyTorch is used for device memory and streams only).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfldce.so")

FLDCE_OK = 0
FLDCE_ERR_INVALID_ARG = -1
FLDCE_ERR_UNSUPPORTED = -2
FLDCE_ERR_WORKSPACE = -3
FLDCE_ERR_CUDA = -4
FLDCE_ERR_DEVICE = -5
FLDCE_ERR_ALIGN = -6
FLDCE_ERR_TOO_LARGE = -7
FLDCE_STATIC_SCRATCH_BYTES = 64 << 20
FLDCE_BF16 = 0
FLDCE_FP32 = 1
FLDCE_FLAG_DW_FP32 = 0x1
FLDCE_FLAG_SKIP_IGNORED = 0x2
FLDCE_FLAG_DH_FP32 = 0x4
FLDCE_FLAG_DW_ACCUMULATE = 0x8
FLDCE_FLAG_FUSED_DH = 0x10

# every symbol include/fldce.h declares
EXPORTS = ("fldce_create", "fldce_workspace_size", "fldce_chunk_size", "fldce_fwd_bwd",
           "fldce_fwd_bwd_noalloc", "fldce_forward", "fldce_fwd_bwd_ex", "fldce_forward_ex",
           "fldce_count_valid", "fldce_vp_stats", "fldce_vp_fwd_bwd",
           "fldce_profile_begin", "fldce_profile_end", "fldce_profile_kind_name",
           "fldce_scale", "fldce_selftest_wait", "fldce_destroy", "fldce_strerror", "fldce_version")
FLDCE_PROF_KINDS = 9


class FldceError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fldce_strerror(status)} (status {status})")


class fldce_config(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("D", ctypes.c_int64),
        ("V", ctypes.c_int64),
        ("max_N", ctypes.c_int64),
        ("chunk_N", ctypes.c_int64),
        ("logit_scale", ctypes.c_float),
        ("label_smoothing", ctypes.c_float),
        ("ignore_index", ctypes.c_int64),
        ("vocab_start", ctypes.c_int64),
        ("vocab_total", ctypes.c_int64),
    ]


class fldce_call(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_void_p),
        ("W", ctypes.c_void_p),
        ("bias", ctypes.c_void_p),
        ("target", ctypes.c_void_p),
        ("p_mask", ctypes.c_void_p),
        ("N", ctypes.c_int64),
        ("total", ctypes.c_float),
        ("grad_out", ctypes.c_float),
        ("count_dev", ctypes.c_void_p),
        ("loss", ctypes.c_void_p),
        ("loss_per_token", ctypes.c_void_p),
        ("lse", ctypes.c_void_p),
        ("argmax", ctypes.c_void_p),
        ("dH", ctypes.c_void_p),
        ("dW", ctypes.c_void_p),
        ("db", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("err_count", ctypes.c_void_p),
        ("stream", ctypes.c_void_p),
        ("dw_ready_event", ctypes.c_void_p),
    ]


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float


def load() -> ctypes.CDLL:
    """Load libfldce.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m linear_diffusion_cross_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.fldce_create.argtypes = [ctypes.POINTER(_P), ctypes.POINTER(fldce_config),
                                 ctypes.POINTER(ctypes.c_size_t)]
    lib.fldce_create.restype = ctypes.c_int
    lib.fldce_workspace_size.argtypes = [_P, _I64, ctypes.POINTER(ctypes.c_size_t)]
    lib.fldce_workspace_size.restype = ctypes.c_int
    lib.fldce_chunk_size.argtypes = [_P, ctypes.POINTER(_I64)]
    lib.fldce_chunk_size.restype = ctypes.c_int
    lib.fldce_fwd_bwd.argtypes = [_P, _P, _P, _P, _P, _I64, _F, _F, _P, _P, _P, _P, _P, _P, _P,
                                  ctypes.c_size_t, _P, _P]
    lib.fldce_fwd_bwd.restype = ctypes.c_int
    lib.fldce_fwd_bwd_noalloc.argtypes = [_P, _P, _P, _P, _P, _I64, _F, _F, _P, _P, _P, _P, _P,
                                          _P, _P, _P]
    lib.fldce_fwd_bwd_noalloc.restype = ctypes.c_int
    lib.fldce_forward.argtypes = [_P, _P, _P, _P, _P, _I64, _F, _P, _P, _P, _P, _P,
                                  ctypes.c_size_t, _P, _P]
    lib.fldce_forward.restype = ctypes.c_int
    lib.fldce_profile_begin.argtypes = [_P, ctypes.c_int]
    lib.fldce_profile_begin.restype = ctypes.c_int
    lib.fldce_profile_end.argtypes = [_P, ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_int32)]
    lib.fldce_profile_end.restype = ctypes.c_int
    lib.fldce_profile_kind_name.argtypes = [ctypes.c_int]
    lib.fldce_profile_kind_name.restype = ctypes.c_char_p
    lib.fldce_fwd_bwd_ex.argtypes = [_P, ctypes.POINTER(fldce_call)]
    lib.fldce_fwd_bwd_ex.restype = ctypes.c_int
    lib.fldce_forward_ex.argtypes = [_P, ctypes.POINTER(fldce_call)]
    lib.fldce_forward_ex.restype = ctypes.c_int
    lib.fldce_vp_stats.argtypes = [_P, ctypes.POINTER(fldce_call), _P]
    lib.fldce_vp_stats.restype = ctypes.c_int
    lib.fldce_vp_fwd_bwd.argtypes = [_P, ctypes.POINTER(fldce_call), _P, ctypes.c_int32]
    lib.fldce_vp_fwd_bwd.restype = ctypes.c_int
    lib.fldce_count_valid.argtypes = [_P, _P, _I64, _P, _P]
    lib.fldce_count_valid.restype = ctypes.c_int
    lib.fldce_selftest_wait.argtypes = [_I64, _P, _P]
    lib.fldce_selftest_wait.restype = ctypes.c_int
    lib.fldce_scale.argtypes = [_P, _I64, ctypes.c_int32, _P, _P]
    lib.fldce_scale.restype = ctypes.c_int
    lib.fldce_destroy.argtypes = [_P]
    lib.fldce_destroy.restype = ctypes.c_int
    lib.fldce_strerror.argtypes = [ctypes.c_int]
    lib.fldce_strerror.restype = ctypes.c_char_p
    lib.fldce_version.argtypes = []
    lib.fldce_version.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr() if x.numel() > 0 else None
    return int(x)


def _stream(s) -> Optional[int]:
    if s is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def _check(status: int, where: str) -> int:
    if status != FLDCE_OK:
        raise FldceError(status, where)
    return status


def fldce_strerror(status: int) -> str:
    return load().fldce_strerror(int(status)).decode()


def fldce_version() -> int:
    return load().fldce_version()


def fldce_create(dtype: int, D: int, V: int, max_N: int, *, chunk_N: int = 0,
                 logit_scale: float = 1.0, label_smoothing: float = 0.0,
                 ignore_index: int = -100, flags: int = 0, vocab_start: int = 0,
                 vocab_total: int = 0):
    """Returns (handle, workspace_bytes for max_N)."""
    cfg = fldce_config(int(dtype), int(flags), int(D), int(V), int(max_N), int(chunk_N),
                       float(logit_scale), float(label_smoothing), int(ignore_index),
                       int(vocab_start), int(vocab_total))
    h = _P()
    ws = ctypes.c_size_t()
    _check(load().fldce_create(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(ws)),
           "fldce_create")
    return h.value, ws.value


def fldce_workspace_size(h: int, N: int) -> int:
    ws = ctypes.c_size_t()
    _check(load().fldce_workspace_size(h, int(N), ctypes.byref(ws)), "fldce_workspace_size")
    return ws.value


def fldce_chunk_size(h) -> int:
    c = _I64()
    _check(load().fldce_chunk_size(h, ctypes.byref(c)), "fldce_chunk_size")
    return c.value


def fldce_fwd_bwd(h, H, W, target, p_mask, N, total, grad_out, loss, loss_per_token, lse,
                  argmax, dH, dW, workspace, workspace_bytes, err_count, stream=None) -> int:
    return _check(load().fldce_fwd_bwd(
        h, _ptr(H), _ptr(W), _ptr(target), _ptr(p_mask), int(N), float(total), float(grad_out),
        _ptr(loss), _ptr(loss_per_token), _ptr(lse), _ptr(argmax), _ptr(dH), _ptr(dW),
        _ptr(workspace), int(workspace_bytes), _ptr(err_count), _stream(stream)), "fldce_fwd_bwd")


def fldce_fwd_bwd_noalloc(h, H, W, target, p_mask, N, total, grad_out, loss, loss_per_token,
                          lse, argmax, dH, dW, err_count, stream=None) -> int:
    """fldce_fwd_bwd with the library's static scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/fldce.h)."""
    return _check(load().fldce_fwd_bwd_noalloc(
        h, _ptr(H), _ptr(W), _ptr(target), _ptr(p_mask), int(N), float(total), float(grad_out),
        _ptr(loss), _ptr(loss_per_token), _ptr(lse), _ptr(argmax), _ptr(dH), _ptr(dW),
        _ptr(err_count), _stream(stream)), "fldce_fwd_bwd_noalloc")


def fldce_forward(h, H, W, target, p_mask, N, total, loss, loss_per_token, lse, argmax,
                  workspace, workspace_bytes, err_count, stream=None) -> int:
    return _check(load().fldce_forward(
        h, _ptr(H), _ptr(W), _ptr(target), _ptr(p_mask), int(N), float(total), _ptr(loss),
        _ptr(loss_per_token), _ptr(lse), _ptr(argmax), _ptr(workspace), int(workspace_bytes),
        _ptr(err_count), _stream(stream)), "fldce_forward")


def fldce_profile_begin(h, max_calls: int) -> int:
    return _check(load().fldce_profile_begin(h, int(max_calls)), "fldce_profile_begin")


def fldce_profile_end(h) -> dict:
    """{kind name: (total ms, launches)} over the window just closed."""
    ms = (ctypes.c_double * FLDCE_PROF_KINDS)()
    n = (ctypes.c_int32 * FLDCE_PROF_KINDS)()
    _check(load().fldce_profile_end(h, ms, n), "fldce_profile_end")
    return {fldce_profile_kind_name(k): (ms[k], n[k]) for k in range(FLDCE_PROF_KINDS)}


def fldce_profile_kind_name(kind: int) -> str:
    r = load().fldce_profile_kind_name(int(kind))
    return r.decode() if r is not None else None


def make_call(**kw) -> fldce_call:
    """A zero-initialised fldce_call; tensors become device pointers."""
    c = fldce_call()
    for k, v in kw.items():
        if k == "stream":
            c.stream = _stream(v)
        elif k == "dw_ready_event":
            handle = None if v is None else (
                v.cuda_event if isinstance(v, torch.cuda.Event) else int(v))
            if v is not None and not handle:
                # a torch.cuda.Event has no CUDA event until its first record
                raise ValueError("dw_ready_event has no CUDA event yet: record it once first")
            c.dw_ready_event = handle
        elif k in ("N", "total", "grad_out", "workspace_bytes"):
            setattr(c, k, v)
        else:
            setattr(c, k, _ptr(v))
    return c


def fldce_fwd_bwd_ex(h, call: fldce_call) -> int:
    return _check(load().fldce_fwd_bwd_ex(h, ctypes.byref(call)), "fldce_fwd_bwd_ex")


def fldce_forward_ex(h, call: fldce_call) -> int:
    return _check(load().fldce_forward_ex(h, ctypes.byref(call)), "fldce_forward_ex")


def fldce_vp_stats(h, call: fldce_call, stats) -> int:
    return _check(load().fldce_vp_stats(h, ctypes.byref(call), _ptr(stats)), "fldce_vp_stats")


def fldce_vp_fwd_bwd(h, call: fldce_call, all_stats, n_shards: int) -> int:
    return _check(load().fldce_vp_fwd_bwd(h, ctypes.byref(call), _ptr(all_stats), int(n_shards)),
                  "fldce_vp_fwd_bwd")


def fldce_count_valid(h, target, N, count, stream=None) -> int:
    return _check(load().fldce_count_valid(h, _ptr(target), int(N), _ptr(count),
                                           _stream(stream)), "fldce_count_valid")


def fldce_scale(x, n, dtype, g, stream=None) -> int:
    return _check(load().fldce_scale(_ptr(x), int(n), int(dtype), _ptr(g), _stream(stream)),
                  "fldce_scale")


def fldce_selftest_wait(limit_ns: int, status, stream=None) -> int:
    return _check(load().fldce_selftest_wait(int(limit_ns), _ptr(status), _stream(stream)),
                  "fldce_selftest_wait")


def fldce_destroy(h) -> int:
    return _check(load().fldce_destroy(h), "fldce_destroy")


_TORCH_DTYPE = {FLDCE_BF16: torch.bfloat16, FLDCE_FP32: torch.float32}


class Plan:
    """A handle, its configuration and a device workspace sized for max_N."""

    def __init__(self, D: int, V: int, max_N: int, *, dtype: torch.dtype = torch.bfloat16,
                 chunk_N: int = 0, logit_scale: float = 1.0, label_smoothing: float = 0.0,
                 ignore_index: int = -100, dw_fp32: bool = False, skip_ignored: bool = False,
                 dh_fp32: bool = False, vocab_start: int = 0, vocab_total: int = 0,
                 dw_accumulate: bool = False, fused_dh: bool = False, device=None):
        code = FLDCE_BF16 if dtype == torch.bfloat16 else FLDCE_FP32
        if _TORCH_DTYPE[code] != dtype:
            raise TypeError(f"unsupported dtype {dtype}")
        self.dtype = dtype
        self.D, self.V, self.max_N = int(D), int(V), int(max_N)
        self.ignore_index = int(ignore_index)
        self.dw_fp32 = bool(dw_fp32)
        self.device = torch.device(device if device is not None else "cuda")
        self.handle, self.workspace_bytes = fldce_create(
            code, D, V, max_N, chunk_N=chunk_N, logit_scale=logit_scale,
            label_smoothing=label_smoothing, ignore_index=ignore_index,
            flags=(FLDCE_FLAG_DW_FP32 if dw_fp32 else 0) |
            (FLDCE_FLAG_SKIP_IGNORED if skip_ignored else 0) |
            (FLDCE_FLAG_DH_FP32 if dh_fp32 else 0) |
            (FLDCE_FLAG_DW_ACCUMULATE if dw_accumulate else 0) |
            (FLDCE_FLAG_FUSED_DH if fused_dh else 0),
            vocab_start=vocab_start, vocab_total=vocab_total)
        self.fused_dh = bool(fused_dh)
        self.dh_fp32 = bool(dh_fp32)
        self.dw_accumulate = bool(dw_accumulate)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)

    def close(self):
        if self.handle is not None:
            fldce_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def outputs(self, N: int, *, want_rows: bool = True, want_argmax: bool = False):
        """Output buffers for N tokens; dW starts at zero for a plan that
        accumulates into it."""
        dev = self.device
        new_dw = torch.zeros if self.dw_accumulate else torch.empty
        out = {
            "loss": torch.empty(1, dtype=torch.float32, device=dev),
            "dH": torch.empty(N, self.D, dtype=torch.float32 if self.dh_fp32 else self.dtype,
                              device=dev),
            "dW": new_dw(self.V, self.D,
                         dtype=torch.float32 if self.dw_fp32 else self.dtype, device=dev),
            "err": torch.empty(2, dtype=torch.int32, device=dev),
        }
        if want_rows:
            out["loss_per_token"] = torch.empty(N, dtype=torch.float32, device=dev)
            out["lse"] = torch.empty(N, dtype=torch.float32, device=dev)
        if want_argmax:
            out["argmax"] = torch.empty(N, dtype=torch.int32, device=dev)
        return out

    def fwd_bwd(self, H, W, target, p_mask, total: float, grad_out: float = 1.0,
                out: Optional[dict] = None, stream=None, bias=None, count_dev=None,
                dw_ready_event=None, **kw) -> dict:
        N = int(H.shape[0])
        if out is None:
            out = self.outputs(N, **kw)
            if bias is not None:
                new_db = torch.zeros if self.dw_accumulate else torch.empty
                out["db"] = new_db(self.V, device=self.device,
                                   dtype=torch.float32 if self.dw_fp32 else self.dtype)
        if bias is None and count_dev is None and dw_ready_event is None:
            fldce_fwd_bwd(self.handle, H, W, target, p_mask, N, total, grad_out, out["loss"],
                          out.get("loss_per_token"), out.get("lse"), out.get("argmax"),
                          out["dH"], out["dW"], self.workspace, self.workspace_bytes,
                          out["err"], stream)
        else:
            call = make_call(H=H, W=W, bias=bias, target=target, p_mask=p_mask, N=N,
                             total=float(total), grad_out=float(grad_out), count_dev=count_dev,
                             loss=out["loss"], loss_per_token=out.get("loss_per_token"),
                             lse=out.get("lse"), argmax=out.get("argmax"), dH=out["dH"],
                             dW=out["dW"], db=out.get("db"), workspace=self.workspace,
                             workspace_bytes=self.workspace_bytes, err_count=out["err"],
                             stream=stream, dw_ready_event=dw_ready_event)
            fldce_fwd_bwd_ex(self.handle, call)
        return out

    def forward(self, H, W, target, p_mask, total: float, out: Optional[dict] = None,
                stream=None, want_argmax: bool = False) -> dict:
        N = int(H.shape[0])
        dev = self.device
        if out is None:
            out = {"loss": torch.empty(1, dtype=torch.float32, device=dev),
                   "loss_per_token": torch.empty(N, dtype=torch.float32, device=dev),
                   "lse": torch.empty(N, dtype=torch.float32, device=dev),
                   "err": torch.empty(2, dtype=torch.int32, device=dev)}
            if want_argmax:
                out["argmax"] = torch.empty(N, dtype=torch.int32, device=dev)
        fldce_forward(self.handle, H, W, target, p_mask, N, total, out["loss"],
                      out.get("loss_per_token"), out.get("lse"), out.get("argmax"),
                      self.workspace, self.workspace_bytes, out["err"], stream)
        return out
