"""ctypes binding of libfa.so (include/fa.h). Argument marshalling only: every step of the
attention forward and backward runs in the library's CUDA kernels.

The functions named like the C entry points (fa_fwd, fa_bwd, fa_bwd_workspace_size,
fa_check_status, fa_last_error_string) take torch CUDA tensors that the caller allocated;
``attention_forward`` / ``attention_backward`` allocate the outputs with torch and call them.
There is no fallback: if libfa.so is missing or the device is not an sm_100 GPU, the calls
raise.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_OK = 0
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
                3: "FA_ERR_MISALIGNED", 4: "FA_ERR_CUDA", 5: "FA_ERR_TIMEOUT",
                6: "FA_ERR_WORKSPACE"}

# (name, restype, argtypes) of every symbol include/fa.h declares.
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_workspace_size": (_Z, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _I, _I, _I, _I, _F, _I, _P]),
    "fa_check_status": (_I, [_P]),
    "fa_last_error_string": (ctypes.c_char_p, []),
    "fa_version": (ctypes.c_char_p, []),
    "fa_profile_enable": (_I, [_I]),
    "fa_profile_read": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong), _I]),
    "fa_kernel_name": (ctypes.c_char_p, [_I]),
    "fa_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_selftest_timeout": (_I, [_I, _P]),
    "fa_debug_stall_next": (_I, [_I, _I, _I]),
    "fa_fwd_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "fa_bwd_ex_workspace_size": (_Z, [_P]),
    "fa_bwd_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P, _P, _P]),
    "fa_fwd_fp8_workspace_size": (_Z, [_P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _F, _F, _F, _P, _P, _P, _P, _Z, _P]),
}

# fa_mask values
MASK_NONE, MASK_CAUSAL, MASK_CAUSAL_BOTTOM_RIGHT = 0, 1, 2


class FaAttnShape(ctypes.Structure):
    """struct fa_attn_shape of include/fa.h."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("N_q", ctypes.c_int), ("N_kv", ctypes.c_int), ("d", ctypes.c_int),
                ("scale", ctypes.c_float), ("mask", ctypes.c_int)]


class FaDropout(ctypes.Structure):
    """struct fa_dropout of include/fa.h."""
    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint)]


def _dropout_arg(dropout):
    """None, or (p, seed, offset) -> a pointer to an fa_dropout (None stays a NULL pointer)."""
    if dropout is None:
        return None
    p, seed, offset = dropout
    return ctypes.byref(FaDropout(float(p), int(seed), int(offset)))


def mask_code(causal) -> int:
    """False / "none" -> no mask; True / "top_left" -> causal aligned at the top left;
    "bottom_right" -> causal aligned at the bottom right (key j visible to query i iff
    j <= i + N_kv - N_q)."""
    if causal is False or causal is None or causal == "none":
        return MASK_NONE
    if causal is True or causal == "top_left":
        return MASK_CAUSAL
    if causal == "bottom_right":
        return MASK_CAUSAL_BOTTOM_RIGHT
    raise ValueError(f"unknown mask {causal!r}")


KERNEL_KINDS = 9

_lib = None


class FaError(RuntimeError):
    def __init__(self, where: str, status: int, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Loads libfa.so (built in-tree by exact_io_aware_66_b200.build); raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m exact_io_aware_66_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(where: str, status: int):
    if status != FA_OK:
        raise FaError(where, status, fa_last_error_string())


def fa_last_error_string() -> str:
    return (lib().fa_last_error_string() or b"").decode()


def fa_version() -> str:
    return lib().fa_version().decode()


def default_scale(d: int) -> float:
    """1/sqrt(d) rounded to fp32 — the value passed to the kernels."""
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32).item())


def _stream_handle(stream, device=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and isinstance(stream, torch.cuda.Stream) and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _one_device(**tensors) -> torch.device:
    """The CUDA device that every argument tensor is on. The library launches on the calling
    thread's current device, so each call below runs with this device made current; tensors on
    different GPUs are refused here rather than handed to a kernel on the wrong one."""
    dev = None
    for name, t in tensors.items():
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {dev}")
    return dev


def _dims(x: torch.Tensor):
    if x.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    return tuple(int(s) for s in x.shape)


def _req(x: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if x.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return x.data_ptr()


def fa_fwd(q, k, v, o, lse, causal: bool = False, scale: float | None = None, stream=None):
    """Forward into caller-allocated o (bf16 [B,H,N,d]) and lse (fp32 [B,H,N])."""
    B, H, N, d = _dims(q)
    for t, n in ((k, "k"), (v, "v"), (o, "o")):
        if _dims(t) != (B, H, N, d):
            raise ValueError(f"{n} shape mismatch")
    if tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    dev = _one_device(q=q, k=k, v=v, o=o, lse=lse)
    ptrs = [_req(q, "q"), _req(k, "k"), _req(v, "v"), _req(o, "o"), _req(lse, "lse", torch.float32)]
    scale = default_scale(d) if scale is None else float(scale)
    with torch.cuda.device(dev):
        st = lib().fa_fwd(*ptrs, B, H, N, d, scale, int(bool(causal)), _stream_handle(stream, dev))
    _check("fa_fwd", st)


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, do, lse, dq, dk, dv, workspace, causal: bool = False,
           scale: float | None = None, stream=None):
    """Backward into caller-allocated dq, dk, dv (bf16 [B,H,N,d]) using a caller-owned
    workspace (uint8 CUDA tensor of at least fa_bwd_workspace_size bytes)."""
    B, H, N, d = _dims(q)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (do, "do"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        if _dims(t) != (B, H, N, d):
            raise ValueError(f"{n} shape mismatch")
    if tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ptrs = [_req(q, "q"), _req(k, "k"), _req(v, "v"), _req(o, "o"), _req(do, "do"),
            _req(lse, "lse", torch.float32), _req(dq, "dq"), _req(dk, "dk"), _req(dv, "dv")]
    dev = _one_device(q=q, k=k, v=v, o=o, do=do, lse=lse, dq=dq, dk=dk, dv=dv,
                      workspace=workspace)
    wbytes = workspace.numel() * workspace.element_size()
    scale = default_scale(d) if scale is None else float(scale)
    with torch.cuda.device(dev):
        st = lib().fa_bwd(*ptrs, workspace.data_ptr(), wbytes, B, H, N, d, scale,
                          int(bool(causal)), _stream_handle(stream, dev))
    _check("fa_bwd", st)


def fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal: bool = False,
                   scale: float | None = None, stream=None):
    """Backward into caller-allocated dq, dk, dv with the library's built-in scratch instead of
    a workspace, for callers that cannot allocate device memory (see include/fa.h: 64 MiB
    limit; calls that overlap on the GPU race on the shared scratch)."""
    B, H, N, d = _dims(q)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (do, "do"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        if _dims(t) != (B, H, N, d):
            raise ValueError(f"{n} shape mismatch")
    if tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    ptrs = [_req(q, "q"), _req(k, "k"), _req(v, "v"), _req(o, "o"), _req(do, "do"),
            _req(lse, "lse", torch.float32), _req(dq, "dq"), _req(dk, "dk"), _req(dv, "dv")]
    dev = _one_device(q=q, k=k, v=v, o=o, do=do, lse=lse, dq=dq, dk=dk, dv=dv)
    scale = default_scale(d) if scale is None else float(scale)
    with torch.cuda.device(dev):
        st = lib().fa_bwd_noalloc(*ptrs, B, H, N, d, scale, int(bool(causal)),
                                  _stream_handle(stream, dev))
    _check("fa_bwd_noalloc", st)


def fa_profile_enable(on: bool = True):
    _check("fa_profile_enable", lib().fa_profile_enable(int(bool(on))))


def fa_profile_read() -> dict:
    """{kernel name: (launches, summed device ms)} since the last read."""
    ms = (ctypes.c_double * KERNEL_KINDS)()
    n = (ctypes.c_longlong * KERNEL_KINDS)()
    _check("fa_profile_read", lib().fa_profile_read(ms, n, KERNEL_KINDS))
    return {lib().fa_kernel_name(i).decode(): (int(n[i]), float(ms[i]))
            for i in range(KERNEL_KINDS)}


def fa_selftest_timeout(limit_us: int = 20000, stream=None):
    """Launches the bounded-wait self-test kernel (see include/fa.h); follow with
    fa_check_status(), which must then raise FaError with FA_ERR_TIMEOUT."""
    _check("fa_selftest_timeout", lib().fa_selftest_timeout(int(limit_us), _stream_handle(stream)))


def fa_debug_stall_next(kind: int, skip: int = 0, limit_us: int = 20000):
    """Arms the failure-detection test hook for the next launch of kernel kind `kind` on this
    thread (0 forward, 2 backward main; -1 disarms): that launch leaves out one load, its wait
    runs out after limit_us and the call's fa_check_status() raises FA_ERR_TIMEOUT."""
    _check("fa_debug_stall_next", lib().fa_debug_stall_next(int(kind), int(skip), int(limit_us)))


def fa_check_status(stream=None):
    """Synchronises the stream and raises FaError if an in-kernel wait timed out."""
    _check("fa_check_status", lib().fa_check_status(_stream_handle(stream)))


def _shape(q, k, v, causal, scale) -> FaAttnShape:
    B, H, N_q, d = _dims(q)
    Bk, H_kv, N_kv, dk = _dims(k)
    if Bk != B or dk != d:
        raise ValueError("k must be [B, H_kv, N_kv, d] with q's B and d")
    if _dims(v) != (B, H_kv, N_kv, d):
        raise ValueError("v shape mismatch")
    scale = default_scale(d) if scale is None else float(scale)
    return FaAttnShape(B, H, H_kv, N_q, N_kv, d, scale, mask_code(causal))


def fa_fwd_ex(q, k, v, o, lse, causal=False, scale: float | None = None, stream=None,
              dropout=None):
    """Forward for q [B,H,N_q,d] and k, v [B,H_kv,N_kv,d] (H a multiple of H_kv) into
    caller-allocated o (like q) and lse (fp32 [B,H,N_q]); causal as in mask_code; dropout None
    or (p, seed, offset) as in include/fa.h."""
    s = _shape(q, k, v, causal, scale)
    if _dims(o) != (s.B, s.H, s.N_q, s.d):
        raise ValueError("o shape mismatch")
    if tuple(lse.shape) != (s.B, s.H, s.N_q):
        raise ValueError("lse must be [B, H, N_q]")
    dev = _one_device(q=q, k=k, v=v, o=o, lse=lse)
    ptrs = [_req(q, "q"), _req(k, "k"), _req(v, "v"), _req(o, "o"), _req(lse, "lse", torch.float32)]
    with torch.cuda.device(dev):
        st = lib().fa_fwd_ex(*ptrs, ctypes.byref(s), _dropout_arg(dropout),
                             _stream_handle(stream, dev))
    _check("fa_fwd_ex", st)


def fa_bwd_ex_workspace_size(B: int, H: int, H_kv: int, N_q: int, N_kv: int, d: int,
                             causal=False) -> int:
    s = FaAttnShape(B, H, H_kv, N_q, N_kv, d, default_scale(d) if d > 0 else 1.0,
                    mask_code(causal))
    return int(lib().fa_bwd_ex_workspace_size(ctypes.byref(s)))


def fa_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, workspace, causal=False,
              scale: float | None = None, stream=None, dropout=None):
    """Backward for the shapes of fa_fwd_ex into caller-allocated dq (like q), dk, dv (like k)
    with a caller-owned workspace of at least fa_bwd_ex_workspace_size bytes; dropout as given
    to the forward that produced o and lse."""
    s = _shape(q, k, v, causal, scale)
    for t, n in ((o, "o"), (do, "do"), (dq, "dq")):
        if _dims(t) != (s.B, s.H, s.N_q, s.d):
            raise ValueError(f"{n} shape mismatch")
    for t, n in ((dk, "dk"), (dv, "dv")):
        if _dims(t) != (s.B, s.H_kv, s.N_kv, s.d):
            raise ValueError(f"{n} shape mismatch")
    if tuple(lse.shape) != (s.B, s.H, s.N_q):
        raise ValueError("lse must be [B, H, N_q]")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ptrs = [_req(q, "q"), _req(k, "k"), _req(v, "v"), _req(o, "o"), _req(do, "do"),
            _req(lse, "lse", torch.float32), _req(dq, "dq"), _req(dk, "dk"), _req(dv, "dv")]
    dev = _one_device(q=q, k=k, v=v, o=o, do=do, lse=lse, dq=dq, dk=dk, dv=dv,
                      workspace=workspace)
    wbytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib().fa_bwd_ex(*ptrs, workspace.data_ptr(), wbytes, ctypes.byref(s),
                             _dropout_arg(dropout), _stream_handle(stream, dev))
    _check("fa_bwd_ex", st)


def _req8(x: torch.Tensor, name: str):
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if x.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise ValueError(f"{name} must hold E4M3 codes (torch.float8_e4m3fn or uint8)")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return x.data_ptr()


def fa_fwd_fp8_workspace_size(B: int, H: int, H_kv: int, N_q: int, N_kv: int, d: int,
                              causal=False) -> int:
    s = FaAttnShape(B, H, H_kv, N_q, N_kv, d, default_scale(d) if d > 0 else 1.0,
                    mask_code(causal))
    return int(lib().fa_fwd_fp8_workspace_size(ctypes.byref(s)))


def fa_fwd_fp8(q8, k8, v8, descale, o, lse, causal=False, scale: float | None = None,
               stream=None, workspace=None):
    """FP8 forward: q8 [B,H,N_q,d], k8 and v8 [B,H_kv,N_kv,d] E4M3 codes with descale =
    (q, k, v) fp32 factors, into caller-allocated o (bf16, like q8) and lse (fp32 [B,H,N_q]).
    Allocates the V^T workspace unless one is given."""
    s = _shape(q8, k8, v8, causal, scale)
    if _dims(o) != (s.B, s.H, s.N_q, s.d):
        raise ValueError("o shape mismatch")
    if tuple(lse.shape) != (s.B, s.H, s.N_q):
        raise ValueError("lse must be [B, H, N_q]")
    if workspace is None:
        workspace = torch.empty(max(16, int(lib().fa_fwd_fp8_workspace_size(ctypes.byref(s)))),
                                dtype=torch.uint8, device=q8.device)
    qd, kd, vd = (float(x) for x in descale)
    dev = _one_device(q8=q8, k8=k8, v8=v8, o=o, lse=lse, workspace=workspace)
    ptrs = [_req8(q8, "q8"), _req8(k8, "k8"), _req8(v8, "v8")]
    with torch.cuda.device(dev):
        st = lib().fa_fwd_fp8(*ptrs, qd, kd, vd, _req(o, "o"), _req(lse, "lse", torch.float32),
                              ctypes.byref(s), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(),
                              _stream_handle(stream, dev))
    _check("fa_fwd_fp8", st)


def attention_forward_fp8(q8, k8, v8, descale, causal=False, scale: float | None = None,
                          stream=None):
    """Returns (o bf16, lse fp32) of the FP8 forward (see fa_fwd_fp8)."""
    B, H, N, d = _dims(q8)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    fa_fwd_fp8(q8, k8, v8, descale, o, lse, causal, scale, stream)
    return o, lse


def attention_forward(q, k, v, causal=False, scale: float | None = None, stream=None,
                      dropout=None):
    """Returns (o, lse) for bf16 CUDA tensors q [B, H, N_q, d] and k, v [B, H_kv, N_kv, d]
    (H_kv = H and N_kv = N_q in the square case); causal as in mask_code; dropout None or
    (p, seed, offset)."""
    B, H, N, d = _dims(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    fa_fwd_ex(q, k, v, o, lse, causal, scale, stream, dropout)
    return o, lse


def attention_backward(q, k, v, o, do, lse, causal=False, scale: float | None = None,
                       stream=None, workspace=None, dropout=None):
    """Returns (dq, dk, dv) for the shapes of attention_forward (dropout as given to it).
    Allocates the workspace unless one is given."""
    B, H, N, d = _dims(q)
    _, H_kv, N_kv, _ = _dims(k)
    if workspace is None:
        workspace = torch.empty(fa_bwd_ex_workspace_size(B, H, H_kv, N, N_kv, d, causal),
                                dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa_bwd_ex(q, k, v, o, do, lse, dq, dk, dv, workspace, causal, scale, stream, dropout)
    return dq, dk, dv
