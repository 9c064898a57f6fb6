"""ctypes binding of libattn.so (include/attn.h).

Argument marshalling only: the functions here turn torch tensors into device
pointers, sizes and the current CUDA stream and call the C ABI; every step of
the computation runs in the library's kernels.  If the library is missing or
a call fails, they raise; there is no fallback.
"""

from __future__ import annotations

import ctypes
import math
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libattn.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "attn.h")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT, ATTN_ERR_SCRATCH_LIMIT, ATTN_ERR_SMEM, \
    ATTN_ERR_RANGE = range(8)
ATTN_FP16, ATTN_BF16 = 0, 1
ATTN_BWD_ALL, ATTN_BWD_PREPROCESS, ATTN_BWD_MAIN, ATTN_BWD_CONVERT = range(4)
ATTN_CAUSAL_NONE, ATTN_CAUSAL_TOP_LEFT, ATTN_CAUSAL_BOTTOM_RIGHT = range(3)
_CAUSAL_NAMES = {"none": ATTN_CAUSAL_NONE, "top_left": ATTN_CAUSAL_TOP_LEFT, "bottom_right": ATTN_CAUSAL_BOTTOM_RIGHT}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, where: str, status: int, message: str):
        super().__init__(f"{where}: {message} (status {status})")
        self.status = status


def load() -> ctypes.CDLL:
    """Loads libattn.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_attention_150_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.attn_fwd.restype = st
    lib.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, vp]
    lib.attn_fwd_fp8.restype = st
    lib.attn_fwd_fp8_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, f, f, f, i, vp]
    lib.attn_fwd_fp8_varlen.restype = st
    lib.attn_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.attn_bwd.restype = st
    lib.attn_bwd_phase.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    lib.attn_bwd_phase.restype = st
    lib.attn_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.attn_bwd_deterministic.restype = st
    lib.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, vp]
    lib.attn_fwd_varlen.restype = st
    lib.attn_bwd_varlen_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.attn_bwd_varlen_workspace_bytes.restype = ctypes.c_size_t
    lib.attn_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i,
                                    vp]
    lib.attn_bwd_varlen.restype = st
    lib.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.attn_bwd_noalloc.restype = st
    lib.attn_bwd_noalloc_max_scratch_bytes.argtypes = []
    lib.attn_bwd_noalloc_max_scratch_bytes.restype = ctypes.c_size_t
    lib.attn_host_step_device_bytes.argtypes = [i, i, i, i, i, i]
    lib.attn_host_step_device_bytes.restype = ctypes.c_size_t
    lib.attn_host_step.argtypes = [vp] * 10 + [ctypes.c_size_t, i, i, i, i, i, f, i, i, i, i, vp]
    lib.attn_host_step.restype = st
    lib.attn_selftest_wait_timeout.argtypes = [i, vp, vp]
    lib.attn_selftest_wait_timeout.restype = st
    lib.attn_last_device_status.argtypes = [vp]
    lib.attn_last_device_status.restype = st
    lib.attn_status_string.argtypes = [st]
    lib.attn_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def declared_symbols() -> list[str]:
    """Names of the functions include/attn.h declares."""
    text = open(HEADER).read()
    return re.findall(r"^\S.*?\b(attn_\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    return load().attn_status_string(status).decode()


def _check(where: str, status: int) -> None:
    if status != ATTN_OK:
        raise AttnError(where, status, status_string(status))


# ---------------------------------------------------------------- raw C ABI

def attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Direct call of attn_fwd with integer device pointers; returns the status."""
    return load().attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, int(causal), dtype, stream)


def attn_fwd_fp8(q, k, v, o, lse, B, H, Nq, Nk, d, scale, descale_q, descale_k, descale_v, causal, stream) -> int:
    """Direct call of attn_fwd_fp8 (E4M3 inputs, bf16 output); returns the status."""
    return load().attn_fwd_fp8(q, k, v, o, lse, B, H, Nq, Nk, d, scale, descale_q, descale_k, descale_v, int(causal),
                               stream)


def attn_fwd_fp8_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k, d, scale, descale_q,
                        descale_k, descale_v, causal, stream) -> int:
    """Direct call of attn_fwd_fp8_varlen; returns the status."""
    return load().attn_fwd_fp8_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k, d, scale,
                                      descale_q, descale_k, descale_v, int(causal), stream)


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Direct call of attn_bwd with integer device pointers; returns the status."""
    return load().attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, int(causal),
                           dtype, stream)


def attn_bwd_phase(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, causal, dtype, phase,
                   stream) -> int:
    """Direct call of attn_bwd_phase (one of the three backward kernels)."""
    return load().attn_bwd_phase(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale,
                                 int(causal), dtype, phase, stream)


def attn_bwd_deterministic(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale, causal, dtype,
                           stream) -> int:
    """Direct call of attn_bwd_deterministic (bit-reproducible dQ)."""
    return load().attn_bwd_deterministic(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, H, Nq, Nk, d, scale,
                                         int(causal), dtype, stream)


def attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Direct call of attn_bwd_noalloc: the backward pass with the library's
    fixed scratch array as workspace, for callers that cannot allocate device
    memory when they call (see include/attn.h)."""
    return load().attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, Nq, Nk, d, scale, int(causal), dtype,
                                   stream)


def attn_bwd_noalloc_max_scratch_bytes() -> int:
    return int(load().attn_bwd_noalloc_max_scratch_bytes())


def attn_host_step_device_bytes(B, H, Nq, Nk, d, chunks) -> int:
    return int(load().attn_host_step_device_bytes(B, H, Nq, Nk, d, chunks))


def attn_host_step(q, k, v, dout, o, lse, dq, dk, dv, device_buffer, device_bytes, B, H, Nq, Nk, d, scale, causal,
                   dtype, chunks, deterministic, stream) -> int:
    """Direct call of attn_host_step (host pointers for the tensors, a device
    pointer for the buffer); returns the status."""
    return load().attn_host_step(q, k, v, dout, o, lse, dq, dk, dv, device_buffer, device_bytes, B, H, Nq, Nk, d,
                                 scale, int(causal), dtype, chunks, int(deterministic), stream)


def attn_bwd_workspace_bytes(B, H, Nq, Nk, d) -> int:
    return int(load().attn_bwd_workspace_bytes(B, H, Nq, Nk, d))


def attn_last_device_status(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(load().attn_last_device_status(stream))


# ---------------------------------------------------------------- tensors

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return ATTN_FP16
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"attention inputs must be float16 or bfloat16, got {t.dtype}")


def _check_tensor(name: str, t: torch.Tensor, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def causal_code(causal) -> int:
    """The C ABI's `causal` value: False/True (top-left), an attn_causal
    integer, or "none" / "top_left" / "bottom_right"."""
    if isinstance(causal, str):
        if causal not in _CAUSAL_NAMES:
            raise ValueError(f"causal must be one of {sorted(_CAUSAL_NAMES)}, got {causal!r}")
        return _CAUSAL_NAMES[causal]
    return int(causal)


def forward(q, k, v, causal=False, scale: float | None = None, out=None, lse=None, stream=None):
    """O, LSE = attention(q, k, v) for q [B,H,Nq,d], k and v [B,H,Nk,d]."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    code = _dtype_code(q)
    _check_tensor("q", q, (B, H, Nq, d), q.dtype)
    _check_tensor("k", k, (B, H, Nk, d), q.dtype)
    _check_tensor("v", v, (B, H, Nk, d), q.dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, (B, H, Nq, d), q.dtype)
    _check_tensor("lse", lse, (B, H, Nq), torch.float32)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    _check("attn_fwd", attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                B, H, Nq, Nk, d, float(scale), causal_code(causal), code, stream))
    return out, lse


def forward_fp8(q, k, v, descale_q: float, descale_k: float, descale_v: float, causal=False,
                scale: float | None = None, out=None, lse=None, stream=None):
    """O (bf16), LSE of attention over E4M3 inputs q [B,H,Nq,128], k and v
    [B,H,Nk,128] (torch.float8_e4m3fn) that stand for descale_x * x."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    e4m3 = torch.float8_e4m3fn
    _check_tensor("q", q, (B, H, Nq, d), e4m3)
    _check_tensor("k", k, (B, H, Nk, d), e4m3)
    _check_tensor("v", v, (B, H, Nk, d), e4m3)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, (B, H, Nq, d), torch.bfloat16)
    _check_tensor("lse", lse, (B, H, Nq), torch.float32)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    _check("attn_fwd_fp8", attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        B, H, Nq, Nk, d, float(scale), float(descale_q), float(descale_k),
                                        float(descale_v), causal_code(causal), stream))
    return out, lse


def backward(q, k, v, out, lse, dout, causal=False, scale: float | None = None,
             dq=None, dk=None, dv=None, workspace=None, stream=None, phase: int = ATTN_BWD_ALL,
             deterministic: bool = False):
    """dQ, dK, dV of attention for the output gradient dout.  `phase` runs
    only one of the three backward kernels (see attn_bwd_phase);
    `deterministic` selects attn_bwd_deterministic (all phases)."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    code = _dtype_code(q)
    for name, t, shp in (("q", q, (B, H, Nq, d)), ("k", k, (B, H, Nk, d)), ("v", v, (B, H, Nk, d)),
                         ("out", out, (B, H, Nq, d)), ("dout", dout, (B, H, Nq, d))):
        _check_tensor(name, t, shp, q.dtype)
    _check_tensor("lse", lse, (B, H, Nq), torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        _check_tensor(name, t, ref.shape, q.dtype)
    nbytes = attn_bwd_workspace_bytes(B, H, Nq, Nk, d)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < nbytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), workspace.data_ptr())
    if deterministic:
        if phase != ATTN_BWD_ALL:
            raise ValueError("the deterministic backward runs all phases")
        _check("attn_bwd_deterministic",
               attn_bwd_deterministic(*ptrs, B, H, Nq, Nk, d, float(scale), causal_code(causal), code, stream))
    else:
        _check("attn_bwd", attn_bwd_phase(*ptrs, B, H, Nq, Nk, d, float(scale), causal_code(causal), code, phase,
                                          stream))
    return dq, dk, dv


# ------------------------------------------------ packed variable-length

def attn_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k, d, scale, causal, dtype,
                    stream) -> int:
    """Direct call of attn_fwd_varlen with integer device pointers."""
    return load().attn_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k, d, scale,
                                  int(causal), dtype, stream)


def attn_bwd_varlen_workspace_bytes(B, H, total_q, max_q, d) -> int:
    return int(load().attn_bwd_varlen_workspace_bytes(B, H, total_q, max_q, d))


def attn_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_q, cu_k, B, H, total_q, total_k, max_q, max_k,
                    d, scale, causal, dtype, deterministic, stream) -> int:
    """Direct call of attn_bwd_varlen with integer device pointers."""
    return load().attn_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_q, cu_k, B, H, total_q, total_k,
                                  max_q, max_k, d, scale, int(causal), dtype, int(deterministic), stream)


def _check_cu(name, cu, B):
    if not cu.is_cuda or cu.dtype != torch.int32 or tuple(cu.shape) != (B + 1,) or not cu.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA int32 tensor of shape ({B + 1},)")


def forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int, causal=False,
                   scale: float | None = None, out=None, lse=None, stream=None):
    """O, LSE of a packed variable-length batch: q [H, total_q, d], k and v
    [H, total_k, d]; sequence b is rows cu_seqlens[b]:cu_seqlens[b+1]."""
    H, total_q, d = q.shape
    total_k = k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    code = _dtype_code(q)
    _check_tensor("q", q, (H, total_q, d), q.dtype)
    _check_tensor("k", k, (H, total_k, d), q.dtype)
    _check_tensor("v", v, (H, total_k, d), q.dtype)
    _check_cu("cu_seqlens_q", cu_seqlens_q, B)
    _check_cu("cu_seqlens_k", cu_seqlens_k, B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, (H, total_q, d), q.dtype)
    _check_tensor("lse", lse, (H, total_q), torch.float32)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    _check("attn_fwd_varlen", attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                              cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, total_q,
                                              total_k, int(max_seqlen_q), int(max_seqlen_k), d, float(scale),
                                              causal_code(causal), code, stream))
    return out, lse


def forward_fp8_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                       descale_q: float, descale_k: float, descale_v: float, causal=False,
                       scale: float | None = None, out=None, lse=None, stream=None):
    """O (bf16), LSE of a packed variable-length batch of E4M3 inputs: q
    [H, total_q, 128], k and v [H, total_k, 128] (torch.float8_e4m3fn)."""
    H, total_q, d = q.shape
    total_k = k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    e4m3 = torch.float8_e4m3fn
    _check_tensor("q", q, (H, total_q, d), e4m3)
    _check_tensor("k", k, (H, total_k, d), e4m3)
    _check_tensor("v", v, (H, total_k, d), e4m3)
    _check_cu("cu_seqlens_q", cu_seqlens_q, B)
    _check_cu("cu_seqlens_k", cu_seqlens_k, B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((H, total_q, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, (H, total_q, d), torch.bfloat16)
    _check_tensor("lse", lse, (H, total_q), torch.float32)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    _check("attn_fwd_fp8_varlen",
           attn_fwd_fp8_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                               cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, total_q, total_k,
                               int(max_seqlen_q), int(max_seqlen_k), d, float(scale), float(descale_q),
                               float(descale_k), float(descale_v), causal_code(causal), stream))
    return out, lse


def backward_varlen(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    causal=False, scale: float | None = None, dq=None, dk=None, dv=None, workspace=None,
                    deterministic: bool = False, stream=None):
    """dQ, dK, dV of forward_varlen for the output gradient dout."""
    H, total_q, d = q.shape
    total_k = k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    code = _dtype_code(q)
    for name, t, shp in (("q", q, (H, total_q, d)), ("k", k, (H, total_k, d)), ("v", v, (H, total_k, d)),
                         ("out", out, (H, total_q, d)), ("dout", dout, (H, total_q, d))):
        _check_tensor(name, t, shp, q.dtype)
    _check_tensor("lse", lse, (H, total_q), torch.float32)
    _check_cu("cu_seqlens_q", cu_seqlens_q, B)
    _check_cu("cu_seqlens_k", cu_seqlens_k, B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = attn_bwd_varlen_workspace_bytes(B, H, total_q, int(max_seqlen_q), d)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < nbytes or not workspace.is_cuda:
        raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    _check("attn_bwd_varlen", attn_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                              lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                              dv.data_ptr(), workspace.data_ptr(), cu_seqlens_q.data_ptr(),
                                              cu_seqlens_k.data_ptr(), B, H, total_q, total_k, int(max_seqlen_q),
                                              int(max_seqlen_k), d, float(scale), causal_code(causal), code,
                                              deterministic, stream))
    return dq, dk, dv


def _check_host(name: str, t: torch.Tensor, shape, dtype) -> None:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def host_step(q, k, v, dout, causal=False, scale: float | None = None, chunks: int = 4,
              deterministic: bool = False, outs=None, device_buffer=None, device=None, stream=None):
    """Forward and backward of host-resident q [B,H,Nq,d], k and v
    [B,H,Nk,d] and dout [B,H,Nq,d] through attn_host_step: the copies of one
    chunk of slices overlap the kernels of another.  Returns (o, lse, dq, dk,
    dv) in host memory (page-locked when allocated here).  The call is
    asynchronous on `stream`: synchronize it before reading the results."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    code = _dtype_code(q)
    for name, t, shp in (("q", q, (B, H, Nq, d)), ("k", k, (B, H, Nk, d)), ("v", v, (B, H, Nk, d)),
                         ("dout", dout, (B, H, Nq, d))):
        _check_host(name, t, shp, q.dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if outs is None:
        outs = (torch.empty((B, H, Nq, d), dtype=q.dtype, pin_memory=True),
                torch.empty((B, H, Nq), dtype=torch.float32, pin_memory=True),
                torch.empty((B, H, Nq, d), dtype=q.dtype, pin_memory=True),
                torch.empty((B, H, Nk, d), dtype=q.dtype, pin_memory=True),
                torch.empty((B, H, Nk, d), dtype=q.dtype, pin_memory=True))
    o, lse, dq, dk, dv = outs
    for name, t, shp, dt in (("o", o, (B, H, Nq, d), q.dtype), ("lse", lse, (B, H, Nq), torch.float32),
                             ("dq", dq, (B, H, Nq, d), q.dtype), ("dk", dk, (B, H, Nk, d), q.dtype),
                             ("dv", dv, (B, H, Nk, d), q.dtype)):
        _check_host(name, t, shp, dt)
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    nbytes = attn_host_step_device_bytes(B, H, Nq, Nk, d, chunks)
    if device_buffer is None:
        device_buffer = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    if not device_buffer.is_cuda or device_buffer.numel() * device_buffer.element_size() < nbytes:
        raise ValueError(f"device_buffer must be a CUDA buffer of at least {nbytes} bytes")
    if device_buffer.device != device:
        raise ValueError(f"device_buffer is on {device_buffer.device}, expected {device}")
    if stream is None:
        stream = torch.cuda.current_stream(device).cuda_stream
    with torch.cuda.device(device):  # the library's internal copy streams belong to the current device
        status = attn_host_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), device_buffer.data_ptr(),
                                device_buffer.numel(), B, H, Nq, Nk, d, float(scale), causal_code(causal), code,
                                int(chunks), deterministic, stream)
    _check("attn_host_step", status)
    return o, lse, dq, dk, dv


def selftest_wait_timeout(limit_us: int, result, stream=None) -> int:
    """Launches the failure-detection self-test (see include/attn.h); result
    is a CUDA int32 tensor of 2 elements.  Returns the launch status."""
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(load().attn_selftest_wait_timeout(int(limit_us), result.data_ptr() if result is not None else None,
                                                  stream))


def device_status(stream=None) -> None:
    """Raises if a kernel of the library recorded an error (e.g. a wait timeout)."""
    _check("attn_last_device_status", attn_last_device_status(stream))
