"""ctypes binding of liblinattn.so (the C ABI in include/linattn.h).

Argument marshalling only: every function checks that the torch tensors it is
handed are contiguous CUDA tensors of the right dtype, reads their shapes and
data pointers, and calls the C entry point of the same name on the current
torch stream (or the stream given).  No step of the computation runs here.
The library is loaded on first use; when it is missing the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT = range(5)
LA_F32, LA_BF16 = 0, 1

_DTYPES = {torch.float32: LA_F32, torch.bfloat16: LA_BF16}
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "liblinattn.so"

_lib = None
_lock = threading.Lock()


class LinAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {la_status_string(status)}"
        if status == LA_ERR_CUDA:
            msg += f" ({last_cuda_error()})"
        super().__init__(msg)
        self.status = status


def lib_path() -> str:
    return os.environ.get("LINATTN_LIB", os.path.join(_HERE, _LIB_NAME))


def load_library():
    """Load liblinattn.so (raises OSError if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise OSError(f"{path} not found: build it with "
                          "`python -m recurrent_decode_la_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        lib.la_state_init.argtypes = [vp, vp, i64, i32, i32, vp]
        lib.la_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, i32,
                                   vp, i32, i64, i32, vp, sz, vp]
        lib.la_prefill_workspace_size.argtypes = [i32, i32, i32, i64, i32, i32, i32, i32]
        lib.la_prefill_workspace_size.restype = sz
        lib.la_decode_step.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
        lib.la_device_status.argtypes = [vp]
        lib.la_selftest_wait_timeout.argtypes = [ctypes.c_double, vp]
        lib.la_selftest_wait_timeout.restype = ctypes.c_int
        lib.la_prefill_path.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp]
        lib.la_prefill_path.restype = ctypes.c_char_p
        lib.la_prefill_kernel.argtypes = [i32, i64, i32, i32, i32, vp, vp, vp, vp, vp]
        lib.la_prefill_kernel.restype = ctypes.c_char_p
        lib.la_resolve_chunk.argtypes = [i32, i32, i32, i32]
        lib.la_status_string.argtypes = [i32]
        lib.la_status_string.restype = ctypes.c_char_p
        lib.la_last_cuda_error.restype = ctypes.c_char_p
        for name in ("la_state_init", "la_prefill", "la_decode_step", "la_device_status",
                     "la_resolve_chunk"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def la_status_string(status: int) -> str:
    return load_library().la_status_string(int(status)).decode()


def last_cuda_error() -> str:
    return load_library().la_last_cuda_error().decode()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr() if t.numel() else None


def _check(status: int, where: str) -> None:
    if status != LA_OK:
        raise LinAttnError(status, where)


def la_state_init(state: torch.Tensor, src: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    """state [..., d_k, d_v] float32 <- src (or zero)."""
    if state.dim() < 2:
        raise ValueError("state must be [..., d_k, d_v]")
    dk, dv = state.shape[-2], state.shape[-1]
    n = state.numel() // max(1, dk * dv)
    if src is not None and src.shape != state.shape:
        raise ValueError("src must have the shape of state")
    _check(load_library().la_state_init(
        _ptr(state, "state", torch.float32), _ptr(src, "src", torch.float32),
        n, dk, dv, _stream(stream)), "la_state_init")


def la_prefill_workspace_size(dtype: torch.dtype, B: int, H: int, T: int, dk: int,
                              dv: int, num_seqs: int = 0, chunk: int = 0) -> int:
    return int(load_library().la_prefill_workspace_size(
        _DTYPES[dtype], B, H, T, dk, dv, num_seqs, chunk))


def la_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
               state: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
               max_seqlen: int = 0, chunk: int = 0,
               workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Chunkwise prefill.  q, k [B,H,T,d_k]; v, o [B,H,T,d_v]; state
    [B,H,d_k,d_v] (or [N,H,d_k,d_v] with cu_seqlens, B == 1)."""
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if q.dim() != 4:
        raise ValueError("q must be [B, H, T, d_k]")
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3] or o.shape != v.shape:
        raise ValueError("q/k/v/o shapes disagree")
    num_seqs = 0
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("cu_seqlens must be int32")
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must hold num_seqs + 1 >= 2 offsets")
        if B != 1:
            raise ValueError("packed input (cu_seqlens) needs B == 1")
        num_seqs = cu_seqlens.numel() - 1
    # the kernels read and write n_units * d_k * d_v floats of state: a smaller
    # buffer would be overrun, so its size is checked here, before any launch
    n_units = (num_seqs if cu_seqlens is not None else B) * H
    if state.numel() != n_units * dk * dv:
        raise ValueError(f"state must hold {n_units} x {dk} x {dv} floats "
                         f"({'num_seqs' if cu_seqlens is not None else 'B'} * H units), got {state.numel()}")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size()
    _check(load_library().la_prefill(
        _ptr(q, "q", q.dtype), _ptr(k, "k", q.dtype), _ptr(v, "v", q.dtype),
        _ptr(o, "o", q.dtype), _ptr(state, "state", torch.float32), _DTYPES[q.dtype],
        B, H, T, dk, dv, _ptr(cu_seqlens, "cu_seqlens"), num_seqs, int(max_seqlen),
        int(chunk), ws_ptr, ws_bytes, _stream(stream)), "la_prefill")


def la_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                   state: torch.Tensor, stream=None) -> None:
    """One decode token per unit.  q, k [B,H,d_k]; v, o [B,H,d_v]; state
    [B,H,d_k,d_v] updated in place."""
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if q.dim() != 3:
        raise ValueError("q must be [B, H, d_k]")
    B, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2] or o.shape != v.shape:
        raise ValueError("q/k/v/o shapes disagree")
    if state.numel() != B * H * dk * dv:
        raise ValueError(f"state must hold {B * H} x {dk} x {dv} floats, got {state.numel()}")
    _check(load_library().la_decode_step(
        _ptr(q, "q", q.dtype), _ptr(k, "k", q.dtype), _ptr(v, "v", q.dtype),
        _ptr(o, "o", q.dtype), _ptr(state, "state", torch.float32), _DTYPES[q.dtype],
        B, H, dk, dv, _stream(stream)), "la_decode_step")


def la_device_status(stream=None) -> int:
    """Synchronise the stream; return the device status code (LA_OK if clean)."""
    return int(load_library().la_device_status(_stream(stream)))


def la_selftest_wait_timeout(timeout_ms: float = 50.0, stream=None) -> None:
    """Launch the bounded-wait diagnostic (see include/linattn.h)."""
    _check(load_library().la_selftest_wait_timeout(float(timeout_ms), _stream(stream)),
           "la_selftest_wait_timeout")


def la_prefill_path(dtype: torch.dtype, dk: int, dv: int, chunk: int = 0,
                    q=None, k=None, v=None, o=None) -> str:
    p = [None if t is None else t.data_ptr() for t in (q, k, v, o)]
    if all(x is None for x in p):
        p = [256] * 4  # aligned placeholders: ask about the shape only
    return load_library().la_prefill_path(_DTYPES[dtype], dk, dv, chunk, *p).decode()


def la_prefill_kernel(dtype: torch.dtype, max_tokens: int, dk: int, dv: int, chunk: int = 0,
                      q=None, k=None, v=None, o=None, state=None) -> str:
    """Which kernel la_prefill runs: "short", "tc", "simt" or "unsupported".
    max_tokens: T (dense) or max_seqlen (packed)."""
    p = [None if t is None else t.data_ptr() for t in (q, k, v, o, state)]
    if all(x is None for x in p):
        p = [256] * 5  # aligned placeholders: ask about the shape only
    return load_library().la_prefill_kernel(_DTYPES[dtype], int(max_tokens), dk, dv, chunk, *p).decode()


def la_resolve_chunk(dtype: torch.dtype, dk: int, dv: int, chunk: int = 0) -> int:
    return int(load_library().la_resolve_chunk(_DTYPES[dtype], dk, dv, chunk))
