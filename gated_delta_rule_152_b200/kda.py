"""Python binding of ``libkda.so`` (the C ABI in ``include/kda.h``).

Argument marshalling only: these functions check shapes and dtypes of torch
tensors, allocate outputs and workspace with torch if the caller did not pass
them, and call the C entry points of the same names on the current CUDA
stream.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback -- if the library is missing or the
device is not a B200 (sm_100) the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = -1
KDA_ERR_UNSUPPORTED = -2
KDA_ERR_MISALIGNED = -3
KDA_ERR_WORKSPACE = -4
KDA_ERR_CUDA = -5
KDA_DTYPE_BF16 = 0
KDA_DTYPE_FP32 = 1
KDA_FLAG_L2NORM_QK = 1
KDA_FLAG_RECURRENT = 2
KDA_FLAG_SCALAR_DECAY = 4
KDA_DEVERR_CU_SEQLENS = 1
KDA_DEVERR_TIMEOUT = 2
KDA_DEVERR_SLOT = 4

EXPORTED = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd_workspace_size_min", "kda_chunk_fwd",
            "kda_chunk_fwd_noalloc", "kda_decode_step",
            "kda_chunk_fwd_slots", "kda_decode_step_slots", "kda_verify_fwd", "kda_workspace_error",
            "kda_selftest_bounded_waits", "kda_topk_workspace_size", "kda_topk_indices",
            "kda_status_string")
KDA_TOPK_MAX_K = 4096

_lock = threading.Lock()
_lib = None


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {status} ({kda_status_string(status)})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkda.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library {path} is missing; build it with "
                               "`python -m gated_delta_rule_152_b200.build`")
        lib = ctypes.CDLL(path)
        P, I32, I64, U32, F32, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                     ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t)
        lib.kda_chunk_fwd_workspace_size.argtypes = [I32, I64, I32, I32, ctypes.c_int]
        lib.kda_chunk_fwd_workspace_size.restype = SZ
        lib.kda_chunk_fwd_workspace_size_min.argtypes = [I32, I64, I32, I32, ctypes.c_int]
        lib.kda_chunk_fwd_workspace_size_min.restype = SZ
        lib.kda_chunk_fwd.argtypes = [P, P, P, P, P, P, I32, I64, I32, I32, ctypes.c_int, F32, U32,
                                      P, P, P, P, SZ, P]
        lib.kda_chunk_fwd.restype = ctypes.c_int
        lib.kda_chunk_fwd_noalloc.argtypes = [P, P, P, P, P, P, I32, I64, I32, I32, ctypes.c_int, F32, U32,
                                              P, P, P, P]
        lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
        lib.kda_decode_step.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, ctypes.c_int, F32, U32, P]
        lib.kda_decode_step.restype = ctypes.c_int
        lib.kda_chunk_fwd_slots.argtypes = [P, P, P, P, P, P, I32, I64, I32, I32, ctypes.c_int, F32, U32,
                                            P, P, I32, P, P, SZ, P]
        lib.kda_chunk_fwd_slots.restype = ctypes.c_int
        lib.kda_decode_step_slots.argtypes = [P, P, P, P, P, P, P, I32, P, I32, I32, I32, ctypes.c_int, F32,
                                              U32, P]
        lib.kda_decode_step_slots.restype = ctypes.c_int
        lib.kda_verify_fwd.argtypes = [P, P, P, P, P, P, I32, I64, I32, I32, ctypes.c_int, F32, U32,
                                       P, P, P, P, SZ, P]
        lib.kda_verify_fwd.restype = ctypes.c_int
        lib.kda_workspace_error.argtypes = [P, ctypes.POINTER(U32), P]
        lib.kda_workspace_error.restype = ctypes.c_int
        lib.kda_selftest_bounded_waits.argtypes = [P, SZ, U32, P]
        lib.kda_selftest_bounded_waits.restype = ctypes.c_int
        lib.kda_topk_workspace_size.argtypes = [I32, I64, I32]
        lib.kda_topk_workspace_size.restype = SZ
        lib.kda_topk_indices.argtypes = [P, I64, I32, I64, I32, P, P, P, P, SZ, P]
        lib.kda_topk_indices.restype = ctypes.c_int
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_status_string.restype = ctypes.c_char_p
        _lib = lib
        return lib


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_FP32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t: torch.Tensor, name: str, shape, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def kda_chunk_fwd_workspace_size(N: int, total_T: int, H: int, d: int = 128,
                                 dtype: torch.dtype = torch.bfloat16) -> int:
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_FP32
    return int(load_library().kda_chunk_fwd_workspace_size(N, total_T, H, d, code))


def kda_chunk_fwd_workspace_size_min(N: int, total_T: int, H: int, d: int = 128,
                                     dtype: torch.dtype = torch.bfloat16) -> int:
    code = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_FP32
    return int(load_library().kda_chunk_fwd_workspace_size_min(N, total_T, H, d, code))


def kda_chunk_fwd(q, k, v, g, beta, cu_seqlens, *, scale: float = 1.0, l2norm: bool = True,
                  initial_state: Optional[torch.Tensor] = None, final_state=True,
                  o: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  recurrent: bool = False, scalar_decay: bool = False,
                  stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Prefill over packed sequences.

    q, k, v: [total_T, H, 128] bf16 or fp32 (same dtype); g: [total_T, H, 128]
    fp32 log-decay ([total_T, H] with ``scalar_decay``, the Gated-DeltaNet
    form); beta: [total_T, H] fp32; cu_seqlens: [N + 1] int32 on the
    device.  ``final_state`` may be True (allocate), False/None (skip) or a
    [N, H, 128, 128] fp32 tensor (may be ``initial_state`` for an in-place
    continuation).  Returns ``(o, final_state)`` with o fp32 [total_T, H, 128].
    """
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_chunk_fwd needs CUDA tensors")
    T, H, d = q.shape
    dt = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, (T, H, d), q.dtype, dev)
    _check(g, "g", (T, H) if scalar_decay else (T, H, d), torch.float32, dev)
    _check(beta, "beta", (T, H), torch.float32, dev)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.device != dev:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
    N = cu_seqlens.numel() - 1
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, H, d, d), torch.float32, dev)
    if final_state is True:
        final_state = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    elif final_state is False:
        final_state = None
    elif final_state is not None:
        _check(final_state, "final_state", (N, H, d, d), torch.float32, dev)
    if o is None:
        o = torch.empty((T, H, d), dtype=torch.float32, device=dev)
    _check(o, "o", (T, H, d), torch.float32, dev)
    if workspace is None:
        # the fp32 / recurrent path uses only the error word; bf16 gets the
        # scratch of the two-pass tensor-core path
        size_fn = (lib.kda_chunk_fwd_workspace_size_min if recurrent or dt == KDA_DTYPE_FP32
                   else lib.kda_chunk_fwd_workspace_size)
        workspace = torch.empty(max(int(size_fn(N, T, H, d, dt)), 256), dtype=torch.uint8, device=dev)
    flags = ((KDA_FLAG_L2NORM_QK if l2norm else 0) | (KDA_FLAG_RECURRENT if recurrent else 0) |
             (KDA_FLAG_SCALAR_DECAY if scalar_decay else 0))
    st = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T, H,
                           d, dt, float(scale), flags, _ptr(initial_state), _ptr(final_state), _ptr(o),
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd")
    return o, final_state


def kda_chunk_fwd_noalloc(q, k, v, g, beta, cu_seqlens, *, scale: float = 1.0, l2norm: bool = True,
                          initial_state: Optional[torch.Tensor] = None, final_state=True,
                          o: Optional[torch.Tensor] = None, recurrent: bool = False,
                          scalar_decay: bool = False, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """kda_chunk_fwd on the library's built-in scratch instead of a workspace
    (see the header: at most KDA_NOALLOC_MAX_SEQS sequences, calls on one
    stream, the first call before any stream capture).  The outputs are
    allocated here if not given; the library call itself allocates nothing.
    Same arguments and results as kda_chunk_fwd."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_chunk_fwd_noalloc needs CUDA tensors")
    T, H, d = q.shape
    dt = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, (T, H, d), q.dtype, dev)
    _check(g, "g", (T, H) if scalar_decay else (T, H, d), torch.float32, dev)
    _check(beta, "beta", (T, H), torch.float32, dev)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.device != dev:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
    N = cu_seqlens.numel() - 1
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, H, d, d), torch.float32, dev)
    if final_state is True:
        final_state = torch.empty((N, H, d, d), dtype=torch.float32, device=dev)
    elif final_state is False:
        final_state = None
    elif final_state is not None:
        _check(final_state, "final_state", (N, H, d, d), torch.float32, dev)
    if o is None:
        o = torch.empty((T, H, d), dtype=torch.float32, device=dev)
    _check(o, "o", (T, H, d), torch.float32, dev)
    flags = ((KDA_FLAG_L2NORM_QK if l2norm else 0) | (KDA_FLAG_RECURRENT if recurrent else 0) |
             (KDA_FLAG_SCALAR_DECAY if scalar_decay else 0))
    st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T, H,
                                   d, dt, float(scale), flags, _ptr(initial_state), _ptr(final_state), _ptr(o),
                                   _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_noalloc")
    return o, final_state


def kda_decode_step(q, k, v, g, beta, state, *, scale: float = 1.0, l2norm: bool = True,
                    o: Optional[torch.Tensor] = None, scalar_decay: bool = False,
                    stream=None) -> torch.Tensor:
    """One decode token per sequence; ``state`` [N, H, 128, 128] fp32 is
    updated in place.  g is [N, H, 128] ([N, H] with ``scalar_decay``).
    Returns o [N, H, 128] fp32."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_decode_step needs CUDA tensors")
    N, H, d = q.shape
    dt = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, (N, H, d), q.dtype, dev)
    _check(g, "g", (N, H) if scalar_decay else (N, H, d), torch.float32, dev)
    _check(beta, "beta", (N, H), torch.float32, dev)
    _check(state, "state", (N, H, d, d), torch.float32, dev)
    if o is None:
        o = torch.empty((N, H, d), dtype=torch.float32, device=dev)
    _check(o, "o", (N, H, d), torch.float32, dev)
    flags = (KDA_FLAG_L2NORM_QK if l2norm else 0) | (KDA_FLAG_SCALAR_DECAY if scalar_decay else 0)
    st = lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(o), N,
                             H, d, dt, float(scale), flags, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step")
    return o


def kda_chunk_fwd_slots(q, k, v, g, beta, cu_seqlens, state_pool, slots, *, scale: float = 1.0,
                        l2norm: bool = True, o: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, recurrent: bool = False,
                        scalar_decay: bool = False, stream=None) -> torch.Tensor:
    """Prefill whose sequences keep their states in a pool: sequence n starts
    from ``state_pool[slots[n]]`` ([num_slots, H, 128, 128] fp32) and its final
    state is written back there.  ``slots``: [N] int32 on the device, distinct.
    Returns o [total_T, H, 128] fp32."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_chunk_fwd_slots needs CUDA tensors")
    T, H, d = q.shape
    dt = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, (T, H, d), q.dtype, dev)
    _check(g, "g", (T, H) if scalar_decay else (T, H, d), torch.float32, dev)
    _check(beta, "beta", (T, H), torch.float32, dev)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.device != dev:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
    N = cu_seqlens.numel() - 1
    _check(slots, "slots", (N,), torch.int32, dev)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (H, d, d):
        raise ValueError("state_pool must be [num_slots, H, 128, 128]")
    _check(state_pool, "state_pool", tuple(state_pool.shape), torch.float32, dev)
    if o is None:
        o = torch.empty((T, H, d), dtype=torch.float32, device=dev)
    _check(o, "o", (T, H, d), torch.float32, dev)
    if workspace is None:
        # the fp32 / recurrent path uses only the error word; bf16 gets the
        # scratch of the two-pass tensor-core path
        size_fn = (lib.kda_chunk_fwd_workspace_size_min if recurrent or dt == KDA_DTYPE_FP32
                   else lib.kda_chunk_fwd_workspace_size)
        workspace = torch.empty(max(int(size_fn(N, T, H, d, dt)), 256), dtype=torch.uint8, device=dev)
    flags = ((KDA_FLAG_L2NORM_QK if l2norm else 0) | (KDA_FLAG_RECURRENT if recurrent else 0) |
             (KDA_FLAG_SCALAR_DECAY if scalar_decay else 0))
    st = lib.kda_chunk_fwd_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T, H,
                                 d, dt, float(scale), flags, _ptr(state_pool), _ptr(slots),
                                 int(state_pool.shape[0]), _ptr(o), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_slots")
    return o


def kda_decode_step_slots(q, k, v, g, beta, state_pool, slots, *, scale: float = 1.0,
                          l2norm: bool = True, o: Optional[torch.Tensor] = None,
                          scalar_decay: bool = False, stream=None) -> torch.Tensor:
    """Decode step whose states live in a pool: sequence n updates
    ``state_pool[slots[n]]`` in place.  Returns o [N, H, 128] fp32."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_decode_step_slots needs CUDA tensors")
    N, H, d = q.shape
    dt = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, (N, H, d), q.dtype, dev)
    _check(g, "g", (N, H) if scalar_decay else (N, H, d), torch.float32, dev)
    _check(beta, "beta", (N, H), torch.float32, dev)
    _check(slots, "slots", (N,), torch.int32, dev)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (H, d, d):
        raise ValueError("state_pool must be [num_slots, H, 128, 128]")
    _check(state_pool, "state_pool", tuple(state_pool.shape), torch.float32, dev)
    if o is None:
        o = torch.empty((N, H, d), dtype=torch.float32, device=dev)
    _check(o, "o", (N, H, d), torch.float32, dev)
    flags = (KDA_FLAG_L2NORM_QK if l2norm else 0) | (KDA_FLAG_SCALAR_DECAY if scalar_decay else 0)
    st = lib.kda_decode_step_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                                   _ptr(slots), int(state_pool.shape[0]), _ptr(o), N, H, d, dt,
                                   float(scale), flags, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step_slots")
    return o


def kda_verify_fwd(q, k, v, g, beta, cu_seqlens, *, initial_state: Optional[torch.Tensor] = None,
                   snapshots: Optional[torch.Tensor] = None, scale: float = 1.0, l2norm: bool = True,
                   o: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   scalar_decay: bool = False, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Multi-token (speculative-verify) step: like kda_chunk_fwd, but returns
    the state after every token, ``snapshots`` [total_T, H, 128, 128] fp32,
    for rolling back to an accepted prefix.  Returns ``(o, snapshots)``."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_verify_fwd needs CUDA tensors")
    T, H, d = q.shape
    dt = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, name, (T, H, d), q.dtype, dev)
    _check(g, "g", (T, H) if scalar_decay else (T, H, d), torch.float32, dev)
    _check(beta, "beta", (T, H), torch.float32, dev)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.device != dev:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
    N = cu_seqlens.numel() - 1
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, H, d, d), torch.float32, dev)
    if snapshots is None:
        snapshots = torch.empty((T, H, d, d), dtype=torch.float32, device=dev)
    _check(snapshots, "snapshots", (T, H, d, d), torch.float32, dev)
    if o is None:
        o = torch.empty((T, H, d), dtype=torch.float32, device=dev)
    _check(o, "o", (T, H, d), torch.float32, dev)
    ws_bytes = int(lib.kda_chunk_fwd_workspace_size_min(N, T, H, d, dt))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    flags = (KDA_FLAG_L2NORM_QK if l2norm else 0) | (KDA_FLAG_SCALAR_DECAY if scalar_decay else 0)
    st = lib.kda_verify_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T, H, d,
                            dt, float(scale), flags, _ptr(initial_state), _ptr(snapshots), _ptr(o),
                            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_verify_fwd")
    return o, snapshots


def kda_selftest_bounded_waits(workspace: torch.Tensor, polls: int = 4096, stream=None) -> None:
    """Enqueue the self-test whose bounded waits must give up (see the header);
    read the outcome with kda_workspace_error(workspace)."""
    st = load_library().kda_selftest_bounded_waits(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                                   int(polls), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_selftest_bounded_waits")


def kda_workspace_error(workspace: torch.Tensor, stream=None) -> int:
    """Read the device error word of a prefill workspace (synchronises)."""
    out = ctypes.c_uint32(0)
    st = load_library().kda_workspace_error(_ptr(workspace), ctypes.byref(out), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_workspace_error")
    return int(out.value)


def kda_topk_workspace_size(rows: int, n: int, k: int = 2048) -> int:
    return int(load_library().kda_topk_workspace_size(rows, n, k))


def kda_topk_indices(scores, k: int = 2048, *, row_lengths: Optional[torch.Tensor] = None,
                     indices: Optional[torch.Tensor] = None, values=False,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """The lightning indexer's selection: per row of ``scores`` ([rows, n]
    fp32 CUDA tensor whose rows are contiguous, any row stride), the indices
    of the k highest scores, best first, ties to the lower index, -1 past the
    row's length.  ``row_lengths``: optional [rows] int32 tokens per row.
    Returns ``indices`` [rows, k] int32 (and the kept scores [rows, k] fp32 if
    ``values`` is True or a tensor)."""
    lib = load_library()
    if scores.device.type != "cuda" or scores.dtype != torch.float32 or scores.dim() != 2:
        raise ValueError("scores must be a 2-D float32 CUDA tensor")
    if scores.stride(1) != 1:
        raise ValueError("scores rows must be contiguous")
    rows, n = scores.shape
    ld = scores.stride(0) if rows > 1 else n
    dev = scores.device
    if row_lengths is not None:
        _check(row_lengths, "row_lengths", (rows,), torch.int32, dev)
    if indices is None:
        indices = torch.empty((rows, k), dtype=torch.int32, device=dev)
    _check(indices, "indices", (rows, k), torch.int32, dev)
    vals = None
    if values is True:
        vals = torch.empty((rows, k), dtype=torch.float32, device=dev)
    elif isinstance(values, torch.Tensor):
        vals = values
        _check(vals, "values", (rows, k), torch.float32, dev)
    need = int(lib.kda_topk_workspace_size(rows, n, k))
    if need == 0:
        raise ValueError("unsupported sizes for kda_topk_indices")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = lib.kda_topk_indices(_ptr(scores), ld, rows, n, k, _ptr(row_lengths), _ptr(indices), _ptr(vals),
                              _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_topk_indices")
    return (indices, vals) if vals is not None else indices
