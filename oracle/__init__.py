"""fp64 CPU oracle for the KDA layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library's product path
(``gated_delta_rule_152_b200``) never imports it and shares no code with it;
the only common dependency is the seeded input generator module, which holds
none of the layer's arithmetic.

* :func:`kda_forward` / :func:`kda_decode` wrap the plain C recurrence in
  ``kda_oracle.c`` (fp64, token by token, OpenMP over independent
  (sequence, head) pairs).  Source: page "GLM-5.3-FLASH" (dimsnsums.com),
  section "How can a layer remember without rereading?", the update rule
  S_t = (I - beta k k^T) Diag(alpha_t) S_{t-1} + beta k v^T; readout
  o_t = scale * S_t^T q_t.
* :mod:`oracle.bruteforce` is an independent numpy formulation with explicit
  d x d matrices, used only to pin the C code on tiny inputs.

Inputs may be torch tensors (any dtype, any device) or numpy arrays; they are
converted exactly to fp64 on the host.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` next to it (gcc, fp64,
    no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", "-std=c99",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.kda_oracle_forward.argtypes = [I64, I64, I64, P, P, P, P, P, P, P, P, P,
                                               ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                               ctypes.c_int]
            lib.kda_oracle_forward.restype = ctypes.c_int
            lib.kda_oracle_decode.argtypes = [I64, I64, I64, P, P, P, P, P, P, P,
                                              ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                              ctypes.c_int]
            lib.kda_oracle_decode.restype = ctypes.c_int
            lib.kda_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def to_f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor (bf16/fp32/...) or array to fp64."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def kda_forward(q, k, v, g, beta, cu_seqlens, initial_state=None, scale: float = 1.0,
                l2norm: bool = True, eps: float = EPS, threads: int = 0):
    """Prefill over packed sequences.  Returns ``(o, final_state)`` in fp64,
    shapes ``[total_T, H, d]`` and ``[N, H, d, d]``."""
    lib = _load()
    q, k, v, g, beta = (to_f64(t) for t in (q, k, v, g, beta))
    cu = np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    T, H, d = q.shape
    N = cu.size - 1
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal total_T")
    s0 = to_f64(initial_state)
    if s0 is not None and s0.shape != (N, H, d, d):
        raise ValueError("initial_state shape mismatch")
    o = np.zeros((T, H, d), dtype=np.float64)
    sT = np.zeros((N, H, d, d), dtype=np.float64)
    rc = lib.kda_oracle_forward(N, H, d, _ptr(cu), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                _ptr(beta), _ptr(s0), _ptr(sT), _ptr(o), float(scale),
                                int(bool(l2norm)), float(eps), int(threads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_forward failed ({rc})")
    return o, sT


def kda_decode(q, k, v, g, beta, state, scale: float = 1.0, l2norm: bool = True,
               eps: float = EPS, threads: int = 0):
    """One decode step.  Returns ``(o, new_state)`` in fp64 (``state`` is not
    modified)."""
    lib = _load()
    q, k, v, g, beta = (to_f64(t) for t in (q, k, v, g, beta))
    S = to_f64(state).copy()
    N, H, d = q.shape
    if S.shape != (N, H, d, d):
        raise ValueError("state shape mismatch")
    o = np.zeros((N, H, d), dtype=np.float64)
    rc = lib.kda_oracle_decode(N, H, d, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                               _ptr(S), _ptr(o), float(scale), int(bool(l2norm)), float(eps),
                               int(threads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_decode failed ({rc})")
    return o, S
