"""kda_chunk_fwd_noalloc, the prefill entry point for callers that cannot
allocate device memory (it runs on a scratch array built into the library
instead of a caller-provided workspace).

Its results must match kda_chunk_fwd's on the same inputs, on two calls in a
row (the second call reuses the scratch the first one left behind).  This
file is collected last so that a run stopping at the first failure has
already run every other test; it passes alone in a fresh process too, where
its first call also does the one-time device set-up.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_152_b200 import inputs as kin
from gated_delta_rule_152_b200 import kda

TOL_BF16 = 2e-2
MAX_SEQS = 16320


def _entry():
    fn = kda.load_library().kda_chunk_fwd_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                   ctypes.c_int, ctypes.c_float, ctypes.c_uint32, P, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _ratio(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return float(np.abs(a - b).max() / np.sqrt(np.mean(b * b)))


def test_noalloc_rejects_too_many_sequences_without_launching():
    from gated_delta_rule_152_b200 import build
    build.build()
    fn = _entry()
    fake = ctypes.c_void_p(0x10000)
    st = fn(fake, fake, fake, fake, fake, fake, MAX_SEQS + 1, 1000, 4, 128, 0, 1.0, 1, None, None,
            fake, None)
    assert st == kda.KDA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    fn = _entry()
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    for seed, lengths in ((31, [100, 0, 257]), (32, [64, 1, 300, 90])):
        x = kin.make_custom_prefill(seed, lengths, heads=3, init_state_std=0.02).to(dev)
        T, H, d = x.q.shape
        N = len(lengths)
        # the allocation-free entry point has only a small fixed scratch, so it
        # runs the fused kernel; give kda_chunk_fwd the minimum workspace too
        ws = torch.zeros(kda.kda_chunk_fwd_workspace_size_min(N, T, H), dtype=torch.uint8, device=dev)
        o_ref, s_ref = kda.kda_chunk_fwd(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens,
                                         initial_state=x.initial_state, workspace=ws)
        o = torch.full_like(o_ref, float("nan"))
        s = torch.full_like(s_ref, float("nan"))
        st = fn(_p(x.q), _p(x.k), _p(x.v), _p(x.g), _p(x.beta), _p(x.cu_seqlens), N, T, H, d,
                kda.KDA_DTYPE_BF16, 1.0, kda.KDA_FLAG_L2NORM_QK, _p(x.initial_state), _p(s), _p(o),
                ctypes.c_void_p(stream.cuda_stream))
        assert st == kda.KDA_OK, kda.kda_status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(o).all() and torch.isfinite(s).all()
        assert _ratio(o, o_ref) <= TOL_BF16
        assert _ratio(s, s_ref) <= TOL_BF16


@pytest.mark.gpu
def test_noalloc_python_binding_matches_the_raw_entry_point():
    # the Python function of the same name, after the raw entry point above
    # has done the one-time device set-up: the same bits on the same inputs
    dev = torch.device("cuda")
    x = kin.make_custom_prefill(33, [200, 7, 64], heads=2, init_state_std=0.02).to(dev)
    T, H, d = x.q.shape
    N = x.cu_seqlens.numel() - 1
    o, s = kda.kda_chunk_fwd_noalloc(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, initial_state=x.initial_state)
    o2 = torch.full_like(o, float("nan"))
    s2 = torch.full_like(s, float("nan"))
    st = _entry()(_p(x.q), _p(x.k), _p(x.v), _p(x.g), _p(x.beta), _p(x.cu_seqlens), N, T, H, d,
                  kda.KDA_DTYPE_BF16, 1.0, kda.KDA_FLAG_L2NORM_QK, _p(x.initial_state), _p(s2), _p(o2),
                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kda.KDA_OK
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(s, s2)
