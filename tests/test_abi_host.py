"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/kda.h, and rejects bad arguments on the host before any
CUDA call (fake, never-dereferenced pointers are enough for that)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_152_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

A = 0x10000          # a fake 16-byte-aligned device address
MIS = 0x10008        # misaligned


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_152_b200 import build
    build.build()
    return kda.load_library()


def test_library_exports_every_declared_function(lib):
    names = header_functions()
    assert set(names) >= {"kda_chunk_fwd", "kda_decode_step", "kda_chunk_fwd_workspace_size",
                          "kda_status_string", "kda_workspace_error"}
    for name in names:
        assert hasattr(lib, name), name
    assert set(kda.EXPORTED) <= set(names)


def test_status_strings(lib):
    assert kda.kda_status_string(0) == "ok"
    for s in range(-5, 0):
        assert kda.kda_status_string(s) not in ("ok", "unknown status")
    assert kda.kda_status_string(-99) == "unknown status"


def test_workspace_size(lib):
    assert lib.kda_chunk_fwd_workspace_size(16, 1000, 32, 128, 0) >= 256 + 64
    assert lib.kda_chunk_fwd_workspace_size(16, 1000, 32, 64, 0) == 0
    assert lib.kda_chunk_fwd_workspace_size(-1, 1000, 32, 128, 0) == 0


def test_workspace_size_ring_and_per_pair_scratch(lib):
    slot = 145 * 1024   # operands of one (64-token chunk, head) pair
    one = lib.kda_chunk_fwd_workspace_size(1, 8192, 32, 128, 0)
    assert 32 * 8 * slot <= one < 64 << 20           # one sequence: a ring of 8 slots per head
    assert lib.kda_chunk_fwd_workspace_size(1, 131072, 32, 128, 0) == one   # independent of length
    # several sequences share each head's ring: the size hardly depends on their number
    # or lengths (16 sequences of up to 16K tokens: under 40 MB, not 9.5 GB)
    two = lib.kda_chunk_fwd_workspace_size(2, 8192, 32, 128, 0)
    sixteen = lib.kda_chunk_fwd_workspace_size(16, 135168, 32, 128, 0)
    assert one <= two <= sixteen < 40 << 20
    many_heads = lib.kda_chunk_fwd_workspace_size(1, 8192, 100, 128, 0)
    assert many_heads >= 128 * 100 * slot            # too many heads for the ring: a slot per pair
    assert lib.kda_chunk_fwd_workspace_size(2, 8192, 100, 128, 0) >= (128 + 1) * 100 * slot
    assert lib.kda_chunk_fwd_workspace_size_min(1, 8192, 32, 128, 0) < 4096


def _chunk(lib, **kw):
    args = dict(q=A, k=A, v=A, g=A, beta=A, cu=A, N=2, T=100, H=4, d=128, dt=0, scale=1.0, flags=1,
                s0=None, sT=None, o=A, ws=A, wsb=4096, stream=None)
    args.update(kw)
    return lib.kda_chunk_fwd(args["q"], args["k"], args["v"], args["g"], args["beta"], args["cu"],
                             args["N"], args["T"], args["H"], args["d"], args["dt"], args["scale"],
                             args["flags"], args["s0"], args["sT"], args["o"], args["ws"], args["wsb"],
                             args["stream"])


def test_chunk_fwd_host_validation(lib):
    assert _chunk(lib, d=64) == kda.KDA_ERR_UNSUPPORTED
    assert _chunk(lib, dt=7) == kda.KDA_ERR_UNSUPPORTED
    assert _chunk(lib, flags=0x80) == kda.KDA_ERR_UNSUPPORTED
    # every documented flag passes validation (then fails later only for lack of a GPU)
    assert _chunk(lib, flags=1 | 2 | 4) == _chunk(lib, flags=1)
    assert _chunk(lib, N=-1) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, H=0) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, T=1 << 31) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, cu=None) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, o=None) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, g=MIS) == kda.KDA_ERR_MISALIGNED
    assert _chunk(lib, s0=MIS) == kda.KDA_ERR_MISALIGNED
    assert _chunk(lib, ws=None) == kda.KDA_ERR_WORKSPACE
    assert _chunk(lib, wsb=16) == kda.KDA_ERR_WORKSPACE


def test_decode_host_validation(lib):
    def dec(**kw):
        a = dict(q=A, k=A, v=A, g=A, beta=A, s=A, o=A, N=4, H=2, d=128, dt=0, scale=1.0, flags=1)
        a.update(kw)
        return lib.kda_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["s"], a["o"], a["N"],
                                   a["H"], a["d"], a["dt"], a["scale"], a["flags"], None)
    assert dec(d=100) == kda.KDA_ERR_UNSUPPORTED
    assert dec(flags=2) == kda.KDA_ERR_UNSUPPORTED   # the recurrent flag is prefill-only
    assert dec(N=-3) == kda.KDA_ERR_INVALID_ARG
    assert dec(s=None) == kda.KDA_ERR_INVALID_ARG
    assert dec(o=MIS) == kda.KDA_ERR_MISALIGNED
    assert dec(N=0) == kda.KDA_OK                    # nothing to do, nothing launched


def test_slot_forms_reject_missing_pool_or_slots(lib):
    P = ctypes.c_void_p
    lib.kda_chunk_fwd_slots.argtypes = [P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int, ctypes.c_float, ctypes.c_uint32, P, P,
                                        ctypes.c_int32, P, P, ctypes.c_size_t, P]
    args = [A, A, A, A, A, A, 2, 100, 4, 128, 0, 1.0, 1]
    assert lib.kda_chunk_fwd_slots(*args, None, A, 8, A, A, 4096, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_slots(*args, A, None, 8, A, A, 4096, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_slots(*args, A, A, 0, A, A, 4096, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_slots(*args, MIS, A, 8, A, A, 4096, None) == kda.KDA_ERR_MISALIGNED


def test_valid_call_without_gpu_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    assert _chunk(lib) in (kda.KDA_ERR_CUDA, kda.KDA_ERR_UNSUPPORTED)


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 2, 128)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(x, x, x, x, torch.zeros(4, 2), torch.tensor([0, 4], dtype=torch.int32))


def test_noalloc_binding_rejects_cpu_tensors_and_bad_shapes():
    import torch
    x = torch.zeros(4, 2, 128)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd_noalloc(x, x, x, x, torch.zeros(4, 2), cu)


def test_selftest_rejects_bad_workspace(lib):
    P = ctypes.c_void_p
    assert lib.kda_selftest_bounded_waits(None, 256, 16, None) == kda.KDA_ERR_WORKSPACE
    assert lib.kda_selftest_bounded_waits(P(A), 64, 16, None) == kda.KDA_ERR_WORKSPACE
    assert lib.kda_selftest_bounded_waits(P(MIS), 256, 16, None) == kda.KDA_ERR_MISALIGNED


def test_topk_host_validation(lib):
    P = ctypes.c_void_p
    ws = kda.kda_topk_workspace_size(4, 1000, 2048)
    assert ws > 0 and kda.kda_topk_workspace_size(4, 1000, kda.KDA_TOPK_MAX_K + 1) == 0
    assert kda.kda_topk_workspace_size(4, 1000, 0) == 0
    # grows with rows and k
    assert kda.kda_topk_workspace_size(8, 1000, 2048) > ws > kda.kda_topk_workspace_size(4, 1000, 64)
    W = 0x100000          # fake 256-byte-aligned workspace
    call = lambda scores, ld, rows, n, k, idx, ws_ptr=W, ws_bytes=ws, lengths=None, vals=None: \
        lib.kda_topk_indices(P(scores) if scores else None, ld, rows, n, k, P(lengths) if lengths else None,
                             P(idx) if idx else None, P(vals) if vals else None, P(ws_ptr) if ws_ptr else None,
                             ws_bytes, None)
    assert call(A, 1000, 4, 1000, 0, A) == kda.KDA_ERR_UNSUPPORTED              # k = 0
    assert call(A, 1000, 4, 1000, 4097, A) == kda.KDA_ERR_UNSUPPORTED           # k above the maximum
    assert call(A, 996, 4, 1000, 16, A) == kda.KDA_ERR_INVALID_ARG              # ld < n
    assert call(A, 1000, 70000, 1000, 16, A) == kda.KDA_ERR_INVALID_ARG         # too many rows
    assert call(A, 1000, 4, 1000, 16, None) == kda.KDA_ERR_INVALID_ARG          # no output
    assert call(A + 2, 1000, 4, 1000, 16, A) == kda.KDA_ERR_MISALIGNED          # scores not 4-byte aligned
    assert call(A, 1000, 4, 1000, 16, A + 1) == kda.KDA_ERR_MISALIGNED          # indices not 4-byte aligned
    assert call(A, 1000, 4, 1000, 16, A, ws_ptr=None) == kda.KDA_ERR_WORKSPACE
    assert call(A, 1000, 4, 1000, 16, A, ws_ptr=W + 16) == kda.KDA_ERR_WORKSPACE   # not 256-byte aligned
    assert call(A, 1000, 4, 1000, 2048, A, ws_bytes=ws - 1) == kda.KDA_ERR_WORKSPACE
    assert call(A, 1000, 0, 1000, 16, None) == kda.KDA_OK                       # nothing to do
