"""GPU parity: the CUDA library against the fp64 oracle, element by element.

Bar (both o and the final state, separately): max|gpu - oracle| <= tol x
RMS(oracle), tol = 1e-4 for fp32 q/k/v and 2e-2 for bf16 q/k/v.  Small cases
span several 64-token chunks and ragged tails; the five named workloads run at
full size on the GPU and are compared on every output the oracle can afford
(all of them, or a subset of heads for the two 130K-token workloads).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_152_b200 import inputs as kin
from gated_delta_rule_152_b200 import kda

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16 = 2e-2


def err_ratio(gpu: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu.detach().double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.abs(g - ref).max()) / max(rms, 1e-300)


def assert_close(gpu, ref, tol, what):
    r = err_ratio(gpu, ref)
    log = os.environ.get("KDA_PARITY_LOG")
    if log:   # optional record of the measured ratios
        with open(log, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
                                "what": what, "max_err_over_rms": r, "tol": tol}) + "\n")
    assert np.isfinite(gpu.detach().cpu().numpy()).all(), f"{what}: non-finite output"
    assert r <= tol, f"{what}: max|err| = {r:.3e} x RMS(ref) > {tol:g}"
    return r


# The bf16 prefill has two tensor-core paths: the two-pass one (prep pass over
# all chunks and the sequential state pass; for a single sequence both run
# overlapped in one launch through a ring of operand slots) runs when the
# workspace holds its scratch -- the binding's default -- and the fused single
# kernel runs with the minimum workspace.
PATHS = ["two_pass", "fused"]


def small_workspace(x: kin.PrefillInputs, dev):
    T, H, _ = x.q.shape
    N = x.cu_seqlens.numel() - 1
    return torch.zeros(kda.kda_chunk_fwd_workspace_size_min(N, T, H), dtype=torch.uint8, device=dev)


def run_both(x: kin.PrefillInputs, recurrent=False, scale=1.0, l2norm=True, heads=None, path="two_pass"):
    dev = torch.device("cuda")
    xd = x.to(dev)
    T, H, _ = x.q.shape
    N = x.cu_seqlens.numel() - 1
    if path == "fused":
        ws = small_workspace(x, dev)
    else:
        ws = torch.zeros(max(kda.kda_chunk_fwd_workspace_size(N, T, H, dtype=x.q.dtype), 256), dtype=torch.uint8,
                         device=dev)
    o, sT = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, scale=scale,
                              l2norm=l2norm, initial_state=xd.initial_state, recurrent=recurrent,
                              workspace=ws)
    torch.cuda.synchronize()
    assert kda.kda_workspace_error(ws) == 0, "a kernel reported an error"
    sel = slice(None) if heads is None else list(heads)
    s0 = None if x.initial_state is None else x.initial_state[:, sel].contiguous()
    o_ref, s_ref = oracle.kda_forward(x.q[:, sel].contiguous(), x.k[:, sel].contiguous(),
                                      x.v[:, sel].contiguous(), x.g[:, sel].contiguous(),
                                      x.beta[:, sel].contiguous(), x.cu_seqlens, s0, scale=scale,
                                      l2norm=l2norm)
    return o[:, sel], sT[:, sel], o_ref, s_ref


def test_tiny_fp32_workload_full():
    x = kin.make_prefill(kin.TINY_FP32)
    o, s, o_ref, s_ref = run_both(x)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(s, s_ref, TOL_FP32, "final state")


@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [200], [0, 5, 64, 130, 1, 257]])
def test_recurrent_kernel_bf16(lengths):
    x = kin.make_custom_prefill(11, lengths, heads=3, init_state_std=0.02)
    o, s, o_ref, s_ref = run_both(x, recurrent=True, scale=0.75)
    assert_close(o, o_ref, TOL_FP32 if sum(lengths) else TOL_FP32, "o")   # fp32 arithmetic throughout
    assert_close(s, s_ref, TOL_FP32, "final state")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("lengths", [[1], [63], [64], [65], [200], [1000]])
def test_chunk_kernel_single_sequence(lengths, path):
    x = kin.make_custom_prefill(21, lengths, heads=2, init_state_std=0.02)
    o, s, o_ref, s_ref = run_both(x, path=path)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


@pytest.mark.parametrize("path", PATHS)
def test_chunk_kernel_varlen_with_empty_and_ragged(path):
    x = kin.make_custom_prefill(22, [0, 5, 64, 130, 1, 257, 0, 128], heads=3, init_state_std=0.05)
    o, s, o_ref, s_ref = run_both(x, scale=0.5, path=path)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")
    # empty sequences: final state equals the initial state exactly
    for n in (0, 6):
        assert torch.equal(s[n].cpu(), x.initial_state[n])


def test_chunk_kernel_without_l2norm():
    x = kin.make_custom_prefill(23, [150, 70], heads=2, init_state_std=0.02)
    # keep |k| near 1 so the un-normalised recurrence stays bounded
    x.q = (x.q.float() / 11.3).to(torch.bfloat16)
    x.k = (x.k.float() / 11.3).to(torch.bfloat16)
    o, s, o_ref, s_ref = run_both(x, l2norm=False)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


@pytest.mark.parametrize("path", PATHS)
def test_chunk_kernel_strong_decay(path):
    # per-chunk decay per channel around 40 nats (inside the tensor-core path's range)
    x = kin.make_custom_prefill(24, [300], heads=2, init_state_std=0.02)
    x.g = x.g * 8.0
    o, s, o_ref, s_ref = run_both(x, path=path)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


def test_chunk_kernel_in_place_state():
    x = kin.make_custom_prefill(25, [100, 33], heads=2, init_state_std=0.02)
    dev = torch.device("cuda")
    xd = x.to(dev)
    state = xd.initial_state.clone()
    o, s = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens,
                             initial_state=state, final_state=state)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
    assert s.data_ptr() == state.data_ptr()
    assert_close(state, s_ref, TOL_BF16, "in-place final state")
    assert_close(o, o_ref, TOL_BF16, "o")


def test_chunk_kernel_split_resume_matches_single_call():
    x = kin.make_custom_prefill(26, [400], heads=2, init_state_std=0.02)
    dev = torch.device("cuda")
    xd = x.to(dev)
    o_full, s_full = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens,
                                       initial_state=xd.initial_state)
    cut = 150
    cu1 = torch.tensor([0, cut], dtype=torch.int32, device=dev)
    cu2 = torch.tensor([0, 400 - cut], dtype=torch.int32, device=dev)
    o1, s1 = kda.kda_chunk_fwd(xd.q[:cut], xd.k[:cut], xd.v[:cut], xd.g[:cut], xd.beta[:cut], cu1,
                               initial_state=xd.initial_state)
    o2, s2 = kda.kda_chunk_fwd(xd.q[cut:].contiguous(), xd.k[cut:].contiguous(), xd.v[cut:].contiguous(),
                               xd.g[cut:].contiguous(), xd.beta[cut:].contiguous(), cu2, initial_state=s1)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
    assert_close(torch.cat([o1, o2]), o_ref, TOL_BF16, "split o")
    assert_close(s2, s_ref, TOL_BF16, "split final state")


def test_zero_tokens_copies_initial_state():
    dev = torch.device("cuda")
    H = 2
    s0 = torch.randn(3, H, 128, 128, device=dev)
    e = torch.empty(0, H, 128, device=dev, dtype=torch.bfloat16)
    cu = torch.zeros(4, dtype=torch.int32, device=dev)
    o, s = kda.kda_chunk_fwd(e, e, e, e.float(), torch.empty(0, H, device=dev), cu, initial_state=s0)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(s, s0)


@pytest.mark.parametrize("path", PATHS)
def test_bad_cu_seqlens_flags_error_and_skips_only_that_sequence(path):
    x = kin.make_custom_prefill(27, [40, 30, 50], heads=2)
    dev = torch.device("cuda")
    xd = x.to(dev)
    # sequence 2 runs backwards (120 -> 60): flagged and skipped; sequences 0
    # and 1 (tokens 0-39 and 40-119) are consistent and do not overlap it
    bad = torch.tensor([0, 40, 120, 60], dtype=torch.int32, device=dev)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(3, 120, 2) if path == "two_pass" else 1024,
                     dtype=torch.uint8, device=dev)
    s0 = torch.randn(3, 2, 128, 128, device=dev)
    sT = torch.full((3, 2, 128, 128), 7.0, device=dev)
    o, s = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, bad, initial_state=s0, final_state=sT,
                             workspace=ws)
    assert kda.kda_workspace_error(ws) & kda.KDA_DEVERR_CU_SEQLENS
    for lo, hi, n in ((0, 40, 0), (40, 120, 1)):
        sl = slice(lo, hi)
        o_ref, s_ref = oracle.kda_forward(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], [0, hi - lo],
                                          s0[n:n + 1].cpu())
        assert_close(o[sl], o_ref, TOL_BF16, f"o of valid sequence {n}")
        assert_close(s[n:n + 1], s_ref, TOL_BF16, f"final state of valid sequence {n}")
    assert torch.all(s[2] == 7.0)   # the skipped sequence's final state is left untouched
    ws.zero_()
    kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, workspace=ws)
    assert kda.kda_workspace_error(ws) == 0


def test_overlapping_sequences_cannot_overrun_the_two_pass_scratch():
    # cu_seqlens [0, 200, 0, 200, 0, 200]: sequences 0, 2 and 4 are each in
    # bounds but cover the same 200 tokens, 12 chunks in all, while the
    # scratch is sized for (200 + 63 * 5) / 64 = 8.  The chunks past the
    # scratch are not computed (sequence 4 is skipped) and the error bit is set.
    x = kin.make_custom_prefill(28, [200], heads=2, init_state_std=0.02)
    dev = torch.device("cuda")
    xd = x.to(dev)
    cu = torch.tensor([0, 200, 0, 200, 0, 200], dtype=torch.int32, device=dev)
    s0 = xd.initial_state.expand(5, -1, -1, -1).contiguous()   # same start, so overlaps agree
    sT = torch.full((5, 2, 128, 128), 7.0, device=dev)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(5, 200, 2), dtype=torch.uint8, device=dev)
    o, s = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, cu, initial_state=s0, final_state=sT,
                             workspace=ws)
    assert kda.kda_workspace_error(ws) & kda.KDA_DEVERR_CU_SEQLENS
    o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
    assert_close(o, o_ref, TOL_BF16, "o of the overlapping sequences")
    for n in (0, 2):
        assert_close(s[n:n + 1], s_ref, TOL_BF16, f"final state of sequence {n}")
    for n in (1, 3, 4):
        assert torch.all(s[n] == 7.0), f"sequence {n} must be skipped"


@pytest.mark.parametrize("path", PATHS)
def test_prefill_8k_workload_full(path):
    x = kin.make_prefill(kin.PREFILL_8K)
    o, s, o_ref, s_ref = run_both(x, path=path)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


def test_prefill_8k_recurrent_path_matches_oracle():
    x = kin.make_prefill(kin.PREFILL_8K, heads=4)
    o, s, o_ref, s_ref = run_both(x, recurrent=True)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(s, s_ref, TOL_FP32, "final state")


def test_prefill_128k_workload_sampled_heads():
    x = kin.make_prefill(kin.PREFILL_128K)
    o, s, o_ref, s_ref = run_both(x, heads=[0, 13, 31])
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


def test_varlen_16_workload_sampled_heads():
    x = kin.make_prefill(kin.VARLEN_16)
    o, s, o_ref, s_ref = run_both(x, heads=[0, 7, 31])
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_small(dtype):
    spec = kin.DecodeSpec("small", 77, 5, 1, 3, dtype)
    tok = kin.make_decode_tokens(spec, 0)
    st = kin.make_decode_state(spec, 0)
    dev = torch.device("cuda")
    td = tok.to(dev)
    sd = st.to(dev)
    o = kda.kda_decode_step(td.q, td.k, td.v, td.g, td.beta, sd, scale=0.9)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_decode(tok.q, tok.k, tok.v, tok.g, tok.beta, st, scale=0.9)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(sd, s_ref, TOL_FP32, "state")


def test_decode_workload_full_layer_two_steps():
    spec = kin.DECODE_256x34
    dev = torch.device("cuda")
    st = kin.make_decode_state(spec, 5)
    sd = st.to(dev)
    ref_state = st
    for step in range(2):
        tok = kin.make_decode_tokens(spec, 5 + 100 * step)
        td = tok.to(dev)
        o = kda.kda_decode_step(td.q, td.k, td.v, td.g, td.beta, sd)
        torch.cuda.synchronize()
        o_ref, ref_state = oracle.kda_decode(tok.q, tok.k, tok.v, tok.g, tok.beta, ref_state)
        # fp32 arithmetic throughout (bf16 inputs are exact in fp32): the tight bound
        assert_close(o, o_ref, TOL_FP32, f"o step {step}")
        assert_close(sd, ref_state, TOL_FP32, f"state step {step}")


# ---------------------------------------------------------------- scalar decay
# Gated-DeltaNet form: one decay per (token, head).  The oracle is the same
# per-channel rule with g broadcast over the channels.

def _scalar_decay_case(seed, lengths, heads=3):
    x = kin.make_custom_prefill(seed, lengths, heads=heads, init_state_std=0.02)
    gs = x.g[..., 0].contiguous()                      # [T, H]
    return x, gs, gs[..., None].expand_as(x.g).contiguous()


@pytest.mark.parametrize("mode", ["recurrent"] + PATHS)
def test_scalar_decay_prefill(mode):
    x, gs, gfull = _scalar_decay_case(41, [0, 70, 257, 64, 1])
    dev = torch.device("cuda")
    xd = x.to(dev)
    recurrent = mode == "recurrent"
    o, s = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, gs.to(dev), xd.beta, xd.cu_seqlens,
                             initial_state=xd.initial_state, recurrent=recurrent, scalar_decay=True,
                             workspace=small_workspace(x, dev) if mode == "fused" else None)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, gfull, x.beta, x.cu_seqlens, x.initial_state)
    tol = TOL_FP32 if recurrent else TOL_BF16
    assert_close(o, o_ref, tol, "o")
    assert_close(s, s_ref, tol, "final state")


def test_scalar_decay_prefill_8k_shape():
    x = kin.make_prefill(kin.PREFILL_8K)
    gs = x.g[..., 0].contiguous()
    dev = torch.device("cuda")
    xd = x.to(dev)
    o, s = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, gs.to(dev), xd.beta, xd.cu_seqlens, scalar_decay=True)
    torch.cuda.synchronize()
    heads = [0, 17]
    gfull = gs[:, heads, None].expand(-1, -1, 128).contiguous()
    o_ref, s_ref = oracle.kda_forward(x.q[:, heads].contiguous(), x.k[:, heads].contiguous(),
                                      x.v[:, heads].contiguous(), gfull, x.beta[:, heads].contiguous(),
                                      x.cu_seqlens)
    assert_close(o[:, heads], o_ref, TOL_BF16, "o")
    assert_close(s[:, heads], s_ref, TOL_BF16, "final state")


def test_scalar_decay_decode():
    spec = kin.DecodeSpec("scalar", 78, 6, 1, 4, torch.bfloat16)
    tok = kin.make_decode_tokens(spec, 0)
    st = kin.make_decode_state(spec, 0)
    gs = tok.g[..., 0].contiguous()
    dev = torch.device("cuda")
    td, sd = tok.to(dev), st.to(dev)
    o = kda.kda_decode_step(td.q, td.k, td.v, gs.to(dev), td.beta, sd, scalar_decay=True)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_decode(tok.q, tok.k, tok.v, gs[..., None].expand_as(tok.g), tok.beta, st)
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(sd, s_ref, TOL_FP32, "state")


# ---------------------------------------------------------------- state pools
# Continuous batching: states live in a pool and sequence n uses slots[n].

@pytest.mark.parametrize("mode", ["recurrent"] + PATHS)
def test_prefill_with_state_pool(mode):
    recurrent = mode == "recurrent"
    dev = torch.device("cuda")
    lengths, slots = [100, 0, 70], [4, 0, 5]
    x = kin.make_custom_prefill(51, lengths, heads=2, init_state_std=0.02)
    pool = torch.randn(6, 2, 128, 128) * 0.02
    pool[slots] = x.initial_state
    pool_d = pool.to(dev)
    xd = x.to(dev)
    o = kda.kda_chunk_fwd_slots(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, pool_d,
                                torch.tensor(slots, dtype=torch.int32, device=dev), recurrent=recurrent,
                                workspace=small_workspace(x, dev) if mode == "fused" else None)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
    tol = TOL_FP32 if recurrent else TOL_BF16
    assert_close(o, o_ref, tol, "o")
    assert_close(pool_d[slots], s_ref, tol, "pooled final states")
    untouched = [i for i in range(6) if i not in slots]
    assert torch.equal(pool_d[untouched].cpu(), pool[untouched])


def test_single_sequence_state_pool_overlapped_path():
    # one sequence: the overlapped prep/state launch, reading and writing the
    # state through a pool slot; 9 chunks wrap the 8-slot operand ring
    dev = torch.device("cuda")
    x = kin.make_custom_prefill(52, [9 * 64 - 5], heads=3, init_state_std=0.02)
    pool = torch.randn(4, 3, 128, 128) * 0.02
    pool[2] = x.initial_state[0]
    pool_d = pool.to(dev)
    xd = x.to(dev)
    o = kda.kda_chunk_fwd_slots(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, pool_d,
                                torch.tensor([2], dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(pool_d[2:3], s_ref, TOL_BF16, "pooled final state")
    assert torch.equal(pool_d[[0, 1, 3]].cpu(), pool[[0, 1, 3]])


def test_packed_sequences_with_many_heads_take_the_two_launch_path():
    # more heads than the overlapped launch takes: the separate prep and state
    # launches over several sequences, an empty one and a ragged tail included
    x = kin.make_custom_prefill(55, [130, 0, 300, 7], heads=100, init_state_std=0.02)
    o, s, o_ref, s_ref = run_both(x, heads=[0, 41, 99])
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")
    assert torch.equal(s[1].cpu(), x.initial_state[1][[0, 41, 99]])   # the empty sequence


def test_ring_with_a_bad_slot_hands_its_chunks_back():
    # several sequences through the overlapped launch (state pool): the middle
    # sequence's slot is out of range, so it is skipped, but the images made for
    # it must still be handed back for the prep role to go on to the third one
    dev = torch.device("cuda")
    x = kin.make_custom_prefill(56, [700, 900, 650], heads=4, init_state_std=0.02)
    xd = x.to(dev)
    pool = torch.zeros(4, 4, 128, 128)
    pool[0], pool[3] = x.initial_state[0], x.initial_state[2]
    pool_d = pool.to(dev)
    T, H = x.total_T, x.heads
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(3, T, H), dtype=torch.uint8, device=dev)
    kda.kda_chunk_fwd_slots(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, pool_d,
                            torch.tensor([0, 9, 3], dtype=torch.int32, device=dev), workspace=ws)
    err = kda.kda_workspace_error(ws)
    assert err & kda.KDA_DEVERR_SLOT and not err & kda.KDA_DEVERR_TIMEOUT
    for n, slot in ((0, 0), (2, 3)):
        cu = x.cu_seqlens.tolist()
        sl = slice(cu[n], cu[n + 1])
        _, s_ref = oracle.kda_forward(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], [0, cu[n + 1] - cu[n]],
                                      x.initial_state[n:n + 1])
        assert_close(pool_d[slot:slot + 1], s_ref, TOL_BF16, f"pooled final state of sequence {n}")


def test_single_sequence_with_many_heads_takes_the_two_launch_path():
    # more heads than the overlapped launch gives state CTAs to: one sequence
    # through the separate prep and state launches
    x = kin.make_custom_prefill(53, [300], heads=100, init_state_std=0.02)
    o, s, o_ref, s_ref = run_both(x, heads=[0, 57, 99])
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


@pytest.mark.parametrize("heads,tokens", [(96, 1280), (1, 2000)])
def test_overlapped_path_at_the_extremes_of_heads(heads, tokens):
    # one sequence through the overlapped launch with the most heads it takes
    # (fewest preparing CTAs) and with one head (most producers waiting for
    # its ring slots, which wrap many times)
    x = kin.make_custom_prefill(54, [tokens], heads=heads, init_state_std=0.02)
    o, s, o_ref, s_ref = run_both(x, heads=sorted({0, heads // 2, heads - 1}))
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


def test_prefill_state_pool_rejects_bad_slot():
    dev = torch.device("cuda")
    x = kin.make_custom_prefill(52, [40, 30], heads=2).to(dev)
    pool = torch.zeros(3, 2, 128, 128, device=dev)
    ws = torch.zeros(1024, dtype=torch.uint8, device=dev)
    kda.kda_chunk_fwd_slots(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, pool,
                            torch.tensor([1, 3], dtype=torch.int32, device=dev), workspace=ws)
    assert kda.kda_workspace_error(ws) & kda.KDA_DEVERR_SLOT
    assert torch.count_nonzero(pool[1]) > 0 and torch.count_nonzero(pool[[0, 2]]) == 0


def test_decode_with_state_pool():
    dev = torch.device("cuda")
    spec = kin.DecodeSpec("pool", 53, 4, 1, 3, torch.bfloat16)
    tok = kin.make_decode_tokens(spec, 0)
    pool = torch.randn(10, 3, 128, 128) * 0.02
    slots = [7, 2, 9, 0]
    pool_d = pool.to(dev)
    td = tok.to(dev)
    o = kda.kda_decode_step_slots(td.q, td.k, td.v, td.g, td.beta, pool_d,
                                  torch.tensor(slots, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.kda_decode(tok.q, tok.k, tok.v, tok.g, tok.beta, pool[slots])
    assert_close(o, o_ref, TOL_FP32, "o")
    assert_close(pool_d[slots], s_ref, TOL_FP32, "pooled states")
    untouched = [i for i in range(10) if i not in slots]
    assert torch.equal(pool_d[untouched].cpu(), pool[untouched])
    # an out-of-range slot skips that sequence: no state is touched and its o rows are NaN
    o2 = torch.full((4, 3, 128), 5.0, device=dev)
    before = pool_d.clone()
    kda.kda_decode_step_slots(td.q, td.k, td.v, td.g, td.beta, pool_d,
                              torch.tensor([7, -1, 9, 10], dtype=torch.int32, device=dev), o=o2)
    torch.cuda.synchronize()
    assert torch.isnan(o2[1]).all() and torch.isnan(o2[3]).all()
    assert torch.isfinite(o2[0]).all() and torch.isfinite(o2[2]).all()
    assert torch.equal(pool_d[[2, 0]], before[[2, 0]])


# ---------------------------------------------------------------- speculative verify
# Draft tokens are verified in one call; the state after every token is kept
# so that a rejected suffix can be rolled back.

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_verify_snapshots_match_prefix_states(dtype):
    dev = torch.device("cuda")
    lengths = [4, 1, 6, 0]
    x = kin.make_custom_prefill(61, lengths, heads=2, dtype=dtype, init_state_std=0.02)
    xd = x.to(dev)
    o, snaps = kda.kda_verify_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens,
                                  initial_state=xd.initial_state)
    torch.cuda.synchronize()
    o_ref, _ = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
    assert_close(o, o_ref, TOL_FP32, "o")
    cu = x.cu_seqlens.tolist()
    for n in range(len(lengths)):
        for t in range(cu[n], cu[n + 1]):   # state after token t = end state of the prefix up to t
            sl = slice(cu[n], t + 1)
            _, s_ref = oracle.kda_forward(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], [0, t + 1 - cu[n]],
                                          x.initial_state[n:n + 1])
            assert_close(snaps[t:t + 1], s_ref[:, :], TOL_FP32, f"snapshot of token {t}")


def test_bounded_waits_give_up_with_an_error_and_the_context_survives():
    # a flag nobody sets and an mbarrier phase that never completes: both
    # bounded waits give up, report KDA_DEVERR_TIMEOUT, and later work runs
    dev = torch.device("cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    kda.kda_selftest_bounded_waits(ws, polls=4096)
    assert kda.kda_workspace_error(ws) & kda.KDA_DEVERR_TIMEOUT
    x = kin.make_custom_prefill(62, [130], heads=2, init_state_std=0.02)
    o, s, o_ref, s_ref = run_both(x)
    assert_close(o, o_ref, TOL_BF16, "o after the self-test")
    assert_close(s, s_ref, TOL_BF16, "final state after the self-test")


@pytest.mark.parametrize("lengths", [[700], [300, 450]])
def test_prefill_replays_from_a_cuda_graph(lengths):
    # the overlapped launch for one and for two sequences, captured once and
    # replayed: the same bits as the eager call
    dev = torch.device("cuda")
    x = kin.make_custom_prefill(61, lengths, heads=4, init_state_std=0.02).to(dev)
    T, H, d = x.q.shape
    N = len(lengths)
    ws = torch.zeros(kda.kda_chunk_fwd_workspace_size(N, T, H), dtype=torch.uint8, device=dev)
    o = torch.empty(T, H, d, device=dev)
    sT = torch.empty(N, H, d, d, device=dev)
    call = lambda: kda.kda_chunk_fwd(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, initial_state=x.initial_state,
                                     final_state=sT, o=o, workspace=ws)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    o_ref, s_ref = o.clone(), sT.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    o.zero_()
    sT.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(sT, s_ref)
    assert kda.kda_workspace_error(ws) == 0


# ---------------------------------------------------------------- strong decay
# Decay rates far beyond the workloads': per-channel decay within a 64-token
# chunk of about 100, 500 and 5,000 nats, three channels at g = -80 per token,
# and a single spike that makes one chunk of a long sequence strong.  The
# two-pass prep takes such chunks' Gram matrices through 16-token block
# references or pairwise exponentials; the fused kernel hands the sequence to
# the token-by-token recurrence.  Every path must still match the oracle.
from tests.chunk_form import gram_level  # noqa: E402

STRONG = {
    "g_1.6_all": lambda g: g.fill_(-1.6),                  # ~100 nats per chunk
    "g_8_third": lambda g: g[..., ::3].fill_(-8.0),        # ~500 nats per chunk on a third of the channels
    "g_80_three": lambda g: g.__setitem__((Ellipsis, [3, 77, 100]), -80.0),   # ~5,000 nats per chunk
    "x40": lambda g: g.mul_(40.0),                         # ~270 nats per chunk on the fastest channel
    "spike": lambda g: g[100, :, 5].fill_(-150.0),         # one token, one channel
    # chunks of all three levels in one sequence: level 1 on chunks 3-4, level 2 on
    # chunk 7, level 0 around them (the state role switches forms chunk by chunk)
    "mixed": lambda g: (g[192:320].fill_(-1.6), g[448:512, :, ::3].fill_(-8.0)),
}


def _strong_input(kind, lengths, heads=2, seed=71):
    x = kin.make_custom_prefill(seed, lengths, heads=heads, init_state_std=0.02)
    STRONG[kind](x.g)
    return x


def _levels(x):
    """The Gram level of every (sequence, head, chunk), on the CPU."""
    cu = x.cu_seqlens.tolist()
    out = set()
    g = x.g.double().numpy()
    for n in range(len(cu) - 1):
        for c0 in range(cu[n], cu[n + 1], 64):
            for h in range(x.heads):
                gc = np.zeros((64, 128))
                L = min(64, cu[n + 1] - c0)
                gc[:L] = g[c0:c0 + L, h]
                out.add(gram_level(np.cumsum(gc, axis=0)))
    return out


@pytest.mark.parametrize("path", ["one_sequence", "two_sequences", "fused"])
@pytest.mark.parametrize("kind,level", [("g_1.6_all", 1), ("g_8_third", 2), ("g_80_three", 2), ("x40", 2),
                                        ("spike", 2), ("mixed", 2)])
def test_prefill_strong_decay(kind, level, path):
    lengths = [640] if path != "two_sequences" else [300, 340]
    x = _strong_input(kind, lengths)
    assert max(_levels(x)) == level   # the case exercises the intended Gram level
    if kind == "mixed" and path == "one_sequence":
        assert _levels(x) == {0, 1, 2}
    o, s, o_ref, s_ref = run_both(x, path="fused" if path == "fused" else "two_pass")
    assert_close(o, o_ref, TOL_BF16, "o")
    assert_close(s, s_ref, TOL_BF16, "final state")


def test_prefill_strong_decay_in_place_state():
    # the fused kernel's fallback restarts from the initial state: with the
    # final state aliasing it, it must not have been overwritten before
    x = _strong_input("g_80_three", [200, 90], heads=2)
    dev = torch.device("cuda")
    xd = x.to(dev)
    for path in ("two_pass", "fused"):
        state = xd.initial_state.clone()
        ws = small_workspace(x, dev) if path == "fused" else None
        o, _ = kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, initial_state=state,
                                 final_state=state, workspace=ws)
        torch.cuda.synchronize()
        o_ref, s_ref = oracle.kda_forward(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, x.initial_state)
        assert_close(o, o_ref, TOL_BF16, f"o ({path})")
        assert_close(state, s_ref, TOL_BF16, f"in-place final state ({path})")
