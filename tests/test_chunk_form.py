"""The 64-token chunk algebra used by the tensor-core kernel, checked on the
CPU against the token-by-token oracle (exact arithmetic), and the operand
precision it runs at (tf32) checked against the 2e-2 x RMS bar."""
import numpy as np
import pytest

import oracle
from gated_delta_rule_152_b200 import inputs as kin
from tests.chunk_form import kda_forward_chunked

f64 = oracle.to_f64


def _case(seed, lengths, heads=2, std=0.02, decay_scale=1.0):
    x = kin.make_custom_prefill(seed, lengths, heads=heads, init_state_std=std)
    g = f64(x.g) * decay_scale
    o, s = oracle.kda_forward(x.q, x.k, x.v, g, x.beta, x.cu_seqlens, x.initial_state, scale=0.8)
    args = (f64(x.q), f64(x.k), f64(x.v), g, f64(x.beta), x.cu_seqlens.tolist(), f64(x.initial_state))
    return args, o, s


@pytest.mark.parametrize("lengths", [[1], [64], [65], [0, 130, 7, 200]])
def test_chunk_algebra_matches_oracle_exactly(lengths):
    args, o, s = _case(3, lengths)
    oc, sc = kda_forward_chunked(*args, scale=0.8)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sc, s, rtol=0, atol=1e-12)


def test_chunk_algebra_with_strong_decay():
    # ~40 nats of decay per channel per chunk: the chunk-end reference keeps
    # every factor finite
    args, o, s = _case(4, [300], decay_scale=8.0)
    oc, sc = kda_forward_chunked(*args, scale=0.8)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-9)
    np.testing.assert_allclose(sc, s, rtol=0, atol=1e-9)


def test_tf32_operands_fit_the_bf16_tolerance_with_margin():
    args, o, s = _case(5, [1500], heads=2)
    oc, sc = kda_forward_chunked(*args, scale=0.8, round_to="tf32")
    err_o = np.abs(oc - o).max() / np.sqrt(np.mean(o * o))
    err_s = np.abs(sc - s).max() / np.sqrt(np.mean(s * s))
    assert err_o < 1e-2 and err_s < 1e-2, (err_o, err_s)


# ---------------------------------------------------------------- chunk-start form
# The form of the two-pass tensor-core prefill: state-side factors relative to
# the chunk start (all in (0, 1]), Gram matrices at level 0, 1 or 2 by the
# chunk's decay.  Each level must reproduce the token-by-token oracle exactly
# (fp64), whatever the decay: the per-chunk decays below run from a few nats
# to several thousand, and one case drives three channels at g = -80 per token.
from tests.chunk_form import kda_forward_chunked_start  # noqa: E402


def _strong_case(kind):
    x = kin.make_custom_prefill(6, [300, 70], heads=2, init_state_std=0.02)
    g = f64(x.g)
    if kind == "per_token_2":          # ~2 nats per token on a third of the channels
        g[:, :, ::3] = -2.0
    elif kind == "x40":                # ~270 nats per chunk on the fastest channel
        g = g * 40.0
    elif kind == "x2000":              # ~13,500 nats per chunk
        g = g * 2000.0
    elif kind == "g80":                # three channels at g = -80 per token
        g[:, :, [3, 77, 100]] = -80.0
    o, s = oracle.kda_forward(x.q, x.k, x.v, g, x.beta, x.cu_seqlens, x.initial_state, scale=0.8)
    args = (f64(x.q), f64(x.k), f64(x.v), g, f64(x.beta), x.cu_seqlens.tolist(), f64(x.initial_state))
    return args, o, s


@pytest.mark.parametrize("kind,expect", [("plain", {0}), ("per_token_2", {0, 1}), ("x40", {0, 2}),
                                         ("x2000", {2}), ("g80", {2})])
def test_chunk_start_form_matches_oracle_at_any_decay(kind, expect):
    args, o, s = _strong_case(kind)
    levels = []
    oc, sc = kda_forward_chunked_start(*args, scale=0.8, levels=levels)
    assert set(levels) == expect
    scale_o, scale_s = np.sqrt(np.mean(o * o)), np.sqrt(np.mean(s * s))
    assert np.abs(oc - o).max() <= 1e-11 * scale_o
    assert np.abs(sc - s).max() <= 1e-11 * scale_s


@pytest.mark.parametrize("level", [1, 2])
def test_gram_levels_agree_where_all_are_finite(level):
    args, o, s = _strong_case("plain")
    oc, sc = kda_forward_chunked_start(*args, scale=0.8, force_level=level)
    np.testing.assert_allclose(oc, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sc, s, rtol=0, atol=1e-12)
