"""Pins of the fp64 oracle against what the page and the mathematics fix.

The page (dimsnsums.com "GLM-5.3-FLASH", section "How can a layer remember
without rereading?") prints one update rule and describes it in words; it has
no worked numbers.  The oracle is therefore pinned by: a hand-worked example
(tests/golden), special cases with closed forms, an independent brute-force
matrix formulation on tiny inputs, and invariants (split/resume, varlen
packing, linearity, a norm bound, delta-rule overwrite and recall).  Each
check is chosen so a plausible slip in the oracle -- a dropped term, a wrong
sign, decay on the wrong axis, S instead of S^T, reading out the state before
the update, erase and decay swapped -- fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.bruteforce import kda_forward_bruteforce
from gated_delta_rule_152_b200 import inputs as kin

D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_3tok.txt")


def rand_case(seed, lengths, H=2, init=True, l2=True, decay_scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    T = sum(lengths)
    q = torch.randn(T, H, D, generator=gen, dtype=torch.float64)
    k = torch.randn(T, H, D, generator=gen, dtype=torch.float64)
    v = torch.randn(T, H, D, generator=gen, dtype=torch.float64)
    g = -torch.nn.functional.softplus(torch.randn(T, H, D, generator=gen, dtype=torch.float64) - 1.0) * decay_scale
    beta = torch.sigmoid(torch.randn(T, H, generator=gen, dtype=torch.float64))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    s0 = torch.randn(len(lengths), H, D, D, generator=gen, dtype=torch.float64) * 0.1 if init else None
    if not l2:
        # without in-layer normalisation keep |k| near 1 so the recurrence stays bounded
        q, k = q / math.sqrt(D), k / math.sqrt(D)
    return [x.numpy() if x is not None else None for x in (q, k, v, g, beta)], cu, \
        (None if s0 is None else s0.numpy())


def _load_golden():
    ins = {"q": np.zeros((3, 1, D)), "k": np.zeros((3, 1, D)), "v": np.zeros((3, 1, D)),
           "alpha": np.ones((3, 1, D)), "beta": np.zeros((3, 1))}
    o_exp = np.zeros((3, 1, D))
    s_exp = np.zeros((1, 1, D, D))
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] == "in":
                name, t, c, val = parts[1], int(parts[2]), parts[3], float(parts[4])
                if name == "beta":
                    ins["beta"][t, 0] = val
                else:
                    ins[name][t, 0, int(c)] = val
            elif parts[0] == "out":
                if parts[1] == "o":
                    o_exp[int(parts[2]), 0, int(parts[3])] = float(parts[4])
                else:
                    s_exp[0, 0, int(parts[2]), int(parts[3])] = float(parts[4])
    g = np.log(ins["alpha"])
    return ins["q"], ins["k"], ins["v"], g, ins["beta"], o_exp, s_exp


def test_golden_worked_example_exact():
    q, k, v, g, beta, o_exp, s_exp = _load_golden()
    o, sT = oracle.kda_forward(q, k, v, g, beta, [0, 3], l2norm=False)
    np.testing.assert_allclose(o, o_exp, rtol=0, atol=1e-15)
    np.testing.assert_allclose(sT, s_exp, rtol=0, atol=1e-15)


def test_golden_worked_example_with_l2norm():
    # Same example with k scaled by 3 and q by 5: with L2-normalisation on,
    # q and k become unit vectors again (up to eps/|x|^2 ~ 1e-7 relative),
    # except q_3 = 5(e0 + e3) which normalises to (e0 + e3)/sqrt(2).
    q, k, v, g, beta, o_exp, s_exp = _load_golden()
    o, sT = oracle.kda_forward(5 * q, 3 * k, v, g, beta, [0, 3], l2norm=True)
    o_exp = o_exp.copy()
    o_exp[2] /= math.sqrt(2.0)
    np.testing.assert_allclose(o, o_exp, rtol=0, atol=1e-6)
    np.testing.assert_allclose(sT, s_exp, rtol=0, atol=1e-6)


def test_I1_beta0_alpha1_leaves_state_unchanged():
    (q, k, v, g, beta), cu, s0 = rand_case(1, [7, 5])
    g[:] = 0.0
    beta[:] = 0.0
    o, sT = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    np.testing.assert_allclose(sT, s0, rtol=0, atol=1e-14)
    for n in range(2):
        for t in range(cu[n], cu[n + 1]):
            for h in range(2):
                qh = q[t, h] / np.sqrt(q[t, h] @ q[t, h] + oracle.EPS)
                np.testing.assert_allclose(o[t, h], s0[n, h].T @ qh, rtol=1e-12, atol=1e-12)


def test_I2_delta_overwrite_reads_back_v():
    # alpha = 1, beta = 1, unit key: S_t^T k_t = v_t exactly, whatever S_{t-1}.
    # Keys are normalised here (not by the layer, whose eps would leave
    # |k|^2 = 1 - eps/|k|^2), so the identity holds to rounding.
    (q, k, v, g, beta), cu, s0 = rand_case(2, [9], init=True)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    g[:] = 0.0
    beta[:] = 1.0
    o, _ = oracle.kda_forward(k, k, v, g, beta, cu, s0, l2norm=False)   # read with q = k
    np.testing.assert_allclose(o, v, rtol=1e-12, atol=1e-12)


def test_I3_orthonormal_recall_and_replacement():
    rng = np.random.default_rng(3)
    n = 40
    Qm, _ = np.linalg.qr(rng.standard_normal((D, D)))
    keys = Qm[:, :n].T                        # n orthonormal keys
    vals = rng.standard_normal((n, D))
    # write all n pairs, then rewrite key 5 with a new value
    newv = rng.standard_normal(D)
    K = np.concatenate([keys, keys[5:6]])[:, None, :]
    V = np.concatenate([vals, newv[None]])[:, None, :]
    T = K.shape[0]
    g = np.zeros((T, 1, D))
    beta = np.ones((T, 1))
    _, sT = oracle.kda_forward(K, K, V, g, beta, [0, T], l2norm=False)
    S = sT[0, 0]
    recalled = keys @ S                        # row j = S^T k_j
    exp = vals.copy()
    exp[5] = newv                              # only the latest value survives
    np.testing.assert_allclose(recalled, exp, rtol=1e-9, atol=1e-9)


def test_I3_capacity_exceeded_breaks_exact_recall():
    # More than 128 distinct keys cannot all be recalled exactly by a 128x128 state.
    rng = np.random.default_rng(4)
    n = 160
    keys = rng.standard_normal((n, D))
    keys /= np.linalg.norm(keys, axis=1, keepdims=True)
    vals = rng.standard_normal((n, D))
    T = n
    _, sT = oracle.kda_forward(keys[:, None], keys[:, None], vals[:, None], np.zeros((T, 1, D)),
                               np.ones((T, 1)), [0, T], l2norm=False)
    err = np.abs(keys @ sT[0, 0] - vals).max()
    assert err > 1e-3


def test_I4_beta0_closed_form_decay():
    (q, k, v, g, beta), cu, s0 = rand_case(5, [11, 6])
    beta[:] = 0.0
    o, sT = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    for n in range(2):
        sl = slice(cu[n], cu[n + 1])
        G = np.cumsum(g[sl], axis=0)           # Gamma_t per channel
        for h in range(2):
            np.testing.assert_allclose(sT[n, h], np.exp(G[-1, h])[:, None] * s0[n, h],
                                       rtol=1e-12, atol=1e-14)
            for i, t in enumerate(range(cu[n], cu[n + 1])):
                qh = q[t, h] / np.sqrt(q[t, h] @ q[t, h] + oracle.EPS)
                np.testing.assert_allclose(o[t, h], s0[n, h].T @ (np.exp(G[i, h]) * qh),
                                           rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("l2", [True, False])
def test_I5_bruteforce_matrix_products(l2):
    (q, k, v, g, beta), cu, s0 = rand_case(6, [5, 0, 9, 16], init=True, l2=l2)
    o, sT = oracle.kda_forward(q, k, v, g, beta, cu, s0, scale=0.7, l2norm=l2)
    ob, sb = kda_forward_bruteforce(q, k, v, g, beta, cu, s0, scale=0.7, l2norm=l2)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(sT, sb, rtol=1e-11, atol=1e-12)


def test_I6_split_resume_and_varlen_packing():
    (q, k, v, g, beta), cu, s0 = rand_case(7, [50], init=True)
    o_full, s_full = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    for cut in (1, 17, 49):
        o1, s1 = oracle.kda_forward(q[:cut], k[:cut], v[:cut], g[:cut], beta[:cut], [0, cut], s0)
        o2, s2 = oracle.kda_forward(q[cut:], k[cut:], v[cut:], g[cut:], beta[cut:], [0, 50 - cut], s1)
        np.testing.assert_allclose(np.concatenate([o1, o2]), o_full, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(s2, s_full, rtol=1e-12, atol=1e-13)
    # packing: three sequences in one call == three separate calls
    lens = [13, 0, 29]
    (q, k, v, g, beta), cu, s0 = rand_case(8, lens, init=True)
    o, sT = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    for n in range(3):
        sl = slice(cu[n], cu[n + 1])
        on, sn = oracle.kda_forward(q[sl], k[sl], v[sl], g[sl], beta[sl], [0, lens[n]], s0[n:n + 1])
        np.testing.assert_allclose(o[sl], on, rtol=0, atol=0)
        np.testing.assert_allclose(sT[n:n + 1], sn, rtol=0, atol=0)
    np.testing.assert_allclose(sT[1], s0[1], rtol=0, atol=0)   # empty sequence: final = initial


def test_I7_linear_in_initial_state_and_values():
    (q, k, v, g, beta), cu, s0 = rand_case(9, [21, 8], init=True)
    (_, _, v2, _, _), _, s02 = rand_case(10, [21, 8], init=True)
    a, b = 0.7, -1.3
    oa, sa = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    ob, sb = oracle.kda_forward(q, k, v2, g, beta, cu, s02)
    oc, sc = oracle.kda_forward(q, k, a * v + b * v2, g, beta, cu, a * s0 + b * s02)
    np.testing.assert_allclose(oc, a * oa + b * ob, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(sc, a * sa + b * sb, rtol=1e-10, atol=1e-12)


def test_I8_frobenius_norm_bound_per_token():
    # With |k| = 1, beta in [0,1], alpha in (0,1]: ||E_t||_2 <= 1, hence
    # ||S_t||_F <= ||S_{t-1}||_F + beta_t ||v_t||.
    (q, k, v, g, beta), cu, s0 = rand_case(11, [30], H=1, init=True)
    S = s0
    for t in range(30):
        _, S_new = oracle.kda_forward(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1],
                                      beta[t:t + 1], [0, 1], S)
        lhs = np.linalg.norm(S_new[0, 0])
        rhs = np.linalg.norm(S[0, 0]) + beta[t, 0] * np.linalg.norm(v[t, 0])
        assert lhs <= rhs * (1 + 1e-12)
        S = S_new


def test_I9_order_of_decay_and_erase():
    # Uniform (scalar, GDN-style) decay commutes with the erase, so both
    # readings of the prose agree; per-channel decay does not, and the oracle
    # must follow the printed product (decay first, then erase).
    (q, k, v, g, beta), cu, s0 = rand_case(12, [12], init=True)
    g_scalar = np.repeat(g[..., :1], D, axis=-1)
    o_s, s_s = oracle.kda_forward(q, k, v, g_scalar, beta, cu, s0)
    ob1, sb1 = kda_forward_bruteforce(q, k, v, g_scalar, beta, cu, s0, order="decay_then_erase")
    ob2, sb2 = kda_forward_bruteforce(q, k, v, g_scalar, beta, cu, s0, order="erase_then_decay")
    np.testing.assert_allclose(o_s, ob1, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(ob1, ob2, rtol=1e-11, atol=1e-11)
    o, _ = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    oo, _ = kda_forward_bruteforce(q, k, v, g, beta, cu, s0, order="erase_then_decay")
    assert np.abs(o - oo).max() > 1e-3


def test_l2norm_is_scale_invariant():
    (q, k, v, g, beta), cu, s0 = rand_case(13, [10])
    o1, s1 = oracle.kda_forward(q, k, v, g, beta, cu, s0)
    o2, s2 = oracle.kda_forward(4.0 * q, 0.5 * k, v, g, beta, cu, s0)
    np.testing.assert_allclose(o1, o2, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(s1, s2, rtol=1e-5, atol=1e-6)


def test_decode_equals_one_token_forward():
    (q, k, v, g, beta), _, _ = rand_case(14, [6], H=3, init=False)
    rng = np.random.default_rng(14)
    S = rng.standard_normal((6, 3, D, D)) * 0.02
    o_dec, S_dec = oracle.kda_decode(q, k, v, g, beta, S)
    o_fwd, S_fwd = oracle.kda_forward(q, k, v, g, beta, np.arange(7), S)
    np.testing.assert_allclose(o_dec, o_fwd, rtol=0, atol=0)
    np.testing.assert_allclose(S_dec, S_fwd, rtol=0, atol=0)


def test_input_generators_are_seeded_and_shaped():
    a = kin.make_prefill(kin.TINY_FP32)
    b = kin.make_prefill(kin.TINY_FP32)
    for x, y in zip((a.q, a.k, a.v, a.g, a.beta), (b.q, b.k, b.v, b.g, b.beta)):
        assert torch.equal(x, y)
    assert a.q.shape == (256, 2, D) and a.q.dtype == torch.float32
    assert (a.g <= 0).all() and ((a.beta > 0) & (a.beta < 1)).all()
    lens = kin.seq_lengths(kin.VARLEN_16)
    assert len(lens) == 16 and all(512 <= x <= 16384 for x in lens)
    t = kin.make_decode_tokens(kin.DECODE_256x34, 3, n_seqs=4)
    assert t.q.shape == (4, 32, D) and t.q.dtype == torch.bfloat16


def test_state_slab_prefix_is_stable():
    # Regenerating a layer slab for fewer sequences reproduces the first rows.
    full = kin.make_decode_state(kin.DECODE_256x34, 7, n_seqs=4)
    part = kin.make_decode_state(kin.DECODE_256x34, 7, n_seqs=2)
    assert torch.equal(full[:2], part)
