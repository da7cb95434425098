"""Brute-force numpy formulation of the KDA recurrence -- TEST INFRASTRUCTURE ONLY.

An independent restatement used to pin the C oracle on tiny inputs: each
token's transition is built as an explicit d x d matrix and multiplied with
numpy ``@``, exactly as the update rule on page "GLM-5.3-FLASH"
(dimsnsums.com), section "How can a layer remember without rereading?", is
printed:

    E_t = (I - beta_t k_t k_t^T) @ Diag(alpha_t)
    S_t = E_t @ S_{t-1} + beta_t * outer(k_t, v_t)
    o_t = scale * S_t^T @ q_t

Cost is O(d^3) per token, so keep T small.  ``order="erase_then_decay"``
evaluates the other reading of the prose (Diag(alpha) applied after the
erase), used only by a test that shows the two readings differ.
"""
from __future__ import annotations

import numpy as np

from . import to_f64, EPS


def _unit(x, l2norm, eps):
    if not l2norm:
        return x
    return x / np.sqrt(np.dot(x, x) + eps)


def kda_forward_bruteforce(q, k, v, g, beta, cu_seqlens, initial_state=None, scale=1.0,
                           l2norm=True, eps=EPS, order="decay_then_erase"):
    q, k, v, g, beta = (to_f64(t) for t in (q, k, v, g, beta))
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    T, H, d = q.shape
    N = len(cu) - 1
    s0 = to_f64(initial_state)
    o = np.zeros((T, H, d))
    sT = np.zeros((N, H, d, d))
    I = np.eye(d)
    for n in range(N):
        for h in range(H):
            S = np.zeros((d, d)) if s0 is None else s0[n, h].copy()
            for t in range(cu[n], cu[n + 1]):
                qt = _unit(q[t, h], l2norm, eps)
                kt = _unit(k[t, h], l2norm, eps)
                A = np.diag(np.exp(g[t, h]))
                erase = I - beta[t, h] * np.outer(kt, kt)
                E = erase @ A if order == "decay_then_erase" else A @ erase
                S = E @ S + beta[t, h] * np.outer(kt, v[t, h])
                o[t, h] = scale * (S.T @ qt)
            sT[n, h] = S
    return o, sT
