"""Chunked form of the KDA recurrence in numpy -- a test helper, not the oracle.

It restates, in fp64, the 64-token chunk algebra that the tensor-core prefill
kernel evaluates, so the derivation can be checked against the token-by-token
oracle independently of GPU numerics (and, with ``round_bf16=True``, so the
error added by rounding the MMA operands to bf16 can be estimated on the CPU).

For one chunk of L tokens with state S on entry (rows = key channels),
Gamma_r = g_0 + ... + g_r (per channel) and Gamma_C = Gamma_{L-1}:

    E_r = exp(Gamma_r - Gamma_C) >= 1,   F_r = exp(Gamma_C - Gamma_r) <= 1
    Kt = k_r * E_r,  Qt = q_r * E_r,  Kb = k_r * F_r          (rows r)
    St = diag(exp(Gamma_C)) S                     (state decayed to chunk end)
    A  = Kt Kb^T  (so A_ri = sum_c k_rc k_ic exp(Gamma_rc - Gamma_ic))
    P  = lower_incl(Qt Kb^T)
    Y  = Kt St,  Z = Qt St
    M  = strict_lower(diag(beta) A),  T = (I + M)^-1,  T' = T diag(beta)
    delta = T' (V - Y),   O = Z + P delta,   S_next = St + Kb^T delta

Unrolling the per-token rule inside the chunk gives
(I + M) delta = diag(beta)(V - K~ S) with K~_r = k_r exp(Gamma_r); K~ S = Kt St
because Kt diag(exp(Gamma_C)) = K~.  The readout and end state follow the
same way.
"""
import numpy as np

C = 64


def _bf16(x):
    """Round an fp64 array to the nearest bf16 value (ties to even)."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def _tf32(x):
    """Round an fp64 array to the nearest tf32 value (10-bit mantissa)."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x1000) >> 13) << 13          # round half away from zero, as cvt.rna
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def kda_forward_chunked(q, k, v, g, beta, cu_seqlens, initial_state=None, scale=1.0,
                        l2norm=True, eps=1e-6, round_bf16=False, round_to=None):
    """``round_to`` in (None, "bf16", "tf32") rounds every MMA operand the way
    the kernel stores it; ``round_bf16=True`` is the same as ``round_to="bf16"``."""
    if round_bf16:
        round_to = "bf16"
    rd = {None: (lambda x: x), "bf16": _bf16, "tf32": _tf32}[round_to]
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    cu = [int(x) for x in cu_seqlens]
    T, H, d = q.shape
    N = len(cu) - 1
    o = np.zeros((T, H, d))
    sT = np.zeros((N, H, d, d))
    for n in range(N):
        for h in range(H):
            S = np.zeros((d, d)) if initial_state is None else np.array(initial_state[n, h], dtype=np.float64)
            for c0 in range(cu[n], cu[n + 1], C):
                L = min(C, cu[n + 1] - c0)
                sl = slice(c0, c0 + L)
                qc, kc = q[sl, h], k[sl, h]
                if l2norm:
                    qc = qc / np.sqrt((qc * qc).sum(-1, keepdims=True) + eps)
                    kc = kc / np.sqrt((kc * kc).sum(-1, keepdims=True) + eps)
                qc = qc * scale
                G = np.cumsum(g[sl, h], axis=0)
                GC = G[-1]
                E = np.exp(G - GC)
                F = np.exp(GC - G)
                Kt, Qt, Kb = rd(kc * E), rd(qc * E), rd(kc * F)
                b = beta[sl, h]
                A = Kt @ Kb.T
                Mm = np.tril(b[:, None] * A, -1)
                Tm = np.linalg.inv(np.eye(L) + Mm)
                Tp = rd(Tm * b[None, :])
                P = rd(np.tril(Qt @ Kb.T))
                St32 = np.exp(GC)[:, None] * S
                St = rd(St32)
                Y, Z = Kt @ St, Qt @ St
                delta = Tp @ rd(v[sl, h]) + Tp @ rd(-Y)
                dl = rd(delta)
                o[sl, h] = Z + P @ dl
                S = St32 + Kb.T @ dl
            sT[n, h] = S
    return o, sT
