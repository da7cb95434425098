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


# ---------------------------------------------------------------------------
# The forms the two-pass tensor-core prefill evaluates.  A chunk whose Gram
# level is 0 (below) keeps the chunk-end form above; any other chunk takes
# every state-side exponent relative to the chunk START, so all its factors
# lie in (0, 1] whatever the decay:
#     Qs = q exp(Gamma_r),  Ks = k exp(Gamma_r),  Kb = k exp(Gamma_C - Gamma_r)
#     W = T' Ks,  U = T' V,  delta = U - W S,  O = Qs S + P delta,
#     S_next = diag(exp(Gamma_C)) S + Kb^T delta,
# with S the state at the chunk start.  Only the intra-chunk Gram matrices
# A_ri = sum_c k_rc k_ic exp(Gamma_rc - Gamma_ic) and P (same with q_r) need
# exponent differences between tokens of the chunk; they are taken in one of
# three ways, chosen per chunk from the decay it carries (LIMIT = the largest
# exponent, in natural-log units, that one factor may hold):
#   level 0, every channel decays by at most LIMIT over the chunk: one product
#     through the chunk end, (q exp(Gamma_r - Gamma_C)) (k exp(Gamma_C - Gamma_i))^T;
#   level 1, every channel decays by at most LIMIT within each 16-token block:
#     with rho_a = Gamma at the last token of block a (rho_-1 = 0),
#     X_r = exp(Gamma_r - rho_{a(r)-1}), Y_i = exp(rho_{b(i)} - Gamma_i) and
#     Z_ab = exp(rho_{a-1} - rho_b) for blocks b <= a, exp(Gamma_r - Gamma_i) =
#     X_r Z_{a(r)b(i)} Y_i, where only Z_aa (the inverse of block a's own
#     decay) exceeds 1;
#   level 2, otherwise: every exp(Gamma_r - Gamma_i) on its own.
# ---------------------------------------------------------------------------
LIMIT = 100.0 * np.log(2.0)
SUB = 16


def gram_level(G, L=None):
    """The level (0, 1, 2) for one chunk's cumulative log-decay G [64, d]
    (rows past the chunk's last token repeat its value)."""
    rho = G[SUB - 1::SUB]                     # [4, d]: Gamma at the last token of each block
    if (-G[-1]).max() <= LIMIT:
        return 0
    prev = np.vstack([np.zeros((1, G.shape[1])), rho[:-1]])
    return 1 if (prev - rho).max() <= LIMIT else 2


def gram(qn, kn, G, level):
    """[P, A] (unmasked 64 x 64) of one chunk at the given level; qn, kn are
    the normalised (and scaled) rows, G the cumulative log-decay, all [64, d]."""
    if level == 0:
        GC = G[-1]
        Qt, Kt, Kb = qn * np.exp(G - GC), kn * np.exp(G - GC), kn * np.exp(GC - G)
        return Qt @ Kb.T, Kt @ Kb.T
    C = G.shape[0]
    if level == 1:
        rho = G[SUB - 1::SUB]
        prev = np.vstack([np.zeros((1, G.shape[1])), rho[:-1]])
        blk = np.arange(C) // SUB
        X = np.exp(G - prev[blk])
        Y = np.exp(rho[blk] - G)
        P = np.zeros((C, C))
        A = np.zeros((C, C))
        for a in range(C // SUB):
            ra = slice(SUB * a, SUB * a + SUB)
            for b in range(a + 1):
                rb = slice(SUB * b, SUB * b + SUB)
                Z = np.exp(prev[a] - rho[b])
                P[ra, rb] = (qn[ra] * X[ra] * Z) @ (kn[rb] * Y[rb]).T
                A[ra, rb] = (kn[ra] * X[ra] * Z) @ (kn[rb] * Y[rb]).T
        return P, A
    E = np.exp(np.minimum(G[:, None, :] - G[None, :, :], 0.0))   # [r, i, c], only i <= r is used
    return np.einsum("rc,ric,ic->ri", qn, E, kn), np.einsum("rc,ric,ic->ri", kn, E, kn)


def kda_forward_chunked_start(q, k, v, g, beta, cu_seqlens, initial_state=None, scale=1.0,
                              l2norm=True, eps=1e-6, force_level=None, levels=None):
    """The forms above, exact (fp64): the chunk-end state form for level-0
    chunks, the chunk-start form otherwise.  ``force_level`` evaluates every
    chunk at that level (where it is finite); ``levels``, if a list, receives
    the level each chunk chose."""
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
                qc, kc = np.zeros((C, d)), np.zeros((C, d))
                qc[:L], kc[:L] = q[sl, h], k[sl, h]
                if l2norm:
                    qc = qc / np.sqrt((qc * qc).sum(-1, keepdims=True) + eps)
                    kc = kc / np.sqrt((kc * kc).sum(-1, keepdims=True) + eps)
                qc = qc * scale
                gc = np.zeros((C, d))
                gc[:L] = g[sl, h]
                G = np.cumsum(gc, axis=0)
                GC = G[-1]
                lvl = gram_level(G) if force_level is None else force_level
                if levels is not None:
                    levels.append(lvl)
                P, A = gram(qc, kc, G, lvl)
                b = np.zeros(C)
                b[:L] = beta[sl, h]
                Mm = np.tril(b[:, None] * A, -1)
                Tp = np.linalg.inv(np.eye(C) + Mm) * b[None, :]
                P = np.tril(P)
                V = np.zeros((C, d))
                V[:L] = v[sl, h]
                Kb = kc * np.exp(GC - G)
                if lvl == 0:   # chunk-end form: the state decayed first, factors up to e^LIMIT
                    Qt, Kt = qc * np.exp(G - GC), kc * np.exp(G - GC)
                    St = np.exp(GC)[:, None] * S
                    W, U = Tp @ Kt, Tp @ V
                    delta = U - W @ St
                    o[sl, h] = (Qt @ St + P @ delta)[:L]
                    S = St + Kb.T @ delta
                else:          # chunk-start form: every factor at most 1
                    Qs, Ks = qc * np.exp(G), kc * np.exp(G)
                    W, U = Tp @ Ks, Tp @ V
                    delta = U - W @ S
                    o[sl, h] = (Qs @ S + P @ delta)[:L]
                    S = np.exp(GC)[:, None] * S + Kb.T @ delta
            sT[n, h] = S
    return o, sT
