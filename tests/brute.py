"""Independent float64 NumPy restatements used to pin the oracle (tiny sizes).

Nothing here is shared with the oracle or the CUDA path.  The conv uses
``np.convolve``, the gates ``np.logaddexp``/``scipy.special.expit``, the
recurrence is expanded into explicit d_k x d_k transition matrices, and the
chunked twins follow the chunkwise (WY/UT) form of the same recurrence: its
factored form, and its affine form (the chunk's terms that multiply the state
collected into one d_k x d_k map) with (I + A)^-1 by recursive doubling.
"""

from __future__ import annotations

import numpy as np
from scipy.special import expit


def conv_silu(x_seq: np.ndarray, hist: np.ndarray, w: np.ndarray) -> np.ndarray:
    """SiLU(causal depthwise conv) of one sequence via np.convolve.

    x_seq [L, C], hist [W-1, C] (oldest first), w [C, W] (last tap on the
    current token).  Returns u [L, C].
    """
    full = np.concatenate([hist, x_seq], axis=0).astype(np.float64)
    L, C = x_seq.shape
    y = np.empty((L, C))
    for c in range(C):
        y[:, c] = np.convolve(full[:, c], w[c, ::-1].astype(np.float64), mode="valid")
    return y * expit(y)


def l2n(x: np.ndarray, eps: float) -> np.ndarray:
    return x / np.sqrt(np.linalg.norm(x) ** 2 + eps)


def gates(a, dt_bias, A_log, b):
    a, dt_bias, A_log, b = (np.asarray(x, np.float64) for x in (a, dt_bias, A_log, b))
    g = -np.exp(A_log) * np.logaddexp(0.0, a + dt_bias)
    return g, np.exp(g), expit(b)


def head_inputs(geo, params, qkv_seq, hist, h):
    """Post-conv, normalised (q, k, v) rows of value head h for one sequence."""
    conv_w = params[0]
    u = conv_silu(qkv_seq, hist, conv_w)
    G = geo.num_v_heads // geo.num_k_heads
    kh = h // G
    dk, dv, Hk = geo.head_k_dim, geo.head_v_dim, geo.num_k_heads
    q = u[:, kh * dk:(kh + 1) * dk]
    k = u[:, Hk * dk + kh * dk:Hk * dk + (kh + 1) * dk]
    v = u[:, 2 * Hk * dk + h * dv:2 * Hk * dk + (h + 1) * dv]
    qh = np.stack([geo.q_scale * l2n(r, geo.l2_eps) for r in q])
    kh_ = np.stack([l2n(r, geo.l2_eps) for r in k])
    return qh, kh_, v


def expansion_states(S0, k, v, alpha, beta):
    """States S_1..S_L from the outer-product expansion
    S_t = Phi_{t,1} S0 + sum_{s<=t} Phi_{t,s+1} beta_s k_s v_s^T,
    Phi_{t,s} = prod_{r=t..s} alpha_r (I - beta_r k_r k_r^T), built explicitly."""
    L, dk = k.shape
    I = np.eye(dk)
    M = [alpha[r] * (I - beta[r] * np.outer(k[r], k[r])) for r in range(L)]
    out = []
    for t in range(L):
        def phi(hi, lo):  # product M[hi] @ M[hi-1] @ ... @ M[lo]; identity if lo > hi
            P = I.copy()
            for r in range(lo, hi + 1):
                P = M[r] @ P
            return P
        S = phi(t, 0) @ S0
        for s in range(t + 1):
            S = S + phi(t, s + 1) @ (beta[s] * np.outer(k[s], v[s]))
        out.append(S)
    return out


def rmsnorm_gate(o, z, w, eps):
    o, z, w = (np.asarray(x, np.float64) for x in (o, z, w))
    return o / np.sqrt(np.mean(o ** 2) + eps) * (1.0 + w) * expit(z)


def prefill(geo, params, qkv, z, a, b, cu, hist, state):
    """Whole prefill by brute force.  Returns (o [T, Hv*dv], state)."""
    conv_w, A_log, dt_bias, norm_w = (np.asarray(p, np.float64) for p in params)
    Hv, dv = geo.num_v_heads, geo.head_v_dim
    T = int(cu[-1])
    o = np.zeros((T, Hv * dv))
    st = np.array(state, np.float64).copy()
    for n in range(len(cu) - 1):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        if t1 == t0:
            continue
        for h in range(Hv):
            qh, kh, v = head_inputs(geo, params, np.asarray(qkv[t0:t1], np.float64), np.asarray(hist[n], np.float64), h)
            g, alpha, beta = gates(np.asarray(a[t0:t1, h], np.float64), dt_bias[h], A_log[h],
                                   np.asarray(b[t0:t1, h], np.float64))
            S0 = st[n, h].T  # stored [dv, dk]
            Ss = expansion_states(S0, kh, v, alpha, beta)
            for t in range(t1 - t0):
                ot = Ss[t].T @ qh[t]
                o[t0 + t, h * dv:(h + 1) * dv] = rmsnorm_gate(ot, np.asarray(z[t0 + t, h * dv:(h + 1) * dv], np.float64),
                                                               norm_w, geo.norm_eps)
            st[n, h] = Ss[-1].T
    return o, st


def chunked_head(S0, q, k, v, g, beta, C):
    """Chunkwise (WY/UT) form of the gated delta rule for one head.

    Within a chunk with cumulative log decay gamma_r = sum_{i<=r} g_i:
      A_ij = beta_i exp(gamma_i - gamma_j) k_i.k_j  (j < i),  T = (I + A)^-1,
      W = T diag(beta e^gamma) K,  U = T diag(beta) V,  Delta = U - W S,
      O = diag(e^gamma) Q S + (M o Q K^T) Delta,  M_ri = exp(gamma_r - gamma_i) (i <= r),
      S <- e^{gamma_L} S + K^T diag(e^{gamma_L - gamma}) Delta.
    S is [dk, dv].  Returns (o [L, dv] before the output norm, S_final).
    """
    L = q.shape[0]
    S = S0.copy()
    outs = []
    for c0 in range(0, L, C):
        c1 = min(L, c0 + C)
        Q, K, V = q[c0:c1], k[c0:c1], v[c0:c1]
        gam = np.cumsum(g[c0:c1])
        bt = beta[c0:c1]
        n = c1 - c0
        diff = gam[:, None] - gam[None, :]
        lower = np.tril(np.ones((n, n)), -1)
        A = (bt[:, None] * np.exp(np.where(lower > 0, diff, 0.0)) * (K @ K.T)) * lower
        Tm = np.linalg.inv(np.eye(n) + A)
        Wm = Tm @ ((bt * np.exp(gam))[:, None] * K)
        Um = Tm @ (bt[:, None] * V)
        D = Um - Wm @ S
        Mm = np.exp(np.where(np.tril(np.ones((n, n))) > 0, diff, -np.inf))
        O = np.exp(gam)[:, None] * (Q @ S) + (Mm * (Q @ K.T)) @ D
        S = np.exp(gam[-1]) * S + K.T @ (np.exp(gam[-1] - gam)[:, None] * D)
        outs.append(O)
    return np.concatenate(outs, axis=0), S


def doubling_inverse(A, base):
    """(I + A)^-1 for a strictly lower triangular A by recursive doubling:
    base x base diagonal blocks by forward substitution, then for b = base,
    2 base, ... every pair of b-blocks merged by T <- T - T (A_off,b T), where
    A_off,b keeps the entries of A whose row and column first fall in
    different halves of a 2b-block.  Padded with zeros to base * 2^k rows."""
    n = A.shape[0]
    Np = base
    while Np < n:
        Np *= 2
    Ap = np.zeros((Np, Np))
    Ap[:n, :n] = A
    T = np.zeros((Np, Np))
    for o in range(0, Np, base):
        blk = Ap[o:o + base, o:o + base]
        for c in range(base):
            t = np.zeros(base)
            for i in range(base):
                t[i] = (1.0 if i == c else 0.0) - (blk[i, :i] @ t[:i] if i else 0.0)
                if i < c:
                    t[i] = 0.0
            T[o:o + base, o + c] = t
    b = base
    while b < Np:
        Aoff = np.zeros((Np, Np))
        for o in range(0, Np, 2 * b):
            Aoff[o + b:o + 2 * b, o:o + b] = Ap[o + b:o + 2 * b, o:o + b]
        T = T - T @ (Aoff @ T)
        b *= 2
    return T[:n, :n]


def affine_head(S0, q, k, v, g, beta, C, base=4):
    """The chunk maps of the gated delta rule collected as affine maps of the
    state, per chunk (same gamma, A, W, U, P as chunked_head, with T from
    doubling_inverse):
      K~ = diag(e^{gamma_L - gamma}) K,   M' = -K~^T W,   Q' = diag(e^gamma) Q - P W,
      O = Q' S + P U,                      S <- e^{gamma_L} S + M' S + K~^T U.
    S is [dk, dv].  Returns (o [L, dv] before the output norm, S_final)."""
    L = q.shape[0]
    S = S0.copy()
    outs = []
    for c0 in range(0, L, C):
        c1 = min(L, c0 + C)
        Q, K, V = q[c0:c1], k[c0:c1], v[c0:c1]
        gam = np.cumsum(g[c0:c1])
        bt = beta[c0:c1]
        n = c1 - c0
        diff = gam[:, None] - gam[None, :]
        lower = np.tril(np.ones((n, n)), -1)
        A = (bt[:, None] * np.exp(np.where(lower > 0, diff, 0.0)) * (K @ K.T)) * lower
        Tm = doubling_inverse(A, base)
        Wm = Tm @ ((bt * np.exp(gam))[:, None] * K)
        Um = Tm @ (bt[:, None] * V)
        P = np.exp(np.where(np.tril(np.ones((n, n))) > 0, diff, -np.inf)) * (Q @ K.T)
        Kt = np.exp(gam[-1] - gam)[:, None] * K
        Mp = -(Kt.T @ Wm)
        Qp = np.exp(gam)[:, None] * Q - P @ Wm
        outs.append(Qp @ S + P @ Um)
        S = np.exp(gam[-1]) * S + Mp @ S + Kt.T @ Um
    return np.concatenate(outs, axis=0), S
