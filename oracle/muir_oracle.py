"""fp64 CPU oracle for the Muir gated delta-rule operator.

TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library, its
Python binding, the benchmark's GPU arm) may import or call this module; only
the tests, the smoke check and the benchmark's CPU-baseline arm do. It shares no
code with the CUDA path.

Sources (web pages about Muir, arXiv 2611.08376):
  [abs]  "Muir: Linear Attention with Sensitivity-Allocated Gating and
         Matched-Filter Readout", arXiv abstract (Astral feed / fugumt copies),
         "Full text": gated delta-rule models decay the state and erase the
         prediction for an incoming key before writing the new value; GDN-2 uses
         channel-wise decay and decoupled erase and write gates; Muir re-weights
         state rows with a matched-filter readout gate.
  [mf]   openai-hub article, section "Muir 先解决了状态里的'强光干扰'": a static
         per-row scale from each row's expected energy, plus a per-token
         (dynamic) modulation of the query at read time.
  [tpu]  openai-hub article, section "为 TPU 重写长序列并行算法", and the liuch.name
         post, bullet "Numerically-stable, large-chunk parallel kernel":
         boundary-pivoted multiplicative decays in (0, 1] with no division, and a
         triangular solve.

Operator, per batch b, head h, token t (all gates already activated):
    x_t = Diag(alpha_t) S_{t-1}                 channel-wise (row) decay
    p_t = x_t^T k_t                             prediction for the incoming key
    S_t = x_t - (e_t*k_t) p_t^T + k_t (w_t*v_t)^T   erase (gated per key row), then write
    qt  = r * g_t * q_t                         static row scale x dynamic query gate
    o_t = S_t^T qt                              matched-filter readout after the write
    y_t = z_t * o_t                             output gate
Readings where the pages are silent are listed in the design notes; the ones
used here: erase acts on key rows with a d_k-vector gate, the readout happens
after the write, the output gate is an elementwise product, no normalisation
happens inside the operator, alpha is passed as log_alpha.

Array layout: q,k,e,g,log_alpha [B,T,H,dk]; v,w,z [B,T,H,dv]; r [H,dk];
states [B,H,dk,dv]. Everything is computed in float64.
"""
from __future__ import annotations

import numpy as np


def _f(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _prep(q, k, v, e, w, g, z, log_alpha, r):
    q, k, v, e, w, g, log_alpha, r = map(_f, (q, k, v, e, w, g, log_alpha, r))
    z = np.ones_like(v) if z is None else _f(z)
    g = np.ones_like(q) if g is None else g  # [mf]: the static-only readout has no dynamic gate (g = 1)
    alpha = np.exp(log_alpha)
    qt = r[None, None] * g * q          # [mf]: static row scale times dynamic query gate
    a = e * k                           # erase direction: erase gate on key rows
    u = w * v                           # write value: write gate on value columns
    return q, k, v, e, w, g, z, alpha, qt, a, u, r


def step(S, alpha_t, k_t, a_t, u_t, qt_t):
    """One token of the recurrence for all (b, h) at once.

    S [B,H,dk,dv]; vectors [B,H,d]. Returns (x, p, S_new, o)."""
    x = alpha_t[..., :, None] * S                                # decay each key row
    p = np.matmul(k_t[..., None, :], x)[..., 0, :]                # p = x^T k
    S_new = x - a_t[..., :, None] * p[..., None, :] + k_t[..., :, None] * u_t[..., None, :]
    o = np.matmul(qt_t[..., None, :], S_new)[..., 0, :]           # o = S^T qt
    return x, p, S_new, o


def forward(q, k, v, e, w, g, z, log_alpha, r, S0=None, return_states=False):
    """Token-by-token recurrence ([abs], [mf]).

    Returns y [B,T,H,dv], S_T [B,H,dk,dv] and, if asked, all states
    [T+1,B,H,dk,dv] (index t holds S_t, index 0 holds S0)."""
    q, k, v, e, w, g, z, alpha, qt, a, u, r = _prep(q, k, v, e, w, g, z, log_alpha, r)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f(S0).copy()
    y = np.empty((B, T, H, dv))
    states = [S.copy()] if return_states else None
    for t in range(T):
        _, _, S, o = step(S, alpha[:, t], k[:, t], a[:, t], u[:, t], qt[:, t])
        y[:, t] = z[:, t] * o
        if return_states:
            states.append(S.copy())
    if return_states:
        return y, S, np.stack(states)
    return y, S


def decode_step(S, q, k, v, e, w, g, z, log_alpha, r):
    """One token for n independent sequences: S [N,H,dk,dv] -> (y [N,H,dv], S_new).

    The same update as forward() with T = 1."""
    y, S_new = forward(q[:, None], k[:, None], v[:, None], e[:, None], w[:, None], g[:, None],
                       None if z is None else z[:, None], log_alpha[:, None], r, S0=S)
    return y[:, 0], S_new


def row_scale(S, exponent=0.5, eps=1e-12):
    """[mf]: the static readout weights state row i by an inverse fractional power
    of its expected energy. Measured over states S [N,H,dk,dv]:
    r[h,i] = (mean_{n,j} S[n,h,i,j]^2 + eps)^(-exponent)."""
    S = _f(S)
    return (np.mean(S * S, axis=(0, 3)) + eps) ** (-exponent)


def backward(q, k, v, e, w, g, z, log_alpha, r, dy, S0=None, dS_T=None, checkpoint_every=64):
    """Reverse-mode of forward(), written out by hand, token by token.

    States are re-created from checkpoints saved every `checkpoint_every` tokens.
    Returns a dict with dq, dk, dv, de, dw, dg, dz, dlog_alpha ([B,T,H,*]), dS0
    [B,H,dk,dv] and dr [H,dk]; dg is None when g is None (the static-only readout).

    With G the cotangent of S_t and do = z * dy_t:
        dz = o * dy,   G += qt do^T,   dqt = S_t do
        from S_t = x - a p^T + k u^T:
            da = -G p,  dp = -G^T a,  du = G^T k,  dk += G u,  dx = G
        from p = x^T k:  dx += k dp^T,  dk += x dp
        from a = e*k:    de = k*da,  dk += e*da
        from u = w*v:    dw = v*du,  dv = w*du
        from qt = r*g*q: dq = r*g*dqt, dg = r*q*dqt, dr += g*q*dqt
        from x = alpha*S_{t-1}: dalpha_i = sum_j dx_ij S_{t-1,ij}, G <- alpha*dx
        dlog_alpha = alpha * dalpha.
    """
    has_g = g is not None
    q, k, v, e, w, g, z, alpha, qt, a, u, r = _prep(q, k, v, e, w, g, z, log_alpha, r)
    dy = _f(dy)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f(S0).copy()
    ck = {}
    for t in range(T):
        if t % checkpoint_every == 0:
            ck[t] = S.copy()
        _, _, S, _ = step(S, alpha[:, t], k[:, t], a[:, t], u[:, t], qt[:, t])

    grads = {n: np.zeros_like(q) for n in ("dq", "dk", "de", "dg", "dlog_alpha")}
    grads.update({n: np.zeros_like(v) for n in ("dv", "dw", "dz")})
    dr = np.zeros_like(r)
    G = np.zeros((B, H, dk, dv)) if dS_T is None else _f(dS_T).copy()
    for seg0 in range(((T - 1) // checkpoint_every) * checkpoint_every, -1, -checkpoint_every):
        seg1 = min(seg0 + checkpoint_every, T)
        prev = [ck[seg0]]
        for t in range(seg0, seg1):
            _, _, s_new, _ = step(prev[-1], alpha[:, t], k[:, t], a[:, t], u[:, t], qt[:, t])
            prev.append(s_new)
        for t in range(seg1 - 1, seg0 - 1, -1):
            S_prev, S_t = prev[t - seg0], prev[t - seg0 + 1]
            x = alpha[:, t][..., :, None] * S_prev
            p = np.matmul(k[:, t][..., None, :], x)[..., 0, :]
            o = np.matmul(qt[:, t][..., None, :], S_t)[..., 0, :]
            do = z[:, t] * dy[:, t]
            grads["dz"][:, t] = o * dy[:, t]
            G = G + qt[:, t][..., :, None] * do[..., None, :]
            dqt = np.matmul(S_t, do[..., :, None])[..., 0]
            da = -np.matmul(G, p[..., :, None])[..., 0]
            dp = -np.matmul(a[:, t][..., None, :], G)[..., 0, :]
            du = np.matmul(k[:, t][..., None, :], G)[..., 0, :]
            dk_t = np.matmul(G, u[:, t][..., :, None])[..., 0] + np.matmul(x, dp[..., :, None])[..., 0] \
                + e[:, t] * da
            dx = G + k[:, t][..., :, None] * dp[..., None, :]
            grads["de"][:, t] = k[:, t] * da
            grads["dk"][:, t] = dk_t
            grads["dw"][:, t] = v[:, t] * du
            grads["dv"][:, t] = w[:, t] * du
            grads["dq"][:, t] = r[None] * g[:, t] * dqt
            grads["dg"][:, t] = r[None] * q[:, t] * dqt
            dr += (g[:, t] * q[:, t] * dqt).sum(0)
            dalpha = (dx * S_prev).sum(-1)
            grads["dlog_alpha"][:, t] = alpha[:, t] * dalpha
            G = alpha[:, t][..., :, None] * dx
    grads["dS0"] = G
    grads["dr"] = dr
    if not has_g:
        grads["dg"] = None
    return grads


# ----------------------------------------------------------------------------
# Chunk algebra ([tpu]): the same operator computed chunk by chunk with
# boundary-pivoted decay products and an explicit triangular solve. Used only to
# check that the chunked form the kernels implement equals the recurrence.
# ----------------------------------------------------------------------------

def pivoted_decay(L_blockwise, t, s, c):
    """Gamma_{t<-s} = prod_{u=s+1..t} alpha_u for -1 <= s <= t inside one chunk,
    as a product of factors that are each exp of a non-positive block-local sum.
    s = -1 means "from the state before the chunk", i.e. prod_{u=0..t} alpha_u.

    L_blockwise [C, dk]: cumulative sum of log_alpha restarted at every block of
    c tokens (so every entry is <= 0). Returns (value [dk], list of factors)."""
    bt = t // c
    if s >= 0 and s // c == bt:
        f = [np.exp(L_blockwise[t] - L_blockwise[s])]            # same block: L_t - L_s <= 0
    else:
        f = []
        if s >= 0:
            end_s = (s // c + 1) * c - 1
            f.append(np.exp(L_blockwise[end_s] - L_blockwise[s]))  # suffix of s's block
            first = s // c + 1
        else:
            first = 0
        for blk in range(first, bt):
            f.append(np.exp(L_blockwise[(blk + 1) * c - 1]))      # whole blocks in between
        f.append(np.exp(L_blockwise[t]))                          # prefix of t's block
    val = np.ones_like(f[0])
    for x in f:
        val = val * x
    return val, f


def chunk_forward(q, k, v, e, w, g, z, log_alpha, r, chunk, sub=16, S0=None, return_factors=False):
    """Chunkwise form of forward() for one chunk size (T % chunk == 0).

    Per chunk with start state S0 and local tokens 1..C:
        M^kk_ts = k_t^T Diag(Gam_{t<-s}) k_s,  M^ka_ts = k_t^T Diag(Gam_{t<-s}) a_s   (s < t)
        N^qk_ts = qt_t^T Diag(Gam_{t<-s}) k_s, N^qa_ts = qt_t^T Diag(Gam_{t<-s}) a_s  (s <= t)
        (I + M^ka) P = (k * Gam_t) S0 + M^kk U          (forward substitution)
        O = (qt * Gam_t) S0 + N^qk U - N^qa P,   y = z * O
        S_C = Diag(Gam_C) S0 + (k * Gam_{C<-t})^T U - (a * Gam_{C<-t})^T P
    Decay products come from pivoted_decay(), never from a division."""
    q, k, v, e, w, g, z, alpha, qt, a, u, r = _prep(q, k, v, e, w, g, z, log_alpha, r)
    la = _f(log_alpha)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    C = chunk
    assert T % C == 0 and C % sub == 0
    S = np.zeros((B, H, dk, dv)) if S0 is None else _f(S0).copy()
    y = np.empty((B, T, H, dv))
    factors = []
    for b in range(B):
        for h in range(H):
            St = S[b, h].copy()
            for c0 in range(0, T, C):
                sl = slice(c0, c0 + C)
                K, A, Q, U = k[b, sl, h], a[b, sl, h], qt[b, sl, h], u[b, sl, h]
                Lb = np.empty((C, dk))
                for t in range(C):
                    Lb[t] = la[b, c0 + t, h] + (Lb[t - 1] if t % sub else 0.0)
                Gam = np.empty((C, C, dk))
                for t in range(C):
                    for s in range(t + 1):
                        Gam[t, s], f = pivoted_decay(Lb, t, s, sub)
                        if return_factors:
                            factors.extend(f)
                Mkk = np.zeros((C, C)); Mka = np.zeros((C, C))
                Nqk = np.zeros((C, C)); Nqa = np.zeros((C, C))
                for t in range(C):
                    for s in range(t + 1):
                        if s < t:
                            Mkk[t, s] = np.sum(K[t] * Gam[t, s] * K[s])
                            Mka[t, s] = np.sum(K[t] * Gam[t, s] * A[s])
                        Nqk[t, s] = np.sum(Q[t] * Gam[t, s] * K[s])
                        Nqa[t, s] = np.sum(Q[t] * Gam[t, s] * A[s])
                g_t = np.empty((C, dk))     # prod_{u<=t} alpha_u: decay from the chunk start through t
                g_suf = np.empty((C, dk))   # prod_{u>t} alpha_u: decay from after t to the chunk end
                for t in range(C):
                    g_t[t], f1 = pivoted_decay(Lb, t, -1, sub)
                    g_suf[t], f2 = pivoted_decay(Lb, C - 1, t, sub)
                    if return_factors:
                        factors.extend(f1 + f2)
                Zr = (K * g_t) @ St + Mkk @ U
                P = np.zeros((C, dv))
                for t in range(C):                       # forward substitution
                    P[t] = Zr[t] - Mka[t, :t] @ P[:t]
                O = (Q * g_t) @ St + Nqk @ U - Nqa @ P
                y[b, sl, h] = z[b, sl, h] * O
                St = g_t[C - 1][:, None] * St + (K * g_suf).T @ U - (A * g_suf).T @ P
            S[b, h] = St
    if return_factors:
        return y, S, factors
    return y, S
