"""Numerical foil (test infrastructure): the chunkwise algorithm with the classic
division-based decay, in fp32, with no pivoting.

The Muir pages (liuch.name post, bullet "Numerically-stable, large-chunk parallel
kernel"; openai-hub article, section on the TPU chunkwise algorithm) contrast
their boundary-pivoted multiplicative decays with the earlier form in which the
chunk Grams use prefix products from the chunk start and their reciprocals,
Gam_{t<-s} = Gam_t / Gam_s, which overflows or underflows fp32 for fast-decaying
channels over long chunks (the pages report NaNs in a quarter of the heads).
This module writes that earlier form out so a test can show it failing where the
pivoted kernel does not. It is never used as a reference for parity.

Per chunk, with Gam_t = prod_{u<=t} alpha_u (from the chunk start), all fp32:
    Kp = K * Gam, Kd = K / Gam, Ad = A / Gam, Qp = Qt * Gam
    M^kk = tril(Kp Kd^T, -1), M^ka = tril(Kp Ad^T, -1)
    N^qk = tril(Qp Kd^T),     N^qa = tril(Qp Ad^T)
    (I + M^ka) P = Kp S0 + M^kk U
    O = Qp S0 + N^qk U - N^qa P,   S_C = Diag(Gam_C) S0 + (K Gam_C / Gam)^T U - (A Gam_C / Gam)^T P
"""
import numpy as np


def forward_unpivoted_fp32(q, k, v, e, w, g, z, log_alpha, r, chunk, S0=None):
    f = np.float32
    q, k, v, e, w, g, la, r = (np.asarray(x, dtype=f) for x in (q, k, v, e, w, g, log_alpha, r))
    z = np.ones_like(v) if z is None else np.asarray(z, dtype=f)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    qt, a, u = r[None, None] * g * q, e * k, w * v
    S = np.zeros((B, H, dk, dv), f) if S0 is None else np.asarray(S0, dtype=f).copy()
    y = np.empty((B, T, H, dv), f)
    tril_s = np.tril(np.ones((chunk, chunk), f), -1)
    tril = np.tril(np.ones((chunk, chunk), f))
    with np.errstate(all="ignore"):
        for c0 in range(0, T, chunk):
            sl = slice(c0, c0 + chunk)
            # [B,H,C,d] views of the chunk
            K, A, Q, U = (x[:, sl].transpose(0, 2, 1, 3) for x in (k, a, qt, u))
            gam = np.exp(np.cumsum(la[:, sl].transpose(0, 2, 1, 3), axis=2, dtype=f)).astype(f)
            Kp, Kd, Ad, Qp = K * gam, K / gam, A / gam, Q * gam
            Mkk = (Kp @ Kd.transpose(0, 1, 3, 2)) * tril_s
            Mka = (Kp @ Ad.transpose(0, 1, 3, 2)) * tril_s
            Nqk = (Qp @ Kd.transpose(0, 1, 3, 2)) * tril
            Nqa = (Qp @ Ad.transpose(0, 1, 3, 2)) * tril
            Zr = Kp @ S + Mkk @ U
            P = np.zeros_like(Zr)
            for t in range(chunk):  # forward substitution
                P[:, :, t] = Zr[:, :, t] - np.einsum("bhs,bhsd->bhd", Mka[:, :, t, :t], P[:, :, :t])
            O = Qp @ S + Nqk @ U - Nqa @ P
            y[:, sl] = (z[:, sl].transpose(0, 2, 1, 3) * O).transpose(0, 2, 1, 3)
            gC = gam[:, :, -1:, :]
            S = gC.transpose(0, 1, 3, 2) * S + (K * gC / gam).transpose(0, 1, 3, 2) @ U \
                - (A * gC / gam).transpose(0, 1, 3, 2) @ P
    return y, S
