"""fp64 numpy restatement of the chunked (WY/UT) form of the delta-rule scan.

Test infrastructure: it mirrors, contraction by contraction, what the chunked CUDA kernel
computes per 64-token chunk, so that the algebra the kernel relies on is checked against
the per-token oracle independently of any GPU code. It shares no code with either.

Per chunk with entering state S0 (dv x dk), g_t = cumulative log decay inside the chunk
(scalar for GDN, per key channel for KDA, 0 for DeltaNet), gamma = exp(g):
  Gram      A[t,i] = beta_t (k_t . k_i) gamma_t/gamma_i  (i < t),  P[t,i] = (q_t . k_i) gamma_t/gamma_i (i <= t)
            (KDA: dot products of k_t*gamma_t, q_t*gamma_t with k_i/gamma_i, channel-wise)
  UT        T = (I + A)^{-1} diag(beta)
  project   X = K S0^T (rows scaled by gamma_t; KDA: (K*gamma) S0^T)   Z = Q S0^T (same scaling)
  residual  Y = V - X
  output    O = Z + (P T) Y
  state     S_C^T = diag(gamma_C) S0^T + Khat^T Y,  Khat^T = K^T diag(gamma_C/gamma) T
            (KDA: Khat^T = diag(gamma_C) (K/gamma)^T T)
"""
import numpy as np

DELTANET, GDN, KDA = 1, 2, 3
C = 64


def chunk_scan(q, k, v, beta, gate, S0, mode, chunk=C, return_parts=False):
    """q, k [T,dk]; v [T,dv]; beta [T]; gate [T] (GDN) / [T,dk] (KDA) / None; S0 [dv,dk]."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    out = np.zeros((T, dv))
    parts = []
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        Kc, Qc, Vc, bc = k[t0:t0 + n], q[t0:t0 + n], v[t0:t0 + n], beta[t0:t0 + n]
        if mode == DELTANET:
            g = np.zeros(n)
        elif mode == GDN:
            g = np.cumsum(np.log(gate[t0:t0 + n]))
        else:
            g = np.cumsum(np.log(gate[t0:t0 + n]), axis=0)  # [n, dk]
        gam = np.exp(g)
        if mode == KDA:
            Kg, Qg, Kn = Kc * gam, Qc * gam, Kc / gam
            G = Kg @ Kn.T
            QK = Qg @ Kn.T
            X = Kg @ S.T
            Z = Qg @ S.T
        else:
            dec = np.exp(g[:, None] - g[None, :])
            G = (Kc @ Kc.T) * dec
            QK = (Qc @ Kc.T) * dec
            X = gam[:, None] * (Kc @ S.T)
            Z = gam[:, None] * (Qc @ S.T)
        A = np.tril(G, -1) * bc[:, None]
        P = np.tril(QK)
        Tm = np.linalg.inv(np.eye(n) + A) * bc[None, :]
        Y = Vc - X
        out[t0:t0 + n] = Z + (P @ Tm) @ Y
        if mode == KDA:
            KhT = gam[-1][:, None] * (Kn.T @ Tm)
            S = (S.T * gam[-1][:, None] + KhT @ Y).T
        else:
            KhT = Kc.T @ (np.exp(g[-1] - g)[:, None] * Tm)
            S = (gam[-1] * S.T + KhT @ Y).T
        if return_parts:
            parts.append(dict(A=A, P=P, T=Tm, Y=Y, KhT=KhT, PT=P @ Tm))
    if return_parts:
        return out, S, parts
    return out, S
