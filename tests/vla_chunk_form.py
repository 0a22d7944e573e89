"""fp64 numpy restatement of the chunked form of the VLA scan that the two CUDA kernels
(A-phase, S-phase) compute per 64-token chunk.

Test infrastructure: it follows the kernels' steps contraction by contraction so that the
algebra they rely on is checked against the per-token oracle with no GPU code involved. It
shares no code with either.

A-phase, chunk entering with the inverse penalty A_c (Woodbury identity over the chunk's
Sherman-Morrison steps):
  M   = I + U A_c U^T = L L^T                 (Cholesky; M >= I for a positive definite A_c)
  W   = L^-1 (U A_c)                          (row t depends on rows <= t of U only)
  Y   = K A_c - tril(K W^T) W                 (row t is A_t k_t)
  alpha_hat_t = Y_t / ||Y_t||,   A_{c+1} = A_c - W^T W
S-phase, chunk entering with S_c (delta rule with read key k_t and write key alpha_hat_t):
  (I + strict_tril(K Alpha^T)) R = V - K S_c^T
  O = Q S_c^T + tril(Q Alpha^T) R,   S_{c+1} = S_c + R^T Alpha
Ratio readout: n is one more row of S whose value is 1 at every token; out = O / (n_t q_t).
"""
import numpy as np

C = 64


def _forward_substitution(L, B):
    """Solve L X = B for lower-triangular L, row by row (the kernels' order)."""
    X = np.array(B, dtype=np.float64)
    for t in range(L.shape[0]):
        X[t] = (X[t] - L[t, :t] @ X[:t]) / L[t, t]
    return X


def _cholesky(M):
    n = M.shape[0]
    L = np.zeros_like(M)
    for j in range(n):
        d = M[j, j] - L[j, :j] @ L[j, :j]
        L[j, j] = np.sqrt(d)
        L[j + 1:, j] = (M[j + 1:, j] - L[j + 1:, :j] @ L[j, :j]) / L[j, j]
    return L


def vla_chunk_scan(q, k, v, u, S0=None, A0=None, n0=None, lambda0=1.0, ratio=False, chunk=C):
    """q, k, v, u [T,d] (one head). Returns (out [T,d], S_final, A_final, n_final)."""
    T, d = q.shape
    A = np.eye(d) / lambda0 if A0 is None else np.array(A0, dtype=np.float64)
    S = np.zeros((d, d)) if S0 is None else np.array(S0, dtype=np.float64)
    n = np.zeros(d) if n0 is None else np.array(n0, dtype=np.float64)
    out = np.zeros((T, d))
    for t0 in range(0, T, chunk):
        m = min(chunk, T - t0)
        Uc, Kc, Qc, Vc = u[t0:t0 + m], k[t0:t0 + m], q[t0:t0 + m], v[t0:t0 + m]
        # A-phase
        UA, KA = Uc @ A, Kc @ A
        L = _cholesky(np.eye(m) + Uc @ UA.T)
        W = _forward_substitution(L, UA)
        Y = KA - np.tril(Kc @ W.T) @ W
        Al = Y / np.linalg.norm(Y, axis=1, keepdims=True)
        A = A - W.T @ W
        # S-phase
        G = np.tril(Kc @ Al.T, -1)
        P = np.tril(Qc @ Al.T)
        unit_l = np.eye(m) + G
        R = _forward_substitution(unit_l, Vc - Kc @ S.T)
        O = Qc @ S.T + P @ R
        if ratio:
            rn = _forward_substitution(unit_l, (1.0 - Kc @ n)[:, None])[:, 0]
            O = O / (Qc @ n + P @ rn)[:, None]
            n = n + rn @ Al
        S = S + R.T @ Al
        out[t0:t0 + m] = O
    return out, S, A, n
