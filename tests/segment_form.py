"""fp64 numpy restatement of a parallel scan over chunk transitions (test infrastructure).

With the chunk quantities of ``chunk_form`` (Gram, UT transform T, PT, Khat^T, decays), one
chunk acts on the transposed state S^T (dk x dv) affinely:

    S^T_c = M_c S^T_{c-1} + b_c,     M_c = D_c - Khat_c^T Kg_c,   b_c = Khat_c^T V_c
    O_c   = E_c S^T_{c-1} + f_c,     E_c = Qg_c - (P T)_c Kg_c,   f_c = (P T)_c V_c

where Kg, Qg are K, Q with rows scaled by gamma_t (KDA: channel-wise), and D_c = gamma_C I
(KDA: diag(gamma_C)). So contiguous segments of chunks can run from a zero state in
parallel while accumulating their transition products. A serial combine over the segments
then gives every segment's true entering state:

    S^T_in(g+1) = Phi_g S^T_in(g) + Z_g,   Phi_g = product of the segment's M_c,
    Z_g = the segment's end state from zero.

Each segment's outputs follow either from a replay from S^T_in(g) (two passes) or from a
correction of its zero-state outputs by the prefix products:

    O_c = O^0_c + E_c Pi_{c-1} S^T_in(g).

It shares no code with the oracle or the CUDA library.
"""
import numpy as np

from chunk_form import DELTANET, KDA, chunk_scan

C = 64


def chunk_affine(q, k, v, beta, gate, mode, chunk=C):
    """Per chunk: (M, b, E, f), the state-independent affine maps above."""
    T, dk = q.shape
    maps = []
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        Kc, Qc, Vc, bc = k[t0:t0 + n], q[t0:t0 + n], v[t0:t0 + n], beta[t0:t0 + n]
        if mode == DELTANET:
            g = np.zeros(n)
        elif mode == KDA:
            g = np.cumsum(np.log(gate[t0:t0 + n]), axis=0)
        else:
            g = np.cumsum(np.log(gate[t0:t0 + n]))
        gam = np.exp(g)
        if mode == KDA:
            Kg, Qg, Kn = Kc * gam, Qc * gam, Kc / gam
            G, QK = Kg @ Kn.T, Qg @ Kn.T
            D = np.diag(gam[-1])
        else:
            dec = np.exp(g[:, None] - g[None, :])
            G, QK = (Kc @ Kc.T) * dec, (Qc @ Kc.T) * dec
            Kg, Qg = gam[:, None] * Kc, gam[:, None] * Qc
            D = gam[-1] * np.eye(dk)
        A = np.tril(G, -1) * bc[:, None]
        Tm = np.linalg.inv(np.eye(n) + A) * bc[None, :]
        PT = np.tril(QK) @ Tm
        KhT = gam[-1][:, None] * (Kn.T @ Tm) if mode == KDA else Kc.T @ (np.exp(g[-1] - g)[:, None] * Tm)
        maps.append((D - KhT @ Kg, KhT @ Vc, Qg - PT @ Kg, PT @ Vc))
    return maps


def segment_scan(q, k, v, beta, gate, S0, mode, bounds, chunk=C, replay=False):
    """Scan split into segments of chunks [bounds[i], bounds[i+1]). Returns (out, S_final,
    entering), where entering lists every segment's entering state (dv x dk). replay=True
    recomputes each segment's outputs with chunk_scan from its entering state instead of
    correcting the zero-state outputs."""
    T, dk = q.shape
    dv = v.shape[1]
    maps = chunk_affine(q, k, v, beta, gate, mode, chunk)
    # pass 1, independent per segment: zero-state outputs, prefix products, segment totals
    seg = []
    for s0, s1 in zip(bounds[:-1], bounds[1:]):
        Z, Pi = np.zeros((dk, dv)), np.eye(dk)
        O0, corr = [], []
        for c in range(s0, s1):
            M, b, E, f = maps[c]
            O0.append(E @ Z + f)
            corr.append(E @ Pi)          # maps the segment's entering state to this chunk's output
            Z, Pi = M @ Z + b, M @ Pi
        seg.append((O0, corr, Pi, Z))
    # serial combine over segments
    ST = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64).T
    entering = []
    for _, _, Phi, Z in seg:
        entering.append(ST)
        ST = Phi @ ST + Z
    # pass 2, independent per segment
    out = np.zeros((T, dv))
    for (s0, s1), (O0, corr, _, _), Sin in zip(zip(bounds[:-1], bounds[1:]), seg, entering):
        t0, t1 = s0 * chunk, min(s1 * chunk, T)
        if replay:
            sl = slice(t0, t1)
            g = None if gate is None else gate[sl]
            out[sl], _ = chunk_scan(q[sl], k[sl], v[sl], beta[sl], g, Sin.T, mode, chunk)
        else:
            for i, c in enumerate(range(s0, s1)):
                n = min(chunk, T - c * chunk)
                out[c * chunk:c * chunk + n] = O0[i] + corr[i] @ Sin
    return out, ST.T, [S.T for S in entering]
