"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-type the oracle's recurrence: each compares it with a closed form,
a brute-force definition of a different shape (causal attention, an explicit matrix
inverse, an SVD), an invariant, or a special case that reduces to another routine.
Each names the passage it follows ("Mechanisms, trade-offs and cross-layer routing of
linear-attention architectures" = the linear-attention overview page; "Variational
Linear Attention (VLA)" = the VLA page).
"""
import numpy as np
import pytest

LINEAR, DELTANET, GDN, KDA = 0, 1, 2, 3


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_dr(rng, B, H, T, dk, dv, mode, unit_k=True, s0=True):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    if unit_k:
        q, k = _unit(q), _unit(k)
    v = rng.standard_normal((B, H, T, dv))
    beta = rng.uniform(0.05, 0.95, (B, H, T))
    gate = None
    if mode == GDN:
        gate = rng.uniform(0.5, 1.0, (B, H, T))
    elif mode == KDA:
        gate = rng.uniform(0.5, 1.0, (B, H, T, dk))
    S0 = rng.standard_normal((B, H, dv, dk)) if s0 else None
    return q, k, v, beta, gate, S0


def _rel(x, y):
    return np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300)


# --- plain linear attention: readout after the write, against brute-force causal attention
# VLA page section 2.1 (S_t = S_{t-1} + v_t k_t^T); overview page "Technical details"
# (y = W phi(q)). o_t = S_t q_t = S0 q_t + sum_{i<=t} (q_t.k_i) v_i  => tril_incl(Q K^T) V.
def test_linear_matches_causal_attention(oracle):
    rng = np.random.default_rng(1)
    B, H, T, dk, dv = 2, 3, 37, 8, 5
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    S0 = rng.standard_normal((B, H, dv, dk))
    out, Sf = oracle.dr_scan(q, k, v, S0=S0, mode=LINEAR)
    mask = np.tril(np.ones((T, T)))  # diagonal included: the token's own write is read
    ref = np.einsum("bhts,bhsv->bhtv", np.einsum("bhtd,bhsd->bhts", q, k) * mask, v)
    ref += np.einsum("bhvd,bhtd->bhtv", S0, q)
    assert _rel(out, ref) < 1e-12
    assert _rel(Sf, S0 + np.einsum("bhtv,bhtd->bhvd", v, k)) < 1e-12
    # a readout taken before the write would miss the diagonal term: make sure it matters
    strict = np.einsum("bhts,bhsv->bhtv", np.einsum("bhtd,bhsd->bhts", q, k) * np.tril(mask, -1), v)
    strict += np.einsum("bhvd,bhtd->bhtv", S0, q)
    assert _rel(out, strict) > 1e-2


# --- alpha = 1, beta = 0 leaves S unchanged (bitwise), readout is S0 q_t
@pytest.mark.parametrize("mode", [DELTANET, GDN, KDA])
def test_identity_when_alpha_one_beta_zero(oracle, mode):
    rng = np.random.default_rng(2)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 1, 2, 19, 6, 4, mode)
    beta = np.zeros_like(beta)
    if gate is not None:
        gate = np.ones_like(gate)
    out, Sf = oracle.dr_scan(q, k, v, beta, gate, S0, mode)
    assert np.array_equal(Sf, S0)
    assert _rel(out, np.einsum("bhvd,bhtd->bhtv", S0, q)) < 1e-13


# --- unit k, beta = 1 => S_t k_t = v_t exactly after the write (read with q = k).
# Overview page "Understanding the key idea": the delta rule writes only the residual of
# the memory's prediction. Holds for alpha != 1 only when the residual is taken against
# the decayed state, which is the reading the oracle implements.
@pytest.mark.parametrize("mode", [DELTANET, GDN, KDA])
def test_exact_recall_unit_k_beta_one(oracle, mode):
    rng = np.random.default_rng(3)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 2, 2, 33, 8, 5, mode)
    out, _ = oracle.dr_scan(k, k, v, np.ones_like(beta), gate, S0, mode)
    assert np.max(np.abs(out - v)) < 1e-12
    if mode != DELTANET:
        # the literal reading (residual against the undecayed state) breaks the invariant
        out_lit, _ = oracle.dr_scan(k, k, v, np.ones_like(beta), gate, S0, mode,
                                    residual_pre_decay=True)
        assert np.max(np.abs(out_lit - v)) > 1e-3


# --- GDN with alpha = 1 is DeltaNet; KDA with uniform channels is GDN (bitwise)
def test_gdn_alpha_one_equals_deltanet(oracle):
    rng = np.random.default_rng(4)
    q, k, v, beta, _, S0 = _rand_dr(rng, 2, 2, 29, 8, 6, DELTANET)
    a, sa = oracle.dr_scan(q, k, v, beta, None, S0, DELTANET)
    b, sb = oracle.dr_scan(q, k, v, beta, np.ones(beta.shape), S0, GDN)
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


def test_kda_uniform_channels_equals_gdn(oracle):
    rng = np.random.default_rng(5)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 2, 2, 29, 8, 6, GDN)
    a, sa = oracle.dr_scan(q, k, v, beta, gate, S0, GDN)
    kda_gate = np.repeat(gate[..., None], 8, axis=-1)
    b, sb = oracle.dr_scan(q, k, v, beta, kda_gate, S0, KDA)
    assert np.array_equal(a, b) and np.array_equal(sa, sb)


# --- decay only (beta = 0): S_T = S0 * prod(alpha) -- scalar (GDN) or per key column (KDA)
# Overview page "Technical details": KDA forgets partially along the key-feature dimension.
@pytest.mark.parametrize("mode", [GDN, KDA])
def test_decay_only_closed_form(oracle, mode):
    rng = np.random.default_rng(6)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 1, 3, 23, 6, 6, mode)
    _, Sf = oracle.dr_scan(q, k, v, np.zeros_like(beta), gate, S0, mode)
    prod = np.prod(gate, axis=2)  # GDN [B,H]; KDA [B,H,dk]
    ref = S0 * (prod[..., None, None] if mode == GDN else prod[:, :, None, :])
    assert _rel(Sf, ref) < 1e-13
    if mode == KDA:  # decaying rows (the value axis) instead would be a different answer
        wrong = S0 * prod[:, :, :, None]
        assert _rel(Sf, wrong) > 1e-2


# --- orthonormal keys: every write sees only its own column, giving a closed form with beta
def _orthonormal_rows(rng, n, d):
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    return Qm[:n]


@pytest.mark.parametrize("mode", [DELTANET, GDN])
def test_orthogonal_keys_closed_form(oracle, mode):
    rng = np.random.default_rng(7)
    T, d, dv = 9, 12, 4
    k = _orthonormal_rows(rng, T, d)[None, None]
    q = _unit(rng.standard_normal((1, 1, T, d)))
    v = rng.standard_normal((1, 1, T, dv))
    beta = rng.uniform(0.1, 0.9, (1, 1, T))
    gate = rng.uniform(0.6, 1.0, (1, 1, T)) if mode == GDN else None
    S0 = rng.standard_normal((1, 1, dv, d))
    _, Sf = oracle.dr_scan(q, k, v, beta, gate, S0, mode)
    a = gate[0, 0] if mode == GDN else np.ones(T)
    for j in range(T):
        kj = k[0, 0, j]
        before = np.prod(a[: j + 1])  # decay applied up to and including step j
        after = np.prod(a[j + 1:])
        pred = before * (S0[0, 0] @ kj)
        ref = after * ((1 - beta[0, 0, j]) * pred + beta[0, 0, j] * v[0, 0, j])
        assert np.max(np.abs(Sf[0, 0] @ kj - ref)) < 1e-12


def test_kda_basis_keys_closed_form(oracle):
    rng = np.random.default_rng(8)
    T, d, dv = 7, 10, 3
    chans = rng.permutation(d)[:T]
    k = np.zeros((1, 1, T, d))
    k[0, 0, np.arange(T), chans] = 1.0
    q = _unit(rng.standard_normal((1, 1, T, d)))
    v = rng.standard_normal((1, 1, T, dv))
    beta = rng.uniform(0.1, 0.9, (1, 1, T))
    gate = rng.uniform(0.5, 1.0, (1, 1, T, d))
    S0 = rng.standard_normal((1, 1, dv, d))
    _, Sf = oracle.dr_scan(q, k, v, beta, gate, S0, KDA)
    a = gate[0, 0]
    written = {int(c): j for j, c in enumerate(chans)}
    for c in range(d):
        if c in written:
            j = written[c]
            pred = np.prod(a[: j + 1, c]) * S0[0, 0][:, c]
            ref = np.prod(a[j + 1:, c]) * ((1 - beta[0, 0, j]) * pred + beta[0, 0, j] * v[0, 0, j])
        else:
            ref = np.prod(a[:, c]) * S0[0, 0][:, c]
        assert np.max(np.abs(Sf[0, 0][:, c] - ref)) < 1e-12


# --- capacity: DeltaNet with beta = 1 and n <= d orthonormal keys recalls every value.
# VLA page section 3.2 (d_h associations per head).
def test_capacity_orthonormal_keys_recall(oracle):
    rng = np.random.default_rng(9)
    d, n = 16, 16
    k = _orthonormal_rows(rng, n, d)[None, None]
    v = rng.standard_normal((1, 1, n, 6))
    _, Sf = oracle.dr_scan(k, k, v, np.ones((1, 1, n)), None, None, DELTANET)
    recalled = np.einsum("vd,nd->nv", Sf[0, 0], k[0, 0])
    assert np.max(np.abs(recalled - v[0, 0])) < 1e-12


# --- resumability and head independence
@pytest.mark.parametrize("mode", [LINEAR, DELTANET, GDN, KDA])
def test_state_carry(oracle, mode):
    rng = np.random.default_rng(10)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 2, 2, 40, 6, 5, mode)
    full, Sfull = oracle.dr_scan(q, k, v, beta, gate, S0, mode)
    c = 17
    g1 = None if gate is None else gate[:, :, :c]
    g2 = None if gate is None else gate[:, :, c:]
    o1, S1 = oracle.dr_scan(q[:, :, :c], k[:, :, :c], v[:, :, :c], beta[:, :, :c], g1, S0, mode)
    o2, S2 = oracle.dr_scan(q[:, :, c:], k[:, :, c:], v[:, :, c:], beta[:, :, c:], g2, S1, mode)
    assert np.array_equal(np.concatenate([o1, o2], axis=2), full)
    assert np.array_equal(S2, Sfull)


def test_head_permutation(oracle):
    rng = np.random.default_rng(11)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 1, 5, 21, 6, 4, KDA)
    out, Sf = oracle.dr_scan(q, k, v, beta, gate, S0, KDA)
    p = np.array([3, 0, 4, 1, 2])
    out_p, Sf_p = oracle.dr_scan(q[:, p], k[:, p], v[:, p], beta[:, p], gate[:, p], S0[:, p], KDA)
    assert np.array_equal(out_p, out[:, p]) and np.array_equal(Sf_p, Sf[:, p])


def test_empty_sequence(oracle):
    rng = np.random.default_rng(12)
    q, k, v, beta, gate, S0 = _rand_dr(rng, 1, 2, 0, 4, 4, GDN)
    out, Sf = oracle.dr_scan(q, k, v, beta, gate, S0, GDN)
    assert out.shape == (1, 2, 0, 4) and np.array_equal(Sf, S0)


# --- VLA (Variational Linear Attention page, sections 2.2-2.3, 3.1)
def _rand_vla(rng, B, H, T, d, u_scale=1.0):
    q = _unit(rng.standard_normal((B, H, T, d)))
    k = _unit(rng.standard_normal((B, H, T, d)))
    v = rng.standard_normal((B, H, T, d))
    u = u_scale * rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    return q, k, v, u


@pytest.mark.parametrize("lam", [1.0, 0.25])
def test_sherman_morrison_matches_explicit_inverse(oracle, lam):
    rng = np.random.default_rng(13)
    d = 6
    q, k, v, u = _rand_vla(rng, 1, 2, 50, d, u_scale=2.0)
    for T in (1, 7, 50):
        _, _, Af = oracle.vla_scan(q[:, :, :T], k[:, :, :T], v[:, :, :T], u[:, :, :T], lambda0=lam)
        for h in range(2):
            M = lam * np.eye(d) + u[0, h, :T].T @ u[0, h, :T]
            assert _rel(Af[0, h], np.linalg.inv(M)) < 1e-12


def test_vla_single_step_from_zero(oracle):
    rng = np.random.default_rng(14)
    d = 8
    q, k, v, u = _rand_vla(rng, 1, 1, 1, d)
    _, Sf, _ = oracle.vla_scan(q, k, v, u, lambda0=0.5)
    A1 = np.linalg.inv(0.5 * np.eye(d) + np.outer(u[0, 0, 0], u[0, 0, 0]))
    a = A1 @ k[0, 0, 0]
    a /= np.linalg.norm(a)
    assert _rel(Sf[0, 0], np.outer(v[0, 0, 0], a)) < 1e-12


def _vla_step_jacobian(oracle, k1, u1, lam):
    """Extract the map S0 -> S1 (v = 0) from the oracle, one basis matrix at a time."""
    d = k1.size
    rows = []
    for b in range(d):
        S0 = np.zeros((1, 1, d, d))
        S0[0, 0, 0, b] = 1.0
        z = np.zeros((1, 1, 1, d))
        _, S1, _ = oracle.vla_scan(z, k1[None, None, None], z, u1[None, None, None], S0=S0,
                                   lambda0=lam)
        rows.append(S1[0, 0, 0])
    return np.array(rows)  # row b = e_b^T J  => J = I - k alpha^T


def test_vla_jacobian_spectral_norm(oracle):
    # Section 3.1 Proposition 2 states ||I - alpha k^T||_2 = 1; as garbled on the page this
    # holds only when alpha = k. For unit vectors with c = alpha.k the exact value is
    # sqrt((3 - 2c + sqrt((3-2c)^2 - 4(1-c)^2)) / 2) >= 1.
    rng = np.random.default_rng(15)
    d = 7
    for trial in range(5):
        k1 = _unit(rng.standard_normal(d))
        u1 = rng.standard_normal(d) * (0.0 if trial == 0 else 1.5)
        J = _vla_step_jacobian(oracle, k1, u1, 1.0)
        A1 = np.linalg.inv(np.eye(d) + np.outer(u1, u1))
        a = A1 @ k1
        a /= np.linalg.norm(a)
        c = float(a @ k1)
        closed = np.sqrt((3 - 2 * c + np.sqrt((3 - 2 * c) ** 2 - 4 * (1 - c) ** 2)) / 2)
        norm = np.linalg.norm(J, 2)
        assert abs(norm - closed) < 1e-10
        assert np.max(np.abs(J - (np.eye(d) - np.outer(k1, a)))) < 1e-12
        if trial == 0:
            assert abs(norm - 1.0) < 1e-12  # alpha = k when A is a multiple of I
        else:
            assert norm >= 1.0 - 1e-12


def test_vla_with_u_zero_is_deltanet_beta_one(oracle):
    rng = np.random.default_rng(16)
    q, k, v, u = _rand_vla(rng, 2, 2, 31, 6)
    S0 = rng.standard_normal((2, 2, 6, 6))
    out, Sf, Af = oracle.vla_scan(q, k, v, np.zeros_like(u), S0=S0, lambda0=2.0)
    ref, Sref = oracle.dr_scan(q, k, v, np.ones(q.shape[:3]), None, S0, DELTANET)
    assert _rel(out, ref) < 1e-12 and _rel(Sf, Sref) < 1e-12
    assert np.array_equal(Af, np.broadcast_to(np.eye(6) / 2.0, Af.shape))


def test_vla_state_carry(oracle):
    rng = np.random.default_rng(17)
    q, k, v, u = _rand_vla(rng, 1, 3, 30, 5)
    full, Sfull, Afull = oracle.vla_scan(q, k, v, u, lambda0=1.0)
    c = 11
    o1, S1, A1 = oracle.vla_scan(q[:, :, :c], k[:, :, :c], v[:, :, :c], u[:, :, :c], lambda0=1.0)
    o2, S2, A2 = oracle.vla_scan(q[:, :, c:], k[:, :, c:], v[:, :, c:], u[:, :, c:], S0=S1, A0=A1)
    assert np.array_equal(np.concatenate([o1, o2], axis=2), full)
    assert np.array_equal(S2, Sfull) and np.array_equal(A2, Afull)


def test_vla_bounded_state_soft(oracle):
    # Section 3.1 Proposition 1 (soft check, not a parity pin): the VLA state stays O(d)
    # while plain accumulation grows with T.
    rng = np.random.default_rng(18)
    d, T = 16, 1000
    q, k, v, u = _rand_vla(rng, 1, 1, T, d)
    _, Sf, _ = oracle.vla_scan(q, k, v, u, lambda0=1.0)
    _, Slin = oracle.dr_scan(q, k, v, None, None, None, LINEAR)
    assert np.linalg.norm(Sf[0, 0]) < 10 * d
    assert np.linalg.norm(Slin[0, 0]) > 3 * np.linalg.norm(Sf[0, 0])


# ====================================================================================
# Gated DeltaNet-2 and the per-token write values (the routed signal of the cross-layer
# routing passages). Overview page, sections "Methodology" and "Technical details":
# Gated DeltaNet-2 separates a per-key-channel erase gate b and a per-value-channel write
# gate w, with e = b (.) kappa, z = w (.) v and the residual r = z - W~ e; the reading
# taken: W~ = alpha S_{t-1}, S_t = W~ + beta r e^T. The write value of a token is
# u_t = beta_t r_t (what the step adds along its key); plain linear attention writes v_t.
# ====================================================================================
GDN2 = 4


def _rand_gdn2(rng, B, H, T, dk, dv):
    q, k, v, beta, gate, S0 = _rand_dr(rng, B, H, T, dk, dv, GDN)
    erase = rng.uniform(0.1, 1.0, (B, H, T, dk))
    write = rng.uniform(0.1, 1.0, (B, H, T, dv))
    return q, k, v, beta, gate, S0, erase, write


def test_gdn2_with_unit_gates_is_gated_deltanet(oracle):
    rng = np.random.default_rng(40)
    q, k, v, beta, gate, S0, _, _ = _rand_gdn2(rng, 2, 2, 33, 6, 5)
    out, Sf, _ = oracle.dr_scan_ex(q, k, v, beta, gate, S0, GDN2, erase=np.ones_like(k),
                                   write=np.ones_like(v))
    ref_out, ref_S = oracle.dr_scan(q, k, v, beta, gate, S0, GDN)
    assert np.array_equal(out, ref_out) and np.array_equal(Sf, ref_S)


def test_gdn2_recalls_the_write_target_along_a_unit_erase_direction(oracle):
    # beta = 1 and a unit e_t = b_t (.) k_t: after the write, S_t e_t = z_t = w_t (.) v_t
    # exactly, whatever the decay (read back with q_t = e_t)
    rng = np.random.default_rng(41)
    B, H, T, dk, dv = 1, 2, 12, 6, 4
    q, k, v, beta, gate, S0, erase, write = _rand_gdn2(rng, B, H, T, dk, dv)
    e = _unit(rng.standard_normal((B, H, T, dk)))
    k = e / erase  # so that b (.) k = e
    out, _, _ = oracle.dr_scan_ex(e, k, v, np.ones_like(beta), gate, S0, GDN2, erase=erase,
                                  write=write)
    assert _rel(out, write * v) < 1e-12
    # the same with the write gate ignored would recall v instead
    assert _rel(write * v, v) > 1e-1


def test_gdn2_without_erase_only_decays(oracle):
    # b = 0: e = 0, nothing is read or written; S_T = (prod alpha) S0 and every write value
    # is beta_t z_t (the whole target, with nothing predicted)
    rng = np.random.default_rng(42)
    q, k, v, beta, gate, S0, _, write = _rand_gdn2(rng, 1, 3, 15, 5, 4)
    out, Sf, u = oracle.dr_scan_ex(q, k, v, beta, gate, S0, GDN2, erase=np.zeros_like(k),
                                   write=write)
    decay = np.prod(gate, axis=-1)[..., None, None]
    assert _rel(Sf, decay * S0) < 1e-13
    assert _rel(u, beta[..., None] * write * v) < 1e-13


def test_gdn2_key_channels_without_erase_are_never_written(oracle):
    # the erase gate is per key channel: a channel with b = 0 at every step keeps only its
    # decayed initial column, whatever the keys and values
    rng = np.random.default_rng(43)
    q, k, v, beta, gate, S0, erase, write = _rand_gdn2(rng, 2, 1, 21, 7, 3)
    off = [1, 4]
    erase[..., off] = 0.0
    _, Sf, _ = oracle.dr_scan_ex(q, k, v, beta, gate, S0, GDN2, erase=erase, write=write)
    decay = np.prod(gate, axis=-1)[..., None, None]
    assert _rel(Sf[..., off], decay * S0[..., off]) < 1e-13
    on = [0, 2, 3, 5, 6]
    assert _rel(Sf[..., on], decay * S0[..., on]) > 1e-2


def test_gdn2_zero_write_gate_erases_along_e(oracle):
    # w = 0, beta = 1, unit e: the write removes what the memory holds along e, S_t e_t = 0
    rng = np.random.default_rng(44)
    B, H, T, dk, dv = 1, 1, 9, 5, 3
    q, k, v, beta, gate, S0, erase, write = _rand_gdn2(rng, B, H, T, dk, dv)
    e = _unit(rng.standard_normal((B, H, T, dk)))
    out, _, _ = oracle.dr_scan_ex(e, e / erase, v, np.ones_like(beta), gate, S0, GDN2,
                                  erase=erase, write=np.zeros_like(write))
    assert np.max(np.abs(out)) < 1e-13


@pytest.mark.parametrize("mode", [LINEAR, DELTANET, GDN, KDA, GDN2])
def test_write_values_rebuild_the_final_state(oracle, mode):
    # every step is S_t = S_{t-1} diag(a_t) + u_t key_t^T, so the exported write values and
    # the decays alone rebuild S_T:  S_T = S0 diag(prod_t a_t) + sum_t u_t key_t^T
    # diag(prod_{s>t} a_s)   (key = e = b (.) k for Gated DeltaNet-2, k otherwise)
    rng = np.random.default_rng(45 + mode)
    B, H, T, dk, dv = 2, 2, 17, 6, 4
    if mode == GDN2:
        q, k, v, beta, gate, S0, erase, write = _rand_gdn2(rng, B, H, T, dk, dv)
    else:
        q, k, v, beta, gate, S0 = _rand_dr(rng, B, H, T, dk, dv, mode)
        erase = write = None
    _, Sf, u = oracle.dr_scan_ex(q, k, v, beta, gate, S0, mode, erase=erase, write=write)
    if mode in (LINEAR, DELTANET):
        a = np.ones((B, H, T, dk))
    elif mode in (GDN, GDN2):
        a = np.repeat(gate[..., None], dk, axis=-1)
    else:
        a = gate
    key = erase * k if mode == GDN2 else k
    after = np.ones_like(a)  # prod_{s>t} a_s per key channel
    for t in range(T - 2, -1, -1):
        after[:, :, t] = after[:, :, t + 1] * a[:, :, t + 1]
    total = after[:, :, 0] * a[:, :, 0]
    rebuilt = S0 * total[:, :, None, :] + np.einsum("bhtv,bhtd->bhvd", u, key * after)
    assert _rel(Sf, rebuilt) < 1e-12
    if mode == LINEAR:
        assert np.array_equal(u, v)


@pytest.mark.parametrize("mode", [DELTANET, GDN, KDA, GDN2])
def test_first_write_value_from_a_zero_state(oracle, mode):
    # with S0 = 0 the first prediction is zero: u_0 = beta_0 v_0 (beta_0 w_0 (.) v_0 for GDN-2)
    rng = np.random.default_rng(50 + mode)
    if mode == GDN2:
        q, k, v, beta, gate, _, erase, write = _rand_gdn2(rng, 1, 2, 3, 4, 5)
    else:
        q, k, v, beta, gate, _ = _rand_dr(rng, 1, 2, 3, 4, 5, mode)
        erase = write = None
    _, _, u = oracle.dr_scan_ex(q, k, v, beta, gate, None, mode, erase=erase, write=write)
    target = write * v if mode == GDN2 else v
    assert _rel(u[:, :, 0], beta[:, :, 0, None] * target[:, :, 0]) < 1e-15


# ====================================================================================
# VLA ratio readout. VLA page, section 2.3: the output is computed as a ratio of
# recurrences, as in standard linear attention, with an ELU+1 feature map. Reading taken:
# the denominator is the same write applied to one more value channel held at 1,
# n_t = n_{t-1} + (1 - n_{t-1} k_t) alpha_hat_t^T, and o_t = S_t q_t / (n_t q_t), with q
# the feature-mapped query and k the unit-norm feature-mapped key (the caller's feature map).
# ====================================================================================
def _elu1(x):
    return np.where(x > 0, x + 1.0, np.exp(x))


def test_vla_ratio_with_basis_keys_is_normalised_linear_attention(oracle):
    # u = 0 keeps A = I / lambda0, so alpha_hat = k; with distinct basis keys every write
    # lands in a fresh direction: S_t = sum_{s<=t} v_s k_s^T and n_t = sum_{s<=t} k_s^T, and
    # the ratio readout is causal linear attention normalised by its own weights (brute force)
    rng = np.random.default_rng(60)
    B, H, d = 1, 3, 8
    T = d
    k = np.zeros((B, H, T, d))
    for h in range(H):
        k[0, h, np.arange(T), rng.permutation(d)] = 1.0
    q = _elu1(rng.standard_normal((B, H, T, d)))
    v = rng.standard_normal((B, H, T, d))
    out, _, _, nf = oracle.vla_scan_ratio(q, k, v, np.zeros_like(v), lambda0=2.0)
    w = np.einsum("bhtd,bhsd->bhts", q, k) * np.tril(np.ones((T, T)))
    ref = np.einsum("bhts,bhsv->bhtv", w, v) / w.sum(-1, keepdims=True)
    assert _rel(out, ref) < 1e-13
    assert _rel(nf, k.sum(2)) < 1e-15


def test_vla_ratio_reads_back_a_constant_value(oracle):
    # when every value is the same vector c (and S0 = c n0^T), S and n follow one recurrence,
    # S_t = c n_t, so every output is exactly c, whatever u, k and q
    rng = np.random.default_rng(61)
    B, H, T, d = 2, 2, 40, 6
    q = _elu1(rng.standard_normal((B, H, T, d)))
    k = _unit(_elu1(rng.standard_normal((B, H, T, d))))
    u = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    c = rng.standard_normal((B, H, d))
    v = np.broadcast_to(c[:, :, None, :], (B, H, T, d)).copy()
    n0 = np.abs(rng.standard_normal((B, H, d)))
    S0 = np.einsum("bhi,bhj->bhij", c, n0)
    out, Sf, _, nf = oracle.vla_scan_ratio(q, k, v, u, S0=S0, n0=n0)
    assert _rel(out, v) < 1e-10
    assert _rel(Sf, np.einsum("bhi,bhj->bhij", c, nf)) < 1e-10


def test_vla_ratio_numerator_is_the_plain_readout(oracle):
    # S and A follow the same recurrence under either readout; the ratio output times the
    # denominator n_t q_t is the plain readout S_t q_t
    rng = np.random.default_rng(62)
    B, H, T, d = 1, 2, 30, 5
    q = _elu1(rng.standard_normal((B, H, T, d)))
    k = _unit(_elu1(rng.standard_normal((B, H, T, d))))
    v = rng.standard_normal((B, H, T, d))
    u = rng.standard_normal((B, H, T, d)) / np.sqrt(d)
    plain, S1, A1 = oracle.vla_scan(q, k, v, u)
    ratio, S2, A2, _ = oracle.vla_scan_ratio(q, k, v, u)
    assert np.array_equal(S1, S2) and np.array_equal(A1, A2)
    # scaling q by a positive number leaves the ratio unchanged but scales the plain readout
    ratio3, _, _, _ = oracle.vla_scan_ratio(3.0 * q, k, v, u)
    assert _rel(ratio3, ratio) < 1e-12
    assert _rel(plain / ratio, np.broadcast_to((plain / ratio)[..., :1], plain.shape)) < 1e-9


# ====================================================================================
# Log-linear attention over a Fenwick hierarchy ("Adaptive memory decay for log-linear
# attention", problem definition and method sections): the prefix [0, t] is split into the
# token itself (level 0) and one block of 2^b earlier tokens per set bit b of t (level b + 1);
# the output is the lambda_t-weighted sum of the levels' linear-attention readouts. The
# oracle keeps the levels as a binary counter; these pins compare it with the pair-wise
# masked form, whose level of (t, s < t) is the bit length of t XOR s.
# ====================================================================================
def _loglinear_inputs(rng, B, H, T, dk, dv):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    L = oracle_levels(T)
    lam = np.log1p(np.exp(0.54 + 0.5 * rng.standard_normal((B, H, T, L))))  # softplus
    return q, k, v, lam


def oracle_levels(T):
    return max(1, int(T - 1).bit_length() + 1)


@pytest.mark.parametrize("T", [1, 2, 7, 64, 100])
def test_loglinear_matches_the_masked_pairwise_form(oracle, T):
    rng = np.random.default_rng(70 + T)
    B, H, dk, dv = 1, 2, 5, 3
    q, k, v, lam = _loglinear_inputs(rng, B, H, T, dk, dv)
    assert oracle.loglinear_levels(T) == lam.shape[-1]
    out = oracle.loglinear_scan(q, k, v, lam)
    t = np.arange(T)[:, None]
    s = np.arange(T)[None, :]
    level = np.vectorize(lambda a, b: int(a ^ b).bit_length())(t, s)  # 0 on the diagonal
    weight = np.take_along_axis(lam, np.broadcast_to(level, (B, H, T, T)), axis=-1)
    weight = weight * (s <= t)
    ref = np.einsum("bhts,bhsv->bhtv", weight * np.einsum("bhtd,bhsd->bhts", q, k), v)
    assert _rel(out, ref) < 1e-12


def test_loglinear_with_unit_weights_is_linear_attention(oracle):
    # lambda = 1 on every level: the levels partition the prefix, so the scan is causal
    # linear attention (and the oracle's plain accumulation from a zero state)
    rng = np.random.default_rng(75)
    B, H, T, dk, dv = 2, 2, 45, 4, 6
    q, k, v, lam = _loglinear_inputs(rng, B, H, T, dk, dv)
    out = oracle.loglinear_scan(q, k, v, np.ones_like(lam))
    ref = np.einsum("bhts,bhsv->bhtv", np.einsum("bhtd,bhsd->bhts", q, k) * np.tril(np.ones((T, T))), v)
    assert _rel(out, ref) < 1e-12
    lin, _ = oracle.dr_scan(q, k, v, mode=LINEAR)
    assert _rel(out, lin) < 1e-12


@pytest.mark.parametrize("level", [0, 1, 2, 3, 5])
def test_loglinear_one_level_reads_one_fenwick_block(oracle, level):
    # weights on one level only: level 0 is the token itself; level b + 1 is the block
    # [hi 2^(b+1), hi 2^(b+1) + 2^b) with hi = t >> (b+1), present when bit b of t is set
    rng = np.random.default_rng(80 + level)
    B, H, T, dk, dv = 1, 1, 50, 3, 2
    q, k, v, lam = _loglinear_inputs(rng, B, H, T, dk, dv)
    one = np.zeros_like(lam)
    one[..., level] = 1.0
    out = oracle.loglinear_scan(q, k, v, one)
    ref = np.zeros_like(out)
    for t in range(T):
        if level == 0:
            block = [t]
        else:
            b = level - 1
            if not (t >> b) & 1:
                continue
            lo = (t >> (b + 1)) << (b + 1)
            block = list(range(lo, lo + (1 << b)))
            assert all(s < t for s in block)
        for s in block:
            ref[:, :, t] += (q[:, :, t] * k[:, :, s]).sum(-1)[..., None] * v[:, :, s]
    assert _rel(out, ref) < 1e-12 if np.any(ref) else np.max(np.abs(out)) == 0.0


def test_loglinear_worked_example(oracle):
    # d = 1, T = 4, lambda_t = (1, 1/2, 1/4) for levels 0, 1, 2:
    # t=0: {0} -> 1 (q0 k0) v0 = 2
    # t=1 (01): {1} + level 1 {0} -> (2*1)*2 + 1/2 (2*2)*1 = 6
    # t=2 (10): {2} + level 2 {0,1} -> (1*1)*4 + 1/4 ((1*2)*1 + (1*1)*2) = 5
    # t=3 (11): {3} + level 1 {2} + level 2 {0,1} -> (1/2*2)*8 + 1/2 (1/2*1)*4
    #           + 1/4 ((1/2*2)*1 + (1/2*1)*2) = 9.5
    q = np.array([1, 2, 1, 0.5])[None, None, :, None]
    k = np.array([2, 1, 1, 2])[None, None, :, None]
    v = np.array([1, 2, 4, 8])[None, None, :, None]
    lam = np.broadcast_to(np.array([1, 0.5, 0.25]), (1, 1, 4, 3))
    out = oracle.loglinear_scan(q, k, v, lam)
    assert np.array_equal(out[0, 0, :, 0], [2, 6, 5, 9.5])
