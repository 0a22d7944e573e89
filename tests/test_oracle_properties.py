"""Property-based pins of the fp64 oracle: the structural pins of test_oracle_pins.py over
random small shapes, sequence lengths (including 0), split points, seeds and variants.

Sources: "Mechanisms, trade-offs and cross-layer routing of linear-attention
architectures" (the overview page), section "Technical details" (delta rule, scalar and
per-key-channel decay); "Variational Linear Attention (VLA)", sections 2.1-2.3.
"""
import numpy as np
import pytest

hyp = pytest.importorskip("hypothesis")
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

LINEAR, DELTANET, GDN, KDA = 0, 1, 2, 3
SETTINGS = settings(max_examples=25, deadline=None, derandomize=True, database=None)

shapes = st.tuples(st.integers(1, 2), st.integers(0, 12), st.integers(1, 6), st.integers(1, 6),
                   st.integers(0, 2**31 - 1))  # H, T, dk, dv, seed


def draw(seed, H, T, dk, dv, mode):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, H, T, dk))
    k = rng.standard_normal((1, H, T, dk))
    k /= np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), 1e-12)
    v = rng.standard_normal((1, H, T, dv))
    beta = rng.uniform(0.05, 0.95, (1, H, T))
    gate = None
    if mode == GDN:
        gate = rng.uniform(0.3, 1.0, (1, H, T))
    elif mode == KDA:
        gate = rng.uniform(0.3, 1.0, (1, H, T, dk))
    S0 = rng.standard_normal((1, H, dv, dk))
    return q, k, v, beta, gate, S0


def rel(x, y):
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-300)) if y.size else 0.0


@SETTINGS
@given(shapes)
def test_linear_is_causal_attention_with_the_diagonal(oracle, shape):
    # VLA page section 2.1: S_t = S_{t-1} + v_t k_t^T, read out after the write
    H, T, dk, dv, seed = shape
    q, k, v, _, _, S0 = draw(seed, H, T, dk, dv, LINEAR)
    out, Sf = oracle.dr_scan(q, k, v, S0=S0, mode=LINEAR)
    mask = np.tril(np.ones((T, T)))
    ref = np.einsum("bhts,bhsv->bhtv", np.einsum("bhtd,bhsd->bhts", q, k) * mask, v)
    ref += np.einsum("bhvd,bhtd->bhtv", S0, q)
    assert rel(out, ref) < 1e-12
    assert rel(Sf, S0 + np.einsum("bhtv,bhtd->bhvd", v, k)) < 1e-12


@SETTINGS
@given(shapes, st.sampled_from([LINEAR, DELTANET, GDN, KDA]), st.floats(0.0, 1.0))
def test_any_split_carries_the_state_exactly(oracle, shape, mode, frac):
    H, T, dk, dv, seed = shape
    q, k, v, beta, gate, S0 = draw(seed, H, T, dk, dv, mode)
    c = int(round(frac * T))
    full, Sfull = oracle.dr_scan(q, k, v, beta, gate, S0, mode)
    part = lambda x, s: None if x is None else np.ascontiguousarray(x[:, :, s])
    o1, S1 = oracle.dr_scan(part(q, slice(0, c)), part(k, slice(0, c)), part(v, slice(0, c)),
                            part(beta, slice(0, c)), part(gate, slice(0, c)), S0, mode)
    o2, S2 = oracle.dr_scan(part(q, slice(c, T)), part(k, slice(c, T)), part(v, slice(c, T)),
                            part(beta, slice(c, T)), part(gate, slice(c, T)), S1, mode)
    assert np.array_equal(np.concatenate([o1, o2], axis=2), full)
    assert np.array_equal(S2, Sfull)


@SETTINGS
@given(shapes)
def test_variants_reduce_to_one_another(oracle, shape):
    # overview page "Technical details": GDN with alpha = 1 is DeltaNet; KDA with the same
    # alpha on every key channel is GDN
    H, T, dk, dv, seed = shape
    q, k, v, beta, gate, S0 = draw(seed, H, T, dk, dv, GDN)
    dn, Sdn = oracle.dr_scan(q, k, v, beta, None, S0, DELTANET)
    g1, Sg1 = oracle.dr_scan(q, k, v, beta, np.ones_like(gate), S0, GDN)
    assert np.array_equal(dn, g1) and np.array_equal(Sdn, Sg1)
    g, Sg = oracle.dr_scan(q, k, v, beta, gate, S0, GDN)
    kda_gate = np.repeat(gate[..., None], dk, axis=-1)
    kd, Skd = oracle.dr_scan(q, k, v, beta, kda_gate, S0, KDA)
    assert np.array_equal(g, kd) and np.array_equal(Sg, Skd)


@SETTINGS
@given(shapes, st.sampled_from([DELTANET, GDN, KDA]))
def test_unit_key_full_write_recalls_the_value(oracle, shape, mode):
    # the delta rule writes only the residual: with |k| = 1 and beta = 1 the state maps the
    # token's key to its value exactly after the write, whatever it held before
    H, T, dk, dv, seed = shape
    T = max(T, 1)
    q, k, v, beta, gate, S0 = draw(seed, H, T, dk, dv, mode)
    for t in range(1, T + 1):
        sl = slice(0, t)
        g = None if gate is None else gate[:, :, sl]
        _, S = oracle.dr_scan(q[:, :, sl], k[:, :, sl], v[:, :, sl], np.ones_like(beta[:, :, sl]),
                              g, S0, mode)
        recall = np.einsum("bhvd,bhd->bhv", S, k[:, :, t - 1])
        assert rel(recall, v[:, :, t - 1]) < 1e-10


@SETTINGS
@given(st.integers(1, 5), st.integers(0, 8), st.floats(0.25, 4.0), st.integers(0, 2**31 - 1))
def test_sherman_morrison_is_the_inverse_penalty(oracle, d, T, lam, seed):
    # VLA page section 2.2: A_t = M_t^{-1} with M_t = lambda0 I + sum u u^T
    rng = np.random.default_rng(seed)
    x = lambda: rng.standard_normal((1, 1, T, d))
    k = x()
    k /= np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), 1e-12)
    u = x()
    _, _, Af = oracle.vla_scan(x(), k, x(), u, lambda0=lam)
    M = lam * np.eye(d) + np.einsum("ti,tj->ij", u[0, 0], u[0, 0])
    assert rel(Af[0, 0], np.linalg.inv(M)) < 1e-10
