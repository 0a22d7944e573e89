"""The chunked WY/UT algebra the tensor-core kernel implements equals the per-token
definition (fp64, up to rounding), for every variant, ragged tails included."""
import numpy as np
import pytest

from chunk_form import chunk_scan

DELTANET, GDN, KDA = 1, 2, 3


def _inputs(rng, T, dk, dv, mode):
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((T, dk)))
    k = unit(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    gate = None
    if mode == GDN:
        gate = np.exp(-np.logaddexp(0, rng.normal(-4, 1, T)))
    elif mode == KDA:
        gate = np.exp(-np.logaddexp(0, rng.normal(-4, 1, (T, dk))))
    S0 = 0.1 * rng.standard_normal((dv, dk))
    return q, k, v, beta, gate, S0


@pytest.mark.parametrize("mode", [DELTANET, GDN, KDA])
@pytest.mark.parametrize("T", [1, 64, 100, 256])
def test_chunk_form_equals_per_token(oracle, mode, T):
    rng = np.random.default_rng(T * 10 + mode)
    dk, dv = 32, 24
    q, k, v, beta, gate, S0 = _inputs(rng, T, dk, dv, mode)
    out, S = chunk_scan(q, k, v, beta, gate, S0, mode)
    g = None if gate is None else gate[None, None]
    ref_out, ref_S = oracle.dr_scan(q[None, None], k[None, None], v[None, None], beta[None, None],
                                    g, S0[None, None], mode)
    scale = max(np.abs(ref_out).max(), 1.0)
    assert np.abs(out - ref_out[0, 0]).max() / scale < 1e-12
    assert np.abs(S - ref_S[0, 0]).max() / max(np.abs(ref_S).max(), 1.0) < 1e-12


def test_chunk_size_does_not_matter(oracle):
    rng = np.random.default_rng(3)
    q, k, v, beta, gate, S0 = _inputs(rng, 200, 16, 16, KDA)
    a, Sa = chunk_scan(q, k, v, beta, gate, S0, KDA, chunk=64)
    b, Sb = chunk_scan(q, k, v, beta, gate, S0, KDA, chunk=16)
    assert np.abs(a - b).max() < 1e-12 and np.abs(Sa - Sb).max() < 1e-12
