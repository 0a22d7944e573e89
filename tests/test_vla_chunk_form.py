"""The chunked VLA algebra the two CUDA kernels implement (Woodbury/Cholesky A-phase, WY
S-phase with read key k and write key alpha_hat) equals the per-token definition in fp64,
ragged tails, entering states and the ratio readout included."""
import numpy as np
import pytest

from vla_chunk_form import vla_chunk_scan


def _inputs(rng, T, d, ratio):
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    elu1 = lambda x: np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    q, k = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    q, k = (elu1(q), unit(elu1(k))) if ratio else (unit(q), unit(k))
    v = rng.standard_normal((T, d))
    u = rng.standard_normal((T, d)) / np.sqrt(d)
    S0 = 0.1 * rng.standard_normal((d, d))
    M = rng.standard_normal((d, d)) / np.sqrt(d)
    A0 = np.linalg.inv(np.eye(d) + M @ M.T)
    n0 = 0.5 + rng.uniform(size=d) / d
    return q, k, v, u, S0, A0, n0


@pytest.mark.parametrize("ratio", [False, True])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_vla_chunk_form_equals_per_token(oracle, T, ratio):
    rng = np.random.default_rng(T + 1000 * ratio)
    d = 16
    q, k, v, u, S0, A0, n0 = _inputs(rng, T, d, ratio)
    got = vla_chunk_scan(q, k, v, u, S0=S0, A0=A0, n0=n0 if ratio else None, ratio=ratio)
    h = lambda x: x[None, None]
    if ratio:
        ref = oracle.vla_scan_ratio(h(q), h(k), h(v), h(u), S0=h(S0), A0=h(A0), n0=h(n0))
    else:
        ref = oracle.vla_scan(h(q), h(k), h(v), h(u), S0=h(S0), A0=h(A0))
    for g, r in zip(got, ref):
        r = np.asarray(r)[0, 0]
        assert np.abs(g - r).max() / max(np.abs(r).max(), 1.0) < 1e-11


def test_vla_chunk_form_chunk_size_does_not_matter(oracle):
    # the Woodbury step over any chunk length is the same map: chunks of 1 token are the
    # Sherman-Morrison recurrence itself
    rng = np.random.default_rng(3)
    q, k, v, u, S0, A0, _ = _inputs(rng, 50, 8, False)
    a = vla_chunk_scan(q, k, v, u, S0=S0, A0=A0, chunk=1)
    b = vla_chunk_scan(q, k, v, u, S0=S0, A0=A0, chunk=17)
    for x, y in zip(a, b):
        assert np.abs(x - y).max() / max(np.abs(y).max(), 1.0) < 1e-11
