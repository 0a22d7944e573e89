"""The parallel scan over chunk transitions (tests/segment_form.py) against the per-token
oracle: any split of the chunks into segments, for every decaying variant and ragged T,
gives the oracle's outputs, final state and state at every segment boundary."""
import numpy as np
import pytest

from chunk_form import DELTANET, GDN, KDA
from segment_form import segment_scan


def draw(seed, T, dk, dv, mode):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((T, dk))), unit(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv))
    beta = rng.uniform(0.05, 0.95, T)
    gate = None
    if mode == GDN:
        gate = rng.uniform(0.6, 1.0, T)
    elif mode == KDA:
        gate = rng.uniform(0.6, 1.0, (T, dk))
    S0 = 0.3 * rng.standard_normal((dv, dk))
    return q, k, v, beta, gate, S0


def rel(x, y):
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-300))


@pytest.mark.parametrize("mode", [DELTANET, GDN, KDA])
@pytest.mark.parametrize("T", [5 * 64 + 17, 6 * 64])
@pytest.mark.parametrize("cuts", [[], [2], [1, 3], [1, 2, 3, 4, 5]])
@pytest.mark.parametrize("replay", [False, True])
def test_segment_scan_matches_the_oracle(oracle, mode, T, cuts, replay):
    dk, dv = 16, 8
    q, k, v, beta, gate, S0 = draw(mode * 100 + T, T, dk, dv, mode)
    n = -(-T // 64)
    bounds = [0] + cuts + [n]
    out, Sf, entering = segment_scan(q, k, v, beta, gate, S0, mode, bounds, replay=replay)
    b = lambda x: None if x is None else x[None, None]
    ref_out, ref_S = oracle.dr_scan(b(q), b(k), b(v), b(beta), b(gate), b(S0), mode)
    assert rel(out, ref_out[0, 0]) < 1e-10
    assert rel(Sf, ref_S[0, 0]) < 1e-10
    for s0, Sin in zip(bounds[:-1], entering):
        t = s0 * 64
        g = None if gate is None else b(gate[:t])
        _, S_at = oracle.dr_scan(b(q[:t]), b(k[:t]), b(v[:t]), b(beta[:t]), g, b(S0), mode)
        assert rel(Sin, S_at[0, 0]) < 1e-10
