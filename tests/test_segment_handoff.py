"""The two facts the segmented Gated DeltaNet scan rests on, checked in fp64 on the oracle.

1. Non-expansive steps. With alpha_t <= 1 and beta_t |k_t|^2 <= 2, one step maps two states
   S and S' to states whose difference is (S - S') diag(alpha)(I - beta k k^T): no value row
   of the difference grows (row-wise 2-norm). Two runs of the scan from different entering
   states therefore never drift further apart, whatever the values.
2. Decay of the hand-off difference. Started from the zero state instead of the true entering
   state, a segment's state after the eight-chunk window differs from the true one by less
   than 2^-16 of the state's largest row norm under the gates of the Gated DeltaNet
   workloads (alpha = exp(-softplus(x)), x ~ N(-4, 1)), far below the device check's 2^-7
   (which leaves room for the kernel's bf16 rounding); with gates all but 1 it stays far
   above 2^-7, the case the device check sends back to the chained kernel. DeltaNet (no gate)
   shrinks the difference only along the keys it writes, about 0.85 per chunk for keys spread
   over all directions: its 48-chunk window leaves about 3e-4.
"""
import numpy as np

from delta_rule_recurrent_chunked_b200 import workloads as wl

WINDOW = 8 * 64
EPS = 2.0 ** -16         # exact arithmetic: the decayed difference alone
DEVICE_EPS = 2.0 ** -7   # the device check's threshold


def _row_norms(x):
    return np.linalg.norm(x, axis=-1)


def _draw(T, gate_mu, seed, mode=wl.GDN):
    w = wl.DRWorkload("handoff", 1, 1, T, 128, 128, mode, "fp32", s0_std=0.1, gate_mu=gate_mu)
    return wl.generate_dr(w, seed)


def test_steps_never_grow_the_difference_of_two_runs(oracle):
    inp = _draw(96, -4.0, seed=11)
    rng = np.random.default_rng(12)
    S_a = inp["S0"].astype(np.float64)
    S_b = S_a + rng.standard_normal(S_a.shape)
    prev = _row_norms(S_a - S_b)
    for t in range(inp["q"].shape[2]):
        sl = lambda x: None if x is None else x[:, :, t:t + 1]
        _, S_a = oracle.dr_scan(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]),
                                sl(inp["gate"]), S_a, wl.GDN)
        _, S_b = oracle.dr_scan(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]),
                                sl(inp["gate"]), S_b, wl.GDN)
        cur = _row_norms(S_a - S_b)
        assert np.all(cur <= prev * (1 + 1e-12) + 1e-300)
        prev = cur


def _handoff_ratio(oracle, gate_mu, seed, mode=wl.GDN, window=WINDOW):
    """Largest row norm of (true - zero-start) state after the window, over the largest row
    norm of the true state, for a segment entered after 2048 tokens."""
    inp = _draw(2048 + window, gate_mu, seed, mode)
    first = {k: (v[:, :, :2048] if k in ("q", "k", "v", "beta", "gate") and v is not None
                 else v) for k, v in inp.items() if k != "workload"}
    _, E0 = oracle.dr_scan(first["q"], first["k"], first["v"], first["beta"], first["gate"],
                           inp["S0"], mode)
    win = {k: (None if inp[k] is None else inp[k][:, :, 2048:])
           for k in ("q", "k", "v", "beta", "gate")}
    _, X = oracle.dr_scan(win["q"], win["k"], win["v"], win["beta"], win["gate"], E0, mode)
    _, Z = oracle.dr_scan(win["q"], win["k"], win["v"], win["beta"], win["gate"], None, mode)
    return float(np.max(_row_norms(X - Z)) / np.max(_row_norms(X)))


def test_window_difference_decays_under_the_workload_gates(oracle):
    for seed in range(3):
        assert _handoff_ratio(oracle, -4.0, seed) < EPS / 100
    # gates all but 1: the window leaves a difference far above the device threshold
    assert _handoff_ratio(oracle, -12.0, 0) > 10 * DEVICE_EPS


def test_deltanet_window_difference_decays_along_the_keys(oracle):
    for seed in range(2):
        assert _handoff_ratio(oracle, 0.0, seed, wl.DELTANET, 48 * 64) < DEVICE_EPS / 10
    # eight chunks are far from enough without a gate
    assert _handoff_ratio(oracle, 0.0, 0, wl.DELTANET, 8 * 64) > 10 * DEVICE_EPS
