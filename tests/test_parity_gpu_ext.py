"""GPU parity of the rows built on the delta-rule recurrence beyond the four variants: Gated
DeltaNet-2 (per-channel erase and write gates) and the per-token write values u_t = beta_t r_t,
through dr_scan_fwd_ex / dr_decode_step_ex, against the fp64 oracle.

Tolerance (max|x - y| / max|y| per tensor: out, S_final and u): 1e-4 for fp32 q/k/v, 2e-2 for
bf16 q/k/v with an fp32 state (oracle fed the bf16-rounded inputs).

Source: "Mechanisms, trade-offs and cross-layer routing of linear-attention architectures",
sections "Methodology" and "Technical details" (Gated DeltaNet-2; the CLER / CLVR routing of a
layer's write signal).
"""
import numpy as np
import pytest

import delta_rule_recurrent_chunked_b200 as drs
from delta_rule_recurrent_chunked_b200 import workloads as wl

from helpers import MODE_NAME, oracle_dr_ex, rel_err, tensor_np, to_device

# the three VLA paths of vla_scan_fwd_ex: the fused cluster kernel (default), the two-kernel
# pair, the per-token kernel
VLA_PATHS = {"fused": {}, "two_kernel": {"two_kernel": True}, "sequential": {"sequential": True}}

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    drs.lib()
    yield
    assert drs.poll_error() == drs.DR_OK


def run_ex(dev, w, force_sequential=False):
    out, Sf, u = drs.scan_ex(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                             mode=MODE_NAME[w.mode], erase=dev["erase"], write=dev["write"],
                             force_sequential=force_sequential)
    torch.cuda.synchronize()
    return out, Sf, u


def check_ex(oracle, w, seed=0, force_sequential=False, heads=None):
    inputs = wl.generate_dr(w, seed)
    dev = to_device(inputs)
    got = run_ex(dev, w, force_sequential)
    if heads is not None:
        inputs = wl.head_slice(inputs, heads)
        got = tuple(tensor_np(t).reshape((w.B * w.H,) + tuple(t.shape[2:]))[heads][None]
                    for t in got)
    else:
        got = tuple(tensor_np(t) for t in got)
    ref = oracle_dr_ex(oracle, inputs)
    errs = [rel_err(g, r) for g, r in zip(got, ref)]
    assert all(e <= TOL[w.dtype] for e in errs), (w, errs)
    assert drs.poll_error() == drs.DR_OK
    return errs


# --- per-token kernel (fp32 state): every variant, write values, fp32 and bf16 inputs
@pytest.mark.parametrize("mode", [wl.LINEAR, wl.DELTANET, wl.GDN, wl.KDA, wl.GDN2])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_sequential_write_values_and_gdn2(oracle, mode, dk, dv, dtype):
    w = wl.DRWorkload("t", 2, 2, 77, dk, dv, mode, dtype, s0_std=0.1, gate_mu=-2.0)
    check_ex(oracle, w, seed=mode + dk + dv, force_sequential=True)


# --- chunked tensor-core kernel: write values on every variant and launch plan, ragged T
@pytest.mark.parametrize("mode", [wl.DELTANET, wl.GDN, wl.KDA, wl.GDN2])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 517])
def test_chunked_write_values_ragged(oracle, mode, T):
    w = wl.DRWorkload("t", 1, 2, T, 128, 128, mode, "bf16", s0_std=0.1)
    check_ex(oracle, w, seed=T + mode)


# split clusters (few heads) and one CTA per (head, value slice) (many heads): the split
# chain CTAs read the write values out of tensor memory one chunk late
@pytest.mark.parametrize("mode", [wl.DELTANET, wl.GDN])
@pytest.mark.parametrize("BH,dv", [(2, 128), (16, 64), (40, 128), (64, 128), (64, 32)])
def test_chunked_write_values_every_plan(oracle, mode, BH, dv):
    plan = drs.chunked_plan(mode, BH, 128, dv)
    assert plan is not None
    w = wl.DRWorkload("t", 1, BH, 300, 128, dv, mode, "bf16", s0_std=0.1)
    check_ex(oracle, w, seed=BH + dv)


# Gated DeltaNet-2 on the chunked path (pre-scaled inputs, then Gated DeltaNet's kernel and
# plan): split clusters for few heads, one CTA per head and slice for many, narrow slices
@pytest.mark.parametrize("BH,dv", [(2, 32), (2, 64), (2, 128), (64, 128), (96, 64)])
def test_chunked_gdn2(oracle, BH, dv):
    assert drs.chunked_plan("gdn2", BH, 128, dv) == drs.chunked_plan("gdn", BH, 128, dv)
    w = wl.DRWorkload("t", 1, BH, 333, 128, dv, wl.GDN2, "bf16", s0_std=0.1)
    check_ex(oracle, w, seed=5 * BH + dv)


def test_chunked_gdn2_strong_decay(oracle):
    w = wl.DRWorkload("t", 1, 4, 300, 128, 128, wl.GDN2, "bf16", s0_std=0.1, gate_mu=2.0)
    check_ex(oracle, w, seed=77)


def test_gdn2_bf16_workload_sampled(oracle):
    w = wl.workload("gdn2_bf16")
    check_ex(oracle, w, heads=[0, 17, 31])


def test_gdn2_with_unit_gates_matches_gdn_on_the_chunked_kernel(oracle):
    # b = w = 1 is Gated DeltaNet: the pre-scaling by 1 is exact and the same kernel and plan
    # follow, so the two calls give the same bits
    w = wl.DRWorkload("t", 1, 4, 200, 128, 128, wl.GDN2, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, 3)
    inputs["erase"] = np.ones_like(inputs["erase"])
    inputs["write"] = np.ones_like(inputs["write"])
    dev = to_device(inputs)
    o2, S2, _ = run_ex(dev, w)
    o1, S1 = drs.scan(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"], mode="gdn")
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_scan_without_write_values_is_unchanged(oracle):
    # dr_scan_fwd_ex with u_out = NULL and dr_scan_fwd give the same bits
    w = wl.DRWorkload("t", 1, 2, 300, 128, 128, wl.GDN, "bf16", s0_std=0.1)
    dev = to_device(wl.generate_dr(w, 8))
    o1, S1 = drs.scan(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"], mode="gdn")
    o2, S2, u = drs.scan_ex(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                            mode="gdn", want_u=False)
    o3, S3, _ = drs.scan_ex(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                            mode="gdn")
    torch.cuda.synchronize()
    assert u is None
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    assert torch.equal(o1, o3) and torch.equal(S1, S3)


def test_gdn2_needs_the_ex_entry_point():
    z = torch.zeros(1, 1, 4, 32, device="cuda")
    b = torch.zeros(1, 1, 4, device="cuda")
    with pytest.raises(drs.DrScanError):
        drs.scan(z, z, z, b, b, None, mode="gdn2")


# --- decode step: Gated DeltaNet-2 and the write value
@pytest.mark.parametrize("mode", [wl.LINEAR, wl.DELTANET, wl.GDN, wl.KDA, wl.GDN2])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 64), (128, 128)])
def test_decode_step_ex(oracle, mode, dtype, dk, dv):
    w = wl.DRWorkload("decode", 3, 5, 1, dk, dv, mode, dtype, s0_std=0.1)
    inputs = wl.generate_dr(w, seed=dk + dv + mode)
    dev = to_device(inputs)
    B, H = w.B, w.H
    sq = lambda t, *tail: None if t is None else t.reshape(B, H, *tail)
    gate = dev["gate"]
    if gate is not None:
        gate = gate.reshape((B, H) + ((dk,) if mode == wl.KDA else ()))
    S = dev["S0"].clone()
    out, u = drs.decode_step_ex(sq(dev["q"], dk), sq(dev["k"], dk), sq(dev["v"], dv),
                                sq(dev["beta"]), gate, S, mode=MODE_NAME[mode],
                                erase=sq(dev["erase"], dk), write=sq(dev["write"], dv))
    torch.cuda.synchronize()
    ref_out, ref_S, ref_u = oracle_dr_ex(oracle, inputs)
    assert rel_err(tensor_np(out), ref_out[:, :, 0]) <= TOL[dtype]
    assert rel_err(tensor_np(S), ref_S) <= TOL[dtype]
    assert rel_err(tensor_np(u), ref_u[:, :, 0]) <= TOL[dtype]


# --- VLA ratio readout ("Variational Linear Attention (VLA)", section 2.3): the normaliser
# n_t = n_{t-1} + (1 - n_{t-1} k_t) alpha_hat_t^T and o_t = S_t q_t / (n_t q_t), fp32, 1e-4
@pytest.mark.parametrize("path", ["fused", "two_kernel", "sequential"])
@pytest.mark.parametrize("d", [32, 96])
def test_vla_ratio_workload(oracle, d, path):
    w = wl.workload(f"vla_ratio_fp32_d{d}")
    inputs = wl.generate_vla(w, 0)
    dev = {k: torch.from_numpy(inputs[k]).cuda() for k in ("q", "k", "v", "u")}
    out, Sf, Af, nf = drs.vla_scan_ratio(dev["q"], dev["k"], dev["v"], dev["u"], lambda0=w.lambda0,
                                         **VLA_PATHS[path])
    torch.cuda.synchronize()
    heads = [0, 13, 31]
    sub = wl.head_slice(inputs, heads)
    ref = oracle.vla_scan_ratio(sub["q"], sub["k"], sub["v"], sub["u"], lambda0=w.lambda0)
    BH = w.B * w.H
    got = [tensor_np(t).reshape((BH,) + tuple(t.shape[2:]))[heads][None] for t in (out, Sf, Af, nf)]
    for g, r in zip(got, ref):
        assert rel_err(g, r) <= 1e-4, rel_err(g, r)


@pytest.mark.parametrize("path", ["fused", "two_kernel", "sequential"])
@pytest.mark.parametrize("d", [32, 64, 96, 128])
@pytest.mark.parametrize("T", [1, 17, 64, 100, 129])
def test_vla_ratio_small_with_initial_state(oracle, d, T, path):
    rng = np.random.default_rng(7 * d + T)
    B, H = 1, 3
    elu1 = lambda x: np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = elu1(rng.standard_normal((B, H, T, d))).astype(np.float32)
    k = unit(elu1(rng.standard_normal((B, H, T, d)))).astype(np.float32)
    v = rng.standard_normal((B, H, T, d)).astype(np.float32)
    u = (rng.standard_normal((B, H, T, d)) / np.sqrt(d)).astype(np.float32)
    S0 = (0.1 * rng.standard_normal((B, H, d, d))).astype(np.float32)
    M = rng.standard_normal((B, H, d, d)) / np.sqrt(d)
    A0 = np.linalg.inv(np.eye(d) + M @ np.swapaxes(M, -1, -2)).astype(np.float32)
    n0 = (0.5 + rng.uniform(size=(B, H, d)) / d).astype(np.float32)
    c = lambda x: torch.from_numpy(x).cuda()
    got = drs.vla_scan_ratio(c(q), c(k), c(v), c(u), S0=c(S0), A0=c(A0), n0=c(n0),
                             **VLA_PATHS[path])
    torch.cuda.synchronize()
    ref = oracle.vla_scan_ratio(q, k, v, u, S0=S0, A0=A0, n0=n0)
    for g, r in zip(got, ref):
        assert rel_err(tensor_np(g), r) <= 1e-4


def test_vla_ratio_keeps_the_plain_state():
    # the ratio readout changes only the output: S and A are the plain scan's
    w = wl.workload("vla_ratio_fp32_d32", T=300)
    inputs = wl.generate_vla(w, 4)
    dev = {k: torch.from_numpy(inputs[k]).cuda() for k in ("q", "k", "v", "u")}
    _, S1, A1 = drs.vla_scan(dev["q"], dev["k"], dev["v"], dev["u"])
    _, S2, A2, _ = drs.vla_scan_ratio(dev["q"], dev["k"], dev["v"], dev["u"])
    torch.cuda.synchronize()
    assert torch.equal(S1, S2) and torch.equal(A1, A2)


def test_vla_ratio_empty_sequence_returns_initial_state():
    d = 32
    z = torch.empty(1, 2, 0, d, device="cuda")
    n0 = torch.rand(1, 2, d, device="cuda")
    _, Sf, Af, nf = drs.vla_scan_ratio(z, z, z, z, n0=n0, lambda0=2.0)
    torch.cuda.synchronize()
    assert torch.equal(nf, n0) and torch.count_nonzero(Sf) == 0
