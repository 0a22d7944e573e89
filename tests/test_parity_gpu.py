"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 oracle.

Tolerance (max|x - y| / max|y| per tensor, out and S_final):
  fp32 q/k/v: 1e-4;   bf16 q/k/v with fp32 state: 2e-2 (oracle fed the bf16-rounded inputs).
Small cases span several 64-token chunks and a ragged tail; the full-size workloads are
checked on sampled heads (heads are independent sequences), in the launch configuration
the benchmark times.
"""
import numpy as np
import pytest

import delta_rule_recurrent_chunked_b200 as drs
from delta_rule_recurrent_chunked_b200 import workloads as wl

from helpers import MODE_NAME, oracle_dr, rel_err, row_rel_err, tensor_np, to_device

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


def run_dr(dev, w, force_sequential=False, want_state=True):
    out, Sf = drs.scan(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                       mode=MODE_NAME[w.mode], want_state=want_state,
                       force_sequential=force_sequential)
    torch.cuda.synchronize()
    return out, Sf


def check_dr(oracle, w, seed=0, force_sequential=False, tol=None):
    inputs = wl.generate_dr(w, seed)
    dev = to_device(inputs)
    out, Sf = run_dr(dev, w, force_sequential)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    tol = tol or TOL[w.dtype]
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= tol and e_S <= tol, (w, e_out, e_S)
    return e_out, e_S


# --- the parity workload: DeltaNet fp32, B1 H2 T256 d32. Besides the tensor-wide metric,
# every row (one token's output, one row of the state) must meet 1e-4 relative to its own
# magnitude.
def test_deltanet_fp32_workload(oracle):
    w = wl.workload("deltanet_fp32")
    inputs = wl.generate_dr(w, 0)
    out, Sf = run_dr(to_device(inputs), w)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    for got, ref in ((tensor_np(out), ref_out), (tensor_np(Sf), ref_S)):
        assert rel_err(got, ref) <= TOL["fp32"]
        assert row_rel_err(got, ref) <= TOL["fp32"], row_rel_err(got, ref)


# --- every variant, fp32 inputs (per-token kernel), ragged T, all head sizes
@pytest.mark.parametrize("mode", [wl.LINEAR, wl.DELTANET, wl.GDN, wl.KDA])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 32), (128, 64), (32, 128), (128, 128)])
@pytest.mark.parametrize("T", [1, 65, 130])
def test_sequential_fp32_variants(oracle, mode, dk, dv, T):
    w = wl.DRWorkload("t", 2, 2, T, dk, dv, mode, "fp32", s0_std=0.1, gate_mu=-2.0)
    check_dr(oracle, w, seed=T + dk + dv)


# --- bf16 inputs on the per-token kernel (the fp32-state baseline path)
@pytest.mark.parametrize("mode", [wl.DELTANET, wl.GDN, wl.KDA])
def test_sequential_bf16(oracle, mode):
    w = wl.DRWorkload("t", 1, 3, 200, 128, 128, mode, "bf16", s0_std=0.1)
    check_dr(oracle, w, seed=3, force_sequential=True)


# --- bf16 inputs through the default dispatch (chunked kernel where it applies)
@pytest.mark.parametrize("mode", [wl.DELTANET, wl.GDN, wl.KDA])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200, 517])
def test_bf16_dispatch_ragged(oracle, mode, T):
    w = wl.DRWorkload("t", 1, 2, T, 128, 128, mode, "bf16", s0_std=0.1)
    check_dr(oracle, w, seed=T)


@pytest.mark.parametrize("dv", [32, 64])
@pytest.mark.parametrize("mode", [wl.GDN, wl.KDA])
def test_bf16_dispatch_narrow_values(oracle, mode, dv):
    w = wl.DRWorkload("t", 2, 2, 300, 128, dv, mode, "bf16", s0_std=0.1)
    check_dr(oracle, w, seed=dv)


# Every branch of the chunked kernel's launch plan: split clusters with four, three or two
# prep CTAs and a three-deep chain slot ring (few heads), with one prep CTA and a two-deep
# ring, and one CTA per (head, value slice) once the heads fill the GPU. The plan is read back
# so that a change of the planner cannot silently drop a branch from the tests.
@pytest.mark.parametrize("mode", [wl.DELTANET, wl.GDN])
@pytest.mark.parametrize("BH,dv,split", [(2, 128, 4), (16, 64, 4), (24, 128, 3), (32, 128, 2),
                                         (40, 128, 1), (40, 64, 1), (46, 128, None),
                                         (64, 128, 0), (64, 32, 0)])
def test_bf16_plan_branches(oracle, mode, BH, dv, split):
    plan = drs.chunked_plan(mode, BH, 128, dv)
    assert plan is not None
    bv, nprep = plan
    assert dv % bv == 0
    if split is not None:
        assert nprep == split, plan
    w = wl.DRWorkload("t", 1, BH, 300, 128, dv, mode, "bf16", s0_std=0.1)
    check_dr(oracle, w, seed=BH + dv)


def test_bf16_strong_decay_gates(oracle):
    # gates near 0.5 per step: summed log-decay over a 64-token chunk reaches about -45
    w = wl.DRWorkload("t", 1, 2, 256, 128, 128, wl.GDN, "bf16", gate_mu=0.0, gate_sigma=0.5)
    check_dr(oracle, w, seed=5)


def _check_with_gates(oracle, w, seed, gate_fn):
    """Parity on a generated workload whose gate array is replaced by gate_fn(inputs) (both
    sides consume the same replaced array)."""
    inputs = wl.generate_dr(w, seed)
    inputs["gate"] = np.ascontiguousarray(gate_fn(inputs), dtype=np.float32)
    dev = to_device(inputs)
    out, Sf = run_dr(dev, w)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert np.isfinite(e_out) and np.isfinite(e_S), (w, e_out, e_S)
    assert e_out <= TOL[w.dtype] and e_S <= TOL[w.dtype], (w, e_out, e_S)
    assert drs.poll_error() == drs.DR_OK


# GDN with alpha about 0.12 per step (x ~ N(2, 1)): a chunk's summed log-decay is about -140,
# far past the point where the factored form exp(g_t) * exp(-g_i) would overflow, so every
# chunk takes the direct exp(g_t - g_i) branch. Split (2 heads) and unsplit (64 heads) plans,
# ragged T.
@pytest.mark.parametrize("BH", [2, 64])
@pytest.mark.parametrize("T", [200, 300])
def test_gdn_bf16_very_strong_decay(oracle, BH, T):
    w = wl.DRWorkload("t", 1, BH, T, 128, 128, wl.GDN, "bf16", s0_std=0.1, gate_mu=2.0)
    _check_with_gates(oracle, w, 20 + BH + T, lambda inp: inp["gate"])


# GDN whose chunks alternate between weak gates (factored branch) and very strong ones
# (direct branch) inside one sequence.
@pytest.mark.parametrize("BH", [2, 64])
def test_gdn_bf16_mixed_decay_chunks(oracle, BH):
    w = wl.DRWorkload("t", 1, BH, 450, 128, 128, wl.GDN, "bf16", s0_std=0.1)

    def gates(inp):
        rng = np.random.default_rng(BH)
        strong = np.exp(-np.logaddexp(0.0, 2.0 + rng.standard_normal(inp["gate"].shape)))
        g = inp["gate"].astype(np.float64).copy()
        chunk = (np.arange(w.T) // 64) % 2 == 1
        g[..., chunk] = strong[..., chunk]
        return g

    _check_with_gates(oracle, w, 31 + BH, gates)


# KDA with strong per-channel gates: x ~ N(0, 1) (alpha about 0.5), x ~ N(1.4, 0.5) (alpha
# about 0.2: a channel's summed log-decay over one chunk about -100, below fp32's exp range)
# and x ~ N(2, 1) (alpha about 0.12, about -140 per chunk), unsplit launches, ragged T.
@pytest.mark.parametrize("mu,sigma", [(0.0, 1.0), (1.4, 0.5), (2.0, 1.0)])
@pytest.mark.parametrize("BH", [2, 48])
def test_kda_bf16_strong_decay(oracle, mu, sigma, BH):
    w = wl.DRWorkload("t", 1, BH, 300, 128, 128, wl.KDA, "bf16", s0_std=0.1, gate_mu=mu,
                      gate_sigma=sigma)
    _check_with_gates(oracle, w, 7 + BH, lambda inp: inp["gate"])


# --- full-size workloads, sampled heads
def _check_sampled(oracle, name, heads, seed=0):
    w = wl.workload(name) if isinstance(name, str) else name
    inputs = wl.generate_dr(w, seed)
    dev = to_device(inputs)
    out, Sf = run_dr(dev, w)
    sub = wl.head_slice(inputs, heads)
    ref_out, ref_S = oracle_dr(oracle, sub)
    o = tensor_np(out).reshape((w.B * w.H,) + tuple(out.shape[2:]))[heads][None]
    s = tensor_np(Sf).reshape((w.B * w.H,) + tuple(Sf.shape[2:]))[heads][None]
    e_out, e_S = rel_err(o, ref_out), rel_err(s, ref_S)
    assert e_out <= TOL[w.dtype] and e_S <= TOL[w.dtype], (name, e_out, e_S)
    return e_out, e_S


def test_gdn_bf16_workload_sampled(oracle):
    _check_sampled(oracle, "gdn_bf16", [0, 13, 31])


def test_kda_bf16_workload_sampled(oracle):
    _check_sampled(oracle, "kda_bf16", [0, 77, 127])


@pytest.mark.parametrize("T", [4096, 8192, 16384, 32768])
def test_gdn_long_workload_sampled(oracle, T):
    _check_sampled(oracle, f"gdn_long_t{T}", [0, 15])


# DeltaNet has no decay, so the rounding of every chunk's bf16 operands stays in the state:
# the long-context shapes (16 heads, split clusters) on the chunked kernel, sampled heads.
@pytest.mark.parametrize("T", [4096, 32768])
def test_deltanet_bf16_long_sampled(oracle, T):
    w = wl.DRWorkload(f"deltanet_long_t{T}", 1, 16, T, 128, 128, wl.DELTANET, "bf16",
                      s0_std=0.1)
    assert drs.chunked_plan("deltanet", 16, 128, 128)[1] > 0  # a split launch
    _check_sampled(oracle, w, [0, 15])


# the same with one CTA per (head, value slice): 64 heads
def test_deltanet_bf16_long_unsplit_sampled(oracle):
    w = wl.DRWorkload("deltanet_long_unsplit", 1, 64, 8192, 128, 128, wl.DELTANET, "bf16",
                      s0_std=0.1)
    assert drs.chunked_plan("deltanet", 64, 128, 128)[1] == 0
    _check_sampled(oracle, w, [0, 63])


# --- edge cases
def test_empty_sequence_copies_state():
    S0 = torch.randn(2, 3, 32, 64, device="cuda")
    q = torch.empty(2, 3, 0, 64, device="cuda")
    v = torch.empty(2, 3, 0, 32, device="cuda")
    beta = torch.empty(2, 3, 0, device="cuda")
    out, Sf = drs.scan(q, q, v, beta, None, S0, mode="deltanet")
    torch.cuda.synchronize()
    assert out.shape == (2, 3, 0, 32) and torch.equal(Sf, S0)
    _, Sf0 = drs.scan(q, q, v, beta, None, None, mode="deltanet")
    torch.cuda.synchronize()
    assert torch.count_nonzero(Sf0) == 0


def test_state_optional_and_carry(oracle):
    w = wl.DRWorkload("t", 1, 2, 256, 128, 128, wl.GDN, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, 9)
    dev = to_device(inputs)
    out_nostate, none = run_dr(dev, w, want_state=False)
    assert none is None
    out, Sf = run_dr(dev, w)
    assert torch.equal(out_nostate, out)
    # resume: two halves with the carried fp32 state equal one pass (up to tolerance)
    h = 128
    half = {k: (None if t is None else t) for k, t in dev.items()}
    a = {k: (t[:, :, :h].contiguous() if t is not None and k != "S0" else t) for k, t in half.items()}
    o1, S1 = drs.scan(a["q"], a["k"], a["v"], a["beta"], a["gate"], dev["S0"], mode="gdn")
    b = {k: (t[:, :, h:].contiguous() if t is not None and k != "S0" else t) for k, t in half.items()}
    o2, S2 = drs.scan(b["q"], b["k"], b["v"], b["beta"], b["gate"], S1, mode="gdn")
    torch.cuda.synchronize()
    ref_out, ref_S = oracle_dr(oracle, inputs)
    assert rel_err(tensor_np(torch.cat([o1, o2], dim=2)), ref_out) <= TOL["bf16"]
    assert rel_err(tensor_np(S2), ref_S) <= TOL["bf16"]


def test_heads_are_independent():
    w = wl.DRWorkload("t", 1, 4, 130, 128, 128, wl.KDA, "bf16")
    dev = to_device(wl.generate_dr(w, 4))
    out, Sf = run_dr(dev, w)
    p = torch.tensor([2, 0, 3, 1], device="cuda")
    perm = {k: (None if t is None else t[:, p].contiguous()) for k, t in dev.items()}
    out_p, Sf_p = run_dr(perm, w)
    assert torch.equal(out_p, out[:, p]) and torch.equal(Sf_p, Sf[:, p])


# --- streams: the library keeps no per-call scratch, so scans on different streams, running
# at the same time on different inputs (split and unsplit launch plans), are independent
def test_concurrent_scans_on_two_streams(oracle):
    cases = [(wl.DRWorkload("t", 1, 2, 700, 128, 128, wl.GDN, "bf16", s0_std=0.1), 11),
             (wl.DRWorkload("t", 1, 64, 200, 128, 128, wl.KDA, "bf16", s0_std=0.1), 12)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    runs = []
    for (w, seed), st in zip(cases, streams):
        inputs = wl.generate_dr(w, seed)
        dev = to_device(inputs)
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            out, Sf = drs.scan(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                               mode=MODE_NAME[w.mode])
        runs.append((w, inputs, out, Sf))
    torch.cuda.synchronize()
    for w, inputs, out, Sf in runs:
        ref_out, ref_S = oracle_dr(oracle, inputs)
        e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
        assert e_out <= TOL["bf16"] and e_S <= TOL["bf16"], (w, e_out, e_S)


# --- single-token decode on a resident state
def decode_inputs(dev, w):
    """Drop the token axis (T = 1) of an uploaded workload: the decode step's shapes."""
    B, H = w.B, w.H
    gate = dev["gate"]
    if gate is not None:
        gate = gate.reshape((B, H) + ((w.dk,) if w.mode == wl.KDA else ()))
    return (dev["q"].reshape(B, H, w.dk), dev["k"].reshape(B, H, w.dk),
            dev["v"].reshape(B, H, w.dv), dev["beta"].reshape(B, H), gate)


@pytest.mark.parametrize("mode", [wl.LINEAR, wl.DELTANET, wl.GDN, wl.KDA])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 128)])
def test_decode_step_matches_one_token_of_the_oracle(oracle, mode, dtype, dk, dv):
    w = wl.DRWorkload("decode", 3, 5, 1, dk, dv, mode, dtype, s0_std=0.1)
    inputs = wl.generate_dr(w, seed=dk + dv + mode)
    dev = to_device(inputs)
    q, k, v, beta, gate = decode_inputs(dev, w)
    S = dev["S0"].clone()
    out = drs.decode_step(q, k, v, beta, gate, S, mode=MODE_NAME[mode])
    torch.cuda.synchronize()
    ref_out, ref_S = oracle_dr(oracle, inputs)
    assert rel_err(tensor_np(out), ref_out[:, :, 0]) <= TOL[dtype]
    assert rel_err(tensor_np(S), ref_S) <= TOL[dtype]


@pytest.mark.parametrize("mode", [wl.DELTANET, wl.GDN, wl.KDA])
def test_decode_steps_replay_the_scan(oracle, mode):
    T = 9
    w = wl.DRWorkload("replay", 2, 3, T, 64, 64, mode, "fp32", s0_std=0.1)
    inputs = wl.generate_dr(w, seed=11 + mode)
    dev = to_device(inputs)
    S = dev["S0"].clone()
    outs = []
    for t in range(T):
        gate = None if dev["gate"] is None else dev["gate"][:, :, t].contiguous()
        outs.append(drs.decode_step(dev["q"][:, :, t].contiguous(), dev["k"][:, :, t].contiguous(),
                                    dev["v"][:, :, t].contiguous(),
                                    dev["beta"][:, :, t].contiguous(), gate, S,
                                    mode=MODE_NAME[mode]))
    torch.cuda.synchronize()
    ref_out, ref_S = oracle_dr(oracle, inputs)
    assert rel_err(tensor_np(torch.stack(outs, dim=2)), ref_out) <= 1e-4
    assert rel_err(tensor_np(S), ref_S) <= 1e-4


def test_gdn_decode_workload_every_head(oracle):
    # the benchmark's decode workload (4096 heads, 256 MiB state), every head checked
    w = wl.workload("gdn_decode_bf16")
    inputs = wl.generate_dr(w, 0)
    dev = to_device(inputs)
    q, k, v, beta, gate = decode_inputs(dev, w)
    S = dev["S0"].clone()
    out = drs.decode_step(q, k, v, beta, gate, S, mode="gdn")
    torch.cuda.synchronize()
    ref_out, ref_S = oracle_dr(oracle, inputs)
    assert rel_err(tensor_np(out), ref_out[:, :, 0]) <= TOL["bf16"]
    assert rel_err(tensor_np(S), ref_S) <= TOL["bf16"]


def test_decode_step_empty_batch_launches_nothing():
    z = torch.empty(0, 4, 128, device="cuda")
    S = torch.empty(0, 4, 128, 128, device="cuda")
    out = drs.decode_step(z, z, z, torch.empty(0, 4, device="cuda"), None, S, mode="deltanet")
    torch.cuda.synchronize()
    assert out.shape == (0, 4, 128)


# --- maximum sizes: element offsets beyond 2^31
def _fill_head(t, h, x):
    t.view(-1, *t.shape[2:])[h] = torch.from_numpy(np.ascontiguousarray(x)).to(t.dtype).to(t.device)


def test_chunked_offsets_beyond_int32(oracle):
    # 16384 heads x 1088 tokens x 128 channels: 2.28e9 elements per q/k/v/out tensor (about
    # 20 GB in all), so the last head's data lies past 2^31 elements. Only the first and last
    # heads carry data; every other head has zero keys, queries and values and must read out
    # exactly zero.
    B, H, T, dk, dv = 128, 128, 1088, 128, 128
    BH = B * H
    assert BH * T * dk > 2**31
    q = torch.zeros(B, H, T, dk, dtype=torch.bfloat16, device="cuda")
    k, v = torch.zeros_like(q), torch.zeros_like(q)
    beta = torch.full((B, H, T), 0.5, device="cuda")
    gate = torch.full((B, H, T), 0.97, device="cuda")
    w = wl.DRWorkload("edge", 1, 2, T, dk, dv, wl.GDN, "bf16")
    small = wl.generate_dr(w, 5)
    for j, h in enumerate((0, BH - 1)):
        for name, t in (("q", q), ("k", k), ("v", v)):
            _fill_head(t, h, small[name][0, j])
        _fill_head(beta, h, small["beta"][0, j])
        _fill_head(gate, h, small["gate"][0, j])
    out, Sf = drs.scan(q, k, v, beta, gate, None, mode="gdn")
    torch.cuda.synchronize()
    ref_out, ref_S = oracle_dr(oracle, small)
    o = out.view(BH, T, dv)
    s = Sf.view(BH, dv, dk)
    for j, h in enumerate((0, BH - 1)):
        assert rel_err(tensor_np(o[h]), ref_out[0, j]) <= TOL["bf16"]
        assert rel_err(tensor_np(s[h]), ref_S[0, j]) <= TOL["bf16"]
    for h in (1, BH // 2, BH - 2):
        assert torch.count_nonzero(o[h]) == 0 and torch.count_nonzero(s[h]) == 0
    del q, k, v, out, Sf, o, s
    torch.cuda.empty_cache()


def test_decode_offsets_beyond_int32(oracle):
    # 139264 heads of 128 x 128 fp32 state: 2.28e9 state elements (9.1 GB) in place
    B, H, dk, dv = 1088, 128, 128, 128
    BH = B * H
    assert BH * dv * dk > 2**31
    w = wl.DRWorkload("edge", 1, 2, 1, dk, dv, wl.KDA, "fp32", s0_std=0.1)
    small = wl.generate_dr(w, 6)
    q = torch.zeros(B, H, dk, device="cuda")
    k, v = torch.zeros_like(q), torch.zeros(B, H, dv, device="cuda")
    beta = torch.full((B, H), 0.5, device="cuda")
    gate = torch.full((B, H, dk), 0.9, device="cuda")
    S = torch.zeros(B, H, dv, dk, device="cuda")
    for j, h in enumerate((0, BH - 1)):
        for name, t in (("q", q), ("k", k), ("v", v), ("beta", beta), ("gate", gate)):
            _fill_head(t, h, small[name][0, j, 0])
        _fill_head(S, h, small["S0"][0, j])
    out = drs.decode_step(q, k, v, beta, gate, S, mode="kda")
    torch.cuda.synchronize()
    ref_out, ref_S = oracle_dr(oracle, small)
    o = out.view(BH, dv)
    s = S.view(BH, dv, dk)
    for j, h in enumerate((0, BH - 1)):
        assert rel_err(tensor_np(o[h]), ref_out[0, j, 0]) <= TOL["fp32"]
        assert rel_err(tensor_np(s[h]), ref_S[0, j]) <= TOL["fp32"]
    for h in (1, BH // 2, BH - 2):
        assert torch.count_nonzero(o[h]) == 0 and torch.count_nonzero(s[h]) == 0
    del q, k, v, S, out, o, s
    torch.cuda.empty_cache()


# --- VLA: the chunked pair (default) and the per-token kernel (sequential=True)
@pytest.mark.parametrize("path", ["fused", "two_kernel", "sequential"])
@pytest.mark.parametrize("d", [32, 96])
def test_vla_workload(oracle, d, path):
    w = wl.workload(f"vla_fp32_d{d}")
    inputs = wl.generate_vla(w, 0)
    dev = {k: torch.from_numpy(inputs[k]).cuda() for k in ("q", "k", "v", "u")}
    out, Sf, Af = drs.vla_scan(dev["q"], dev["k"], dev["v"], dev["u"], lambda0=w.lambda0,
                               **VLA_PATHS[path])
    torch.cuda.synchronize()
    heads = [0, 9, 31]
    sub = wl.head_slice(inputs, heads)
    ref_out, ref_S, ref_A = oracle.vla_scan(sub["q"], sub["k"], sub["v"], sub["u"], lambda0=w.lambda0)
    o = tensor_np(out).reshape(32, w.T, d)[heads][None]
    s = tensor_np(Sf).reshape(32, d, d)[heads][None]
    a = tensor_np(Af).reshape(32, d, d)[heads][None]
    for got, ref in ((o, ref_out), (s, ref_S), (a, ref_A)):
        assert rel_err(got, ref) <= 1e-4
        assert row_rel_err(got, ref) <= 1e-4, row_rel_err(got, ref)


@pytest.mark.parametrize("path", ["fused", "two_kernel", "sequential"])
@pytest.mark.parametrize("d", [32, 64, 96, 128])
@pytest.mark.parametrize("T", [1, 17, 64, 65, 100, 129])
def test_vla_small_with_initial_state(oracle, d, T, path):
    rng = np.random.default_rng(d + T)
    B, H = 1, 3
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((B, H, T, d))).astype(np.float32)
    k = unit(rng.standard_normal((B, H, T, d))).astype(np.float32)
    v = rng.standard_normal((B, H, T, d)).astype(np.float32)
    u = (rng.standard_normal((B, H, T, d)) / np.sqrt(d)).astype(np.float32)
    S0 = (0.1 * rng.standard_normal((B, H, d, d))).astype(np.float32)
    M = rng.standard_normal((B, H, d, d)) / np.sqrt(d)
    A0 = np.linalg.inv(np.eye(d) + M @ np.swapaxes(M, -1, -2)).astype(np.float32)
    c = lambda x: torch.from_numpy(x).cuda()
    out, Sf, Af = drs.vla_scan(c(q), c(k), c(v), c(u), S0=c(S0), A0=c(A0), **VLA_PATHS[path])
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    ro, rs, ra = oracle.vla_scan(q, k, v, u, S0=S0, A0=A0)
    assert rel_err(tensor_np(out), ro) <= 1e-4
    assert rel_err(tensor_np(Sf), rs) <= 1e-4
    assert rel_err(tensor_np(Af), ra) <= 1e-4


def test_vla_empty_sequence_returns_initial_state():
    d = 32
    z = torch.empty(1, 2, 0, d, device="cuda")
    out, Sf, Af = drs.vla_scan(z, z, z, z, lambda0=4.0)
    torch.cuda.synchronize()
    eye = torch.eye(d, device="cuda") / 4.0
    assert torch.count_nonzero(Sf) == 0 and torch.allclose(Af, eye.expand_as(Af))


@pytest.mark.parametrize("d", [32, 96, 128])
def test_vla_chunked_long_sequence_with_state(oracle, d):
    # 1000 tokens: 15 full chunks and a ragged one, entering S0 and A0 (a positive definite
    # inverse penalty), every head against the oracle
    rng = np.random.default_rng(40 + d)
    B, H, T = 2, 2, 1000
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((B, H, T, d))).astype(np.float32)
    k = unit(rng.standard_normal((B, H, T, d))).astype(np.float32)
    v = rng.standard_normal((B, H, T, d)).astype(np.float32)
    u = (rng.standard_normal((B, H, T, d)) / np.sqrt(d)).astype(np.float32)
    S0 = (0.1 * rng.standard_normal((B, H, d, d))).astype(np.float32)
    M = rng.standard_normal((B, H, d, d)) / np.sqrt(d)
    A0 = np.linalg.inv(np.eye(d) + M @ np.swapaxes(M, -1, -2)).astype(np.float32)
    c = lambda x: torch.from_numpy(x).cuda()
    out, Sf, Af = drs.vla_scan(c(q), c(k), c(v), c(u), S0=c(S0), A0=c(A0))
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    ro, rs, ra = oracle.vla_scan(q, k, v, u, S0=S0, A0=A0)
    for got, ref in ((out, ro), (Sf, rs), (Af, ra)):
        assert rel_err(tensor_np(got), ref) <= 1e-4
        assert row_rel_err(tensor_np(got), ref) <= 1e-4


def test_vla_fused_many_clusters_d128(oracle):
    # 80 heads at d = 128: clusters of 5 CTAs, 400 CTAs in all, more than one wave on the
    # device; first, middle and last heads against the oracle
    w = wl.VLAWorkload("vla_many", B=4, H=20, T=150, d=128)
    inputs = wl.generate_vla(w, 12)
    dev = {k: torch.from_numpy(inputs[k]).cuda() for k in ("q", "k", "v", "u")}
    out, Sf, Af = drs.vla_scan(dev["q"], dev["k"], dev["v"], dev["u"])
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    heads = [0, 41, 79]
    sub = wl.head_slice(inputs, heads)
    ref = oracle.vla_scan(sub["q"], sub["k"], sub["v"], sub["u"])
    got = [tensor_np(t).reshape((80,) + tuple(t.shape[2:]))[heads][None] for t in (out, Sf, Af)]
    for g, r in zip(got, ref):
        assert rel_err(g, r) <= 1e-4


@pytest.mark.parametrize("d", [32, 64, 96, 128])
def test_vla_fused_equals_two_kernel_bitwise(d):
    # the fused kernel hands W and K A_c to the S-phase CTAs, which form alpha_hat with the
    # same code the two-kernel form's A-phase runs (two slot pairs up to d = 96, one at 128);
    # the arithmetic is the same, so every output must match bit for bit
    w = wl.VLAWorkload(f"vla_ratio_d{d}", B=2, H=4, T=700, d=d, ratio=True)
    inputs = wl.generate_vla(w, 9)
    dev = {k: torch.from_numpy(inputs[k]).cuda() for k in ("q", "k", "v", "u")}
    a = drs.vla_scan_ratio(dev["q"], dev["k"], dev["v"], dev["u"])
    b = drs.vla_scan_ratio(dev["q"], dev["k"], dev["v"], dev["u"], two_kernel=True)
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_vla_chunked_non_positive_definite_a0_is_reported():
    # A0 = -10 I is no inverse penalty: I + U A0 U^T has a negative pivot, which the chunked
    # kernel reports instead of returning numbers
    d, T = 32, 64
    rng = np.random.default_rng(5)
    x = torch.from_numpy((rng.standard_normal((1, 1, T, d)) / np.sqrt(d)).astype(np.float32)).cuda()
    A0 = -10.0 * torch.eye(d, device="cuda").expand(1, 1, d, d).contiguous()
    drs.vla_scan(x, x, x, x, A0=A0)
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_ERR_NOT_SPD
    assert drs.poll_error() == drs.DR_OK


# --- failure path: a bounded wait that runs out latches a status, nothing hangs
def test_timeout_is_reported_and_cleared():
    rc = drs.lib().dr_debug_timeout_probe(1000, drs._stream_handle(torch.device("cuda")))
    assert rc == drs.DR_OK
    assert drs.poll_error() == drs.DR_ERR_TIMEOUT
    assert drs.poll_error() == drs.DR_OK
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
