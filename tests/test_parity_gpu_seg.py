"""GPU parity of the segmented scan of Gated DeltaNet and KDA (few heads, long sequences).

dr_scan_fwd cuts each head into segments that run at once from zero states; every segment
but the last runs eight chunks on into the next one, carrying its state, and writes the
outputs there. The zero-start outputs after that window are kept only where a device-side
check shows the two states at the window's end agree (and no token's step could grow a
difference); otherwise the chained kernel reruns the call. These tests pin
both outcomes against the fp64 oracle at the bf16 tolerance (2e-2, max|x - y| / max|y|), and
pin the fallback against the chained kernel bit for bit.
"""
import numpy as np
import pytest

import delta_rule_recurrent_chunked_b200 as drs
from delta_rule_recurrent_chunked_b200 import workloads as wl

from helpers import oracle_dr, oracle_dr_ex, rel_err, tensor_np, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    drs.lib()
    yield
    assert drs.poll_error() == drs.DR_OK


def _scan(dev, mode, chained=False, want_u=False):
    out, Sf, u = drs.scan_ex(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                             mode=mode, erase=dev["erase"], write=dev["write"], want_u=want_u,
                             chained=chained)
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    return out, Sf, u


def test_plan_segments_only_gated_deltanet_with_few_heads():
    plan = drs.chunked_plan_ex
    assert plan("gdn", 16, 8192, 128, 128) == (64, 2, 2)
    assert plan("gdn", 16, 4096, 128, 128)[2] == 2
    assert plan("gdn", 16, 32768, 128, 128)[2] == 2
    assert plan("gdn", 2, 32768, 128, 128)[2] == 16
    assert plan("gdn", 1, 8192, 128, 128)[2] == 4
    assert plan("gdn2", 16, 8192, 128, 128)[2] == 2
    # the chained plan is kept when asked for, when the heads already fill the GPU, for a T
    # that is not a multiple of 64 or too short to cut in two, and for the other variants
    assert plan("gdn", 16, 8192, 128, 128, chained=True) == drs.chunked_plan("gdn", 16, 128, 128) + (1,)
    assert plan("gdn", 32, 32768, 128, 128)[2] == 1
    assert plan("gdn", 16, 4096 + 64, 128, 128)[2] == 1
    assert plan("gdn", 2, 4095, 128, 128)[2] == 1
    assert plan("gdn", 2, 4096 - 64, 128, 128)[2] == 1
    # DeltaNet: a 48-chunk window, segments of at least 96 chunks
    assert plan("deltanet", 16, 32768, 128, 128) == (64, 2, 2)
    assert plan("deltanet", 2, 32768, 128, 128)[2] == 4
    assert plan("deltanet", 16, 8192, 128, 128)[2] == 1
    # KDA: one CTA per segment with every value channel
    assert plan("kda", 16, 32768, 128, 128) == (128, 0, 8)
    assert plan("kda", 2, 32768, 128, 128) == (128, 0, 16)
    assert plan("kda", 4, 8192, 128, 64) == (64, 0, 4)
    assert plan("kda", 128, 4096, 128, 128)[2] == 1


@pytest.mark.parametrize("B,H,T,s0", [(1, 2, 8192, True), (1, 2, 16384, False), (2, 3, 8192, True),
                                      (1, 1, 16384, True), (1, 16, 4096, True)])
def test_segmented_gdn_matches_oracle(oracle, B, H, T, s0):
    w = wl.DRWorkload("gdn_seg", B, H, T, 128, 128, wl.GDN, "bf16", s0_std=0.1 if s0 else 0.0)
    assert drs.chunked_plan_ex("gdn", B * H, T, 128, 128)[2] > 1
    inputs = wl.generate_dr(w, seed=3)
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, _ = _scan(dev, "gdn")
    # the checks passed: the zero-start outputs after the window were kept, nothing reran
    after = drs.segment_counters()
    assert (after[0] - before[0], after[1] - before[1]) == (1, 0)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= TOL and e_S <= TOL, (e_out, e_S)
    out_c, Sf_c, _ = _scan(dev, "gdn", chained=True)
    assert rel_err(tensor_np(out), tensor_np(out_c)) <= 1e-2
    assert rel_err(tensor_np(Sf), tensor_np(Sf_c)) <= 1e-2


def _fallback_equals_chained(oracle, inputs):
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, _ = _scan(dev, "gdn")
    after = drs.segment_counters()
    assert (after[0] - before[0], after[1] - before[1]) == (1, 1)
    out_c, Sf_c, _ = _scan(dev, "gdn", chained=True)
    assert torch.equal(out, out_c) and torch.equal(Sf, Sf_c)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= TOL and e_S <= TOL, (e_out, e_S)


# gates all but 1: the state difference barely decays over the window, the check fails and
# the chained kernel recomputes the call
def test_weak_decay_falls_back_to_the_chained_scan(oracle):
    w = wl.DRWorkload("gdn_weak", 1, 2, 8192, 128, 128, wl.GDN, "bf16", s0_std=0.1,
                      gate_mu=-12.0)
    _fallback_equals_chained(oracle, wl.generate_dr(w, seed=4))


# one token whose step can grow a difference (beta |k|^2 = 3.6 > 2), with the usual decay
# that would pass the hand-off check on its own
def test_expanding_step_falls_back_to_the_chained_scan(oracle):
    w = wl.DRWorkload("gdn_expand", 1, 2, 8192, 128, 128, wl.GDN, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, seed=5)
    inputs["k"][0, 1, 2900] *= 2.0  # bf16 values: exact
    inputs["k_raw"] = wl.bf16_bits(inputs["k"])
    inputs["beta"][0, 1, 2900] = 0.9
    _fallback_equals_chained(oracle, inputs)


# a gate above 1 on one token (outside the documented range, still computed by the chained
# kernel): the segmented result is not used
def test_gate_above_one_falls_back_to_the_chained_scan(oracle):
    w = wl.DRWorkload("gdn_gate_gt1", 1, 2, 8192, 128, 128, wl.GDN, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, seed=6)
    inputs["gate"][0, 0, 3000] = 1.2
    _fallback_equals_chained(oracle, inputs)


def test_segmented_write_values_and_gdn2(oracle):
    for mode in (wl.GDN, wl.GDN2):
        w = wl.DRWorkload("seg_ex", 1, 2, 8192, 128, 128, mode, "bf16", s0_std=0.1)
        inputs = wl.generate_dr(w, seed=7)
        dev = to_device(inputs)
        name = "gdn" if mode == wl.GDN else "gdn2"
        assert drs.chunked_plan_ex(name, 2, 8192, 128, 128)[2] > 1
        before = drs.segment_counters()
        out, Sf, u = _scan(dev, name, want_u=True)
        after = drs.segment_counters()
        assert (after[0] - before[0], after[1] - before[1]) == (1, 0)
        ref_out, ref_S, ref_u = oracle_dr_ex(oracle, inputs)
        errs = (rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S),
                rel_err(tensor_np(u), ref_u))
        assert max(errs) <= TOL, (name, errs)


# the segmented call leaves nothing behind that changes the next call: two calls in a row,
# and a chained call between them, give the same result
def test_segmented_calls_in_a_row_agree():
    w = wl.DRWorkload("gdn_seg_rep", 1, 4, 8192, 128, 128, wl.GDN, "bf16", s0_std=0.1)
    dev = to_device(wl.generate_dr(w, seed=8))
    a = _scan(dev, "gdn")
    _scan(dev, "gdn", chained=True)
    b = _scan(dev, "gdn")
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# without S_final the check kernel has no final state to copy; the outputs are unchanged
def test_segmented_without_final_state(oracle):
    w = wl.DRWorkload("gdn_seg_nostate", 1, 2, 8192, 128, 128, wl.GDN, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, seed=9)
    dev = to_device(inputs)
    out, Sf, _ = drs.scan_ex(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"], dev["S0"],
                             mode="gdn", want_state=False, want_u=False)
    torch.cuda.synchronize()
    assert Sf is None and drs.poll_error() == drs.DR_OK
    ref_out, _ = oracle_dr(oracle, inputs)
    assert rel_err(tensor_np(out), ref_out) <= TOL
    out2, _, _ = _scan(dev, "gdn")
    assert torch.equal(out, out2)


# two segmented calls in flight on two streams take scratch of their own
def test_segmented_calls_on_two_streams(oracle):
    ws = [wl.DRWorkload(f"gdn_seg_s{i}", 1, 2, 8192, 128, 128, wl.GDN, "bf16", s0_std=0.1)
          for i in range(2)]
    inputs = [wl.generate_dr(w, seed=20 + i) for i, w in enumerate(ws)]
    devs = [to_device(x) for x in inputs]
    streams = [torch.cuda.Stream() for _ in devs]
    torch.cuda.synchronize()
    results = []
    for dev, st in zip(devs, streams):
        with torch.cuda.stream(st):
            results.append(drs.scan(dev["q"], dev["k"], dev["v"], dev["beta"], dev["gate"],
                                    dev["S0"], mode="gdn"))
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    for x, (out, Sf) in zip(inputs, results):
        ref_out, ref_S = oracle_dr(oracle, x)
        assert rel_err(tensor_np(out), ref_out) <= TOL and rel_err(tensor_np(Sf), ref_S) <= TOL


# narrower value heads run the segment launch on the split instances with 32 and 16 value
# channels per chain CTA
@pytest.mark.parametrize("dv", [32, 64])
def test_segmented_gdn_narrow_values(oracle, dv):
    w = wl.DRWorkload("gdn_seg_dv", 1, 4, 8192, 128, dv, wl.GDN, "bf16", s0_std=0.1)
    plan = drs.chunked_plan_ex("gdn", 4, 8192, 128, dv)
    assert plan[0] == dv // 2 and plan[2] > 1, plan
    inputs = wl.generate_dr(w, seed=10 + dv)
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, _ = _scan(dev, "gdn")
    after = drs.segment_counters()
    assert (after[0] - before[0], after[1] - before[1]) == (1, 0)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= TOL and e_S <= TOL, (dv, e_out, e_S)


# KDA: the segment launch is the unsplit kernel with every value channel in one CTA
@pytest.mark.parametrize("H,T,dv,s0", [(2, 8192, 128, True), (4, 8192, 64, False),
                                       (1, 16384, 128, True)])
def test_segmented_kda_matches_oracle(oracle, H, T, dv, s0):
    w = wl.DRWorkload("kda_seg", 1, H, T, 128, dv, wl.KDA, "bf16", s0_std=0.1 if s0 else 0.0)
    assert drs.chunked_plan_ex("kda", H, T, 128, dv)[2] > 1
    inputs = wl.generate_dr(w, seed=30 + H)
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, _ = _scan(dev, "kda")
    after = drs.segment_counters()
    assert (after[0] - before[0], after[1] - before[1]) == (1, 0)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= TOL and e_S <= TOL, (e_out, e_S)
    out_c, Sf_c, _ = _scan(dev, "kda", chained=True)
    assert rel_err(tensor_np(out), tensor_np(out_c)) <= 1e-2
    assert rel_err(tensor_np(Sf), tensor_np(Sf_c)) <= 1e-2


def _kda_fallback_equals_chained(oracle, inputs):
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, _ = _scan(dev, "kda")
    after = drs.segment_counters()
    assert (after[0] - before[0], after[1] - before[1]) == (1, 1)
    out_c, Sf_c, _ = _scan(dev, "kda", chained=True)
    assert torch.equal(out, out_c) and torch.equal(Sf, Sf_c)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= TOL and e_S <= TOL, (e_out, e_S)


# per-channel gates all but 1: too little decay over the window, the chained kernel reruns
def test_kda_weak_decay_falls_back_to_the_chained_scan(oracle):
    w = wl.DRWorkload("kda_weak", 1, 2, 8192, 128, 128, wl.KDA, "bf16", s0_std=0.1,
                      gate_mu=-12.0)
    _kda_fallback_equals_chained(oracle, wl.generate_dr(w, seed=40))


# one channel of one token's gate above 1
def test_kda_gate_above_one_falls_back_to_the_chained_scan(oracle):
    w = wl.DRWorkload("kda_gt1", 1, 2, 8192, 128, 128, wl.KDA, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, seed=41)
    inputs["gate"][0, 1, 5000, 17] = 1.2
    _kda_fallback_equals_chained(oracle, inputs)


# one token whose step can grow a difference (beta |k|^2 = 3.6 > 2)
def test_kda_expanding_step_falls_back_to_the_chained_scan(oracle):
    w = wl.DRWorkload("kda_expand", 1, 2, 8192, 128, 128, wl.KDA, "bf16", s0_std=0.1)
    inputs = wl.generate_dr(w, seed=42)
    inputs["k"][0, 0, 6000] *= 2.0  # bf16 values: exact
    inputs["k_raw"] = wl.bf16_bits(inputs["k"])
    inputs["beta"][0, 0, 6000] = 0.9
    _kda_fallback_equals_chained(oracle, inputs)


# DeltaNet has no gate: the hand-off difference shrinks only along the keys written, over a
# 48-chunk window
@pytest.mark.parametrize("H,T", [(2, 16384), (2, 32768)])
def test_segmented_deltanet_matches_oracle(oracle, H, T):
    w = wl.DRWorkload("deltanet_seg", 1, H, T, 128, 128, wl.DELTANET, "bf16", s0_std=0.1)
    assert drs.chunked_plan_ex("deltanet", H, T, 128, 128)[2] > 1
    inputs = wl.generate_dr(w, seed=50 + H)
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, _ = _scan(dev, "deltanet")
    after = drs.segment_counters()
    assert (after[0] - before[0], after[1] - before[1]) == (1, 0)
    ref_out, ref_S = oracle_dr(oracle, inputs)
    e_out, e_S = rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S)
    assert e_out <= TOL and e_S <= TOL, (e_out, e_S)


# the write values through the segment launch of every variant, and DR_CHAINED leaving the
# segment counters alone
@pytest.mark.parametrize("mode,T", [(wl.KDA, 8192), (wl.DELTANET, 16384)])
def test_segmented_write_values_kda_deltanet(oracle, mode, T):
    name = "kda" if mode == wl.KDA else "deltanet"
    w = wl.DRWorkload("seg_u", 1, 2, T, 128, 128, mode, "bf16", s0_std=0.1)
    assert drs.chunked_plan_ex(name, 2, T, 128, 128)[2] > 1
    inputs = wl.generate_dr(w, seed=60 + mode)
    dev = to_device(inputs)
    before = drs.segment_counters()
    out, Sf, u = _scan(dev, name, want_u=True)
    mid = drs.segment_counters()
    assert (mid[0] - before[0], mid[1] - before[1]) == (1, 0)
    ref_out, ref_S, ref_u = oracle_dr_ex(oracle, inputs)
    errs = (rel_err(tensor_np(out), ref_out), rel_err(tensor_np(Sf), ref_S),
            rel_err(tensor_np(u), ref_u))
    assert max(errs) <= TOL, (name, errs)
    _scan(dev, name, chained=True, want_u=True)
    assert drs.segment_counters() == mid
