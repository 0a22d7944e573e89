"""Worked examples (``tests/golden/*.json``): tiny dyadic cases of every scan variant.

The inputs are dyadic rationals, so every intermediate value of the recurrence is exact
in fp64 and every input is exact in bf16. The stored expected values were written by
``tests/golden/make_golden.py`` from the oracle; here they are pinned against the same
cases worked by hand (the steps are in each fixture's ``derivation``), the oracle is
checked to reproduce them bit for bit, and (``-m gpu``) the CUDA paths run the same
inputs zero-padded to their supported sizes.

Sources: "Mechanisms, trade-offs and cross-layer routing of linear-attention
architectures" (aitrends.kr), section "Technical details" (delta rule, Gated DeltaNet,
Kimi Delta Attention); "Variational Linear Attention (VLA)" (gist.science 2605.11196),
sections 2.2-2.3.
"""
import json
import os

import numpy as np
import pytest

from helpers import rel_err

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
CASES = ["deltanet_d2_t2", "gdn_d2_t3", "kda_d2_t2", "gdn2_d2_t2", "vla_d3_t2",
         "vla_ratio_d3_t2"]

# The same cases worked by hand from the per-token definitions (fractions written out).
HAND = {
    # u: the write values beta_t r_t of the derivations' residuals r
    "deltanet_d2_t2": {
        "out": [[1, 0], [0, 2]],
        "S_final": [[1 / 2, -1 / 2], [1, 1]],
        "u": [[1, 0], [-1 / 2, 1]],
    },
    "gdn_d2_t3": {
        "out": [[1, 2], [5 / 2, 1], [1 / 16, 5 / 8]],
        "S_final": [[9 / 16, 1 / 2], [5 / 8, 0]],
        "u": [[1, 2], [2, 0], [7 / 16, 3 / 8]],
    },
    "kda_d2_t2": {
        "out": [[5 / 4, 9 / 4], [1 / 8, 5 / 4]],
        "S_final": [[3 / 4, 1 / 8], [5 / 4, 5 / 4]],
        "u": [[1 / 4, -1 / 4], [-1 / 8, 3 / 4]],
    },
    "gdn2_d2_t2": {
        "out": [[5 / 4, 1], [5 / 2, 9 / 4]],
        "S_final": [[2, 1 / 2], [2, 1 / 4]],
        "u": [[3 / 4, 1], [11 / 8, 3 / 2]],
    },
    "vla_d3_t2": {
        "out": [[1, 2, 3], [-1, -1, -3]],
        "S_final": [[1, -1, 0], [2, -1, 0], [3, -3, 0]],
        "A_final": [[3 / 4, -1 / 4, -1 / 4], [-1 / 4, 3 / 4, -1 / 4], [-1 / 4, -1 / 4, 3 / 4]],
    },
    "vla_ratio_d3_t2": {
        "out": [[1, 2, 3], [1 / 2, 3 / 2, 3 / 2]],
        "S_final": [[1, -2, 0], [2, -3, 0], [3, -6, 0]],
        "A_final": [[3 / 4, -1 / 4, -1 / 4], [-1 / 4, 3 / 4, -1 / 4], [-1 / 4, -1 / 4, 3 / 4]],
        "n_final": [1, -1, 0],
    },
}


def load(name):
    with open(os.path.join(GOLDEN, name + ".json")) as f:
        return json.load(f)


def bh(x):
    return np.asarray(x, np.float64)[None, None]


def run_oracle(oracle, fx, residual_pre_decay=False):
    x = fx["inputs"]
    if fx["mode"] == "vla":
        out, Sf, Af = oracle.vla_scan(bh(x["q"]), bh(x["k"]), bh(x["v"]), bh(x["u"]),
                                      lambda0=x["lambda0"])
        return {"out": out[0, 0], "S_final": Sf[0, 0], "A_final": Af[0, 0]}
    if fx["mode"] == "vla_ratio":
        out, Sf, Af, nf = oracle.vla_scan_ratio(bh(x["q"]), bh(x["k"]), bh(x["v"]), bh(x["u"]),
                                                lambda0=x["lambda0"])
        return {"out": out[0, 0], "S_final": Sf[0, 0], "A_final": Af[0, 0], "n_final": nf[0, 0]}
    mode = {"deltanet": oracle.DELTANET, "gdn": oracle.GDN, "kda": oracle.KDA,
            "gdn2": oracle.GDN2}[fx["mode"]]
    beta = np.asarray(x["beta"], np.float64)[None, None]
    gate = bh(x["gate"]) if "gate" in x else None
    S0 = np.asarray(x["S0"], np.float64)[None, None] if "S0" in x else None
    erase = bh(x["erase"]) if "erase" in x else None
    write = bh(x["write"]) if "write" in x else None
    out, Sf, u = oracle.dr_scan_ex(bh(x["q"]), bh(x["k"]), bh(x["v"]), beta, gate, S0, mode,
                                   erase=erase, write=write,
                                   residual_pre_decay=residual_pre_decay)
    return {"out": out[0, 0], "S_final": Sf[0, 0], "u": u[0, 0]}


@pytest.mark.parametrize("name", CASES)
def test_fixture_matches_the_hand_derivation(name):
    fx = load(name)
    assert fx["cite"] and fx["derivation"]
    for key, want in HAND[name].items():
        assert np.array_equal(np.asarray(fx["expected"][key]), np.asarray(want, np.float64)), key


@pytest.mark.parametrize("name", CASES)
def test_oracle_reproduces_the_fixture_exactly(oracle, name):
    fx = load(name)
    got = run_oracle(oracle, fx)
    for key, want in fx["expected"].items():
        assert np.array_equal(got[key], np.asarray(want)), key


def test_gdn2_example_recalls_its_write_target():
    # the reading's exact-recall property on the worked example: at t = 2, beta = 1 and
    # e2 = (1,0) is a unit vector, so S2 e2 = z2 = w2 (.) v2 = (2, 2)
    fx = load("gdn2_d2_t2")
    S2 = np.asarray(fx["expected"]["S_final"])
    assert np.array_equal(S2 @ np.array([1.0, 0.0]), [2.0, 2.0])


def test_gdn_example_separates_the_two_residual_readings(oracle):
    # Residual against the undecayed state at t = 3: r = (1,1) - S2 k3 = (1/2, 0), so
    # S3 = [[3/8, 1/2], [1/4, 0]] and o3 = (-1/8, 1/4); the first two steps agree.
    fx = load("gdn_d2_t3")
    got = run_oracle(oracle, fx, residual_pre_decay=True)
    assert np.array_equal(got["S_final"], [[3 / 8, 1 / 2], [1 / 4, 0]])
    assert np.array_equal(got["out"], [[1, 2], [5 / 2, 1], [-1 / 8, 1 / 4]])


# --- the CUDA paths on the same inputs -------------------------------------------------
@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import delta_rule_recurrent_chunked_b200 as drs

    drs.lib()
    yield torch, drs
    assert drs.poll_error() == drs.DR_OK


def pad(x, shape, fill=0.0):
    a = np.full(shape, fill, np.float64)
    x = np.asarray(x, np.float64)
    a[tuple(slice(0, n) for n in x.shape)] = x
    return a


def bf16_tensor(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["deltanet_d2_t2", "gdn_d2_t3", "kda_d2_t2", "gdn2_d2_t2"])
@pytest.mark.parametrize("path", ["fp32_sequential", "bf16_chunked"])
def test_cuda_scan_on_the_worked_examples(cuda, name, path):
    torch, drs = cuda
    fx = load(name)
    x = fx["inputs"]
    T, d = np.asarray(x["q"]).shape
    dk, dv = (32, 32) if path == "fp32_sequential" else (128, 32)
    assert drs.chunked_applies(fx["mode"], path == "bf16_chunked", dk, dv) == (path == "bf16_chunked")
    q, k = pad(x["q"], (T, dk)), pad(x["k"], (T, dk))
    v = pad(x["v"], (T, dv))
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32))[None, None].cuda()
    if path == "fp32_sequential":
        tq, tk, tv = f32(q), f32(k), f32(v)
    else:
        tq, tk, tv = (bf16_tensor(torch, a)[None, None].cuda() for a in (q, k, v))
    beta = torch.tensor(x["beta"], dtype=torch.float32, device="cuda")[None, None]
    gate = erase = write = None
    if fx["mode"] in ("gdn", "gdn2"):
        gate = torch.tensor(x["gate"], dtype=torch.float32, device="cuda")[None, None]
    elif fx["mode"] == "kda":
        gate = f32(pad(x["gate"], (T, dk), fill=1.0))
    if fx["mode"] == "gdn2":
        erase, write = f32(pad(x["erase"], (T, dk))), f32(pad(x["write"], (T, dv)))
    S0 = f32(pad(x["S0"], (dv, dk))) if "S0" in x else None
    out, Sf, u = drs.scan_ex(tq, tk, tv, beta, gate, S0, mode=fx["mode"], erase=erase,
                             write=write, force_sequential=path == "fp32_sequential")
    torch.cuda.synchronize()
    out, Sf, u = (a.double().cpu().numpy()[0, 0] for a in (out, Sf, u))
    tol = 1e-4 if path == "fp32_sequential" else 2e-2
    for got, key in ((out[:, :d], "out"), (Sf[:d, :d], "S_final"), (u[:, :d], "u")):
        assert rel_err(got, np.asarray(fx["expected"][key])) <= tol, key
    # zero key and value channels receive nothing from the real ones
    assert not np.any(out[:, d:]) and not np.any(Sf[d:, :]) and not np.any(Sf[:, d:])
    assert not np.any(u[:, d:])


@pytest.mark.gpu
def test_cuda_vla_on_the_worked_example(cuda):
    torch, drs = cuda
    fx = load("vla_d3_t2")
    x = fx["inputs"]
    T, d = np.asarray(x["q"]).shape
    D = 32
    t = lambda a: torch.from_numpy(np.ascontiguousarray(pad(a, (T, D)), np.float32))[None, None].cuda()
    out, Sf, Af = drs.vla_scan(t(x["q"]), t(x["k"]), t(x["v"]), t(x["u"]), lambda0=x["lambda0"])
    torch.cuda.synchronize()
    out, Sf, Af = (a.double().cpu().numpy()[0, 0] for a in (out, Sf, Af))
    for got, key in ((out[:, :d], "out"), (Sf[:d, :d], "S_final"), (Af[:d, :d], "A_final")):
        assert rel_err(got, np.asarray(fx["expected"][key])) <= 1e-4, key
    assert not np.any(out[:, d:]) and not np.any(Sf[d:, :]) and not np.any(Sf[:, d:])
    eye = np.eye(D)
    assert np.allclose(Af[d:, d:], eye[d:, d:]) and not np.any(Af[:d, d:]) and not np.any(Af[d:, :d])


@pytest.mark.gpu
def test_cuda_vla_ratio_on_the_worked_example(cuda):
    torch, drs = cuda
    fx = load("vla_ratio_d3_t2")
    x = fx["inputs"]
    T, d = np.asarray(x["q"]).shape
    D = 32
    t = lambda a: torch.from_numpy(np.ascontiguousarray(pad(a, (T, D)), np.float32))[None, None].cuda()
    got = drs.vla_scan_ratio(t(x["q"]), t(x["k"]), t(x["v"]), t(x["u"]), lambda0=x["lambda0"])
    torch.cuda.synchronize()
    out, Sf, Af, nf = (a.double().cpu().numpy()[0, 0] for a in got)
    for g, key in ((out[:, :d], "out"), (Sf[:d, :d], "S_final"), (Af[:d, :d], "A_final"),
                   (nf[:d], "n_final")):
        assert rel_err(g, np.asarray(fx["expected"][key])) <= 1e-4, key
    assert not np.any(nf[d:]) and not np.any(out[:, d:])
