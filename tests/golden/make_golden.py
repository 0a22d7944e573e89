"""Write the worked-example fixtures in this folder (``*.json``).

Each fixture is a tiny hand-chosen case whose inputs are dyadic rationals: every
intermediate value of the recurrence is then exact in fp64, and the inputs are exact
in bf16, so the same case checks the fp64 oracle bit for bit and the CUDA paths within
their tolerances. The stored expected values are written here by calling the oracle
only; ``tests/test_golden.py`` pins them against a derivation by hand (the steps are
also stored in each fixture) and runs the CUDA paths on the same inputs.

Run from the repository root:  python tests/golden/make_golden.py
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402  (test infrastructure: the only import this script makes)

DR_PAGE = ('"Mechanisms, trade-offs and cross-layer routing of linear-attention architectures" '
           '(aitrends.kr), section "Technical details": delta-rule write with residual '
           'r = v - W kappa, gated (scalar alpha) and per-key-channel (Kimi) decays')
VLA_PAGE = ('"Variational Linear Attention (VLA)" (gist.science 2605.11196), sections 2.2-2.3: '
            'Sherman-Morrison update of A = M^-1, alpha_hat = A k_hat / ||A k_hat||, '
            'S_t = S_{t-1} + (v - S_{t-1} k_hat) alpha_hat^T')

GDN2_PAGE = ('"Mechanisms, trade-offs and cross-layer routing of linear-attention architectures" '
             '(aitrends.kr), sections "Methodology" and "Technical details": Gated DeltaNet-2 '
             'with per-channel erase b and write w, e = b (.) kappa, z = w (.) v, residual '
             'r = z - W~ e (W~ the decayed memory), written along e')

VLA_RATIO_PAGE = VLA_PAGE + ('; section 2.3: the output is a ratio of recurrences, as in linear '
                             'attention; the denominator is the same write on a value held at 1, '
                             'n_t = n_{t-1} + (1 - n_{t-1} k_hat) alpha_hat^T, o_t = S_t q / (n_t q)')

CASES = {
    "deltanet_d2_t2": dict(
        mode=oracle.DELTANET,
        cite=DR_PAGE + "; DeltaNet (alpha = 1)",
        q=[[1, 0], [1, 1]], k=[[1, 0], [1, 1]], v=[[2, 0], [0, 2]], beta=[0.5, 0.5],
        derivation=[
            "t=1: S0 = 0, r = v1 = (2,0), S1 = 1/2 (2,0)^T (1,0) = [[1,0],[0,0]], o1 = S1 q1 = (1,0)",
            "t=2: S1 k2 = (1,0), r = (0,2) - (1,0) = (-1,2), "
            "S2 = S1 + 1/2 (-1,2)^T (1,1) = [[1/2,-1/2],[1,1]], o2 = S2 (1,1) = (0,2)",
        ]),
    "gdn_d2_t3": dict(
        mode=oracle.GDN,
        cite=DR_PAGE + "; Gated DeltaNet, residual against the decayed state",
        q=[[1, 0], [1, 1], [1, -1]], k=[[1, 0], [0, 1], [1, 0]], v=[[2, 4], [4, 0], [1, 1]],
        beta=[0.5, 0.5, 0.5], gate=[0.5, 0.5, 0.25],
        derivation=[
            "t=1: S1 = 1/2 (2,4)^T (1,0) = [[1,0],[2,0]], o1 = (1,2)",
            "t=2: alpha S1 = [[1/2,0],[1,0]], (alpha S1) k2 = (0,0), r = (4,0), "
            "S2 = [[1/2,2],[1,0]], o2 = S2 (1,1) = (5/2,1)",
            "t=3: alpha S2 = [[1/8,1/2],[1/4,0]], (alpha S2) k3 = (1/8,1/4), r = (7/8,3/4), "
            "S3 = [[9/16,1/2],[5/8,0]], o3 = S3 (1,-1) = (1/16,5/8)",
            "(residual against the undecayed state instead: r3 = (1,1) - S2 k3 = (1/2,0), "
            "S3 = [[3/8,1/2],[1/4,0]], o3 = (-1/8,1/4))",
        ]),
    "kda_d2_t2": dict(
        mode=oracle.KDA,
        cite=DR_PAGE + "; Kimi Delta Attention, alpha scales the key-channel columns of S",
        q=[[1, 1], [0, 1]], k=[[1, 0], [0, 1]], v=[[1, 1], [0, 2]], beta=[0.5, 0.5],
        gate=[[0.5, 0.25], [1.0, 0.5]], S0=[[1, 2], [3, 4]],
        derivation=[
            "t=1: S0 diag(1/2,1/4) = [[1/2,1/2],[3/2,1]], its k1 column (1/2,3/2), r = (1/2,-1/2), "
            "S1 = [[3/4,1/2],[5/4,1]], o1 = S1 (1,1) = (5/4,9/4)",
            "t=2: S1 diag(1,1/2) = [[3/4,1/4],[5/4,1/2]], its k2 column (1/4,1/2), r = (-1/4,3/2), "
            "S2 = [[3/4,1/8],[5/4,5/4]], o2 = S2 (0,1) = (1/8,5/4)",
        ]),
    "gdn2_d2_t2": dict(
        mode=oracle.GDN2,
        cite=GDN2_PAGE,
        q=[[1, 0], [1, 1]], k=[[1, 1], [1, 0]], v=[[2, 4], [4, 2]], beta=[0.5, 1.0],
        gate=[0.5, 0.5], erase=[[1, 0], [1, 1]], write=[[1, 0.5], [0.5, 1]], S0=[[1, 2], [0, 1]],
        derivation=[
            "t=1: e = b (.) k = (1,0), z = w (.) v = (2,2), W~ = S0/2 = [[1/2,1],[0,1/2]], "
            "W~ e = (1/2,0), r = (3/2,2), u = beta r = (3/4,1), S1 = W~ + u e^T = [[5/4,1],[1,1/2]], "
            "o1 = S1 (1,0) = (5/4,1)",
            "t=2: e = (1,0), z = (2,2), W~ = S1/2 = [[5/8,1/2],[1/2,1/4]], W~ e = (5/8,1/2), "
            "r = (11/8,3/2), u = r (beta = 1), S2 = [[2,1/2],[2,1/4]] (S2 e = z), "
            "o2 = S2 (1,1) = (5/2,9/4)",
            "(written along k instead of e: S1 = W~ + u k1^T = [[5/4,7/4],[1,3/2]])",
        ]),
    "vla_d3_t2": dict(
        mode="vla",
        cite=VLA_PAGE,
        q=[[1, 1, 1], [0, 1, 1]], k=[[2, 1, 1], [1, 2, 1]], v=[[1, 2, 3], [0, 1, 0]],
        u=[[1, 1, 1], [0, 0, 0]], lambda0=1.0,
        derivation=[
            "t=1: A0 = I, z = A0 u1 = (1,1,1), 1 + u1.z = 4, A1 = I - J/4 (J all ones); "
            "A1 k1 = (1,0,0), alpha_hat = e1, S1 = (1,2,3)^T e1^T, o1 = S1 q1 = (1,2,3)",
            "t=2: u2 = 0 leaves A2 = A1; A2 k2 = (0,1,0), alpha_hat = e2, S1 k2 = (1,2,3), "
            "r = (0,1,0) - (1,2,3) = (-1,-1,-3), S2 = S1 + r e2^T = [[1,-1,0],[2,-1,0],[3,-3,0]], "
            "o2 = S2 (0,1,1) = (-1,-1,-3)",
        ]),
    "vla_ratio_d3_t2": dict(
        mode="vla_ratio",
        cite=VLA_RATIO_PAGE,
        q=[[1, 1, 1], [3, 1, 1]], k=[[2, 1, 1], [2, 4, 2]], v=[[1, 2, 3], [0, 1, 0]],
        u=[[1, 1, 1], [0, 0, 0]], lambda0=1.0,
        derivation=[
            "t=1: as vla_d3_t2, A1 = I - J/4, A1 k1 = (1,0,0), alpha_hat = e1, S1 = (1,2,3)^T e1^T; "
            "n1 = 0 + (1 - 0) e1 = e1, n1 q1 = 1, o1 = S1 q1 / 1 = (1,2,3)",
            "t=2: u2 = 0 leaves A2 = A1; A2 k2 = (0,2,0), alpha_hat = e2, S1 k2 = (2,4,6), "
            "r = (-2,-3,-6), S2 = [[1,-2,0],[2,-3,0],[3,-6,0]]; n1 k2 = 2, n2 = e1 + (1-2) e2 "
            "= (1,-1,0); S2 q2 = (1,3,3), n2 q2 = 2, o2 = (1/2,3/2,3/2)",
        ]),
}


def _bh(x):
    """A [T, ...] list as a [1, 1, T, ...] float64 array."""
    return np.asarray(x, np.float64)[None, None]


def build_case(name: str, spec: dict) -> dict:
    fx = {"case": name, "cite": spec["cite"], "derivation": spec["derivation"],
          "mode": spec["mode"] if spec["mode"] in ("vla", "vla_ratio") else
          {oracle.DELTANET: "deltanet", oracle.GDN: "gdn", oracle.KDA: "kda",
           oracle.GDN2: "gdn2"}[spec["mode"]]}
    inputs = {key: spec[key] for key in ("q", "k", "v", "beta", "gate", "erase", "write", "S0",
                                         "u", "lambda0")
              if key in spec}
    fx["inputs"] = inputs
    if spec["mode"] == "vla":
        out, Sf, Af = oracle.vla_scan(_bh(spec["q"]), _bh(spec["k"]), _bh(spec["v"]),
                                      _bh(spec["u"]), lambda0=spec["lambda0"])
        fx["expected"] = {"out": out[0, 0].tolist(), "S_final": Sf[0, 0].tolist(),
                          "A_final": Af[0, 0].tolist()}
    elif spec["mode"] == "vla_ratio":
        out, Sf, Af, nf = oracle.vla_scan_ratio(_bh(spec["q"]), _bh(spec["k"]), _bh(spec["v"]),
                                                _bh(spec["u"]), lambda0=spec["lambda0"])
        fx["expected"] = {"out": out[0, 0].tolist(), "S_final": Sf[0, 0].tolist(),
                          "A_final": Af[0, 0].tolist(), "n_final": nf[0, 0].tolist()}
    else:
        beta = np.asarray(spec["beta"], np.float64)[None, None]
        gate = None if "gate" not in spec else _bh(spec["gate"])
        S0 = None if "S0" not in spec else np.asarray(spec["S0"], np.float64)[None, None]
        erase = None if "erase" not in spec else _bh(spec["erase"])
        write = None if "write" not in spec else _bh(spec["write"])
        out, Sf, u = oracle.dr_scan_ex(_bh(spec["q"]), _bh(spec["k"]), _bh(spec["v"]), beta, gate,
                                       S0, spec["mode"], erase=erase, write=write)
        # u: the per-token write values beta_t r_t
        fx["expected"] = {"out": out[0, 0].tolist(), "S_final": Sf[0, 0].tolist(),
                          "u": u[0, 0].tolist()}
    return fx


def main() -> None:
    for name, spec in CASES.items():
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(build_case(name, spec), f, indent=1)
            f.write("\n")
        print("wrote", name + ".json")


if __name__ == "__main__":
    main()
