"""Shared test helpers: device upload of generated workloads, oracle references, metrics."""
from __future__ import annotations

import numpy as np

from delta_rule_recurrent_chunked_b200 import workloads as wl

MODE_NAME = {wl.LINEAR: "linear", wl.DELTANET: "deltanet", wl.GDN: "gdn", wl.KDA: "kda",
             wl.GDN2: "gdn2"}


def rel_err(x, y) -> float:
    """max|x - y| / max|y| over a whole tensor (the tolerance metric for out and S_final)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    if y.size == 0:
        return 0.0
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-30))


def row_rel_err(x, y, floor=1e-3) -> float:
    """Row-wise relative error: the largest, over rows (last axis), of max|x - y| over the
    row divided by max|y| over the row, with that denominator floored at floor * max|y| of
    the whole tensor (a row whose reference is all but zero is measured against the tensor's
    scale instead). Stricter than rel_err for rows of small magnitude."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    if y.size == 0:
        return 0.0
    x = x.reshape(-1, y.shape[-1])
    y = y.reshape(-1, y.shape[-1])
    scale = max(float(np.max(np.abs(y))), 1e-30)
    den = np.maximum(np.max(np.abs(y), axis=1), floor * scale)
    return float(np.max(np.max(np.abs(x - y), axis=1) / den))


def to_device(inputs: dict, device="cuda"):
    """Upload a generated delta-rule workload: returns a dict of torch tensors."""
    import torch

    w = inputs["workload"]
    dev = {}
    for name in ("q", "k", "v"):
        raw = inputs[name + "_raw"]
        if w.dtype == "bf16":
            t = torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(raw))
        dev[name] = t.to(device)
    for name in ("beta", "gate", "S0", "erase", "write"):
        arr = inputs.get(name)
        dev[name] = None if arr is None else torch.from_numpy(np.ascontiguousarray(arr)).to(device)
    return dev


def oracle_dr(oracle, inputs: dict):
    w = inputs["workload"]
    return oracle.dr_scan(inputs["q"], inputs["k"], inputs["v"], inputs["beta"], inputs["gate"],
                          inputs["S0"], w.mode)


def oracle_dr_ex(oracle, inputs: dict):
    """(out, S_final, write values) of the oracle, every variant including Gated DeltaNet-2."""
    w = inputs["workload"]
    return oracle.dr_scan_ex(inputs["q"], inputs["k"], inputs["v"], inputs["beta"],
                             inputs["gate"], inputs["S0"], w.mode, erase=inputs.get("erase"),
                             write=inputs.get("write"))


def tensor_np(t):
    import torch

    return t.detach().to(torch.float64).cpu().numpy()
