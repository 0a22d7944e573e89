"""Shared test helpers: device upload of generated workloads, oracle references, metrics."""
from __future__ import annotations

import numpy as np

from delta_rule_recurrent_chunked_b200 import workloads as wl

MODE_NAME = {wl.LINEAR: "linear", wl.DELTANET: "deltanet", wl.GDN: "gdn", wl.KDA: "kda"}


def rel_err(x, y) -> float:
    """max|x - y| / max|y| over a whole tensor (the tolerance metric for out and S_final)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    if y.size == 0:
        return 0.0
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-30))


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
    for name in ("beta", "gate", "S0"):
        arr = inputs.get(name)
        dev[name] = None if arr is None else torch.from_numpy(np.ascontiguousarray(arr)).to(device)
    return dev


def oracle_dr(oracle, inputs: dict):
    w = inputs["workload"]
    return oracle.dr_scan(inputs["q"], inputs["k"], inputs["v"], inputs["beta"], inputs["gate"],
                          inputs["S0"], w.mode)


def tensor_np(t):
    import torch

    return t.detach().to(torch.float64).cpu().numpy()
