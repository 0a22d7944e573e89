"""Seeded synthetic inputs for the delta-rule scan workloads.

This module only draws random numbers and casts them; it holds none of the scan's
arithmetic. Both the CUDA path (through the tests and the benchmark) and the fp64
oracle consume exactly the arrays it returns, so they always see the same values.

Recipe (one ``numpy.random.default_rng(seed)`` per workload, fp64 draws in this order):
  delta-rule family: q, k, v, beta-logit, gate-x, [Gated DeltaNet-2: erase-logit,
                     write-logit], S0
  VLA:               q, k, v, u
  log-linear:        q, k, v, lambda-x
then q and k (VLA: k_hat, q_hat) are L2-normalised per token, beta = sigmoid(logit),
alpha = exp(-softplus(x)) (the gate value in (0, 1), not its log), and q/k/v are rounded
to the workload's input type (bf16 by round-to-nearest-even, else fp32). Gated
DeltaNet-2's erase and write gates are sigmoid(N(0,1)) per (b,h,t,channel). beta, alpha, the
gates and S0 are always fp32. The oracle is fed these rounded values upcast to fp64.

Workloads (shapes and distributions as the method's benchmark configurations state):
  deltanet_fp32     B1  H2  T256  dk=dv=32   fp32, alpha = 1, S0 = 0
  gdn_bf16          B4  H8  T4096 dk=dv=128  bf16, scalar alpha, x ~ N(-4, 1) per (b,h,t)
  kda_bf16          B8  H16 T4096 dk=dv=128  bf16, per-key-channel alpha, x ~ N(-4,1) per (b,h,t,c)
  gdn_long_t{T}     B1  H16 T in {4096, 8192, 16384, 32768} dk=dv=128 bf16, S0 ~ N(0, 0.1^2)
  gdn2_bf16         B4  H8  T4096 dk=dv=128  bf16, gates as gdn_bf16, erase/write sigmoid(N(0,1))
  vla_fp32_d{d}     B4  H8  T4096 d in {32, 96} fp32, A0 = I (lambda0 = 1), u ~ N(0,1)/sqrt(d)
  vla_ratio_fp32_d{d}  as vla_fp32_d{d} with the ratio readout: the same draws, with the ELU+1
                    feature map on q and k before k is L2-normalised (q stays unnormalised)
  loglinear_bf16    B4  H8  T4096 dk=dv=128  bf16, level weights lambda = softplus(0.54 + 0.5 x),
                    x ~ N(0,1) per (b,h,t,level): around softplus(0.54) = 1, the page's
                    initial value, with content-dependent spread; 13 levels
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

LINEAR, DELTANET, GDN, KDA, GDN2 = 0, 1, 2, 3, 4
MODE_NAMES = {LINEAR: "linear", DELTANET: "deltanet", GDN: "gdn", KDA: "kda", GDN2: "gdn2"}


@dataclass(frozen=True)
class DRWorkload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    mode: int
    dtype: str  # "bf16" or "fp32" for q/k/v/out
    s0_std: float = 0.0
    gate_mu: float = -4.0
    gate_sigma: float = 1.0
    decode: bool = False  # T = 1 steps on a state resident in HBM (dr_decode_step)

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T


@dataclass(frozen=True)
class LogLinearWorkload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T

    @property
    def levels(self) -> int:
        return max(1, int(self.T - 1).bit_length() + 1)


@dataclass(frozen=True)
class VLAWorkload:
    name: str
    B: int
    H: int
    T: int
    d: int
    lambda0: float = 1.0
    ratio: bool = False  # ratio readout o = S q / (n q) on ELU+1 features

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T


WORKLOADS = {
    "deltanet_fp32": DRWorkload("deltanet_fp32", 1, 2, 256, 32, 32, DELTANET, "fp32"),
    "gdn_bf16": DRWorkload("gdn_bf16", 4, 8, 4096, 128, 128, GDN, "bf16"),
    "kda_bf16": DRWorkload("kda_bf16", 8, 16, 4096, 128, 128, KDA, "bf16"),
}
for _T in (4096, 8192, 16384, 32768):
    WORKLOADS[f"gdn_long_t{_T}"] = DRWorkload(f"gdn_long_t{_T}", 1, 16, _T, 128, 128, GDN, "bf16",
                                              s0_std=0.1)
# long-context KDA with few heads (not one of the timed configurations; the segmented scan's
# KDA case)
WORKLOADS["kda_long_t32768"] = DRWorkload("kda_long_t32768", 1, 16, 32768, 128, 128, KDA, "bf16",
                                          s0_std=0.1)
WORKLOADS["gdn2_bf16"] = DRWorkload("gdn2_bf16", 4, 8, 4096, 128, 128, GDN2, "bf16")
WORKLOADS["loglinear_bf16"] = LogLinearWorkload("loglinear_bf16", 4, 8, 4096, 128, 128)
# streaming decode: one token per step for 4096 heads whose 256 MiB fp32 state stays in HBM
WORKLOADS["gdn_decode_bf16"] = DRWorkload("gdn_decode_bf16", 128, 32, 1, 128, 128, GDN, "bf16",
                                          s0_std=0.1, decode=True)
for _d in (32, 96):
    WORKLOADS[f"vla_fp32_d{_d}"] = VLAWorkload(f"vla_fp32_d{_d}", 4, 8, 4096, _d)
    WORKLOADS[f"vla_ratio_fp32_d{_d}"] = VLAWorkload(f"vla_ratio_fp32_d{_d}", 4, 8, 4096, _d,
                                                     ratio=True)


def workload(name: str, **overrides):
    """Look up a named workload; keyword overrides shrink it (e.g. T=65, B=1)."""
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to bf16 (nearest-even); return the raw 16-bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _as_input(x: np.ndarray, dtype: str):
    """Return (values as fp32 after rounding to dtype, raw array to upload)."""
    if dtype == "bf16":
        bits = bf16_bits(x)
        return bf16_to_f32(bits), bits
    f = np.ascontiguousarray(x, dtype=np.float32)
    return f, f


def generate_dr(w: DRWorkload, seed: int = 0) -> dict:
    """Draw one delta-rule workload. Values are fp32 numpy arrays already rounded to
    the input type; ``*_raw`` are what goes to the device (uint16 bf16 bits or fp32)."""
    rng = np.random.default_rng(seed)
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    q = _unit_rows(rng.standard_normal((B, H, T, dk)))
    k = _unit_rows(rng.standard_normal((B, H, T, dk)))
    v = rng.standard_normal((B, H, T, dv))
    logit = rng.standard_normal((B, H, T))
    beta = (1.0 / (1.0 + np.exp(-logit))).astype(np.float32)
    gate = erase = write = None
    if w.mode in (GDN, GDN2):
        x = w.gate_mu + w.gate_sigma * rng.standard_normal((B, H, T))
        gate = np.exp(-np.logaddexp(0.0, x)).astype(np.float32)
    elif w.mode == KDA:
        x = w.gate_mu + w.gate_sigma * rng.standard_normal((B, H, T, dk))
        gate = np.exp(-np.logaddexp(0.0, x)).astype(np.float32)
    if w.mode == GDN2:
        erase = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T, dk))))).astype(np.float32)
        write = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T, dv))))).astype(np.float32)
    S0 = None
    if w.s0_std > 0.0:
        S0 = (w.s0_std * rng.standard_normal((B, H, dv, dk))).astype(np.float32)
    out = {"workload": w, "beta": beta, "gate": gate, "S0": S0, "erase": erase, "write": write}
    for name, arr in (("q", q), ("k", k), ("v", v)):
        out[name], out[name + "_raw"] = _as_input(arr, w.dtype)
    return out


def _elu1(x: np.ndarray) -> np.ndarray:
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def generate_vla(w: VLAWorkload, seed: int = 0) -> dict:
    rng = np.random.default_rng(seed)
    B, H, T, d = w.B, w.H, w.T, w.d
    q = rng.standard_normal((B, H, T, d))
    k = rng.standard_normal((B, H, T, d))
    if w.ratio:  # the ELU+1 feature map; only the key is normalised
        q, k = _elu1(q), _unit_rows(_elu1(k))
    else:
        q, k = _unit_rows(q), _unit_rows(k)
    q, k = q.astype(np.float32), k.astype(np.float32)
    v = rng.standard_normal((B, H, T, d)).astype(np.float32)
    u = (rng.standard_normal((B, H, T, d)) / np.sqrt(d)).astype(np.float32)
    return {"workload": w, "q": q, "k": k, "v": v, "u": u, "S0": None, "A0": None, "n0": None}


def generate_loglinear(w: LogLinearWorkload, seed: int = 0) -> dict:
    rng = np.random.default_rng(seed)
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv
    q = _unit_rows(rng.standard_normal((B, H, T, dk)))
    k = _unit_rows(rng.standard_normal((B, H, T, dk)))
    v = rng.standard_normal((B, H, T, dv))
    x = rng.standard_normal((B, H, T, w.levels))
    lam = np.logaddexp(0.0, 0.54 + 0.5 * x).astype(np.float32)
    out = {"workload": w, "lam": lam}
    for name, arr in (("q", q), ("k", k), ("v", v)):
        out[name], out[name + "_raw"] = _as_input(arr, "bf16")
    return out


def generate(w, seed: int = 0) -> dict:
    if isinstance(w, VLAWorkload):
        return generate_vla(w, seed)
    if isinstance(w, LogLinearWorkload):
        return generate_loglinear(w, seed)
    return generate_dr(w, seed)


def head_slice(inputs: dict, heads) -> dict:
    """Restrict a generated workload to a list of flat (b*H + h) head indices
    (heads are independent sequences). Returns arrays shaped [1, len(heads), ...]."""
    w = inputs["workload"]
    out = {"workload": w}
    for key, arr in inputs.items():
        if key == "workload" or arr is None:
            out[key] = arr
            continue
        flat = arr.reshape((w.B * w.H,) + arr.shape[2:])
        out[key] = flat[list(heads)][None]
    return out
