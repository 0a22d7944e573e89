"""GPU parity of the log-linear attention scan (loglinear_scan_fwd) against the fp64 oracle.

"Adaptive memory decay for log-linear attention", problem definition and method sections: a
Fenwick-tree hierarchy of memories, outputs weighted over the levels by lambda_t^(l).
Tolerance: bf16 q/k/v with fp32 level states, max|x - y| / max|y| <= 2e-2 (oracle fed the
bf16-rounded inputs).
"""
import numpy as np
import pytest

import delta_rule_recurrent_chunked_b200 as drs
from delta_rule_recurrent_chunked_b200 import workloads as wl

from helpers import rel_err, tensor_np

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


def upload(inputs):
    dev = {}
    for name in ("q", "k", "v"):
        raw = np.ascontiguousarray(inputs[name + "_raw"])
        dev[name] = torch.from_numpy(raw.view(np.int16)).view(torch.bfloat16).cuda()
    dev["lam"] = torch.from_numpy(np.ascontiguousarray(inputs["lam"])).cuda()
    return dev


def check(oracle, w, seed, heads=None, lam_fn=None):
    inputs = wl.generate_loglinear(w, seed)
    if lam_fn is not None:
        inputs["lam"] = np.ascontiguousarray(lam_fn(inputs["lam"]), dtype=np.float32)
    dev = upload(inputs)
    out = drs.loglinear_scan(dev["q"], dev["k"], dev["v"], dev["lam"])
    torch.cuda.synchronize()
    got = tensor_np(out)
    if heads is not None:
        inputs = wl.head_slice(inputs, heads)
        got = got.reshape((w.B * w.H,) + got.shape[2:])[heads][None]
    ref = oracle.loglinear_scan(inputs["q"], inputs["k"], inputs["v"], inputs["lam"])
    e = rel_err(got, ref)
    assert e <= TOL, (w, e)
    return e


# ragged T: one chunk, a partial chunk, many chunks (every Fenwick level up to 2^5 chunks)
@pytest.mark.parametrize("T", [1, 5, 64, 65, 130, 1000, 2049])
def test_loglinear_ragged(oracle, T):
    check(oracle, wl.LogLinearWorkload("t", 1, 3, T, 128, 128), seed=T)


@pytest.mark.parametrize("dv", [32, 64])
def test_loglinear_narrow_values(oracle, dv):
    check(oracle, wl.LogLinearWorkload("t", 2, 2, 777, 128, dv), seed=dv)


def test_loglinear_workload_sampled(oracle):
    check(oracle, wl.workload("loglinear_bf16"), seed=0, heads=[0, 11, 31])


def test_loglinear_long_context_sampled(oracle):
    # 512 chunks: all nine chunk levels of the block-state counter
    check(oracle, wl.LogLinearWorkload("t", 1, 4, 32768, 128, 128), seed=3, heads=[0, 3])


@pytest.mark.parametrize("level", [0, 3, 7, 9, 12])
def test_loglinear_one_level(oracle, level):
    # weight on one level only: in-chunk levels (0-6) and block-state levels (7+)
    def one(lam):
        z = np.zeros_like(lam)
        z[..., level] = 1.0
        return z
    check(oracle, wl.LogLinearWorkload("t", 1, 2, 3000, 128, 128), seed=level, lam_fn=one)


def test_loglinear_rejects_too_few_levels():
    q = torch.zeros(1, 1, 100, 128, dtype=torch.bfloat16, device="cuda")
    lam = torch.ones(1, 1, 100, 7, device="cuda")  # 100 tokens need 8 levels
    with pytest.raises(drs.DrScanError):
        drs.loglinear_scan(q, q, q, lam)
