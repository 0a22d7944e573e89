"""vla_scan_fwd_noalloc: the chunked VLA scan for callers that must not allocate device
memory (a serving engine that hands all device memory to its own allocator up front, or a
step where a driver allocation could block). Its scratch is a fixed array compiled into the
library instead of pool memory, so its results must be those of vla_scan_fwd_ex, call after
call, with the array still holding the previous call's contents.

This file is collected last on purpose: a run that stops at the first failure has run every
other test before this one."""
import ctypes

import numpy as np
import pytest

import delta_rule_recurrent_chunked_b200 as drs
from delta_rule_recurrent_chunked_b200 import workloads as wl

A = 0x10000  # a fake, 16-byte aligned address: validation rejects before any dereference


def _call_noalloc(B, H, T, d, flags=0):
    P = ctypes.c_void_p
    return drs.lib().vla_scan_fwd_noalloc(P(A), P(A), P(A), P(A), None, None, None, 1.0, P(A),
                                          None, None, None, B, H, T, d, flags, None)


def test_noalloc_rejects_requests_above_its_array():
    drs.lib()
    too_many = drs.VLA_NOALLOC_MAX_FLOATS // (4 * 64) + 1  # tokens
    assert _call_noalloc(1, 4, too_many, 64) == drs.DR_ERR_SCRATCH_LIMIT
    assert "scratch" in drs.status_string(drs.DR_ERR_SCRATCH_LIMIT)
    assert _call_noalloc(1, 4, 8, 64, flags=drs.VLA_SEQUENTIAL) == drs.DR_ERR_INVALID_ARG
    assert _call_noalloc(1, 4, 8, 48) == drs.DR_ERR_UNSUPPORTED
    assert _call_noalloc(0, 4, 8, 64) == drs.DR_OK


def _run(name, inputs, ratio):
    import torch

    w = inputs["workload"]
    dev = {k: torch.from_numpy(inputs[k]).cuda() for k in ("q", "k", "v", "u")}
    shp = (w.B, w.H)
    out = torch.empty_like(dev["v"])
    Sf = torch.empty(shp + (w.d, w.d), device="cuda")
    Af = torch.empty(shp + (w.d, w.d), device="cuda")
    nf = torch.empty(shp + (w.d,), device="cuda") if ratio else None
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    flags = drs.VLA_RATIO_READOUT if ratio else 0
    rc = getattr(drs.lib(), name)(p(dev["q"]), p(dev["k"]), p(dev["v"]), p(dev["u"]), None, None,
                                  None, 1.0, p(out), p(Sf), p(Af), p(nf), w.B, w.H, w.T, w.d,
                                  flags, drs._stream_handle(out.device))
    assert rc == drs.DR_OK, drs.status_string(rc)
    torch.cuda.synchronize()
    assert drs.poll_error() == drs.DR_OK
    return [t.cpu().numpy() for t in (out, Sf, Af, nf) if t is not None]


@pytest.mark.gpu
@pytest.mark.parametrize("ratio", [False, True])
def test_noalloc_matches_the_pool_entry_point_on_two_calls_in_a_row(ratio):
    # two different requests back to back: the second finds the first one's directions
    # still in the array and must not depend on them
    cases = [wl.VLAWorkload("noalloc_a", B=2, H=3, T=300, d=64, ratio=ratio),
             wl.VLAWorkload("noalloc_b", B=1, H=5, T=129, d=32, ratio=ratio)]
    for seed, w in enumerate(cases):
        inputs = wl.generate_vla(w, 20 + seed)
        ref = _run("vla_scan_fwd_ex", inputs, ratio)
        got = _run("vla_scan_fwd_noalloc", inputs, ratio)
        for g, r in zip(got, ref):
            err = np.abs(g - r).max() / np.abs(r).max()
            assert err <= 1e-4, (w.name, err)
