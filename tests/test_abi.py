"""C-ABI library checks that need no GPU: it loads, exports every symbol the header
declares, and rejects bad arguments with the documented status codes before touching
the device (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

import delta_rule_recurrent_chunked_b200 as drs
from delta_rule_recurrent_chunked_b200 import build as drbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "drscan.h")


@pytest.fixture(scope="module")
def lib():
    drbuild.build_library()
    return drs.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    assert set(header_functions()) == set(drs.SIGNATURES), header_functions()


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", drs.LIB_PATH]).decode()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in header_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_version_and_status_strings(lib):
    assert lib.dr_version() >= 100
    codes = [drs.DR_OK, drs.DR_ERR_INVALID_ARG, drs.DR_ERR_UNSUPPORTED, drs.DR_ERR_CUDA,
             drs.DR_ERR_TIMEOUT, drs.DR_ERR_DEVICE_BOUNDS, drs.DR_ERR_GATE_RANGE,
             drs.DR_ERR_NOT_SPD]
    texts = [drs.status_string(c) for c in codes]
    assert all(t and t != "unknown status" for t in texts)
    assert len(set(texts)) == len(texts)
    assert drs.status_string(12345) == "unknown status"


A = 0x10000  # a fake, 16-byte aligned address: validation rejects before any dereference


def call_dr(lib, q=A, k=A, v=A, beta=A, gate=A, S0=None, out=A, Sf=None, B=1, H=1, T=8, dk=32,
            dv=32, mode=drs.DR_GDN):
    P = ctypes.c_void_p
    return lib.dr_scan_fwd(P(q), P(k), P(v), P(beta), P(gate), P(S0), P(out), P(Sf), B, H, T,
                           dk, dv, mode, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), drs.DR_ERR_INVALID_ARG),
    (dict(out=None), drs.DR_ERR_INVALID_ARG),
    (dict(beta=None), drs.DR_ERR_INVALID_ARG),
    (dict(gate=None), drs.DR_ERR_INVALID_ARG),
    (dict(gate=None, mode=drs.DR_KDA), drs.DR_ERR_INVALID_ARG),
    (dict(k=A + 4), drs.DR_ERR_INVALID_ARG),
    (dict(S0=A + 8), drs.DR_ERR_INVALID_ARG),
    (dict(Sf=A + 2), drs.DR_ERR_INVALID_ARG),
    (dict(T=-1), drs.DR_ERR_INVALID_ARG),
    (dict(B=-2), drs.DR_ERR_INVALID_ARG),
    (dict(dk=0), drs.DR_ERR_INVALID_ARG),
    (dict(mode=7), drs.DR_ERR_INVALID_ARG),
    (dict(mode=drs.DR_GDN | 0x800), drs.DR_ERR_INVALID_ARG),
    (dict(dk=48), drs.DR_ERR_UNSUPPORTED),
    (dict(dv=256), drs.DR_ERR_UNSUPPORTED),
    (dict(B=0), drs.DR_OK),                      # empty batch: nothing to launch
    (dict(H=0, T=0), drs.DR_OK),
    (dict(q=None, k=None, v=None, out=None, beta=None, gate=None, B=0), drs.DR_OK),
    (dict(q=A + 4, B=0), drs.DR_ERR_INVALID_ARG),  # misaligned is an error even when unused
])
def test_dr_scan_argument_validation(lib, kw, code):
    assert call_dr(lib, **kw) == code


def test_linear_and_deltanet_need_no_gate(lib):
    # a valid request reaches the launch; with B*H == 0 there is nothing to launch
    assert call_dr(lib, beta=None, gate=None, mode=drs.DR_LINEAR, B=0) == drs.DR_OK
    assert call_dr(lib, gate=None, mode=drs.DR_DELTANET, B=0) == drs.DR_OK


def call_decode(lib, q=A, k=A, v=A, beta=A, gate=A, S=A, out=A, B=1, H=1, dk=32, dv=32,
                mode=drs.DR_GDN):
    P = ctypes.c_void_p
    return lib.dr_decode_step(P(q), P(k), P(v), P(beta), P(gate), P(S), P(out), B, H, dk, dv, mode,
                              None)


@pytest.mark.parametrize("kw,code", [
    (dict(S=None), drs.DR_ERR_INVALID_ARG),
    (dict(q=None), drs.DR_ERR_INVALID_ARG),
    (dict(out=None), drs.DR_ERR_INVALID_ARG),
    (dict(beta=None), drs.DR_ERR_INVALID_ARG),
    (dict(gate=None), drs.DR_ERR_INVALID_ARG),
    (dict(gate=None, mode=drs.DR_KDA), drs.DR_ERR_INVALID_ARG),
    (dict(S=A + 8), drs.DR_ERR_INVALID_ARG),
    (dict(v=A + 2), drs.DR_ERR_INVALID_ARG),
    (dict(B=-1), drs.DR_ERR_INVALID_ARG),
    (dict(dv=0), drs.DR_ERR_INVALID_ARG),
    (dict(mode=7), drs.DR_ERR_INVALID_ARG),
    (dict(mode=drs.DR_GDN | drs.DR_FORCE_SEQUENTIAL), drs.DR_ERR_INVALID_ARG),  # scan-only flag
    (dict(dk=48), drs.DR_ERR_UNSUPPORTED),
    (dict(dv=256), drs.DR_ERR_UNSUPPORTED),
    (dict(B=0), drs.DR_OK),
    (dict(q=None, k=None, v=None, beta=None, gate=None, S=None, out=None, H=0), drs.DR_OK),
    (dict(beta=None, gate=None, mode=drs.DR_LINEAR, B=0), drs.DR_OK),
    (dict(S=A + 4, B=0), drs.DR_ERR_INVALID_ARG),  # misaligned is an error even when unused
])
def test_decode_step_argument_validation(lib, kw, code):
    assert call_decode(lib, **kw) == code


def call_vla(lib, q=A, k=A, v=A, u=A, S0=None, A0=None, lam=1.0, out=A, B=1, H=1, T=8, d=32):
    P = ctypes.c_void_p
    return lib.vla_scan_fwd(P(q), P(k), P(v), P(u), P(S0), P(A0), lam, P(out), None, None, B, H,
                            T, d, None)


@pytest.mark.parametrize("kw,code", [
    (dict(u=None), drs.DR_ERR_INVALID_ARG),
    (dict(q=A + 4), drs.DR_ERR_INVALID_ARG),
    (dict(lam=0.0), drs.DR_ERR_INVALID_ARG),
    (dict(lam=-1.0), drs.DR_ERR_INVALID_ARG),
    (dict(T=-5), drs.DR_ERR_INVALID_ARG),
    (dict(d=48), drs.DR_ERR_UNSUPPORTED),
    (dict(d=256), drs.DR_ERR_UNSUPPORTED),
    (dict(B=0), drs.DR_OK),
])
def test_vla_argument_validation(lib, kw, code):
    assert call_vla(lib, **kw) == code


def call_vla_ex(lib, flags, B=1, n0=None):
    P = ctypes.c_void_p
    return lib.vla_scan_fwd_ex(P(A), P(A), P(A), P(A), None, None, P(n0), 1.0, P(A), None, None,
                               None, B, 1, 8, 32, flags, None)


def test_vla_ex_flags(lib):
    assert call_vla_ex(lib, 0x8) == drs.DR_ERR_INVALID_ARG
    assert call_vla_ex(lib, drs.VLA_SEQUENTIAL | 0x10) == drs.DR_ERR_INVALID_ARG
    assert call_vla_ex(lib, drs.VLA_SEQUENTIAL, n0=A) == drs.DR_ERR_INVALID_ARG  # n0: ratio only
    assert call_vla_ex(lib, drs.VLA_SEQUENTIAL | drs.VLA_TWO_KERNEL) == drs.DR_ERR_INVALID_ARG
    for flags in (0, drs.VLA_SEQUENTIAL, drs.VLA_TWO_KERNEL, drs.VLA_RATIO_READOUT,
                  drs.VLA_RATIO_READOUT | drs.VLA_SEQUENTIAL,
                  drs.VLA_RATIO_READOUT | drs.VLA_TWO_KERNEL):
        assert call_vla_ex(lib, flags, B=0) == drs.DR_OK


def test_timeout_probe_rejects_bad_limits(lib):
    assert lib.dr_debug_timeout_probe(0, None) == drs.DR_ERR_INVALID_ARG
    assert lib.dr_debug_timeout_probe(10**7, None) == drs.DR_ERR_INVALID_ARG


def test_chunked_plan_rejects_before_querying_the_device(lib):
    bv, npr = ctypes.c_int(-1), ctypes.c_int(-1)
    call = lambda mode, BH, dk, dv, a=ctypes.byref(bv), b=ctypes.byref(npr): \
        lib.dr_chunked_plan(mode, BH, dk, dv, a, b)
    assert call(drs.DR_GDN | drs.DR_IN_BF16, 4, 128, 128, None, None) == drs.DR_ERR_INVALID_ARG
    assert call(drs.DR_GDN | drs.DR_IN_BF16, 0, 128, 128) == drs.DR_ERR_INVALID_ARG
    assert call(drs.DR_GDN | 0x4000, 4, 128, 128) == drs.DR_ERR_INVALID_ARG
    # fp32 inputs, forced sequential, other shapes and plain linear attention use the
    # per-token kernel: no plan, both outputs zeroed
    for mode, dk, dv in [(drs.DR_GDN, 128, 128),
                         (drs.DR_GDN | drs.DR_IN_BF16 | drs.DR_FORCE_SEQUENTIAL, 128, 128),
                         (drs.DR_GDN | drs.DR_IN_BF16, 64, 128),
                         (drs.DR_KDA | drs.DR_IN_BF16, 128, 96),
                         (drs.DR_LINEAR | drs.DR_IN_BF16, 128, 128)]:
        bv.value, npr.value = -1, -1
        assert call(mode, 4, dk, dv) == drs.DR_ERR_UNSUPPORTED
        assert (bv.value, npr.value) == (0, 0)


def test_chunked_plan_ex_rejects_before_querying_the_device(lib):
    bv, npr, ns = ctypes.c_int(-1), ctypes.c_int(-1), ctypes.c_int(-1)
    call = lambda mode, BH, T, dk, dv, c=ctypes.byref(ns): lib.dr_chunked_plan_ex(
        mode, BH, T, dk, dv, ctypes.byref(bv), ctypes.byref(npr), c)
    assert call(drs.DR_GDN | drs.DR_IN_BF16, 4, 4096, 128, 128, None) == drs.DR_ERR_INVALID_ARG
    assert call(drs.DR_GDN | drs.DR_IN_BF16, 4, -1, 128, 128) == drs.DR_ERR_INVALID_ARG
    assert call(drs.DR_GDN | drs.DR_IN_BF16, 0, 4096, 128, 128) == drs.DR_ERR_INVALID_ARG
    assert call(drs.DR_GDN | drs.DR_IN_BF16 | 0x4000, 4, 4096, 128, 128) == drs.DR_ERR_INVALID_ARG
    # the per-token kernel's requests: no plan, one segment
    ns.value = -1
    assert call(drs.DR_GDN | drs.DR_IN_BF16 | drs.DR_CHAINED | drs.DR_FORCE_SEQUENTIAL, 4, 4096,
                128, 128) == drs.DR_ERR_UNSUPPORTED
    assert (bv.value, npr.value, ns.value) == (0, 0, 1)


def test_scan_accepts_the_chained_flag_and_rejects_unknown_bits(lib):
    # B*H = 0: validated, nothing launched
    P = ctypes.c_void_p
    for mode, code in [(drs.DR_GDN | drs.DR_IN_BF16 | drs.DR_CHAINED, drs.DR_OK),
                       (drs.DR_GDN | drs.DR_IN_BF16 | 0x800, drs.DR_ERR_INVALID_ARG)]:
        assert lib.dr_scan_fwd(None, None, None, None, None, None, None, None, 0, 4, 64, 128,
                               128, mode, None) == code


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(drs, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(drs, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        drs.lib()


C_CALLER = r"""
#include "drscan.h"
int main(void) {
    int bv = 0, np = 0;
    int (*scan)(const void*, const void*, const void*, const float*, const float*, const float*,
                void*, float*, int, int, int, int, int, int, cudaStream_t) = dr_scan_fwd;
    int (*decode)(const void*, const void*, const void*, const float*, const float*, float*,
                  void*, int, int, int, int, int, cudaStream_t) = dr_decode_step;
    (void)scan;
    (void)decode;
    (void)vla_scan_fwd;
    (void)dr_poll_error;
    (void)dr_debug_timeout_probe;
    /* host-only calls: a request rejected before any device query, status text, version */
    if (dr_chunked_plan(DR_GDN | DR_IN_BF16, 0, 128, 128, &bv, &np) != DR_ERR_INVALID_ARG) return 1;
    if (!dr_status_string(DR_ERR_TIMEOUT)[0]) return 2;
    return dr_version() > 0 ? 0 : 3;
}
"""


def test_header_serves_a_plain_c_caller(lib, tmp_path):
    # the boundary is a C ABI: a C99 program compiles against the header without warnings,
    # links against the library and makes its host-only calls
    import shutil

    cuda_inc = "/usr/local/cuda/include"
    if not shutil.which("gcc") or not os.path.exists(os.path.join(cuda_inc, "cuda_runtime.h")):
        pytest.skip("needs gcc and the CUDA runtime headers")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(drs.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
                           "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src),
                           "-L", libdir, "-ldrscan", f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    assert subprocess.run([str(exe)]).returncode == 0
