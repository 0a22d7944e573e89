"""B200-native forward recurrent-memory scan of delta-rule linear attention.

Thin Python binding over the C-ABI library ``libdrscan.so`` (declared in
``include/drscan.h``). This module only marshals arguments: it checks tensor dtypes,
shapes and devices, passes raw device pointers and the current CUDA stream, and raises
on a non-zero status. Every step of the scan runs in the library's CUDA kernels; there
is no CPU fallback, and a missing library is an error.

    out, S_final = scan(q, k, v, beta, gate, S0=None, mode="gdn")
    out, S_final, u = scan_ex(q, k, v, beta, gate, S0=None, mode="gdn2", erase=b, write=w)
    out, S_final, A_final = vla_scan(q, k, v, u, S0=None, A0=None, lambda0=1.0)
    out = decode_step(q, k, v, beta, gate, S, mode="gdn")     # S updated in place
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdrscan.so")

DR_LINEAR, DR_DELTANET, DR_GDN, DR_KDA, DR_GDN2 = 0, 1, 2, 3, 4
DR_IN_BF16 = 0x100
DR_FORCE_SEQUENTIAL = 0x200
DR_CHAINED = 0x400
DR_OK, DR_ERR_INVALID_ARG, DR_ERR_UNSUPPORTED, DR_ERR_CUDA, DR_ERR_TIMEOUT, DR_ERR_DEVICE_BOUNDS = (
    0, -1, -2, -3, -4, -5)
DR_ERR_GATE_RANGE = -6
DR_ERR_NOT_SPD = -7
DR_ERR_SCRATCH_LIMIT = -8
VLA_NOALLOC_MAX_FLOATS = 16777216
MODES = {"linear": DR_LINEAR, "deltanet": DR_DELTANET, "gdn": DR_GDN, "kda": DR_KDA,
         "gdn2": DR_GDN2}

# Every function the C ABI exports, with its ctypes signature.
_VP, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "dr_scan_fwd": ([_VP] * 8 + [_I] * 6 + [_VP], _I),
    "dr_scan_fwd_ex": ([_VP] * 11 + [_I] * 6 + [_VP], _I),
    "dr_decode_step": ([_VP] * 7 + [_I] * 5 + [_VP], _I),
    "dr_decode_step_ex": ([_VP] * 10 + [_I] * 5 + [_VP], _I),
    "vla_scan_fwd": ([_VP] * 6 + [_F] + [_VP] * 3 + [_I] * 4 + [_VP], _I),
    "vla_scan_fwd_ex": ([_VP] * 7 + [_F] + [_VP] * 4 + [_I] * 5 + [_VP], _I),
    "vla_scan_fwd_noalloc": ([_VP] * 7 + [_F] + [_VP] * 4 + [_I] * 5 + [_VP], _I),
    "loglinear_scan_fwd": ([_VP] * 5 + [_I] * 7 + [_VP], _I),
    "dr_status_string": ([_I], ctypes.c_char_p),
    "dr_poll_error": ([_VP], _I),
    "dr_debug_timeout_probe": ([_I, _VP], _I),
    "dr_chunked_plan": ([_I, ctypes.c_longlong, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)], _I),
    "dr_chunked_plan_ex": ([_I, ctypes.c_longlong, _I, _I, _I, ctypes.POINTER(_I),
                            ctypes.POINTER(_I), ctypes.POINTER(_I)], _I),
    "dr_segment_counters": ([ctypes.POINTER(ctypes.c_ulonglong)] * 2, _I),
    "dr_version": ([], _I),
}

_lib = None


class DrScanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({status_string(status)})")


def lib():
    """Load libdrscan.so (built in-tree). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m delta_rule_recurrent_chunked_b200.build` (nvcc, sm_100a)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (argtypes, restype) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = argtypes
            fn.restype = restype
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().dr_status_string(int(status)).decode()


def _stream_handle(device):
    import torch

    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, shape, dtype, device):
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def scan(q, k, v, beta=None, gate=None, S0=None, mode="gdn", want_state=True,
         force_sequential=False, out=None, S_final=None, chained=False):
    """Delta-rule scan on the GPU. q, k: [B,H,T,dk]; v: [B,H,T,dv] (bf16 or fp32, same
    dtype); beta: [B,H,T] fp32; gate: alpha values, [B,H,T] (gdn) or [B,H,T,dk] (kda) fp32;
    S0: [B,H,dv,dk] fp32 or None. chained=True keeps Gated DeltaNet off the segmented scan
    (DR_CHAINED). Returns (out like v, S_final fp32 or None)."""
    import torch

    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q/k/v must be bf16 or fp32")
    _check(q, "q", (B, H, T, dk), q.dtype, dev)
    _check(k, "k", (B, H, T, dk), q.dtype, dev)
    _check(v, "v", (B, H, T, dv), q.dtype, dev)
    if variant != DR_LINEAR:
        _check(beta, "beta", (B, H, T), torch.float32, dev)
    else:
        beta = None
    if variant == DR_GDN:
        _check(gate, "gate", (B, H, T), torch.float32, dev)
    elif variant == DR_KDA:
        _check(gate, "gate", (B, H, T, dk), torch.float32, dev)
    else:
        gate = None
    if S0 is not None:
        _check(S0, "S0", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    _check(out, "out", (B, H, T, dv), q.dtype, dev)
    if want_state and S_final is None:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", (B, H, dv, dk), torch.float32, dev)
    flags = variant | (DR_IN_BF16 if q.dtype == torch.bfloat16 else 0)
    if force_sequential:
        flags |= DR_FORCE_SEQUENTIAL
    if chained:
        flags |= DR_CHAINED
    rc = lib().dr_scan_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(S0), _ptr(out),
                           _ptr(S_final), B, H, T, dk, dv, flags, _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "dr_scan_fwd")
    return out, S_final


def scan_ex(q, k, v, beta=None, gate=None, S0=None, mode="gdn", erase=None, write=None,
            want_state=True, want_u=True, force_sequential=False, out=None, S_final=None,
            u_out=None, chained=False):
    """scan() with Gated DeltaNet-2 and the per-token write values, through dr_scan_fwd_ex.
    mode "gdn2" takes gate [B,H,T] (alpha), erase [B,H,T,dk] (b) and write [B,H,T,dv] (w),
    fp32. Returns (out, S_final or None, u or None): u [B,H,T,dv] like v holds the write
    values beta_t r_t."""
    import torch

    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q/k/v must be bf16 or fp32")
    _check(q, "q", (B, H, T, dk), q.dtype, dev)
    _check(k, "k", (B, H, T, dk), q.dtype, dev)
    _check(v, "v", (B, H, T, dv), q.dtype, dev)
    if variant != DR_LINEAR:
        _check(beta, "beta", (B, H, T), torch.float32, dev)
    else:
        beta = None
    if variant in (DR_GDN, DR_GDN2):
        _check(gate, "gate", (B, H, T), torch.float32, dev)
    elif variant == DR_KDA:
        _check(gate, "gate", (B, H, T, dk), torch.float32, dev)
    else:
        gate = None
    if variant == DR_GDN2:
        _check(erase, "erase", (B, H, T, dk), torch.float32, dev)
        _check(write, "write", (B, H, T, dv), torch.float32, dev)
    else:
        erase = write = None
    if S0 is not None:
        _check(S0, "S0", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    _check(out, "out", (B, H, T, dv), q.dtype, dev)
    if want_state and S_final is None:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    if S_final is not None:
        _check(S_final, "S_final", (B, H, dv, dk), torch.float32, dev)
    if want_u and u_out is None:
        u_out = torch.empty((B, H, T, dv), dtype=q.dtype, device=dev)
    if u_out is not None:
        _check(u_out, "u_out", (B, H, T, dv), q.dtype, dev)
    flags = variant | (DR_IN_BF16 if q.dtype == torch.bfloat16 else 0)
    if force_sequential:
        flags |= DR_FORCE_SEQUENTIAL
    if chained:
        flags |= DR_CHAINED
    rc = lib().dr_scan_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(erase),
                              _ptr(write), _ptr(S0), _ptr(out), _ptr(S_final), _ptr(u_out),
                              B, H, T, dk, dv, flags, _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "dr_scan_fwd_ex")
    return out, S_final, u_out


def decode_step_ex(q, k, v, beta=None, gate=None, S=None, mode="gdn", erase=None, write=None,
                   want_u=True, out=None, u_out=None):
    """decode_step() with Gated DeltaNet-2 (erase [B,H,dk], write [B,H,dv]) and the write
    value u [B,H,dv], through dr_decode_step_ex. Returns (out, u or None)."""
    import torch

    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q/k/v must be bf16 or fp32")
    _check(q, "q", (B, H, dk), q.dtype, dev)
    _check(k, "k", (B, H, dk), q.dtype, dev)
    _check(v, "v", (B, H, dv), q.dtype, dev)
    if variant != DR_LINEAR:
        _check(beta, "beta", (B, H), torch.float32, dev)
    else:
        beta = None
    if variant in (DR_GDN, DR_GDN2):
        _check(gate, "gate", (B, H), torch.float32, dev)
    elif variant == DR_KDA:
        _check(gate, "gate", (B, H, dk), torch.float32, dev)
    else:
        gate = None
    if variant == DR_GDN2:
        _check(erase, "erase", (B, H, dk), torch.float32, dev)
        _check(write, "write", (B, H, dv), torch.float32, dev)
    else:
        erase = write = None
    if S is None:
        raise ValueError("decode_step_ex needs the state S (updated in place)")
    _check(S, "S", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=dev)
    _check(out, "out", (B, H, dv), q.dtype, dev)
    if want_u and u_out is None:
        u_out = torch.empty((B, H, dv), dtype=q.dtype, device=dev)
    if u_out is not None:
        _check(u_out, "u_out", (B, H, dv), q.dtype, dev)
    flags = variant | (DR_IN_BF16 if q.dtype == torch.bfloat16 else 0)
    rc = lib().dr_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(erase),
                                 _ptr(write), _ptr(S), _ptr(out), _ptr(u_out), B, H, dk, dv,
                                 flags, _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "dr_decode_step_ex")
    return out, u_out


def decode_step(q, k, v, beta=None, gate=None, S=None, mode="gdn", out=None):
    """One token of the delta-rule recurrence on a resident state, on the GPU.
    q, k: [B,H,dk]; v: [B,H,dv] (bf16 or fp32, same dtype); beta: [B,H] fp32; gate:
    alpha values, [B,H] (gdn) or [B,H,dk] (kda) fp32; S: [B,H,dv,dk] fp32, updated in
    place. Returns out [B,H,dv] like v."""
    import torch

    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q/k/v must be bf16 or fp32")
    _check(q, "q", (B, H, dk), q.dtype, dev)
    _check(k, "k", (B, H, dk), q.dtype, dev)
    _check(v, "v", (B, H, dv), q.dtype, dev)
    if variant != DR_LINEAR:
        _check(beta, "beta", (B, H), torch.float32, dev)
    else:
        beta = None
    if variant == DR_GDN:
        _check(gate, "gate", (B, H), torch.float32, dev)
    elif variant == DR_KDA:
        _check(gate, "gate", (B, H, dk), torch.float32, dev)
    else:
        gate = None
    if S is None:
        raise ValueError("decode_step needs the state S (updated in place)")
    _check(S, "S", (B, H, dv, dk), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=dev)
    _check(out, "out", (B, H, dv), q.dtype, dev)
    flags = variant | (DR_IN_BF16 if q.dtype == torch.bfloat16 else 0)
    rc = lib().dr_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(S),
                              _ptr(out), B, H, dk, dv, flags, _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "dr_decode_step")
    return out


def vla_scan(q, k, v, u, S0=None, A0=None, lambda0=1.0, want_state=True, out=None,
             sequential=False, two_kernel=False):
    """VLA Sherman-Morrison scan on the GPU (fp32). q, k, v, u: [B,H,T,d];
    S0, A0: [B,H,d,d] or None. Returns (out, S_final, A_final). The chunked scan runs as one
    fused cluster kernel by default; two_kernel=True runs its two phases as separate kernels
    (with pool scratch), sequential=True the per-token kernel."""
    import torch

    B, H, T, d = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("u", u)):
        _check(t, name, (B, H, T, d), torch.float32, dev)
    for name, t in (("S0", S0), ("A0", A0)):
        if t is not None:
            _check(t, name, (B, H, d, d), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, d), dtype=torch.float32, device=dev)
    _check(out, "out", (B, H, T, d), torch.float32, dev)
    Sf = torch.empty((B, H, d, d), dtype=torch.float32, device=dev) if want_state else None
    Af = torch.empty((B, H, d, d), dtype=torch.float32, device=dev) if want_state else None
    flags = _vla_path_flags(sequential, two_kernel)
    rc = lib().vla_scan_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(S0), _ptr(A0), None,
                               float(lambda0), _ptr(out), _ptr(Sf), _ptr(Af), None, B, H, T,
                               d, flags, _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "vla_scan_fwd_ex")
    return out, Sf, Af


VLA_RATIO_READOUT = 0x1
VLA_SEQUENTIAL = 0x2
VLA_TWO_KERNEL = 0x4


def _vla_path_flags(sequential: bool, two_kernel: bool) -> int:
    return (VLA_SEQUENTIAL if sequential else 0) | (VLA_TWO_KERNEL if two_kernel else 0)


def vla_scan_ratio(q, k, v, u, S0=None, A0=None, n0=None, lambda0=1.0, want_state=True,
                   out=None, sequential=False, two_kernel=False):
    """VLA scan with the ratio readout o_t = S_t q_t / (n_t q_t) (fp32), through
    vla_scan_fwd_ex. q: [B,H,T,d] feature-mapped queries (phi(q)); k: unit-norm
    feature-mapped keys; n0: [B,H,d] or None. Returns (out, S_final, A_final, n_final).
    two_kernel / sequential select the other paths, as in vla_scan."""
    import torch

    B, H, T, d = q.shape
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("u", u)):
        _check(t, name, (B, H, T, d), torch.float32, dev)
    for name, t in (("S0", S0), ("A0", A0)):
        if t is not None:
            _check(t, name, (B, H, d, d), torch.float32, dev)
    if n0 is not None:
        _check(n0, "n0", (B, H, d), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, d), dtype=torch.float32, device=dev)
    _check(out, "out", (B, H, T, d), torch.float32, dev)
    Sf = torch.empty((B, H, d, d), dtype=torch.float32, device=dev) if want_state else None
    Af = torch.empty((B, H, d, d), dtype=torch.float32, device=dev) if want_state else None
    nf = torch.empty((B, H, d), dtype=torch.float32, device=dev) if want_state else None
    rc = lib().vla_scan_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(S0), _ptr(A0), _ptr(n0),
                               float(lambda0), _ptr(out), _ptr(Sf), _ptr(Af), _ptr(nf), B, H, T,
                               d, VLA_RATIO_READOUT | _vla_path_flags(sequential, two_kernel),
                               _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "vla_scan_fwd_ex")
    return out, Sf, Af, nf


def loglinear_levels(T: int) -> int:
    """Level weights a log-linear scan of T tokens needs: level 0 plus one per bit of T - 1."""
    return max(1, int(T - 1).bit_length() + 1)


def loglinear_scan(q, k, v, lam, out=None):
    """Log-linear attention over a Fenwick hierarchy of memories, through loglinear_scan_fwd.
    q, k: [B,H,T,dk] bf16; v: [B,H,T,dv] bf16; lam: [B,H,T,L] fp32 level weights
    (L >= loglinear_levels(T)). Returns out [B,H,T,dv] bf16."""
    import torch

    B, H, T, dk = q.shape
    dv = v.shape[-1]
    L = lam.shape[-1]
    dev = q.device
    _check(q, "q", (B, H, T, dk), torch.bfloat16, dev)
    _check(k, "k", (B, H, T, dk), torch.bfloat16, dev)
    _check(v, "v", (B, H, T, dv), torch.bfloat16, dev)
    _check(lam, "lambda", (B, H, T, L), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.bfloat16, device=dev)
    _check(out, "out", (B, H, T, dv), torch.bfloat16, dev)
    rc = lib().loglinear_scan_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), B, H, T, dk,
                                  dv, L, DR_IN_BF16, _stream_handle(dev))
    if rc != DR_OK:
        raise DrScanError(rc, "loglinear_scan_fwd")
    return out


def poll_error(device=None) -> int:
    """Synchronise the current stream and return/clear the device status word."""
    import torch

    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    return int(lib().dr_poll_error(_stream_handle(dev)))


def chunked_plan(mode, BH: int, dk: int, dv: int) -> tuple:
    """(value channels per chain CTA, prep CTAs per head; 0 = unsplit) that dr_scan_fwd uses
    for bf16 inputs on the current device, or None when the chunked kernel does not apply."""
    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    bv, nprep = ctypes.c_int(0), ctypes.c_int(0)
    st = lib().dr_chunked_plan(variant | DR_IN_BF16, int(BH), int(dk), int(dv),
                               ctypes.byref(bv), ctypes.byref(nprep))
    if st == DR_ERR_UNSUPPORTED:
        return None
    if st != DR_OK:
        raise DrScanError(st, "dr_chunked_plan")
    return bv.value, nprep.value


def chunked_plan_ex(mode, BH: int, T: int, dk: int, dv: int, chained=False) -> tuple:
    """(value channels per chain CTA, prep CTAs per head, segments per head) for bf16 inputs
    of length T on the current device, or None when the chunked kernel does not apply. With
    more than one segment the first two describe the launches over B*H*segments sequences."""
    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    bv, nprep, nseg = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    flags = variant | DR_IN_BF16 | (DR_CHAINED if chained else 0)
    st = lib().dr_chunked_plan_ex(flags, int(BH), int(T), int(dk), int(dv), ctypes.byref(bv),
                                  ctypes.byref(nprep), ctypes.byref(nseg))
    if st == DR_ERR_UNSUPPORTED:
        return None
    if st != DR_OK:
        raise DrScanError(st, "dr_chunked_plan_ex")
    return bv.value, nprep.value, nseg.value


def segment_counters(device=None) -> tuple:
    """(segmented scans, chained reruns after a failed hand-off check) on the device since
    the library was loaded; waits for the device's work first."""
    import torch

    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        scans, reruns = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
        st = lib().dr_segment_counters(ctypes.byref(scans), ctypes.byref(reruns))
    if st != DR_OK:
        raise DrScanError(st, "dr_segment_counters")
    return scans.value, reruns.value


def chunked_applies(mode, dtype_is_bf16: bool, dk: int, dv: int) -> bool:
    """Whether dr_scan_fwd runs the chunked tensor-core kernel for this request."""
    variant = MODES[mode] if isinstance(mode, str) else int(mode)
    return (dtype_is_bf16 and dk == 128 and dv in (32, 64, 128)
            and variant in (DR_DELTANET, DR_GDN, DR_KDA, DR_GDN2))
