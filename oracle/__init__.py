"""fp64 CPU oracle of the delta-rule recurrent-memory scan (forward).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package; the product path (the CUDA library and
its Python binding) never does, and shares no code with it.

The arithmetic lives in ``dr_oracle.c`` (plain C, fp64, one token at a time, OpenMP
over independent (batch, head) sequences). This module compiles it with gcc on first
use and marshals numpy arrays through ctypes. See the C file's header for the
sources on the pages and for the readings taken where the pages are silent.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, brute-force definitions and invariants the pages fix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

LINEAR, DELTANET, GDN, KDA, GDN2 = 0, 1, 2, 3, 4

_lib = None


def build(force: bool = False) -> str:
    """Compile dr_oracle.c into liboracle.so (gcc -O2 -fopenmp); return the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_dr_scan.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp] + [ctypes.c_int] * 7
        lib.oracle_dr_scan.restype = ctypes.c_int
        lib.oracle_dr_scan_ex.argtypes = [dp] * 11 + [ctypes.c_int] * 7
        lib.oracle_dr_scan_ex.restype = ctypes.c_int
        lib.oracle_vla_scan.argtypes = [dp] * 6 + [ctypes.c_double] + [dp] * 3 + [ctypes.c_int] * 4
        lib.oracle_vla_scan.restype = ctypes.c_int
        lib.oracle_vla_scan_ex.argtypes = ([dp] * 7 + [ctypes.c_double] + [dp] * 4
                                           + [ctypes.c_int] * 5)
        lib.oracle_vla_scan_ex.restype = ctypes.c_int
        lib.oracle_loglinear_scan.argtypes = [dp] * 5 + [ctypes.c_int] * 6
        lib.oracle_loglinear_scan.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (all host cores unless OMP_NUM_THREADS says otherwise)."""
    return int(_load().oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def dr_scan(q, k, v, beta=None, gate=None, S0=None, mode=DELTANET, residual_pre_decay=False,
            want_state=True):
    """Per-token delta-rule scan in fp64.

    q, k: [B,H,T,dk]; v: [B,H,T,dv]; beta: [B,H,T] (ignored for LINEAR);
    gate: None (LINEAR, DELTANET), [B,H,T] (GDN) or [B,H,T,dk] (KDA), alpha values;
    S0: [B,H,dv,dk] or None (zeros). Returns (out [B,H,T,dv], S_final [B,H,dv,dk] or None).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, T):
        raise ValueError("shape mismatch")
    beta = _f64(beta) if mode != LINEAR else None
    gate = _f64(gate) if mode in (GDN, KDA) else None
    if beta is not None and beta.shape != (B, H, T):
        raise ValueError("beta shape")
    if gate is not None:
        want = (B, H, T) if mode == GDN else (B, H, T, dk)
        if gate.shape != want:
            raise ValueError("gate shape")
    S0 = _f64(S0)
    if S0 is not None and S0.shape != (B, H, dv, dk):
        raise ValueError("S0 shape")
    out = np.empty((B, H, T, dv), np.float64)
    Sf = np.empty((B, H, dv, dk), np.float64) if want_state else None
    rc = _load().oracle_dr_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(S0),
                                _ptr(out), _ptr(Sf), B, H, T, dk, dv, int(mode),
                                int(bool(residual_pre_decay)))
    if rc != 0:
        raise RuntimeError(f"oracle_dr_scan failed ({rc})")
    return out, Sf


def dr_scan_ex(q, k, v, beta=None, gate=None, S0=None, mode=DELTANET, erase=None, write=None,
               residual_pre_decay=False):
    """Per-token delta-rule scan in fp64, every variant including Gated DeltaNet-2, also
    returning the per-token write values u_t = beta_t r_t (v_t for plain linear attention).

    As dr_scan, plus: mode GDN2 takes gate [B,H,T] (alpha), erase [B,H,T,dk] (b) and
    write [B,H,T,dv] (w). Returns (out, S_final, u [B,H,T,dv]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, T):
        raise ValueError("shape mismatch")
    beta = _f64(beta) if mode != LINEAR else None
    gate = _f64(gate) if mode in (GDN, KDA, GDN2) else None
    if beta is not None and beta.shape != (B, H, T):
        raise ValueError("beta shape")
    if gate is not None:
        want = (B, H, T, dk) if mode == KDA else (B, H, T)
        if gate.shape != want:
            raise ValueError("gate shape")
    if mode == GDN2:
        erase, write = _f64(erase), _f64(write)
        if erase is None or erase.shape != (B, H, T, dk):
            raise ValueError("erase shape")
        if write is None or write.shape != (B, H, T, dv):
            raise ValueError("write shape")
    else:
        erase = write = None
    S0 = _f64(S0)
    if S0 is not None and S0.shape != (B, H, dv, dk):
        raise ValueError("S0 shape")
    out = np.empty((B, H, T, dv), np.float64)
    Sf = np.empty((B, H, dv, dk), np.float64)
    u = np.empty((B, H, T, dv), np.float64)
    rc = _load().oracle_dr_scan_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate),
                                   _ptr(erase), _ptr(write), _ptr(S0), _ptr(out), _ptr(Sf),
                                   _ptr(u), B, H, T, dk, dv, int(mode),
                                   int(bool(residual_pre_decay)))
    if rc != 0:
        raise RuntimeError(f"oracle_dr_scan_ex failed ({rc})")
    return out, Sf, u


def vla_scan(q, k, v, u, S0=None, A0=None, lambda0=1.0, want_state=True):
    """Per-token VLA Sherman-Morrison scan in fp64.

    q, k, v, u: [B,H,T,d]; S0, A0: [B,H,d,d] or None (zeros, I/lambda0).
    Returns (out [B,H,T,d], S_final, A_final) (the last two None unless want_state).
    """
    q, k, v, u = _f64(q), _f64(k), _f64(v), _f64(u)
    B, H, T, d = q.shape
    for x in (k, v, u):
        if x.shape != q.shape:
            raise ValueError("shape mismatch")
    S0, A0 = _f64(S0), _f64(A0)
    for x in (S0, A0):
        if x is not None and x.shape != (B, H, d, d):
            raise ValueError("state shape")
    out = np.empty((B, H, T, d), np.float64)
    Sf = np.empty((B, H, d, d), np.float64) if want_state else None
    Af = np.empty((B, H, d, d), np.float64) if want_state else None
    rc = _load().oracle_vla_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(S0), _ptr(A0),
                                 float(lambda0), _ptr(out), _ptr(Sf), _ptr(Af), B, H, T, d)
    if rc != 0:
        raise RuntimeError(f"oracle_vla_scan failed ({rc})")
    return out, Sf, Af


def vla_scan_ratio(q, k, v, u, S0=None, A0=None, n0=None, lambda0=1.0):
    """Per-token VLA scan in fp64 with the ratio readout o_t = S_t q_t / (n_t q_t), where
    n_t = n_{t-1} + (1 - n_{t-1} k_t) alpha_hat_t^T is the same write applied to a value
    held at 1. q: [B,H,T,d] the feature-mapped queries; k: the unit-norm feature-mapped keys;
    n0: [B,H,d] or None (zeros). Returns (out, S_final, A_final, n_final)."""
    q, k, v, u = _f64(q), _f64(k), _f64(v), _f64(u)
    B, H, T, d = q.shape
    for x in (k, v, u):
        if x.shape != q.shape:
            raise ValueError("shape mismatch")
    S0, A0, n0 = _f64(S0), _f64(A0), _f64(n0)
    for x in (S0, A0):
        if x is not None and x.shape != (B, H, d, d):
            raise ValueError("state shape")
    if n0 is not None and n0.shape != (B, H, d):
        raise ValueError("n0 shape")
    out = np.empty((B, H, T, d), np.float64)
    Sf = np.empty((B, H, d, d), np.float64)
    Af = np.empty((B, H, d, d), np.float64)
    nf = np.empty((B, H, d), np.float64)
    rc = _load().oracle_vla_scan_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(u), _ptr(S0), _ptr(A0),
                                    _ptr(n0), float(lambda0), _ptr(out), _ptr(Sf), _ptr(Af),
                                    _ptr(nf), B, H, T, d, 1)
    if rc != 0:
        raise RuntimeError(f"oracle_vla_scan_ex failed ({rc})")
    return out, Sf, Af, nf


def loglinear_levels(T: int) -> int:
    """Levels a log-linear scan of T tokens needs: level 0 plus one per bit of T - 1."""
    return max(1, int(T - 1).bit_length() + 1)


def loglinear_scan(q, k, v, lam):
    """Log-linear attention over a Fenwick hierarchy of linear-attention memories, fp64,
    one token at a time (binary-counter form). q, k: [B,H,T,dk]; v: [B,H,T,dv];
    lam: [B,H,T,L] level weights (L >= loglinear_levels(T)). Returns out [B,H,T,dv]."""
    q, k, v, lam = _f64(q), _f64(k), _f64(v), _f64(lam)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    L = lam.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, T) or lam.shape[:3] != (B, H, T):
        raise ValueError("shape mismatch")
    out = np.empty((B, H, T, dv), np.float64)
    rc = _load().oracle_loglinear_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(out), B, H, T,
                                       dk, dv, L)
    if rc != 0:
        raise RuntimeError(f"oracle_loglinear_scan failed ({rc})")
    return out
