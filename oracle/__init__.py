"""fp64 CPU oracle for the gated delta-rule forward recurrence.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg (and its ``--impl reference`` arm) may import
this package. It shares no code with the CUDA library: the token loop lives in
``pdn_oracle.c`` (plain C, fp64, one POSIX thread per (batch, head) chain), the
chunk-form cross-check in ``chunked.py`` (numpy, fp64).

Parity status
-------------
* token loop (every variant): pinned by closed forms, brute force and the
  least-squares identity (tests/test_oracle_pins.py);
* backward (every variant): the analytic reverse-time adjoint, pinned by
  central finite differences of the token loop on every input;
* diagonal preconditioner: pinned by its invariants; the page-level constants
  (centring, eps, base of the exponential) are readings of the pages, so the
  match with the original paper is **parity unpinned** for those constants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

VARIANTS = {"DN": 0, "GDN": 1, "KDA": 2, "PDN": 3, "PGDN": 4, "PKDA": 5,
            "FG2_GDN": 6, "GDN2": 7, "PLA": 8, "FG2_GDN_PLUS": 9}
DECAYS = {"none": 0, "scalar": 1, "channel": 2}
PRECOND_VARIANTS = ("PDN", "PGDN", "PKDA", "PLA")


def build(force: bool = False) -> str:
    """Compile ``pdn_oracle.c`` into ``liboracle.so`` next to it (gcc)."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
            return _LIB
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L",
                               "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
        return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        D = ctypes.POINTER(ctypes.c_double)
        I = ctypes.c_int
        lib.oracle_forward.restype = I
        lib.oracle_forward.argtypes = [I, I, I, I, I, I, I, D, D, D, D, D, D, D, D, D,
                                       ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                       D, D, D, I]
        lib.oracle_generic.restype = I
        lib.oracle_generic.argtypes = [I, I, I, I, I, D, D, D, D, D, D, ctypes.c_double,
                                       D, D, I]
        lib.oracle_backward.restype = I
        lib.oracle_backward.argtypes = [I, I, I, I, I, I, I, D, D, D, D, D, D, D, D, D,
                                        ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                        D, D, D, D, D, D, D, D, D, D, D]
        lib.oracle_precond.restype = I
        lib.oracle_precond.argtypes = [I, I, D, D, ctypes.c_double, ctypes.c_double, D, D]
        _lib = lib
    return _lib


def _f64(a):
    """Upcast an input (numpy array or torch tensor, any float dtype) to a
    contiguous float64 numpy array, exactly (every bf16/fp32 value is an fp64)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor, without importing torch here
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(variant, q, k, v, log_alpha=None, beta=None, erase=None, write=None,
            S0=None, A0=None, q_scale=1.0, x=1.5, eps=1e-6, nthreads=0,
            want_o=True):
    """Run the token-by-token recurrence for ``variant``.

    Shapes: q, k [B,T,H,dk]; v [B,T,H,dv]; log_alpha None | [B,T,H] (scalar
    decay) | [B,T,H,dk] (channel decay); beta [B,T,H] | [B,T,H,dk] (FG2_GDN,
    FG2_GDN_PLUS: the key-side gain); erase [B,T,H,dk] (GDN2); write
    [B,T,H,dv] (GDN2's write gate, FG2_GDN_PLUS's value-side gain);
    S0 [B,H,dv,dk]; A0 [B,H,dk].
    Returns (o [B,T,H,dv] or None, S_T [B,H,dv,dk], A_T [B,H,dk]) in fp64.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, dk = k.shape
    dv = v.shape[3]
    la, be, er, wr = _f64(log_alpha), _f64(beta), _f64(erase), _f64(write)
    s0, a0 = _f64(S0), _f64(A0)
    decay = 0 if la is None else (1 if la.ndim == 3 else 2)
    o = np.zeros((B, T, H, dv), np.float64) if want_o else None
    ST = np.zeros((B, H, dv, dk), np.float64)
    AT = np.zeros((B, H, dk), np.float64)
    rc = lib.oracle_forward(VARIANTS[variant], decay, B, T, H, dk, dv,
                            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(er),
                            _ptr(wr), _ptr(s0), _ptr(a0), float(q_scale), float(x),
                            float(eps), _ptr(o), _ptr(ST), _ptr(AT), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_forward failed with code %d" % rc)
    return o, ST, AT


def backward(variant, q, k, v, log_alpha=None, beta=None, erase=None, write=None,
             S0=None, A0=None, q_scale=1.0, x=1.5, eps=1e-6, dO=None, dST=None):
    """Gradients of a scalar loss L with dL/do = dO [B,T,H,dv] and
    dL/dS_T = dST [B,H,dv,dk] (either may be None = 0), through the token loop
    of ``forward``: a dict with q, k, v, log_alpha, beta, erase, write, S0, A0
    (None for inputs the variant does not take). Pinned by finite differences."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, dk = k.shape
    dv = v.shape[3]
    la, be, er, wr = _f64(log_alpha), _f64(beta), _f64(erase), _f64(write)
    s0, a0, do, dst = _f64(S0), _f64(A0), _f64(dO), _f64(dST)
    decay = 0 if la is None else (1 if la.ndim == 3 else 2)
    g = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v),
         "log_alpha": None if la is None else np.zeros_like(la),
         "beta": None if be is None else np.zeros_like(be),
         "erase": None if er is None else np.zeros_like(er),
         "write": None if wr is None else np.zeros_like(wr),
         "S0": np.zeros((B, H, dv, dk)), "A0": np.zeros((B, H, dk))}
    rc = lib.oracle_backward(VARIANTS[variant], decay, B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                             _ptr(la), _ptr(be), _ptr(er), _ptr(wr), _ptr(s0), _ptr(a0),
                             float(q_scale), float(x), float(eps), _ptr(do), _ptr(dst),
                             _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["log_alpha"]),
                             _ptr(g["beta"]), _ptr(g["erase"]), _ptr(g["write"]), _ptr(g["S0"]),
                             _ptr(g["A0"]))
    if rc != 0:
        raise ValueError("oracle_backward failed with code %d" % rc)
    if variant not in PRECOND_VARIANTS:
        g["A0"] = None
    return g


def generic(q, r, w, u, log_alpha=None, S0=None, q_scale=1.0, nthreads=0):
    """Generic delta step with caller-given read key r, write key w and target u
    (all [B,T,H,d]); log_alpha None or channel [B,T,H,dk]. Returns (o, S_T)."""
    lib = _load()
    q, r, w, u = _f64(q), _f64(r), _f64(w), _f64(u)
    la, s0 = _f64(log_alpha), _f64(S0)
    B, T, H, dk = r.shape
    dv = u.shape[3]
    o = np.zeros((B, T, H, dv), np.float64)
    ST = np.zeros((B, H, dv, dk), np.float64)
    rc = lib.oracle_generic(B, T, H, dk, dv, _ptr(q), _ptr(r), _ptr(w), _ptr(u),
                            _ptr(la), _ptr(s0), float(q_scale), _ptr(o), _ptr(ST),
                            int(nthreads))
    if rc != 0:
        raise ValueError("oracle_generic failed with code %d" % rc)
    return o, ST


def precond(k, A0=None, x=1.5, eps=1e-6):
    """Preconditioner coefficients B_t [T,dk] and final accumulator A_T [dk]
    for one key sequence k [T,dk]."""
    lib = _load()
    k = _f64(k)
    T, dk = k.shape
    a0 = _f64(A0)
    Bc = np.zeros((T, dk), np.float64)
    AT = np.zeros((dk,), np.float64)
    rc = lib.oracle_precond(T, dk, _ptr(k), _ptr(a0), float(x), float(eps),
                            _ptr(Bc), _ptr(AT))
    if rc != 0:
        raise ValueError("oracle_precond failed with code %d" % rc)
    return Bc, AT
