"""Shared helpers for the GPU parity tests: run the CUDA path through the C
ABI and the fp64 oracle on the same seeded inputs, and compare them.

Error metric (the reading of "max relative error" used throughout): the
normalised max-abs error  max|gpu - ref| / max|ref|, computed separately over
the outputs o and over the final state S_T. Bars: 1e-4 for fp32 inputs,
2e-2 for bf16 inputs with an fp32 state. Alongside it every check records,
without gating on it, the elementwise relative error
max |gpu - ref| / max(|ref|, 1e-3 rms(ref)); the session summary lists it.
"""
import numpy as np
import torch

import oracle
from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import (PRECOND_VARIANTS, Workload,
                                                               make_inputs, slice_chain)

TOL = {"f32": 1e-4, "bf16": 2e-2}

# (test workload name, dtype, normalised error of o, of S_T, elementwise
# relative error of o, of S_T), appended by every assert_parity call
REPORT = []


def nmax_err(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = np.abs(ref).max()
    if denom == 0:
        return float(np.abs(gpu).max())
    return float(np.abs(gpu - ref).max() / denom)


def elem_rel_err(gpu, ref, floor=1e-3):
    """max |gpu - ref| / max(|ref|, floor * rms(ref)), elementwise."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    den = np.maximum(np.abs(ref), floor * rms)
    if rms == 0:
        return float(np.abs(gpu).max())
    return float((np.abs(gpu - ref) / den).max())


def gates(inputs):
    return {n: inputs[n] for n in ("log_alpha", "beta", "erase", "write")}


def run_gpu(w: Workload, inputs, S0=None, A0=None, impl="auto", chunk=None):
    dev = torch.device("cuda")
    d = {n: (t.to(dev) if t is not None else None) for n, t in inputs.items()}
    o, ST, AT = pdn.chunk_fwd(w.variant, d["q"], d["k"], d["v"], **gates(d),
                              S0=None if S0 is None else S0.to(dev),
                              A0=None if A0 is None else A0.to(dev),
                              chunk=chunk or w.chunk, impl=impl, q_scale=w.q_scale,
                              precond_x=w.precond_x, precond_eps=w.precond_eps)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    return o, ST, AT


def run_oracle(w: Workload, inputs, S0=None, A0=None):
    return oracle.forward(w.variant, inputs["q"], inputs["k"], inputs["v"],
                          log_alpha=inputs["log_alpha"], beta=inputs["beta"],
                          erase=inputs["erase"], write=inputs["write"], S0=S0, A0=A0,
                          q_scale=w.q_scale, x=w.precond_x, eps=w.precond_eps)


def assert_parity(w: Workload, o_gpu, ST_gpu, AT_gpu, o_ref, ST_ref, AT_ref, tol=None, tol_a=1e-5):
    tol = TOL[w.dtype] if tol is None else tol
    og = o_gpu.float().cpu().numpy()
    sg = ST_gpu.cpu().numpy()
    e_o = nmax_err(og, o_ref)
    e_s = nmax_err(sg, ST_ref)
    r_o = elem_rel_err(og, o_ref)
    r_s = elem_rel_err(sg, ST_ref)
    REPORT.append((w.name, w.dtype, e_o, e_s, r_o, r_s))
    msg = "%s: err(o)=%.3g err(S_T)=%.3g tol=%.3g (elementwise rel: o %.3g, S_T %.3g)" % (
        w.name, e_o, e_s, tol, r_o, r_s)
    assert e_o <= tol and e_s <= tol, msg
    if w.variant in PRECOND_VARIANTS and AT_gpu is not None:
        e_a = nmax_err(AT_gpu.cpu().numpy(), AT_ref)
        assert e_a <= tol_a, "%s: err(A_T)=%.3g" % (w.name, e_a)
    return e_o, e_s
