"""fp64 definition of the fused prologue (TEST INFRASTRUCTURE ONLY).

The kernels can take raw projections and apply, per token and head, the
activations the workloads otherwise apply before the recurrence: L2
normalisation of q and k over the head dimension, sigmoid of the gains and
gates, and a softplus or log-sigmoid decay. This module writes those maps out
in numpy fp64; the oracle of the fused path is ``oracle.forward`` on
``apply(raw, ...)``. Bits as in the C ABI (pdn.h, PDN_PRO_*).
Pinned by closed forms and by scipy's reference functions
(tests/test_oracle_pins.py).
"""
from __future__ import annotations

import numpy as np

L2NORM_QK, SIGMOID_GATES, DECAY_SOFTPLUS, DECAY_LOGSIGMOID = 1, 2, 4, 8


def l2_normalise(x):
    """x / max(||x||, 1e-12) over the last axis."""
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-12)


def sigmoid(x):
    """1 / (1 + e^-x), evaluated without overflow on either side."""
    x = np.asarray(x, np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def softplus(x):
    """log(1 + e^x) = max(x, 0) + log(1 + e^-|x|)."""
    x = np.asarray(x, np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def apply(raw: dict, prologue: int, decay_scale: float = 1.0) -> dict:
    """The activated inputs (float64) of raw projections ``raw`` (the keys of
    the workload generator: q, k, v, log_alpha, beta, erase, write)."""
    out = {}
    for n, a in raw.items():
        if a is None:
            out[n] = None
            continue
        if hasattr(a, "detach"):
            a = a.detach().to("cpu").double().numpy()
        out[n] = np.asarray(a, np.float64)
    if prologue & L2NORM_QK:
        out["q"] = l2_normalise(out["q"])
        out["k"] = l2_normalise(out["k"])
    if prologue & SIGMOID_GATES:
        for n in ("beta", "erase", "write"):
            if out.get(n) is not None:
                out[n] = sigmoid(out[n])
    if out.get("log_alpha") is not None:
        if prologue & DECAY_SOFTPLUS:
            out["log_alpha"] = -decay_scale * softplus(out["log_alpha"])
        elif prologue & DECAY_LOGSIGMOID:
            out["log_alpha"] = -softplus(-out["log_alpha"])
    return out
