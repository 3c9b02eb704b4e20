"""fp64 stand-ins for the per-segment operations of the sequence-parallel
prefill (test infrastructure): the oracle's token loop for the forward and the
transition, numpy for the key energy, the accumulator sum and the composition.
They let the orchestration in linear_recurrence_sequence_chunked_b200.seqpar
run on CPU ranks (gloo) and be checked against one token loop over the whole
sequence."""
import numpy as np
import torch

import oracle
from oracle import prologue as oracle_prologue

PRECOND = ("PDN", "PGDN", "PKDA", "PLA")


def _t(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a))


class OracleOps:
    def __init__(self, variant, q_scale=1.0, precond_x=1.5, precond_eps=1e-6, prologue=0,
                 decay_scale=1.0):
        self.variant = variant
        self.precond = variant in PRECOND
        self.kw = dict(q_scale=q_scale, x=precond_x, eps=precond_eps)
        self.pro = (prologue, decay_scale)

    def _act(self, x):
        return oracle_prologue.apply(x, *self.pro)

    def key_energy(self, x):
        k = self._act(x)["k"]
        return _t(np.sum(k * k, axis=1))

    def accumulate(self, parts, n, base):
        out = parts[:n].double().sum(0) if n > 0 else torch.zeros_like(parts[0], dtype=torch.float64)
        return out + (0 if base is None else base.double())

    def forward(self, x, S0, A0):
        a = self._act(x)
        o, ST, AT = oracle.forward(self.variant, a["q"], a["k"], a["v"], log_alpha=a["log_alpha"],
                                   beta=a["beta"], erase=a["erase"], write=a["write"], S0=S0,
                                   A0=A0, **self.kw)
        return _t(o), _t(ST), _t(AT)

    def transition(self, x, A0):
        a = self._act(x)
        B, T, H, dk = a["k"].shape
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        _, ST, _ = oracle.forward(self.variant, a["q"], a["k"], np.zeros((B, T, H, dk)),
                                  log_alpha=a["log_alpha"], beta=a["beta"], erase=a["erase"],
                                  write=None if a["write"] is None else np.zeros((B, T, H, dk)) + a["write"][..., :dk],
                                  S0=eye, A0=A0, want_o=False, **self.kw)
        return _t(ST)

    def compose(self, S_in, A, B_add):
        out = B_add.double().clone()
        if S_in is not None:
            out += torch.matmul(S_in.double(), A.double())
        return out
