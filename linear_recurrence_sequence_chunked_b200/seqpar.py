"""Sequence-parallel prefill: one long sequence cut into segments, one per
rank, joined by exchanges of small per-(batch, head) tensors ("FG2-GDN", ja
§4, 32k-token contexts).

Every update acts on the state by right-multiplication, so segment g maps its
start state affinely, S_end = S_start A_g + B_g. Rank g:
  1. preconditioned variants: its key energy E_g; all-gather; the accumulator
     at its start is A0 + sum_{h<g} E_h (its coefficients depend on it);
  2. B_g = final state of its segment from S = 0; A_g = the segment's
     transition (the chunked forward with zero targets from the identity);
  3. all-gather (A_g, B_g); S_start(g) = fold of S -> S A_h + B_h over h < g
     from the sequence's S0;
  4. its outputs: the chunked forward of its segment from S_start(g).
Every arithmetic step runs in the library's kernels (``CudaOps``);
torch.distributed only moves tensors (the all-gathers). ``SegmentPrefill``
exposes the phases so that a test can run several segments in one process.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch

from . import pdn


class CudaOps:
    """The per-segment operations through the C ABI, on one CUDA device."""

    def __init__(self, variant: str, decay: str, chunk: int = 64, impl: str = "auto",
                 q_scale: float = 1.0, precond_x: float = 1.5, precond_eps: float = 1e-6,
                 prologue: int = 0, decay_scale: float = 1.0):
        self.variant = variant
        self.decay = decay
        self.kw = dict(chunk=chunk, impl=impl, q_scale=q_scale, precond_x=precond_x,
                       precond_eps=precond_eps, prologue=prologue, decay_scale=decay_scale)
        self.precond = variant in pdn.PRECOND_VARIANTS

    def _problem(self, x, T=None):
        B, Tx, H, dk = x["k"].shape
        dv = x["v"].shape[3] if x.get("v") is not None else dk
        kw = self.kw
        return pdn.make_problem(self.variant, B, Tx if T is None else T, H, dk, dv, x["k"].dtype,
                                self.decay, kw["chunk"], kw["impl"], kw["q_scale"],
                                kw["precond_x"], kw["precond_eps"], kw["prologue"],
                                kw["decay_scale"])

    @staticmethod
    def _stream(x):
        return torch.cuda.current_stream(x["k"].device).cuda_stream

    def key_energy(self, x):
        B, T, H, dk = x["k"].shape
        E = torch.empty(B, H, dk, dtype=torch.float32, device=x["k"].device)
        t = pdn.make_tensors(None, x["k"], None, None, AT=E)
        pdn._check(pdn.pdn_key_energy(self._problem(x), t, self._stream(x)), "pdn_key_energy")
        return E

    def accumulate(self, parts, n, base):
        out = torch.empty_like(parts[0])
        rc = pdn.pdn_accumulate(n, parts[0].numel(), parts.data_ptr(),
                                None if base is None else base.data_ptr(), out.data_ptr(),
                                torch.cuda.current_stream(parts.device).cuda_stream)
        pdn._check(rc, "pdn_accumulate")
        return out

    def forward(self, x, S0, A0):
        kw = self.kw
        return pdn.chunk_fwd(self.variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"],
                             beta=x["beta"], erase=x["erase"], write=x["write"], S0=S0, A0=A0,
                             **kw)

    def transition(self, x, A0):
        B, T, H, dk = x["k"].shape
        p = self._problem(x)
        p.d_v = dk
        ws_bytes = pdn.pdn_chunk_fwd_workspace(p)
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x["k"].device)
        A = torch.empty(B, H, dk, dk, dtype=torch.float32, device=x["k"].device)
        AT = torch.empty(B, H, dk, dtype=torch.float32, device=x["k"].device) if self.precond else None
        t = pdn.make_tensors(x["q"], x["k"], None, None, x["log_alpha"], x["beta"], x["erase"],
                             x["write"], ST=A, A0=A0, AT=AT)
        pdn._check(pdn.pdn_chunk_transition(p, t, ws.data_ptr(), ws.numel(), self._stream(x)),
                   "pdn_chunk_transition")
        return A

    def compose(self, S_in, A, B_add):
        BH = A.shape[0] * A.shape[1]
        dv, dk = B_add.shape[2], B_add.shape[3]
        out = torch.empty_like(B_add)
        rc = pdn.pdn_state_compose(BH, dv, dk, None if S_in is None else S_in.data_ptr(),
                                   A.data_ptr(), B_add.data_ptr(), out.data_ptr(),
                                   torch.cuda.current_stream(A.device).cuda_stream)
        pdn._check(rc, "pdn_state_compose")
        return out


class SegmentPrefill:
    """The phases of one rank's segment (``x``: that segment's inputs)."""

    def __init__(self, ops, x: dict, rank: int):
        self.ops, self.x, self.rank = ops, x, rank
        self.A_start = None

    def energy(self):
        """Phase 1 (preconditioned variants): this segment's key energy."""
        return self.ops.key_energy(self.x)

    def local(self, energies, A0):
        """Phase 2: the accumulator at this segment's start (from the gathered
        energies, stacked [world, ...], or None), then (A_g, B_g)."""
        if self.ops.precond:
            self.A_start = self.ops.accumulate(energies, self.rank, A0)
        _, B_g, _ = self.ops.forward(self.x, None, self.A_start)
        A_g = self.ops.transition(self.x, self.A_start)
        return A_g, B_g

    def finish(self, A_all, B_all, S0):
        """Phase 3: the start state from the segments before this one, then
        this segment's outputs: (o, S at its end, accumulator at its end)."""
        S = S0
        for g in range(self.rank):
            S = self.ops.compose(S, A_all[g], B_all[g])
        return self.ops.forward(self.x, S, self.A_start)


def seqpar_forward(ops, x: dict, rank: int, world: int,
                   all_gather: Callable[[torch.Tensor], torch.Tensor],
                   S0: Optional[torch.Tensor] = None, A0: Optional[torch.Tensor] = None):
    """Rank ``rank``'s part of a sequence-parallel prefill over ``world``
    ranks. ``x`` holds this rank's segment (segments in rank order);
    ``all_gather(t)`` returns the ``world`` ranks' tensors stacked on a new
    first axis; S0 and A0 are the sequence's initial state and accumulator
    (the same on every rank). Returns (o of this segment, state at its end,
    accumulator at its end); rank world - 1 holds the sequence's final state."""
    seg = SegmentPrefill(ops, x, rank)
    energies = all_gather(seg.energy()) if ops.precond else None
    A_g, B_g = seg.local(energies, A0)
    A_all, B_all = all_gather(A_g), all_gather(B_g)
    return seg.finish(A_all, B_all, S0)


def nccl_all_gather(group=None):
    """all_gather over torch.distributed (NCCL for CUDA tensors), stacked."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out

    return gather
