"""Seeded synthetic inputs for the gated delta-rule forward and decode.

This module only draws random numbers in a fixed order and shapes them; it
holds none of the recurrence's arithmetic, so both the CUDA path and the fp64
oracle consume its tensors. Draw order (one ``torch.Generator`` seeded per
workload): q, k, v, beta, decay, erase, write. Everything is drawn in fp32,
q and k are L2-normalised per token and head, then tensors are cast to the
workload dtype (scalar beta and scalar log-decay stay fp32).

The shapes stand in for the 340M-1.3B language-model layers the pages train
(hidden 2048 = 16 heads x 128); no dataset is involved.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

DECAY_OF_VARIANT = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar",
                    "KDA": "channel", "PKDA": "channel"}
PRECOND_VARIANTS = ("PDN", "PGDN", "PKDA", "PLA")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    variant: str            # DN GDN KDA PDN PGDN PKDA FG2_GDN GDN2 PLA FG2_GDN_PLUS
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str              # "f32" | "bf16"
    decay: str              # "none" | "scalar" | "channel"
    decay_recipe: str = "softplus"   # "softplus": -0.1*softplus(N(0,1)); "sigmoid": log sigmoid(N(2,1));
                                     # "strong": 2 * decay_mean * sigmoid(N(0,1)) (mean decay_mean)
    decay_mean: float = 0.0          # mean per-token log decay of the "strong" recipe
    hard_decay: bool = False         # channel 3 (channel decay) or every 7th token (scalar) at log alpha = -30
    chunk: int = 64
    precond_x: float = 1.5
    precond_eps: float = 1e-6
    q_scale: float = 1.0
    seed: int = 0
    decode_steps: int = 0   # >0: a decode workload (T == decode_steps tokens per sequence)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The workloads the build is measured and checked on.
WORKLOADS = {
    # Preconditioned DeltaNet, fp32, tiny: parity at 1e-4.
    "pdn_f32_small": Workload("pdn_f32_small", "PDN", 1, 512, 2, 64, 64, "f32", "none"),
    # Preconditioned GDN, bf16 inputs, fp32 state: the headline forward layer.
    "pgdn_bf16_4k": Workload("pgdn_bf16_4k", "PGDN", 4, 4096, 16, 128, 128, "bf16", "scalar"),
    # Preconditioned KDA at the 1.3B-layer shape, channel decay from sigmoid(N(2,1)).
    "pkda_bf16_8k": Workload("pkda_bf16_8k", "PKDA", 8, 8192, 16, 128, 128, "bf16", "channel",
                             decay_recipe="sigmoid"),
    # FG2-GDN and Gated DeltaNet-2 at 32k tokens, channel decay.
    "fg2_bf16_32k": Workload("fg2_bf16_32k", "FG2_GDN", 2, 32768, 16, 128, 128, "bf16", "channel"),
    "gdn2_bf16_32k": Workload("gdn2_bf16_32k", "GDN2", 2, 32768, 16, 128, 128, "bf16", "channel"),
    # Preconditioned linear attention (scalar decay) and FG2-GDN+ (channel
    # decay) at the headline layer shape.
    "pla_bf16_4k": Workload("pla_bf16_4k", "PLA", 4, 4096, 16, 128, 128, "bf16", "scalar"),
    "fg2p_bf16_4k": Workload("fg2p_bf16_4k", "FG2_GDN_PLUS", 4, 4096, 16, 128, 128, "bf16",
                             "channel"),
    # Recurrent decode of Preconditioned GDN: 256 sequences x 16 heads, 1024 steps.
    "pgdn_decode_256": Workload("pgdn_decode_256", "PGDN", 256, 1024, 16, 128, 128, "bf16",
                                "scalar", decode_steps=1024),
}


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_inputs(w: Workload, device="cpu", B: Optional[int] = None, T: Optional[int] = None,
                generator_device: Optional[str] = None) -> dict:
    """Draw the inputs of workload ``w`` (optionally with B or T overridden).

    Returns a dict with q, k, v, log_alpha, beta, erase, write (None where the
    variant does not use them). ``generator_device`` picks where the random
    numbers are drawn (defaults to ``device``); the same (seed, generator
    device, shape) always gives the same tensors.
    """
    B = w.B if B is None else B
    T = w.T if T is None else T
    gdev = torch.device(generator_device or device)
    g = torch.Generator(device=gdev)
    g.manual_seed(w.seed)
    dt = w.torch_dtype
    H, dk, dv = w.H, w.dk, w.dv

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=gdev, dtype=torch.float32)

    q = _l2n(randn(B, T, H, dk)).to(dt)
    k = _l2n(randn(B, T, H, dk)).to(dt)
    v = randn(B, T, H, dv).to(dt)
    beta = None
    if w.variant in ("FG2_GDN", "FG2_GDN_PLUS"):
        beta = torch.sigmoid(randn(B, T, H, dk)).to(dt)
    elif w.variant != "GDN2":
        beta = torch.sigmoid(randn(B, T, H))
    log_alpha = None
    if w.decay != "none":
        shape = (B, T, H) if w.decay == "scalar" else (B, T, H, dk)
        z = randn(*shape)
        if w.decay_recipe == "sigmoid":
            la = torch.nn.functional.logsigmoid(z + 2.0)
        elif w.decay_recipe == "strong":
            la = 2.0 * w.decay_mean * torch.sigmoid(z)
        else:
            la = -0.1 * torch.nn.functional.softplus(z)
        if w.hard_decay:
            if w.decay == "scalar":
                la[:, ::7] = -30.0
            else:
                la[..., 3] = -30.0
        log_alpha = la if w.decay == "scalar" else la.to(dt)
    erase = write = None
    if w.variant == "GDN2":
        erase = torch.sigmoid(randn(B, T, H, dk)).to(dt)
        write = torch.sigmoid(randn(B, T, H, dv)).to(dt)
    elif w.variant == "FG2_GDN_PLUS":  # the value-side gain vector
        write = torch.sigmoid(randn(B, T, H, dv)).to(dt)
    out = dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, erase=erase, write=write)
    return {n: (t.to(device) if t is not None else None) for n, t in out.items()}


# fused-prologue bits (pdn.h PDN_PRO_*)
PRO_L2NORM_QK, PRO_SIGMOID_GATES, PRO_DECAY_SOFTPLUS, PRO_DECAY_LOGSIGMOID = 1, 2, 4, 8


def raw_prologue(w: Workload):
    """(prologue bits, decay scale) that turn the raw projections of
    ``make_raw_inputs(w)`` into the inputs ``make_inputs(w)`` draws."""
    bits = PRO_L2NORM_QK | PRO_SIGMOID_GATES
    if w.decay == "none":
        return bits, 1.0
    if w.decay_recipe == "sigmoid":
        return bits | PRO_DECAY_LOGSIGMOID, 1.0
    if w.decay_recipe == "softplus":
        return bits | PRO_DECAY_SOFTPLUS, 0.1
    raise ValueError("no raw form for the %r decay recipe" % w.decay_recipe)


def make_raw_inputs(w: Workload, device="cpu", B: Optional[int] = None, T: Optional[int] = None,
                    generator_device: Optional[str] = None) -> dict:
    """The raw projections behind ``make_inputs(w)``: the same seed and draw
    order, with the activations left to a fused prologue (q and k not
    normalised, gains and gates as logits, the decay as its pre-activation
    z, or z + 2 for the log-sigmoid recipe)."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    gdev = torch.device(generator_device or device)
    g = torch.Generator(device=gdev)
    g.manual_seed(w.seed)
    dt = w.torch_dtype
    H, dk, dv = w.H, w.dk, w.dv

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=gdev, dtype=torch.float32)

    q = randn(B, T, H, dk).to(dt)
    k = randn(B, T, H, dk).to(dt)
    v = randn(B, T, H, dv).to(dt)
    beta = None
    if w.variant in ("FG2_GDN", "FG2_GDN_PLUS"):
        beta = randn(B, T, H, dk).to(dt)
    elif w.variant != "GDN2":
        beta = randn(B, T, H)
    log_alpha = None
    if w.decay != "none":
        raw_prologue(w)  # rejects recipes without a raw form
        shape = (B, T, H) if w.decay == "scalar" else (B, T, H, dk)
        z = randn(*shape)
        if w.decay_recipe == "sigmoid":
            z = z + 2.0
        log_alpha = z if w.decay == "scalar" else z.to(dt)
    erase = write = None
    if w.variant == "GDN2":
        erase = randn(B, T, H, dk).to(dt)
        write = randn(B, T, H, dv).to(dt)
    elif w.variant == "FG2_GDN_PLUS":
        write = randn(B, T, H, dv).to(dt)
    out = dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, erase=erase, write=write)
    return {n: (t.to(device) if t is not None else None) for n, t in out.items()}


def slice_chain(inputs: dict, b: int, h: int, t0: int = 0, t1: Optional[int] = None) -> dict:
    """The inputs of one (batch, head) chain over tokens [t0, t1), as a B=1,
    H=1 problem on the CPU (used to check sampled chains of large workloads)."""
    out = {}
    for n, t in inputs.items():
        if t is None:
            out[n] = None
            continue
        s = t[b:b + 1, t0:t1, h:h + 1]
        out[n] = s.to("cpu")
    return out
