"""GPU parity of the fused prologue: raw projections in, the kernels apply L2
normalisation of q and k, sigmoid gains and gates and the softplus or
log-sigmoid decay themselves. The oracle is the fp64 recurrence on the same
raw inputs passed through the fp64 prologue (oracle.prologue)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import prologue as oracle_prologue
from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import (WORKLOADS, Workload, make_inputs,
                                                               make_raw_inputs, raw_prologue,
                                                               slice_chain)

from parity_util import TOL, assert_parity, nmax_err

pytestmark = pytest.mark.gpu

CASES = [("PGDN", "scalar", "softplus"), ("PKDA", "channel", "sigmoid"),
         ("KDA", "channel", "softplus"), ("FG2_GDN", "channel", "softplus"),
         ("GDN2", "channel", "sigmoid"), ("FG2_GDN_PLUS", "channel", "softplus"),
         ("PLA", "scalar", "softplus"), ("PDN", "none", "softplus")]


def oracle_on_raw(w, raw, S0=None, A0=None):
    bits, scale = raw_prologue(w)
    a = oracle_prologue.apply(raw, bits, scale)
    return oracle.forward(w.variant, a["q"], a["k"], a["v"], log_alpha=a["log_alpha"],
                          beta=a["beta"], erase=a["erase"], write=a["write"], S0=S0, A0=A0,
                          q_scale=w.q_scale, x=w.precond_x, eps=w.precond_eps)


def gpu_on_raw(w, raw, impl, S0=None, A0=None):
    bits, scale = raw_prologue(w)
    d = {n: (t.cuda() if t is not None else None) for n, t in raw.items()}
    o, ST, AT = pdn.chunk_fwd(w.variant, d["q"], d["k"], d["v"], log_alpha=d["log_alpha"],
                              beta=d["beta"], erase=d["erase"], write=d["write"],
                              S0=None if S0 is None else S0.cuda(),
                              A0=None if A0 is None else A0.cuda(), impl=impl,
                              q_scale=w.q_scale, precond_x=w.precond_x,
                              precond_eps=w.precond_eps, prologue=bits, decay_scale=scale)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    return o, ST, AT


@pytest.mark.parametrize("impl,dtype,d", [("tc", "bf16", 128), ("simt", "bf16", 64),
                                          ("simt", "f32", 64)])
@pytest.mark.parametrize("variant,decay,recipe", CASES)
def test_fused_prologue_matches_oracle(variant, decay, recipe, impl, dtype, d):
    w = Workload("pro-%s-%s" % (variant, impl), variant, 2, 150, 2, d, d, dtype, decay,
                 decay_recipe=recipe, q_scale=0.9)
    raw = make_raw_inputs(w)
    g = torch.Generator().manual_seed(6)
    S0 = 0.3 * torch.randn(w.B, w.H, d, d, generator=g)
    A0 = torch.rand(w.B, w.H, d, generator=g) if variant in pdn.PRECOND_VARIANTS else None
    o, ST, AT = gpu_on_raw(w, raw, impl, S0, A0)
    # the kernels normalise k themselves (fp32, then bf16 as operands), so the
    # accumulator of k.k carries that rounding: 1e-3 for A_T
    assert_parity(w, o, ST, AT, *oracle_on_raw(w, raw, S0, A0), tol_a=1e-3)


@pytest.mark.parametrize("variant,decay,recipe", CASES[:4])
def test_fused_prologue_equals_separate_activations(variant, decay, recipe):
    """The raw projections through the fused prologue and the workload's own
    activated inputs (same seed, activations applied before the call) give the
    same outputs up to the rounding of the activated inputs to bf16."""
    w = Workload("pro-eq-%s" % variant, variant, 2, 200, 2, 128, 128, "bf16", decay,
                 decay_recipe=recipe)
    o1, S1, _ = gpu_on_raw(w, make_raw_inputs(w), "tc")
    x = {n: (t.cuda() if t is not None else None) for n, t in make_inputs(w).items()}
    o2, S2, _ = pdn.chunk_fwd(w.variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"],
                              beta=x["beta"], erase=x["erase"], write=x["write"])
    torch.cuda.synchronize()
    assert nmax_err(o1.float().cpu().numpy(), o2.float().cpu().numpy()) < 2e-2
    assert nmax_err(S1.cpu().numpy(), S2.cpu().numpy()) < 2e-2


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
@pytest.mark.parametrize("variant,decay,recipe", CASES)
def test_fused_prologue_decode(variant, decay, recipe, dtype, d):
    """Decode with raw token projections (both decode kernels: d = 128 takes
    the streaming kernel, d = 64 the generic one)."""
    w = Workload("pro-dec-%s" % variant, variant, 3, 10, 2, d, d, dtype, decay,
                 decay_recipe=recipe, q_scale=1.1)
    raw = make_raw_inputs(w)
    bits, scale = raw_prologue(w)
    S = torch.zeros(w.B, w.H, d, d, device="cuda")
    A = torch.zeros(w.B, w.H, d, device="cuda") if variant in pdn.PRECOND_VARIANTS else None
    dev = {n: (t.cuda() if t is not None else None) for n, t in raw.items()}
    outs = []
    for t in range(w.T):
        sl = {n: (v[:, t:t + 1].contiguous() if v is not None else None) for n, v in dev.items()}
        outs.append(pdn.decode_step(w.variant, sl["q"], sl["k"], sl["v"], S, A,
                                    log_alpha=sl["log_alpha"], beta=sl["beta"], erase=sl["erase"],
                                    write=sl["write"], q_scale=w.q_scale, prologue=bits,
                                    decay_scale=scale))
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    ro, rS, rA = oracle_on_raw(w, raw)
    o = torch.cat(outs, dim=1)
    assert nmax_err(o.float().cpu().numpy(), ro) <= TOL[dtype]
    assert nmax_err(S.cpu().numpy(), rS) <= TOL[dtype]
    if A is not None:
        assert nmax_err(A.cpu().numpy(), rA) <= 1e-3


def test_fused_prologue_headline_layer_sampled_chains():
    """The headline layer (Preconditioned GDN, B4 T4096 H16 d128) from raw
    projections, in the launch configuration the bench times; three sampled
    (batch, head) chains checked against the oracle over all 4096 tokens."""
    w = WORKLOADS["pgdn_bf16_4k"]
    raw = make_raw_inputs(w, device="cuda", generator_device="cuda")
    o, ST, AT = gpu_on_raw(w, raw, "auto")
    for b, h in [(0, 0), (2, 9), (3, 15)]:
        xs = slice_chain(raw, b, h)
        ro, rS, rA = oracle_on_raw(w.replace(B=1, H=1), xs)
        assert nmax_err(o[b:b + 1, :, h:h + 1].float().cpu().numpy(), ro) <= 2e-2
        assert nmax_err(ST[b:b + 1, h:h + 1].cpu().numpy(), rS) <= 2e-2
        assert nmax_err(AT[b:b + 1, h:h + 1].cpu().numpy(), rA) <= 1e-3
