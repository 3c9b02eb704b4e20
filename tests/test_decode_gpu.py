"""GPU parity of the decode step: tokens fed one at a time through
pdn_decode_step must reproduce the oracle's token recurrence, and decoding
after a chunked prefill must continue it."""
import numpy as np
import pytest
import torch

from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import WORKLOADS, Workload, make_inputs

from parity_util import TOL, nmax_err, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

VARIANTS = ["DN", "GDN", "KDA", "PDN", "PGDN", "PKDA", "FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"]
DECAY = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar",
         "KDA": "channel", "PKDA": "channel", "FG2_GDN": "channel", "GDN2": "channel",
         "PLA": "scalar", "FG2_GDN_PLUS": "channel"}


def decode_all(w, x, S, A, steps):
    """Run `steps` decode calls on device copies; returns o [B,steps,H,dv]."""
    dev = torch.device("cuda")
    d = {n: (t.to(dev) if t is not None else None) for n, t in x.items()}
    outs = []
    for t in range(steps):
        sl = {n: (v[:, t:t + 1].contiguous() if v is not None else None) for n, v in d.items()}
        outs.append(pdn.decode_step(w.variant, sl["q"], sl["k"], sl["v"], S, A,
                                    log_alpha=sl["log_alpha"], beta=sl["beta"], erase=sl["erase"],
                                    write=sl["write"], q_scale=w.q_scale, precond_x=w.precond_x,
                                    precond_eps=w.precond_eps))
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    return torch.cat(outs, dim=1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_decode_matches_oracle(variant, dtype):
    w = Workload("dec", variant, 3, 20, 2, 64, 64, dtype, DECAY[variant], q_scale=0.9)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(3)
    S0 = 0.3 * torch.randn(w.B, w.H, w.dv, w.dk, generator=g)
    A0 = torch.rand(w.B, w.H, w.dk, generator=g) if variant in ("PDN", "PGDN", "PKDA", "PLA") else None
    S = S0.cuda()
    A = A0.cuda() if A0 is not None else None
    o = decode_all(w, x, S, A, w.T)
    ro, rS, rA = run_oracle(w, x, S0, A0)
    tol = TOL[dtype]
    assert nmax_err(o.float().cpu().numpy(), ro) <= tol
    assert nmax_err(S.cpu().numpy(), rS) <= tol
    if A is not None:
        assert nmax_err(A.cpu().numpy(), rA) <= 1e-6


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 128), (128, 64), (128, 128)])
def test_decode_head_dims(dk, dv):
    w = Workload("dec", "PGDN", 2, 5, 3, dk, dv, "f32", "scalar")
    x = make_inputs(w)
    S = torch.zeros(w.B, w.H, dv, dk, device="cuda")
    A = torch.zeros(w.B, w.H, dk, device="cuda")
    o = decode_all(w, x, S, A, w.T)
    ro, rS, _ = run_oracle(w, x)
    assert nmax_err(o.cpu().numpy(), ro) <= 1e-4
    assert nmax_err(S.cpu().numpy(), rS) <= 1e-4


def test_prefill_then_decode_continues_forward():
    """Chunked prefill over 200 tokens, then 8 decode steps, equals one
    forward over 208 tokens (fixed-size state carried between calls)."""
    w = Workload("pd", "PKDA", 2, 208, 4, 128, 128, "bf16", "channel")
    x = make_inputs(w)
    o_full, S_full, A_full = run_gpu(w, x)
    xp = {n: (t[:, :200] if t is not None else None) for n, t in x.items()}
    xd = {n: (t[:, 200:] if t is not None else None) for n, t in x.items()}
    _, S, A = run_gpu(w.replace(T=200), xp)
    o_dec = decode_all(w, xd, S, A, 8)
    assert nmax_err(o_dec.float().cpu().numpy(), o_full[:, 200:].float().cpu().numpy()) < 2e-2
    assert nmax_err(S.cpu().numpy(), S_full.cpu().numpy()) < 1e-2


def test_decode_workload_shape_sampled():
    """The decode workload's shape (256 sequences x 16 heads, d 128, fp32
    state, bf16 tokens) for 16 steps, every chain checked against the oracle."""
    w = WORKLOADS["pgdn_decode_256"].replace(T=16)
    x = make_inputs(w, device="cuda", generator_device="cuda")
    S = torch.zeros(w.B, w.H, w.dv, w.dk, device="cuda")
    A = torch.zeros(w.B, w.H, w.dk, device="cuda")
    o = decode_all(w, x, S, A, 16)
    xc = {n: (t.cpu() if t is not None else None) for n, t in x.items()}
    ro, rS, rA = run_oracle(w, xc)
    assert nmax_err(o.float().cpu().numpy(), ro) <= 2e-2
    assert nmax_err(S.cpu().numpy(), rS) <= 2e-2
    assert nmax_err(A.cpu().numpy(), rA) <= 1e-6


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_decode_d128_many_heads(variant, dtype):
    """d = 128 with more (batch, head) items than SMs, so the persistent
    streaming kernel cycles each CTA through its ring of state buffers."""
    w = Workload("dec128", variant, 40, 3, 8, 128, 128, dtype, DECAY[variant], q_scale=1.1)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(4)
    S0 = 0.2 * torch.randn(w.B, w.H, 128, 128, generator=g)
    A0 = torch.rand(w.B, w.H, 128, generator=g) if variant in ("PDN", "PGDN", "PKDA", "PLA") else None
    S = S0.cuda()
    A = A0.cuda() if A0 is not None else None
    o = decode_all(w, x, S, A, w.T)
    ro, rS, rA = run_oracle(w, x, S0, A0)
    tol = TOL[dtype]
    assert nmax_err(o.float().cpu().numpy(), ro) <= tol
    assert nmax_err(S.cpu().numpy(), rS) <= tol
    if A is not None:
        assert nmax_err(A.cpu().numpy(), rA) <= 1e-6


def test_decode_workload_full_1024_steps_sampled_chains():
    """The decode workload as configured: 256 sequences x 16 heads, d 128,
    fp32 state, one bf16 token per sequence per step for all 1024 steps. The
    outputs of every step and the final state of sampled (batch, head)
    chains are checked against the oracle over all 1024 tokens, so drift of
    the fp32 state over the whole run would show."""
    w = WORKLOADS["pgdn_decode_256"]
    steps = w.decode_steps
    x = make_inputs(w.replace(T=steps), device="cuda", generator_device="cuda")
    S = torch.zeros(w.B, w.H, w.dv, w.dk, device="cuda")
    A = torch.zeros(w.B, w.H, w.dk, device="cuda")
    o = decode_all(w, x, S, A, steps)
    for b, h in [(0, 0), (97, 5), (255, 15), (128, 9)]:
        xs = {n: (t[b:b + 1, :, h:h + 1].cpu() if t is not None else None) for n, t in x.items()}
        ro, rS, rA = run_oracle(w.replace(B=1, H=1, T=steps), xs)
        eo = nmax_err(o[b:b + 1, :, h:h + 1].float().cpu().numpy(), ro)
        es = nmax_err(S[b:b + 1, h:h + 1].cpu().numpy(), rS)
        ea = nmax_err(A[b:b + 1, h:h + 1].cpu().numpy(), rA)
        assert eo <= 2e-2 and es <= 2e-2 and ea <= 1e-5, (b, h, eo, es, ea)
