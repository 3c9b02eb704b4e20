"""GPU parity: the CUDA chunked forward (through the C ABI) against the fp64
oracle, element by element, on the same seeded inputs."""
import numpy as np
import pytest
import torch

from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import WORKLOADS, Workload, make_inputs

from parity_util import TOL, assert_parity, run_gpu, run_oracle, nmax_err

pytestmark = pytest.mark.gpu

VARIANTS = ["DN", "GDN", "KDA", "PDN", "PGDN", "PKDA", "FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"]
DECAY = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar",
         "KDA": "channel", "PKDA": "channel", "FG2_GDN": "channel", "GDN2": "channel",
         "PLA": "scalar", "FG2_GDN_PLUS": "channel"}
IMPLS = ["simt", "auto"]


def small(variant, dtype, B=2, T=150, H=3, d=64, dv=None, decay=None, seed=0, **kw):
    return Workload("small-%s-%s" % (variant, dtype), variant, B, T, H, d, d if dv is None else dv,
                    dtype, decay or DECAY[variant], seed=seed, **kw)


def rand_state(w, seed=1, scale=0.3):
    g = torch.Generator().manual_seed(seed)
    S0 = scale * torch.randn(w.B, w.H, w.dv, w.dk, generator=g)
    A0 = torch.rand(w.B, w.H, w.dk, generator=g) * 2.0 if w.variant in ("PDN", "PGDN", "PKDA", "PLA") else None
    return S0, A0


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_variants_small(variant, dtype, impl):
    """Every variant, ragged T (2 full chunks + a tail), random S0/A0, q_scale != 1."""
    w = small(variant, dtype, q_scale=0.8)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    o, ST, AT = run_gpu(w, x, S0, A0, impl=impl)
    ro, rS, rA = run_oracle(w, x, S0, A0)
    assert_parity(w, o, ST, AT, ro, rS, rA)


@pytest.mark.parametrize("decay", ["none", "scalar", "channel"])
@pytest.mark.parametrize("variant", ["FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"])
def test_free_decay_variants(variant, decay):
    w = small(variant, "bf16", decay=decay, T=97)
    x = make_inputs(w)
    o, ST, AT = run_gpu(w, x)
    assert_parity(w, o, ST, AT, *run_oracle(w, x))


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 128, 200])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_lengths_and_chunks(T, chunk):
    w = small("PKDA", "f32", B=1, H=2, T=T, d=32, chunk=chunk)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    o, ST, AT = run_gpu(w, x, S0, A0, impl="simt")
    assert_parity(w, o, ST, AT, *run_oracle(w, x, S0, A0))


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 48), (48, 128)])
def test_head_dims(dk, dv):
    w = small("PGDN", "f32", B=1, H=2, T=80, d=dk, dv=dv)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    o, ST, AT = run_gpu(w, x, S0, A0)
    assert_parity(w, o, ST, AT, *run_oracle(w, x, S0, A0))


def test_pdn_fp32_workload_full():
    """The fp32 Preconditioned DeltaNet workload (B1 H2 T512 d64, chunk 64),
    every output checked at 1e-4."""
    w = WORKLOADS["pdn_f32_small"]
    x = make_inputs(w)
    o, ST, AT = run_gpu(w, x)
    assert_parity(w, o, ST, AT, *run_oracle(w, x), tol=1e-4)


def test_empty_sequence_returns_initial_state():
    w = small("PGDN", "bf16", T=0)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    o, ST, AT = run_gpu(w, x, S0, A0)
    assert o.numel() == 0
    torch.testing.assert_close(ST.cpu(), S0, rtol=0, atol=0)
    torch.testing.assert_close(AT.cpu(), A0, rtol=0, atol=0)


@pytest.mark.parametrize("variant", ["PGDN", "PKDA", "GDN2"])
def test_continuation_matches_single_pass(variant):
    """fwd(T1) then fwd(T2 | S_T1, A_T1) equals fwd(T1 + T2), T1 not a
    multiple of the chunk (the split moves every chunk boundary)."""
    w = small(variant, "f32", B=2, H=2, T=300, d=64)
    x = make_inputs(w)
    o, ST, AT = run_gpu(w, x)
    x1 = {n: (t[:, :137] if t is not None else None) for n, t in x.items()}
    x2 = {n: (t[:, 137:] if t is not None else None) for n, t in x.items()}
    o1, S1, A1 = run_gpu(w.replace(T=137), x1)
    o2, S2, A2 = run_gpu(w.replace(T=163), x2, S1.cpu(), None if A1 is None else A1.cpu())
    oc = torch.cat([o1, o2], dim=1)
    assert nmax_err(oc.cpu().numpy(), o.cpu().numpy()) < 1e-5
    assert nmax_err(S2.cpu().numpy(), ST.cpu().numpy()) < 1e-5


def test_deterministic():
    w = small("PKDA", "bf16", B=2, H=4, T=300, d=128)
    x = make_inputs(w)
    a = run_gpu(w, x)
    b = run_gpu(w, x)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bounded_wait_reports_timeout():
    """A device wait that nothing completes gives up after its poll limit and
    reports PDN_ERR_TIMEOUT; the context stays usable afterwards."""
    s = torch.cuda.current_stream().cuda_stream
    assert pdn.pdn_get_device_error(s) == pdn.PDN_OK
    assert pdn.pdn_selftest_bounded_wait(1000, s) == pdn.PDN_OK
    assert pdn.pdn_get_device_error(s) == pdn.PDN_ERR_TIMEOUT
    assert pdn.pdn_get_device_error(s) == pdn.PDN_OK  # cleared
    w = small("GDN", "f32", T=40)
    x = make_inputs(w)
    o, ST, AT = run_gpu(w, x)
    assert_parity(w, o, ST, AT, *run_oracle(w, x))


def test_misaligned_device_pointer_rejected():
    w = small("GDN", "bf16", T=8)
    x = {n: (t.cuda() if t is not None else None) for n, t in make_inputs(w).items()}
    buf = torch.empty(x["q"].numel() + 8, dtype=torch.bfloat16, device="cuda")
    q_bad = buf[1:1 + x["q"].numel()].view_as(x["q"])
    with pytest.raises(pdn.PdnError) as e:
        pdn.chunk_fwd("GDN", q_bad, x["k"], x["v"], log_alpha=x["log_alpha"], beta=x["beta"])
    assert e.value.code == pdn.PDN_ERR_INVALID_ARG
