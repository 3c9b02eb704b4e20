"""GPU checks of the sequence-parallel prefill pieces through the C ABI
(segment transition, key energy, accumulator sum, state composition) against
their definitions, and of the whole protocol with several segments run in one
process against one token loop over the sequence (ranks that wait on each
other are not run as separate processes on one GPU)."""
import numpy as np
import pytest
import torch

import oracle
from linear_recurrence_sequence_chunked_b200 import pdn, seqpar
from linear_recurrence_sequence_chunked_b200.workloads import (Workload, make_inputs,
                                                               make_raw_inputs, raw_prologue)

from parity_util import TOL, nmax_err
from seqpar_oracle_ops import OracleOps

pytestmark = pytest.mark.gpu

CASES = [("PGDN", "scalar"), ("PKDA", "channel"), ("GDN2", "channel"), ("FG2_GDN_PLUS", "channel"),
         ("PLA", "scalar"), ("KDA", "channel"), ("DN", "none")]


def cuda(x):
    return {n: (t.cuda() if t is not None else None) for n, t in x.items()}


@pytest.mark.parametrize("impl,dtype,d", [("tc", "bf16", 128), ("simt", "f32", 64)])
@pytest.mark.parametrize("variant,decay", CASES)
def test_transition_matches_product_of_steps(variant, decay, impl, dtype, d):
    """A_seg = prod_t Diag(alpha_t)(I - r_t w_t^T): the oracle's token loop with
    zero targets from the identity state."""
    w = Workload("tr", variant, 2, 150, 2, d, d, dtype, decay, seed=4)
    x = make_inputs(w)
    A0 = torch.rand(2, 2, d) if variant in pdn.PRECOND_VARIANTS else None
    ops = seqpar.CudaOps(variant, decay, impl=impl)
    A = ops.transition(cuda(x), None if A0 is None else A0.cuda())
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    ref = OracleOps(variant).transition(x, None if A0 is None else A0.double().numpy())
    assert nmax_err(A.cpu().numpy(), ref.numpy()) <= TOL[dtype]


@pytest.mark.parametrize("prologue", [0, pdn.PRO_L2NORM_QK])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_key_energy(dtype, prologue):
    w = Workload("ke", "PGDN", 3, 333, 4, 128, 128, dtype, "scalar", seed=5)
    x = make_raw_inputs(w) if prologue else make_inputs(w)
    A0 = torch.rand(3, 4, 128)
    ops = seqpar.CudaOps("PGDN", "scalar", prologue=prologue)
    k = x["k"].double().numpy()
    if prologue:
        k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    E = ops.key_energy(cuda(x))
    torch.cuda.synchronize()
    np.testing.assert_allclose(E.cpu().numpy(), np.sum(k * k, axis=1), rtol=2e-5, atol=1e-5)
    # with a start value: AT = A0 + sum
    t = pdn.make_tensors(None, cuda(x)["k"], None, None, A0=A0.cuda(), AT=E)
    assert pdn.pdn_key_energy(ops._problem(x), t, torch.cuda.current_stream().cuda_stream) == pdn.PDN_OK
    torch.cuda.synchronize()
    np.testing.assert_allclose(E.cpu().numpy(), A0.numpy() + np.sum(k * k, axis=1), rtol=2e-5, atol=1e-5)


@pytest.mark.parametrize("dv,dk", [(128, 128), (64, 128), (128, 48), (16, 16)])
def test_state_compose_and_accumulate(dv, dk):
    g = torch.Generator(device="cuda").manual_seed(6)
    S = torch.randn(3, 5, dv, dk, device="cuda", generator=g)
    A = torch.randn(3, 5, dk, dk, device="cuda", generator=g) / dk ** 0.5
    Bm = torch.randn(3, 5, dv, dk, device="cuda", generator=g)
    ops = seqpar.CudaOps("PGDN", "scalar")
    out = ops.compose(S, A, Bm)
    out0 = ops.compose(None, A, Bm)
    torch.cuda.synchronize()
    ref = torch.matmul(S.double(), A.double()) + Bm.double()
    assert (out.double() - ref).abs().max().item() < 1e-4
    assert torch.equal(out0, Bm)
    parts = torch.randn(4, 3, 5, dk, device="cuda", generator=g)
    base = torch.randn(3, 5, dk, device="cuda", generator=g)
    for n in range(5):
        acc = ops.accumulate(parts, n, base)
        torch.cuda.synchronize()
        ref = base.double() + parts[:n].double().sum(0)
        assert (acc.double() - ref).abs().max().item() < 1e-5


@pytest.mark.parametrize("segments", [2, 4])
@pytest.mark.parametrize("variant,decay", CASES)
def test_sequence_parallel_matches_one_pass(variant, decay, segments):
    """The protocol with ``segments`` segments in one process on the tensor-core
    path (bf16, d = 128, T = 700, segment bounds off the chunk grid) against the
    oracle over the whole sequence, and the final state against one
    pdn_chunk_fwd over the whole sequence."""
    w = Workload("sp-%s" % variant, variant, 2, 700, 2, 128, 128, "bf16", decay, seed=7)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(8)
    S0 = 0.3 * torch.randn(2, 2, 128, 128, generator=g)
    A0 = torch.rand(2, 2, 128, generator=g) if variant in pdn.PRECOND_VARIANTS else None
    bounds = [0] + [int(w.T * (i + 1) / segments) + 13 * (i % 2) for i in range(segments - 1)] + [w.T]
    ops = seqpar.CudaOps(variant, decay, impl="tc")
    xd = cuda(x)
    segs = [seqpar.SegmentPrefill(ops, {n: (t[:, bounds[i]:bounds[i + 1]].contiguous()
                                            if t is not None else None) for n, t in xd.items()}, i)
            for i in range(segments)]
    energies = torch.stack([s.energy() for s in segs]) if ops.precond else None
    A0d = None if A0 is None else A0.cuda()
    loc = [s.local(energies, A0d) for s in segs]
    A_all = torch.stack([a for a, _ in loc])
    B_all = torch.stack([b for _, b in loc])
    res = [s.finish(A_all, B_all, S0.cuda()) for s in segs]
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    o = torch.cat([r[0] for r in res], dim=1)
    ro, rS, rA = oracle.forward(variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"],
                                beta=x["beta"], erase=x["erase"], write=x["write"], S0=S0, A0=A0)
    assert nmax_err(o.float().cpu().numpy(), ro) <= 2e-2
    assert nmax_err(res[-1][1].cpu().numpy(), rS) <= 2e-2
    if A0 is not None:
        assert nmax_err(res[-1][2].cpu().numpy(), rA) <= 1e-5
