"""GPU parity under strong decay. The pages bound the decay only to (0, 1)
(KDA's D_t = Diag(alpha_t), alpha_t in (0,1)^{d_k}, "Gated DeltaNet-2" ja §1;
the scalar gate of GDN likewise), so a chunk's cumulative decay can fall far
below anything fp32 represents. Mean per-token log decays of -1.5, -3 and -10
(e^-96 .. e^-640 over a 64-token chunk) and one key channel (or, for scalar
decay, every 7th token) at log alpha = -30 must all match the oracle at the
usual bars, on both chunk kernels and on decode."""
import pytest
import torch

from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import Workload, make_inputs

from parity_util import TOL, assert_parity, nmax_err, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

DECAY = {"GDN": "scalar", "PGDN": "scalar", "KDA": "channel", "PKDA": "channel",
         "FG2_GDN": "channel", "GDN2": "channel", "PLA": "channel", "FG2_GDN_PLUS": "channel"}
STRENGTHS = [-1.5, -3.0, -10.0, "hard"]


def strong(variant, mean, dtype="bf16", B=2, T=150, H=2, d=128, decay=None):
    decay = decay or DECAY[variant]
    if mean == "hard":
        return Workload("hard-%s" % variant, variant, B, T, H, d, d, dtype, decay,
                        hard_decay=True, q_scale=0.9)
    return Workload("strong%g-%s" % (mean, variant), variant, B, T, H, d, d, dtype, decay,
                    decay_recipe="strong", decay_mean=mean, q_scale=0.9)


def rand_state(w, seed=5):
    g = torch.Generator().manual_seed(seed)
    S0 = 0.3 * torch.randn(w.B, w.H, w.dv, w.dk, generator=g)
    A0 = torch.rand(w.B, w.H, w.dk, generator=g) if w.variant in ("PDN", "PGDN", "PKDA", "PLA") else None
    return S0, A0


@pytest.mark.parametrize("mean", STRENGTHS)
@pytest.mark.parametrize("variant", list(DECAY))
def test_strong_decay_tensor_core_path(variant, mean):
    w = strong(variant, mean)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    assert pdn.pdn_chunk_fwd_impl(pdn.make_problem(w.variant, w.B, w.T, w.H, 128, 128, torch.bfloat16,
                                                   w.decay)) == pdn.IMPLS["tc"]
    o, ST, AT = run_gpu(w, x, S0, A0, impl="tc")
    assert torch.isfinite(o.float()).all() and torch.isfinite(ST).all()
    assert_parity(w, o, ST, AT, *run_oracle(w, x, S0, A0))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mean", STRENGTHS)
@pytest.mark.parametrize("variant", list(DECAY))
def test_strong_decay_cuda_core_path(variant, mean, dtype):
    w = strong(variant, mean, dtype=dtype, d=64)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    o, ST, AT = run_gpu(w, x, S0, A0, impl="simt")
    assert torch.isfinite(o.float()).all() and torch.isfinite(ST).all()
    assert_parity(w, o, ST, AT, *run_oracle(w, x, S0, A0))


@pytest.mark.parametrize("decay", ["scalar", "channel"])
@pytest.mark.parametrize("variant", ["FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"])
def test_strong_decay_free_decay_variants(variant, decay):
    w = strong(variant, -3.0, decay=decay, T=200)
    x = make_inputs(w)
    o, ST, AT = run_gpu(w, x, impl="tc")
    assert_parity(w, o, ST, AT, *run_oracle(w, x))


def test_strong_decay_mixed_with_mild_chunks():
    """Strong decay in some chunks and mild decay in others, in one sequence:
    the flagged sub-chunks take the exact pairwise sums, the rest the
    factorised products, and the state passes between them."""
    w = strong("PKDA", -10.0, T=320, B=2, H=3)
    x = make_inputs(w)
    mild = make_inputs(w.replace(decay_recipe="softplus"))
    la = x["log_alpha"].clone()
    la[:, 64:192] = mild["log_alpha"][:, 64:192]  # chunks 1 and 2 mild
    la[:, 200:210] = -40.0                         # a burst inside chunk 3
    x["log_alpha"] = la
    o, ST, AT = run_gpu(w, x, impl="tc")
    assert_parity(w, o, ST, AT, *run_oracle(w, x))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mean", STRENGTHS)
@pytest.mark.parametrize("variant", list(DECAY))
def test_strong_decay_decode(variant, mean, dtype):
    w = strong(variant, mean, dtype=dtype, B=3, T=12, H=2)
    x = make_inputs(w)
    S0, A0 = rand_state(w)
    S = S0.cuda()
    A = A0.cuda() if A0 is not None else None
    dev = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
    outs = []
    for t in range(w.T):
        sl = {n: (v[:, t:t + 1].contiguous() if v is not None else None) for n, v in dev.items()}
        outs.append(pdn.decode_step(w.variant, sl["q"], sl["k"], sl["v"], S, A,
                                    log_alpha=sl["log_alpha"], beta=sl["beta"], erase=sl["erase"],
                                    write=sl["write"], q_scale=w.q_scale))
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    o = torch.cat(outs, dim=1)
    ro, rS, rA = run_oracle(w, x, S0, A0)
    assert nmax_err(o.float().cpu().numpy(), ro) <= TOL[dtype]
    assert nmax_err(S.cpu().numpy(), rS) <= TOL[dtype]
