"""GPU parity of the backward: pdn_chunk_bwd through the C ABI against the
fp64 oracle's reverse-mode gradient of the token loop (itself pinned by
central finite differences), on the same seeded inputs and cotangents.

The CUDA backward runs in fp32 for both input dtypes (bf16 inputs are widened
exactly), so one bar holds for both: normalised max-abs error <= 2e-4 per
gradient tensor (the forward's fp32 bar 1e-4, doubled for the extra passes:
the decay gradient is a suffix sum over every later token)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import prologue as oracle_prologue
from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import (WORKLOADS, Workload, make_inputs,
                                                               make_raw_inputs, raw_prologue,
                                                               slice_chain)

from parity_util import REPORT, elem_rel_err, nmax_err

pytestmark = pytest.mark.gpu

TOL_BWD = 2e-4
VARIANTS = ["DN", "GDN", "KDA", "PDN", "PGDN", "PKDA", "FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"]
DECAY = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar",
         "KDA": "channel", "PKDA": "channel", "FG2_GDN": "channel", "GDN2": "channel",
         "PLA": "scalar", "FG2_GDN_PLUS": "channel"}
PRECOND = ("PDN", "PGDN", "PKDA", "PLA")


def small(variant, dtype, B=2, T=150, H=3, dk=64, dv=None, decay=None, seed=0, **kw):
    return Workload("bwd-%s-%s" % (variant, dtype), variant, B, T, H, dk, dk if dv is None else dv,
                    dtype, decay or DECAY[variant], seed=seed, **kw)


def states(w, seed=1, scale=0.3):
    g = torch.Generator().manual_seed(seed)
    S0 = scale * torch.randn(w.B, w.H, w.dv, w.dk, generator=g)
    A0 = torch.rand(w.B, w.H, w.dk, generator=g) * 2.0 if w.variant in PRECOND else None
    return S0, A0


def cotangents(w, seed=5):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dO = torch.randn(w.B, w.T, w.H, w.dv, generator=g).to(dt)
    dST = 0.5 * torch.randn(w.B, w.H, w.dv, w.dk, generator=g)
    return dO, dST


def run_gpu(w, x, S0, A0, dO, dST):
    dev = torch.device("cuda")
    d = {n: (t.to(dev) if t is not None else None) for n, t in x.items()}
    on = lambda t: None if t is None else t.to(dev)
    g = pdn.chunk_bwd(w.variant, d["q"], d["k"], d["v"], dO=on(dO), dST=on(dST),
                      log_alpha=d["log_alpha"], beta=d["beta"], erase=d["erase"], write=d["write"],
                      S0=on(S0), A0=on(A0), q_scale=w.q_scale, precond_x=w.precond_x,
                      precond_eps=w.precond_eps)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    return {n: (None if t is None else t.cpu().numpy()) for n, t in g.items()}


def run_oracle(w, x, S0, A0, dO, dST):
    return oracle.backward(w.variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"],
                           beta=x["beta"], erase=x["erase"], write=x["write"], S0=S0, A0=A0,
                           q_scale=w.q_scale, x=w.precond_x, eps=w.precond_eps, dO=dO, dST=dST)


def assert_grads(w, gg, gr, tol=TOL_BWD, label=""):
    bad = []
    for name, ref in gr.items():
        if ref is None:
            assert gg[name] is None, name
            continue
        e = nmax_err(gg[name], ref)
        REPORT.append(("%s%s:d%s" % (w.name, label, name), w.dtype, e, 0.0,
                       elem_rel_err(gg[name], ref), 0.0))
        if not e <= tol:
            bad.append((name, e))
    assert not bad, bad


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_backward_variants(variant, dtype):
    """Every variant: ragged T (two 64-token scan blocks and a tail), random
    S0 / A0 / dO / dS_T, q_scale != 1."""
    w = small(variant, dtype, q_scale=0.8)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    assert_grads(w, run_gpu(w, x, S0, A0, dO, dST), run_oracle(w, x, S0, A0, dO, dST))


@pytest.mark.parametrize("decay", ["none", "scalar", "channel"])
@pytest.mark.parametrize("variant", ["FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"])
def test_backward_free_decay(variant, decay):
    w = small(variant, "bf16", decay=decay, T=97)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    assert_grads(w, run_gpu(w, x, S0, A0, dO, dST), run_oracle(w, x, S0, A0, dO, dST))


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 129])
def test_backward_lengths(T):
    """Token counts around the 16-token staging chunks and the 64-token scan
    blocks; d = 32 leaves three quarters of each warp's lanes without a key
    channel."""
    w = small("PKDA", "f32", B=1, H=2, T=T, dk=32)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    assert_grads(w, run_gpu(w, x, S0, A0, dO, dST), run_oracle(w, x, S0, A0, dO, dST))


@pytest.mark.parametrize("dk,dv", [(128, 64), (48, 80), (128, 128), (16, 16)])
@pytest.mark.parametrize("variant", ["GDN2", "PGDN", "FG2_GDN_PLUS"])
def test_backward_head_dims(variant, dk, dv):
    w = small(variant, "bf16", B=1, H=2, T=70, dk=dk, dv=dv)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    assert_grads(w, run_gpu(w, x, S0, A0, dO, dST), run_oracle(w, x, S0, A0, dO, dST))


@pytest.mark.parametrize("which", ["dO", "dST", "both"])
def test_backward_absent_cotangents(which):
    """A NULL cotangent is zero: the loss reads only o, only S_T, or neither."""
    w = small("PKDA", "f32", T=40)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    if which in ("dO", "both"):
        dO = None
    if which in ("dST", "both"):
        dST = None
    gg = run_gpu(w, x, S0, A0, dO, dST)
    gr = run_oracle(w, x, S0, A0, dO, dST)
    if which == "both":
        for n, t in gg.items():
            if t is not None:
                assert np.abs(t).max() == 0.0, n
    else:
        assert_grads(w, gg, gr)


@pytest.mark.parametrize("variant", ["GDN", "KDA", "PKDA", "GDN2"])
def test_backward_strong_decay(variant):
    """Decays down to the per-token floor: the token-level backward never
    divides by a cumulative decay, so it stays exact at any strength."""
    w = small(variant, "f32", T=130, decay_recipe="strong", decay_mean=-20.0)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    assert_grads(w, run_gpu(w, x, S0, A0, dO, dST), run_oracle(w, x, S0, A0, dO, dST))


@pytest.mark.parametrize("name,chains", [("pgdn_bf16_4k", [(0, 0), (3, 15)]),
                                         ("pkda_bf16_8k", [(7, 15)]),
                                         ("gdn2_bf16_32k", [(1, 9)])])
def test_backward_full_size_sampled(name, chains):
    """Full-size workloads: the whole backward on the GPU, the oracle on
    sampled (batch, head) chains over all T tokens."""
    check_sampled_chains(WORKLOADS[name], chains)


@pytest.mark.parametrize("name,chains", [("pgdn_bf16_4k", [(3, 15)]),
                                         ("pkda_bf16_8k", [(7, 15)]),
                                         ("gdn2_bf16_32k", [(1, 9)])])
def test_backward_training_mode_full_size_sampled(name, chains):
    """The training mode at full size (GDN-2 32k through the time-segmented
    forward): sampled chains against the oracle over all T tokens."""
    check_sampled_chains(WORKLOADS[name], chains, training=True)


@pytest.mark.parametrize("variant,dk,dv,B", [("PKDA", 128, 128, 5), ("GDN2", 64, 64, 10),
                                            ("FG2_GDN_PLUS", 128, 128, 5), ("GDN2", 48, 80, 8),
                                            ("PGDN", 32, 32, 10), ("PGDN", 32, 32, 6),
                                            ("GDN2", 64, 32, 6)])
def test_backward_many_chains_ragged(variant, dk, dv, B):
    """Enough (batch, head) pairs for the row sweeps' unrolled chunk loop, in
    each layout the dispatch picks: 8 rows per warp with 4, 2 and 1 key
    channels per lane (B = 5, 10, 10 at d_k = 128, 64, 32) and 4 rows per
    warp with 1 and 2 (B = 6 at d_v = 32). The token count leaves a ragged
    last chunk of 3 tokens (and d_v = 80 a partial group of rows); sampled
    chains, the last one included."""
    w = small(variant, "bf16", B=B, T=203, H=16, dk=dk, dv=dv)
    check_sampled_chains(w, [(0, 0), (w.B // 2, 7), (w.B - 1, w.H - 1)])


def check_sampled_chains(w, chains, training=False):
    """The whole backward on the GPU, the oracle on the sampled chains; with
    `training`, the training mode (forward with saving, backward from the
    saved values) at the bf16 bar its saved values carry."""
    x = make_inputs(w, device="cuda")
    g = torch.Generator().manual_seed(11)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dO = torch.randn(w.B, w.T, w.H, w.dv, generator=g).to(dt)
    dST = 0.5 * torch.randn(w.B, w.H, w.dv, w.dk, generator=g)
    kw = dict(log_alpha=x["log_alpha"], beta=x["beta"], erase=x["erase"], write=x["write"],
              q_scale=w.q_scale, precond_x=w.precond_x, precond_eps=w.precond_eps)
    extra = {}
    if training:
        saved = {}
        _, ST, _ = pdn.chunk_fwd(w.variant, x["q"], x["k"], x["v"], saved=saved, **kw)
        extra = dict(saved=saved, ST=ST)
    gd = pdn.chunk_bwd(w.variant, x["q"], x["k"], x["v"], dO=dO.cuda(), dST=dST.cuda(), **kw,
                       **extra)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    for b, h in chains:
        xs = slice_chain(x, b, h)
        gr = oracle.backward(w.variant, xs["q"], xs["k"], xs["v"], log_alpha=xs["log_alpha"],
                             beta=xs["beta"], erase=xs["erase"], write=xs["write"],
                             q_scale=w.q_scale, x=w.precond_x, eps=w.precond_eps,
                             dO=dO[b:b + 1, :, h:h + 1], dST=dST[b:b + 1, h:h + 1])
        gs = {}
        for n, t in gd.items():
            if t is None:
                gs[n] = None
            elif n == "S0":
                gs[n] = t[b:b + 1, h:h + 1].cpu().numpy()
            elif n == "A0":
                gs[n] = t[b:b + 1, h:h + 1].cpu().numpy()
            else:
                gs[n] = t[b:b + 1, :, h:h + 1].cpu().numpy()
        if training:
            assert_grads(w, gs, gr, tol=2e-2, label="[saved,b%d,h%d]" % (b, h))
        else:
            assert_grads(w, gs, gr, label="[b%d,h%d]" % (b, h))


def test_backward_is_deterministic():
    """Fixed-order reductions throughout (no atomics): two runs agree bitwise."""
    w = small("PKDA", "bf16", T=150)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    a = run_gpu(w, x, S0, A0, dO, dST)
    b = run_gpu(w, x, S0, A0, dO, dST)
    for n in a:
        if a[n] is not None:
            assert np.array_equal(a[n], b[n]), n


@pytest.mark.parametrize("variant,recipe,dtype,dk", [("PGDN", "softplus", "bf16", 64),
                                                    ("GDN2", "sigmoid", "bf16", 64),
                                                    ("FG2_GDN_PLUS", "softplus", "f32", 32),
                                                    ("PKDA", "sigmoid", "f32", 32),
                                                    ("PLA", "softplus", "bf16", 32),
                                                    ("FG2_GDN", "sigmoid", "bf16", 32)])
def test_backward_prologue_finite_differences(variant, recipe, dtype, dk):
    """With the fused prologue (raw projections in: L2 normalisation of q and
    k, sigmoid gains and gates, softplus or log-sigmoid decay) the gradients
    are with respect to the raw inputs. Checked element by element against
    central differences of L = sum(dO . o) + sum(dST . S_T), with o and S_T
    from the fp64 oracle on the activated inputs, at sampled elements of every
    input tensor."""
    w = Workload("bwdpro-%s" % variant, variant, 1, 37, 2, dk, dk, dtype, DECAY[variant],
                 decay_recipe=recipe, seed=3)
    raw = make_raw_inputs(w)
    bits, dscale = raw_prologue(w)
    dO, dST = cotangents(w)
    dev = torch.device("cuda")
    d = {n: (t.to(dev) if t is not None else None) for n, t in raw.items()}
    g = pdn.chunk_bwd(w.variant, d["q"], d["k"], d["v"], dO=dO.to(dev), dST=dST.to(dev),
                      log_alpha=d["log_alpha"], beta=d["beta"], erase=d["erase"],
                      write=d["write"], q_scale=w.q_scale, precond_x=w.precond_x,
                      precond_eps=w.precond_eps, prologue=bits, decay_scale=dscale)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    base = {n: (t.double().numpy() if t is not None else None) for n, t in raw.items()}
    dO64, dST64 = dO.double().numpy(), dST.double().numpy()

    def loss(x):
        a = oracle_prologue.apply(x, bits, dscale)
        o, ST, _ = oracle.forward(w.variant, a["q"], a["k"], a["v"], log_alpha=a["log_alpha"],
                                  beta=a["beta"], erase=a["erase"], write=a["write"],
                                  q_scale=w.q_scale, x=w.precond_x, eps=w.precond_eps)
        return float((o * dO64).sum() + (ST * dST64).sum())

    rng = np.random.default_rng(1)
    bad = []
    for name in ("q", "k", "v", "log_alpha", "beta", "erase", "write"):
        if base[name] is None:
            assert g[name] is None, name
            continue
        G = g[name].cpu().numpy()
        gmax = float(np.abs(G).max())
        for _ in range(4):
            idx = tuple(int(rng.integers(0, n)) for n in base[name].shape)
            h = 1e-5 * max(1.0, abs(base[name][idx]))
            xp, xm = dict(base), dict(base)
            xp[name], xm[name] = base[name].copy(), base[name].copy()
            xp[name][idx] += h
            xm[name][idx] -= h
            fd = (loss(xp) - loss(xm)) / (2 * h)
            if not abs(G[idx] - fd) <= 2e-3 * gmax + 1e-6:
                bad.append((name, idx, float(G[idx]), fd, gmax))
    assert not bad, bad


@pytest.mark.parametrize("variant,T", [("PGDN", 200), ("GDN2", 130), ("PKDA", 257),
                                       ("FG2_GDN_PLUS", 64), ("PLA", 100)])
def test_backward_training_mode(variant, T):
    """Training mode: the tensor-core forward also leaves every token's delta
    and the chunk-start states (pdn_chunk_fwd_save) and the backward reuses
    them instead of its forward sweep (pdn_chunk_bwd_saved). Saving leaves
    the forward's outputs bitwise unchanged; the gradients, which carry the
    forward's bf16-operand rounding, meet the bf16 bar against the oracle."""
    w = small(variant, "bf16", B=2, T=T, H=2, dk=128)
    x = make_inputs(w)
    S0, A0 = states(w)
    dO, dST = cotangents(w)
    dev = torch.device("cuda")
    d = {n: (t.to(dev) if t is not None else None) for n, t in x.items()}
    kw = dict(log_alpha=d["log_alpha"], beta=d["beta"], erase=d["erase"], write=d["write"],
              S0=S0.to(dev), A0=None if A0 is None else A0.to(dev), q_scale=w.q_scale,
              precond_x=w.precond_x, precond_eps=w.precond_eps)
    o1, ST1, AT1 = pdn.chunk_fwd(w.variant, d["q"], d["k"], d["v"], **kw)
    saved = {}
    o2, ST2, AT2 = pdn.chunk_fwd(w.variant, d["q"], d["k"], d["v"], saved=saved, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(ST1, ST2)
    g = pdn.chunk_bwd(w.variant, d["q"], d["k"], d["v"], dO=dO.to(dev), dST=dST.to(dev),
                      saved=saved, ST=ST2, **kw)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    gg = {n: (None if t is None else t.cpu().numpy()) for n, t in g.items()}
    assert_grads(w, gg, run_oracle(w, x, S0, A0, dO, dST), tol=2e-2, label="[saved]")


@pytest.mark.parametrize("variant,recipe", [("PGDN", "softplus"), ("GDN2", "sigmoid"),
                                            ("PKDA", "sigmoid")])
def test_backward_training_mode_prologue(variant, recipe):
    """Training mode from raw projections (fused prologue in both directions):
    the saved deltas and states are those of the activated inputs, and the
    gradients with respect to the raw projections match the exact backward's
    (itself pinned by finite differences) within the bf16 bar."""
    w = Workload("trainpro-%s" % variant, variant, 2, 150, 2, 128, 128, "bf16", DECAY[variant],
                 decay_recipe=recipe, seed=11)
    raw = make_raw_inputs(w, device="cuda")
    bits, dscale = raw_prologue(w)
    dO, dST = cotangents(w)
    dO, dST = dO.cuda(), dST.cuda()
    kw = dict(log_alpha=raw["log_alpha"], beta=raw["beta"], erase=raw["erase"],
              write=raw["write"], q_scale=w.q_scale, precond_x=w.precond_x,
              precond_eps=w.precond_eps, prologue=bits, decay_scale=dscale)
    o1, ST1, _ = pdn.chunk_fwd(w.variant, raw["q"], raw["k"], raw["v"], **kw)
    saved = {}
    o2, ST2, _ = pdn.chunk_fwd(w.variant, raw["q"], raw["k"], raw["v"], saved=saved, **kw)
    gs = pdn.chunk_bwd(w.variant, raw["q"], raw["k"], raw["v"], dO=dO, dST=dST, saved=saved,
                       ST=ST2, **kw)
    ge = pdn.chunk_bwd(w.variant, raw["q"], raw["k"], raw["v"], dO=dO, dST=dST, **kw)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    assert torch.equal(o1, o2) and torch.equal(ST1, ST2)
    for n, t in ge.items():
        if t is not None:
            e = nmax_err(gs[n].cpu().numpy(), t.cpu().numpy())
            assert e <= 2e-2, (n, e)


def test_backward_training_mode_time_segments():
    """Training mode through the time-segmented forward (few chains, a long
    sequence): the reused deltas and states index the whole sequence; the
    gradients match the exact backward within the bf16 bar."""
    w = small("PGDN", "bf16", B=1, T=4096, H=16, dk=128)
    x = make_inputs(w, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(5)
    dO = torch.randn(w.B, w.T, w.H, w.dv, generator=gen, device="cuda").to(torch.bfloat16)
    dST = torch.randn(w.B, w.H, w.dv, w.dk, generator=gen, device="cuda")
    kw = dict(log_alpha=x["log_alpha"], beta=x["beta"], precond_x=w.precond_x,
              precond_eps=w.precond_eps)
    saved = {}
    _, ST, _ = pdn.chunk_fwd(w.variant, x["q"], x["k"], x["v"], saved=saved, **kw)
    gs = pdn.chunk_bwd(w.variant, x["q"], x["k"], x["v"], dO=dO, dST=dST, saved=saved, ST=ST, **kw)
    ge = pdn.chunk_bwd(w.variant, x["q"], x["k"], x["v"], dO=dO, dST=dST, **kw)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    for n, t in ge.items():
        if t is not None:
            e = nmax_err(gs[n].cpu().numpy(), t.cpu().numpy())
            assert e <= 2e-2, (n, e)
