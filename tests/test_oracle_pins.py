"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a closed form, a brute-force expansion, the recursive least-squares
identity, or an invariant the pages state -- so that a dropped term, a wrong
sign or index, or transposed read/write keys fails at least one of them.

Sources: "Preconditioned DeltaNet" (gist.science, ja/de/fr), "Gated
DeltaNet-2" (ja), "FG2-GDN" (ja). Section names are given per test.
"""
import numpy as np
import pytest

import oracle
from oracle import chunked
from oracle import prologue

VARIANTS = ["DN", "GDN", "KDA", "PDN", "PGDN", "PKDA", "FG2_GDN", "GDN2", "PLA", "FG2_GDN_PLUS"]
DECAY = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar",
         "KDA": "channel", "PKDA": "channel", "FG2_GDN": "channel", "GDN2": "channel",
         "PLA": "channel", "FG2_GDN_PLUS": "channel"}


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_inputs(variant, B=2, T=9, H=2, dk=8, dv=8, seed=0, decay=None, S0=True):
    rng = np.random.default_rng(seed)
    decay = DECAY[variant] if decay is None else decay
    d = dict(q=unit(rng.standard_normal((B, T, H, dk))),
             k=unit(rng.standard_normal((B, T, H, dk))),
             v=rng.standard_normal((B, T, H, dv)))
    if variant in ("FG2_GDN", "FG2_GDN_PLUS"):
        d["beta"] = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))
    elif variant != "GDN2":
        d["beta"] = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    if decay == "scalar":
        d["log_alpha"] = -0.3 * np.abs(rng.standard_normal((B, T, H)))
    elif decay == "channel":
        d["log_alpha"] = -0.3 * np.abs(rng.standard_normal((B, T, H, dk)))
    if variant == "GDN2":
        d["erase"] = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))
        d["write"] = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dv))))
    if variant == "FG2_GDN_PLUS":
        d["write"] = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dv))))
    if S0:
        d["S0"] = 0.5 * rng.standard_normal((B, H, dv, dk))
    return d


def decay_cum(log_alpha, shape_bthk):
    """Cumulative decay multipliers prod_{s<=t} alpha_s, [B,T,H,dk]."""
    B, T, H, dk = shape_bthk
    if log_alpha is None:
        return np.ones((B, T, H, dk))
    la = log_alpha if log_alpha.ndim == 4 else np.repeat(log_alpha[..., None], dk, axis=3)
    return np.exp(np.cumsum(la, axis=1))


# ---------------------------------------------------------------- P1
@pytest.mark.parametrize("variant", VARIANTS)
def test_p1_zero_gain_leaves_only_decay(variant):
    """beta = 0 (GDN-2: erase = write = 0) removes the delta step, so
    S_t = S_0 Diag(prod alpha) and o_t = S_0 Diag(prod alpha) q_t: decay and
    state orientation ("Gated DeltaNet-2" ja §1, decay D_t = Diag(alpha_t))."""
    d = rand_inputs(variant, seed=1)
    for n in ("beta", "erase", "write"):
        if n in d:
            d[n] = np.zeros_like(d[n])
    # (PLA reads out through the preconditioned query B_t . q: x = 1 makes B = 1)
    o, ST, _ = oracle.forward(variant, **d, q_scale=0.7, x=1.0 if variant == "PLA" else 1.5)
    cum = decay_cum(d.get("log_alpha"), d["k"].shape)
    B, T, H, _ = d["k"].shape
    for b in range(B):
        for h in range(H):
            for t in range(T):
                St = d["S0"][b, h] * cum[b, t, h][None, :]
                np.testing.assert_allclose(o[b, t, h], 0.7 * St @ d["q"][b, t, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(ST[b, h], d["S0"][b, h] * cum[b, T - 1, h][None, :], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- P2
@pytest.mark.parametrize("pv,base", [("PDN", "DN"), ("PGDN", "GDN"), ("PKDA", "KDA")])
def test_p2_identity_preconditioner_reduces_to_base(pv, base):
    """x = 1 confines B_t to [1, 1], i.e. P = I, and the preconditioned variant
    is its base variant exactly ("Preconditioned DeltaNet" fr §2.C)."""
    d = rand_inputs(pv, seed=2)
    o1, S1, _ = oracle.forward(pv, **d, x=1.0)
    o2, S2, _ = oracle.forward(base, **d)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


# ---------------------------------------------------------------- P3
@pytest.mark.parametrize("decay,base", [("scalar", "GDN"), ("channel", "KDA")])
def test_p3_fg2_equal_beta_vector_is_gdn(decay, base):
    """An all-equal per-channel beta vector c makes FG2-GDN's sqrt(beta) on k
    and v equal to a scalar gain c ("FG2-GDN" ja §2.1)."""
    d = rand_inputs("FG2_GDN", seed=3, decay=decay)
    c = d["beta"][..., 0]
    d["beta"] = np.repeat(c[..., None], d["k"].shape[3], axis=3)
    o1, S1, _ = oracle.forward("FG2_GDN", **d)
    d["beta"] = c
    o2, S2, _ = oracle.forward(base, **d)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- P4
@pytest.mark.parametrize("decay,base", [("scalar", "GDN"), ("channel", "KDA")])
def test_p4_gdn2_tied_gates_reduce(decay, base):
    """Erase and write gates tied to one scalar beta give KDA, and with a
    scalar decay Gated DeltaNet ("Gated DeltaNet-2" ja §1, last paragraph)."""
    d = rand_inputs("GDN2", seed=4, decay=decay)
    rng = np.random.default_rng(44)
    B, T, H, dk = d["k"].shape
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    d["erase"] = np.repeat(beta[..., None], dk, axis=3)
    d["write"] = np.repeat(beta[..., None], d["v"].shape[3], axis=3)
    o1, S1, _ = oracle.forward("GDN2", **d)
    d2 = {n: d[n] for n in ("q", "k", "v", "log_alpha", "S0")}
    o2, S2, _ = oracle.forward(base, **d2, beta=beta)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- P5
@pytest.mark.parametrize("variant", ["DN", "GDN", "KDA", "FG2_GDN", "GDN2"])
def test_p5_delta_rule_writes_exactly(variant):
    """With unit-norm keys and a full gain (beta = 1, erase gate 1), one delta
    step makes the state map the read key to its target exactly,
    S_t k_t = u_t, whatever the decay: the exact-recall property of the delta
    rule viewed as online least squares ("Preconditioned DeltaNet" ja §1).
    Reading with q = k therefore returns u_t at every step."""
    d = rand_inputs(variant, seed=5)
    d["q"] = d["k"].copy()
    for n in ("beta", "erase"):
        if n in d:
            d[n] = np.ones_like(d[n])
    o, _, _ = oracle.forward(variant, **d)
    target = d["v"] * (d["write"] if variant == "GDN2" else 1.0)
    np.testing.assert_allclose(o, target, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("variant", ["PDN", "PGDN", "PKDA"])
def test_p5_preconditioned_write_key_normalised(variant):
    """For the preconditioned variants w_t = beta_t (B_t . k_t) and the read
    key is k_t (apply-to-key: "Preconditioned DeltaNet" de §2, read/write key).
    Choosing beta_t = 1 / sum_i B_ti k_ti^2 makes w_t.k_t = 1, so
    S_t k_t = v_t exactly. A swap of read and write keys would fail this."""
    d = rand_inputs(variant, seed=6)
    B, T, H, dk = d["k"].shape
    beta = np.zeros((B, T, H))
    for b in range(B):
        for h in range(H):
            Bc, _ = oracle.precond(d["k"][b, :, h], x=1.5)
            beta[b, :, h] = 1.0 / np.sum(Bc * d["k"][b, :, h] ** 2, axis=1)
    d["beta"] = beta
    d["q"] = d["k"].copy()
    o, _, _ = oracle.forward(variant, **d, x=1.5)
    np.testing.assert_allclose(o, d["v"], rtol=1e-11, atol=1e-12)


def test_p5_generic_any_normalised_pair():
    """Generic step: whenever w_t.r_t = 1, S_t r_t = u_t."""
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 1, 12, 2, 6, 5
    r = rng.standard_normal((B, T, H, dk))
    w = rng.standard_normal((B, T, H, dk))
    w = w / np.sum(w * r, axis=3, keepdims=True)
    u = rng.standard_normal((B, T, H, dv))
    la = -0.2 * np.abs(rng.standard_normal((B, T, H, dk)))
    o, _ = oracle.generic(r, r, w, u, log_alpha=la, S0=rng.standard_normal((B, H, dv, dk)))
    np.testing.assert_allclose(o, u, rtol=1e-10, atol=1e-11)


# ---------------------------------------------------------------- P6
def variant_vectors(variant, d, b, t, h, Bc=None):
    k, v = d["k"][b, t, h], d["v"][b, t, h]
    if variant in ("DN", "GDN", "KDA"):
        return k, d["beta"][b, t, h] * k, v
    if variant in ("PDN", "PGDN", "PKDA"):
        return k, d["beta"][b, t, h] * Bc[t] * k, v
    if variant == "FG2_GDN":
        sb = np.sqrt(d["beta"][b, t, h])
        return sb * k, sb * k, sb * v
    if variant == "PLA":
        return np.zeros_like(k), d["beta"][b, t, h] * k, v
    if variant == "FG2_GDN_PLUS":
        sk = np.sqrt(d["beta"][b, t, h])
        return sk * k, sk * k, np.sqrt(d["write"][b, t, h]) * v
    return d["erase"][b, t, h] * k, k, d["write"][b, t, h] * v


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("T", [1, 2, 3])
def test_p6_brute_force_product_expansion(variant, T):
    """For T <= 3 the state is the explicit sum of products
    S_T = S_0 prod_s D_s (I - r_s w_s^T) + sum_t u_t w_t^T prod_{s>t} D_s (I - r_s w_s^T),
    formed with d_k x d_k matrices (the generic update written out)."""
    d = rand_inputs(variant, B=1, T=T, H=1, dk=5, dv=5 if variant == "FG2_GDN" else 4, seed=10 + T)
    o, ST, AT = oracle.forward(variant, **d, q_scale=1.3)
    dk = 5
    Bc = None
    if variant in ("PDN", "PGDN", "PKDA", "PLA"):
        Bc, _ = oracle.precond(d["k"][0, :, 0], x=1.5)
    la = d.get("log_alpha")
    mats, outer = [], []
    for t in range(T):
        r, w, u = variant_vectors(variant, d, 0, t, 0, Bc)
        if la is None:
            Dm = np.eye(dk)
        elif la.ndim == 3:
            Dm = np.exp(la[0, t, 0]) * np.eye(dk)
        else:
            Dm = np.diag(np.exp(la[0, t, 0]))
        mats.append(Dm @ (np.eye(dk) - np.outer(r, w)))
        outer.append(np.outer(u, w))
    for tt in range(1, T + 1):
        S = d["S0"][0, 0].copy()
        for s in range(tt):
            S = S @ mats[s]
        for t in range(tt):
            term = outer[t]
            for s in range(t + 1, tt):
                term = term @ mats[s]
            S = S + term
        qt = d["q"][0, tt - 1, 0] * (Bc[tt - 1] if variant == "PLA" else 1.0)
        np.testing.assert_allclose(o[0, tt - 1, 0], 1.3 * S @ qt, rtol=1e-12, atol=1e-12)
        if tt == T:
            np.testing.assert_allclose(ST[0, 0], S, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- PLA and FG2-GDN+
@pytest.mark.parametrize("decay", ["none", "scalar", "channel"])
def test_pla_identity_preconditioner_is_decayed_linear_attention(decay):
    """PLA with x = 1 (B_t = 1) is linear attention with the gain and the
    decay axes: no erase, so
    o_t = q_scale (S_0 Diag(prod_{s<=t} alpha_s) + sum_{s<=t} beta_s v_s (k_s . prod_{s<tau<=t} alpha_tau)^T) q_t,
    written out as the explicit sum ("Preconditioned DeltaNet" ja §2.1:
    linear attention; fr §2.D: decay and gain axes)."""
    d = rand_inputs("PLA", seed=31, decay=decay, T=10)
    o, ST, _ = oracle.forward("PLA", **d, x=1.0, q_scale=0.8)
    B, T, H, dk = d["k"].shape
    la = d.get("log_alpha")
    for b in range(B):
        for h in range(H):
            if la is None:
                lac = np.zeros((T, dk))
            elif la.ndim == 3:
                lac = np.repeat(la[b, :, h][:, None], dk, axis=1)
            else:
                lac = la[b, :, h]
            for t in range(T):
                S = d["S0"][b, h] * np.exp(lac[: t + 1].sum(axis=0))[None, :]
                for s in range(t + 1):
                    g = np.exp(lac[s + 1: t + 1].sum(axis=0))
                    S = S + d["beta"][b, s, h] * np.outer(d["v"][b, s, h], d["k"][b, s, h] * g)
                np.testing.assert_allclose(o[b, t, h], 0.8 * S @ d["q"][b, t, h], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(ST[b, h], S, rtol=1e-11, atol=1e-12)


def test_pla_preconditions_the_query_only():
    """Apply-to-query ("Preconditioned DeltaNet" fr §2.A): the preconditioner
    touches only the read-out, so PLA's state is the same for every x, and its
    output is the x = 1 output read with the query B_t . q_t; the accumulator
    A is the running sum of k . k either way."""
    d = rand_inputs("PLA", seed=32, T=12)
    o15, S15, A15 = oracle.forward("PLA", **d, x=1.5)
    o1, S1, A1 = oracle.forward("PLA", **d, x=1.0)
    np.testing.assert_array_equal(S15, S1)
    B, T, H, dk = d["k"].shape
    qB = d["q"].copy()
    for b in range(B):
        for h in range(H):
            Bc, _ = oracle.precond(d["k"][b, :, h], x=1.5)
            qB[b, :, h] *= Bc
    oq, _, _ = oracle.forward("PLA", **dict(d, q=qB), x=1.0)
    np.testing.assert_allclose(o15, oq, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(A15, np.sum(d["k"] ** 2, axis=1), rtol=1e-13)


@pytest.mark.parametrize("decay", ["scalar", "channel"])
def test_fg2_plus_reductions(decay):
    """FG2-GDN+ ("FG2-GDN" ja §2.2: separate key-side and value-side gain
    vectors): beta^v = beta^k is FG2-GDN exactly; beta^k = 1 is the delta rule
    with unit gain on the values sqrt(beta^v) . v (KDA, or GDN for scalar
    decay); beta^v = 0 with S_0 = 0 writes nothing."""
    d = rand_inputs("FG2_GDN_PLUS", seed=33, decay=decay)
    d["write"] = d["beta"].copy()
    o1, S1, _ = oracle.forward("FG2_GDN_PLUS", **d)
    o2, S2, _ = oracle.forward("FG2_GDN", **{n: a for n, a in d.items() if n != "write"})
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    d = rand_inputs("FG2_GDN_PLUS", seed=34, decay=decay)
    d["beta"] = np.ones_like(d["beta"])
    o3, S3, _ = oracle.forward("FG2_GDN_PLUS", **d)
    base = {n: d[n] for n in ("q", "k", "log_alpha", "S0")}
    base["v"] = np.sqrt(d["write"]) * d["v"]
    base["beta"] = np.ones(d["k"].shape[:3])
    o4, S4, _ = oracle.forward("GDN" if decay == "scalar" else "KDA", **base)
    np.testing.assert_allclose(o3, o4, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S3, S4, rtol=1e-12, atol=1e-13)
    d = rand_inputs("FG2_GDN_PLUS", seed=35, decay=decay, S0=False)
    d["write"] = np.zeros_like(d["write"])
    o5, S5, _ = oracle.forward("FG2_GDN_PLUS", **d)
    assert not o5.any() and not S5.any()


# ---------------------------------------------------------------- fused prologue
def test_prologue_maps_closed_forms_and_references():
    """The prologue's maps against closed forms and scipy's reference
    implementations: sigmoid(0) = 1/2, softplus(0) = log 2, log sigmoid(x) =
    -softplus(-x), sigmoid(x) + sigmoid(-x) = 1; unit norms after L2
    normalisation, direction kept, zero vectors stay zero."""
    from scipy.special import expit, log_expit
    x = np.linspace(-60, 60, 241)
    np.testing.assert_allclose(prologue.sigmoid(x), expit(x), rtol=1e-15, atol=0)
    np.testing.assert_allclose(-prologue.softplus(-x), log_expit(x), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(prologue.sigmoid(x) + prologue.sigmoid(-x), 1.0, rtol=0, atol=1e-15)
    assert prologue.sigmoid(np.array([0.0]))[0] == 0.5
    assert prologue.softplus(np.array([0.0]))[0] == np.log(2.0)
    np.testing.assert_allclose(prologue.softplus(np.array([30.0, -30.0])),
                               [30.0 + np.exp(-30.0), np.exp(-30.0)], rtol=1e-12)
    rng = np.random.default_rng(40)
    v = rng.standard_normal((5, 7, 16)) * 3.0
    n = prologue.l2_normalise(v)
    np.testing.assert_allclose(np.linalg.norm(n, axis=-1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(n * np.linalg.norm(v, axis=-1, keepdims=True), v, rtol=1e-14)
    assert not prologue.l2_normalise(np.zeros((2, 4))).any()


def test_prologue_apply_selects_by_bits():
    """Each bit touches only its tensors; the decay bits map log_alpha."""
    rng = np.random.default_rng(41)
    raw = dict(q=rng.standard_normal((1, 3, 2, 4)), k=rng.standard_normal((1, 3, 2, 4)),
               v=rng.standard_normal((1, 3, 2, 4)), log_alpha=rng.standard_normal((1, 3, 2)),
               beta=rng.standard_normal((1, 3, 2)), erase=None, write=None)
    a = prologue.apply(raw, 0)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        np.testing.assert_array_equal(a[n], raw[n])
    a = prologue.apply(raw, prologue.L2NORM_QK | prologue.SIGMOID_GATES | prologue.DECAY_SOFTPLUS, 0.1)
    np.testing.assert_array_equal(a["v"], raw["v"])
    np.testing.assert_allclose(np.linalg.norm(a["k"], axis=-1), 1.0, rtol=1e-15)
    np.testing.assert_allclose(a["beta"], 1 / (1 + np.exp(-raw["beta"])), rtol=1e-15)
    np.testing.assert_allclose(a["log_alpha"], -0.1 * np.log1p(np.exp(raw["log_alpha"])), rtol=1e-14)
    a = prologue.apply(raw, prologue.DECAY_LOGSIGMOID)
    np.testing.assert_allclose(a["log_alpha"], np.log(1 / (1 + np.exp(-raw["log_alpha"]))), rtol=1e-14)
    np.testing.assert_array_equal(a["beta"], raw["beta"])


# ---------------------------------------------------------------- backward
def _loss(variant, d, dO, dST, **kw):
    o, ST, _ = oracle.forward(variant, **d, **kw)
    return float(np.sum(o * dO) + np.sum(ST * dST))


@pytest.mark.parametrize("decay", ["none", "scalar", "channel"])
@pytest.mark.parametrize("variant", VARIANTS)
def test_backward_matches_central_differences(variant, decay):
    """The analytic backward of the token loop equals central finite
    differences of the forward, on every element of every input (q, k, v, the
    decay, the gains and gates, S0 and A0), for L = <o, dO> + <S_T, dST>. The
    gate-aware backward of "Gated DeltaNet-2" (ja §3) is this gradient."""
    fixed = {"DN": "none", "PDN": "none", "GDN": "scalar", "PGDN": "scalar", "KDA": "channel",
             "PKDA": "channel"}
    if variant in fixed and fixed[variant] != decay:
        pytest.skip("decay fixed by the variant")
    dk = dv = 4
    d = rand_inputs(variant, B=1, T=5, H=2, dk=dk, dv=dv, seed=50, decay=decay)
    if decay != "none":
        d["log_alpha"] = d["log_alpha"] * 3.0  # stronger decay
    if variant in ("PDN", "PGDN", "PKDA", "PLA"):
        d["A0"] = np.random.default_rng(51).uniform(0.2, 1.0, (1, 2, dk))
    rng = np.random.default_rng(52)
    dO = rng.standard_normal(d["v"].shape)
    dST = rng.standard_normal(d["S0"].shape)
    kw = dict(q_scale=0.8, x=1.5)
    g = oracle.backward(variant, **d, dO=dO, dST=dST, **kw)
    h = 1e-6
    for name, arr in d.items():
        ga = g[name]
        assert ga is not None and ga.shape == arr.shape, name
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            x0 = arr[idx]
            arr[idx] = x0 + h
            lp = _loss(variant, d, dO, dST, **kw)
            arr[idx] = x0 - h
            lm = _loss(variant, d, dO, dST, **kw)
            arr[idx] = x0
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(ga, num, rtol=2e-6, atol=2e-7, err_msg=name)


@pytest.mark.parametrize("decay", ["scalar", "channel"])
def test_decay_gradient_suffix_sum(decay):
    """The decay gradient as a suffix sum over tokens (the form the CUDA
    backward uses; no per-token state): with psi_t,i the cotangent of
    log alpha_t,i and S_t = P_t + delta_t w_t^T,
        psi_t = psi_{t+1} + q'_t . dq'_t - w_t . dw_t + r_t . dr_t,
        psi_T,i = sum_j S_T[j,i] dS_T[j,i].
    Checked in fp64 against the oracle's directly computed gradient
    (sum_j S_{t-1}[j,i] dP_t[j,i] alpha_t,i) on GDN-2, whose (r, w, q')
    cotangents follow from its input gradients: dr = derase / k,
    dw = dk - e . dr, dq' = dq."""
    rng = np.random.default_rng(61)
    d = rand_inputs("GDN2", B=1, T=12, H=2, dk=6, dv=5, seed=60, decay=decay)
    d["log_alpha"] = d["log_alpha"] * 2.0
    dO = rng.standard_normal(d["v"].shape)
    dST = rng.standard_normal(d["S0"].shape)
    g = oracle.backward("GDN2", **d, dO=dO, dST=dST, q_scale=0.7)
    _, ST, _ = oracle.forward("GDN2", d["q"], d["k"], d["v"], log_alpha=d["log_alpha"],
                           erase=d["erase"], write=d["write"], S0=d["S0"], q_scale=0.7)
    k, e, q = d["k"], d["erase"], d["q"]
    dr = g["erase"] / k
    dw = g["k"] - e * dr
    r, w = e * k, k
    term = q * g["q"] - w * dw + r * dr                      # [B,T,H,dk]
    psi = np.einsum("bhji,bhji->bhi", ST, dST)[:, None]        # psi_T, [B,1,H,dk]
    suffix = np.flip(np.cumsum(np.flip(term, axis=1), axis=1), axis=1) + psi
    want = suffix.sum(axis=3) if decay == "scalar" else suffix
    np.testing.assert_allclose(g["log_alpha"], want, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- P7
@pytest.mark.parametrize("lam", [0.5, 2.0])
def test_p7_exact_preconditioning_is_least_squares(lam):
    """Theorem 3.1 ("Preconditioned DeltaNet" ja §2.1, fr §2.A): with the
    exact inverse key Gram matrix applied to the write key (apply-to-key),
    DeltaNet (beta = 1, no decay, S_0 = 0) recovers the least-squares map
    S_t = (sum_i v_i k_i^T) G_t^{-1}, G_t = lam I + sum_i k_i k_i^T, and its
    read-out equals linear attention with the preconditioner applied to the
    query (apply-to-query). Exercises the generic step with a dense,
    non-symmetric read/write key pair."""
    rng = np.random.default_rng(8)
    T, dk, dv = 20, 6, 4
    k = rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    q = rng.standard_normal((T, dk))
    G = lam * np.eye(dk)
    C = np.zeros((dv, dk))
    w = np.zeros((T, dk))
    o_ls = np.zeros((T, dv))
    for t in range(T):
        G = G + np.outer(k[t], k[t])
        C = C + np.outer(v[t], k[t])
        w[t] = np.linalg.solve(G, k[t])
        o_ls[t] = C @ np.linalg.solve(G, q[t])
    o, ST = oracle.generic(q[None, :, None], k[None, :, None], w[None, :, None], v[None, :, None])
    np.testing.assert_allclose(o[0, :, 0], o_ls, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(ST[0, 0], C @ np.linalg.inv(G), rtol=1e-9, atol=1e-10)


# ---------------------------------------------------------------- P8 and preconditioner invariants
@pytest.mark.parametrize("x", [1.2, 1.5, 2.0])
def test_p8_preconditioner_range(x):
    """B_t stays inside [1/x, x] ("Preconditioned DeltaNet" de §2,
    "Stabilitätsverbesserung"; fr §2.C), also for heavy-tailed accumulators."""
    rng = np.random.default_rng(9)
    k = rng.standard_normal((300, 16)) * np.exp(2 * rng.standard_normal(16))[None, :]
    Bc, _ = oracle.precond(k, x=x)
    assert np.all(Bc >= 1 / x - 1e-15) and np.all(Bc <= x + 1e-15)
    assert Bc.max() > 1.0 and Bc.min() < 1.0


def test_precond_identity_and_symmetry():
    """Centring: equal accumulators give B = 1; with d_k = 2 the centred logs
    are opposite, so B_0 B_1 = 1; x = 1 gives B = 1 everywhere."""
    rng = np.random.default_rng(10)
    signs = rng.choice([-1.0, 1.0], size=(50, 8))
    Bc, _ = oracle.precond(signs / np.sqrt(8.0), x=1.5)
    np.testing.assert_allclose(Bc, 1.0, rtol=0, atol=1e-14)
    k2 = rng.standard_normal((40, 2))
    Bc2, _ = oracle.precond(k2, x=1.7)
    np.testing.assert_allclose(Bc2[:, 0] * Bc2[:, 1], 1.0, rtol=1e-13)
    Bc1, _ = oracle.precond(rng.standard_normal((30, 8)), x=1.0)
    np.testing.assert_array_equal(Bc1, 1.0)


def test_precond_decreasing_in_accumulated_energy():
    """P_t = Diag(A_t)^{-1}: channels with more accumulated key energy get a
    smaller coefficient ("Preconditioned DeltaNet" fr §2.B)."""
    rng = np.random.default_rng(11)
    k = rng.standard_normal((64, 12)) * np.linspace(0.2, 3.0, 12)[None, :]
    Bc, AT = oracle.precond(k, x=1.5)
    A = np.cumsum(k * k, axis=0)
    for t in range(64):
        order = np.argsort(A[t])
        assert np.all(np.diff(Bc[t, order]) <= 1e-15)
    np.testing.assert_allclose(AT, A[-1], rtol=1e-13)
    _, AT2 = oracle.precond(k, A0=np.full(12, 3.0), x=1.5)
    np.testing.assert_allclose(AT2, A[-1] + 3.0, rtol=1e-13)


def test_p8_eigenvalue_control_and_bounded_state():
    """x <= 2 keeps the non-unit eigenvalue 1 - beta k~^T k of the transition
    in [-1, 1) for unit keys and beta in (0, 1) ("Preconditioned DeltaNet"
    fr §2.C), and the state stays bounded over a 32k-token random stream."""
    rng = np.random.default_rng(12)
    T, dk, dv = 32768, 16, 16
    k = unit(rng.standard_normal((1, T, 1, dk)))
    Bc, _ = oracle.precond(k[0, :, 0], x=2.0)
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1))))
    lam = 1 - beta[0, :, 0] * np.sum(Bc * k[0, :, 0] ** 2, axis=1)
    assert np.all(lam >= -1.0) and np.all(lam < 1.0)
    v = rng.standard_normal((1, T, 1, dv))
    o, ST, _ = oracle.forward("PDN", k.copy(), k, v, beta=beta, x=2.0)
    assert np.isfinite(o).all()
    assert np.linalg.norm(ST) < 20 * np.sqrt(dv)
    assert np.abs(o).max() < 50


# ---------------------------------------------------------------- P9
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 37, 100, 128])
def test_p9_chunk_form_equals_token_loop(chunk, T):
    """The chunkwise WY/UT form ("Gated DeltaNet-2" ja §3: decay absorbed into
    the erase/write matrices, lower-triangular (I+T)^{-1} solve for the
    auxiliaries Y and U) reproduces the token recurrence to fp64 rounding, for
    every chunk length and a ragged tail."""
    rng = np.random.default_rng(13 + T)
    B, H, dk, dv = 1, 2, 8, 6
    q = unit(rng.standard_normal((B, T, H, dk)))
    r = unit(rng.standard_normal((B, T, H, dk)))
    w = 0.8 * unit(rng.standard_normal((B, T, H, dk))) * rng.uniform(0.3, 1.2, (B, T, H, dk))
    u = rng.standard_normal((B, T, H, dv))
    la = -0.2 * np.abs(rng.standard_normal((B, T, H, dk)))
    S0 = rng.standard_normal((B, H, dv, dk))
    o1, S1 = oracle.generic(q, r, w, u, log_alpha=la, S0=S0, q_scale=0.9)
    o2, S2 = chunked.chunk_forward(q, r, w, u, log_alpha=la, S0=S0, chunk=chunk, q_scale=0.9)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("mean_log_alpha", [-1.5, -3.0, -10.0, "hard"])
@pytest.mark.parametrize("chunk", [16, 64])
def test_p9_chunk_form_under_strong_decay(mean_log_alpha, chunk):
    """The chunk form stays equal to the token loop however strong the decay:
    the pages bound alpha only to (0, 1) (KDA's D_t = Diag(alpha_t),
    "Gated DeltaNet-2" ja §1), so mean per-token log decays of -1.5, -3 and -10
    (whole-chunk decays of e^-96 .. e^-640 per channel) and one channel at
    log alpha = -30 on every token ("hard") must all reproduce the recurrence,
    down to fp64 rounding."""
    rng = np.random.default_rng(29)
    B, T, H, dk, dv = 1, 150, 2, 8, 6
    q = unit(rng.standard_normal((B, T, H, dk)))
    r = unit(rng.standard_normal((B, T, H, dk)))
    w = 0.8 * unit(rng.standard_normal((B, T, H, dk))) * rng.uniform(0.3, 1.2, (B, T, H, dk))
    u = rng.standard_normal((B, T, H, dv))
    if mean_log_alpha == "hard":
        la = -0.1 * np.abs(rng.standard_normal((B, T, H, dk)))
        la[..., 3] = -30.0
    else:
        la = 2.0 * mean_log_alpha * rng.uniform(0.0, 1.0, (B, T, H, dk))
    S0 = rng.standard_normal((B, H, dv, dk))
    o1, S1 = oracle.generic(q, r, w, u, log_alpha=la, S0=S0, q_scale=0.9)
    o2, S2 = chunked.chunk_forward(q, r, w, u, log_alpha=la, S0=S0, chunk=chunk, q_scale=0.9)
    assert np.isfinite(o2).all() and np.isfinite(S2).all()
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-11)


# ---------------------------------------------------------------- P10
@pytest.mark.parametrize("variant", VARIANTS)
def test_p10_continuation(variant):
    """The fixed-size state is the whole carry ("Gated DeltaNet-2" ja,
    problem statement: constant-memory decoding): running T1 tokens, then T2
    tokens from (S_T1, A_T1), equals one run over T1 + T2 tokens."""
    d = rand_inputs(variant, T=11, seed=14)
    o, ST, AT = oracle.forward(variant, **d)
    d1 = {n: (a[:, :5] if n not in ("S0",) else a) for n, a in d.items()}
    d2 = {n: a[:, 5:] for n, a in d.items() if n != "S0"}
    oa, Sa, Aa = oracle.forward(variant, **d1)
    ob, Sb, Ab = oracle.forward(variant, **d2, S0=Sa, A0=Aa)
    np.testing.assert_array_equal(np.concatenate([oa, ob], axis=1), o)
    np.testing.assert_array_equal(Sb, ST)
    np.testing.assert_array_equal(Ab, AT)


def test_oracle_rejects_bad_arguments():
    d = rand_inputs("FG2_GDN", dk=8, dv=6)
    with pytest.raises(ValueError):
        oracle.forward("FG2_GDN", **d)  # FG2 needs d_k == d_v
    d = rand_inputs("FG2_GDN_PLUS")
    del d["write"]
    with pytest.raises(ValueError):
        oracle.forward("FG2_GDN_PLUS", **d)  # the value-side gain is required
    d = rand_inputs("GDN2")
    del d["erase"]
    with pytest.raises(ValueError):
        oracle.forward("GDN2", **d)


def test_threads_do_not_change_results():
    d = rand_inputs("PKDA", B=3, H=3, T=20, seed=15)
    o1, S1, A1 = oracle.forward("PKDA", **d, nthreads=1)
    o2, S2, A2 = oracle.forward("PKDA", **d, nthreads=5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    np.testing.assert_array_equal(A1, A2)
