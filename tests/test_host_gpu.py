"""pdn_chunk_fwd_host (inputs and outputs in page-locked host memory, copies
overlapped with the compute over slices of the batch) against pdn_chunk_fwd
on device buffers: the batch elements are independent chains, so every
output must be bitwise the same for any number of slices; and against the
oracle once."""
import pytest
import torch

from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import Workload, make_inputs

from parity_util import assert_parity, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

DECAY = {"PGDN": "scalar", "PKDA": "channel", "FG2_GDN": "channel", "GDN2": "channel",
         "DN": "none", "PLA": "scalar", "FG2_GDN_PLUS": "channel"}
GATES = ("log_alpha", "beta", "erase", "write")


def host_run(w, x, S0, A0, slices):
    dev = torch.device("cuda")
    hx = {n: (t.pin_memory() if t is not None else None) for n, t in x.items()}
    ho = torch.empty(w.B, w.T, w.H, w.dv, dtype=x["v"].dtype).pin_memory()
    hS0 = S0.pin_memory() if S0 is not None else None
    hA0 = A0.pin_memory() if A0 is not None else None
    hST = torch.empty(w.B, w.H, w.dv, w.dk).pin_memory()
    precond = w.variant in pdn.PRECOND_VARIANTS
    hAT = torch.empty(w.B, w.H, w.dk).pin_memory() if precond else None
    dx = {n: (torch.empty_like(t, device=dev) if t is not None else None) for n, t in hx.items()}
    do = torch.empty(ho.shape, dtype=ho.dtype, device=dev)
    dS0 = torch.empty_like(hS0, device=dev) if hS0 is not None else None
    dA0 = torch.empty_like(hA0, device=dev) if hA0 is not None else None
    dST = torch.empty(hST.shape, device=dev)
    dAT = torch.empty(hAT.shape, device=dev) if precond else None
    prob = pdn.make_problem(w.variant, w.B, w.T, w.H, w.dk, w.dv, x["k"].dtype, w.decay)
    ws_bytes = pdn.pdn_chunk_fwd_workspace(prob)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    th = pdn.make_host_tensors(hx["q"], hx["k"], hx["v"], ho, *(hx[n] for n in GATES),
                               S0=hS0, ST=hST, A0=hA0, AT=hAT)
    td = pdn.make_tensors(dx["q"], dx["k"], dx["v"], do, *(dx[n] for n in GATES),
                          S0=dS0, ST=dST, A0=dA0, AT=dAT)
    stream = torch.cuda.current_stream().cuda_stream
    rc = pdn.pdn_chunk_fwd_host(prob, th, td, ws.data_ptr(), ws.numel(), slices, stream)
    assert rc == pdn.PDN_OK, pdn.pdn_status_string(rc)
    torch.cuda.synchronize()
    assert pdn.device_error() == pdn.PDN_OK
    return ho, hST, hAT


@pytest.mark.parametrize("variant", ["PGDN", "PKDA", "FG2_GDN", "GDN2", "DN", "PLA", "FG2_GDN_PLUS"])
def test_host_path_matches_device_path(variant):
    w = Workload("host-" + variant, variant, 3, 130, 2, 128, 128, "bf16", DECAY[variant])
    x = make_inputs(w)
    g = torch.Generator().manual_seed(7)
    S0 = 0.2 * torch.randn(w.B, w.H, 128, 128, generator=g)
    A0 = torch.rand(w.B, w.H, 128, generator=g) if variant in pdn.PRECOND_VARIANTS else None
    ref = run_gpu(w, x, S0, A0)
    for slices in (1, 2, 3):
        o, ST, AT = host_run(w, x, S0, A0, slices)
        assert torch.equal(o, ref[0].cpu()), (variant, slices)
        assert torch.equal(ST, ref[1].cpu()), (variant, slices)
        if AT is not None:
            assert torch.equal(AT, ref[2].cpu()), (variant, slices)


def test_host_path_parity_with_oracle():
    w = Workload("host-oracle", "PGDN", 2, 200, 2, 128, 128, "bf16", "scalar")
    x = make_inputs(w)
    o, ST, AT = host_run(w, x, None, None, 2)
    assert_parity(w, o, ST, AT, *run_oracle(w, x))


@pytest.mark.parametrize("variant", ["PGDN", "GDN2"])
def test_host_path_odd_token_head_count(variant):
    """T * H odd (131 x 1): slice 1's fp32 scalar-gate pointers sit 4 bytes
    off a 16-byte boundary, which the scalar gates allow; every slicing gives
    the device path's outputs bitwise."""
    w = Workload("host-odd-" + variant, variant, 3, 131, 1, 128, 128, "bf16", DECAY[variant])
    x = make_inputs(w)
    ref = run_gpu(w, x)
    for slices in (2, 3):
        o, ST, AT = host_run(w, x, None, None, slices)
        assert torch.equal(o, ref[0].cpu()), (variant, slices)
        assert torch.equal(ST, ref[1].cpu()), (variant, slices)


def device_runs(w, x, S0, A0, slices):
    """The device path cut the way pdn_chunk_fwd_host cuts sequences when
    slices > B: per batch element, runs of whole chunks in order, each
    pdn_chunk_fwd continuing from the previous run's S_T and A_T."""
    dev = torch.device("cuda")
    N = (w.T + 63) // 64
    runs = min(-(-slices // w.B), N)
    L = -(-N // runs)
    runs = -(-N // L)
    os, Ss, As = [], [], []
    for b in range(w.B):
        S = S0[b:b + 1].to(dev) if S0 is not None else None
        A = A0[b:b + 1].to(dev) if A0 is not None else None
        ob = []
        for j in range(runs):
            t0, t1 = j * L * 64, (w.T if j + 1 == runs else (j + 1) * L * 64)
            sl = {n: (t[b:b + 1, t0:t1].contiguous().to(dev) if t is not None else None)
                  for n, t in x.items()}
            o, S, A = pdn.chunk_fwd(w.variant, sl["q"], sl["k"], sl["v"],
                                    **{n: sl[n] for n in GATES}, S0=S, A0=A)
            ob.append(o)
        os.append(torch.cat(ob, 1))
        Ss.append(S)
        As.append(A)
    torch.cuda.synchronize()
    o = torch.cat(os, 0).cpu()
    ST = torch.cat(Ss, 0).cpu()
    AT = torch.cat(As, 0).cpu() if As[0] is not None else None
    return o, ST, AT


@pytest.mark.parametrize("variant,dk,dtype", [("PGDN", 128, "bf16"), ("GDN2", 128, "bf16"),
                                              ("PKDA", 128, "bf16"), ("PGDN", 64, "f32")])
def test_host_path_cuts_sequences_into_runs(variant, dk, dtype):
    """slices > B: every sequence is also cut into runs of whole chunks that
    hand the state and accumulator on through the device S_T and A_T. The
    outputs equal the device path cut at the same chunk boundaries bitwise,
    and the oracle within the parity bar; runs of 2, 3 and 5 per sequence
    (the last with a ragged 44-token tail)."""
    w = Workload("host-runs-" + variant, variant, 2, 300, 2, dk, dk, dtype, DECAY[variant])
    x = make_inputs(w)
    g = torch.Generator().manual_seed(9)
    S0 = 0.2 * torch.randn(w.B, w.H, dk, dk, generator=g)
    A0 = torch.rand(w.B, w.H, dk, generator=g) if variant in pdn.PRECOND_VARIANTS else None
    for slices in (3, 5, 10):
        o, ST, AT = host_run(w, x, S0, A0, slices)
        ro, rS, rA = device_runs(w, x, S0, A0, slices)
        assert torch.equal(o, ro), (variant, slices)
        assert torch.equal(ST, rS), (variant, slices)
        if AT is not None:
            assert torch.equal(AT, rA), (variant, slices)
    assert_parity(w, o, ST, AT, *run_oracle(w, x, S0, A0))
