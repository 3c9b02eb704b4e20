"""The allocation-free chunked forward (pdn_chunk_fwd_noalloc), for callers
that cannot allocate a device workspace: its scratch is a fixed array inside
the library. Checked through the C ABI against the workspace entry point
(pdn_chunk_fwd) on two calls in a row, and against its size limit. This file
is collected last so a run that stops at the first failure has already run
every other test."""
import ctypes

import pytest
import torch

from linear_recurrence_sequence_chunked_b200 import pdn
from linear_recurrence_sequence_chunked_b200.workloads import Workload, make_inputs

from parity_util import TOL, nmax_err

pytestmark = pytest.mark.gpu


def _buffers(w, x):
    dev = torch.device("cuda")
    d = {n: (t.to(dev) if t is not None else None) for n, t in x.items()}
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=torch.bfloat16, device=dev)
    ST = torch.empty(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=dev)
    AT = (torch.empty(w.B, w.H, w.dk, dtype=torch.float32, device=dev)
          if w.variant in pdn.PRECOND_VARIANTS else None)
    t = pdn.make_tensors(d["q"], d["k"], d["v"], o, d["log_alpha"], d["beta"], d["erase"],
                         d["write"], ST=ST, AT=AT)
    return d, t, o, ST, AT


def _problem(w):
    return pdn.make_problem(w.variant, w.B, w.T, w.H, w.dk, w.dv, torch.bfloat16, w.decay, 64,
                            "tc", w.q_scale, w.precond_x, w.precond_eps)


def test_noalloc_matches_workspace_entry_point_two_calls():
    """Calls in a row on the one array: 40 chunk blocks, then 48, then a
    smaller call (4 blocks, ragged tail) after the larger ones, so stale
    contents from an earlier call would show; then the largest problem the
    array takes (809 blocks)."""
    stream = torch.cuda.current_stream().cuda_stream
    cases = [Workload("na1", "PGDN", 2, 300, 4, 128, 128, "bf16", "scalar", seed=11),
             Workload("na2", "PKDA", 1, 500, 6, 128, 128, "bf16", "channel", seed=12),
             Workload("na3", "PGDN", 1, 100, 2, 128, 128, "bf16", "scalar", seed=13),
             Workload("na4", "GDN", 1, 809 * 64 - 10, 1, 128, 128, "bf16", "scalar", seed=14)]
    results = []
    for w in cases:  # calls in a row, each reusing the array
        x = make_inputs(w)
        _, t, o, ST, AT = _buffers(w, x)
        assert pdn.pdn_chunk_fwd_noalloc(_problem(w), t, stream) == pdn.PDN_OK
        torch.cuda.synchronize()
        assert pdn.device_error() == pdn.PDN_OK
        results.append((w, x, o.clone(), ST.clone(), None if AT is None else AT.clone()))
    for w, x, o_na, S_na, A_na in results:
        d = {n: (t.cuda() if t is not None else None) for n, t in x.items()}
        o, ST, AT = pdn.chunk_fwd(w.variant, d["q"], d["k"], d["v"], log_alpha=d["log_alpha"],
                                  beta=d["beta"], impl="tc", precond_x=w.precond_x,
                                  precond_eps=w.precond_eps)
        torch.cuda.synchronize()
        tol = TOL["bf16"]
        assert nmax_err(o_na.float().cpu().numpy(), o.float().cpu().numpy()) <= tol
        assert nmax_err(S_na.cpu().numpy(), ST.cpu().numpy()) <= tol
        if A_na is not None:
            assert nmax_err(A_na.cpu().numpy(), AT.cpu().numpy()) <= 1e-6


def test_noalloc_rejects_problems_beyond_the_array():
    w = Workload("na-big", "PGDN", 4, 4096, 16, 128, 128, "bf16", "scalar")  # 4096 chunk blocks
    fake = 0x7f0000000000
    t = pdn.PdnTensors(q=fake, k=fake, v=fake, log_alpha=fake, beta=fake, o=fake)
    assert pdn.pdn_chunk_fwd_noalloc(_problem(w), t, None) == pdn.PDN_ERR_WORKSPACE
    # one chunk block past the limit (810 blocks), rejected before any launch
    big = _problem(w.replace(B=1, H=1, T=810 * 64))
    assert pdn.pdn_chunk_fwd_noalloc(big, t, None) == pdn.PDN_ERR_WORKSPACE
    small = _problem(w.replace(B=1, H=1, T=64))
    small.d_k = 64  # not a shape the tensor-core path takes
    assert pdn.pdn_chunk_fwd_noalloc(small, t, None) == pdn.PDN_ERR_UNSUPPORTED
