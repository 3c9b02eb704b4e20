"""Sequence-parallel prefill on CPU ranks: the orchestration of
linear_recurrence_sequence_chunked_b200.seqpar over a world-size-2 gloo
process group, with fp64 stand-ins for the per-segment operations, against
one token loop over the whole sequence; and its single-process phases for
1..4 segments."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
from linear_recurrence_sequence_chunked_b200 import seqpar  # noqa: E402
from linear_recurrence_sequence_chunked_b200.workloads import Workload, make_inputs  # noqa: E402
from seqpar_oracle_ops import OracleOps  # noqa: E402

CASES = [("PGDN", "scalar"), ("PKDA", "channel"), ("GDN2", "channel"), ("FG2_GDN_PLUS", "channel"),
         ("PLA", "scalar"), ("DN", "none")]


def _inputs(variant, decay, T=37):
    w = Workload("sp", variant, 2, T, 2, 8, 8, "f32", decay, seed=3)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(9)
    S0 = 0.3 * torch.randn(2, 2, 8, 8, generator=g, dtype=torch.float64)
    A0 = torch.rand(2, 2, 8, generator=g, dtype=torch.float64) if variant in ("PDN", "PGDN", "PKDA", "PLA") else None
    return w, {n: (t.double().numpy() if t is not None else None) for n, t in x.items()}, S0, A0


def _segment(x, bounds, g):
    t0, t1 = bounds[g], bounds[g + 1]
    return {n: (a[:, t0:t1].copy() if a is not None else None) for n, a in x.items()}


def _full(variant, x, S0, A0):
    return oracle.forward(variant, x["q"], x["k"], x["v"], log_alpha=x["log_alpha"], beta=x["beta"],
                          erase=x["erase"], write=x["write"], S0=S0, A0=A0)


def _worker(rank, world, port, variant, decay, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, x, S0, A0 = _inputs(variant, decay)
        bounds = [0, 20, w.T]  # uneven segments, not on chunk boundaries

        def gather(t):
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t.contiguous())
            return torch.stack(parts)

        o, S, A = seqpar.seqpar_forward(OracleOps(variant), _segment(x, bounds, rank), rank, world,
                                        gather, S0=S0, A0=A0)
        out[rank] = (o.numpy(), S.numpy(), None if A is None else A.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("variant,decay", [("PKDA", "channel"), ("GDN2", "channel")])
def test_two_gloo_ranks_match_one_pass(variant, decay):
    port = 29600 + (os.getpid() % 900)
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, variant, decay, out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    w, x, S0, A0 = _inputs(variant, decay)
    o, ST, AT = _full(variant, x, S0.numpy(), None if A0 is None else A0.numpy())
    np.testing.assert_allclose(np.concatenate([res[0][0], res[1][0]], axis=1), o, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(res[1][1], ST, rtol=1e-9, atol=1e-10)
    if AT is not None and variant in ("PKDA",):
        np.testing.assert_allclose(res[1][2], AT, rtol=1e-12)


@pytest.mark.parametrize("segments", [1, 2, 3, 4])
@pytest.mark.parametrize("variant,decay", CASES)
def test_phases_in_one_process_match_one_pass(variant, decay, segments):
    """The same protocol with the all-gathers done in one process: phase 1 for
    every segment, gather, phase 2, gather, phase 3."""
    w, x, S0, A0 = _inputs(variant, decay)
    bounds = np.linspace(0, w.T, segments + 1).astype(int).tolist()
    ops = OracleOps(variant)
    segs = [seqpar.SegmentPrefill(ops, _segment(x, bounds, g), g) for g in range(segments)]
    energies = torch.stack([s.energy() for s in segs]) if ops.precond else None
    loc = [s.local(energies, A0) for s in segs]
    A_all = torch.stack([a for a, _ in loc])
    B_all = torch.stack([b for _, b in loc])
    res = [s.finish(A_all, B_all, S0) for s in segs]
    o, ST, AT = _full(variant, x, S0.numpy(), None if A0 is None else A0.numpy())
    np.testing.assert_allclose(torch.cat([r[0] for r in res], dim=1).numpy(), o, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(res[-1][1].numpy(), ST, rtol=1e-9, atol=1e-10)
