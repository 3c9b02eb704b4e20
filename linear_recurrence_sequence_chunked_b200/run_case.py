"""Run one workload through the library a few times: a fixed, small command to
point a profiler at (``ncu ... python -m linear_recurrence_sequence_chunked_b200.run_case
--op fwd --workload gdn2_bf16_32k --batch 1 --tokens 8192``).

``--op fwd`` calls pdn_chunk_fwd, ``bwd`` pdn_chunk_bwd (from random dO and
dS_T), ``train`` pdn_chunk_fwd_save then pdn_chunk_bwd_saved (training mode),
``decode`` pdn_decode_step once per token. Inputs are the seeded
synthetic ones of ``workloads.py``; ``--batch`` and ``--tokens`` override the
workload's B and T. Exits non-zero if a call fails or the device error word is
set.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import pdn
from .workloads import WORKLOADS, make_inputs


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="pgdn_bf16_4k", choices=sorted(WORKLOADS))
    ap.add_argument("--op", default="fwd", choices=("fwd", "bwd", "train", "decode"))
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--calls", type=int, default=2)
    args = ap.parse_args(argv)
    w = WORKLOADS[args.workload]
    over = {}
    if args.batch:
        over["B"] = args.batch
    if args.tokens:
        over["T"] = args.tokens
    if over:
        w = w.replace(**over)
    dev = torch.device("cuda")
    if args.op == "decode":
        x = make_inputs(w, device=dev, T=args.calls)
        S = torch.zeros(w.B, w.H, w.dv, w.dk, device=dev)
        A = torch.zeros(w.B, w.H, w.dk, device=dev) if w.variant in pdn.PRECOND_VARIANTS else None
        for s in range(args.calls):
            sl = {n: (t[:, s:s + 1].contiguous() if t is not None else None) for n, t in x.items()}
            pdn.decode_step(w.variant, sl["q"], sl["k"], sl["v"], S, A, log_alpha=sl["log_alpha"],
                            beta=sl["beta"], erase=sl["erase"], write=sl["write"],
                            q_scale=w.q_scale, precond_x=w.precond_x, precond_eps=w.precond_eps)
    else:
        x = make_inputs(w, device=dev)
        g = {n: x[n] for n in ("log_alpha", "beta", "erase", "write")}
        kw = dict(q_scale=w.q_scale, precond_x=w.precond_x, precond_eps=w.precond_eps)
        if args.op == "fwd":
            for _ in range(args.calls):
                pdn.chunk_fwd(w.variant, x["q"], x["k"], x["v"], **g, chunk=w.chunk, **kw)
        else:
            gen = torch.Generator(device=dev).manual_seed(7)
            dO = torch.randn(w.B, w.T, w.H, w.dv, generator=gen, device=dev).to(x["v"].dtype)
            dST = torch.randn(w.B, w.H, w.dv, w.dk, generator=gen, device=dev)
            for _ in range(args.calls):
                if args.op == "train":
                    saved = {}
                    _, ST, _ = pdn.chunk_fwd(w.variant, x["q"], x["k"], x["v"], **g, chunk=w.chunk,
                                             saved=saved, **kw)
                    pdn.chunk_bwd(w.variant, x["q"], x["k"], x["v"], dO=dO, dST=dST, **g,
                                  saved=saved, ST=ST, **kw)
                else:
                    pdn.chunk_bwd(w.variant, x["q"], x["k"], x["v"], dO=dO, dST=dST, **g, **kw)
    torch.cuda.synchronize()
    if pdn.device_error() != pdn.PDN_OK:
        print("device error word set", file=sys.stderr)
        return 1
    print("ok: %s %s B=%d T=%d H=%d, %d calls" % (args.op, w.name, w.B, w.T, w.H, args.calls))
    return 0


if __name__ == "__main__":
    sys.exit(main())
