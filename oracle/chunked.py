"""fp64 chunk form of the generic delta step (TEST INFRASTRUCTURE ONLY).

The pages describe a chunkwise-parallel form of the same recurrence: the decay
is absorbed into the erase and write matrices and a lower-triangular system
(I + T)^{-1} is solved to get an erase-side auxiliary Y and a write-side
auxiliary U ("Gated DeltaNet-2", ja §3 "efficient chunkwise parallel
training"; "Preconditioned DeltaNet", ja §2.3 "chunkwise parallelisation";
"FG2-GDN", ja §2.3 "DPLR structure"). This module writes that form out with
numpy so a test can check, before any kernel exists, that the chunk algebra
the kernels use reproduces the token loop. It is a cross-check of the
algebra, not a second definition: the definition is the token loop in
pdn_oracle.c.

Per chunk of C tokens with state S0 (d_v x d_k) and cumulative in-chunk log
decay G_t = sum_{s<=t} log alpha_s (per key channel):
    M_ts = sum_i r_ti w_si e^{G_ti - G_si}        (s < t)
    P_ts = sum_i q_ti w_si e^{G_ti - G_si}        (s <= t)
    Rh = e^{G} . r,  Qh = e^{G} . q,  Wb = e^{G_C - G} . w
    Y  = (I + M)^{-1} Rh,  U~ = (I + M)^{-1} u
    D  = U~ - Y S0^T
    O  = q_scale (Qh S0^T + P D)
    S_C = S0 Diag(e^{G_C}) + D^T Wb
The decay between two tokens of a chunk is formed from the difference
G_t - G_s <= 0 itself, never as the product e^{G_t} e^{-G_s}: the pages put no
floor on the decay (KDA's D_t = Diag(alpha_t), alpha_t in (0,1)^{d_k},
"Gated DeltaNet-2" ja §1), and for strong decay e^{-G_s} overflows even fp64.
"""
from __future__ import annotations

import numpy as np


def chunk_forward(q, r, w, u, log_alpha=None, S0=None, chunk=64, q_scale=1.0):
    """Shapes as oracle.generic: q, r, w [B,T,H,dk]; u [B,T,H,dv]; log_alpha
    None or [B,T,H,dk]; S0 [B,H,dv,dk]. Returns (o [B,T,H,dv], S_T)."""
    q, r, w, u = (np.asarray(a, np.float64) for a in (q, r, w, u))
    B, T, H, dk = r.shape
    dv = u.shape[3]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk)) if S0 is None else np.array(S0[b, h], np.float64)
            for c0 in range(0, T, chunk):
                c1 = min(T, c0 + chunk)
                if log_alpha is None:
                    G = np.zeros((c1 - c0, dk))
                else:
                    G = np.cumsum(np.asarray(log_alpha[b, c0:c1, h], np.float64), axis=0)
                n = c1 - c0
                low = np.tril(np.ones((n, n), bool))
                # E[t, s, i] = e^{G_ti - G_si} for s <= t, 0 above the diagonal
                diff = G[:, None, :] - G[None, :, :]
                E = np.exp(np.where(low[:, :, None], diff, -np.inf))
                rc, wc, qc = r[b, c0:c1, h], w[b, c0:c1, h], q[b, c0:c1, h]
                M = np.tril(np.einsum("ti,si,tsi->ts", rc, wc, E), -1)
                P = np.einsum("ti,si,tsi->ts", qc, wc, E)
                Rh = np.exp(G) * rc
                Qh = np.exp(G) * qc
                Wb = np.exp(G[-1][None, :] - G) * wc
                Tinv = np.linalg.inv(np.eye(c1 - c0) + M)
                Y = Tinv @ Rh
                Ut = Tinv @ u[b, c0:c1, h]
                D = Ut - Y @ S.T
                o[b, c0:c1, h] = q_scale * (Qh @ S.T + P @ D)
                S = S * np.exp(G[-1])[None, :] + D.T @ Wb
            ST[b, h] = S
    return o, ST
