"""Sequential residual codebook fit on the GPU, driven from Python through the C ABI.

Order of the steps (review, "What carries the argument": the codebook is fit by EM and R
residual rounds refine the reconstruction): for round r, seed the round's codebook from
the residual rows (Forgy: entry c of group j is sub-vector j of row init(r)[c]), run
`iters` calls of commvq_em_step, then advance the residuals with one commvq_encode round
against the final codebook (its residual output). All arithmetic runs in the library's
kernels; this module gathers the seed rows and orders the calls. With a checkpoint path the
fit is saved after every EM step and resumed from that file (checkpoint.py).
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np
import torch

from . import api
from .checkpoint import FitSteps, resumable_fit


def fit_codebook(rows: torch.Tensor, R: int, n_codes: int, iters: int,
                 init_indices: Callable[[int, int], np.ndarray], g: int = 8,
                 sse_history: bool = False, checkpoint: Optional[str] = None, seed: int = 0,
                 on_step: Optional[Callable[[int, int], None]] = None):
    """rows [N, d] float32 on the device -> codebook [R, d/g, Nc', g] float32 (and the
    per-step SSE of each round run in this call when sse_history). checkpoint: a file to save
    the fit's progress to after every EM step and to resume from (same d, g, R, Nc', iters and
    seed), giving the uninterrupted fit's codebook bit for bit. on_step(r, it) is called after
    each EM step (after its checkpoint is written)."""
    N, d = rows.shape
    G = d // g
    dev = rows.device
    cfg1 = api.Config(d=d, g=g, R=1, n_codes=n_codes, q_heads=1, kv_heads=1)
    ws = torch.empty(api.em_workspace_bytes(cfg1, N), dtype=torch.uint8, device=dev)
    hist = {}
    cur = [-1]   # the round being fit (-1: a round resumed part-way from a checkpoint)

    def em_step(res, cb_r):
        sse = torch.zeros(1, dtype=torch.float64, device=dev)
        api.em_step(cfg1, res, cb_r, sse_out=sse, workspace=ws)
        hist.setdefault(cur[0], []).append(sse)
        return cb_r

    def seed_round(res, r):
        cur[0] = r
        idx = torch.from_numpy(np.asarray(init_indices(r, N), dtype=np.int64)).to(dev)
        return res.index_select(0, idx).reshape(n_codes, G, g).permute(1, 0, 2).contiguous()

    def advance(res, cb_r):
        nxt = torch.empty_like(res)
        api.encode(cfg1, res.view(N, 1, d), cb_r.unsqueeze(0), residual_out=nxt.view(N, 1, d))
        return nxt

    def from_numpy(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)

    steps = FitSteps(em_step=em_step, advance=advance, seed_round=seed_round,
                     to_numpy=lambda t: t.detach().cpu().numpy(), from_numpy=from_numpy)
    rounds = resumable_fit(rows.contiguous(), R, g, n_codes, iters, steps, path=checkpoint, seed=seed,
                           on_step=on_step)
    cb = torch.stack(rounds).contiguous()
    if sse_history:
        return cb, [[float(x.item()) for x in hist[r]] for r in sorted(k for k in hist if k >= 0)]
    return cb
