"""Sequential residual codebook fit on the GPU, driven from Python through the C ABI.

Order of the steps (review, "What carries the argument": the codebook is fit by EM and R
residual rounds refine the reconstruction): for round r, seed the round's codebook from
the residual rows (Forgy: entry c of group j is sub-vector j of row init(r)[c]), run
`iters` calls of commvq_em_step, then advance the residuals with one commvq_encode round
against the final codebook (its residual output). All arithmetic runs in the library's
kernels; this module gathers the seed rows and orders the calls.
"""
from __future__ import annotations

from typing import Callable

import numpy as np
import torch

from . import api


def fit_codebook(rows: torch.Tensor, R: int, n_codes: int, iters: int,
                 init_indices: Callable[[int, int], np.ndarray], g: int = 8,
                 sse_history: bool = False):
    """rows [N, d] float32 on the device -> codebook [R, d/g, Nc', g] float32 (and the
    per-step SSE of each round when sse_history)."""
    N, d = rows.shape
    G = d // g
    cfg1 = api.Config(d=d, g=g, R=1, n_codes=n_codes, q_heads=1, kv_heads=1)
    ws = torch.empty(api.em_workspace_bytes(cfg1, N), dtype=torch.uint8, device=rows.device)
    res = rows.contiguous()
    rounds, hist = [], []
    for r in range(R):
        idx = torch.from_numpy(np.asarray(init_indices(r, N), dtype=np.int64)).to(rows.device)
        cb_r = res.index_select(0, idx).reshape(n_codes, G, g).permute(1, 0, 2).contiguous()
        sse = torch.zeros(max(iters, 1), dtype=torch.float64, device=rows.device)
        for it in range(iters):
            api.em_step(cfg1, res, cb_r, sse_out=sse[it:it + 1], workspace=ws)
        nxt = torch.empty_like(res)
        api.encode(cfg1, res.view(N, 1, d), cb_r.unsqueeze(0), residual_out=nxt.view(N, 1, d))
        res = nxt
        rounds.append(cb_r)
        hist.append(sse[:iters])
    cb = torch.stack(rounds).contiguous()
    if sse_history:
        return cb, [h.cpu().tolist() for h in hist]
    return cb
