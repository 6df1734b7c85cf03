"""Shared fixtures for parity tests: seeded inputs (from synth), oracle-side codebooks,
and the attention error metric.

Every expected value here comes from the CPU oracle; nothing is taken from the CUDA path.
"""
from __future__ import annotations

import functools

import numpy as np

from decode_attention_commvq_b200 import synth
from oracle import oracle as O

# Attention tolerance: max over (b, h) of max_i |o_i - r_i| / max_i |r_i|.
TOL_F32 = 2e-3    # fp32 inputs (the tiny workload)
TOL_BF16 = 5e-3   # bf16 queries


def tol_for(w: synth.Workload) -> float:
    return TOL_F32 if w.q_dtype == "f32" else TOL_BF16


def rel_err(out: np.ndarray, ref: np.ndarray) -> float:
    """max over leading (b, h) of max_i |o - r| / max_i |r|."""
    o = out.reshape(-1, out.shape[-1]).astype(np.float64)
    r = ref.reshape(-1, ref.shape[-1]).astype(np.float64)
    num = np.abs(o - r).max(axis=1)
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return float((num / den).max())


@functools.lru_cache(maxsize=None)
def oracle_codebooks(w: synth.Workload):
    """(kcb, vcb) [R, d/g, Nc', g] float32 for a workload: N(0,1) entries for the tiny
    workload, otherwise the oracle's sequential EM fit on the seeded fitting rows."""
    if w.codebook == "normal":
        return synth.normal_codebook(w, True), synth.normal_codebook(w, False)
    out = []
    for key in (True, False):
        rows = synth.fit_rows(w, key)
        cb, _ = O.fit_codebook(rows, w.R, w.g, w.n_codes, w.em_iters,
                               lambda r, N, key=key: synth.forgy_indices(w, key, r, N))
        out.append(cb)
    return tuple(out)


def q_as_f64(w: synth.Workload, q_stored: np.ndarray) -> np.ndarray:
    return synth.as_f32(q_stored, w.q_dtype).astype(np.float64)


def to_torch_q(q_stored: np.ndarray, dtype: str, device):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(q_stored.view(np.int16)).to(device).view(torch.bfloat16)
    if dtype == "f16":
        return torch.from_numpy(q_stored).to(device)
    return torch.from_numpy(q_stored.astype(np.float32)).to(device)
