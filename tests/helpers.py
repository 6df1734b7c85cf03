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
        # the threaded face gives the single-threaded fit bit for bit (pinned in
        # test_oracle_pins.py), in a fraction of the time
        cb, _ = O.fit_codebook(rows, w.R, w.g, w.n_codes, w.em_iters,
                               lambda r, N, key=key: synth.forgy_indices(w, key, r, N),
                               threads=O.host_threads())
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


# Planted near ties for the encoder (the spec's rule: the two smallest fp32 distances d1 <= d2
# of a decision form a near tie when d2 - d1 <= 1e-5 * d2). One 8-scalar group, residual 0, so
# the distance of an entry is the fp32 fused sum of its squared coordinates; every coordinate
# is an integer and every partial sum stays below 2^24, so each distance is exact:
#   D2  = 1024^2                          = 1048576
#   IN  = 1023^2 + 45^2 + 3^2 + 1 + 1 + 1 = 1048566   (d2 - d1 = 10 <= 10.4858: a near tie)
#   OUT = 1023^2 + 45^2 + 3^2 + 1 + 1     = 1048565   (d2 - d1 = 11 >  10.4858: not one)
#   MID = 1024^2 + 4^2                    = 1048592
#   FAR = 2000^2                          = 4000000
NEAR_TIE_ENTRIES = {
    "D2": [1024, 0, 0, 0, 0, 0, 0, 0],
    "IN": [1023, 45, 3, 1, 1, 1, 0, 0],
    "OUT": [1023, 45, 3, 1, 1, 0, 0, 0],
    "MID": [1024, 4, 0, 0, 0, 0, 0, 0],
    "FAR": [2000, 0, 0, 0, 0, 0, 0, 0],
}
# (entry order in the sub-codebook, expected code, expected near-tie count). The second-best
# distance appears before the best (it must be kept when the best is replaced), after it (it
# must be picked up by the else branch), and is lowered after a farther second (it must be
# replaced by the closer one).
NEAR_TIE_CASES = [
    (("D2", "IN"), 1, 1),
    (("IN", "D2"), 0, 1),
    (("D2", "OUT"), 1, 0),
    (("OUT", "D2"), 0, 0),
    (("IN", "FAR", "MID", "D2"), 0, 1),
    (("FAR", "MID", "IN"), 2, 0),
    (("MID", "D2", "IN"), 2, 1),
]


def near_tie_case(order):
    """Codebook [1, 1, len(order), 8] float32 and one zero row [1, 8] for a planted case."""
    cb = np.array([[[NEAR_TIE_ENTRIES[k] for k in order]]], dtype=np.float32)
    return cb, np.zeros((1, 8), dtype=np.float32)


class Guarded:
    """A device buffer with 256 canary bytes (0xA5) on each side: `t` is the caller's tensor (16-
    and 256-byte alignment kept), `intact()` tells whether the kernels wrote only inside it."""
    PAD = 256
    CANARY = 0xA5

    def __init__(self, shape, dtype, device):
        import torch
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((n + 2 * self.PAD,), self.CANARY, dtype=torch.uint8, device=device)
        self.t = self.raw[self.PAD:self.PAD + n].view(dtype).view(shape)

    def intact(self) -> bool:
        import torch
        r = self.raw
        return bool(torch.all(r[:self.PAD] == self.CANARY).item() and
                    torch.all(r[self.PAD + self.n:] == self.CANARY).item())
