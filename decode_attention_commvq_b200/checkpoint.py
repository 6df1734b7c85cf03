"""Codebook checkpoints and a resumable sequential codebook fit.

Codebooks are the only state a CommVQ cache carries across calls (one key and one value
codebook per layer, [R, d/g, Nc', g] float32). A fit runs R residual rounds of `iters` EM steps
each (review, "What carries the argument": codebooks fit by EM, residual rounds). This module
stores a fit's progress in a small binary file and resumes it at the (round, iteration) where
it stopped; a resumed fit gives the uninterrupted fit's codebook bit for bit, because every step
is deterministic and the residuals of the finished rounds are recomputed from their codebooks.

File layout (little-endian), 64-byte header then the codebook:
    0  8 bytes  magic b"CMVQCB\\x00\\x01"
    8  u32      format version (1)
   12  u32      d        16 u32 g       20 u32 R (rounds of the full fit)
   24  u32      Nc'      28 u32 rounds_done (rounds whose codebook is final)
   32  u32      iters_done (EM steps applied to round rounds_done's codebook; 0 = not started)
   36  u32      iters (EM steps per round of the fit)
   40  u64      seed (the caller's fit seed, checked on resume)
   48  u32      stored rounds (rounds_done, plus one when iters_done > 0)
   52  12 bytes reserved (zero)
   64  float32  [stored rounds, d/g, Nc', g]
No arithmetic of the method lives here: the fit's steps come from the caller (the library's GPU
calls in fit.py, or any other implementation of the same two steps).
"""
from __future__ import annotations

import os
import struct
from dataclasses import dataclass
from typing import Callable, Optional

import numpy as np

MAGIC = b"CMVQCB\x00\x01"
VERSION = 1
_HEADER = struct.Struct("<8sIIIIIIIIQI12s")
assert _HEADER.size == 64


@dataclass(frozen=True)
class FitState:
    d: int
    g: int
    R: int
    n_codes: int
    rounds_done: int
    iters_done: int
    iters: int
    seed: int

    @property
    def finished(self) -> bool:
        return self.rounds_done >= self.R


def save(path: str, codebook: np.ndarray, state: FitState) -> None:
    """Write `codebook` [stored rounds, d/g, Nc', g] float32 and `state` to path atomically
    (a temporary file in the same directory, then a rename)."""
    cb = np.ascontiguousarray(codebook, dtype=np.float32)
    stored = state.rounds_done + (1 if state.iters_done > 0 and not state.finished else 0)
    want = (stored, state.d // state.g, state.n_codes, state.g)
    if cb.shape != want:
        raise ValueError(f"codebook shape {cb.shape} does not match the state's {want}")
    head = _HEADER.pack(MAGIC, VERSION, state.d, state.g, state.R, state.n_codes, state.rounds_done,
                        state.iters_done, state.iters, state.seed, stored, b"\0" * 12)
    tmp = f"{path}.tmp{os.getpid()}"
    with open(tmp, "wb") as f:
        f.write(head)
        f.write(cb.tobytes())
        f.flush()
        os.fsync(f.fileno())
    os.replace(tmp, path)


def load(path: str):
    """Read a checkpoint: (codebook [stored rounds, d/g, Nc', g] float32, FitState). Raises
    ValueError for a file that is not a checkpoint of this format or whose size is wrong."""
    with open(path, "rb") as f:
        raw = f.read()
    if len(raw) < _HEADER.size:
        raise ValueError(f"{path}: too short for a codebook checkpoint")
    magic, ver, d, g, R, nc, rdone, idone, iters, seed, stored, _ = _HEADER.unpack_from(raw)
    if magic != MAGIC:
        raise ValueError(f"{path}: not a codebook checkpoint (bad magic)")
    if ver != VERSION:
        raise ValueError(f"{path}: format version {ver}, this reader knows {VERSION}")
    if g <= 0 or d <= 0 or d % g or R <= 0 or nc <= 0 or rdone > R or idone > iters:
        raise ValueError(f"{path}: inconsistent header (d={d}, g={g}, R={R}, Nc'={nc}, "
                         f"rounds_done={rdone}, iters_done={idone}, iters={iters})")
    state = FitState(d, g, R, nc, rdone, idone, iters, seed)
    want_stored = rdone + (1 if idone > 0 and rdone < R else 0)
    if stored != want_stored:
        raise ValueError(f"{path}: {stored} stored rounds, the header implies {want_stored}")
    n = stored * (d // g) * nc * g
    if len(raw) != _HEADER.size + 4 * n:
        raise ValueError(f"{path}: {len(raw) - _HEADER.size} data bytes, expected {4 * n}")
    cb = np.frombuffer(raw, dtype="<f4", offset=_HEADER.size, count=n).reshape(stored, d // g, nc, g).copy()
    return cb, state


@dataclass
class FitSteps:
    """The two steps of a sequential fit, on whatever arrays the implementation uses:
    em_step(residual_rows, round_codebook) -> the round codebook after one EM step;
    advance(residual_rows, round_codebook) -> the residual rows after one encoder round;
    seed_round(residual_rows, r) -> the round's initial codebook (e.g. Forgy);
    to_numpy / from_numpy convert a round codebook for the checkpoint file."""
    em_step: Callable
    advance: Callable
    seed_round: Callable
    to_numpy: Callable
    from_numpy: Callable


def resumable_fit(rows, R: int, g: int, n_codes: int, iters: int, steps: FitSteps, path: Optional[str] = None,
                  seed: int = 0, on_step: Optional[Callable[[int, int], None]] = None):
    """Sequential residual fit of R rounds x iters EM steps, saved to `path` after every step and
    resumed from it when it holds a checkpoint of the same (d, g, R, Nc', iters, seed). Returns the
    list of R round codebooks (in the steps' array type). on_step(r, it) is called after each EM
    step has been saved (a hook for callers; tests use it to interrupt a fit)."""
    d = int(rows.shape[1])
    G = d // g
    done, r0, it0, partial = [], 0, 0, None
    if path and os.path.exists(path):
        cb, st = load(path)
        if (st.d, st.g, st.R, st.n_codes, st.iters, st.seed) != (d, g, R, n_codes, iters, seed):
            raise ValueError(f"{path}: checkpoint of another fit ({st}), not d={d}, g={g}, R={R}, "
                             f"Nc'={n_codes}, iters={iters}, seed={seed}")
        done = [steps.from_numpy(cb[r]) for r in range(st.rounds_done)]
        r0, it0 = st.rounds_done, st.iters_done
        if it0 > 0 and r0 < R:
            partial = steps.from_numpy(cb[r0])
    res = rows
    for cb_r in done:                       # residuals of the finished rounds, recomputed
        res = steps.advance(res, cb_r)

    def snapshot(rounds_done, iters_done, current):
        if not path:
            return
        arrs = [steps.to_numpy(c) for c in done]
        if current is not None:
            arrs.append(steps.to_numpy(current))
        cb = np.stack(arrs) if arrs else np.zeros((0, G, n_codes, g), dtype=np.float32)
        save(path, cb, FitState(d, g, R, n_codes, rounds_done, iters_done, iters, seed))

    for r in range(r0, R):
        if r == r0 and partial is not None:
            cb_r, it_start = partial, it0
        else:
            cb_r, it_start = steps.seed_round(res, r), 0
        for it in range(it_start, iters):
            cb_r = steps.em_step(res, cb_r)
            if it + 1 < iters:
                snapshot(r, it + 1, cb_r)
            else:
                done.append(cb_r)
                snapshot(r + 1, 0, None)
            if on_step:
                on_step(r, it)
        if iters == 0:
            done.append(cb_r)
            snapshot(r + 1, 0, None)
        res = steps.advance(res, cb_r)
    return done
