"""Python face of the CommVQ CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg use
this module. It loads ``libcommvq_oracle.so`` (plain C, built with
``-ffp-contract=off``; see ``commvq_oracle.c`` for the definitions and their
sources) and marshals numpy arrays. The codebook-fit driver below strings the C
primitives together in the order the pages give (CommVQ machine review, "What
carries the argument": codebooks fit by EM, R residual rounds).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "commvq_oracle.c")
LIB = os.path.join(HERE, "libcommvq_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c99"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (a test checker, not part of the product)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        _lib.oracle_encode.argtypes = [P, I64, I, I, I, I, P, P, P, P]
        _lib.oracle_decode.argtypes = [P, I64, I, I, I, I, P, P]
        _lib.oracle_scores_plain.argtypes = [P, P, I64, I64, I, ctypes.c_double, P]
        _lib.oracle_scores_table.argtypes = [P, P, I64, I64, I, I, I, I, P, ctypes.c_double, P]
        _lib.oracle_attend.argtypes = [P, P, P, P, I, I, I, I, ctypes.c_double, P, P]
        _lib.oracle_em_step.argtypes = [P, I64, I, I, I, P, P, P]
        _lib.oracle_values_hist.argtypes = [P, P, I64, I64, I, I, I, I, P, P, P]
        _lib.oracle_em_soft_step.argtypes = [P, I64, I, I, I, P, ctypes.c_double, P]
        _lib.oracle_rope.argtypes = [P, P, I64, I, ctypes.c_double, P]
        _lib.oracle_attend_dense.argtypes = [P, P, P, P, I, I, I, I, P, P]
        _lib.oracle_decode_bits.argtypes = [P, I64, I, P, I, P]
        _lib.oracle_em_update.argtypes = [P, I64, I, I, I, P, P]
        for f in ("oracle_encode", "oracle_decode", "oracle_scores_plain", "oracle_scores_table",
                  "oracle_attend", "oracle_em_step", "oracle_values_hist", "oracle_em_soft_step",
                  "oracle_rope", "oracle_attend_dense", "oracle_decode_bits", "oracle_em_update"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def host_threads() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _pieces(n: int, threads: int):
    """[start, stop) ranges splitting n items into at most `threads` contiguous pieces."""
    k = max(1, min(int(threads), n))
    edges = [n * i // k for i in range(k + 1)]
    return [(edges[i], edges[i + 1]) for i in range(k) if edges[i + 1] > edges[i]]


def _run_pieces(fn, pieces):
    """Run fn(a, b) for every piece, on threads when there are several (each call is one
    single-threaded C call on disjoint data; ctypes releases the GIL around it)."""
    if len(pieces) <= 1:
        return [fn(a, b) for a, b in pieces]
    with ThreadPoolExecutor(len(pieces)) as ex:
        return list(ex.map(lambda ab: fn(*ab), pieces))


def encode(x: np.ndarray, cb: np.ndarray, want_residual: bool = False, threads: int = 1):
    """Residual nearest-codeword codes of rows x[..., d] against cb [R, d/g, Nc', g].
    threads > 1 splits the rows into contiguous pieces encoded at once (each row's result does
    not depend on the others, so the output is the same).

    Returns (codes [..., R, d/g] int32, near_tie_count[, residual [..., d] fp32])."""
    R, G, Nc, g = cb.shape
    d = G * g
    lead = x.shape[:-1]
    xf = _c(x.reshape(-1, d).astype(np.float32), np.float32)   # f16 widens exactly
    n = xf.shape[0]
    cbf = _c(cb, np.float32)
    codes = np.empty((n, R, G), dtype=np.int32)
    res = np.empty((n, d), dtype=np.float32) if want_residual else None

    def piece(a, b):   # rows a..b-1: their own codes, residuals and near-tie count
        ties = ctypes.c_int64(0)
        _check(lib().oracle_encode(_p(xf[a:b]), b - a, d, g, R, Nc, _p(cbf), _p(codes[a:b]),
                                   None if res is None else _p(res[a:b]), ctypes.byref(ties)), "encode")
        return int(ties.value)

    ties = sum(_run_pieces(piece, _pieces(n, threads)))
    codes = codes.reshape(*lead, R, G)
    if want_residual:
        return codes, ties, res.reshape(*lead, d)
    return codes, ties


def decode(codes: np.ndarray, cb: np.ndarray) -> np.ndarray:
    """Sum of the selected codewords in fp64: codes [..., R, d/g] -> [..., d]."""
    R, G, Nc, g = cb.shape
    d = G * g
    lead = codes.shape[:-2]
    cc = _c(codes.reshape(-1, R, G), np.int32)
    out = np.empty((cc.shape[0], d), dtype=np.float64)
    _check(lib().oracle_decode(_p(cc), cc.shape[0], d, g, R, Nc, _p(_c(cb, np.float32)), _p(out)),
           "decode")
    return out.reshape(*lead, d)


def scores_plain(q: np.ndarray, keys: np.ndarray, base: float) -> np.ndarray:
    """Plain RoPE scores of one query [d] against decoded keys [T, d] at positions 0..T-1."""
    qd = _c(q, np.float64)
    kd = _c(keys, np.float64)
    T, d = kd.shape
    out = np.empty(T, dtype=np.float64)
    _check(lib().oracle_scores_plain(_p(qd), _p(kd), d, T, d, float(base), _p(out)), "scores_plain")
    return out


def scores_table(q: np.ndarray, codes: np.ndarray, cb: np.ndarray, base: float) -> np.ndarray:
    """Scores of one query [d] through the query x codebook table; codes [T, R, d/g]."""
    R, G, Nc, g = cb.shape
    d = G * g
    cc = _c(codes, np.int32)
    T = cc.shape[0]
    out = np.empty(T, dtype=np.float64)
    _check(lib().oracle_scores_table(_p(_c(q, np.float64)), _p(cc), R * G, T, d, g, R, Nc,
                                     _p(_c(cb, np.float32)), float(base), _p(out)), "scores_table")
    return out


def values_hist(p: np.ndarray, codes: np.ndarray, cb: np.ndarray):
    """Value output through histograms: weights p [T], codes [T, R, d/g].
    Returns (o [d] fp64, H [R, d/g, Nc'] fp64)."""
    R, G, Nc, g = cb.shape
    d = G * g
    cc = _c(codes, np.int32)
    T = cc.shape[0]
    o = np.empty(d, dtype=np.float64)
    H = np.empty((R, G, Nc), dtype=np.float64)
    _check(lib().oracle_values_hist(_p(_c(p, np.float64)), _p(cc), R * G, T, d, g, R, Nc,
                                    _p(_c(cb, np.float32)), _p(H), _p(o)), "values_hist")
    return o, H


def bits_per_scalar(R: int, n_codes: int, g: int) -> float:
    """Average stored bits per scalar, R * log2(Nc') / g (Eq. 21 as the review quotes it)."""
    return R * float(np.log2(n_codes)) / g


def reduction_vs_fp16(bits: float) -> float:
    """Fraction of an FP16 cache saved at `bits` per scalar."""
    return 1.0 - bits / 16.0


def kv_cache_bytes(tokens: int, layers: int, kv_dim: int, batch: int, bits: float) -> float:
    """Bytes of a K+V cache: 2 tensors x batch x tokens x layers x kv_dim x bits / 8."""
    return 2.0 * batch * tokens * layers * kv_dim * bits / 8.0


def attend(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, offsets: np.ndarray,
           base: float):
    """Plain decode attention on decoded caches. q [B, Hq, d]; khat/vhat [sum T, Hkv, d].
    Returns (out [B, Hq, d] fp64, lse [B, Hq] fp64)."""
    B, Hq, d = q.shape
    Hkv = khat.shape[1]
    out = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    _check(lib().oracle_attend(_p(_c(q, np.float64)), _p(_c(khat, np.float64)),
                               _p(_c(vhat, np.float64)), _p(_c(offsets, np.int64)), B, Hq, Hkv, d,
                               float(base), _p(out), _p(lse)), "attend")
    return out, lse


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rows x [n, d] rotated to positions pos [n] (fp64): the key rows a decompress-then-attend
    implementation stores."""
    xd = _c(x, np.float64)
    n, d = xd.shape
    out = np.empty_like(xd)
    _check(lib().oracle_rope(_p(xd), _p(_c(pos, np.int64)), n, d, float(base), _p(out)), "rope")
    return out


def rope_cache(khat: np.ndarray, offsets: np.ndarray, base: float) -> np.ndarray:
    """A decoded key cache [sum T, Hkv, d] rotated row by row to its in-sequence positions."""
    N, Hkv, d = khat.shape
    pos = np.concatenate([np.arange(offsets[b + 1] - offsets[b]) for b in range(len(offsets) - 1)]
                         + [np.zeros(0, np.int64)]).astype(np.int64)
    return rope(khat.reshape(N * Hkv, d), np.repeat(pos, Hkv), base).reshape(N, Hkv, d)


def attend_dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, offsets: np.ndarray):
    """Dense decode attention on keys that already carry their rotation. q [B, Hq, d];
    k/v [sum T, Hkv, d]. Returns (out [B, Hq, d] fp64, lse [B, Hq] fp64)."""
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    out = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    _check(lib().oracle_attend_dense(_p(_c(q, np.float64)), _p(_c(k, np.float64)), _p(_c(v, np.float64)),
                                     _p(_c(offsets, np.int64)), B, Hq, Hkv, d, _p(out), _p(lse)),
           "attend_dense")
    return out, lse


def decode_bits(bits: np.ndarray, C: np.ndarray) -> np.ndarray:
    """The binary value code: bits [T, Nc/8] uint8 (bit n = byte n/8, bit n%8) and value codebook
    C [Nc, dkv] -> rows [T, dkv] fp64, the sum of the rows of C whose bit is set."""
    Nc, dkv = C.shape
    b = _c(bits, np.uint8)
    T = b.shape[0]
    out = np.empty((T, dkv), dtype=np.float64)
    _check(lib().oracle_decode_bits(_p(b), T, Nc, _p(_c(C, np.float32)), dkv, _p(out)), "decode_bits")
    return out


def attend_binv(q: np.ndarray, k_codes: np.ndarray, v_bits: np.ndarray, offsets: np.ndarray,
                kcb: np.ndarray, C: np.ndarray, base: float):
    """Decode attention with CommVQ keys (codes [sum T, Hkv, R, d/g]) and binary values
    (bits [sum T, Nc/8] over all Hkv*d value dims): decode both, then attend."""
    Hkv = k_codes.shape[1]
    d = q.shape[-1]
    vhat = decode_bits(v_bits, C).reshape(-1, Hkv, d)
    return attend(q, decode(k_codes, kcb), vhat, offsets, base)


def attend_codes(q: np.ndarray, k_codes: np.ndarray, v_codes: np.ndarray, offsets: np.ndarray,
                 kcb: np.ndarray, vcb: np.ndarray, base: float, threads: int = 1):
    """Decode attention straight from codes [sum T, Hkv, R, d/g]: decode, then attend.
    threads > 1 attends the KV heads' query groups at once (each (b, h) result is computed on
    its own, so the output is the same)."""
    Hkv = k_codes.shape[1]
    if threads <= 1 or Hkv == 1:
        return attend(q, decode(k_codes, kcb), decode(v_codes, vcb), offsets, base)
    B, Hq, d = q.shape
    G = Hq // Hkv
    out = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)

    def piece(a, b):   # KV heads a..b-1 and their query heads, decoded one head at a time
        for kvh in range(a, b):
            khat = decode(k_codes[:, kvh:kvh + 1], kcb)
            vhat = decode(v_codes[:, kvh:kvh + 1], vcb)
            o, l = attend(q[:, kvh * G:(kvh + 1) * G], khat, vhat, offsets, base)
            out[:, kvh * G:(kvh + 1) * G] = o
            lse[:, kvh * G:(kvh + 1) * G] = l

    _run_pieces(piece, _pieces(Hkv, threads))
    return out, lse


def em_step(rows: np.ndarray, cb_round: np.ndarray):
    """One EM step on residual rows [N, d] for one round's codebook [d/g, Nc', g].
    Returns (new codebook, codes [N, d/g], sse)."""
    G, Nc, g = cb_round.shape
    d = G * g
    rf = _c(rows, np.float32)
    N = rf.shape[0]
    cb = _c(cb_round, np.float32).copy()
    codes = np.empty((N, G), dtype=np.int32)
    sse = ctypes.c_double(0.0)
    _check(lib().oracle_em_step(_p(rf), N, d, g, Nc, _p(cb), _p(codes), ctypes.byref(sse)),
           "em_step")
    return cb, codes, float(sse.value)


def em_soft_step(rows: np.ndarray, cb_round: np.ndarray, tau: float):
    """One soft-assignment EM step at temperature tau. Returns (new codebook, sse)."""
    G, Nc, g = cb_round.shape
    d = G * g
    rf = _c(rows, np.float32)
    cb = _c(cb_round, np.float32).copy()
    sse = ctypes.c_double(0.0)
    _check(lib().oracle_em_soft_step(_p(rf), rf.shape[0], d, g, Nc, _p(cb), float(tau),
                                     ctypes.byref(sse)), "em_soft_step")
    return cb, float(sse.value)


def forgy_init(rows: np.ndarray, idx: np.ndarray, g: int) -> np.ndarray:
    """Round codebook [d/g, Nc', g] whose entry c of group j is sub-vector j of row idx[c]."""
    N, d = rows.shape
    G = d // g
    return np.ascontiguousarray(rows[idx].reshape(len(idx), G, g).transpose(1, 0, 2),
                                dtype=np.float32)


def em_update(rows: np.ndarray, cb_round: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """The EM step's closed-form update on given assignments codes [N, d/g]: a new codebook."""
    G, Nc, g = cb_round.shape
    rf = _c(rows, np.float32)
    cb = _c(cb_round, np.float32).copy()
    _check(lib().oracle_em_update(_p(rf), rf.shape[0], G * g, g, Nc, _p(_c(codes, np.int32)), _p(cb)),
           "em_update")
    return cb


def fit_codebook(rows: np.ndarray, R: int, g: int, n_codes: int, iters: int, init_indices,
                 threads: int = 1):
    """Sequential residual fit: for each round, Forgy init from that round's residual rows,
    `iters` EM steps, then advance the residuals by one encoder round against the final
    codebook. init_indices(r, N) -> row indices. Returns (cb [R, d/g, Nc', g], sse history).
    threads > 1 makes each step's assignments with the threaded encoder (the EM step's own
    rule) and applies the update on them: the same codebooks bit for bit, and no SSE history
    (None)."""
    res = _c(rows, np.float32).copy()
    N, d = res.shape
    rounds, hist = [], []
    for r in range(R):
        cb_r = forgy_init(res, init_indices(r, N), g)
        h = []
        for _ in range(iters):
            if threads > 1:
                codes, _ = encode(res, cb_r[None], threads=threads)
                cb_r = em_update(res, cb_r, codes[:, 0])
            else:
                cb_r, _, sse = em_step(res, cb_r)
                h.append(sse)
        hist.append(h)
        rounds.append(cb_r)
        _, _, res = encode(res, cb_r[None], want_residual=True, threads=threads)
    return np.stack(rounds).astype(np.float32), (hist if threads <= 1 else None)


def time_call(fn, *a, **kw):
    t0 = time.perf_counter()
    out = fn(*a, **kw)
    return out, time.perf_counter() - t0
