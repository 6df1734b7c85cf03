"""Seeded synthetic inputs shared by the CUDA path, the CPU oracle and the bench.

This module holds workload shapes and random draws only. It contains none of the
method's arithmetic (no distances, no rotary phases, no softmax, no codebook
fitting), so both sides of every parity test can take their inputs from here.

Every draw is ``numpy.random.default_rng([seed, stream, sub])`` (PCG64) followed
by ``standard_normal`` in float64 and one cast to the stated storage type.

Stream ids:
    0  codebooks and codebook-fitting rows (sub 0: key codebook, 1: value
       codebook, 2: key fitting rows, 3: value fitting rows)
    1  key cache rows (sub = sequence index)
    2  value cache rows (sub = sequence index)
    3  decode queries
    4  outlier-channel permutation
    5  ragged sequence lengths
    6  Forgy initial-entry permutations (sub = 2 * tensor + round; tensor 0 = K, 1 = V)
    7  uniform random key codes (full-size attention parity)
    8  uniform random value codes (full-size attention parity)

The workloads follow the CommVQ pages (CommVQ: Commutative Vector Quantization for
KV Cache Compression, "What carries the argument": g consecutive scalars share one
index, R residual rounds, R*log2(Nc')/g bits per scalar) at LLaMA-3.1-8B layer
shape (32 query heads, 8 KV heads, d = 128).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

STREAM_CODEBOOK = 0
STREAM_K = 1
STREAM_V = 2
STREAM_Q = 3
STREAM_OUTLIER = 4
STREAM_LENGTHS = 5
STREAM_FORGY = 6
STREAM_KCODES = 7
STREAM_VCODES = 8

SUB_KCB, SUB_VCB, SUB_KROWS, SUB_VROWS = 0, 1, 2, 3


@dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic workload."""

    name: str
    seed: int
    d: int = 128
    g: int = 8
    R: int = 2
    n_codes: int = 256
    q_heads: int = 32
    kv_heads: int = 8
    rope_base: float = 500000.0
    batch: int = 1
    seq_len: int = 32768               # fixed length (ignored when ragged)
    ragged: Optional[tuple] = None     # (lo, hi) inclusive, per-sequence lengths
    kv_dtype: str = "f16"              # storage type of K/V rows before encoding
    q_dtype: str = "bf16"
    n_outliers: int = 8                # key channels scaled by outlier_scale
    outlier_scale: float = 10.0
    codebook: str = "em"               # "em": fitted; "normal": entries ~ N(0,1)
    em_rows: int = 4096
    em_iters: int = 5                  # per round
    encode_tokens: int = 0             # >0: encode-only workload (tokens x kv_heads rows)
    fit_seed: Optional[int] = None     # seed of the codebook fit and outlier channels
    v_bits: int = 0                    # > 0: values in the binary code with this many rows

    @property
    def cb_seed(self) -> int:
        return self.seed if self.fit_seed is None else self.fit_seed

    @property
    def groups(self) -> int:
        return self.d // self.g

    @property
    def code_bytes(self) -> int:
        return 1 if self.n_codes <= 256 else 2

    def lengths(self) -> np.ndarray:
        """Per-sequence cached lengths T_b (stream 5)."""
        if self.ragged is None:
            return np.full(self.batch, self.seq_len, dtype=np.int64)
        lo, hi = self.ragged
        rng = np.random.default_rng([self.seed, STREAM_LENGTHS, 0])
        return rng.integers(lo, hi, size=self.batch, endpoint=True).astype(np.int64)

    def offsets(self) -> np.ndarray:
        L = self.lengths()
        return np.concatenate([[0], np.cumsum(L)]).astype(np.int64)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The workloads, in order: tiny fp32 case, 2-bit 32K layer, 1-bit 128K layer, ragged batch of
# 16, the encode + codebook-fit workload, the pages' own g = 64 setting at 2 and 1 bits, and
# the binary value code.
WORKLOADS = [
    Workload(name="tiny_fp32_T256_R1_N16", seed=0, R=1, n_codes=16, q_heads=1, kv_heads=1,
             rope_base=10000.0, seq_len=256, kv_dtype="f32", q_dtype="f32", n_outliers=0,
             codebook="normal"),
    Workload(name="llama8b_2bit_T32768", seed=1, R=2, seq_len=32768),
    Workload(name="llama8b_1bit_T131072", seed=2, fit_seed=1, R=1, seq_len=131072),
    Workload(name="llama8b_2bit_batch16_ragged", seed=3, fit_seed=1, R=2, batch=16,
             ragged=(4096, 8192)),
    Workload(name="encode_fit_131072x8", seed=4, R=2, encode_tokens=131072, em_rows=65536,
             em_iters=10),
    # the pages' own hyper-parameters: 64 scalars per index, 64 entries, 21 (2-bit) or 11
    # (1-bit) residual rounds: R * log2(64) / 64 = 1.97 and 1.03 bits per scalar
    Workload(name="pages_g64_2bit_T32768", seed=5, g=64, R=21, n_codes=64, seq_len=32768),
    Workload(name="pages_g64_1bit_T32768", seed=6, fit_seed=5, g=64, R=11, n_codes=64, seq_len=32768),
    # the pages' binary value code (2048 rows over the 1024-dim KV row: 2 bits per scalar) with
    # the 2-bit layer's keys
    Workload(name="llama8b_binv2048_T32768", seed=7, fit_seed=1, R=2, seq_len=32768, v_bits=2048),
]
# The 1-bit layer and the ragged batch take their codebooks (and outlier channels) from
# the 2-bit layer's fit seed: under sequential residual fitting the R=1 codebook is
# round 0 of the same fit on the same rows.


def rng(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), int(sub)])


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (round to nearest even) -> bfloat16 bits (round to nearest even)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def cast(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Cast float64 draws to the storage type. bf16 is returned as uint16 bits."""
    if dtype == "f32":
        return x64.astype(np.float32)
    if dtype == "f16":
        return x64.astype(np.float16)
    if dtype == "bf16":
        return to_bf16_bits(x64)
    raise ValueError(dtype)


def as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float32 view of stored values (f16 and bf16 widen exactly)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x)
    return x.astype(np.float32)


def outlier_channels(w: Workload) -> np.ndarray:
    """The key channels scaled by w.outlier_scale: first n of a seeded permutation of 0..d-1."""
    if w.n_outliers == 0:
        return np.zeros(0, dtype=np.int64)
    perm = rng(w.cb_seed, STREAM_OUTLIER, 0).permutation(w.d)
    return np.sort(perm[: w.n_outliers])


def _rows64(w: Workload, stream: int, sub: int, n: int, key: bool) -> np.ndarray:
    seed = w.cb_seed if stream == STREAM_CODEBOOK else w.seed
    x = rng(seed, stream, sub).standard_normal((n, w.d))
    if key and w.n_outliers:
        x[:, outlier_channels(w)] *= w.outlier_scale
    return x


def kv_rows(w: Workload, key: bool, T: int, sub: int = 0, dtype: Optional[str] = None) -> np.ndarray:
    """Pre-RoPE key (key=True) or value rows for one sequence: [T, kv_heads, d]."""
    stream = STREAM_K if key else STREAM_V
    x = _rows64(w, stream, sub, T * w.kv_heads, key).reshape(T, w.kv_heads, w.d)
    return cast(x, dtype or w.kv_dtype)


def kv_cache_rows(w: Workload, key: bool, dtype: Optional[str] = None) -> np.ndarray:
    """Rows for all sequences concatenated along T: [sum T_b, kv_heads, d]."""
    L = w.lengths()
    parts = [kv_rows(w, key, int(L[b]), sub=b, dtype=dtype) for b in range(w.batch)]
    return np.concatenate(parts, axis=0)


def encode_rows(w: Workload, key: bool, tokens: int, dtype: Optional[str] = None,
                chunk: int = 8192) -> np.ndarray:
    """[tokens, kv_heads, d] rows for the encode workload, drawn in fixed chunks of tokens
    (sub = chunk index) so that any chunk can be regenerated on its own."""
    out = np.empty((tokens, w.kv_heads, w.d), dtype=np.float16 if (dtype or w.kv_dtype) == "f16"
                   else np.float32)
    for ci, t0 in enumerate(range(0, tokens, chunk)):
        n = min(chunk, tokens - t0)
        out[t0:t0 + n] = kv_rows(w, key, n, sub=ci, dtype=dtype)
    return out


def queries(w: Workload) -> np.ndarray:
    """Post-RoPE decode queries [batch, q_heads, d] in w.q_dtype (bf16 as uint16 bits)."""
    x = rng(w.seed, STREAM_Q, 0).standard_normal((w.batch, w.q_heads, w.d))
    return cast(x, w.q_dtype)


def normal_codebook(w: Workload, key: bool) -> np.ndarray:
    """[R, d/g, Nc', g] float32 codebook with entries ~ N(0, 1)."""
    sub = SUB_KCB if key else SUB_VCB
    x = rng(w.cb_seed, STREAM_CODEBOOK, sub).standard_normal((w.R, w.groups, w.n_codes, w.g))
    return x.astype(np.float32)


def fit_rows(w: Workload, key: bool) -> np.ndarray:
    """[em_rows, d] float32 codebook-fitting rows, same distribution as the cache rows
    (cast through the cache's storage type, then widened exactly)."""
    sub = SUB_KROWS if key else SUB_VROWS
    x = _rows64(w, STREAM_CODEBOOK, sub, w.em_rows, key)
    return as_f32(cast(x, w.kv_dtype), w.kv_dtype)


def forgy_indices(w: Workload, key: bool, rnd: int, n_rows: int) -> np.ndarray:
    """Row indices whose sub-vectors seed round `rnd`'s codebook (first Nc' of a permutation)."""
    tensor = 0 if key else 1
    perm = rng(w.cb_seed, STREAM_FORGY, 2 * tensor + rnd).permutation(n_rows)
    if n_rows >= w.n_codes:
        return perm[: w.n_codes].astype(np.int64)
    reps = -(-w.n_codes // n_rows)
    return np.tile(perm, reps)[: w.n_codes].astype(np.int64)


def uniform_codes(w: Workload, key: bool, total_T: int) -> np.ndarray:
    """[total_T, kv_heads, R, d/g] codes drawn uniformly in [0, Nc')."""
    stream = STREAM_KCODES if key else STREAM_VCODES
    c = rng(w.seed, stream, 0).integers(0, w.n_codes, size=(total_T, w.kv_heads, w.R, w.groups))
    return c.astype(np.uint8 if w.code_bytes == 1 else np.uint16)


def value_bits(w: Workload, total_T: int) -> np.ndarray:
    """[total_T, v_bits / 8] uint8 binary value codes, every bit uniform (stream 8, sub 1)."""
    return rng(w.seed, STREAM_VCODES, 1).integers(0, 256, size=(total_T, w.v_bits // 8), dtype=np.uint8)


def binary_value_codebook(w: Workload) -> np.ndarray:
    """C [v_bits, kv_heads * d] float32, entries N(0, 2 / v_bits): with half the bits set a decoded
    value row is ~N(0, 1) per scalar (stream 0, sub 4)."""
    x = rng(w.cb_seed, STREAM_CODEBOOK, 4).standard_normal((w.v_bits, w.kv_heads * w.d))
    return (x * np.sqrt(2.0 / w.v_bits)).astype(np.float32)
