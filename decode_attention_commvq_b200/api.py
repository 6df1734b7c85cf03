"""ctypes binding of libcommvq_b200.so (the C ABI declared in include/commvq.h).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels. PyTorch supplies device memory and the current stream. There is no CPU
fallback: if the shared library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcommvq_b200.so")

F32, F16, BF16 = 0, 1, 2
ATTN_AUTO, ATTN_TABLE, ATTN_DECODE_MMA, ATTN_GENERIC = 0, 1, 2, 3
ATTEND_PREPARED = 1

STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "WORKSPACE", 5: "DEVICE_CHECK"}

EXPORTS = ("commvq_encode", "commvq_encode_kv", "commvq_attend_workspace_bytes", "commvq_attend_decode", "commvq_attend_prepare",
           "commvq_attend_decode_noalloc", "commvq_em_workspace_bytes", "commvq_em_step",
           "commvq_em_step_soft", "commvq_decompress_workspace_bytes", "commvq_decompress",
           "commvq_dense_decode_workspace_bytes", "commvq_dense_decode",
           "commvq_attend_binv_workspace_bytes", "commvq_attend_decode_binv",
           "commvq_copy_async", "commvq_workspace_error", "commvq_status_string", "commvq_abi_version")


class CConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("g", ctypes.c_int32), ("R", ctypes.c_int32),
                ("n_codes", ctypes.c_int32), ("q_heads", ctypes.c_int32),
                ("kv_heads", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("code_bytes", ctypes.c_int32)]


class CAttendOptions(ctypes.Structure):
    _fields_ = [("algo", ctypes.c_int32), ("splits", ctypes.c_int32),
                ("main_start", ctypes.c_void_p), ("main_stop", ctypes.c_void_p),
                ("flags", ctypes.c_int32)]


class CommVQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status_string(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m decode_attention_commvq_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    CP = ctypes.POINTER(CConfig)
    OP = ctypes.POINTER(CAttendOptions)
    lib.commvq_encode.argtypes = [CP, P, I32, I64, P, P, P, P, P]
    lib.commvq_encode.restype = I32
    lib.commvq_encode_kv.argtypes = [CP, P, P, I32, I64, P, P, P, P, P, P]
    lib.commvq_encode_kv.restype = I32
    lib.commvq_attend_workspace_bytes.argtypes = [CP, I32, I64, OP]
    lib.commvq_attend_workspace_bytes.restype = SZ
    lib.commvq_attend_decode.argtypes = [CP, P, I32, P, P, P, I32, I64, P, P, P, P, P, SZ, OP, P]
    lib.commvq_attend_decode.restype = I32
    lib.commvq_attend_prepare.argtypes = [CP, I32, I64, P, P, P, SZ, OP, P]
    lib.commvq_attend_prepare.restype = I32
    lib.commvq_attend_decode_noalloc.argtypes = [CP, P, I32, P, P, P, I32, I64, P, P, P, P, OP, P]
    lib.commvq_attend_decode_noalloc.restype = I32
    lib.commvq_em_workspace_bytes.argtypes = [CP, I64]
    lib.commvq_em_workspace_bytes.restype = SZ
    lib.commvq_em_step.argtypes = [CP, P, I64, P, P, P, P, SZ, P]
    lib.commvq_em_step.restype = I32
    lib.commvq_em_step_soft.argtypes = [CP, P, I64, P, ctypes.c_float, P, P, SZ, P]
    lib.commvq_em_step_soft.restype = I32
    lib.commvq_decompress_workspace_bytes.argtypes = [CP, I64]
    lib.commvq_decompress_workspace_bytes.restype = SZ
    lib.commvq_decompress.argtypes = [CP, P, P, P, I32, I64, P, P, I32, P, P, P, SZ, P]
    lib.commvq_decompress.restype = I32
    lib.commvq_dense_decode_workspace_bytes.argtypes = [CP, I32, I64, OP]
    lib.commvq_dense_decode_workspace_bytes.restype = SZ
    lib.commvq_dense_decode.argtypes = [CP, P, I32, P, P, I32, P, I32, I64, P, P, P, SZ, OP, P]
    lib.commvq_dense_decode.restype = I32
    lib.commvq_attend_binv_workspace_bytes.argtypes = [CP, I32, I32, I64]
    lib.commvq_attend_binv_workspace_bytes.restype = SZ
    lib.commvq_attend_decode_binv.argtypes = [CP, P, I32, P, P, I32, P, I32, I64, P, P, P, P, P, SZ, I32, P]
    lib.commvq_attend_decode_binv.restype = I32
    lib.commvq_copy_async.argtypes = [P, P, SZ, P]
    lib.commvq_copy_async.restype = I32
    lib.commvq_workspace_error.argtypes = [P, ctypes.POINTER(I32), P]
    lib.commvq_workspace_error.restype = I32
    lib.commvq_status_string.argtypes = [I32]
    lib.commvq_status_string.restype = ctypes.c_char_p
    lib.commvq_abi_version.argtypes = []
    lib.commvq_abi_version.restype = I32
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.commvq_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != 0:
        raise CommVQError(status, what)


@dataclass(frozen=True)
class Config:
    d: int = 128
    g: int = 8
    R: int = 2
    n_codes: int = 256
    q_heads: int = 32
    kv_heads: int = 8
    rope_base: float = 500000.0

    @property
    def code_bytes(self) -> int:
        return 1 if self.n_codes <= 256 else 2

    @property
    def groups(self) -> int:
        return self.d // self.g

    def c(self) -> CConfig:
        return CConfig(self.d, self.g, self.R, self.n_codes, self.q_heads, self.kv_heads,
                       float(self.rope_base), self.code_bytes)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


_DT = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}


def code_dtype(cfg: Config):
    return torch.uint8 if cfg.code_bytes == 1 else torch.int16


def encode(cfg: Config, x: torch.Tensor, codebook: torch.Tensor, codes: Optional[torch.Tensor] = None,
           near_ties: Optional[torch.Tensor] = None, residual_out: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """commvq_encode: x [T, kv_heads, d] f16/f32 -> codes [T, kv_heads, R, d/g]."""
    T = x.shape[0]
    if codes is None:
        codes = torch.empty((T, cfg.kv_heads, cfg.R, cfg.groups), dtype=code_dtype(cfg),
                            device=x.device)
    cc = cfg.c()
    _check(LIB.commvq_encode(ctypes.byref(cc), _ptr(x), _DT[x.dtype], T, _ptr(codebook),
                             _ptr(codes), _ptr(near_ties), _ptr(residual_out), _stream(stream)),
           "commvq_encode")
    return codes


def encode_kv(cfg: Config, k_x: torch.Tensor, v_x: torch.Tensor, k_codebook: torch.Tensor,
              v_codebook: torch.Tensor, k_codes: torch.Tensor, v_codes: torch.Tensor,
              near_ties: Optional[torch.Tensor] = None, stream=None):
    """commvq_encode_kv: the key rows k_x and value rows v_x [T, kv_heads, d] (same shape and dtype)
    into k_codes / v_codes [T, kv_heads, R, d/g] in one launch."""
    if k_x.shape != v_x.shape or k_x.dtype != v_x.dtype:
        raise ValueError("k_x and v_x must have the same shape and dtype")
    cc = cfg.c()
    _check(LIB.commvq_encode_kv(ctypes.byref(cc), _ptr(k_x), _ptr(v_x), _DT[k_x.dtype], int(k_x.shape[0]),
                                _ptr(k_codebook), _ptr(v_codebook), _ptr(k_codes), _ptr(v_codes), _ptr(near_ties),
                                _stream(stream)), "commvq_encode_kv")
    return k_codes, v_codes


def _opts(algo: int, splits: int, events=None, flags: int = 0) -> CAttendOptions:
    o = CAttendOptions(int(algo), int(splits), None, None, int(flags))
    if events is not None:
        o.main_start = ctypes.c_void_p(events[0].cuda_event)
        o.main_stop = ctypes.c_void_p(events[1].cuda_event)
    return o


def attend_workspace_bytes(cfg: Config, B: int, max_T: int, algo: int = ATTN_AUTO, splits: int = 0) -> int:
    cc = cfg.c()
    o = _opts(algo, splits)
    return int(LIB.commvq_attend_workspace_bytes(ctypes.byref(cc), int(B), int(max_T), ctypes.byref(o)))


def attend_workspace(cfg: Config, B: int, max_T: int, device, algo: int = ATTN_AUTO, splits: int = 0):
    n = attend_workspace_bytes(cfg, B, max_T, algo, splits)
    if n == 0:
        raise CommVQError(1, "commvq_attend_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def attend_decode(cfg: Config, q: torch.Tensor, k_codes: torch.Tensor, v_codes: torch.Tensor,
                  seq_offsets: torch.Tensor, max_T: int, k_codebook: torch.Tensor,
                  v_codebook: torch.Tensor, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  algo: int = ATTN_AUTO, splits: int = 0, want_lse: bool = True, stream=None,
                  main_events=None, prepared: bool = False):
    """commvq_attend_decode: returns (out [B, q_heads, d] f32, lse [B, q_heads] f32 or None).
    main_events: optional (start, stop) torch.cuda.Event pair recorded around the main kernel.
    prepared: the workspace holds this layer's prepared state (attend_prepare)."""
    B = q.shape[0]
    if out is None:
        out = torch.empty((B, cfg.q_heads, cfg.d), dtype=torch.float32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.q_heads), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = attend_workspace(cfg, B, max_T, q.device, algo, splits)
    cc = cfg.c()
    o = _opts(algo, splits, main_events, ATTEND_PREPARED if prepared else 0)
    _check(LIB.commvq_attend_decode(ctypes.byref(cc), _ptr(q), _DT[q.dtype], _ptr(k_codes),
                                    _ptr(v_codes), _ptr(seq_offsets), int(B), int(max_T),
                                    _ptr(k_codebook), _ptr(v_codebook), _ptr(out), _ptr(lse),
                                    _ptr(workspace), workspace.numel(), ctypes.byref(o),
                                    _stream(stream)), "commvq_attend_decode")
    return out, lse


def attend_prepare(cfg: Config, B: int, max_T: int, k_codebook: torch.Tensor, v_codebook: torch.Tensor,
                   workspace: torch.Tensor, algo: int = ATTN_AUTO, splits: int = 0, stream=None):
    """commvq_attend_prepare: writes the codebook-dependent state into the workspace once, for
    later attend_decode(..., prepared=True) calls with the same shapes and codebooks."""
    cc = cfg.c()
    o = _opts(algo, splits)
    _check(LIB.commvq_attend_prepare(ctypes.byref(cc), int(B), int(max_T), _ptr(k_codebook), _ptr(v_codebook),
                                     _ptr(workspace), workspace.numel(), ctypes.byref(o), _stream(stream)),
           "commvq_attend_prepare")
    return workspace


def attend_decode_noalloc(cfg: Config, q: torch.Tensor, k_codes: torch.Tensor, v_codes: torch.Tensor,
                          seq_offsets: torch.Tensor, max_T: int, k_codebook: torch.Tensor,
                          v_codebook: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                          algo: int = ATTN_AUTO, splits: int = 0, stream=None, prepared: bool = False):
    """commvq_attend_decode_noalloc: the library's fixed internal scratch instead of a
    workspace (for callers that cannot allocate device memory). out/lse are caller-owned."""
    cc = cfg.c()
    o = _opts(algo, splits, None, ATTEND_PREPARED if prepared else 0)
    _check(LIB.commvq_attend_decode_noalloc(ctypes.byref(cc), _ptr(q), _DT[q.dtype], _ptr(k_codes),
                                            _ptr(v_codes), _ptr(seq_offsets), int(q.shape[0]),
                                            int(max_T), _ptr(k_codebook), _ptr(v_codebook), _ptr(out),
                                            _ptr(lse), ctypes.byref(o), _stream(stream)),
           "commvq_attend_decode_noalloc")
    return out, lse


def em_workspace_bytes(cfg: Config, N: int) -> int:
    cc = cfg.c()
    return int(LIB.commvq_em_workspace_bytes(ctypes.byref(cc), int(N)))


def em_step(cfg: Config, rows: torch.Tensor, codebook_round: torch.Tensor,
            codes_out: Optional[torch.Tensor] = None, sse_out: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None):
    """commvq_em_step: updates codebook_round [d/g, Nc', g] in place."""
    N = rows.shape[0]
    if workspace is None:
        n = em_workspace_bytes(cfg, N)
        if n == 0:
            raise CommVQError(1, "commvq_em_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=rows.device)
    cc = cfg.c()
    _check(LIB.commvq_em_step(ctypes.byref(cc), _ptr(rows), int(N), _ptr(codebook_round),
                              _ptr(codes_out), _ptr(sse_out), _ptr(workspace), workspace.numel(),
                              _stream(stream)), "commvq_em_step")
    return codebook_round


def em_step_soft(cfg: Config, rows: torch.Tensor, codebook_round: torch.Tensor, tau: float,
                 sse_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None):
    """commvq_em_step_soft: soft-assignment EM step at temperature tau, in place."""
    N = rows.shape[0]
    if workspace is None:
        n = em_workspace_bytes(cfg, N)
        if n == 0:
            raise CommVQError(1, "commvq_em_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=rows.device)
    cc = cfg.c()
    _check(LIB.commvq_em_step_soft(ctypes.byref(cc), _ptr(rows), int(N), _ptr(codebook_round),
                                   float(tau), _ptr(sse_out), _ptr(workspace), workspace.numel(),
                                   _stream(stream)), "commvq_em_step_soft")
    return codebook_round


def decompress_workspace_bytes(cfg: Config, max_T: int) -> int:
    cc = cfg.c()
    return int(LIB.commvq_decompress_workspace_bytes(ctypes.byref(cc), int(max_T)))


def decompress(cfg: Config, k_codes: torch.Tensor, v_codes: torch.Tensor, seq_offsets: torch.Tensor,
               max_T: int, k_codebook: torch.Tensor, v_codebook: torch.Tensor,
               out_dtype=torch.bfloat16, k_out: Optional[torch.Tensor] = None,
               v_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None):
    """commvq_decompress: codes [total_T, kv_heads, R, d/g] -> dense rows (k rotated, v),
    each [total_T, kv_heads, d] of out_dtype (bf16 or f16)."""
    N = k_codes.shape[0]
    shape = (N, cfg.kv_heads, cfg.d)
    if k_out is None:
        k_out = torch.empty(shape, dtype=out_dtype, device=k_codes.device)
    if v_out is None:
        v_out = torch.empty(shape, dtype=out_dtype, device=k_codes.device)
    if workspace is None:
        n = decompress_workspace_bytes(cfg, max_T)
        if n == 0:
            raise CommVQError(1, "commvq_decompress_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=k_codes.device)
    cc = cfg.c()
    _check(LIB.commvq_decompress(ctypes.byref(cc), _ptr(k_codes), _ptr(v_codes), _ptr(seq_offsets),
                                 int(seq_offsets.numel() - 1), int(max_T), _ptr(k_codebook),
                                 _ptr(v_codebook), _DT[k_out.dtype], _ptr(k_out), _ptr(v_out),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "commvq_decompress")
    return k_out, v_out


def dense_decode_workspace_bytes(cfg: Config, B: int, max_T: int, splits: int = 0) -> int:
    cc = cfg.c()
    o = _opts(ATTN_AUTO, splits)
    return int(LIB.commvq_dense_decode_workspace_bytes(ctypes.byref(cc), int(B), int(max_T), ctypes.byref(o)))


def dense_decode(cfg: Config, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_offsets: torch.Tensor,
                 max_T: int, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, splits: int = 0, want_lse: bool = True,
                 stream=None, main_events=None):
    """commvq_dense_decode over dense rows k, v [total_T, kv_heads, d] (bf16 or f16; keys
    already rotated). Returns (out [B, q_heads, d] f32, lse [B, q_heads] f32 or None)."""
    B = q.shape[0]
    if out is None:
        out = torch.empty((B, cfg.q_heads, cfg.d), dtype=torch.float32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.q_heads), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = dense_decode_workspace_bytes(cfg, B, max_T, splits)
        if n == 0:
            raise CommVQError(1, "commvq_dense_decode_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    cc = cfg.c()
    o = _opts(ATTN_AUTO, splits, main_events)
    _check(LIB.commvq_dense_decode(ctypes.byref(cc), _ptr(q), _DT[q.dtype], _ptr(k), _ptr(v), _DT[k.dtype],
                                   _ptr(seq_offsets), int(B), int(max_T), _ptr(out), _ptr(lse),
                                   _ptr(workspace), workspace.numel(), ctypes.byref(o), _stream(stream)),
           "commvq_dense_decode")
    return out, lse


def attend_binv_workspace_bytes(cfg: Config, n_bits: int, B: int, max_T: int) -> int:
    cc = cfg.c()
    return int(LIB.commvq_attend_binv_workspace_bytes(ctypes.byref(cc), int(n_bits), int(B), int(max_T)))


def attend_decode_binv(cfg: Config, q: torch.Tensor, k_codes: torch.Tensor, v_bits: torch.Tensor,
                       seq_offsets: torch.Tensor, max_T: int, k_codebook: torch.Tensor, v_codebook: torch.Tensor,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, want_lse: bool = True, prepared: bool = False,
                       stream=None):
    """commvq_attend_decode_binv: CommVQ keys, binary values v_bits [total_T, n_bits/8] uint8
    with codebook C [n_bits, kv_heads * d]. prepared: the workspace holds the key side's state
    from an earlier call with the same cfg, B, max_T and key codebook. Returns (out, lse)."""
    if prepared and workspace is None:
        raise ValueError("prepared=True needs the workspace of an earlier call")
    B = q.shape[0]
    n_bits = v_codebook.shape[0]
    if out is None:
        out = torch.empty((B, cfg.q_heads, cfg.d), dtype=torch.float32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, cfg.q_heads), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = attend_binv_workspace_bytes(cfg, n_bits, B, max_T)
        if n == 0:
            raise CommVQError(2, "commvq_attend_binv_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    cc = cfg.c()
    _check(LIB.commvq_attend_decode_binv(ctypes.byref(cc), _ptr(q), _DT[q.dtype], _ptr(k_codes), _ptr(v_bits),
                                         int(n_bits), _ptr(seq_offsets), int(B), int(max_T), _ptr(k_codebook),
                                         _ptr(v_codebook), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                         ATTEND_PREPARED if prepared else 0, _stream(stream)),
           "commvq_attend_decode_binv")
    return out, lse


def copy_async(dst: torch.Tensor, src: torch.Tensor, stream=None):
    """commvq_copy_async: src's bytes into dst by one kernel; either tensor may be device memory or
    pinned host memory that the device maps at its host address (see host_mapped)."""
    n = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < n:
        raise ValueError("dst is smaller than src")
    _check(LIB.commvq_copy_async(_ptr(dst), _ptr(src), n, _stream(stream)), "commvq_copy_async")
    return dst


def host_mapped(t: torch.Tensor) -> bool:
    """Whether pinned host tensor t is device-accessible at its host address (mapped pinned memory
    under unified addressing), as the CUDA runtime reports it."""
    if t.is_cuda or not t.is_pinned():
        return False
    try:
        from cuda.bindings import runtime as rt
    except Exception:
        return False
    err, dptr = rt.cudaHostGetDevicePointer(t.data_ptr(), 0)
    return err == rt.cudaError_t.cudaSuccess and int(dptr) == t.data_ptr()


def workspace_error(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(0)
    st = LIB.commvq_workspace_error(_ptr(workspace), ctypes.byref(v), _stream(stream))
    if st not in (0, 5):
        raise CommVQError(st, "commvq_workspace_error")
    return int(v.value)


def abi_version() -> int:
    return int(LIB.commvq_abi_version())
