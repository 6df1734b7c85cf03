"""CPU checks of the C ABI: the library builds and loads, exports every function the
header declares, and rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "commvq.h")


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import build
    build.build()
    from decode_attention_commvq_b200 import api as A
    return A


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(commvq_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("commvq_encode", "commvq_attend_decode", "commvq_em_step",
              "commvq_attend_workspace_bytes", "commvq_em_workspace_bytes",
              "commvq_workspace_error", "commvq_status_string", "commvq_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(api):
    lib = ctypes.CDLL(api.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(api.EXPORTS) == set(declared_functions())


def test_status_strings_and_version(api):
    assert api.abi_version() == 2
    for s in range(6):
        assert api.status_string(s)
    assert "unknown" in api.status_string(99)


def _cfg(api, **kw):
    base = dict(d=128, g=8, R=2, n_codes=256, q_heads=32, kv_heads=8, rope_base=5e5)
    base.update(kw)
    return api.Config(**base)


FAKE = 0x10000  # a 256-byte-aligned non-null address; never dereferenced by these calls


def _attend(api, cfg, B=1, max_T=100, ws_bytes=1 << 20, q=FAKE, kc=FAKE, vc=FAKE, offs=FAKE,
            kcb=FAKE, vcb=FAKE, out=FAKE, lse=None, ws=FAKE, qdt=2, opts=None):
    cc = cfg.c()
    P = ctypes.c_void_p
    return api.LIB.commvq_attend_decode(ctypes.byref(cc), P(q), qdt, P(kc), P(vc), P(offs), B, max_T,
                                        P(kcb), P(vcb), P(out), P(lse) if lse else None, P(ws),
                                        ws_bytes, ctypes.byref(opts) if opts else None, None)


def test_attend_rejects_bad_arguments(api):
    INVALID, UNSUP, WS = 1, 2, 4
    cfg = _cfg(api)
    assert _attend(api, _cfg(api, q_heads=30)) == INVALID          # Hq % Hkv
    assert _attend(api, _cfg(api, g=7)) == INVALID                  # d % g
    assert _attend(api, _cfg(api, n_codes=0)) == INVALID
    assert _attend(api, _cfg(api, rope_base=-1.0)) == INVALID
    assert _attend(api, _cfg(api, d=64)) == UNSUP
    assert _attend(api, _cfg(api, g=128)) == UNSUP                  # group width
    assert _attend(api, _cfg(api, R=40)) == UNSUP
    assert _attend(api, _cfg(api, n_codes=512), opts=api.CAttendOptions(2, 0)) == UNSUP   # MMA: uint16 codes
    assert _attend(api, _cfg(api, g=64, n_codes=64), opts=api.CAttendOptions(1, 0)) == UNSUP   # table: g = 8 only
    assert _attend(api, cfg, q=0) == INVALID
    assert _attend(api, cfg, q=FAKE + 8) == INVALID                 # misaligned
    assert _attend(api, cfg, ws=FAKE + 16) == INVALID               # workspace alignment
    assert _attend(api, cfg, qdt=7) == INVALID
    assert _attend(api, cfg, B=-1) == INVALID
    assert _attend(api, cfg, ws_bytes=16) == WS
    assert _attend(api, cfg, B=0) == 0                               # no-op
    bad = api.CAttendOptions(4, 0)
    assert _attend(api, cfg, opts=bad) == INVALID
    bad = api.CAttendOptions(0, -2)
    assert _attend(api, cfg, opts=bad) == INVALID


def test_workspace_sizes(api):
    cfg = _cfg(api)
    one = api.attend_workspace_bytes(cfg, 1, 32768, algo=api.ATTN_TABLE, splits=4)
    assert one == 256 + 32 * 4 * 528
    assert api.attend_workspace_bytes(cfg, 16, 8192, algo=api.ATTN_TABLE, splits=1) == 256 + 16 * 32 * 528
    # decode-and-rotate form: partials, two fp16 codebook images, the score buffer
    mma = api.attend_workspace_bytes(cfg, 1, 32768, algo=api.ATTN_DECODE_MMA, splits=148)
    part = 256 + 32 * 148 * 528
    img = 512 * 256
    phase = 64 * 8 + 128 * 64 * 8 + 64 * 8
    want = -(-part // 256) * 256 + 2 * img + -(-phase // 256) * 256 + 32768 * 32 * 4
    assert mma == -(-want // 256) * 256
    assert api.attend_workspace_bytes(cfg, 1, 32768) == api.attend_workspace_bytes(
        cfg, 1, 32768, algo=api.ATTN_DECODE_MMA)
    # shapes the decode-and-rotate form does not take
    assert api.attend_workspace_bytes(_cfg(api, R=3, n_codes=64), 1, 10, algo=api.ATTN_DECODE_MMA) == 0
    assert api.attend_workspace_bytes(_cfg(api, R=3, n_codes=64), 1, 10) > 0   # AUTO -> table
    assert api.attend_workspace_bytes(_cfg(api, q_heads=30), 1, 10) == 0
    em = api.em_workspace_bytes(cfg, 65536)
    assert em >= 32 * 16 * 256 * (8 * 8 + 4)
    assert api.em_workspace_bytes(cfg, 0) == 0
    assert api.em_workspace_bytes(_cfg(api, n_codes=5000), 10) == 0


def test_encode_and_em_reject_bad_arguments(api):
    INVALID, UNSUP = 1, 2
    P = ctypes.c_void_p
    cc = _cfg(api).c()
    enc = api.LIB.commvq_encode
    assert enc(ctypes.byref(cc), P(FAKE), 1, 0, P(FAKE), P(FAKE), None, None, None) == 0   # T = 0
    assert enc(ctypes.byref(cc), None, 1, 5, P(FAKE), P(FAKE), None, None, None) == INVALID
    assert enc(ctypes.byref(cc), P(FAKE + 4), 1, 5, P(FAKE), P(FAKE), None, None, None) == INVALID
    assert enc(ctypes.byref(cc), P(FAKE), 2, 5, P(FAKE), P(FAKE), None, None, None) == UNSUP  # bf16 rows
    c2 = _cfg(api, n_codes=300).c()                  # code_bytes must be 2
    c2.code_bytes = 1
    assert enc(ctypes.byref(c2), P(FAKE), 1, 5, P(FAKE), P(FAKE), None, None, None) == INVALID
    em = api.LIB.commvq_em_step
    assert em(ctypes.byref(cc), P(FAKE), 0, P(FAKE), None, None, P(FAKE), 1 << 30, None) == INVALID
    assert em(ctypes.byref(cc), P(FAKE), 100, P(FAKE), None, None, P(FAKE), 16, None) == 4
    c3 = _cfg(api, n_codes=5000).c()
    assert em(ctypes.byref(c3), P(FAKE), 100, P(FAKE), None, None, P(FAKE), 1 << 30, None) == UNSUP


def test_soft_em_rejects_bad_temperature(api):
    P = ctypes.c_void_p
    cc = _cfg(api).c()
    f = api.LIB.commvq_em_step_soft
    for tau in (0.0, -1.0, float("nan"), float("inf")):
        assert f(ctypes.byref(cc), P(FAKE), 100, P(FAKE), tau, None, P(FAKE), 1 << 30, None) == 1


def _decomp(api, cfg, B=1, max_T=100, kc=FAKE, vc=FAKE, offs=FAKE, kcb=FAKE, vcb=FAKE, odt=2,
            ko=FAKE, vo=FAKE, ws=FAKE, ws_bytes=1 << 24):
    cc = cfg.c()
    P = ctypes.c_void_p
    return api.LIB.commvq_decompress(ctypes.byref(cc), P(kc), P(vc), P(offs), B, max_T, P(kcb), P(vcb),
                                     odt, P(ko), P(vo), P(ws), ws_bytes, None)


def _dense(api, cfg, B=1, max_T=100, q=FAKE, k=FAKE, v=FAKE, kvdt=2, offs=FAKE, out=FAKE, ws=FAKE,
           ws_bytes=1 << 24, opts=None):
    cc = cfg.c()
    P = ctypes.c_void_p
    return api.LIB.commvq_dense_decode(ctypes.byref(cc), P(q), 2, P(k), P(v), kvdt, P(offs), B, max_T,
                                       P(out), None, P(ws), ws_bytes, ctypes.byref(opts) if opts else None,
                                       None)


def test_decompress_and_dense_reject_bad_arguments(api):
    INVALID, UNSUP, WS = 1, 2, 4
    cfg = _cfg(api)
    assert _decomp(api, cfg, B=0) == 0
    assert _decomp(api, cfg, odt=0) == INVALID                       # fp32 output
    assert _decomp(api, cfg, kc=0) == INVALID
    assert _decomp(api, cfg, ko=FAKE + 8) == INVALID                 # misaligned output
    assert _decomp(api, cfg, ws_bytes=1024) == WS
    assert _decomp(api, _cfg(api, R=3)) == UNSUP
    assert _decomp(api, _cfg(api, n_codes=512)) == UNSUP
    assert _decomp(api, _cfg(api, q_heads=12, kv_heads=3)) == UNSUP   # KV heads not in {1,2,4,8}
    assert _decomp(api, cfg, max_T=-1) == INVALID
    assert _dense(api, cfg, B=0) == 0
    assert _dense(api, cfg, kvdt=0) == INVALID                       # fp32 rows
    assert _dense(api, cfg, q=0) == INVALID
    assert _dense(api, cfg, k=FAKE + 4) == INVALID
    assert _dense(api, cfg, ws_bytes=512) == WS
    assert _dense(api, _cfg(api, q_heads=12, kv_heads=3)) == UNSUP   # KV heads not in {1,2,4,8}
    assert _dense(api, _cfg(api, q_heads=32, kv_heads=1)) == UNSUP   # 32 heads per group
    assert _dense(api, cfg, opts=api.CAttendOptions(0, 513)) == INVALID


def test_decompress_and_dense_workspace_sizes(api):
    cfg = _cfg(api)
    img = 2 * 16 * 256 * 16
    want = 256 + 2 * img + 128 * 32 * 16 + 256 * 32 * 16            # header, images, tables
    assert api.decompress_workspace_bytes(cfg, 32768) == want
    assert api.decompress_workspace_bytes(_cfg(api, R=3), 10) == 0
    assert api.dense_decode_workspace_bytes(cfg, 1, 32768, splits=8) == 256 + 32 * 8 * 528
    # 2 KV heads: 4 warps per head write their own partials
    c2 = _cfg(api, q_heads=8, kv_heads=2)
    assert api.dense_decode_workspace_bytes(c2, 2, 1000, splits=3) == 256 + 2 * 8 * 3 * 4 * 528
    assert api.dense_decode_workspace_bytes(_cfg(api, q_heads=12, kv_heads=3), 1, 10) == 0


def test_prepare_rejects_bad_arguments(api):
    INVALID, UNSUP, WS = 1, 2, 4
    P = ctypes.c_void_p
    f = api.LIB.commvq_attend_prepare
    cc = _cfg(api).c()
    assert f(ctypes.byref(cc), 0, 100, P(FAKE), P(FAKE), P(FAKE), 1 << 24, None, None) == 0   # B = 0
    assert f(ctypes.byref(cc), 1, 100, None, P(FAKE), P(FAKE), 1 << 24, None, None) == INVALID
    assert f(ctypes.byref(cc), 1, 100, P(FAKE + 4), P(FAKE), P(FAKE), 1 << 24, None, None) == INVALID
    assert f(ctypes.byref(cc), 1, 100, P(FAKE), P(FAKE), P(FAKE + 16), 1 << 24, None, None) == INVALID
    assert f(ctypes.byref(cc), 1, 100, P(FAKE), P(FAKE), P(FAKE), 64, None, None) == WS
    assert f(ctypes.byref(cc), -1, 100, P(FAKE), P(FAKE), P(FAKE), 1 << 24, None, None) == INVALID
    c5 = _cfg(api, R=40).c()
    assert f(ctypes.byref(c5), 1, 100, P(FAKE), P(FAKE), P(FAKE), 1 << 24, None, None) == UNSUP
    o = api.CAttendOptions(api.ATTN_DECODE_MMA, 0, None, None, 0)
    c3 = _cfg(api, R=3, n_codes=64).c()
    assert f(ctypes.byref(c3), 1, 100, P(FAKE), P(FAKE), P(FAKE), 1 << 24, ctypes.byref(o), None) == UNSUP


def test_generic_algo_workspace(api):
    """The pages' setting (g = 64, Nc' = 64, R = 21) resolves to the generic algorithm: partials
    for every warp of a KV head (8 / KV) plus the phasor tables (128 offsets + one chunk per
    128 positions, 512 B each)."""
    cfg = _cfg(api, g=64, n_codes=64, R=21)
    n = api.attend_workspace_bytes(cfg, 1, 32768, splits=4)
    part = 256 + 32 * 4 * 1 * 528
    want = -(-part // 256) * 256 + (128 + 256) * 512
    assert n == -(-want // 256) * 256
    assert api.attend_workspace_bytes(cfg, 1, 32768, splits=4, algo=api.ATTN_GENERIC) == n
    assert api.attend_workspace_bytes(cfg, 1, 32768, algo=api.ATTN_DECODE_MMA) == 0
    assert api.attend_workspace_bytes(_cfg(api, g=64, n_codes=64, R=21, q_heads=64, kv_heads=2), 1, 10) == 0


def _binv(api, cfg, n_bits=2048, B=1, max_T=100, q=FAKE, qdt=2, kc=FAKE, bits=FAKE, offs=FAKE, kcb=FAKE,
          C=FAKE, out=FAKE, ws=FAKE, ws_bytes=1 << 28, flags=0):
    cc = cfg.c()
    P = ctypes.c_void_p
    return api.LIB.commvq_attend_decode_binv(ctypes.byref(cc), P(q), qdt, P(kc), P(bits), n_bits, P(offs), B,
                                             max_T, P(kcb), P(C), P(out), None, P(ws), ws_bytes, flags, None)


def test_binary_value_code_rejects_bad_arguments(api):
    INVALID, UNSUP, WS = 1, 2, 4
    cfg = _cfg(api)
    assert _binv(api, cfg, B=0) == 0
    assert _binv(api, cfg, n_bits=1000) == UNSUP                     # not a multiple of 1024
    assert _binv(api, cfg, n_bits=9216) == UNSUP                     # above 8192
    assert _binv(api, cfg, n_bits=0) == INVALID
    assert _binv(api, _cfg(api, R=3)) == UNSUP                       # keys off the decode-and-rotate shape
    assert _binv(api, _cfg(api, q_heads=64, kv_heads=8)) == UNSUP    # more than 32 query heads
    assert _binv(api, cfg, qdt=7) == INVALID
    assert _binv(api, cfg, bits=0) == INVALID
    assert _binv(api, cfg, C=FAKE + 4) == INVALID                    # misaligned codebook
    assert _binv(api, cfg, max_T=-1) == INVALID
    assert _binv(api, cfg, ws_bytes=4096) == WS


def test_binary_value_code_workspace_holds_the_key_side_and_the_sums(api):
    """At least the decode-and-rotate workspace plus one split's H [Hq, n_bits] fp32 (the split
    count falls as the bit count grows, so the size need not grow with the bits)."""
    cfg = _cfg(api)
    base = api.attend_workspace_bytes(cfg, 1, 32768, algo=api.ATTN_DECODE_MMA)
    for n_bits in (1024, 2048, 8192):
        assert api.attend_binv_workspace_bytes(cfg, n_bits, 1, 32768) >= base + 32 * n_bits * 4
    assert api.attend_binv_workspace_bytes(cfg, 2048, -1, 10) == 0


def test_copy_rejects_bad_arguments(api):
    f = api.LIB.commvq_copy_async
    P = ctypes.c_void_p
    assert f(P(FAKE), P(FAKE + 4096), 0, None) == 0            # nothing to copy
    assert f(None, P(FAKE), 64, None) == 1                     # null destination
    assert f(P(FAKE), None, 64, None) == 1                     # null source
    assert f(P(FAKE + 8), P(FAKE + 4096), 64, None) == 1       # misaligned destination
    assert f(P(FAKE), P(FAKE + 4104), 64, None) == 1           # misaligned source
    assert f(P(FAKE), P(FAKE + 32), 64, None) == 1             # overlapping ranges
