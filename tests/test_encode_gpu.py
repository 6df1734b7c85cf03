"""Encoder parity: CUDA codes must equal the oracle's bit for bit (ties to the lowest
index), with the same near-tie count and the same fp32 residual."""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import oracle_codebooks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _cfg(api, w):
    return api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                      kv_heads=w.kv_heads, rope_base=w.rope_base)


def _run(api, cfg, x_np, cb_np, gpu, residual=False):
    x = torch.from_numpy(x_np).to(gpu)
    cb = torch.from_numpy(cb_np).to(gpu)
    ties = torch.zeros(1, dtype=torch.int64, device=gpu)
    res = torch.empty(x.shape, dtype=torch.float32, device=gpu) if residual else None
    codes = api.encode(cfg, x, cb, near_ties=ties, residual_out=res)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    if cfg.code_bytes == 2:
        c = c.view(np.uint16)
    return c.astype(np.int64), int(ties.item()), (res.cpu().numpy() if residual else None)


def _compare(api, cfg, x_np, cb_np, gpu, residual=True):
    got, ties, res = _run(api, cfg, x_np, cb_np, gpu, residual)
    want, want_ties, want_res = O.encode(x_np, cb_np, want_residual=True)
    assert got.shape == want.shape
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{len(mism)} code mismatches, first at {mism[:5]}"
    assert ties == want_ties
    if residual:
        assert np.array_equal(res.view(np.uint32), want_res.astype(np.float32).view(np.uint32))
    return want_ties


def test_encode_tiny_workload(api, gpu):
    w = synth.WORKLOADS[0]
    kcb, vcb = oracle_codebooks(w)
    cfg = _cfg(api, w)
    for key, cb in ((True, kcb), (False, vcb)):
        x = synth.kv_cache_rows(w, key)          # fp32 rows
        _compare(api, cfg, x, cb, gpu)


@pytest.mark.parametrize("key", [True, False])
def test_encode_2bit_layer_slice(api, gpu, key):
    w = synth.WORKLOADS[1]
    kcb, vcb = oracle_codebooks(w)
    cfg = _cfg(api, w)
    x = synth.kv_rows(w, key, T=1027)            # fp16, ragged tail vs 512-row blocks
    _compare(api, cfg, x, kcb if key else vcb, gpu)


def test_encode_1bit_layer_slice(api, gpu):
    w = synth.WORKLOADS[2]
    kcb, _ = oracle_codebooks(w)
    cfg = _cfg(api, w)
    x = synth.kv_rows(w, True, T=300)
    _compare(api, cfg, x, kcb, gpu)


@pytest.mark.parametrize("key", [True, False])
def test_encode_full_workload_with_its_own_codebooks(api, gpu, key):
    """The encode workload at full size: all 131072 x 8 fp16 rows of K (outlier channels) or V,
    encoded with the workload's own codebooks (the oracle's fit: 10 EM iterations per round on
    65536 rows). The codes of 1000 seeded positions (8000 rows) plus the first and the last
    position equal the oracle's bit for bit, and so do the near-tie count and the residuals of
    those rows encoded on their own."""
    w = synth.WORKLOADS[4]
    kcb, vcb = oracle_codebooks(w)
    cb = kcb if key else vcb
    cfg = _cfg(api, w)
    x = synth.encode_rows(w, key, w.encode_tokens)
    got, _, _ = _run(api, cfg, x, cb, gpu)
    rng = np.random.default_rng(124 + int(key))
    toks = np.sort(rng.choice(np.arange(1, w.encode_tokens - 1), 1000, replace=False))
    toks = np.concatenate([[0], toks, [w.encode_tokens - 1]])
    want, want_ties, want_res = O.encode(x[toks], cb, want_residual=True, threads=O.host_threads())
    assert np.array_equal(got[toks], want)
    sub_codes, sub_ties, sub_res = _run(api, cfg, np.ascontiguousarray(x[toks]), cb, gpu, residual=True)
    assert np.array_equal(sub_codes, want)
    assert sub_ties == want_ties
    assert np.array_equal(sub_res.view(np.uint32), want_res.astype(np.float32).view(np.uint32))


def test_encode_uint16_codes_and_multi_tile(api, gpu):
    rng = np.random.default_rng(7)
    for Nc, R in ((300, 2), (1500, 1), (2, 3)):
        cfg = api.Config(d=64, g=8, R=R, n_codes=Nc, q_heads=1, kv_heads=3)
        cb = rng.standard_normal((R, 8, Nc, 8)).astype(np.float32)
        x = rng.standard_normal((97, 3, 64)).astype(np.float16)
        _compare(api, cfg, x, cb, gpu)


def test_encode_ties_and_duplicates(api, gpu):
    cfg = api.Config(d=16, g=8, R=1, n_codes=8, q_heads=1, kv_heads=1)
    cb = np.zeros((1, 2, 8, 8), dtype=np.float32)
    cb[0, :, 3] = 1.0
    cb[0, :, 6] = 1.0        # duplicate of entry 3
    cb[0, :, 0] = -2.0
    x = np.ones((5, 1, 16), dtype=np.float32)
    t = _compare(api, cfg, x, cb, gpu)
    assert t == 10
    got, _, _ = _run(api, cfg, x, cb, gpu)
    assert np.all(got == 3)


def test_encode_empty(api, gpu):
    w = synth.WORKLOADS[1]
    cfg = _cfg(api, w)
    x = torch.empty((0, 8, 128), dtype=torch.float16, device=gpu)
    cb = torch.zeros((2, 16, 256, 8), dtype=torch.float32, device=gpu)
    codes = api.encode(cfg, x, cb)
    assert codes.shape == (0, 8, 2, 16)


@pytest.mark.parametrize("wi", [1, 5])
@pytest.mark.parametrize("tokens", [1, 3, 40])
def test_few_rows_take_the_warp_encoder(gpu, wi, tokens):
    """A decode step encodes one new position: up to 4096 (row, group) units go through the
    warp-per-unit kernel. Codes, near-tie counts and residuals equal the oracle's, at the
    library's g = 8 (R = 2, 256 entries) and the pages' g = 64 (R = 21, 64 entries)."""
    from decode_attention_commvq_b200 import api
    w = synth.WORKLOADS[wi]
    cfg = api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads, kv_heads=w.kv_heads)
    kcb, _ = oracle_codebooks(w)
    x = synth.kv_rows(w, True, tokens, sub=777, dtype="f16")
    ref, ties, res_ref = O.encode(x, kcb, want_residual=True)
    nt = torch.zeros(1, dtype=torch.int64, device=gpu)
    res = torch.empty(x.shape, dtype=torch.float32, device=gpu)
    codes = api.encode(cfg, torch.from_numpy(x).to(gpu), torch.from_numpy(kcb).to(gpu), near_ties=nt,
                       residual_out=res)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy().astype(np.int64), ref.astype(np.int64))
    assert int(nt.item()) == ties
    assert np.array_equal(res.cpu().numpy(), res_ref)


def test_warp_encoder_ties_and_tiny_codebooks(gpu):
    """Exact ties (duplicated entries) go to the lowest index and count as near ties; fewer
    entries (5) than lanes."""
    from decode_attention_commvq_b200 import api
    rng = np.random.default_rng(97)
    cb = rng.standard_normal((2, 16, 5, 8)).astype(np.float32)
    cb[:, :, 3] = cb[:, :, 1]                       # entries 1 and 3 identical
    x = cb[0, :, 1].reshape(1, 1, 128).astype(np.float32) + 0.0   # row = entry 1 exactly
    cfg = api.Config(d=128, g=8, R=2, n_codes=5, q_heads=1, kv_heads=1)
    nt = torch.zeros(1, dtype=torch.int64, device=gpu)
    codes = api.encode(cfg, torch.from_numpy(x).to(gpu), torch.from_numpy(cb).to(gpu), near_ties=nt)
    torch.cuda.synchronize()
    ref, ties = O.encode(x, cb)
    assert np.array_equal(codes.cpu().numpy().astype(np.int64), ref.astype(np.int64))
    assert int(nt.item()) == ties and ties >= 16
    assert (codes.cpu().numpy()[0, 0, 0] == 1).all()


@pytest.mark.parametrize("rows", [1, 5000])
def test_planted_near_ties(api, gpu, rows):
    """The planted near ties of tests/helpers.py (gaps just inside and just outside 1e-5 * d2,
    second-best distances before, after and lowered after the best) through the warp encoder
    (1 row) and the block encoder (5000 rows, more than 4096 units): the planted code in every
    row and exactly the planted count per row."""
    from tests.helpers import NEAR_TIE_CASES, near_tie_case
    for order, code, ties in NEAR_TIE_CASES:
        cb, x = near_tie_case(order)
        cfg = api.Config(d=8, g=8, R=1, n_codes=len(order), q_heads=1, kv_heads=1)
        xs = np.ascontiguousarray(np.repeat(x.reshape(1, 1, 8), rows, axis=0))
        got, n, _ = _run(api, cfg, xs, cb, gpu)
        assert (got == code).all(), order
        assert n == ties * rows, order


@pytest.mark.parametrize("tokens", [1, 700])
def test_encode_kv_equals_two_encodes(api, gpu, tokens):
    """commvq_encode_kv (key and value rows in one launch; 1 token takes the warp encoder, 700 the
    block encoder) gives the codes and near-tie count of the oracle on each tensor."""
    w = synth.WORKLOADS[1]
    kcb, vcb = oracle_codebooks(w)
    cfg = _cfg(api, w)
    kx = synth.kv_rows(w, True, tokens, sub=555, dtype="f16")
    vx = synth.kv_rows(w, False, tokens, sub=555, dtype="f16")
    kc = torch.empty((tokens, w.kv_heads, w.R, w.groups), dtype=torch.uint8, device=gpu)
    vc = torch.empty_like(kc)
    nt = torch.zeros(1, dtype=torch.int64, device=gpu)
    api.encode_kv(cfg, torch.from_numpy(kx).to(gpu), torch.from_numpy(vx).to(gpu), torch.from_numpy(kcb).to(gpu),
                  torch.from_numpy(vcb).to(gpu), kc, vc, near_ties=nt)
    torch.cuda.synchronize()
    ref_k, tk = O.encode(kx, kcb)
    ref_v, tv = O.encode(vx, vcb)
    assert np.array_equal(kc.cpu().numpy().astype(np.int64), ref_k)
    assert np.array_equal(vc.cpu().numpy().astype(np.int64), ref_v)
    assert int(nt.item()) == tk + tv
