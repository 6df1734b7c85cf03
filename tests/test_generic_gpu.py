"""The pages' own hyper-parameters (CommVQ review, "Assumptions & free parameters": g = 64
scalars per index, Nc' = 64 entries, R = 21 rounds for 2 bits and 11 for 1 bit): the encoder and
the hard EM step against the oracle bit for bit, and the GENERIC attention algorithm against
the oracle's attention from codes; GENERIC also on the library's g = 8 workloads and with
two-byte codes.

GENERIC decodes, rotates and accumulates in fp32, so its bound is fp32's, not the fp16 bound of
the fast forms. A decoded row's R fp32 additions err by <= R * 2^-24 of the summed entry
magnitudes (~1.3e-6 at R = 21), the fp64-derived phasors by a few 2^-24, the 128-term dot by
<= ~8 * 2^-24 of sum |q_i k_i|. With keys whose outlier channels are 10x, sum |q_i k_i| / sqrt d
reaches ~50, so a score moves by <= ~1e-4 and a softmax-weighted output by a relative
<= ~2e-4. The bound below, 5e-4, keeps a 2.5x margin."""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import oracle_codebooks, q_as_f64, rel_err, to_torch_q

pytestmark = pytest.mark.gpu

TOL_GENERIC = 5e-4
GENERIC = 3


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _cfg(api, w):
    return api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                      kv_heads=w.kv_heads, rope_base=w.rope_base)


def _codes_gpu(c, w, gpu):
    dt = np.uint8 if w.code_bytes == 1 else np.int16
    return torch.from_numpy(np.ascontiguousarray(c.astype(np.int64).astype(dt))).to(gpu)


@pytest.mark.parametrize("wi", [5, 6])
def test_encoder_pages_setting_bit_exact(api, gpu, wi):
    """512 positions x 8 KV heads of keys (with outlier channels) and values through the GPU
    encoder and the oracle: identical codes, near-tie counts and residuals."""
    w = synth.WORKLOADS[wi].with_(seq_len=512)
    cfg = _cfg(api, w)
    kcb, vcb = oracle_codebooks(synth.WORKLOADS[wi])
    for key, cb in ((True, kcb), (False, vcb)):
        x = synth.kv_cache_rows(w, key)                        # [512, 8, 128] fp16
        ref, ties = O.encode(x, cb)
        res_ref = O.encode(x, cb, want_residual=True)[2]
        xt = torch.from_numpy(x).to(gpu)
        nt = torch.zeros(1, dtype=torch.int64, device=gpu)
        res = torch.empty(x.shape, dtype=torch.float32, device=gpu)
        codes = api.encode(cfg, xt, torch.from_numpy(cb).to(gpu), near_ties=nt, residual_out=res)
        torch.cuda.synchronize()
        assert np.array_equal(codes.cpu().numpy().astype(np.int64), ref.astype(np.int64))
        assert int(nt.item()) == ties
        assert np.array_equal(res.cpu().numpy(), res_ref)


@pytest.mark.parametrize("g", [16, 32, 64])
def test_encoder_other_group_widths(api, gpu, g):
    """Normal codebooks, 4 rounds, 100 entries, fp32 rows: bit-exact codes at g = 16, 32, 64."""
    rng = np.random.default_rng(80 + g)
    R, Nc, d = 4, 100, 128
    cb = rng.standard_normal((R, d // g, Nc, g)).astype(np.float32)
    x = rng.standard_normal((300, 2, d)).astype(np.float32)
    cfg = api.Config(d=d, g=g, R=R, n_codes=Nc, q_heads=2, kv_heads=2)
    codes = api.encode(cfg, torch.from_numpy(x).to(gpu), torch.from_numpy(cb).to(gpu))
    torch.cuda.synchronize()
    ref, _ = O.encode(x, cb)
    assert np.array_equal(codes.cpu().numpy().astype(np.int64), ref.astype(np.int64))


def test_em_step_pages_setting(api, gpu):
    """One hard EM step at g = 64, Nc' = 64 on the 2-bit setting's key fitting rows: the
    oracle's assignments, entries within 1 ulp (fp64 sums in another order), SSE to 1e-12."""
    w = synth.WORKLOADS[5]
    cfg = _cfg(api, w)
    rows = synth.fit_rows(w, True)
    cb0 = O.forgy_init(rows, synth.forgy_indices(w, True, 0, rows.shape[0]), w.g)
    cb = torch.from_numpy(cb0.copy()).to(gpu)
    codes = torch.empty((rows.shape[0], w.d // w.g), dtype=torch.uint8, device=gpu)
    sse = torch.zeros(1, dtype=torch.float64, device=gpu)
    api.em_step(cfg, torch.from_numpy(rows).to(gpu), cb, codes_out=codes, sse_out=sse)
    torch.cuda.synchronize()
    cb_o, codes_o, sse_o = O.em_step(rows, cb0)
    assert np.array_equal(codes.cpu().numpy().astype(np.int64), codes_o.astype(np.int64))
    ia = cb.cpu().numpy().view(np.int32).astype(np.int64)
    ib = cb_o.astype(np.float32).view(np.int32).astype(np.int64)
    assert np.abs(ia - ib).max() <= 1
    assert abs(float(sse.item()) - sse_o) <= 1e-12 * abs(sse_o)


def _attend(api, w, q_np, kc, vc, offs, kcb, vcb, gpu, algo=GENERIC, splits=0):
    cfg = _cfg(api, w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    max_T = int(np.diff(offs).max())
    out, lse = api.attend_decode(cfg, q, _codes_gpu(kc, w, gpu), _codes_gpu(vc, w, gpu), offsets, max_T,
                                 torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu),
                                 algo=algo, splits=splits)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("wi", [5, 6])
@pytest.mark.parametrize("splits", [0, 3])
def test_generic_pages_setting(api, gpu, wi, splits):
    """2048 encoded positions at g = 64, Nc' = 64, R = 21 / 11; all 32 heads; AUTO resolves to
    GENERIC for this shape."""
    w = synth.WORKLOADS[wi].with_(seq_len=2048)
    kcb, vcb = oracle_codebooks(synth.WORKLOADS[wi])
    kc, _ = O.encode(synth.kv_cache_rows(w, True), kcb)
    vc, _ = O.encode(synth.kv_cache_rows(w, False), vcb)
    q = synth.queries(w)
    offs = w.offsets()
    out, lse = _attend(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo=0, splits=splits)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    assert rel_err(out, ref) <= TOL_GENERIC
    assert np.allclose(lse, ref_lse, rtol=1e-5, atol=1e-4)


def test_generic_pages_setting_full_size_sampled(api, gpu):
    """The full 32768-position 2-bit layer at the pages' setting, uniform codes; the oracle
    computes four heads."""
    w = synth.WORKLOADS[5]
    kcb, vcb = oracle_codebooks(w)
    offs = w.offsets()
    kc = synth.uniform_codes(w, True, int(offs[-1]))
    vc = synth.uniform_codes(w, False, int(offs[-1]))
    q = synth.queries(w)
    out, _ = _attend(api, w, q, kc, vc, offs, kcb, vcb, gpu)
    qf = q_as_f64(w, q)
    for h in (0, 7, 20, 31):
        kvh = h // (w.q_heads // w.kv_heads)
        ref, _ = O.attend_codes(qf[:, h:h + 1], kc[:, kvh:kvh + 1], vc[:, kvh:kvh + 1], offs, kcb, vcb, w.rope_base)
        assert rel_err(out[0, h], ref[0, 0]) <= TOL_GENERIC


@pytest.mark.parametrize("wi,T", [(0, None), (1, 3000), (3, None)])
def test_generic_on_g8_workloads(api, gpu, wi, T):
    """GENERIC on the library's own layout: the tiny fp32 case (16 entries, one round), 3000
    encoded positions of the 2-bit layer, and the ragged batch of 16 (uniform codes)."""
    w = synth.WORKLOADS[wi] if T is None else synth.WORKLOADS[wi].with_(seq_len=T)
    kcb, vcb = oracle_codebooks(synth.WORKLOADS[wi])
    offs = w.offsets()
    if wi == 3:
        kc = synth.uniform_codes(w, True, int(offs[-1]))
        vc = synth.uniform_codes(w, False, int(offs[-1]))
        heads = [(0, 0), (5, 17), (15, 31)]
    else:
        kc, _ = O.encode(synth.kv_cache_rows(w, True), kcb)
        vc, _ = O.encode(synth.kv_cache_rows(w, False), vcb)
        heads = None
    q = synth.queries(w)
    out, _ = _attend(api, w, q, kc, vc, offs, kcb, vcb, gpu)
    qf = q_as_f64(w, q)
    if heads is None:
        ref, _ = O.attend_codes(qf, kc, vc, offs, kcb, vcb, w.rope_base)
        assert rel_err(out, ref) <= TOL_GENERIC
    else:
        group = w.q_heads // w.kv_heads
        for b, h in heads:
            sl = slice(offs[b], offs[b + 1])
            ref, _ = O.attend_codes(qf[b:b + 1, h:h + 1], kc[sl, h // group:h // group + 1],
                                    vc[sl, h // group:h // group + 1], np.array([0, offs[b + 1] - offs[b]]),
                                    kcb, vcb, w.rope_base)
            assert rel_err(out[b, h], ref[0, 0]) <= TOL_GENERIC


def test_generic_two_byte_codes_and_checked_codes(api, gpu):
    """300 entries (uint16 codes), g = 16, 3 rounds, 2 KV heads x 16 query heads, two sequences;
    then one code out of range: clamped to the last entry and reported in the error word."""
    rng = np.random.default_rng(91)
    w = synth.Workload(name="u16", seed=91, g=16, R=3, n_codes=300, q_heads=32, kv_heads=2,
                       batch=2, ragged=(100, 700), n_outliers=0, codebook="normal")
    kcb, vcb = synth.normal_codebook(w, True), synth.normal_codebook(w, False)
    offs = w.offsets()
    N = int(offs[-1])
    kc = rng.integers(0, 300, size=(N, 2, 3, 8))
    vc = rng.integers(0, 300, size=(N, 2, 3, 8))
    q = synth.queries(w)
    out, _ = _attend(api, w, q, kc, vc, offs, kcb, vcb, gpu)
    ref, _ = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    assert rel_err(out, ref) <= TOL_GENERIC
    cfg = _cfg(api, w)
    bad = kc.copy()
    bad[3, 1, 2, 5] = 4000
    ws = api.attend_workspace(cfg, 2, int(np.diff(offs).max()), gpu, algo=GENERIC)
    api.attend_decode(cfg, to_torch_q(q, w.q_dtype, gpu), _codes_gpu(bad, w, gpu), _codes_gpu(vc, w, gpu),
                      torch.from_numpy(offs).to(gpu), int(np.diff(offs).max()),
                      torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu), workspace=ws, algo=GENERIC)
    assert api.workspace_error(ws) == 1
