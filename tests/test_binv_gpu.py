"""Binary value code (CommVQ review, "Assumptions & free parameters": one bit per codebook row
over the whole KV dimension, v_t = s_t^T C): commvq_attend_decode_binv against the oracle's
attention on decoded values, within the attention bounds of the other parity tests (2e-3 fp32
query / 5e-3 bf16 query, max relative error per (b, h)).

The key side is the decode-and-rotate scores kernel (same error as there). On the value side
each softmax weight enters the tensor cores as 24-bit fixed point (absolute error <= 2^-25,
i.e. at most fp16's relative 2^-11 for weights >= 2^-14), H = sum_t p_t s_t is summed exactly in
int32 and contracted with the fp32 C in fp32, so the value side adds less than the fp16 value
codebook of the CommVQ value path."""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import oracle_codebooks, q_as_f64, rel_err, to_torch_q, tol_for

pytestmark = pytest.mark.gpu

W_BINV = synth.WORKLOADS[7]


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _cfg(api, w):
    return api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                      kv_heads=w.kv_heads, rope_base=w.rope_base)


def _key_codebook(w):
    # the binary-value workload's key fit is the 2-bit layer's (same fit seed and rows)
    return oracle_codebooks(synth.WORKLOADS[1])[0] if w.codebook != "normal" else synth.normal_codebook(w, True)


def _run(api, w, q_np, kc, bits, offs, kcb, C, gpu, **kw):
    cfg = _cfg(api, w)
    max_T = int(np.diff(offs).max())
    out, lse = api.attend_decode_binv(
        cfg, to_torch_q(q_np, w.q_dtype, gpu),
        torch.from_numpy(np.ascontiguousarray(kc.astype(np.uint8))).to(gpu),
        torch.from_numpy(bits).to(gpu), torch.from_numpy(offs.astype(np.int64)).to(gpu), max_T,
        torch.from_numpy(kcb).to(gpu), torch.from_numpy(C).to(gpu), **kw)
    torch.cuda.synchronize()
    return out.cpu().numpy(), (lse.cpu().numpy() if lse is not None else None)


@pytest.mark.parametrize("n_bits", [1024, 2048, 4096])
def test_encoded_keys_all_heads(api, gpu, n_bits):
    """3000 oracle-encoded key positions (several splits, a ragged 16-position tail), all 32
    heads; 1, 2 and 4 bits per value scalar."""
    w = W_BINV.with_(seq_len=3000, v_bits=n_bits)
    kcb = _key_codebook(w)
    kc, _ = O.encode(synth.kv_cache_rows(w, True), kcb)
    offs = w.offsets()
    bits = synth.value_bits(w, int(offs[-1]))
    C = synth.binary_value_codebook(w)
    q = synth.queries(w)
    out, lse = _run(api, w, q, kc, bits, offs, kcb, C, gpu)
    ref, ref_lse = O.attend_binv(q_as_f64(w, q), kc, bits, offs, kcb, C, w.rope_base)
    assert rel_err(out, ref) <= tol_for(w)
    assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)


def test_degenerate_lengths(api, gpu):
    """One batch with an empty sequence (zero output, lse -inf), a single position, 17 positions
    (one tile and one), and 283: uniform key codes, 2048 bits."""
    w = W_BINV.with_(batch=4, ragged=None)
    offs = np.array([0, 0, 1, 18, 301], dtype=np.int64)
    N = int(offs[-1])
    kcb = _key_codebook(w)
    kc = synth.uniform_codes(w, True, N)
    bits = synth.value_bits(w, N)
    C = synth.binary_value_codebook(w)
    q = synth.queries(w)
    out, lse = _run(api, w, q, kc, bits, offs, kcb, C, gpu)
    assert np.all(out[0] == 0.0) and np.all(np.isneginf(lse[0]))
    ref, ref_lse = O.attend_binv(q_as_f64(w, q)[1:], kc, bits, offs[1:], kcb, C, w.rope_base)
    assert rel_err(out[1:], ref) <= tol_for(w)
    assert np.allclose(lse[1:], ref_lse, rtol=1e-3, atol=5e-3)
    # a single position: the output is that position's decoded value row, exactly up to fp32
    v1 = O.decode_bits(bits[0:1], C).reshape(w.kv_heads, w.d)
    group = w.q_heads // w.kv_heads
    for h in range(w.q_heads):
        assert np.abs(out[1, h] - v1[h // group]).max() <= 1e-5 * np.abs(v1).max()


def test_fp32_query_head_shapes(api, gpu):
    """fp32 queries, normal codebooks, 16 entries, one round: 4 KV heads x 8 query heads and 1 KV
    head x 8 query heads, 700 positions."""
    for kv, hq in ((4, 32), (1, 8)):
        w = synth.Workload(name="binv_f32", seed=73, R=1, n_codes=16, q_heads=hq, kv_heads=kv,
                           seq_len=700, kv_dtype="f32", q_dtype="f32", n_outliers=0, codebook="normal",
                           v_bits=1024)
        kcb = synth.normal_codebook(w, True)
        kc = synth.uniform_codes(w, True, 700)
        offs = w.offsets()
        bits = synth.value_bits(w, 700)
        C = synth.binary_value_codebook(w)
        q = synth.queries(w)
        out, lse = _run(api, w, q, kc, bits, offs, kcb, C, gpu)
        ref, ref_lse = O.attend_binv(q_as_f64(w, q), kc, bits, offs, kcb, C, w.rope_base)
        assert rel_err(out, ref) <= tol_for(w)
        assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)


def test_ragged_batch_sampled(api, gpu):
    """The ragged batch of 16 (4096-8192 positions each) with binary values, uniform key codes;
    the oracle computes three (sequence, head) pairs."""
    w = synth.WORKLOADS[3].with_(v_bits=2048)
    kcb = _key_codebook(w)
    offs = w.offsets()
    N = int(offs[-1])
    kc = synth.uniform_codes(w, True, N)
    bits = synth.value_bits(w, N)
    C = synth.binary_value_codebook(w)
    q = synth.queries(w)
    out, _ = _run(api, w, q, kc, bits, offs, kcb, C, gpu, want_lse=False)
    qf = q_as_f64(w, q)
    group = w.q_heads // w.kv_heads
    for b, h in ((0, 0), (7, 13), (15, 31)):
        kvh = h // group
        sl = slice(offs[b], offs[b + 1])
        ref, _ = O.attend_binv(qf[b:b + 1, h:h + 1], kc[sl, kvh:kvh + 1], bits[sl],
                               np.array([0, offs[b + 1] - offs[b]]), kcb,
                               np.ascontiguousarray(C[:, kvh * w.d:(kvh + 1) * w.d]), w.rope_base)
        assert rel_err(out[b, h], ref[0, 0]) <= tol_for(w)


def test_full_size_sampled(api, gpu):
    """The full 32768-position workload with 2048 value bits in the launch configuration the
    bench times (uniform key codes); the oracle computes four heads."""
    w = W_BINV
    kcb = _key_codebook(w)
    offs = w.offsets()
    N = int(offs[-1])
    kc = synth.uniform_codes(w, True, N)
    bits = synth.value_bits(w, N)
    C = synth.binary_value_codebook(w)
    q = synth.queries(w)
    out, _ = _run(api, w, q, kc, bits, offs, kcb, C, gpu)
    qf = q_as_f64(w, q)
    group = w.q_heads // w.kv_heads
    for h in (0, 9, 22, 31):
        kvh = h // group
        ref, _ = O.attend_binv(qf[:, h:h + 1], kc[:, kvh:kvh + 1], bits, offs, kcb,
                               np.ascontiguousarray(C[:, kvh * w.d:(kvh + 1) * w.d]), w.rope_base)
        assert rel_err(out[0, h], ref[0, 0]) <= tol_for(w)


def test_unsupported_shapes_and_workspace(api, gpu):
    """n_bits not a multiple of 1024, above 8192, or keys off the decode-and-rotate shape are
    refused before any launch; a short workspace is reported."""
    w = W_BINV
    cfg = _cfg(api, w)
    assert api.attend_binv_workspace_bytes(cfg, 1000, 1, 100) == 0
    assert api.attend_binv_workspace_bytes(cfg, 9216, 1, 100) == 0
    assert api.attend_binv_workspace_bytes(_cfg(api, synth.WORKLOADS[5]), 2048, 1, 100) == 0
    n = api.attend_binv_workspace_bytes(cfg, 2048, 1, 100)
    assert n > 0
    offs = np.array([0, 100], dtype=np.int64)
    kcb = _key_codebook(w)
    kc = synth.uniform_codes(w, True, 100)
    bits = synth.value_bits(w, 100)
    C = synth.binary_value_codebook(w)
    ws = torch.empty(n - 256, dtype=torch.uint8, device=gpu)
    with pytest.raises(api.CommVQError):
        _run(api, w, synth.queries(w), kc, bits, offs, kcb, C, gpu, workspace=ws)


def test_prepared_workspace_reuse(api, gpu):
    """A second call on the same workspace with the prepared flag (key state kept) gives the
    same output bit for bit, and the error word stays clear."""
    w = W_BINV.with_(seq_len=1000)
    kcb = _key_codebook(w)
    offs = w.offsets()
    kc = synth.uniform_codes(w, True, 1000)
    bits = synth.value_bits(w, 1000)
    C = synth.binary_value_codebook(w)
    q = synth.queries(w)
    ws = torch.empty(api.attend_binv_workspace_bytes(_cfg(api, w), w.v_bits, 1, 1000), dtype=torch.uint8,
                     device=gpu)
    out0, lse0 = _run(api, w, q, kc, bits, offs, kcb, C, gpu, workspace=ws)
    out1, lse1 = _run(api, w, q, kc, bits, offs, kcb, C, gpu, workspace=ws, prepared=True)
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)
    assert api.workspace_error(ws) == 0


def test_many_waves_of_ctas(api, gpu):
    """8192 value bits (32 slices of 256 rows) for 20 sequences of 1 KV head x 8 query heads:
    ~640 CTAs of the bit-plane kernel, several per SM in turn, each holding all of tensor
    memory while it runs."""
    rng = np.random.default_rng(77)
    lens = rng.integers(1, 300, size=20)
    w = synth.Workload(name="binv_waves", seed=77, R=2, n_codes=256, q_heads=8, kv_heads=1, batch=20,
                       seq_len=300, n_outliers=0, codebook="normal", v_bits=8192)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(offs[-1])
    kcb = synth.normal_codebook(w, True)
    kc = synth.uniform_codes(w, True, N)
    bits = synth.value_bits(w, N)
    C = synth.binary_value_codebook(w)
    q = synth.queries(w)
    out, lse = _run(api, w, q, kc, bits, offs, kcb, C, gpu)
    ref, ref_lse = O.attend_binv(q_as_f64(w, q), kc, bits, offs, kcb, C, w.rope_base)
    assert rel_err(out, ref) <= tol_for(w)
    assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)
