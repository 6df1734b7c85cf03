"""Sequence lengths outside [0, max_T] and the prepared state across decode steps.

A sequence whose offsets give more rows than max_T is truncated to max_T rows, and one whose
offsets decrease is read as empty; either sets bit 2 of the device error word (the call
completes, nothing traps). The expected outputs come from the oracle run on the clamped
sequences. The error word of a later call with valid lengths on the same workspace is 0 again:
each call's last kernel publishes and clears the bits its kernels set.
"""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import q_as_f64, rel_err, to_torch_q, tol_for

pytestmark = pytest.mark.gpu

LENGTH_BIT = 4


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _cfg(api, w):
    return api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                      kv_heads=w.kv_heads, rope_base=w.rope_base)


# three sequences: 300 rows; 500 rows against max_T = 400 (truncated); offsets that go back by
# 100 rows (a negative length, read as empty)
BAD_OFFS = np.array([0, 300, 800, 700], dtype=np.int64)
MAX_T = 400
CLAMPED = [(0, 300), (300, 400), (800, 0)]   # (first row, rows) the call must attend to


def _inputs(w):
    total = int(BAD_OFFS.max())
    kc = synth.uniform_codes(w, True, total)
    vc = synth.uniform_codes(w, False, total)
    kcb = synth.normal_codebook(w, True)
    vcb = synth.normal_codebook(w, False)
    return kc, vc, kcb, vcb


def _clamped_reference(w, q, kc, vc, kcb, vcb, values=None):
    """The oracle per sequence on the rows the clamped lengths select."""
    outs, lses = [], []
    for b, (r0, n) in enumerate(CLAMPED):
        qb = q_as_f64(w, q)[b:b + 1]
        offs = np.array([0, n], dtype=np.int64)
        if values is None:
            o, l = O.attend_codes(qb, kc[r0:r0 + n], vc[r0:r0 + n], offs, kcb, vcb, w.rope_base)
        else:
            o, l = O.attend_binv(qb, kc[r0:r0 + n], values[r0:r0 + n], offs, kcb, vcb, w.rope_base)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs), np.concatenate(lses)


def _check(out, lse, ref, ref_lse, w):
    assert rel_err(out[:2], ref[:2]) <= tol_for(w)
    assert np.allclose(lse[:2], ref_lse[:2], rtol=1e-3, atol=5e-3)
    assert np.all(out[2] == 0.0) and np.all(np.isneginf(lse[2]))


@pytest.mark.parametrize("algo", [1, 2, 3])
def test_bad_lengths_are_clamped_and_reported(api, gpu, algo):
    w = synth.WORKLOADS[1].with_(batch=3, ragged=None, seq_len=MAX_T, codebook="normal")
    kc, vc, kcb, vcb = _inputs(w)
    cfg = _cfg(api, w)
    q_np = synth.queries(w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    kct, vct = torch.from_numpy(kc).to(gpu), torch.from_numpy(vc).to(gpu)
    kcbt, vcbt = torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu)
    ws = api.attend_workspace(cfg, 3, MAX_T, gpu, algo=algo)
    out, lse = api.attend_decode(cfg, q, kct, vct, torch.from_numpy(BAD_OFFS).to(gpu), MAX_T, kcbt, vcbt,
                                 workspace=ws, algo=algo)
    assert api.workspace_error(ws) == LENGTH_BIT
    ref, ref_lse = _clamped_reference(w, q_np, kc, vc, kcb, vcb)
    _check(out.cpu().numpy(), lse.cpu().numpy(), ref, ref_lse, w)
    good = torch.tensor([0, 300, 700, 800], dtype=torch.int64, device=gpu)
    api.attend_decode(cfg, q, kct, vct, good, MAX_T, kcbt, vcbt, workspace=ws, algo=algo)
    assert api.workspace_error(ws) == 0


def test_bad_lengths_with_prepared_state(api, gpu):
    """The decode-and-rotate path with COMMVQ_ATTEND_PREPARED clears no word at the start of a
    call: the bit of a bad call must still be gone after the next good one."""
    w = synth.WORKLOADS[1].with_(batch=3, ragged=None, seq_len=MAX_T, codebook="normal")
    kc, vc, kcb, vcb = _inputs(w)
    cfg = _cfg(api, w)
    q = to_torch_q(synth.queries(w), w.q_dtype, gpu)
    kct, vct = torch.from_numpy(kc).to(gpu), torch.from_numpy(vc).to(gpu)
    kcbt, vcbt = torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu)
    ws = api.attend_workspace(cfg, 3, MAX_T, gpu, algo=2)
    api.attend_prepare(cfg, 3, MAX_T, kcbt, vcbt, ws, algo=2)
    good = torch.tensor([0, 300, 700, 800], dtype=torch.int64, device=gpu)
    bad = torch.from_numpy(BAD_OFFS).to(gpu)
    for offs, want in ((good, 0), (bad, LENGTH_BIT), (good, 0), (bad, LENGTH_BIT), (good, 0)):
        api.attend_decode(cfg, q, kct, vct, offs, MAX_T, kcbt, vcbt, workspace=ws, algo=2, prepared=True)
        assert api.workspace_error(ws) == want


def test_binary_values_bad_lengths(api, gpu):
    w = synth.WORKLOADS[7].with_(batch=3, ragged=None, seq_len=MAX_T, codebook="normal")
    kc, _, kcb, _ = _inputs(w)
    bits = synth.value_bits(w, int(BAD_OFFS.max()))
    C = synth.binary_value_codebook(w)
    cfg = _cfg(api, w)
    q_np = synth.queries(w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    ws = torch.empty(api.attend_binv_workspace_bytes(cfg, w.v_bits, 3, MAX_T), dtype=torch.uint8, device=gpu)
    args = (cfg, q, torch.from_numpy(kc).to(gpu), torch.from_numpy(bits).to(gpu))
    cb = (torch.from_numpy(kcb).to(gpu), torch.from_numpy(C).to(gpu))
    out, lse = api.attend_decode_binv(*args, torch.from_numpy(BAD_OFFS).to(gpu), MAX_T, *cb, workspace=ws)
    assert api.workspace_error(ws) == LENGTH_BIT
    ref, ref_lse = _clamped_reference(w, q_np, kc, None, kcb, C, values=bits)
    _check(out.cpu().numpy(), lse.cpu().numpy(), ref, ref_lse, w)
    good = torch.tensor([0, 300, 700, 800], dtype=torch.int64, device=gpu)
    api.attend_decode_binv(*args, good, MAX_T, *cb, workspace=ws, prepared=True)
    assert api.workspace_error(ws) == 0


def test_comparator_bad_lengths(api, gpu):
    """commvq_decompress skips the rows past max_T and commvq_dense_decode attends to the
    clamped sequences; both report bit 2."""
    w = synth.WORKLOADS[1].with_(batch=3, ragged=None, seq_len=MAX_T, codebook="normal")
    kc, vc, kcb, vcb = _inputs(w)
    cfg = _cfg(api, w)
    total = int(BAD_OFFS.max())
    kct, vct = torch.from_numpy(kc).to(gpu), torch.from_numpy(vc).to(gpu)
    kcbt, vcbt = torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu)
    bad = torch.from_numpy(BAD_OFFS).to(gpu)
    k_rows = torch.zeros((total, w.kv_heads, w.d), dtype=torch.bfloat16, device=gpu)
    v_rows = torch.zeros_like(k_rows)
    ws = torch.empty(api.decompress_workspace_bytes(cfg, MAX_T), dtype=torch.uint8, device=gpu)
    api.decompress(cfg, kct, vct, bad, MAX_T, kcbt, vcbt, k_out=k_rows, v_out=v_rows, workspace=ws)
    assert api.workspace_error(ws) == LENGTH_BIT
    # rows 700..799 of sequence 1 lie past max_T: not written
    assert torch.count_nonzero(k_rows[700:800]).item() == 0
    q_np = synth.queries(w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    wsd = torch.empty(api.dense_decode_workspace_bytes(cfg, 3, MAX_T), dtype=torch.uint8, device=gpu)
    out, lse = api.dense_decode(cfg, q, k_rows, v_rows, bad, MAX_T, workspace=wsd)
    assert api.workspace_error(wsd) == LENGTH_BIT
    ref, ref_lse = _clamped_reference(w, q_np, kc, vc, kcb, vcb)
    # dense rows are bf16: the comparator's own bound
    o = out.cpu().numpy()
    assert rel_err(o[:2], ref[:2]) <= 2e-2
    assert np.all(o[2] == 0.0) and np.all(np.isneginf(lse.cpu().numpy()[2]))
    good = torch.tensor([0, 300, 700, 800], dtype=torch.int64, device=gpu)
    api.dense_decode(cfg, q, k_rows, v_rows, good, MAX_T, workspace=wsd)
    assert api.workspace_error(wsd) == 0


def test_prepared_state_survives_other_step_shapes(api, gpu):
    """commvq_attend_prepare with B = 1 and max_T = 1000 (63 splits), then decode steps with
    COMMVQ_ATTEND_PREPARED at max_T = 3000 (148 splits) and at B = 2: the prepared images sit at
    fixed workspace offsets, so the results equal unprepared calls bit for bit."""
    w = synth.WORKLOADS[1].with_(seq_len=3000, codebook="normal")
    cfg = _cfg(api, w)
    kcb = torch.from_numpy(synth.normal_codebook(w, True)).to(gpu)
    vcb = torch.from_numpy(synth.normal_codebook(w, False)).to(gpu)
    big = max(api.attend_workspace_bytes(cfg, 1, 3000, algo=2), api.attend_workspace_bytes(cfg, 2, 3000, algo=2))
    ws = torch.empty(big, dtype=torch.uint8, device=gpu)
    api.attend_prepare(cfg, 1, 1000, kcb, vcb, ws, algo=2)
    for B, T in ((1, 3000), (2, 1500), (1, 1000)):
        wb = w.with_(batch=B, seq_len=T)
        kc = torch.from_numpy(synth.uniform_codes(wb, True, B * T)).to(gpu)
        vc = torch.from_numpy(synth.uniform_codes(wb, False, B * T)).to(gpu)
        q = to_torch_q(synth.queries(wb), w.q_dtype, gpu)
        offs = torch.from_numpy(wb.offsets()).to(gpu)
        out_p, lse_p = api.attend_decode(cfg, q, kc, vc, offs, T, kcb, vcb, workspace=ws, algo=2, prepared=True)
        out_u, lse_u = api.attend_decode(cfg, q, kc, vc, offs, T, kcb, vcb, algo=2)
        torch.cuda.synchronize()
        assert torch.equal(out_p, out_u) and torch.equal(lse_p, lse_u)
    assert api.workspace_error(ws) == 0
