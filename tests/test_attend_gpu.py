"""Decode-attention parity: CUDA output vs the fp64 oracle (decompress, RoPE, softmax)
within 2e-3 (fp32 query) / 5e-3 (bf16 query) max relative error per (b, h), on every
workload, every algorithm and several split counts; plus the degenerate cases."""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import Guarded, oracle_codebooks, q_as_f64, rel_err, to_torch_q, tol_for

pytestmark = pytest.mark.gpu

ALGOS = [1, 2]   # table path, decode-and-rotate path


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _cfg(api, w):
    return api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                      kv_heads=w.kv_heads, rope_base=w.rope_base)


def _codes_np_to_gpu(c, gpu):
    return torch.from_numpy(np.ascontiguousarray(c.astype(np.uint8))).to(gpu)


def _run(api, w, q_np, kc, vc, offs, kcb, vcb, gpu, algo=0, splits=0):
    """One attention call with out, lse and the workspace inside canary guard bands, which must
    be untouched afterwards."""
    cfg = _cfg(api, w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    max_T = int(np.diff(offs).max()) if len(offs) > 1 else 0
    B = len(offs) - 1
    out_g = Guarded((B, w.q_heads, w.d), torch.float32, gpu)
    lse_g = Guarded((B, w.q_heads), torch.float32, gpu)
    ws_g = Guarded((api.attend_workspace_bytes(cfg, B, max_T, algo, splits),), torch.uint8, gpu)
    out, lse = api.attend_decode(cfg, q, _codes_np_to_gpu(kc, gpu), _codes_np_to_gpu(vc, gpu),
                                 offsets, max_T, torch.from_numpy(kcb).to(gpu),
                                 torch.from_numpy(vcb).to(gpu), out=out_g.t, lse=lse_g.t, workspace=ws_g.t,
                                 algo=algo, splits=splits)
    torch.cuda.synchronize()
    assert out_g.intact() and lse_g.intact() and ws_g.intact(), "a kernel wrote outside its buffer"
    return out.cpu().numpy(), lse.cpu().numpy()


def _encoded_inputs(w, T=None):
    """Seeded K/V rows encoded by the oracle (small sizes)."""
    kcb, vcb = oracle_codebooks(w)
    if T is not None:
        w = w.with_(seq_len=T)
    kx = synth.kv_cache_rows(w, True)
    vx = synth.kv_cache_rows(w, False)
    kc, _ = O.encode(kx, kcb)
    vc, _ = O.encode(vx, vcb)
    return w, kc, vc, kcb, vcb


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_tiny_workload(api, gpu, algo, splits):
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[0])
    q = synth.queries(w)
    offs = w.offsets()
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo, splits)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    assert rel_err(out, ref) <= tol_for(w)
    assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("splits", [0, 2, 7])
def test_2bit_layer_short_context_all_heads(api, gpu, algo, splits):
    """All 32 heads on 3000 encoded positions: several 256-position chunks and a ragged tail."""
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=3000)
    q = synth.queries(w)
    offs = w.offsets()
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo, splits)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    assert rel_err(out, ref) <= tol_for(w)
    assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)


def _full_size_all_heads(api, gpu, w, algo=0, splits=0):
    """Full-size workload with uniform random codes (attention does not depend on how codes
    were made); the oracle computes every (sequence, query head), its KV heads on the host's
    cores at once."""
    kcb, vcb = oracle_codebooks(w)
    offs = w.offsets()
    total = int(offs[-1])
    kc = synth.uniform_codes(w, True, total)
    vc = synth.uniform_codes(w, False, total)
    q = synth.queries(w)
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo, splits)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base, threads=O.host_threads())
    assert rel_err(out, ref) <= tol_for(w)
    assert np.all(np.abs(lse - ref_lse) <= 1e-3 * np.maximum(1.0, np.abs(ref_lse)))
    return out


@pytest.mark.parametrize("algo", ALGOS)
def test_2bit_layer_full_size(api, gpu, algo):
    """All 32 heads over 32768 positions."""
    _full_size_all_heads(api, gpu, synth.WORKLOADS[1], algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_1bit_layer_full_size(api, gpu, algo):
    """All 32 heads over 131072 positions."""
    _full_size_all_heads(api, gpu, synth.WORKLOADS[2], algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_ragged_batch_full_size(api, gpu, algo):
    """Every (sequence, head) of the ragged batch of 16."""
    _full_size_all_heads(api, gpu, synth.WORKLOADS[3], algo)


@pytest.mark.parametrize("algo", ALGOS)
def test_split_count_invariance(api, gpu, algo):
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=2000)
    q = synth.queries(w)
    offs = w.offsets()
    outs = [_run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo, s)[0] for s in (1, 2, 5, 16)]
    # The table path keeps softmax weights in fp32, so splits change only fp32 rounding. The
    # decode-and-rotate path feeds the weights to the tensor cores in fp16 relative to each
    # split's own maximum (rounding up to 2^-11 relative), so its bound is fp16's.
    bound = 1e-5 if algo == 1 else 1e-3
    for o in outs[1:]:
        assert rel_err(o, outs[0]) <= bound


@pytest.mark.parametrize("algo", ALGOS)
def test_degenerate_lengths(api, gpu, algo):
    """Empty sequences (out 0, lse -inf), a single position (out = its value), and
    lengths shorter than the split count, mixed in one ragged batch."""
    w = synth.WORKLOADS[1].with_(batch=5, ragged=(0, 0))
    kcb, vcb = oracle_codebooks(synth.WORKLOADS[1])
    lens = np.array([0, 1, 3, 0, 300])
    offs = np.concatenate([[0], np.cumsum(lens)])
    total = int(offs[-1])
    kc = synth.uniform_codes(w, True, total)
    vc = synth.uniform_codes(w, False, total)
    q = synth.queries(w)
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo, splits=4)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    for b in (0, 3):
        assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
    for b in (1, 2, 4):
        assert rel_err(out[b], ref[b]) <= tol_for(w)
    row = int(offs[1])                               # sequence 1's only position
    vhat = O.decode(vc[row:row + 1], vcb)[0]         # [Hkv, d]
    for h in range(w.q_heads):
        assert np.allclose(out[1, h], vhat[h // 4], rtol=1e-3, atol=1e-3)


@pytest.mark.parametrize("algo", ALGOS)
def test_zero_query_gives_mean_value(api, gpu, algo):
    w = synth.WORKLOADS[1].with_(seq_len=777)
    kcb, vcb = oracle_codebooks(synth.WORKLOADS[1])
    offs = w.offsets()
    kc = synth.uniform_codes(w, True, 777)
    vc = synth.uniform_codes(w, False, 777)
    q = np.zeros((1, w.q_heads, w.d), dtype=np.uint16)    # bf16 zeros
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo)
    vhat = O.decode(vc, vcb)                               # [T, Hkv, d]
    mean = vhat.mean(0)
    # table path: fp32 value codebook; decode-and-rotate path: fp16 codebook entries
    # (2^-12 relative rounding each, fixed per entry)
    bound = 1e-4 if algo == 1 else 2e-3
    for h in range(w.q_heads):
        assert rel_err(out[0, h], mean[h // 4]) <= bound
    assert np.allclose(lse, np.log(777), rtol=1e-5)


@pytest.mark.parametrize("algo", ALGOS)
def test_out_of_range_codes_are_flagged_not_trapped(api, gpu, algo):
    """Nc' = 16 with uint8 codes: a code >= 16 is clamped to 15 and recorded in the
    workspace error word; the call itself completes."""
    w = synth.WORKLOADS[0]
    kcb, vcb = oracle_codebooks(w)
    cfg = _cfg(api, w)
    kc = synth.uniform_codes(w, True, 256)
    vc = synth.uniform_codes(w, False, 256)
    kc[17, 0, 0, 3] = 200
    vc[40, 0, 0, 9] = 16
    q = to_torch_q(synth.queries(w), w.q_dtype, gpu)
    offs = torch.tensor([0, 256], dtype=torch.int64, device=gpu)
    ws = api.attend_workspace(cfg, 1, 256, gpu, algo=algo)
    out, _ = api.attend_decode(cfg, q, _codes_np_to_gpu(kc, gpu), _codes_np_to_gpu(vc, gpu), offs, 256,
                               torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu),
                               workspace=ws, algo=algo)
    assert api.workspace_error(ws) == 1
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[17, 0, 0, 3] = 15
    vc2[40, 0, 0, 9] = 15
    out2, _ = api.attend_decode(cfg, q, _codes_np_to_gpu(kc2, gpu), _codes_np_to_gpu(vc2, gpu), offs,
                                256, torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu),
                                workspace=ws, algo=algo)
    assert api.workspace_error(ws) == 0
    # value histograms accumulate with shared-memory float atomics: equal up to rounding order
    assert rel_err(out.cpu().numpy(), out2.cpu().numpy()) <= 1e-6


def test_workspace_too_small_is_rejected(api, gpu):
    w = synth.WORKLOADS[0]
    cfg = _cfg(api, w)
    ws = torch.empty(64, dtype=torch.uint8, device=gpu)
    z = torch.zeros(1, w.q_heads, w.d, dtype=torch.float32, device=gpu)
    codes = torch.zeros(256, 1, 1, 16, dtype=torch.uint8, device=gpu)
    cb = torch.zeros(1, 16, 16, 8, dtype=torch.float32, device=gpu)
    offs = torch.tensor([0, 256], dtype=torch.int64, device=gpu)
    with pytest.raises(api.CommVQError) as e:
        api.attend_decode(cfg, z, codes, codes, offs, 256, cb, cb, workspace=ws)
    assert e.value.status == 4


@pytest.mark.parametrize("algo", ALGOS)
def test_long_split_refreshes_phasors(api, gpu, algo):
    """One split of 4500 positions: the decode-and-rotate path advances its phasors by
    recurrence and rebuilds them exactly every 16 stages (2048 positions)."""
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=4500)
    q = synth.queries(w)
    offs = w.offsets()
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo, splits=1)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    assert rel_err(out, ref) <= tol_for(w)
    assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)


SHAPES = [
    # (q_heads, kv_heads, R, n_codes, q_dtype)
    (32, 8, 2, 256, "f16"),
    (32, 8, 2, 256, "f32"),
    (8, 8, 2, 256, "bf16"),     # no grouping
    (16, 2, 2, 256, "bf16"),    # 8 query heads per KV head
    (8, 4, 1, 256, "bf16"),
    (4, 1, 2, 64, "bf16"),      # smaller codebook: run-time entry count, codes checked
    (6, 2, 1, 100, "f32"),
]


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "q%d_kv%d_R%d_N%d_%s" % s)
def test_shapes_and_query_types(api, gpu, algo, shape):
    Hq, Hkv, R, Nc, qdt = shape
    w = synth.WORKLOADS[1].with_(q_heads=Hq, kv_heads=Hkv, R=R, n_codes=Nc, q_dtype=qdt,
                                 batch=3, ragged=(100, 700), codebook="normal")
    kcb = synth.normal_codebook(w, True)
    vcb = synth.normal_codebook(w, False)
    offs = w.offsets()
    total = int(offs[-1])
    kc = synth.uniform_codes(w, True, total)
    vc = synth.uniform_codes(w, False, total)
    q = synth.queries(w)
    out, lse = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
    assert rel_err(out, ref) <= tol_for(w)
    assert np.allclose(lse, ref_lse, rtol=1e-3, atol=5e-3)


@pytest.mark.parametrize("algo", ALGOS)
def test_prepared_workspace_is_identical(api, gpu, algo):
    """commvq_attend_prepare once, then decode steps with COMMVQ_ATTEND_PREPARED: the same
    results as unprepared calls, for two different queries on one prepared workspace (the
    same bits on the decode-and-rotate path; the table path adds histogram weights with
    shared-memory atomics, whose order varies, so there within 1e-6)."""
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=3000)
    cfg = _cfg(api, w)
    offs = w.offsets()
    max_T = int(np.diff(offs).max())
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    kcg, vcg = _codes_np_to_gpu(kc, gpu), _codes_np_to_gpu(vc, gpu)
    kcbt, vcbt = torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu)
    ws = api.attend_workspace(cfg, 1, max_T, gpu, algo)
    api.attend_prepare(cfg, 1, max_T, kcbt, vcbt, ws, algo=algo)
    q0 = synth.queries(w)
    q1 = synth.queries(w.with_(seed=w.seed + 7))
    for q_np in (q0, q1):
        q = to_torch_q(q_np, w.q_dtype, gpu)
        out_p, lse_p = api.attend_decode(cfg, q, kcg, vcg, offsets, max_T, kcbt, vcbt, workspace=ws,
                                         algo=algo, prepared=True)
        out_u, lse_u = api.attend_decode(cfg, q, kcg, vcg, offsets, max_T, kcbt, vcbt, algo=algo)
        torch.cuda.synchronize()
        if algo == 2:
            assert torch.equal(out_p, out_u) and torch.equal(lse_p, lse_u)
        else:
            assert rel_err(out_p.cpu().numpy(), out_u.cpu().numpy()) <= 1e-6
            assert torch.allclose(lse_p, lse_u, rtol=1e-6, atol=1e-6)
        ref, _ = O.attend_codes(q_as_f64(w, q_np), kc, vc, offs, kcb, vcb, w.rope_base)
        assert rel_err(out_p.cpu().numpy(), ref) <= tol_for(w)
    assert api.workspace_error(ws) == 0


def test_prepared_state_survives_a_longer_context(api, gpu, algo=2):
    """The prepared state sits at fixed workspace offsets: prepared once at a short context,
    it serves PREPARED decode steps at that length and at a longer one, where the split count,
    and so the size of the per-split buffers, differ (1000 positions: 63 splits; 3000: 148)."""
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=3000)
    cfg = _cfg(api, w)
    kcg, vcg = _codes_np_to_gpu(kc, gpu), _codes_np_to_gpu(vc, gpu)
    kcbt, vcbt = torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu)
    ws = api.attend_workspace(cfg, 1, 3000, gpu, algo)
    api.attend_prepare(cfg, 1, 1000, kcbt, vcbt, ws, algo=algo)
    q_np = synth.queries(w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    for T in (1000, 3000, 1000):
        offs = np.array([0, T], dtype=np.int64)
        offsets = torch.from_numpy(offs).to(gpu)
        out_p, _ = api.attend_decode(cfg, q, kcg[:T], vcg[:T], offsets, T, kcbt, vcbt, workspace=ws,
                                     algo=algo, prepared=True)
        out_u, _ = api.attend_decode(cfg, q, kcg[:T], vcg[:T], offsets, T, kcbt, vcbt, algo=algo)
        torch.cuda.synchronize()
        assert torch.equal(out_p, out_u), T
        ref, _ = O.attend_codes(q_as_f64(w, q_np), kc[:T], vc[:T], offs, kcb, vcb, w.rope_base)
        assert rel_err(out_p.cpu().numpy(), ref) <= tol_for(w)
    assert api.workspace_error(ws) == 0


def test_many_queries_within_bound(api, gpu):
    """The bf16 bound on 6 seeded queries x 32 heads (192 heads) over 3000 encoded positions of
    the 2-bit layer, decode-and-rotate path: the tail of the error distribution, not one
    query's."""
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=3000)
    offs = w.offsets()
    worst = 0.0
    for seed in range(11, 17):
        q = synth.queries(w.with_(seed=seed))
        out, _ = _run(api, w, q, kc, vc, offs, kcb, vcb, gpu, algo=2)
        ref, _ = O.attend_codes(q_as_f64(w, q), kc, vc, offs, kcb, vcb, w.rope_base)
        worst = max(worst, rel_err(out, ref))
    assert worst <= tol_for(w), worst


@pytest.mark.parametrize("algo", ALGOS)
def test_timing_events_outside_and_inside_a_capture(api, gpu, algo):
    """The caller's main-kernel events are recorded on direct launches and inside a CUDA
    graph capture alike, and do not change the result."""
    w, kc, vc, kcb, vcb = _encoded_inputs(synth.WORKLOADS[1], T=1000)
    cfg = _cfg(api, w)
    offs = w.offsets()
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    kcg, vcg = _codes_np_to_gpu(kc, gpu), _codes_np_to_gpu(vc, gpu)
    kcbt, vcbt = torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu)
    q = to_torch_q(synth.queries(w), w.q_dtype, gpu)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    ev[0].record()   # torch times only events it has recorded once itself
    ev[1].record()
    ws = api.attend_workspace(cfg, 1, 1000, gpu, algo)
    out_e, _ = api.attend_decode(cfg, q, kcg, vcg, offsets, 1000, kcbt, vcbt, workspace=ws, algo=algo,
                                 main_events=ev)
    torch.cuda.synchronize()
    assert ev[0].elapsed_time(ev[1]) > 0
    out_p, _ = api.attend_decode(cfg, q, kcg, vcg, offsets, 1000, kcbt, vcbt, workspace=ws, algo=algo)
    torch.cuda.synchronize()
    assert rel_err(out_e.cpu().numpy(), out_p.cpu().numpy()) <= 1e-6
    stream = torch.cuda.Stream()
    out_g = torch.empty_like(out_p)
    with torch.cuda.stream(stream):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            api.attend_decode(cfg, q, kcg, vcg, offsets, 1000, kcbt, vcbt, out=out_g, workspace=ws,
                              algo=algo, stream=stream, main_events=ev)
        g.replay()
    torch.cuda.synchronize()
    assert ev[0].elapsed_time(ev[1]) > 0
    assert rel_err(out_g.cpu().numpy(), out_p.cpu().numpy()) <= 1e-6
