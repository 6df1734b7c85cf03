"""EM-step parity: assignments bit-exact with the oracle's, codebook entries equal to the
oracle's fp64-mean update (summation order differs, so at most 1 ulp apart), SSE within
1e-12 relative, and the step deterministic run to run."""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _ulp_diff(a: np.ndarray, b: np.ndarray) -> int:
    ia = a.astype(np.float32).view(np.int32).astype(np.int64)
    ib = b.astype(np.float32).view(np.int32).astype(np.int64)
    return int(np.abs(ia - ib).max())


def _gpu_step(api, cfg, rows, cb_round, gpu):
    r = torch.from_numpy(rows).to(gpu)
    cb = torch.from_numpy(cb_round.copy()).to(gpu)
    codes = torch.empty((rows.shape[0], cfg.d // cfg.g), dtype=api.code_dtype(cfg), device=gpu)
    sse = torch.zeros(1, dtype=torch.float64, device=gpu)
    api.em_step(cfg, r, cb, codes_out=codes, sse_out=sse)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    if cfg.code_bytes == 2:
        c = c.view(np.uint16)
    return cb.cpu().numpy(), c.astype(np.int64), float(sse.item())


def _check(api, cfg, rows, cb0, gpu):
    cb_g, codes_g, sse_g = _gpu_step(api, cfg, rows, cb0, gpu)
    cb_o, codes_o, sse_o = O.em_step(rows, cb0)
    assert np.array_equal(codes_g, codes_o)
    assert _ulp_diff(cb_g, cb_o) <= 1
    assert abs(sse_g - sse_o) <= 1e-12 * abs(sse_o)
    return cb_g


@pytest.mark.parametrize("key", [True, False])
def test_em_step_fitting_rows(api, gpu, key):
    """The 2-bit layer's 4096 fitting rows, Forgy init, two consecutive steps."""
    w = synth.WORKLOADS[1]
    cfg = api.Config(d=128, g=8, R=1, n_codes=256, q_heads=32, kv_heads=8)
    rows = synth.fit_rows(w, key)
    cb = O.forgy_init(rows, synth.forgy_indices(w, key, 0, rows.shape[0]), 8)
    cb1 = _check(api, cfg, rows, cb, gpu)
    _check(api, cfg, rows, O.em_step(rows, cb)[0], gpu)
    assert cb1.shape == (16, 256, 8)


def test_em_step_encode_workload_rows(api, gpu):
    """The encode workload's 65536 fitting rows (keys with outlier channels)."""
    w = synth.WORKLOADS[4]
    cfg = api.Config(d=128, g=8, R=1, n_codes=256, q_heads=32, kv_heads=8)
    rows = synth.fit_rows(w, True)
    cb = O.forgy_init(rows, synth.forgy_indices(w, True, 0, rows.shape[0]), 8)
    _check(api, cfg, rows, cb, gpu)


def test_em_step_ragged_rows_and_empty_entries(api, gpu):
    rng = np.random.default_rng(5)
    cfg = api.Config(d=32, g=8, R=1, n_codes=300, q_heads=1, kv_heads=1)
    rows = rng.standard_normal((2049 + 513, 32)).astype(np.float32)
    cb = rng.standard_normal((4, 300, 8)).astype(np.float32) * 3     # many entries stay empty
    _check(api, cfg, rows, cb, gpu)


def test_em_step_deterministic(api, gpu):
    w = synth.WORKLOADS[1]
    cfg = api.Config(d=128, g=8, R=1, n_codes=256, q_heads=32, kv_heads=8)
    rows = synth.fit_rows(w, True)
    cb = O.forgy_init(rows, synth.forgy_indices(w, True, 0, rows.shape[0]), 8)
    a = _gpu_step(api, cfg, rows, cb, gpu)
    b = _gpu_step(api, cfg, rows, cb, gpu)
    assert np.array_equal(a[0].view(np.uint32), b[0].view(np.uint32))
    assert a[2] == b[2]


def _gpu_soft(api, cfg, rows, cb_round, tau, gpu):
    r = torch.from_numpy(rows).to(gpu)
    cb = torch.from_numpy(cb_round.copy()).to(gpu)
    sse = torch.zeros(1, dtype=torch.float64, device=gpu)
    api.em_step_soft(cfg, r, cb, tau, sse_out=sse)
    torch.cuda.synchronize()
    return cb.cpu().numpy(), float(sse.item())


@pytest.mark.parametrize("tau", [0.5, 4.0, 40.0])
def test_soft_em_step_matches_oracle(api, gpu, tau):
    """Soft assignment at three temperatures on the 2-bit layer's key fitting rows."""
    w = synth.WORKLOADS[1]
    cfg = api.Config(d=128, g=8, R=1, n_codes=256, q_heads=32, kv_heads=8)
    rows = synth.fit_rows(w, True)
    cb = O.forgy_init(rows, synth.forgy_indices(w, True, 0, rows.shape[0]), 8)
    got, sse = _gpu_soft(api, cfg, rows, cb, tau, gpu)
    want, want_sse = O.em_soft_step(rows, cb, tau)
    scale = np.abs(want).max()
    assert np.abs(got - want).max() <= 2e-5 * scale
    assert abs(sse - want_sse) <= 1e-12 * abs(want_sse)


def test_soft_em_cold_limit_is_the_hard_step(api, gpu):
    w = synth.WORKLOADS[1]
    cfg = api.Config(d=128, g=8, R=1, n_codes=256, q_heads=32, kv_heads=8)
    rows = synth.fit_rows(w, False)
    cb = O.forgy_init(rows, synth.forgy_indices(w, False, 0, rows.shape[0]), 8)
    soft, _ = _gpu_soft(api, cfg, rows, cb, 1e-30, gpu)
    hard, _, _ = O.em_step(rows, cb)
    assert _ulp_diff(soft, hard) <= 1


def test_soft_em_deterministic_and_small_codebooks(api, gpu):
    rng = np.random.default_rng(9)
    cfg = api.Config(d=32, g=8, R=1, n_codes=300, q_heads=1, kv_heads=1)
    rows = rng.standard_normal((777, 32)).astype(np.float32)
    cb = rng.standard_normal((4, 300, 8)).astype(np.float32)
    a, sa = _gpu_soft(api, cfg, rows, cb, 2.0, gpu)
    b, sb = _gpu_soft(api, cfg, rows, cb, 2.0, gpu)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32)) and sa == sb
    want, _ = O.em_soft_step(rows, cb, 2.0)
    assert np.abs(a - want).max() <= 2e-5 * np.abs(want).max()


def test_checkpointed_fit_resumes_bit_for_bit(gpu, tmp_path):
    """The GPU codebook fit (fit.py) saved after every EM step, interrupted part-way through round
    1 and resumed from the file, ends with the uninterrupted fit's codebook bit for bit."""
    from decode_attention_commvq_b200 import fit
    w = synth.WORKLOADS[1].with_(em_rows=1024, em_iters=3)
    rows = torch.from_numpy(synth.fit_rows(w, True)).to(gpu)
    init = lambda r, N: synth.forgy_indices(w, True, r, N)
    full = fit.fit_codebook(rows, w.R, w.n_codes, w.em_iters, init)
    p = str(tmp_path / "k.bin")

    class Stop(Exception):
        pass

    def stop(r, it):
        if (r, it) == (1, 0):
            raise Stop()

    with pytest.raises(Stop):
        fit.fit_codebook(rows, w.R, w.n_codes, w.em_iters, init, checkpoint=p, seed=1, on_step=stop)
    resumed = fit.fit_codebook(rows, w.R, w.n_codes, w.em_iters, init, checkpoint=p, seed=1)
    torch.cuda.synchronize()
    assert torch.equal(full, resumed)
