"""The no-allocation decode-attention entry point.

commvq_attend_decode_noalloc serves callers that cannot allocate device memory: for example
a plugin inside a host framework that owns the device allocator, or a latency-critical loop
where a cudaMalloc (which may synchronise the device) is not allowed. It runs the same
attention as commvq_attend_decode with the library's fixed internal scratch (32 MiB per
device) in place of a caller-provided workspace.

These tests call it through the C ABI and compare it with commvq_attend_decode and with the
CPU oracle on the same inputs, on two calls in a row (the second call finds the first call's
leftovers in the shared scratch). COMMVQ_ATTEND_PREPARED is refused: prepared state kept in
the shared array could belong to another layer. This file is named so that pytest collects it
last; each test stands on its own.
"""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from tests.helpers import rel_err, to_torch_q, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _inputs(api, w, gpu):
    cfg = api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                     kv_heads=w.kv_heads, rope_base=w.rope_base)
    offs = w.offsets()
    total = int(offs[-1])
    kc = torch.from_numpy(synth.uniform_codes(w, True, total)).to(gpu)
    vc = torch.from_numpy(synth.uniform_codes(w, False, total)).to(gpu)
    kcb = torch.from_numpy(synth.normal_codebook(w, True)).to(gpu)
    vcb = torch.from_numpy(synth.normal_codebook(w, False)).to(gpu)
    q = to_torch_q(synth.queries(w), w.q_dtype, gpu)
    return cfg, q, kc, vc, torch.from_numpy(offs).to(gpu), int(np.diff(offs).max()), kcb, vcb


@pytest.mark.parametrize("wi", [1, 3])
@pytest.mark.parametrize("algo", [1, 2])
def test_noalloc_matches_workspace_entry_point_twice(api, gpu, wi, algo):
    """The 2-bit 32K layer (~7 MiB of scratch) and the ragged batch of 16 (~20 MiB)."""
    w = synth.WORKLOADS[wi]
    cfg, q, kc, vc, offs, max_T, kcb, vcb = _inputs(api, w, gpu)
    ref_out, ref_lse = api.attend_decode(cfg, q, kc, vc, offs, max_T, kcb, vcb, algo=algo)
    torch.cuda.synchronize()
    ref_out, ref_lse = ref_out.cpu().numpy(), ref_lse.cpu().numpy()
    for _ in range(2):
        out = torch.full((w.batch, w.q_heads, w.d), float("nan"), dtype=torch.float32, device=gpu)
        lse = torch.full((w.batch, w.q_heads), float("nan"), dtype=torch.float32, device=gpu)
        api.attend_decode_noalloc(cfg, q, kc, vc, offs, max_T, kcb, vcb, out, lse, algo=algo)
        torch.cuda.synchronize()
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(l).all()
        assert rel_err(o, ref_out) <= tol_for(w)
        assert np.allclose(l, ref_lse, rtol=1e-5, atol=1e-5)


def test_noalloc_rejects_requests_beyond_its_scratch(api, gpu):
    """A 1M-position request needs far more than the 32 MiB scratch: rejected, nothing runs."""
    w = synth.WORKLOADS[1]
    cfg = api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                     kv_heads=w.kv_heads, rope_base=w.rope_base)
    assert api.attend_workspace_bytes(cfg, 1, 1 << 20) > 32 << 20
    q = torch.zeros((1, w.q_heads, w.d), dtype=torch.bfloat16, device=gpu)
    codes = torch.zeros((16, w.kv_heads, w.R, w.groups), dtype=torch.uint8, device=gpu)
    cb = torch.zeros((w.R, w.groups, w.n_codes, w.g), dtype=torch.float32, device=gpu)
    offs = torch.tensor([0, 16], dtype=torch.int64, device=gpu)
    out = torch.zeros((1, w.q_heads, w.d), dtype=torch.float32, device=gpu)
    with pytest.raises(api.CommVQError) as e:
        api.attend_decode_noalloc(cfg, q, codes, codes, offs, 1 << 20, cb, cb, out)
    assert e.value.status == 4
    assert torch.count_nonzero(out).item() == 0


def test_noalloc_rejects_the_prepared_flag(api, gpu):
    """Layer A, then layer B (other codebooks), both without the flag, then layer A with
    COMMVQ_ATTEND_PREPARED: the shared array holds layer B's images by then, so the flagged call
    must be refused (INVALID_ARG) and leave the caller's output untouched."""
    w = synth.WORKLOADS[1].with_(seq_len=2048)
    cfg, q, kc, vc, offs, max_T, kcb_a, vcb_a = _inputs(api, w, gpu)
    wb = w.with_(seed=w.seed + 11)
    kcb_b = torch.from_numpy(synth.normal_codebook(wb, True)).to(gpu)
    vcb_b = torch.from_numpy(synth.normal_codebook(wb, False)).to(gpu)
    out = torch.empty((w.batch, w.q_heads, w.d), dtype=torch.float32, device=gpu)
    for kcb, vcb in ((kcb_a, vcb_a), (kcb_b, vcb_b)):
        api.attend_decode_noalloc(cfg, q, kc, vc, offs, max_T, kcb, vcb, out, algo=2)
    sentinel = torch.full_like(out, 7.0)
    out.copy_(sentinel)
    with pytest.raises(api.CommVQError) as e:
        api.attend_decode_noalloc(cfg, q, kc, vc, offs, max_T, kcb_a, vcb_a, out, algo=2, prepared=True)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert torch.equal(out, sentinel)


def test_noalloc_matches_the_oracle(api, gpu):
    """The no-allocation call against the CPU oracle directly (not only against the workspace
    call), on 3000 positions of the 2-bit layer's shape with uniform codes, twice in a row."""
    from oracle import oracle as O
    from tests.helpers import q_as_f64
    w = synth.WORKLOADS[1].with_(seq_len=3000, codebook="normal")
    cfg = api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                     kv_heads=w.kv_heads, rope_base=w.rope_base)
    offs = w.offsets()
    kc = synth.uniform_codes(w, True, 3000)
    vc = synth.uniform_codes(w, False, 3000)
    kcb = synth.normal_codebook(w, True)
    vcb = synth.normal_codebook(w, False)
    q_np = synth.queries(w)
    ref, ref_lse = O.attend_codes(q_as_f64(w, q_np), kc, vc, offs, kcb, vcb, w.rope_base)
    args = (cfg, to_torch_q(q_np, w.q_dtype, gpu), torch.from_numpy(kc).to(gpu), torch.from_numpy(vc).to(gpu),
            torch.from_numpy(offs).to(gpu), 3000, torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu))
    for _ in range(2):
        out = torch.full((1, w.q_heads, w.d), float("nan"), dtype=torch.float32, device=gpu)
        lse = torch.full((1, w.q_heads), float("nan"), dtype=torch.float32, device=gpu)
        api.attend_decode_noalloc(*args, out, lse)
        torch.cuda.synchronize()
        assert rel_err(out.cpu().numpy(), ref) <= tol_for(w)
        assert np.allclose(lse.cpu().numpy(), ref_lse, rtol=1e-3, atol=5e-3)


def test_noalloc_on_a_second_device(api):
    """The array's address is looked up once per device, with that device current: a call with
    cuda:1 current must use cuda:1's copy and match the workspace call there."""
    if torch.cuda.device_count() < 2:
        pytest.skip("one visible device")
    dev = torch.device("cuda:1")
    w = synth.WORKLOADS[1].with_(seq_len=2048)
    with torch.cuda.device(dev):
        cfg, q, kc, vc, offs, max_T, kcb, vcb = _inputs(api, w, dev)
        ref, _ = api.attend_decode(cfg, q, kc, vc, offs, max_T, kcb, vcb)
        out = torch.empty_like(ref)
        api.attend_decode_noalloc(cfg, q, kc, vc, offs, max_T, kcb, vcb, out)
        torch.cuda.synchronize(dev)
        assert rel_err(out.cpu().numpy(), ref.cpu().numpy()) <= 1e-6
