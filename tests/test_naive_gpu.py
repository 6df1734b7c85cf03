"""Parity of the decompress-then-attend comparator (CommVQ review, "What carries the argument"
and Table 5: the "naive implementation of the same quantization").

* commvq_decompress: every written element against the oracle's fp64 decode + RoPE, within the
  bound of the roundings the kernel takes (fp16 codebook entries, an fp16 round sum, one final
  rounding to the output type).
* commvq_dense_decode: against the oracle's dense attention on the same 16-bit rows; the only
  rounding is the softmax weights to the row type before the second product.
* Both together: against the oracle's attention straight from the codes.
Every expected value and every bound is computed from oracle outputs and the seeded inputs."""
import numpy as np
import pytest
import torch

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import TOL_BF16, oracle_codebooks, q_as_f64, rel_err, to_torch_q

pytestmark = pytest.mark.gpu

U16 = 2.0 ** -11    # unit roundoff of fp16 (11 significant bits)
UOUT = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


@pytest.fixture(scope="module")
def api():
    from decode_attention_commvq_b200 import api as A
    return A


def _cfg(api, w):
    return api.Config(d=w.d, g=w.g, R=w.R, n_codes=w.n_codes, q_heads=w.q_heads,
                      kv_heads=w.kv_heads, rope_base=w.rope_base)


def _gpu_codes(c, gpu):
    return torch.from_numpy(np.ascontiguousarray(c.astype(np.uint8))).to(gpu)


def _abs_sum(codes: np.ndarray, cb: np.ndarray) -> np.ndarray:
    """sum_r |cb[r, j, code, :]| per element: codes [N, KV, R, G] -> [N, KV, d]."""
    R, G, Nc, g = cb.shape
    N, KV = codes.shape[:2]
    out = np.zeros((N, KV, G, g))
    for r in range(R):
        for j in range(G):
            out[:, :, j] += np.abs(cb[r, j][codes[:, :, r, j].astype(np.int64)])
    return out.reshape(N, KV, G * g)


def _decompress_bounds(codes, cb, R, ref, u_out, rotated):
    """Elementwise bound on |decompressed - exact|: the fp16 entries and the fp16 sum each
    round by at most U16 of the summed magnitudes A, or by half the fp16 subnormal spacing
    (2^-25) below fp16's normal range (R + 1 roundings); a rotation is orthogonal, so a pair's
    error moves at most sqrt 2 times its larger component's; the fp32 rotation adds a few
    2^-24 A; the final rounding adds u_out of the result."""
    A = _abs_sum(codes, cb)
    if rotated:
        pm = np.maximum(A[..., 0::2], A[..., 1::2])
        A = np.repeat(pm, 2, axis=-1) * np.sqrt(2.0)
    pre = (R + 1) * (U16 * A + 2.0 ** -25 * (np.sqrt(2.0) if rotated else 1.0)) + 2.0 ** -21 * A
    return u_out * np.abs(ref) + (1.0 + u_out) * pre + 1e-30


def _sample_rows(offs: np.ndarray, limit: int, seed: int) -> np.ndarray:
    N = int(offs[-1])
    if N <= limit:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    edges = np.concatenate([offs[:-1], offs[1:] - 1])
    edges = edges[(edges >= 0) & (edges < N)]
    return np.unique(np.concatenate([edges, rng.choice(N, size=limit, replace=False)]))


def _decompress(api, w, kc, vc, offs, kcb, vcb, gpu, dtype):
    cfg = _cfg(api, w)
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    max_T = int(np.diff(offs).max()) if len(offs) > 1 else 0
    ko, vo = api.decompress(cfg, _gpu_codes(kc, gpu), _gpu_codes(vc, gpu), offsets, max_T,
                            torch.from_numpy(kcb).to(gpu), torch.from_numpy(vcb).to(gpu), out_dtype=dtype)
    torch.cuda.synchronize()
    return ko, vo


def _check_decompress(w, kc, vc, offs, kcb, vcb, ko, vo, dtype, rows):
    pos = rows - offs[np.searchsorted(offs, rows, side="right") - 1]       # in-sequence positions
    khat = O.decode(kc[rows], kcb)                                         # [n, KV, d]
    n, KV, d = khat.shape
    k_ref = O.rope(khat.reshape(n * KV, d), np.repeat(pos, KV), w.rope_base).reshape(n, KV, d)
    v_ref = O.decode(vc[rows], vcb)
    ridx = torch.from_numpy(rows.astype(np.int64)).to(ko.device)
    k_got = ko[ridx].double().cpu().numpy()
    v_got = vo[ridx].double().cpu().numpy()
    kb = _decompress_bounds(kc[rows], kcb, w.R, k_ref, UOUT[dtype], True)
    vb = _decompress_bounds(vc[rows], vcb, w.R, v_ref, UOUT[dtype], False)
    assert np.all(np.abs(k_got - k_ref) <= kb), float((np.abs(k_got - k_ref) / kb).max())
    assert np.all(np.abs(v_got - v_ref) <= vb), float((np.abs(v_got - v_ref) / vb).max())


def _encoded(w, T=None):
    kcb, vcb = oracle_codebooks(w)
    if T is not None:
        w = w.with_(seq_len=T)
    kc, _ = O.encode(synth.kv_cache_rows(w, True), kcb)
    vc, _ = O.encode(synth.kv_cache_rows(w, False), vcb)
    return w, kc, vc, kcb, vcb


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("wi,T", [(0, None), (1, 3000)])
def test_decompress_encoded_workloads(api, gpu, wi, T, dtype):
    """The tiny workload (one round, 16 entries: the checked-code path) and 3000 encoded
    positions of the 2-bit layer; every element."""
    w, kc, vc, kcb, vcb = _encoded(synth.WORKLOADS[wi], T)
    offs = w.offsets()
    ko, vo = _decompress(api, w, kc, vc, offs, kcb, vcb, gpu, dtype)
    _check_decompress(w, kc, vc, offs, kcb, vcb, ko, vo, dtype, np.arange(int(offs[-1])))


@pytest.mark.parametrize("wi", [1, 2, 3])
def test_decompress_full_size_sampled_rows(api, gpu, wi):
    """Full-size workloads with uniform codes (2-bit 32K, 1-bit 128K, the ragged batch of 16);
    a seeded sample of rows plus every sequence's first and last row."""
    w = synth.WORKLOADS[wi]
    kcb, vcb = oracle_codebooks(w)
    offs = w.offsets()
    total = int(offs[-1])
    kc = synth.uniform_codes(w, True, total)
    vc = synth.uniform_codes(w, False, total)
    ko, vo = _decompress(api, w, kc, vc, offs, kcb, vcb, gpu, torch.bfloat16)
    _check_decompress(w, kc, vc, offs, kcb, vcb, ko, vo, torch.bfloat16, _sample_rows(offs, 3000, wi))


def _dense_inputs(rng, offs, Hq, Hkv, d=128):
    N = int(offs[-1])
    q = rng.standard_normal((len(offs) - 1, Hq, d)).astype(np.float32)
    k = (rng.standard_normal((N, Hkv, d)) * 1.5).astype(np.float32)
    v = rng.standard_normal((N, Hkv, d)).astype(np.float32)
    return q, k, v


def _to_dtype(x: np.ndarray, dtype, gpu):
    t = torch.from_numpy(x).to(dtype)
    return t.to(gpu), t.double().numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("Hq,Hkv,offs,splits", [
    (32, 8, [0, 1000], 0),
    (32, 8, [0, 1000], 5),
    (16, 1, [0, 333, 333, 334, 2000], 0),
    (16, 2, [0, 17, 530], 3),
    (4, 4, [0, 4096], 0),
    (8, 8, [0, 1], 0),
])
def test_dense_decode_matches_oracle(api, gpu, dtype, Hq, Hkv, offs, splits):
    """Every KV-head count the kernel takes, up to 16 heads per group, ragged and empty
    sequences, one-position sequences, several split counts. q has the row type, so the
    products are exact and the softmax-weight rounding (u of the row type) is the only
    rounding beyond fp32: |o - r| <= u * sum_t p_t |v_t| (+ fp32 slack)."""
    rng = np.random.default_rng(71 + Hq + Hkv + splits)
    offs = np.array(offs)
    q, k, v = _dense_inputs(rng, offs, Hq, Hkv)
    qg, qd = _to_dtype(q, dtype, gpu)
    kg, kd = _to_dtype(k, dtype, gpu)
    vg, vd = _to_dtype(v, dtype, gpu)
    cfg = api.Config(d=128, g=8, R=2, n_codes=256, q_heads=Hq, kv_heads=Hkv)
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    out, lse = api.dense_decode(cfg, qg, kg, vg, offsets, int(np.diff(offs).max()), splits=splits)
    torch.cuda.synchronize()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    ref, ref_lse = O.attend_dense(qd, kd, vd, offs)
    mag, _ = O.attend_dense(qd, kd, np.abs(vd), offs)
    bound = UOUT[dtype] * mag + 2.0 ** -16 * np.abs(ref).max()
    assert np.all(np.abs(out - ref) <= bound), float((np.abs(out - ref) / np.maximum(bound, 1e-30)).max())
    fin = np.isfinite(ref_lse)
    assert np.allclose(lse[fin], ref_lse[fin], rtol=0, atol=1e-4)
    assert np.all(lse[~fin] == -np.inf) and np.all(out[~np.isfinite(ref_lse)] == 0)


def _naive(api, w, q_np, kc, vc, offs, kcb, vcb, gpu, dtype):
    ko, vo = _decompress(api, w, kc, vc, offs, kcb, vcb, gpu, dtype)
    cfg = _cfg(api, w)
    q = to_torch_q(q_np, w.q_dtype, gpu)
    offsets = torch.from_numpy(offs.astype(np.int64)).to(gpu)
    out, lse = api.dense_decode(cfg, q, ko, vo, offsets, int(np.diff(offs).max()))
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _bf16_end_to_end_bound(w, qf, kc, vc, offs, kcb, vcb):
    """First-order bound for the bf16 store: key errors dk move each score by at most
    ds_t = sum_i |q_i| dk_ti / sqrt d, so every weight moves by a factor within
    e^{+-2 max ds}; value errors dv add sum_t p_t dv_t; the weight rounding adds
    2^-8 sum_t p_t |v_t|. The weighted sums come from the oracle's own softmax."""
    u = 2.0 ** -8
    khat, vhat = O.decode(kc, kcb), O.decode(vc, vcb)
    k_ref = O.rope_cache(khat, offs, w.rope_base)
    dk = _decompress_bounds(kc, kcb, w.R, k_ref, u, True)
    dv = _decompress_bounds(vc, vcb, w.R, vhat, u, False)
    mag, _ = O.attend(qf, khat, np.abs(vhat), offs, w.rope_base)
    dvs, _ = O.attend(qf, khat, dv, offs, w.rope_base)
    group = w.q_heads // w.kv_heads
    bound = np.zeros_like(mag)
    for b in range(len(offs) - 1):
        sl = slice(offs[b], offs[b + 1])
        for h in range(w.q_heads):
            ds = (np.abs(qf[b, h])[None, :] * dk[sl, h // group]).sum(-1).max() / np.sqrt(w.d)
            bound[b, h] = (np.expm1(2 * ds) + u) * mag[b, h] + dvs[b, h]
    return bound


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_naive_path_end_to_end(api, gpu, dtype):
    """Decompress + dense decode on 3000 encoded positions of the 2-bit layer, all 32 heads,
    against the oracle's attention from codes. With an fp16 store the errors are those of the
    fused path's fp16 operands and the fused path's bound (5e-3) holds; the bf16 store gets
    the first-order bound of its own roundings."""
    w, kc, vc, kcb, vcb = _encoded(synth.WORKLOADS[1], 3000)
    q = synth.queries(w)
    offs = w.offsets()
    out, _ = _naive(api, w, q, kc, vc, offs, kcb, vcb, gpu, dtype)
    qf = q_as_f64(w, q)
    ref, _ = O.attend_codes(qf, kc, vc, offs, kcb, vcb, w.rope_base)
    if dtype == torch.float16:
        assert rel_err(out, ref) <= TOL_BF16
    else:
        bound = _bf16_end_to_end_bound(w, qf, kc, vc, offs, kcb, vcb)
        assert np.all(np.abs(out - ref) <= bound + 1e-6 * np.abs(ref).max())
