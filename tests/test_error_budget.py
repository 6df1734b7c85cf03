"""The decode-and-rotate path's error budget, on the CPU: the kernels' roundings emulated in
numpy around oracle values, against the oracle's exact attention (CommVQ machine review, "What
carries the argument": decoding is a sum of codewords; the bound is the bf16-input tolerance).

Roundings emulated: key and value codebook entries to fp16; the keys' R-round sum exact (the
kernels add the rounds in fp32) and the values' R-round sum in fp16; the rotation in fp64 (the
kernel's fp32 rotation adds ~1e-7); and the rotated key rounded to one fp16 operand (the fast
kernels, attend_fast.cu) or carried as two fp16 terms (attend_mma.cu, exact to ~2^-22). The tests
pin the design decisions: with the key rounds summed exactly, one fp16 operand keeps the worst
head clear of the 5e-3 bound; an fp16 sum of the key rounds would take it past the bound."""
import numpy as np

from decode_attention_commvq_b200 import synth
from oracle import oracle as O
from tests.helpers import TOL_BF16, oracle_codebooks, q_as_f64, rel_err


def _f16(x):
    return x.astype(np.float16).astype(np.float64)


def _decode_f16(codes, cb16, sum16=True):
    """Sum of fp16 entries; each partial sum rounded to fp16 when sum16 (else exact)."""
    R, G, Nc, g = cb16.shape
    out = np.zeros(codes.shape[:2] + (G, g))
    for r in range(R):
        for j in range(G):
            e = cb16[r, j][codes[:, :, r, j]]
            out[:, :, j] = (_f16(out[:, :, j] + e) if sum16 else out[:, :, j] + e) if r else e
    return out.reshape(codes.shape[:2] + (G * g,))


def test_rotated_key_operand_keeps_a_margin():
    w = synth.WORKLOADS[1].with_(seq_len=3000)
    kcb, vcb = oracle_codebooks(synth.WORKLOADS[1])
    kc, _ = O.encode(synth.kv_cache_rows(w, True), kcb)
    vc, _ = O.encode(synth.kv_cache_rows(w, False), vcb)
    offs = w.offsets()
    k_exact = O.rope_cache(O.decode(kc, kcb), offs, w.rope_base)
    v_exact = O.decode(vc, vcb)
    k16 = O.rope_cache(_decode_f16(kc, _f16(kcb), sum16=False), offs, w.rope_base)   # fp16 entries, exact sum
    v16 = _decode_f16(vc, _f16(vcb))
    one_term, two_term = 0.0, 0.0
    for seed in (1, 2, 3, 4):
        q = q_as_f64(w, synth.queries(w.with_(seed=seed)))
        ref, _ = O.attend_dense(q, k_exact, v_exact, offs)
        o1, _ = O.attend_dense(q, _f16(k16), v16, offs)
        o2, _ = O.attend_dense(q, k16, v16, offs)
        one_term = max(one_term, rel_err(o1, ref))
        two_term = max(two_term, rel_err(o2, ref))
    assert one_term <= 0.85 * TOL_BF16, one_term    # the fast kernels
    assert two_term <= 0.6 * TOL_BF16, two_term     # attend_mma.cu
    assert one_term > two_term


def test_key_rounds_summed_exactly_at_full_length():
    """All 32 heads over 32768 positions of the 2-bit layer with uniform codes (the full-size
    parity workload): with the kernels' roundings the worst head stays well inside the bound;
    summing the two key rounds in fp16 instead would take it past the bound."""
    w = synth.WORKLOADS[1]
    kcb, vcb = oracle_codebooks(w)
    offs = w.offsets()
    T = int(offs[-1])
    kc = synth.uniform_codes(w, True, T)
    vc = synth.uniform_codes(w, False, T)
    q = q_as_f64(w, synth.queries(w))
    ref, _ = O.attend_dense(q, O.rope_cache(O.decode(kc, kcb), offs, w.rope_base), O.decode(vc, vcb), offs)
    v16 = _decode_f16(vc, _f16(vcb))
    kernel_like, _ = O.attend_dense(q, _f16(O.rope_cache(_decode_f16(kc, _f16(kcb), sum16=False), offs,
                                                         w.rope_base)), v16, offs)   # one fp16 operand
    fp16_key_sum, _ = O.attend_dense(q, O.rope_cache(_decode_f16(kc, _f16(kcb)), offs, w.rope_base), v16, offs)
    assert rel_err(kernel_like, ref) <= 0.8 * TOL_BF16
    assert rel_err(fp16_key_sum, ref) > TOL_BF16


def test_binary_value_weights_in_three_digits_add_almost_nothing():
    """The binary value code's value side, emulated: each softmax weight p = 2^(s - m) <= 1 as
    24-bit fixed point q = round(p (2^24 - 1)) in three 8-bit digits, the bit-plane sums
    sum_t s_t[n] q_t exact in integers, the contraction with C in fp64 (the kernel's is fp32).
    Against the exact attention on decoded values the output moves by far less than the bf16
    tolerance: each weight is carried to 2^-25 absolute, so the relative change of the output is
    at most ~2^-25 x (positions / sum of weights). Here it is 1.0e-7; fp16 weights would give
    2.3e-5."""
    rng = np.random.default_rng(79)
    T, Nc, d = 3000, 2048, 128
    s = rng.standard_normal(T) * 3.0                       # log2-domain scores, a few units apart
    p = np.exp2(s - s.max())                               # split maximum: every weight <= 1
    q = np.rint(p * (2 ** 24 - 1)).astype(np.int64)
    digits = [(q >> sh) & 0xFF for sh in (16, 8, 0)]
    assert np.array_equal(digits[0] * 65536 + digits[1] * 256 + digits[2], q)
    bits = rng.integers(0, 2, size=(T, Nc), dtype=np.int64)
    C = rng.standard_normal((Nc, d)) * np.sqrt(2.0 / Nc)
    H_int = sum(bits.T @ dg * (256 ** (2 - i)) for i, dg in enumerate(digits))   # exact integers
    out = (H_int / (2 ** 24 - 1)) @ C / p.sum()
    ref = (bits.T @ p) @ C / p.sum()
    err = np.abs(out - ref).max() / np.abs(ref).max()
    assert err < 1e-5
    assert err < TOL_BF16 / 100
