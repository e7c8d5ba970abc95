"""Accuracy of the two approximations the CUDA kernels use, checked on the CPU
with float32 arithmetic written out step by step (numpy), against float64.

1. The attention kernel evaluates a quarter of its exponentials 2^x on the
   FMA pipes: x = n + f with n = round(x) obtained by adding 1.5 * 2^23, a
   cubic for 2^f on [-1/2, 1/2], and n added to the exponent field.  The
   probabilities it feeds are rounded to bf16 (relative step 2^-8), so a
   relative error of 1e-4 is invisible there.
2. The QKV epilogue computes the RoPE angle t * omega_j modulo one turn in
   float32 from a split frequency f_j = omega_j / (2 pi) = fh_j + fl_j, with
   fh_j short enough that t * fh_j is exact.  The angle then goes to the
   hardware sine / cosine on [-pi, pi] (absolute error about 4e-7 there,
   which this test does not model); the phase itself must be right to ~1e-7
   turns for every position of the sequence.
"""
import numpy as np

F32 = np.float32
MAGIC = F32(12582912.0)  # 1.5 * 2^23
C0, C1, C2, C3 = F32(0.99992812), F32(0.69326097), F32(0.24261054), F32(0.05517132)


def exp2_poly(x):
    x = np.asarray(x, dtype=F32)
    xc = np.maximum(x, F32(-125.0))
    y = (xc + MAGIC).astype(F32)
    f = (xc - (y - MAGIC).astype(F32)).astype(F32)
    p = ((C3 * f + C2).astype(F32) * f + C1).astype(F32)
    p = (p * f + C0).astype(F32)
    bits = (p.view(np.int32).astype(np.int64) + (y.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    r = bits.astype(np.uint32).view(F32)
    return np.where(x < F32(-125.0), F32(0.0), r)


def test_exp2_poly_relative_error():
    x = np.linspace(-125.0, 8.0, 400001, dtype=np.float64).astype(F32)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_exp2_poly_masked_and_integers():
    assert exp2_poly(np.array([-np.inf], dtype=F32))[0] == 0.0
    assert exp2_poly(np.array([-200.0], dtype=F32))[0] == 0.0
    ints = np.arange(-125, 9, dtype=F32)
    got = exp2_poly(ints).astype(np.float64)
    assert np.allclose(got, np.exp2(ints.astype(np.float64)), rtol=1e-4, atol=0)


def split_freqs(base, D, tbits):
    f = base ** (-2.0 * np.arange(D // 2) / D) / (2.0 * np.pi)
    m, e = np.frexp(f)
    keep = 24 - tbits
    fh = np.ldexp(np.rint(np.ldexp(f, keep - e)), e - keep)
    return f, fh.astype(F32), (f - fh).astype(F32)


def phase_turns(t, fh, fl):
    tf = F32(t)
    p = (tf * fh).astype(F32)           # exact: t has <= tbits bits, fh <= 24 - tbits
    p = (p - np.floor(p)).astype(F32)
    p = (tf * fl + p).astype(F32)
    return (p - np.rint(p)).astype(F32)


def test_rope_phase_split_is_exact_enough():
    for T in (256, 2048, 8192):
        tbits = int(np.ceil(np.log2(T)))
        f, fh, fl = split_freqs(1e5, 128, tbits)
        # t * fh exact in float32 for every position
        for t in (T - 1, T // 2 + 1, 1):
            prod = F32(t) * fh
            assert np.array_equal(prod.astype(np.float64), t * fh.astype(np.float64))
        worst = 0.0
        for t in range(0, T, max(1, T // 257)):
            got = phase_turns(t, fh, fl).astype(np.float64)
            exact = t * f
            err = np.abs(((got - exact) + 0.5) % 1.0 - 0.5)
            worst = max(worst, err.max())
        assert worst < 2e-7, (T, worst)
