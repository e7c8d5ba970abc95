"""Accuracy of an approximation the CUDA kernels use, checked on the CPU
with float32 arithmetic written out step by step (numpy), against float64.

The QKV epilogue computes the RoPE angle t * omega_j modulo one turn in
float32 from a split frequency f_j = omega_j / (2 pi) = fh_j + fl_j, with fh_j
short enough that t * fh_j is exact.  The angle then goes to the hardware
sine / cosine on [-pi, pi] (absolute error about 4e-7 there, which this test
does not model); the phase itself must be right to ~1e-7 turns for every
position of the sequence.
"""
import numpy as np

F32 = np.float32


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


def _f32_fma(a, b, c):
    """fma in float32: one rounding of the exact a * b + c."""
    return F32(np.float64(a) * np.float64(b) + np.float64(c))


def test_rope_angle_steps_by_rotation():
    """Where a warp's 32 rows are 32 consecutive positions, the QKV epilogue
    takes each lane's first angle (rows 4 i + r, i = 0..7) from the phase
    above and reaches the next seven by rotating with cos / sin of the exact
    step 4 f (two fmas per component).  Modelled here with float32 products
    and float32 fmas, cosine / sine of the float32 angles in float64 (the
    hardware adds ~4e-7 to each); the seven steps must stay within 2e-6 of the
    exact cos / sin of 2 pi t f, far below bf16's 2^-9."""
    worst = 0.0
    for T in (2048, 8192):
        tbits = int(np.ceil(np.log2(T)))
        f, fh, fl = split_freqs(1e5, 128, tbits)
        for t0 in (0, 4, T // 2 + 1, T - 32):
            q = (phase_turns(t0, fh, fl) * F32(2 * np.pi)).astype(F32)
            d = (phase_turns(4, fh, fl) * F32(2 * np.pi)).astype(F32)
            c, s = np.cos(q.astype(np.float64)).astype(F32), np.sin(q.astype(np.float64)).astype(F32)
            dc, ds = np.cos(d.astype(np.float64)).astype(F32), np.sin(d.astype(np.float64)).astype(F32)
            for i in range(8):
                t = t0 + 4 * i
                ang = 2 * np.pi * ((t * f) % 1.0)
                worst = max(worst, np.abs(c - np.cos(ang)).max(), np.abs(s - np.sin(ang)).max())
                cn = np.array([_f32_fma(a, b, -F32(x * y)) for a, b, x, y in zip(c, dc, s, ds)], dtype=F32)
                sn = np.array([_f32_fma(a, b, F32(x * y)) for a, b, x, y in zip(s, dc, c, ds)], dtype=F32)
                c, s = cn, sn
    assert worst < 2e-6, worst
