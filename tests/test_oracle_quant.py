"""Pins for the oracle's quantizers (CPU only).

Each check is independent of the formula it pins: exact rational arithmetic
(fractions), brute-force nearest-code search, a library Hadamard matrix, or a
closed-form special case.
"""
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

from oracle import quant as Q
from oracle import codebook as CB


def _rng(seed=0):
    return np.random.Generator(np.random.PCG64(seed))


def _blocks(n, seed=0, scale=1.0):
    r = _rng(seed)
    x = (r.standard_normal((n, 32)) * scale).astype(np.float16)
    return x


def _ulp32(x: float) -> Fraction:
    m, e = np.frexp(np.float32(x))
    return Fraction(2) ** (int(e) - 24)


# ------------------------------------------------------------------ q8_0

def check_q8_0(quantize, x16):
    codes, d16 = quantize(x16)
    xb = x16.astype(np.float32).reshape(-1, 32)
    cb = codes.reshape(-1, 32).astype(int)
    for i in range(xb.shape[0]):
        amax = Fraction(float(np.abs(xb[i]).max()))
        # the fp32 scale is the float nearest amax/127 (exact rational check)
        d32 = np.float32(np.divide(np.float32(float(amax)), np.float32(127)))
        assert abs(Fraction(float(d32)) - amax / 127) <= _ulp32(float(d32)) / 2
        assert d16.reshape(-1)[i] == np.float16(d32)
        if amax == 0:
            assert (cb[i] == 0).all()
            continue
        for j in range(32):
            t = Fraction(float(np.divide(xb[i, j], d32, dtype=np.float32)))
            # brute force: nearest integer in [-127, 127], ties away from zero
            best = min(range(-127, 128), key=lambda c: (abs(t - c), -abs(c)))
            assert cb[i, j] == best, (i, j, float(t), cb[i, j], best)
        # the extreme element always reaches +-127
        j = int(np.argmax(np.abs(xb[i])))
        assert abs(cb[i, j]) == 127


def test_q8_0_bruteforce_random():
    check_q8_0(Q.quantize_q8_0, _blocks(24, seed=1))


def test_q8_0_special_blocks():
    x = np.zeros((6, 32), dtype=np.float16)
    x[1, 5] = -3.0                               # single nonzero
    x[2] = np.arange(32) - 16                    # ramp: -16..15
    x[3, ::2] = 1.5                              # ties of |x|
    x[3, 1::2] = -1.5
    x[4] = np.float16(6.0e-5)                    # subnormal-ish fp16 values
    x[5] = np.float16(65504.0)                   # fp16 max
    check_q8_0(Q.quantize_q8_0, x)
    codes, d = Q.quantize_q8_0(x)
    assert (codes[0] == 0).all() and d[0, 0] == 0
    assert codes[1, 5] == -127 and (np.delete(codes[1], 5) == 0).all()
    # ramp: x/d = (i-16)*127/16 -> element 0 is -127, element 17 (x=1) is 8 (7.9375 rounds up)
    assert codes[2, 0] == -127 and codes[2, 17] == 8 and codes[2, 16] == 0


def test_q8_0_dequant_error_bound():
    x = _blocks(64, seed=2, scale=3.0)
    codes, d16 = Q.quantize_q8_0(x)
    xh = Q.dequantize_q8_0(codes, d16)
    d32 = np.abs(x.astype(np.float32)).max(axis=1) / np.float32(127)
    err = np.abs(xh - x.astype(np.float64))
    # half a step plus the fp16 rounding of the scale times |q| <= 127
    bound = d32[:, None] / 2 + 127 * np.abs(d16.astype(np.float64) - d32[:, None]) + 1e-12
    assert (err <= bound).all()


# ------------------------------------------------------------------ q4_0

def check_q4_0(quantize, x16):
    codes, d16 = quantize(x16)
    xb = x16.astype(np.float32).reshape(-1, 32)
    cb = codes.reshape(-1, 32).astype(int)
    for i in range(xb.shape[0]):
        j0 = int(np.argmax(np.abs(xb[i])))
        m = xb[i, j0]
        if m == 0:
            assert (cb[i] == 8).all()
            continue
        d32 = np.float32(np.divide(m, np.float32(-8), dtype=np.float32))
        assert Fraction(float(d32)) == Fraction(float(m)) / -8     # exact: power of two
        assert d16.reshape(-1)[i] == np.float16(d32)
        # the signed extreme decodes exactly: (0 - 8) * (m / -8) = m
        assert cb[i, j0] == 0
        for j in range(32):
            t = Fraction(float(np.divide(xb[i, j], d32, dtype=np.float32)))
            # brute force: nearest (q - 8) for q in 0..15, ties toward +inf, clamp at 15
            best = min(range(16), key=lambda c: (abs(t - (c - 8)), -c))
            assert cb[i, j] == best, (i, j, float(t), cb[i, j], best)


def test_q4_0_bruteforce_random():
    check_q4_0(Q.quantize_q4_0, _blocks(24, seed=3))


def test_q4_0_special_blocks():
    x = np.zeros((4, 32), dtype=np.float16)
    x[1, 3] = -2.0
    x[1, 7] = 2.0             # |x| tie: first index (negative) wins -> d = 0.25
    x[2, 0] = 5.0
    x[2, 1] = -5.0 + 0.0
    x[3] = np.arange(32) - 12
    check_q4_0(Q.quantize_q4_0, x)
    codes, d = Q.quantize_q4_0(x)
    assert (codes[0] == 8).all()
    assert float(d[1, 0]) == 0.25 and codes[1, 3] == 0 and codes[1, 7] == 15
    # positive extreme 5: d = -0.625; x = -5 -> t = 8 -> floor(16.5) clamps to 15
    assert float(d[2, 0]) == -0.625 and codes[2, 0] == 0 and codes[2, 1] == 15


def test_nibble_packing_convention():
    codes = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    packed = Q.pack_nibbles(codes)
    assert packed.tolist() == [[0x21, 0x43, 0x0F]]
    assert (Q.unpack_nibbles(packed) == codes).all()


# ------------------------------------------------------------------ rotation + lut4

@pytest.mark.parametrize("D", [64, 128])
def test_wht_matches_library_hadamard(D):
    r = _rng(4)
    x = r.integers(-50, 50, size=(5, D)).astype(np.float32)     # exact in fp32
    ref = x.astype(np.float64) @ scipy.linalg.hadamard(D).T
    assert (Q.wht_f32(x).astype(np.float64) == ref).all()
    assert (Q.hadamard_f64(D) == scipy.linalg.hadamard(D)).all()


@pytest.mark.parametrize("D", [64, 128])
def test_rotation_is_orthogonal(D):
    r = _rng(5)
    s = np.where(r.random(D) < 0.5, -1, 1).astype(np.int8)
    x = r.standard_normal((7, D))
    y = Q.rotate_f64(x, s)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(Q.unrotate_f64(y, s), x, atol=1e-12)
    # unit vectors go to +-1/sqrt(D) everywhere
    e0 = np.zeros(D); e0[0] = 1.0
    np.testing.assert_allclose(np.abs(Q.rotate_f64(e0, s)), np.full(D, 1 / np.sqrt(D)), rtol=1e-14)


@pytest.mark.parametrize("D", [64, 128])
def test_lut4_quantizer(D):
    r = _rng(6)
    s = np.where(r.random(D) < 0.5, -1, 1).astype(np.int8)
    cb = CB.lloyd_max_f16(16, 1.0 / np.sqrt(D))
    x = (r.standard_normal((40, D)) * 2).astype(np.float16)
    x[0] = 0
    idx, n = Q.quantize_lut4(x, s, cb)
    # zero vector: norm 0 and every index is the one straddling 0 (symmetric codebook)
    assert n[0] == 0 and (idx[0] == 7).all()
    # the norm is the vector norm (rotation is orthogonal), to fp32 + fp16 precision
    nn = np.linalg.norm(x.astype(np.float64), axis=1)
    np.testing.assert_allclose(n[1:].astype(np.float64), nn[1:], rtol=1e-3)
    # each index is the nearest centroid to the unit-norm rotated coordinate
    u = Q.rotate_f64(x.astype(np.float64), s) / np.maximum(nn, 1e-300)[:, None]
    c = cb.astype(np.float64)
    near = np.argmin(np.abs(u[..., None] - c), axis=-1)
    mid = 0.5 * (c[:-1] + c[1:])
    close = np.min(np.abs(u[..., None] - mid), axis=-1) < 1e-5
    assert ((idx == near) | close)[1:].all()
    assert (idx <= 15).all()
    # reconstruction error is the codebook's: relative MSE close to the Gaussian distortion
    xh = Q.unrotate_f64(Q.dequantize_lut4(idx, n, cb), s)
    rel = np.sum((xh - x.astype(np.float64)) ** 2, axis=1)[1:] / nn[1:] ** 2
    assert 0.003 < rel.mean() < 0.02


def test_lut4_bitexact_against_fp64_where_unambiguous():
    # the fp32 pipeline must agree with an fp64 evaluation of the same steps except
    # for coordinates that sit within rounding of a threshold.
    D = 128
    r = _rng(7)
    s = np.where(r.random(D) < 0.5, -1, 1).astype(np.int8)
    cb = CB.lloyd_max_f16(16, 1.0 / np.sqrt(D))
    x = r.standard_normal((30, D)).astype(np.float16)
    idx, n = Q.quantize_lut4(x, s, cb)
    y = Q.rotate_f64(x.astype(np.float64), s)
    nn = np.linalg.norm(y, axis=1)
    u = y / nn[:, None]
    t = 0.5 * (cb[:-1].astype(np.float64) + cb[1:].astype(np.float64))
    ref = (u[..., None] > t).sum(-1)
    ambiguous = np.min(np.abs(u[..., None] - t), axis=-1) < 1e-6
    assert ((idx == ref) | ambiguous).all()
    assert (n == nn.astype(np.float16)).mean() > 0.95


# ---------------------------------------------------------------- nvfp4

def _e2m1_table_from_bits():
    """E2M1 magnitudes from the bit layout (2 exponent bits, bias 1, 1 mantissa bit;
    exponent 0 is subnormal), independent of the oracle's table."""
    out = []
    for code in range(8):
        e, m = code >> 1, code & 1
        out.append(Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1))
    return out


def _nearest_even_brute(x: Fraction, table):
    best = None
    for i, v in enumerate(table):
        d = abs(x - v)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def test_e4m3_encoding_matches_torch_float8():
    # independent reference: PyTorch's float8_e4m3fn cast (round to nearest even)
    import torch
    rng = np.random.Generator(np.random.PCG64(21))
    t = np.concatenate([rng.random(2000) * 448, np.exp(rng.uniform(-12, 6, 2000)),
                        Q.E4M3_MAGNITUDES, (Q.E4M3_MAGNITUDES[1:] + Q.E4M3_MAGNITUDES[:-1]) / 2])
    t = t[t <= 448].astype(np.float32)
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(Q.e4m3_encode(t), ref)
    assert np.array_equal(Q.e4m3_decode(np.arange(127)),
                          torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy())
    assert Q.e4m3_encode(np.float32([1e4]))[0] == 126           # saturates at 448


def test_e2m1_encoding_brute_force():
    table = _e2m1_table_from_bits()
    assert [float(v) for v in table] == list(Q.E2M1_MAGNITUDES)
    rng = np.random.Generator(np.random.PCG64(22))
    mids = [float((a + b) / 2) for a, b in zip(table[:-1], table[1:])]
    vals = np.concatenate([rng.uniform(-8, 8, 3000), mids, [-m for m in mids], [0.0, -0.0, 6.0, 7.0, -9.0]])
    vals = vals.astype(np.float32)
    got = Q.e2m1_encode(vals)
    for v, c in zip(vals, got):
        mag = _nearest_even_brute(abs(Fraction(float(v))), table)
        want = mag | (8 if np.signbit(v) else 0)
        assert c == want, (v, c, want)


def test_nvfp4_quantizer_steps_exact():
    rng = np.random.Generator(np.random.PCG64(23))
    x = (rng.standard_normal((40, 128)) * rng.choice([0.01, 1.0, 50.0], (40, 1))).astype(np.float16)
    codes, words = Q.quantize_nvfp4(x)
    raw = words.view(np.uint8)
    table = _e2m1_table_from_bits()
    e4 = {i: Fraction(float(v)) for i, v in enumerate(Q.E4M3_MAGNITUDES)}
    for i in range(len(x)):
        xf = [Fraction(float(v)) for v in x[i].astype(np.float32)]
        amax = max(abs(v) for v in xf)
        g = np.float32(raw[i, 8:12].view(np.float32)[0])
        assert abs(Fraction(float(g)) - amax / 2688) <= _ulp32(float(g)) / 2     # fp32(amax / 2688)
        six_g = np.float32(np.float32(6.0) * g)
        for b in range(8):
            blk = xf[16 * b:16 * b + 16]
            t = np.float32(np.float32(max(abs(v) for v in blk)) / six_g)
            sc = raw[i, b]
            assert sc == _nearest_even_brute(Fraction(float(t)), [e4[k] for k in range(127)])
            den = np.float32(g * np.float32(float(e4[sc])))
            for j in range(16):
                v = np.float32(np.float32(float(blk[j])) / den) if den > 0 else np.float32(0.0)
                c = codes[i, 16 * b + j]
                want = _nearest_even_brute(abs(Fraction(float(v))), table) | (8 if np.signbit(v) else 0)
                assert den == 0 or c == want


def test_nvfp4_special_vectors_and_error_bound():
    D = 64
    zero = np.zeros((1, D), dtype=np.float16)
    c, w = Q.quantize_nvfp4(zero)
    assert not c.any() and not w.any()
    # values exactly representable as e2m1 * e4m3 * g round-trip exactly
    x = np.zeros((1, D), dtype=np.float16)
    x[0, :8] = [6, 4, 3, 2, 1.5, 1, 0.5, -6]
    c, w = Q.quantize_nvfp4(x)
    xh = Q.dequantize_nvfp4(c, w)
    assert np.allclose(xh[0, :8], x[0, :8].astype(np.float64), rtol=1e-6)
    # tiny negatives keep their sign bit; reconstruction error within half an e2m1 step
    rng = np.random.Generator(np.random.PCG64(24))
    x = (rng.standard_normal((50, D)) * 2).astype(np.float16)
    c, w = Q.quantize_nvfp4(x)
    xh = Q.dequantize_nvfp4(c, w)
    raw = w.view(np.uint8)
    g = raw[:, 4:8].copy().view(np.float32)[:, 0].astype(np.float64)
    s = Q.e4m3_decode(raw[:, :4]).astype(np.float64)                      # [50, 4]
    unit = (s * g[:, None])[:, :, None]                                     # value of 1.0 per block
    err = np.abs(xh - x.astype(np.float64)).reshape(50, 4, 16)
    mag = np.abs(x.astype(np.float64)).reshape(50, 4, 16) / unit
    step = np.where(mag < 2, 0.5, np.where(mag < 4, 1.0, 2.0))              # e2m1 spacing there
    assert (err <= (step / 2) * unit * (1 + 1e-6) + 1e-12).all()
    assert Q.nvfp4_scale_row_words(128) == 8 and Q.nvfp4_scale_row_words(64) == 4


# ------------------------------------------------------------------ exhaustive fp16 sweep

def _all_finite_fp16():
    """Every finite fp16 value (both zeros, subnormals, normals up to +-65504)."""
    bits = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    v = bits.view(np.float16)
    return v[np.isfinite(v)]


def test_q8_0_q4_0_exhaustive_single_block_sweep():
    # For every finite fp16 value v, the block [v, -v, 0, ..., 0]: a tie of |x| between
    # the first two elements, subnormals, zeros and +-65504 included.  Expected values
    # come from exact rational arithmetic, not from the quantizers' fp32 path.
    v = _all_finite_fp16()
    x = np.zeros((v.size, 32), dtype=np.float16)
    x[:, 0] = v
    x[:, 1] = -v
    c8, d8 = Q.quantize_q8_0(x)
    c4, d4 = Q.quantize_q4_0(x)
    c8 = c8.astype(int)
    c4 = c4.astype(int)
    nz = v != 0
    s = np.sign(v.astype(np.float64)).astype(int)
    # q8_0: the extreme of either sign reaches +-127, the rest stay 0
    assert (c8[nz, 0] == 127 * s[nz]).all() and (c8[nz, 1] == -127 * s[nz]).all()
    assert (c8[:, 2:] == 0).all() and (c8[~nz] == 0).all() and (d8[~nz] == 0).all()
    # q8_0 scale: fp16 of the fp32 value nearest |v| / 127 (checked exactly on every value)
    for val, dh in zip(v[nz][::7], d8[nz][::7, 0]):
        exact = Fraction(abs(float(val))) / 127
        d32 = np.float32(float(exact))  # candidate; must be within half an fp32 ulp of exact
        assert abs(Fraction(float(d32)) - exact) <= _ulp32(float(d32)) / 2
        assert dh == np.float16(d32)
    # q4_0: the first of the tied extremes wins: d = v / -8 (exact, then rounded to fp16),
    # v -> code 0, -v -> 16 clamped to 15, zeros -> 8
    assert (c4[nz, 0] == 0).all() and (c4[nz, 1] == 15).all()
    assert (c4[:, 2:] == 8).all() and (c4[~nz] == 8).all()
    want_d4 = np.array([np.float16(float(Fraction(float(a)) / -8)) for a in v[nz]], dtype=np.float16)
    assert (d4[nz, 0].view(np.uint16) == want_d4.view(np.uint16)).all()
