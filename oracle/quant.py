"""Block quantizers of the KV cache (oracle side; test infrastructure only).

Every quantizer takes float16 vectors ``x[..., D]`` (D a multiple of 32) and
works in IEEE float32 with round-to-nearest-even, one operation at a time, so
that the resulting integer codes are fixed to the bit: numpy float32 array
operations are single IEEE operations, so no fused multiply-add or wider
intermediate can creep in.  Integer decisions (a code, a codebook index) are
taken on these float32 values; the dequantized cache is then formed in fp64.

Formats (the readings this library fixes where the pages give no arithmetic):

q8_0   blocks of 32 along the head dimension.
       amax = max |x_i|;  d = fp32(amax / 127);
       q_i = round-half-away-from-zero(fp32(x_i / d)) clamped to [-127, 127]
       (q = 0 when d == 0);  stored scale = fp16_rne(d);  x_hat = q * d16.
q4_0   blocks of 32.  m = the signed element of largest |x| (lowest index on a tie);
       d = fp32(m / -8);  q_i = min(15, floor(fp32(fp32(x_i / d) + 8.5)))
       (q = 8 when d == 0);  stored scale = fp16_rne(d);  x_hat = (q - 8) * d16.
lut4   rotated 4-bit codebook (TurboQuant-style, Walsh-Hadamard rotation named in
       section "Почему это работает для любой квантизации" of the tproger page).
       y = c * H_D (s (.) x) with s the fixed random signs, H_D the Sylvester
       Hadamard matrix applied as butterfly stages h = 1, 2, ..., D/2 in fp32
       (each pair (a, b) -> (a + b, a - b)), then multiplied by c = fp32(1/sqrt(D));
       ss = pairwise tree sum of fp32(y_i^2) with strides D/2, D/4, ..., 1;
       n = fp32(sqrt(ss));  u_i = fp32(y_i / n)  (u = 0 when n == 0);
       thresholds t_k = fp32(fp32(c_k + c_{k+1}) * 0.5) from the fp16 codebook;
       idx_i = #{k : u_i > t_k};  stored norm = fp16_rne(n);
       x_hat' = n16 * c16[idx]  (in the rotated domain).

nvfp4  (named in the tproger page's opening summary among the schemes the method
       works with; the page gives no arithmetic).  Blocks of 16 along the head
       dimension, E2M1 codes with an E4M3 block scale and a per-vector fp32 scale:
       amax = max |x_i| over the vector;  g = fp32(amax / 2688)  (2688 = 6 * 448, the
       largest E2M1 value times the largest E4M3 value);  per block
       s = e4m3(fp32(amax_b / fp32(6 * g)))  (0 when g == 0);
       code_i = e2m1(fp32(x_i / fp32(g * s)))  (0 when g * s == 0);
       x_hat = e2m1_value(code) * s * g.  e4m3 / e2m1 round to nearest with ties to
       the even code and saturate at the largest finite value (448 / 6); e2m1 keeps
       the sign (a negative value that rounds to zero gives the code of -0).
       Scale row (little-endian bytes): the D/16 E4M3 codes, the 4 bytes of g, zero
       padding to a multiple of 8 bytes.

Packing of 4-bit codes: element 2j in the low nibble of byte j, element 2j+1 in
the high nibble.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
BLOCK = 32


def _blocks(x16: np.ndarray) -> np.ndarray:
    D = x16.shape[-1]
    assert D % BLOCK == 0, "head_dim must be a multiple of 32"
    return x16.astype(np.float32).reshape(x16.shape[:-1] + (D // BLOCK, BLOCK))


def quantize_q8_0(x16: np.ndarray):
    """Return (codes int8 [..., D], scales float16 [..., D/32])."""
    x = _blocks(x16)
    amax = np.abs(x).max(axis=-1)                               # exact
    d = np.divide(amax, F32(127.0), dtype=np.float32)           # one fp32 division
    zero = d == 0
    dsafe = np.where(zero, F32(1.0), d).astype(np.float32)
    t = np.divide(x, dsafe[..., None], dtype=np.float32)        # fp32 x / d
    t64 = t.astype(np.float64)                                  # exact widening
    q = np.sign(t64) * np.floor(np.abs(t64) + 0.5)              # half away from zero (exact in fp64)
    q = np.clip(q, -127, 127)
    q[zero] = 0
    return q.astype(np.int8).reshape(x16.shape), d.astype(np.float16)


def quantize_q4_0(x16: np.ndarray):
    """Return (codes uint8 in [0, 15] [..., D] (unpacked), scales float16 [..., D/32])."""
    x = _blocks(x16)
    i = np.argmax(np.abs(x), axis=-1)                           # first index of the largest |x|
    m = np.take_along_axis(x, i[..., None], axis=-1)[..., 0]    # signed extreme
    d = np.divide(m, F32(-8.0), dtype=np.float32)
    zero = d == 0
    dsafe = np.where(zero, F32(1.0), d).astype(np.float32)
    t = np.divide(x, dsafe[..., None], dtype=np.float32)
    u = np.add(t, F32(8.5), dtype=np.float32)
    q = np.minimum(np.floor(u), 15)
    q[zero] = 8
    return q.astype(np.uint8).reshape(x16.shape), d.astype(np.float16)


def wht_f32(x: np.ndarray) -> np.ndarray:
    """Unnormalized Sylvester-Hadamard transform along the last axis, fp32 butterflies
    in the stage order h = 1, 2, 4, ..., D/2."""
    y = np.array(x, dtype=np.float32, copy=True)
    D = y.shape[-1]
    lead = y.shape[:-1]
    h = 1
    while h < D:
        z = y.reshape(lead + (D // (2 * h), 2, h))
        a = z[..., 0, :]
        b = z[..., 1, :]
        y = np.stack([np.add(a, b, dtype=np.float32), np.subtract(a, b, dtype=np.float32)],
                     axis=-2).reshape(lead + (D,))
        h *= 2
    return y


def rotation_scale_f32(D: int) -> np.float32:
    """c = fp32(1 / sqrt(D)), the constant that makes c * H_D orthogonal."""
    return F32(1.0 / np.sqrt(float(D)))


def quantize_lut4(x16: np.ndarray, signs: np.ndarray, codebook16: np.ndarray):
    """Return (idx uint8 [..., D], norms float16 [...]).

    ``signs``: D entries +1/-1; ``codebook16``: 16 float16 centroids, increasing.
    """
    D = x16.shape[-1]
    s = np.asarray(signs, dtype=np.float32)
    x = np.multiply(x16.astype(np.float32), s, dtype=np.float32)       # exact sign flips
    y = np.multiply(wht_f32(x), rotation_scale_f32(D), dtype=np.float32)
    v = np.multiply(y, y, dtype=np.float32)
    stride = D // 2
    while stride >= 1:
        v = np.add(v[..., :stride], v[..., stride:2 * stride], dtype=np.float32)
        stride //= 2
    n = np.sqrt(v[..., 0], dtype=np.float32)                            # correctly rounded
    zero = n == 0
    nsafe = np.where(zero, F32(1.0), n).astype(np.float32)
    u = np.divide(y, nsafe[..., None], dtype=np.float32)
    u[zero] = 0
    cb = np.asarray(codebook16, dtype=np.float16).astype(np.float32)
    t = np.multiply(np.add(cb[:-1], cb[1:], dtype=np.float32), F32(0.5), dtype=np.float32)
    idx = (u[..., None] > t).sum(axis=-1)
    return idx.astype(np.uint8), n.astype(np.float16)


# ---------------------------------------------------------------- packing

def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., D] values in 0..15 -> [..., D/2] bytes (2j low nibble, 2j+1 high nibble)."""
    c = codes.astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = packed.astype(np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# ---------------------------------------------------------------- dequant (fp64)

def dequantize_q8_0(codes: np.ndarray, scales16: np.ndarray) -> np.ndarray:
    c = codes.astype(np.float64).reshape(codes.shape[:-1] + (codes.shape[-1] // BLOCK, BLOCK))
    return (c * scales16.astype(np.float64)[..., None]).reshape(codes.shape)


def dequantize_q4_0(codes: np.ndarray, scales16: np.ndarray) -> np.ndarray:
    c = (codes.astype(np.float64) - 8.0).reshape(codes.shape[:-1] + (codes.shape[-1] // BLOCK, BLOCK))
    return (c * scales16.astype(np.float64)[..., None]).reshape(codes.shape)


def dequantize_lut4(idx: np.ndarray, norms16: np.ndarray, codebook16: np.ndarray) -> np.ndarray:
    """Rotated-domain reconstruction n * c[idx]."""
    cb = np.asarray(codebook16, dtype=np.float16).astype(np.float64)
    return norms16.astype(np.float64)[..., None] * cb[idx.astype(np.int64)]


def hadamard_f64(D: int) -> np.ndarray:
    """Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(D)
    bits = np.bitwise_and(i[:, None], i[None, :])
    pop = np.zeros_like(bits)
    b = bits.copy()
    while b.any():
        pop += b & 1
        b >>= 1
    return np.where(pop % 2 == 0, 1.0, -1.0)


def rotate_f64(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R x with R = c H diag(s), in fp64 (used for the query)."""
    D = x.shape[-1]
    H = hadamard_f64(D)
    return (np.asarray(x, dtype=np.float64) * signs.astype(np.float64)) @ H.T / np.sqrt(D)


def unrotate_f64(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """R^T y = diag(s) c H y (H is symmetric), in fp64 (used for the output)."""
    D = y.shape[-1]
    H = hadamard_f64(D)
    return (np.asarray(y, dtype=np.float64) @ H.T / np.sqrt(D)) * signs.astype(np.float64)


# ---------------------------------------------------------------- nvfp4

NV_BLOCK = 16
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # codes 0..7; bit 3 = sign


def _e4m3_magnitudes() -> np.ndarray:
    """Value of every non-negative E4M3 code 0..126 (code 127 is NaN): exponent bits 3..6
    with bias 7, three mantissa bits; exponent 0 is subnormal (m / 8) 2^-6."""
    vals = []
    for code in range(127):
        e, m = code >> 3, code & 7
        vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


E4M3_MAGNITUDES = _e4m3_magnitudes()


def _nearest_even(mag: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the increasing `table` (ties -> the even index);
    values beyond the last entry saturate to it."""
    mag = np.asarray(mag, dtype=np.float64)
    dist = np.abs(mag[..., None] - table)            # exact: float32 inputs, exact table
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    idx = np.arange(len(table))
    # among the (at most two, adjacent) nearest entries take the even index
    even = np.where(cand & (idx % 2 == 0), idx, len(table))
    pick = even.min(axis=-1)
    first = np.where(cand, idx, len(table)).min(axis=-1)
    return np.where(pick < len(table), pick, first)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32)
    code = _nearest_even(np.abs(v), E2M1_MAGNITUDES).astype(np.uint8)
    return np.where(np.signbit(v), code | 8, code).astype(np.uint8)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code).astype(np.int64)
    mag = E2M1_MAGNITUDES[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_encode(t: np.ndarray) -> np.ndarray:
    """Non-negative float32 -> E4M3 code (nearest, ties to even, saturating at 448)."""
    return _nearest_even(np.asarray(t, dtype=np.float32), E4M3_MAGNITUDES).astype(np.uint8)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    return E4M3_MAGNITUDES[np.asarray(code).astype(np.int64) & 127]


def nvfp4_scale_row_words(D: int) -> int:
    return (D // NV_BLOCK + 4 + 7) // 8 * 4


def quantize_nvfp4(x16: np.ndarray):
    """Returns (codes [..., D] E2M1 bit patterns, scale rows [..., nvfp4_scale_row_words(D)]
    as uint16 words)."""
    x = np.asarray(x16).astype(np.float32)
    D = x.shape[-1]
    assert D % NV_BLOCK == 0
    xb = x.reshape(x.shape[:-1] + (D // NV_BLOCK, NV_BLOCK))
    amax = np.abs(x).max(axis=-1)                                   # [...]
    g = (amax / F32(2688.0)).astype(np.float32)
    six_g = (F32(6.0) * g).astype(np.float32)
    amax_b = np.abs(xb).max(axis=-1)                                # [..., B]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(six_g[..., None] > 0, amax_b / six_g[..., None], F32(0.0)).astype(np.float32)
    sc = e4m3_encode(t)                                             # [..., B]
    s = e4m3_decode(sc).astype(np.float32)
    den = (g[..., None] * s).astype(np.float32)                     # [..., B]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(den[..., None] > 0, xb / den[..., None], F32(0.0)).astype(np.float32)
    codes = np.where(den[..., None] > 0, e2m1_encode(v), np.uint8(0)).reshape(x.shape)
    nw = nvfp4_scale_row_words(D)
    row = np.zeros(x.shape[:-1] + (2 * nw,), dtype=np.uint8)
    row[..., : D // NV_BLOCK] = sc
    row[..., D // NV_BLOCK: D // NV_BLOCK + 4] = g[..., None].view(np.uint8)
    return codes.astype(np.int64), row.view(np.uint16)


def dequantize_nvfp4(codes: np.ndarray, words: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes)
    D = codes.shape[-1]
    raw = np.ascontiguousarray(np.asarray(words, dtype=np.uint16)).view(np.uint8)
    sc = raw[..., : D // NV_BLOCK]
    g = np.ascontiguousarray(raw[..., D // NV_BLOCK: D // NV_BLOCK + 4]).view(np.float32)[..., 0]
    s = e4m3_decode(sc).astype(np.float64)
    vals = e2m1_decode(codes).reshape(codes.shape[:-1] + (D // NV_BLOCK, NV_BLOCK))
    return (vals * s[..., None] * g.astype(np.float64)[..., None, None]).reshape(codes.shape)


# ---------------------------------------------------------------- whole cache

def quantize(fmt: str, x16: np.ndarray, signs=None, codebook16=None):
    """Logical planes of one cache tensor: (codes [..., D] unpacked ints, scales fp16)."""
    if fmt == "q8_0":
        return quantize_q8_0(x16)
    if fmt == "q4_0":
        return quantize_q4_0(x16)
    if fmt == "lut4":
        idx, n = quantize_lut4(x16, signs, codebook16)
        return idx, n[..., None]
    if fmt == "nvfp4":
        return quantize_nvfp4(x16)
    raise ValueError(fmt)


def dequantize(fmt: str, codes, scales16, codebook16=None) -> np.ndarray:
    if fmt == "q8_0":
        return dequantize_q8_0(codes, scales16)
    if fmt == "q4_0":
        return dequantize_q4_0(codes, scales16)
    if fmt == "lut4":
        return dequantize_lut4(codes, scales16[..., 0], codebook16)
    if fmt == "nvfp4":
        return dequantize_nvfp4(codes, scales16)
    raise ValueError(fmt)
