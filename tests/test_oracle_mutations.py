"""Planted mistakes: each test builds a plausibly wrong variant of one oracle step
(on the CPU) and checks that the pin guarding that step rejects it.  This is the
evidence that the pins are sharp enough to catch a dropped term, a wrong sign
or index, or an off-by-half rounding."""
import math

import numpy as np
import pytest
import scipy.linalg

from oracle import attention as A
from oracle import quant as Q
from tests.test_oracle_quant import check_q8_0, check_q4_0, _blocks
from tests.test_oracle_attention import brute_force_attention


def test_q8_0_truncation_instead_of_rounding_is_caught():
    def bad(x16):
        x = x16.astype(np.float32).reshape(-1, 32)
        d = np.abs(x).max(1) / np.float32(127)
        q = np.trunc(x / d[:, None])
        return q.astype(np.int8).reshape(x16.shape), d.astype(np.float16)[:, None]
    with pytest.raises(AssertionError):
        check_q8_0(bad, _blocks(8, seed=11))


def test_q4_0_missing_half_offset_is_caught():
    def bad(x16):
        x = x16.astype(np.float32).reshape(-1, 32)
        i = np.argmax(np.abs(x), 1)
        d = x[np.arange(len(x)), i] / np.float32(-8)
        q = np.minimum(np.floor(x / d[:, None] + np.float32(8.0)), 15)
        return q.astype(np.uint8).reshape(x16.shape), d.astype(np.float16)[:, None]
    with pytest.raises(AssertionError):
        check_q4_0(bad, _blocks(8, seed=12))


def test_q4_0_unsigned_extreme_is_caught():
    def bad(x16):
        x = x16.astype(np.float32).reshape(-1, 32)
        d = np.abs(x).max(1) / np.float32(-8)        # drops the sign of the extreme
        q = np.minimum(np.floor(x / d[:, None] + np.float32(8.5)), 15)
        return q.astype(np.uint8).reshape(x16.shape), d.astype(np.float16)[:, None]
    with pytest.raises(AssertionError):
        check_q4_0(bad, _blocks(8, seed=13))


def test_wht_missing_stage_is_caught():
    D = 64
    x = np.random.Generator(np.random.PCG64(14)).integers(-9, 9, (3, D)).astype(np.float32)
    y = x.copy()
    h = 1
    while h < D // 2:                                 # last stage dropped
        z = y.reshape(3, D // (2 * h), 2, h)
        y = np.stack([z[:, :, 0] + z[:, :, 1], z[:, :, 0] - z[:, :, 1]], 2).reshape(3, D)
        h *= 2
    assert not np.array_equal(y, x @ scipy.linalg.hadamard(D).T)


def test_combine_without_rescale_is_caught():
    r = np.random.Generator(np.random.PCG64(15))
    q, k, v = r.standard_normal((3, 8)), r.standard_normal((40, 8)) * 3, r.standard_normal((40, 8))
    parts = [(0, 7), (7, 40)]
    os_, ms, ls = [], [], []
    for a, b in parts:
        s = q @ k[a:b].T
        mm = s.max(1)
        p = np.exp(s - mm[:, None])
        os_.append(p @ v[a:b]); ms.append(mm); ls.append(p.sum(1))
    bad = sum(os_) / sum(ls)[:, None]                 # forgets e^{m_s - M}
    dense, _ = A.dense_attention(q, k, v, 1.0)
    assert not np.allclose(bad, dense, rtol=1e-6)


def test_denominator_over_kept_only_is_caught():
    r = np.random.Generator(np.random.PCG64(16))
    q, k, v = r.standard_normal((2, 16)), r.standard_normal((50, 16)), r.standard_normal((50, 16))
    s = (q @ k.T) * 0.25
    # wrong: l sums only kept positions (tau = 1 keeps only split maxima)
    outs = []
    for g in range(2):
        num, den, M = np.zeros(16), 0.0, s[g].max()
        for a in range(0, 50, 12):
            seg = s[g, a:a + 12]
            num += math.exp(seg.max() - M) * v[a + int(np.argmax(seg))]
            den += math.exp(seg.max() - M)
        outs.append(num / den)
    good = A.sparse_v_attention(q, k, v, 0.25, 1.0, 12)["out"]
    assert not np.allclose(np.array(outs), good, rtol=1e-6)


def test_gqa_modulo_mapping_is_caught():
    r = np.random.Generator(np.random.PCG64(17))
    Hq, Hkv, D, N = 8, 2, 16, 20
    q = r.standard_normal((Hq, D))
    k = r.standard_normal((N, Hkv, D))
    v = r.standard_normal((N, Hkv, D))
    hq = 1                                            # floor(1 / 4) = 0, but 1 % 2 = 1
    right = brute_force_attention(q[hq:hq + 1], k[:, hq // (Hq // Hkv)], v[:, hq // (Hq // Hkv)], 0.25)
    wrong = brute_force_attention(q[hq:hq + 1], k[:, hq % Hkv], v[:, hq % Hkv], 0.25)
    assert not np.allclose(right, wrong)
