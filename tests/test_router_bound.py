"""CPU pins of the arithmetic behind the certified router of token batches.

The router of 64 tokens and more writes router rows and tokens as scaled
integers q (|q| < 2^30) in four signed base-256 digits, forms every logit from
the 16 exact digit products, and certifies its top-K selection with a bound
eps on the logit's error:

    eps = ||W_e - wh_e|| ||x_t|| + ||wh_e|| ||x_t - xh_t||
          + 7u max|W_e| sqrt(H) ||xh_t|| + 2u |v|,          u = 2^-53

These tests restate that arithmetic in numpy, independently of the CUDA
code, and check it against exact rational arithmetic (fractions.Fraction):
the digits reconstruct q exactly and stay in [-128, 127], the 16 scaled digit
products sum to qw . qx exactly, and the computed logit lies within eps of
the exact logit Wr_e . x_t + b_e, on random rows and on rows chosen to stress
the bound (wide dynamic range, subnormal values, one dominant element).
"""
import zlib
from fractions import Fraction

import numpy as np
import pytest

U = 2.0 ** -53
NORM_UP = 1.0 + 1e-10


def split_rows(rows):
    """Per row: scale exponent s with max|row| 2^-s in [2^29, 2^30), q = rint(row 2^-s),
    and the four signed base-256 digits of q (digit 0 most significant)."""
    rows = np.asarray(rows, dtype=np.float64)
    s = np.zeros(rows.shape[0], dtype=np.int64)
    for i, r in enumerate(rows):
        amax = np.abs(r).max()
        if amax > 0:
            s[i] = np.frexp(np.float32(amax))[1] - 30
    q = np.rint(np.ldexp(rows, -s[:, None])).astype(np.int64)
    d = np.zeros((4,) + q.shape, dtype=np.int64)
    rest = q.copy()
    for p in (3, 2, 1):
        d[p] = ((rest & 0xFF) ^ 0x80) - 0x80
        rest = (rest - d[p]) >> 8
    d[0] = rest
    return s, q, d


def logits(wr, bias, x):
    """Logits as the certified router forms them (exact digit products, three
    fp64 additions of the digit-plane terms, scale, bias) and their bounds."""
    H = wr.shape[1]
    r, qw, dw = split_rows(wr)
    s, qx, dx = split_rows(x)
    P = np.einsum("peh,qth->pqte", dw, dx)  # exact int64
    w8 = [2.0 ** 24, 2.0 ** 16, 2.0 ** 8, 1.0]
    term = [sum(P[p, q].astype(np.float64) * w8[q] for q in range(4)) * w8[p] for p in range(4)]
    v = ((term[0] + term[1]) + term[2]) + term[3]
    v = np.ldexp(v, s[:, None] + r[None, :]) + np.asarray(bias, dtype=np.float64)[None, :]
    wh = np.ldexp(qw.astype(np.float64), r[:, None])
    xh = np.ldexp(qx.astype(np.float64), s[:, None])
    wd = np.sqrt(((wr - wh) ** 2).sum(1)) * NORM_UP
    wq = np.sqrt((wh ** 2).sum(1)) * NORM_UP
    wg = 7 * U * np.abs(wr).max(1) * np.sqrt(H) * NORM_UP
    xn = np.sqrt((x ** 2).sum(1)) * NORM_UP
    xd = np.sqrt(((x - xh) ** 2).sum(1)) * NORM_UP
    xq = np.sqrt((xh ** 2).sum(1)) * NORM_UP
    eps = (wd[None] * xn[:, None] + wq[None] * xd[:, None] + wg[None] * xq[:, None]) * (1 + 1e-9) \
        + 2.3e-16 * np.abs(v) + 1e-300
    return v, eps, (qw, dw, qx, dx, P)


def exact(wr, bias, x, t, e):
    return sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(wr[e], x[t])) + Fraction(float(bias[e]))


def test_digits_reconstruct_and_stay_in_range():
    rng = np.random.default_rng(1)
    q = np.concatenate([rng.integers(-(2 ** 30) + 64, 2 ** 30 - 64, 20000),
                        np.array([0, 1, -1, 127, 128, -128, -129, 2 ** 30 - 64, -(2 ** 30) + 64])])
    rows = q.astype(np.float64)[None, :] * 2.0 ** -40  # the scale of this row maps its largest back to q
    s, qq, d = split_rows(rows)
    assert np.array_equal(qq[0], np.rint(np.ldexp(rows[0], -s[0])).astype(np.int64))
    assert d.min() >= -128 and d.max() <= 127
    assert np.abs(d[0]).max() <= 65
    assert np.array_equal(d[0] * 2 ** 24 + d[1] * 2 ** 16 + d[2] * 2 ** 8 + d[3], qq)


def test_digit_bytes_equal_the_offset_word_form():
    """The GPU extracts the four digits as the bytes of (q + 0x808080) xor 0x808080."""
    rng = np.random.default_rng(2)
    q = rng.integers(-(2 ** 30) + 64, 2 ** 30 - 64, 50000)
    _, _, d = split_rows(q.astype(np.float64)[None, :] * 2.0 ** -31)
    qq = split_rows(q.astype(np.float64)[None, :] * 2.0 ** -31)[1][0]
    word = ((qq + 0x808080) & 0xFFFFFFFF) ^ 0x808080
    for p in range(4):
        byte = (word >> (8 * (3 - p))) & 0xFF
        assert np.array_equal(np.where(byte >= 128, byte - 256, byte), d[p][0])


def test_digit_products_sum_to_the_integer_dot_product():
    rng = np.random.default_rng(3)
    wr = rng.standard_normal((5, 256)).astype(np.float32).astype(np.float64)
    x = rng.standard_normal((4, 256)).astype(np.float32).astype(np.float64)
    _, _, (qw, dw, qx, dx, P) = logits(wr, np.zeros(5), x)
    total = sum(P[p, q] * 2 ** (8 * (6 - p - q)) for p in range(4) for q in range(4))
    ref = np.array([[sum(int(a) * int(b) for a, b in zip(qx[t], qw[e])) for e in range(5)] for t in range(4)])
    assert np.array_equal(total, ref)
    assert np.abs(P).max() < 2 ** 31  # int32 accumulation cannot overflow


def _rows(kind, n, H, rng):
    if kind == "gauss_f32":
        return rng.standard_normal((n, H)).astype(np.float32).astype(np.float64)
    if kind == "gauss_bf16":
        f = rng.standard_normal((n, H)).astype(np.float32)
        b = ((f.view(np.uint32) + 0x7FFF + ((f.view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint32) << 16
        return b.view(np.float32).astype(np.float64)
    if kind == "wide_range":  # magnitudes over 2^-40 .. 2^10
        return (rng.standard_normal((n, H)) * np.exp2(rng.uniform(-40, 10, (n, H)))).astype(np.float32).astype(np.float64)
    if kind == "subnormal":
        return (rng.standard_normal((n, H)) * 2.0 ** -140).astype(np.float32).astype(np.float64)
    if kind == "one_dominant":
        r = rng.standard_normal((n, H)) * 1e-3
        r[:, 7] = 1e4
        return r.astype(np.float32).astype(np.float64)
    raise ValueError(kind)


@pytest.mark.parametrize("wkind,xkind", [("gauss_f32", "gauss_f32"), ("gauss_f32", "gauss_bf16"),
                                         ("wide_range", "gauss_f32"), ("gauss_f32", "wide_range"),
                                         ("subnormal", "one_dominant"), ("one_dominant", "subnormal")])
def test_logit_error_within_the_bound(wkind, xkind):
    rng = np.random.default_rng(zlib.crc32(f"{wkind}/{xkind}".encode()))
    H, E, T = 192, 6, 5
    wr = _rows(wkind, E, H, rng) * 0.02
    wr = wr.astype(np.float32).astype(np.float64)
    x = _rows(xkind, T, H, rng)
    bias = rng.standard_normal(E).astype(np.float32).astype(np.float64)
    v, eps, _ = logits(wr, bias, x)
    for t in range(T):
        for e in range(E):
            err = abs(Fraction(float(v[t, e])) - exact(wr, bias, x, t, e))
            assert err <= Fraction(float(eps[t, e])), (t, e, float(err), eps[t, e])


def test_bound_is_tight_enough_to_certify_typical_logits():
    """At the full hidden size with N(0, 0.02) router rows and N(0, 1) tokens the
    bound is about 5e-8, far below the typical gap between the 8th and 9th
    largest of 256 logits (~0.1 of their spread of ~1.6)."""
    rng = np.random.default_rng(5)
    H = 6144
    wr = (rng.standard_normal((4, H)) * 0.02).astype(np.float32).astype(np.float64)
    x = rng.standard_normal((2, H)).astype(np.float32).astype(np.float64)
    _, eps, _ = logits(wr, np.zeros(4), x)
    assert eps.max() < 2e-7
