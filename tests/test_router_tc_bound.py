"""Host restatement of the tensor-core router's fixed-point slices and of its bound (no GPU).

The kernel (route_tc.cu) writes each bf16 row v as X_i = rint(v_i 2^q) with q = 148 - e1
(e1: the row's largest biased exponent, at least 1), splits X = 2^16 h + 2^8 m + l into int8
slices, multiplies the slices pairwise into five int32 accumulators by pair weight, and bounds
|l - l~| by 2^-(qx+qw) (Sx/2 + Sw/2 + H/4), S = sum |X|, where l~ = 2^-(qx+qw) sum_s 2^(8(4-s)) A_s.
These tests restate those rules from the bf16 bit patterns and check, with exact rational
arithmetic, that the slices are in range and recompose X, that the accumulators fit int32 and
recompose sum X W, that the Horner partial sums stay below the bound the kernel uses for their
fp64 roundings, and that the logit bound holds on random and adversarial rows.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def quantize_row(bits):
    e = (bits.astype(np.int64) >> 7) & 0xFF
    emax = int(e.max()) if bits.size else 0
    e1 = emax if emax > 0 else 1
    q = 148 - e1
    m8 = np.where(e > 0, 0x80 | (bits & 0x7F), bits & 0x7F).astype(np.int64)
    sh = np.where(e > 0, e, 1) - e1 + 14
    X = np.zeros(bits.shape, np.int64)
    for i in range(bits.size):
        s = int(sh[i])
        m = int(m8[i])
        if s >= 0:
            v = m << s
        elif s < -8:
            v = 0
        else:
            k = -s
            q0, rem, half = m >> k, m & ((1 << k) - 1), 1 << (k - 1)
            v = q0 + (1 if (rem > half or (rem == half and (q0 & 1))) else 0)
        X[i] = -v if bits[i] & 0x8000 else v
    X1 = (X + 128) >> 8
    lo = X - X1 * 256
    hi = (X1 + 128) >> 8
    mi = X1 - hi * 256
    return q, X, (hi, mi, lo)


def exact(bits):
    """bf16 bit patterns -> exact Fractions."""
    out = []
    for b in bits.tolist():
        e = (b >> 7) & 0xFF
        m = (0x80 | (b & 0x7F)) if e else (b & 0x7F)
        v = Fraction(m) * Fraction(2) ** ((e if e else 1) - 134)
        out.append(-v if b & 0x8000 else v)
    return out


def check_pair(xb, wb):
    qx, X, xs_ = quantize_row(xb)
    qw, Wq, ws_ = quantize_row(wb)
    for Y, (h, m, l) in ((X, xs_), (Wq, ws_)):
        assert np.all(np.abs(Y) < 1 << 22)
        assert np.all((h >= -64) & (h <= 64))
        assert np.all((m >= -128) & (m <= 127)) and np.all((l >= -128) & (l <= 127))
        assert np.array_equal(65536 * h + 256 * m + l, Y)
        assert np.all(np.abs(h) * 65536 + np.abs(m) * 256 + np.abs(l) <= np.abs(Y) + (1 << 17))
    acc = [0] * 5
    for i in range(3):
        for j in range(3):
            acc[i + j] += int(np.dot(ws_[i].astype(np.int64), xs_[j].astype(np.int64)))
    for a in acc:
        assert abs(a) < 1 << 31
    v, big = 0, int(np.dot(np.abs(X) + (1 << 17), np.abs(Wq) + (1 << 17)))
    for k, a in enumerate(acc):                     # the kernel's Horner steps, exactly
        v = v * 256 + a
        assert abs(v) * (1 << (8 * (4 - k))) <= big
    assert v == int(np.dot(X, Wq))
    scale = Fraction(2) ** (-(qx + qw))
    l_tilde = scale * v
    xs, ws = exact(xb), exact(wb)
    l = sum(a * b for a, b in zip(xs, ws))
    H = xb.size
    bound = scale * (Fraction(int(np.abs(X).sum()), 2) + Fraction(int(np.abs(Wq).sum()), 2) + Fraction(H, 4))
    assert abs(l - l_tilde) <= bound
    for vals, q, Y in ((xs, qx, X), (ws, qw, Wq)):   # each value within half a step of its grid point
        step = Fraction(2) ** (-q)
        assert all(abs(a - int(y) * step) <= step / 2 for a, y in zip(vals, Y.tolist()))
    return abs(l - l_tilde), bound


def bits_of(vals):
    return oracle.round_bf16(np.asarray(vals, np.float64))


@pytest.mark.parametrize("seed", range(6))
def test_random_rows(seed):
    rng = np.random.default_rng(seed)
    H = 256
    x = bits_of(rng.normal(0.0, 1.0, H))
    w = bits_of(rng.normal(0.0, 0.02, H))
    err, bound = check_pair(x, w)
    assert err <= bound


def test_wide_range_subnormals_zeros_and_extremes():
    rng = np.random.default_rng(9)
    H = 192
    xv = rng.normal(0.0, 1.0, H) * np.exp2(rng.integers(-40, 2, H))
    xv[:4] = [64.0, -64.0, 0.0, -0.0]
    x = bits_of(xv)
    x[10:14] = [0x0001, 0x8003, 0x007F, 0x0080]        # subnormals and the smallest normal
    wv = rng.normal(0.0, 0.02, H) * np.exp2(rng.integers(-30, 1, H))
    w = bits_of(wv)
    w[20:22] = [0x7F7F, 0xFF7F]                        # the largest finite bf16 values
    check_pair(x, w)


def test_zero_and_constant_rows():
    H = 64
    z = np.zeros(H, np.uint16)
    one = bits_of(np.ones(H))
    assert check_pair(z, one)[0] == 0
    assert check_pair(one, one)[0] == 0                # powers of two are exact on the grid
    q, X, _ = quantize_row(one)
    assert q == 148 - 127 and np.all(X == 1 << 21)


def test_the_bound_is_nearly_reached_and_a_dropped_term_is_caught():
    """x = one value 64 and H-1 values 239 * 2^-20 (each rounds down by 0.47 of its grid step),
    w = 2^-6 everywhere (exact on its grid): the error is 0.47/0.5 of the w~.dx term, so the
    bound is nearly tight and the bound without that term fails."""
    H = 128
    x = np.full(H, (114 << 7) | (239 & 0x7F), np.uint16)   # 239 * 2^(114 - 134)
    x[0] = bits_of([64.0])[0]
    w = bits_of(np.full(H, 2.0 ** -6))
    err, bound = check_pair(x, w)
    qx, X, _ = quantize_row(x)
    qw, Wq, _ = quantize_row(w)
    w_term = Fraction(2) ** (-(qx + qw)) * Fraction(int(np.abs(Wq).sum()), 2)
    assert err > Fraction(9, 10) * w_term
    assert err > bound - w_term
