"""Pins of the oracle's NVFP4 (W4A4) functions against what the format and the
mathematics fix: brute-force nearest-grid rounding, the format's closed-form
decode, exact round trips of representable tensors, error bounds, the nibble
packing order, and identity experts whose output has a closed form.

NVFP4 here is NVIDIA's published format (the pages name it for the W4A4
release without defining it): E2M1 elements, one E4M3 scale per 16
elements along the contraction dimension, one fp32 scale per tensor.
"""
import numpy as np
import pytest

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def brute_e2m1(v: float) -> int:
    """Nearest of the 8 magnitudes by distance; ties to the even code; saturate at 6."""
    a = abs(float(v))
    d = np.abs(GRID - min(a, 6.0))
    best = np.flatnonzero(d == d.min())
    c = int(best[0]) if len(best) == 1 else int(next(b for b in best if b % 2 == 0))
    return (8 if np.signbit(v) else 0) | c


def f32(x):
    return np.float32(x)


def bf16_bits(v):
    """Exact bf16 bits of values that are representable in bf16."""
    a = np.asarray(v, dtype=np.float32)
    bits = a.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "value not representable in bf16"
    return (bits >> 16).astype(np.uint16)


def test_e2m1_decode_matches_the_format_definition():
    q = np.arange(16, dtype=np.uint8)
    s, e, m = q >> 3, (q >> 1) & 3, q & 1
    ref = np.where(e == 0, m * 0.5, 2.0 ** (e - 1.0) * (1 + m / 2.0)) * np.where(s == 1, -1.0, 1.0)
    assert np.array_equal(oracle.e2m1_decode(q).astype(np.float64), ref)


def test_e2m1_encode_is_nearest_with_ties_to_even():
    rng = np.random.default_rng(5)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    vals = np.concatenate([GRID, mids, np.nextafter(mids, 0), np.nextafter(mids, 10), [6.5, 100.0, 1e-30],
                           rng.uniform(0, 7, 3000)]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    got = oracle.e2m1_encode(vals)
    ref = np.array([brute_e2m1(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_representable_tensor_round_trips():
    """Blocks built from grid values times a power of two, each reaching 6 * 2^k: the
    codes are exactly the grid codes, and the values come back to within the fp32
    rounding of the tensor scale amax / 2688 (2688 = 2^7 * 21 is not a power of two)."""
    rng = np.random.default_rng(6)
    rows, K = 8, 64
    x = np.empty((rows, K), np.float32)
    for r in range(rows):
        for b in range(K // 16):
            k = int(rng.integers(-6, 4))
            blk = rng.choice(GRID, 16) * rng.choice([-1.0, 1.0], 16)
            blk[int(rng.integers(16))] = 6.0   # every block reaches 6 * 2^k
            x[r, b * 16:(b + 1) * 16] = blk * 2.0 ** k
    bits = bf16_bits(x)
    s_t = oracle.nvfp4_tensor_scale(bits)
    codes, scales = oracle.quantize_nvfp4(bits, s_t)
    q = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(rows, K)
    mag = np.abs(x) / (np.max(np.abs(x.reshape(rows, K // 16, 16)), axis=2, keepdims=True) / 6.0).repeat(16, 2).reshape(rows, K)
    ref_codes = np.array([brute_e2m1(np.copysign(m, v)) for m, v in zip(mag.ravel(), x.ravel())]).reshape(rows, K)
    assert np.array_equal(q, ref_codes)
    deq = oracle.dequantize_nvfp4(codes, scales, s_t)
    assert np.all(np.abs(deq - x) <= 2.0 ** -22 * np.abs(x))


def test_block_maximum_encodes_to_six_and_errors_are_bounded():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)      # truncation gives bf16 values
    xv = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    s_t = oracle.nvfp4_tensor_scale(bits)
    assert s_t == f32(f32(np.max(np.abs(xv))) / f32(2688.0))
    codes, scales = oracle.quantize_nvfp4(bits, s_t)
    deq = oracle.dequantize_nvfp4(codes, scales, s_t)
    S = oracle.e4m3_decode(scales).astype(np.float64)
    e = np.repeat(np.float32(S) * s_t, 16, axis=1).astype(np.float64)           # fl32(S_b * s_t)
    q = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(16, 256)
    blocks = np.abs(xv).reshape(16, 16, 16)
    qb = q.reshape(16, 16, 16)
    amax_pos = blocks.argmax(axis=2)
    top = np.take_along_axis(qb, amax_pos[..., None], axis=2)[..., 0] & 7
    assert np.all(top == 7)                                    # the block maximum maps to +-6
    err = np.abs(xv - deq)
    mag = np.abs(xv) / e
    half = np.where(mag < 2, 0.25, np.where(mag < 4, 0.5, 1.0)) * e   # half the grid spacing
    assert np.all(err <= half * (1 + 1e-12) + 1e-300)
    assert np.all(np.sign(deq) * np.sign(xv) >= 0)


def test_packing_puts_the_even_element_in_the_low_nibble():
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = [6.0, 0.5, 1.0, 0.0, 2.0, 3.0, 4.0, 1.5] * 2
    x[0, 16] = 6.0
    bits = bf16_bits(x)
    codes, scales = oracle.quantize_nvfp4(bits, oracle.nvfp4_tensor_scale(bits))
    assert codes[0, 0] == (7 | (1 << 4)) and codes[0, 1] == (2 | (0 << 4))
    assert codes[0, 2] == (4 | (5 << 4)) and codes[0, 3] == (6 | (3 << 4))
    assert scales[0, 1] == scales[0, 0] and np.all(codes[0, 9:] == 0)


def test_zero_blocks_and_tensor():
    z = np.zeros((2, 32), np.uint16)
    assert oracle.nvfp4_tensor_scale(z) == f32(1.0)
    codes, scales = oracle.quantize_nvfp4(z, f32(1.0))
    assert not codes.any() and not scales.any()


def quant_dequant_fp32(a32, th):
    """fp32 row -> NVFP4 (blocks of 16, tensor scale th) -> dequantised fp64, from the
    pinned E2M1 / E4M3 encoders and the format's rules."""
    out = np.empty(a32.shape[0])
    for b in range(a32.shape[0] // 16):
        blk = a32[b * 16:(b + 1) * 16]
        amax = np.float32(np.max(np.abs(blk)))
        S = oracle.e4m3_decode(oracle.e4m3_encode(np.array([f32(f32(amax / f32(6.0)) / th)], np.float32)))[0]
        e = f32(f32(S) * th)
        q = oracle.e2m1_encode((blk / e).astype(np.float32)) if e != 0 else np.zeros(16, np.uint8)
        out[b * 16:(b + 1) * 16] = oracle.e2m1_decode(q).astype(np.float64) * float(S) * float(th)
    return out


@pytest.mark.parametrize("c", [1.0, 2.0, 0.25])
def test_identity_experts_have_a_closed_form(c):
    """W_up[e] = c [I | 0], W_down[e] = [I ; 0]: each dequantises to a diagonal (c and 1
    up to the rounding of the tensor scale), so z_f = w_ff x_f, y_j = deq(H)_j for j < F
    and y_j = 0 beyond."""
    H, F, E = 64, 32, 2
    wu = np.zeros((E, F, H), np.float32)
    wd = np.zeros((E, H, F), np.float32)
    for e in range(E):
        wu[e, :, :F] = c * np.eye(F)
        wd[e, :F, :] = np.eye(F)
    bank_up = oracle.quantize_bank_nvfp4(bf16_bits(wu))
    bank_down = oracle.quantize_bank_nvfp4(bf16_bits(wd))
    Wu = oracle.dequantize_nvfp4(bank_up[0][0], bank_up[1][0], bank_up[2][0])
    Wd = oracle.dequantize_nvfp4(bank_down[0][0], bank_down[1][0], bank_down[2][0])
    assert np.count_nonzero(Wu) == F and np.count_nonzero(Wd) == F
    assert np.all(np.abs(np.diag(Wu[:, :F]) - c) <= 2.0 ** -22 * c)
    rng = np.random.default_rng(8)
    x = bf16_bits(np.round(rng.standard_normal((3, H)) * 8) / 8)
    tx, th = f32(0.01), f32(0.02)
    cx, sx = oracle.quantize_nvfp4(x, tx)
    dx = oracle.dequantize_nvfp4(cx, sx, tx)
    y = oracle.expert_rows_nvfp4(cx, sx, np.array([0, 1, 0], np.int32), bank_up, bank_down,
                                 np.array([0, 1], np.int32), tx, th)
    assert not y[:, F:].any()
    for r in range(3):
        a32 = np.float32(np.maximum(np.diag(Wu[:, :F]) * dx[r, :F], 0.0) ** 2)
        ref = np.diag(Wd[:F, :]) * quant_dequant_fp32(a32, th)
        assert np.max(np.abs(y[r, :F] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_expert_equals_dense_products_of_dequantised_tensors():
    """The expert's two contractions against numpy matmuls of the dequantised banks
    (random weights), with the hidden row quantised by the pinned encoders."""
    rng = np.random.default_rng(9)
    H, F = 96, 48
    wu = (rng.standard_normal((1, F, H)) * 0.05).astype(np.float32)
    wd = (rng.standard_normal((1, H, F)) * 0.05).astype(np.float32)
    to_bits = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)
    bank_up = oracle.quantize_bank_nvfp4(to_bits(wu))
    bank_down = oracle.quantize_bank_nvfp4(to_bits(wd))
    x = to_bits(rng.standard_normal((2, H)).astype(np.float32))
    tx = oracle.nvfp4_tensor_scale(x)
    th = f32(0.05)
    cx, sx = oracle.quantize_nvfp4(x, tx)
    y = oracle.expert_rows_nvfp4(cx, sx, np.zeros(2, np.int32), bank_up, bank_down, np.array([0], np.int32), tx, th)
    Wu = oracle.dequantize_nvfp4(bank_up[0][0], bank_up[1][0], bank_up[2][0])
    Wd = oracle.dequantize_nvfp4(bank_down[0][0], bank_down[1][0], bank_down[2][0])
    dx = oracle.dequantize_nvfp4(cx, sx, tx)
    a = np.maximum(dx @ Wu.T, 0.0) ** 2
    for r in range(2):
        ref = Wd @ quant_dequant_fp32(np.float32(a[r]), th)
        assert np.max(np.abs(y[r] - ref)) <= 1e-9 * max(1.0, np.max(np.abs(ref)))
