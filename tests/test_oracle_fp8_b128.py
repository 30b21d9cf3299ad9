"""Pins of the oracle's FP8_B128 experts (bloomery issue page, section 3 "Kernel
dispatch" and the FP8 release: FP8_B128 scales, the 64-value tail of K = 1856,
physical K 1920).  Reading: E4M3 codes with one fp32 scale per block of 128
consecutive values along K of each row, K zero-padded to a multiple of 128,
block scale amax / 448 over the block's real values; a scalar scale maps to
FP8_B128 as equal block scales; activations keep static scalar scales.

The pins: scalar scales mapped to FP8_B128 reproduce the scalar-scale expert;
block scales and codes against torch's E4M3 conversion; exact round trips of
representable blocks; one block's scale moves alone; the padded tail changes
nothing; and the expert against numpy products of the dequantised operands.
"""
import numpy as np
import torch

import oracle

F32 = np.float32


def bf16(a):
    """fp32 values -> bf16 bits (round to nearest even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def vals(bits):
    return oracle.bf16_to_f64(bits)


def torch_e4m3(v32):
    """Saturating E4M3 codes: torch rounds to nearest even but turns values past 448 into NaN,
    so clip first (for finite values saturation is the same as clipping)."""
    v = np.clip(np.ascontiguousarray(v32, dtype=np.float32), -448.0, 448.0)
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def rand_bank(rng, n, rows, K, sigma=0.02):
    return bf16(rng.standard_normal((n, rows, K)) * sigma)


def test_scalar_scales_map_to_b128_and_reproduce_the_scalar_expert():
    """The normaliser's mapping: per-tensor codes and scale as equal block scales give the
    scalar-scale expert (F = 192 has a 64-value tail block)."""
    rng = np.random.default_rng(21)
    H, F, n = 256, 192, 3
    wu, wd = rand_bank(rng, n, F, H), rand_bank(rng, n, H, F)
    qu, su = oracle.quantize_bank_fp8(wu)
    qd, sd = oracle.quantize_bank_fp8(wd)
    bu = oracle.scalar_to_fp8_b128(qu, su, H)
    bd = oracle.scalar_to_fp8_b128(qd, sd, F)
    assert bd[0].shape == (n, H, 256) and not bd[0][..., F:].any()
    x = bf16(rng.standard_normal((5, H)))
    sx, sh = F32(0.01), F32(0.002)
    ex = np.array([0, 2, 1, 2, 0], np.int32)
    slot = oracle.identity_slot(n)
    ref = oracle.expert_rows_fp8(oracle.quantize_act_fp8(x, sx), ex, qu, su, qd, sd, slot, sx, sh)
    got = oracle.expert_rows_fp8_b128(oracle.quantize_act_fp8_b128(x, sx), ex, bu, bd, slot, sx, sh, H, F)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_block_scales_and_codes_against_torch_e4m3():
    rng = np.random.default_rng(22)
    rows, K = 6, 1856
    w = bf16(rng.standard_normal((rows, K)) * 0.05)
    w[2, 128:256] = 0                                   # an all-zero block
    w[3, 1800] = bf16(np.array([7.5], np.float32))[0]   # a large value in the 64-value tail block
    q, s = oracle.quantize_fp8_b128(w)
    assert q.shape == (rows, 1920) and s.shape == (rows, 15)
    assert not q[:, K:].any()                           # padding codes are zero
    wv = vals(w).astype(np.float32)
    for b in range(15):
        k0, k1 = b * 128, min(b * 128 + 128, K)
        amax = np.max(np.abs(wv[:, k0:k1]), axis=1)
        exp = np.where(amax > 0, (amax / F32(448.0)).astype(np.float32), F32(1.0))
        assert np.array_equal(s[:, b], exp)
        assert np.array_equal(q[:, k0:k1], torch_e4m3((wv[:, k0:k1] / exp[:, None]).astype(np.float32)))
    assert s[3, 14] == F32(F32(7.5) / F32(448.0))       # the tail block's scale comes from its 64 values
    assert s[2, 1] == 1.0 and not q[2, 128:256].any()


def test_representable_blocks_round_trip_exactly():
    """Blocks of E4M3 values times 2^k whose maximum is 448 * 2^k: scale 2^k, exact codes."""
    rng = np.random.default_rng(23)
    grid = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float64)
    grid = grid[np.isfinite(grid)]
    rows, K = 4, 320                                    # 2.5 blocks
    x = np.empty((rows, K))
    for r in range(rows):
        for b in range(3):
            k0, k1 = b * 128, min(b * 128 + 128, K)
            kexp = int(rng.integers(-12, -4))
            blk = rng.choice(grid, k1 - k0) * rng.choice([-1.0, 1.0], k1 - k0)
            blk[int(rng.integers(k1 - k0))] = 448.0
            x[r, k0:k1] = blk * 2.0 ** kexp
    bits = bf16(x)
    assert np.array_equal(vals(bits), x)                # E4M3 values times 2^k are bf16 values
    q, s = oracle.quantize_fp8_b128(bits)
    deq = oracle.e4m3_decode(q).astype(np.float64) * np.repeat(s.astype(np.float64), 128, axis=1)
    assert np.array_equal(deq[:, :K], x)


def test_one_block_scale_moves_alone():
    rng = np.random.default_rng(24)
    w = bf16(rng.standard_normal((3, 640)) * 0.03)
    q0, s0 = oracle.quantize_fp8_b128(w)
    w2 = w.copy()
    w2[1, 256:384] = bf16(vals(w[1, 256:384]) * 4.0)    # exact: a power of two
    q1, s1 = oracle.quantize_fp8_b128(w2)
    assert np.array_equal(q0, q1)
    changed = s0 != s1
    assert changed.sum() == 1 and changed[1, 2] and s1[1, 2] == 4 * s0[1, 2]


def test_padding_the_input_to_physical_K_changes_nothing():
    rng = np.random.default_rng(25)
    w = bf16(rng.standard_normal((4, 1856)) * 0.02)
    wp = np.zeros((4, 1920), np.uint16)
    wp[:, :1856] = w
    q, s = oracle.quantize_fp8_b128(w)
    qp, sp = oracle.quantize_fp8_b128(wp)
    assert np.array_equal(q, qp) and np.array_equal(s, sp)


def test_expert_equals_numpy_products_of_dequantised_operands():
    rng = np.random.default_rng(26)
    H, F, n = 384, 320, 2                               # F: two blocks and a 64-value tail
    wu, wd = rand_bank(rng, n, F, H), rand_bank(rng, n, H, F)
    bu, bd = oracle.quantize_fp8_b128(wu), oracle.quantize_fp8_b128(wd)
    x = bf16(rng.standard_normal((3, H)))
    sx, sh = F32(0.009), F32(0.004)
    qx = oracle.quantize_act_fp8_b128(x, sx)
    y = oracle.expert_rows_fp8_b128(qx, np.array([1, 0, 1], np.int32), bu, bd, oracle.identity_slot(n), sx, sh,
                                    H, F)
    Hp, Fp = 384, 384
    for r, e in enumerate([1, 0, 1]):
        Wu = oracle.e4m3_decode(bu[0][e]).astype(np.float64) * np.repeat(bu[1][e].astype(np.float64), 128, axis=1)
        Wd = oracle.e4m3_decode(bd[0][e]).astype(np.float64) * np.repeat(bd[1][e].astype(np.float64), 128, axis=1)
        xd = oracle.e4m3_decode(qx[r]).astype(np.float64) * float(sx)
        z = Wu @ xd
        a32 = (np.maximum(z, 0.0) ** 2).astype(np.float32)
        qa = np.zeros(Fp, np.uint8)
        qa[:F] = torch_e4m3((a32 / sh).astype(np.float32))
        ref = Wd @ (oracle.e4m3_decode(qa).astype(np.float64) * float(sh))
        assert np.max(np.abs(y[r] - ref)) <= 1e-12 * np.max(np.abs(ref))
