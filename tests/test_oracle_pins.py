"""Pins of the oracle to something other than itself.

Each test checks one oracle function against what the pages and the
mathematics fix: exact rational arithmetic and brute-force sorting, a
library softmax, closed forms for identity-like experts, a dense torch fp64
reformulation, the zero-padding invariance of the audio.cpp model page
("Q4_K, Q3_K and Q2_K expert profiles": routed-bank inputs padded to 2,816
and 2,048 with zeros leave outputs and routing unchanged), relabelling
equivariance and an exhaustive check of the FP8 code maps against torch.
"""
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from synth import workloads as W

TINY = W.WORKLOADS[0]


def tiny_inputs(w=TINY, bias=None):
    x = W.host_x(w)
    wr = W.host_router(w)
    wu = W.host_w_up(w)
    wd = W.host_w_down(w)
    return x, wr, bias, wu, wd


def to_bits(a: np.ndarray) -> np.ndarray:
    """float32 values that are exactly bf16 -> bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
    return (bits >> 16).astype(np.uint16)


def exact_logits(x, wr, bias=None):
    xf = oracle.bf16_to_f64(x)
    wf = oracle.bf16_to_f64(wr)
    T, H = xf.shape
    E = wf.shape[0]
    out = [[None] * E for _ in range(T)]
    xq = [[Fraction(v) for v in row] for row in xf]
    wq = [[Fraction(v) for v in row] for row in wf]
    for t in range(T):
        for e in range(E):
            s = sum(a * b for a, b in zip(xq[t], wq[e]))
            if bias is not None:
                s += Fraction(float(bias[e]))
            out[t][e] = s
    return out


# --------------------------------------------------------------------------- routing

def test_fixed_point_logits_within_bound_of_exact_sum():
    x, wr, _, _, _ = tiny_inputs()
    L = oracle.router_logits_fx(x[:6], wr)
    ex = exact_logits(x[:6], wr)
    bound = Fraction(TINY.H, 2 ** 41)
    for t in range(6):
        for e in range(TINY.E):
            assert abs(Fraction(int(L[t, e]), 2 ** 40) - ex[t][e]) <= bound


def test_topk_equals_brute_force_sort_of_exact_logits():
    x, wr, _, _, _ = tiny_inputs()
    ex = exact_logits(x, wr)
    L, idx, w = oracle.route(x, wr, None, TINY.K)
    for t in range(TINY.T):
        order = sorted(range(TINY.E), key=lambda e: (-ex[t][e], e))
        assert list(idx[t]) == order[:TINY.K]


def test_ties_go_to_the_lower_expert_index():
    x, wr, _, _, _ = tiny_inputs()
    wr = wr.copy()
    wr[5] = wr[1]          # experts 1 and 5 now have identical logits for every token
    wr[6] = wr[1]
    bias = np.zeros(TINY.E, dtype=np.float32)
    bias[[1, 5, 6]] = 50.0  # and they are the three best
    L, idx, w = oracle.route(x, wr, bias, 3)
    assert np.all(idx == np.array([1, 5, 6]))
    assert np.allclose(w, 1.0 / 3.0, rtol=0, atol=1e-15)


def test_weights_equal_library_softmax_renormalised():
    x, wr, _, _, _ = tiny_inputs()
    bias = W.zipf_bias(11, TINY.E)
    L, idx, w = oracle.route(x, wr, bias, TINY.K)
    ex = exact_logits(x, wr, bias)
    for t in range(TINY.T):
        p = scipy.special.softmax(np.array([float(v) for v in ex[t]]))
        sel = p[idx[t]]
        assert np.allclose(w[t], sel / sel.sum(), rtol=1e-12, atol=0)


def test_routing_invariants_decode_shape_router():
    w = W.WORKLOADS[1]
    x = W.host_x(w)[:32]
    wr = W.host_router(w)
    L, idx, wt = oracle.route(x, wr, None, w.K)
    assert np.allclose(wt.sum(1), 1.0, atol=1e-12)
    assert np.all(wt > 0)
    for t in range(32):
        assert len(set(idx[t].tolist())) == w.K
        assert idx[t].min() >= 0 and idx[t].max() < w.E
        sel = L[t, idx[t]]
        rest = np.delete(L[t], idx[t])
        assert sel.min() >= rest.max()
        assert np.all(np.diff(sel) <= 0)


def test_one_hot_bias_selects_the_planted_experts():
    x, wr, _, _, _ = tiny_inputs()
    bias = np.zeros(TINY.E, dtype=np.float32)
    bias[6] = 100.0
    bias[3] = 99.0
    L, idx, w = oracle.route(x, wr, bias, 2)
    assert np.all(idx[:, 0] == 6) and np.all(idx[:, 1] == 3)
    lw = np.log(w[:, 0] / w[:, 1])          # softmax ratio = exp(logit difference)
    assert np.allclose(lw, (L[:, 6] - L[:, 3]).astype(np.float64) * 2.0 ** -40, rtol=0, atol=1e-12)
    assert np.all(np.abs(lw - 1.0) < 2.0)


def test_fixed_point_logits_match_float64_matmul():
    w = W.WORKLOADS[1]
    x = W.host_x(w)[:8]
    wr = W.host_router(w)
    L = oracle.router_logits_fx(x, wr).astype(np.float64) * 2.0 ** -40
    ref = oracle.bf16_to_f64(x) @ oracle.bf16_to_f64(wr).T
    assert np.max(np.abs(L - ref)) < 1e-9


# --------------------------------------------------------------------------- permutation

def test_permute_equals_stable_argsort():
    w = W.WORKLOADS[3]
    x = W.host_x(w)[:200]
    wr = W.host_router(w)
    _, idx, _ = oracle.route(x, wr, W.host_bias(w), w.K)
    counts, offsets, perm_src, inv_row = oracle.permute(idx, w.E)
    flat = idx.reshape(-1)
    assert np.array_equal(perm_src, np.argsort(flat, kind="stable").astype(np.int32))
    assert np.array_equal(counts, np.bincount(flat, minlength=w.E).astype(np.int32))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
    assert np.array_equal(perm_src[inv_row], np.arange(flat.size))
    assert np.array_equal(inv_row[perm_src], np.arange(flat.size))
    assert (counts == 0).any()           # the Zipf bias leaves some experts empty
    for e in range(w.E):
        seg = perm_src[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all(flat[seg] == e)


# --------------------------------------------------------------------------- experts

def identity_like_banks(w, c):
    """W_up[e] = c_e [I | 0] (F x H),  W_down[e] = [I ; 0] (H x F)."""
    wu = np.zeros((w.E, w.F, w.H), dtype=np.float32)
    wd = np.zeros((w.E, w.H, w.F), dtype=np.float32)
    for e in range(w.E):
        wu[e, np.arange(w.F), np.arange(w.F)] = c[e]
        wd[e, np.arange(w.F), np.arange(w.F)] = 1.0
    return to_bits(wu), to_bits(wd)


def test_identity_experts_closed_form():
    x, wr, _, _, _ = tiny_inputs()
    c = np.array([1.0 + e / 8.0 for e in range(TINY.E)], dtype=np.float32)
    wu, wd = identity_like_banks(TINY, c)
    r = oracle.moe_layer_bf16(x, wr, None, wu, wd, TINY.K)
    xf = oracle.bf16_to_f64(x)
    relu2 = np.maximum(xf[:, :TINY.F], 0.0) ** 2
    gain = (r["w"] * (c.astype(np.float64)[r["idx"]] ** 2)).sum(1)
    expect = np.zeros_like(xf)
    expect[:, :TINY.F] = gain[:, None] * relu2
    assert np.allclose(r["out"], expect, rtol=1e-14, atol=0)


def test_identity_experts_unit_gain_is_routing_independent():
    x, wr, _, _, _ = tiny_inputs()
    wu, wd = identity_like_banks(TINY, np.ones(TINY.E, dtype=np.float32))
    r = oracle.moe_layer_bf16(x, wr, W.zipf_bias(5, TINY.E), wu, wd, TINY.K)
    xf = oracle.bf16_to_f64(x)
    assert np.allclose(r["out"][:, :TINY.F], np.maximum(xf[:, :TINY.F], 0) ** 2, rtol=1e-14)
    assert np.all(r["out"][:, TINY.F:] == 0)


def test_dense_masked_reformulation_torch_fp64():
    for wl in (TINY, W.Workload("mid", 12, 512, 16, 4, 192, seed=9)):
        x, wr, _, wu, wd = tiny_inputs(wl)
        bias = W.zipf_bias(wl.seed, wl.E)
        r = oracle.moe_layer_bf16(x, wr, bias, wu, wd, wl.K)
        X = torch.from_numpy(oracle.bf16_to_f64(x))
        R = torch.from_numpy(oracle.bf16_to_f64(wr))
        U = torch.from_numpy(oracle.bf16_to_f64(wu))
        D = torch.from_numpy(oracle.bf16_to_f64(wd))
        logits = X @ R.T + torch.from_numpy(bias.astype(np.float64))
        p = torch.softmax(logits, dim=-1)
        top = torch.topk(logits, wl.K, dim=-1)
        gaps = (top.values[:, :-1] - top.values[:, 1:]).min()
        assert gaps > 1e-8  # no near-ties, so the library's order is the unique one
        assert np.array_equal(top.indices.numpy(), r["idx"])
        gate = torch.zeros_like(p).scatter(1, top.indices, p.gather(1, top.indices))
        gate = gate / gate.sum(1, keepdim=True)
        dense = torch.zeros_like(X)
        for e in range(wl.E):
            y = torch.relu(X @ U[e].T) ** 2 @ D[e].T
            dense += gate[:, e:e + 1] * y
        ref = dense.numpy()
        assert np.max(np.abs(r["out"] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_zero_padding_to_2816_and_2048_changes_nothing():
    wl = W.Workload("pad", 6, 2688, 8, 2, 1856, seed=21)
    x, wr, _, wu, wd = tiny_inputs(wl)
    base = oracle.moe_layer_bf16(x, wr, None, wu, wd, wl.K)
    HP, FP = 2816, 2048
    xp = np.zeros((wl.T, HP), np.uint16); xp[:, :wl.H] = x
    wrp = np.zeros((wl.E, HP), np.uint16); wrp[:, :wl.H] = wr
    wup = np.zeros((wl.E, FP, HP), np.uint16); wup[:, :wl.F, :wl.H] = wu
    wdp = np.zeros((wl.E, HP, FP), np.uint16); wdp[:, :wl.H, :wl.F] = wd
    pad = oracle.moe_layer_bf16(xp, wrp, None, wup, wdp, wl.K)
    assert np.array_equal(pad["logits"], base["logits"])
    assert np.array_equal(pad["idx"], base["idx"])
    assert np.array_equal(pad["w"], base["w"])
    assert np.array_equal(pad["out"][:, :wl.H], base["out"])
    assert np.all(pad["out"][:, wl.H:] == 0)


def test_expert_relabelling_equivariance():
    x, wr, _, wu, wd = tiny_inputs()
    bias = W.zipf_bias(2, TINY.E)
    base = oracle.moe_layer_bf16(x, wr, bias, wu, wd, TINY.K)
    pi = np.array([3, 7, 0, 5, 1, 6, 2, 4])          # expert e gets label pi[e]
    inv = np.argsort(pi)
    rl = oracle.moe_layer_bf16(x, wr[inv], bias[inv], wu[inv], wd[inv], TINY.K)
    assert np.array_equal(rl["idx"], pi[base["idx"]])
    assert np.array_equal(rl["out"], base["out"])


def test_expert_subset_slot_map():
    x, wr, _, wu, wd = tiny_inputs()
    full = oracle.moe_layer_bf16(x, wr, None, wu, wd, TINY.K, tokens=[3, 9])
    used = sorted(set(full["idx"].reshape(-1).tolist()))
    slot = -np.ones(TINY.E, np.int32)
    slot[used] = np.arange(len(used))
    sub = oracle.moe_layer_bf16(x, wr, None, wu[used], wd[used], TINY.K, tokens=[3, 9], slot=slot)
    assert np.array_equal(sub["out"], full["out"])
    with pytest.raises(ValueError):
        bad = slot.copy(); bad[used[0]] = -1
        oracle.moe_layer_bf16(x, wr, None, wu[used], wd[used], TINY.K, tokens=[3, 9], slot=bad)


def test_combine_order_and_residual():
    rng = np.random.default_rng(0)
    y = rng.standard_normal((3, 4, 5))
    w = rng.random((3, 4))
    res = to_bits(np.float32([[1.0, -2.0, 0.5, 0.0, 3.0]] * 3))
    out = oracle.combine(y, w, res)
    expect = oracle.bf16_to_f64(res).copy()
    for t in range(3):
        acc = np.zeros(5)
        for k in range(4):
            acc = acc + w[t, k] * y[t, k]
        expect[t] += acc
    assert np.array_equal(out, expect)


# --------------------------------------------------------------------------- FP8

def all_bf16_values():
    return (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)


def test_e4m3_encode_exhaustive_over_bf16_against_torch():
    v = all_bf16_values()
    q = oracle.e4m3_encode(v)
    fin = np.isfinite(v)
    small = fin & (np.abs(v) <= 448.0)
    ref = torch.from_numpy(v[small]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q[small], ref)
    big = fin & (np.abs(v) > 448.0) | np.isinf(v)
    assert np.all((q[big] & 0x7F) == 0x7E)
    assert np.all((q[big] >> 7) == (np.signbit(v[big])).astype(np.uint8))
    assert np.all((q[np.isnan(v)] & 0x7F) == 0x7F)


def test_e4m3_encode_random_fp32_against_torch():
    rng = np.random.default_rng(1)
    mant = rng.integers(0, 2 ** 23, 400_000, dtype=np.uint32)
    expo = rng.integers(100, 136, 400_000, dtype=np.uint32)   # 2^-27 .. 2^8
    sign = rng.integers(0, 2, 400_000, dtype=np.uint32)
    v = ((sign << 31) | (expo << 23) | mant).view(np.float32)
    v = v[np.abs(v) <= 448.0]
    q = oracle.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_e4m3_decode_all_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(v), nan)
    assert np.array_equal(v[~nan], ref[~nan])
    assert v[0x7E] == 448.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9


def test_tensor_quantiser_scale_and_error_bound():
    k = synth.key(4, 3, 0)
    w = synth.normal_bf16(k, 1856 * 64, 0.02)
    q, s = oracle.quantize_tensor_fp8(w)
    wf = oracle.bf16_to_f64(w)
    assert s == np.float32(np.float32(np.abs(wf).max()) / np.float32(448.0))
    assert np.any((q & 0x7F) == 0x7E)
    deq = oracle.e4m3_decode(q).astype(np.float64) * float(s)
    normal = np.abs(wf) >= 2.0 ** -6 * float(s) * 1.0001
    rel = np.abs(deq - wf)[normal] / np.abs(wf)[normal]
    assert rel.max() <= 2.0 ** -4 * 1.0001
    assert np.all(np.abs(deq - wf)[~normal] <= 2.0 ** -10 * float(s) * 1.0001)


def test_fp8_expert_equals_bf16_expert_on_exactly_representable_values():
    H, F = 64, 32
    rng = np.random.default_rng(3)
    qd = rng.integers(0, 256, (1, H, F), dtype=np.uint8)
    qd[(qd & 0x7F) == 0x7F] = 0x38            # no NaN codes
    qu = np.zeros((1, F, H), np.uint8)
    qu[0, np.arange(F), np.arange(F)] = 0x38   # 1.0 on the diagonal
    xs = np.float32(rng.choice([0.0, 1.0, -1.0, 2.0, 0.5, -4.0, 0.25], H))
    qx = oracle.e4m3_encode(xs)[None, :]
    y8 = oracle.expert_rows_fp8(qx, np.zeros(1, np.int32), qu, np.float32([1.0]), qd,
                                np.float32([1.0]), np.zeros(1, np.int32), 1.0, 1.0)
    wu = to_bits(oracle.e4m3_decode(qu))
    wd = to_bits(oracle.e4m3_decode(qd))
    y16 = oracle.expert_rows_bf16(xs.astype(np.float64)[None, :], np.zeros(1, np.int32), wu, wd,
                                  np.zeros(1, np.int32))
    assert np.array_equal(y8, y16)


def test_fp8_scales_enter_linearly():
    H, F = 64, 32
    rng = np.random.default_rng(4)
    qu = rng.integers(0, 0x70, (1, F, H), dtype=np.uint8)
    qd = rng.integers(0, 0x70, (1, H, F), dtype=np.uint8)
    qx = rng.integers(0, 0x70, (1, H), dtype=np.uint8)
    ex, slot = np.zeros(1, np.int32), np.zeros(1, np.int32)
    y1 = oracle.expert_rows_fp8(qx, ex, qu, np.float32([1.0]), qd, np.float32([1.0]), slot, 1.0, 1e6)
    # doubling the down scale doubles y exactly; s_u*s_x enters only as a product
    y2 = oracle.expert_rows_fp8(qx, ex, qu, np.float32([1.0]), qd, np.float32([2.0]), slot, 1.0, 1e6)
    assert np.array_equal(y2, 2.0 * y1)
    y3 = oracle.expert_rows_fp8(qx, ex, qu, np.float32([0.5]), qd, np.float32([1.0]), slot, 2.0, 1e6)
    assert np.array_equal(y3, y1)


# --------------------------------------------------------------------------- normalisation, rounding

def test_rmsnorm_against_torch_fp64_within_one_bf16_rounding():
    k = synth.key(4, 7, 3)
    x = synth.normal_bf16(k, 64 * 2688, 3.0).reshape(64, 2688)
    u = oracle.rmsnorm_bf16(x, 1e-5)
    X = torch.from_numpy(oracle.bf16_to_f64(x))
    ref = (X / torch.sqrt((X * X).mean(-1, keepdim=True) + 1e-5)).numpy()
    got = oracle.bf16_to_f64(u)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)
    assert np.allclose(np.sqrt((got ** 2).mean(1)), 1.0, atol=3e-3)


def test_round_bf16_picks_the_nearest_value():
    rng = np.random.default_rng(5)
    v = rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 20, 200_000))
    b = oracle.round_bf16(v)
    r = oracle.bf16_to_f64(b)
    up = oracle.bf16_to_f64((b.astype(np.int32) + 1).astype(np.uint16))
    dn = oracle.bf16_to_f64((b.astype(np.int32) - 1).astype(np.uint16))
    err = np.abs(r - v)
    assert np.all(err <= np.abs(up - v)) and np.all(err <= np.abs(dn - v))
    halves = v[:1000].astype(np.float32).astype(np.float64)
    assert np.array_equal(oracle.round_bf16(halves),
                          torch.from_numpy(halves.astype(np.float32)).bfloat16().view(torch.int16).numpy().astype(np.uint16))
