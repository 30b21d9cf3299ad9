"""GPU parity of the FP8_B128 W8A8 experts against the oracle (bloomery issue
page, section 3: FP8_B128 scales with the 64-value tail of K = 1856).  The
bank quantiser must give the oracle's codes and block scales bit for bit; the
layer output is compared within FP8_TOL = 3e-2 of max|ref| (the H codes follow
fp32 accumulators whose summation order differs from the oracle's, as in the
scalar-scale FP8 path)."""
import numpy as np
import pytest
import torch

import oracle
from synth import workloads as W

from _gpu import FP8_TOL, dev, dev_bf16, host_f64, inputs, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def gpu_bank(moe, bank):
    n, rows, K = bank.shape
    Kp = moe.b128_kp(K)
    codes = torch.empty(n, rows, Kp, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, rows, Kp // 128, dtype=torch.float32, device="cuda")
    moe.quantize_fp8_b128(dev_bf16(bank), codes, scales)
    torch.cuda.synchronize()
    return codes, scales


@pytest.mark.parametrize("shape", [(3, 1856, 2688), (2, 2688, 1856), (4, 64, 208), (2, 130, 16)])
def test_b128_quantiser_bit_exact(moe, shape):
    n, rows, K = shape
    import synth
    bank = synth.normal_bf16(synth.key(50 + n, 3, rows), n * rows * K, W.SIGMA_W).reshape(n, rows, K)
    bank[0, 0, :min(K, 128)] = 0                      # an all-zero block
    bank[-1, -1, -1] = np.uint16(0x40F0)              # 7.5 in the last (tail) block
    codes, scales = gpu_bank(moe, bank)
    q, s = oracle.quantize_fp8_b128(bank)
    assert np.array_equal(codes.cpu().numpy(), q)
    assert np.array_equal(scales.cpu().numpy(), s)


def b128_case(moe, w, h, tokens=None):
    bu, bd = oracle.quantize_fp8_b128(h["wu"]), oracle.quantize_fp8_b128(h["wd"])
    cu, su = gpu_bank(moe, h["wu"])
    cd, sd = gpu_bank(moe, h["wd"])
    assert np.array_equal(cd.cpu().numpy(), bd[0]) and np.array_equal(su.cpu().numpy(), bu[1])
    sx, sh = oracle.calibrate_fp8(h["x"][:64], h["wr"], h["bias"], h["wu"], w.K)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, fp8_b128=True)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    moe.forward(dims, dev_bf16(h["x"]), dev_bf16(h["wr"]), None if h["bias"] is None else dev(h["bias"]), cu, cd,
                out, ws, scales=moe.fp8_scales(su, sd, float(sx), float(sh)), topk_idx=idx)
    moe.check_device_error()
    r = oracle.moe_layer_fp8_b128(h["x"], h["wr"], h["bias"], bu, bd, sx, sh, w.K, w.H, w.F, tokens=tokens)
    got = host_f64(out) if tokens is None else host_f64(out)[tokens]
    gi = idx.cpu().numpy() if tokens is None else idx.cpu().numpy()[tokens]
    assert np.array_equal(gi, r["idx"])
    return rel_err(got, r["out"])


@pytest.mark.parametrize("w", [W.WORKLOADS[0], W.Workload("b128_ragged_T37_F192", 37, 512, 16, 4, 192, seed=51),
                               W.Workload("b128_tails_H272_F208", 21, 272, 8, 3, 208, seed=52),
                               W.Workload("b128_hot_T300", 300, 256, 4, 2, 128, seed=53)],
                         ids=lambda w: w.name)
def test_b128_forward_parity_small(moe, w):
    assert b128_case(moe, w, inputs(w)) <= FP8_TOL


def test_b128_forward_parity_decode_shape(moe):
    """H = 2688 (21 blocks) and F = 1856 (15 blocks, the last with 64 values)."""
    w = W.Workload("b128_decode_T64", 64, 2688, 128, 6, 1856, seed=54)
    assert b128_case(moe, w, inputs(w), tokens=np.arange(0, 64, 7)) <= FP8_TOL


@pytest.mark.parametrize("one_launch", [1, 0], ids=["one_launch_ffn", "two_launches"])
def test_b128_expired_wait_is_reported(moe, one_launch):
    """One launch: the list's first up unit withholds its report, so the down units of its entry
    wait in vain.  Two launches: block 0's producer withholds its first load.  Either way the
    status is MOE_ETIMEOUT and the next call is right."""
    moe.debug_set(8, one_launch)
    try:
        _b128_expired_wait_case(moe)
    finally:
        moe.debug_set(8, 1)


def _b128_expired_wait_case(moe):
    w = W.WORKLOADS[0]
    h = inputs(w)
    cu, su = gpu_bank(moe, h["wu"])
    cd, sd = gpu_bank(moe, h["wd"])
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, fp8_b128=True)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    sc = moe.fp8_scales(su, sd, 0.01, 0.01)
    moe.debug_set(1, 20_000_000)
    moe.debug_set(2, 1)
    try:
        moe.forward(dims, dev_bf16(h["x"]), dev_bf16(h["wr"]), None, cu, cd, out, ws, scales=sc)
        assert moe.check_device_error_status() == moe.MOE_ETIMEOUT
    finally:
        moe.debug_set(2, 0)
        moe.debug_set(1, 0)
    moe.forward(dims, dev_bf16(h["x"]), dev_bf16(h["wr"]), None, cu, cd, out, ws, scales=sc)
    moe.check_device_error()


def test_b128_forward_parity_prefill_shape(moe):
    """The prefill workload with FP8_B128 experts (T = 4096, 128 experts, ~192 rows per
    expert, so every expert's rows span several 64-row tiles): routing bit for bit on every
    token, the output on sampled tokens within FP8_TOL.  The banks are made and quantised on
    the device from the seeded bf16 masters; the oracle quantises the used experts' masters
    itself (the quantiser is bit-exact, above)."""
    import synth
    w = W.WORKLOADS[10]
    sx, sh = W.fp8_b128_scales(w)
    stream = torch.cuda.current_stream().cuda_stream
    banks = []
    for tid, shape in ((synth.T_WUP, (w.E, w.F, w.H)), (synth.T_WDOWN, (w.E, w.H, w.F))):
        t = torch.empty(*shape, dtype=torch.bfloat16, device="cuda")
        synth.normal_bf16_device(synth.key(w.seed, tid, 0), t.numel(), W.SIGMA_W, t.data_ptr(), stream)
        n, rows, K = shape
        kp = moe.b128_kp(K)
        codes = torch.empty(n, rows, kp, dtype=torch.uint8, device="cuda")
        sc = torch.empty(n, rows, kp // 128, dtype=torch.float32, device="cuda")
        moe.quantize_fp8_b128(t, codes, sc)
        banks.append((codes, sc))
        del t
    (cu, su), (cd, sd) = banks
    x, wr = W.host_x(w), W.host_router(w)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, fp8_b128=True)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    moe.forward(dims, dev_bf16(x), dev_bf16(wr), None, cu, cd, out, ws,
                scales=moe.fp8_scales(su, sd, float(sx), float(sh)), topk_idx=idx)
    moe.check_device_error()

    _, ridx, _ = oracle.route(x, wr, None, w.K)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    rng = np.random.default_rng(10)
    tok = np.unique(np.concatenate([[0, w.T - 1], rng.choice(w.T, size=6, replace=False)]))
    used = sorted(set(ridx[tok].reshape(-1).tolist()))
    slot = -np.ones(w.E, np.int32)
    slot[used] = np.arange(len(used))
    bu = oracle.quantize_fp8_b128(W.host_w_up(w, experts=used))
    bd = oracle.quantize_fp8_b128(W.host_w_down(w, experts=used))
    r = oracle.moe_layer_fp8_b128(x, wr, None, bu, bd, sx, sh, w.K, w.H, w.F, tokens=tok, slot=slot)
    assert np.array_equal(r["idx"], ridx[tok])
    assert rel_err(host_f64(out)[tok], r["out"]) <= FP8_TOL


@pytest.mark.parametrize("w", [W.WORKLOADS[0], W.Workload("b128_ragged_T37_F192", 37, 512, 16, 4, 192, seed=51),
                               W.Workload("b128_tails_H272_F208", 21, 272, 8, 3, 208, seed=52),
                               W.Workload("b128_hot_T300", 300, 256, 4, 2, 128, seed=53),
                               W.Workload("b128_decode_T64", 64, 2688, 128, 6, 1856, seed=54),
                               W.Workload("b128_T700", 700, 512, 16, 4, 320, seed=55)],
                         ids=lambda w: w.name)
def test_b128_one_launch_ffn_equals_two_launches_bitwise(moe, w):
    """Both projections in one launch run the same block sums in the same order for every
    (token, feature), so the output is the same bit for bit as with two launches, although the
    one launch cuts experts into tiles of at most 64 rows and the two launches into up to 128
    (T = 700 here, 175 rows per expert)."""
    h = inputs(w)
    cu, su = gpu_bank(moe, h["wu"])
    cd, sd = gpu_bank(moe, h["wd"])
    sx, sh = oracle.calibrate_fp8(h["x"][:64], h["wr"], h["bias"], h["wu"], w.K)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, fp8_b128=True)
    ws = moe.alloc_workspace(dims)
    sc = moe.fp8_scales(su, sd, float(sx), float(sh))
    x, wr = dev_bf16(h["x"]), dev_bf16(h["wr"])
    bias = None if h["bias"] is None else dev(h["bias"])
    outs = []
    for one in (1, 0):
        moe.debug_set(8, one)
        try:
            out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            moe.forward(dims, x, wr, bias, cu, cd, out, ws, scales=sc)
            moe.check_device_error()
            outs.append(out)
        finally:
            moe.debug_set(8, 1)
    assert torch.equal(outs[0], outs[1])
