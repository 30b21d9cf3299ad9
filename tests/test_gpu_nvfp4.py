"""GPU parity of the NVFP4 (W4A4) experts against the oracle.

The quantisers (weight banks with their tensor scales; activations with a
static tensor scale) must give the oracle's codes and block scales bit for
bit.  The layer output is compared within NVFP4_TOL = 3e-2 of max|ref|: the
two sides accumulate the expert products in different orders, so the fp32
ReLU^2 values differ in the last bits and a value next to a rounding point
of the 4-bit grid can take the neighbouring code; one such flip moves one
hidden element by one grid step (at most a third of its block's maximum),
about 1 % of the output's maximum at these shapes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

from _gpu import dev, dev_bf16, host_f64, inputs, rel_err

pytestmark = pytest.mark.gpu

NVFP4_TOL = 3e-2


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def ksp(K):
    return (K // 16 + 15) // 16 * 16


def gpu_bank(moe, bank):
    n, rows, K = bank.shape
    codes = torch.empty(n, rows, K // 2, dtype=torch.uint8, device="cuda")
    block = torch.empty(n, rows, ksp(K), dtype=torch.uint8, device="cuda")
    tscale = torch.empty(n, dtype=torch.float32, device="cuda")
    moe.quantize_nvfp4(dev_bf16(bank), codes, block, tscale)
    torch.cuda.synchronize()
    return codes, block, tscale


@pytest.mark.parametrize("shape", [(8, 128, 256), (3, 1856, 2688), (2, 2688, 1856), (5, 64, 96)])
def test_weight_quantiser_bit_exact(moe, shape):
    n, rows, K = shape
    bank = synth.normal_bf16(synth.key(40 + n, 3, rows), n * rows * K, W.SIGMA_W).reshape(n, rows, K)
    bank[0, 0, :16] = 0                  # an all-zero block
    codes, block, tscale = gpu_bank(moe, bank)
    c_ref, s_ref, t_ref = oracle.quantize_bank_nvfp4(bank)
    assert np.array_equal(tscale.cpu().numpy(), t_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    b = block.cpu().numpy()
    assert np.array_equal(b[..., :K // 16], s_ref)
    assert not b[..., K // 16:].any()     # padding is zero


@pytest.mark.parametrize("x_scale", [0.0023, 1.0 / 2688.0, 0.05, 1.7e-5])
def test_activation_quantiser_bit_exact(moe, x_scale):
    rows, H = 300, 2688
    x = synth.normal_bf16(synth.key(41, 1, 0), rows * H, 1.0).reshape(rows, H)
    x[1] = 0                                                         # zero row
    x[2, :64] = np.uint16(0x7F7F)                                    # large values saturate
    x[3, ::7] = np.uint16(0x0001)                                    # tiny values
    codes = torch.empty(rows, H // 2, dtype=torch.uint8, device="cuda")
    block = torch.empty(rows, ksp(H), dtype=torch.uint8, device="cuda")
    moe.quantize_act_nvfp4(dev_bf16(x), codes, block, x_scale)
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.quantize_nvfp4(x, np.float32(x_scale))
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    b = block.cpu().numpy()
    assert np.array_equal(b[:, :H // 16], s_ref) and not b[:, H // 16:].any()


def nvfp4_case(moe, w, h, tokens=None, slot_experts=None, ws_fill=None):
    """Quantise banks on the GPU (checked bit-exact against the oracle), calibrate static
    tensor scales with the oracle, run the layer on both sides.  ws_fill: a byte written over
    the whole workspace first (0x7F is an E4M3 NaN: stale workspace bytes must not reach the
    tensor cores as scales)."""
    bank_up = oracle.quantize_bank_nvfp4(h["wu"])
    bank_down = oracle.quantize_bank_nvfp4(h["wd"])
    cu, bu, tu = gpu_bank(moe, h["wu"])
    cd, bd, td = gpu_bank(moe, h["wd"])
    assert np.array_equal(cu.cpu().numpy(), bank_up[0]) and np.array_equal(td.cpu().numpy(), bank_down[2])
    tx, th = oracle.calibrate_nvfp4(h["x"][:64], h["wr"], h["bias"], h["wu"], w.K)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, nvfp4=True)
    ws = moe.alloc_workspace(dims)
    if ws_fill is not None:
        ws.fill_(ws_fill)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    sc = moe.nvfp4_scales(tu, td, float(tx), float(th), bu, bd)
    moe.forward(dims, dev_bf16(h["x"]), dev_bf16(h["wr"]), None if h["bias"] is None else dev(h["bias"]), cu, cd,
                out, ws, scales=sc, topk_idx=idx)
    moe.check_device_error()
    r = oracle.moe_layer_nvfp4(h["x"], h["wr"], h["bias"], bank_up, bank_down, tx, th, w.K, tokens=tokens)
    got = host_f64(out) if tokens is None else host_f64(out)[tokens]
    assert np.array_equal(idx.cpu().numpy() if tokens is None else idx.cpu().numpy()[tokens], r["idx"])
    return rel_err(got, r["out"])


@pytest.mark.parametrize("w", [W.WORKLOADS[0], W.Workload("nvfp4_ragged_T37", 37, 512, 16, 4, 192, seed=26),
                               W.Workload("nvfp4_tail_F224_T300", 300, 256, 8, 3, 224, seed=27)],
                         ids=lambda w: w.name)
def test_nvfp4_forward_parity_small(moe, w):
    assert nvfp4_case(moe, w, inputs(w)) <= NVFP4_TOL


@pytest.mark.parametrize("w", [W.Workload("nvfp4_tail_F224_T300", 300, 256, 8, 3, 224, seed=27),
                               W.Workload("nvfp4_tail_H288_F96", 40, 288, 8, 2, 96, seed=29)],
                         ids=lambda w: w.name)
def test_nvfp4_forward_ignores_stale_workspace_bytes(moe, w):
    """K = 224 (or 96, 288) is not a whole stage of 256: the last stage's padding blocks are
    masked, so a workspace full of E4M3 NaN bytes gives the same, finite result."""
    assert nvfp4_case(moe, w, inputs(w), ws_fill=0x7F) <= NVFP4_TOL


def test_nvfp4_forward_parity_decode_shape(moe):
    w = W.Workload("nvfp4_decode_T64", 64, 2688, 128, 6, 1856, seed=28)
    assert nvfp4_case(moe, w, inputs(w), tokens=np.arange(0, 64, 9)) <= NVFP4_TOL


def test_nvfp4_forward_parity_prefill_shape(moe):
    """4096 tokens: tiles of up to 256 token rows (two fp16 stage buffers), sampled tokens."""
    w = W.Workload("nvfp4_prefill_T4096", 4096, 2688, 128, 6, 1856, seed=29)
    assert nvfp4_case(moe, w, inputs(w), tokens=np.arange(3, 4096, 611)) <= NVFP4_TOL


@pytest.mark.parametrize("one_launch", [1, 0], ids=["one_launch_ffn", "two_launches"])
def test_nvfp4_expired_wait_is_reported(moe, one_launch):
    """One launch: the list's first up unit withholds its report, so the down units of its entry
    wait in vain.  Two launches: block 0's producer withholds its first load.  Either way the
    status is MOE_ETIMEOUT and the next call is right."""
    moe.debug_set(8, one_launch)
    try:
        _nvfp4_expired_wait_case(moe)
    finally:
        moe.debug_set(8, 1)


def _nvfp4_expired_wait_case(moe):
    w = W.WORKLOADS[0]
    h = inputs(w)
    cu, bu, tu = gpu_bank(moe, h["wu"])
    cd, bd, td = gpu_bank(moe, h["wd"])
    _, ridx, _ = oracle.route(h["x"], h["wr"], None, w.K)
    _, offsets, perm_src, _ = oracle.permute(ridx, w.E)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, nvfp4=True)
    ws = moe.alloc_workspace(dims)
    y = torch.empty(w.T * w.K, w.H, dtype=torch.bfloat16, device="cuda")
    sc = moe.nvfp4_scales(tu, td, 0.01, 0.01, bu, bd)
    moe.debug_set(1, 20_000_000)
    moe.debug_set(2, 1)
    try:
        moe.expert_ffn(dims, dev_bf16(h["x"]), dev(offsets), dev(perm_src), cu, cd, sc, y, ws)
        assert moe.check_device_error_status() == moe.MOE_ETIMEOUT
    finally:
        moe.debug_set(2, 0)
        moe.debug_set(1, 0)
    moe.expert_ffn(dims, dev_bf16(h["x"]), dev(offsets), dev(perm_src), cu, cd, sc, y, ws)
    moe.check_device_error()


@pytest.mark.parametrize("w", [W.WORKLOADS[0], W.Workload("nvfp4_ragged_T37", 37, 512, 16, 4, 192, seed=26),
                               W.Workload("nvfp4_tail_F224_T300", 300, 256, 8, 3, 224, seed=27),
                               W.Workload("nvfp4_decode_T64", 64, 2688, 128, 6, 1856, seed=28),
                               W.Workload("nvfp4_prefill_T4096", 4096, 2688, 128, 6, 1856, seed=29)],
                         ids=lambda w: w.name)
def test_nvfp4_one_launch_ffn_equals_two_launches_bitwise(moe, w):
    """Both projections in one launch run the same units (same tiles, same accumulation order,
    the same quantisation of H), so the layer output is the same bit for bit as with two
    launches, at both TMEM layouts (tiles of up to 64 rows on two CTAs per SM, and up to 224)."""
    h = inputs(w)
    cu, bu, tu = gpu_bank(moe, h["wu"])
    cd, bd, td = gpu_bank(moe, h["wd"])
    tx, th = oracle.calibrate_nvfp4(h["x"][:64], h["wr"], h["bias"], h["wu"], w.K)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, nvfp4=True)
    ws = moe.alloc_workspace(dims)
    sc = moe.nvfp4_scales(tu, td, float(tx), float(th), bu, bd)
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
