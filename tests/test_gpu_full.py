"""GPU parity at full workload sizes, the FP8 W8A8 path, the RMS norm of the
chained stack, the device twin of the input generator, and the bounded-wait
failure path.

Full-size cases compare the whole routing and permutation bit for bit and
the layer output on sampled tokens (tokens never interact, so the oracle can
compute any subset exactly)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

from _gpu import BF16_TOL, FP8_TOL, dev, dev_bf16, device_inputs, host_bits, host_f64, inputs, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def device_bank(key, n, sigma, shape):
    t = torch.empty(*shape, dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(key, n, sigma, t.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return t


def test_device_generator_matches_host_generator():
    for (seed, tid, layer, sigma, n, off) in [(1, 3, 0, 0.02, 1 << 20, 0), (2, 1, 0, 1.0, 300_001, 12345),
                                              (4, 4, 22, 0.02, 77_777, 5 << 30)]:
        k = synth.key(seed, tid, layer)
        d = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        synth.normal_bf16_device(k, n, sigma, d.data_ptr(), torch.cuda.current_stream().cuda_stream, offset=off)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(d), synth.normal_bf16(k, n, sigma, offset=off))


# --------------------------------------------------------------------------- full size

@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_full_size_routing_permutation_and_sampled_outputs(moe, cfg):
    w = W.WORKLOADS[cfg]
    x = W.host_x(w)
    wr = W.host_router(w)
    bias = W.host_bias(w)
    wu_d = device_bank(synth.key(w.seed, synth.T_WUP, 0), w.E * w.F * w.H, W.SIGMA_W, (w.E, w.F, w.H))
    wd_d = device_bank(synth.key(w.seed, synth.T_WDOWN, 0), w.E * w.H * w.F, W.SIGMA_W, (w.E, w.H, w.F))
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    moe.forward(dims, dev_bf16(x), dev_bf16(wr), None if bias is None else dev(bias), wu_d, wd_d, out, ws,
                topk_idx=idx, topk_w=wt)
    moe.check_device_error()

    _, ridx, rw = oracle.route(x, wr, bias, w.K)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.max(np.abs(wt.cpu().numpy() - rw)) <= 1e-5
    counts, offsets, perm_src, inv_row = oracle.permute(ridx, w.E)
    g = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (w.E, w.E + 1, w.T * w.K, w.T * w.K)]
    moe.permute(dims, idx, *g, ws=ws)
    moe.check_device_error()
    for got, ref in zip(g, (counts, offsets, perm_src, inv_row)):
        assert np.array_equal(got.cpu().numpy(), ref)

    rng = np.random.default_rng(cfg)
    tok = np.unique(np.concatenate([[0, w.T - 1], rng.choice(w.T, size=min(w.T, 40), replace=False)]))
    used = sorted(set(ridx[tok].reshape(-1).tolist()))
    slot = -np.ones(w.E, np.int32)
    slot[used] = np.arange(len(used))
    r = oracle.moe_layer_bf16(x, wr, bias, W.host_w_up(w, experts=used), W.host_w_down(w, experts=used), w.K,
                              tokens=tok, slot=slot)
    assert rel_err(host_f64(out)[tok], r["out"]) <= BF16_TOL


# --------------------------------------------------------------------------- FP8 W8A8

def test_quantize_fp8_bit_exact(moe):
    w = W.WORKLOADS[0]
    for bank in (W.host_w_up(w), W.host_w_down(w),
                 synth.normal_bf16(synth.key(4, 3, 7), 4 * 1856 * 2688, 0.02).reshape(4, 1856, 2688)):
        q_ref, s_ref = oracle.quantize_bank_fp8(bank)
        codes = torch.empty(bank.shape, dtype=torch.uint8, device="cuda")
        scales = torch.empty(bank.shape[0], dtype=torch.float32, device="cuda")
        moe.quantize_fp8(dev_bf16(bank), codes, scales)
        torch.cuda.synchronize()
        assert np.array_equal(scales.cpu().numpy(), s_ref)
        assert np.array_equal(codes.cpu().numpy(), q_ref)


def test_quantize_fp8_zero_tensor_and_saturation(moe):
    bank = np.zeros((2, 64), np.uint16)
    bank[1, :4] = [0x3F80, 0xBF80, 0x4000, 0x0001]        # 1, -1, 2, tiny
    q_ref, s_ref = oracle.quantize_bank_fp8(bank)
    codes = torch.empty(bank.shape, dtype=torch.uint8, device="cuda")
    scales = torch.empty(2, dtype=torch.float32, device="cuda")
    moe.quantize_fp8(dev_bf16(bank), codes, scales)
    torch.cuda.synchronize()
    assert np.array_equal(scales.cpu().numpy(), s_ref) and s_ref[0] == 1.0
    assert np.array_equal(codes.cpu().numpy(), q_ref)


def _act_scales():
    sc = [np.float32(v) for v in (1.0, 0.001, 37.0, 448.0, 1.0 / 3.0, 0.0371, 2.0 ** -20, 6.1e4)]
    for sx, sh in W.chain_scales():
        sc += [sx, sh]
    rng = np.random.default_rng(31)
    sc += [np.float32(v) for v in np.exp(rng.uniform(np.log(1e-4), np.log(1e3), 16))]
    return sc


def test_activation_codes_match_a_correctly_rounded_division_for_every_bf16(moe):
    """Every bf16 bit pattern but NaN, at every static scale of the chain workload and
    24 more: the kernel's E4M3 codes of x / s (a reciprocal quotient with one FMA
    correction) equal the oracle's, which divides with one correctly rounded fp32
    division."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    nan = ((bits & 0x7F80) == 0x7F80) & ((bits & 0x007F) != 0)
    bits = np.where(nan, np.uint16(0), bits).reshape(256, 256)
    x = dev_bf16(bits)
    codes = torch.empty(256, 256, dtype=torch.uint8, device="cuda")
    for s in _act_scales():
        moe.quantize_act_fp8(x, codes, float(s))
        torch.cuda.synchronize()
        ref = oracle.quantize_act_fp8(bits, float(s)).reshape(256, 256)
        got = codes.cpu().numpy()
        assert np.array_equal(got, ref), (float(s), int(np.sum(got != ref)))


@pytest.mark.parametrize("scale", [1.0, 0.001, 37.0])
def test_rmsnorm_bit_exact(moe, scale):
    x = synth.normal_bf16(synth.key(4, 7, 1), 300 * 2688, scale).reshape(300, 2688)
    u = torch.empty(300, 2688, dtype=torch.bfloat16, device="cuda")
    moe.rmsnorm(dev_bf16(x), u, 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(u), oracle.rmsnorm_bf16(x, 1e-5))


def fp8_case(moe, w, x, wr, bias, wu, wd, tokens=None):
    """Quantise banks on both sides, calibrate static scales with the oracle, run both."""
    qu, su = oracle.quantize_bank_fp8(wu)
    qd, sd = oracle.quantize_bank_fp8(wd)
    sx, sh = oracle.calibrate_fp8(x[:64], wr, bias, wu, w.K)
    cu = torch.empty(wu.shape, dtype=torch.uint8, device="cuda")
    cd = torch.empty(wd.shape, dtype=torch.uint8, device="cuda")
    gsu = torch.empty(w.E, dtype=torch.float32, device="cuda")
    gsd = torch.empty(w.E, dtype=torch.float32, device="cuda")
    moe.quantize_fp8(dev_bf16(wu), cu, gsu)
    moe.quantize_fp8(dev_bf16(wd), cd, gsd)
    torch.cuda.synchronize()
    assert np.array_equal(cu.cpu().numpy(), qu) and np.array_equal(gsd.cpu().numpy(), sd)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, fp8=True)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    sc = moe.fp8_scales(gsu, gsd, float(sx), float(sh))
    moe.forward(dims, dev_bf16(x), dev_bf16(wr), None if bias is None else dev(bias), cu, cd, out, ws,
                scales=sc, topk_idx=idx)
    moe.check_device_error()
    r = oracle.moe_layer_fp8(x, wr, bias, qu, su, qd, sd, sx, sh, w.K, tokens=tokens)
    got = host_f64(out) if tokens is None else host_f64(out)[tokens]
    ridx = r["idx"]
    assert np.array_equal(idx.cpu().numpy() if tokens is None else idx.cpu().numpy()[tokens], ridx)
    return rel_err(got, r["out"])


@pytest.mark.parametrize("w", [W.WORKLOADS[0], W.Workload("fp8_ragged_T37", 37, 512, 16, 4, 192, seed=16),
                               W.Workload("fp8_tail_F208", 21, 272, 8, 3, 208, seed=17)],
                         ids=lambda w: w.name)
def test_fp8_forward_parity_small(moe, w):
    h = inputs(w)
    assert fp8_case(moe, w, h["x"], h["wr"], h["bias"], h["wu"], h["wd"]) <= FP8_TOL


def test_fp8_forward_parity_decode_shape(moe):
    w = W.Workload("fp8_decode_T64", 64, 2688, 128, 6, 1856, seed=18)
    h = inputs(w)
    assert fp8_case(moe, w, h["x"], h["wr"], None, h["wu"], h["wd"], tokens=np.arange(0, 64, 5)) <= FP8_TOL


# --------------------------------------------------------------------------- bounded waits

@pytest.mark.parametrize("one_launch", [1, 0], ids=["one_launch_ffn", "two_launches"])
def test_expired_wait_is_reported_and_the_context_stays_usable(moe, one_launch):
    """Two launches: block 0's producer withholds its first load, so the MMA's wait expires.
    One launch: the first up unit of the list withholds its report, so the down units of its entry
    wait on the counter in vain.  Either way the status is MOE_ETIMEOUT and the next call is
    right."""
    moe.debug_set(8, one_launch)
    try:
        _expired_wait_case(moe)
    finally:
        moe.debug_set(8, 1)


def _expired_wait_case(moe):
    w = W.WORKLOADS[0]
    h = inputs(w)
    d = device_inputs(h)
    _, ridx, _ = oracle.route(h["x"], h["wr"], None, w.K)
    _, offsets, perm_src, _ = oracle.permute(ridx, w.E)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    y = torch.empty(w.T * w.K, w.H, dtype=torch.bfloat16, device="cuda")
    moe.debug_set(1, 20_000_000)   # 20 ms limit on every bounded wait
    moe.debug_set(2, 1)            # block 0 withholds its first load (or unit 0 its report)
    try:
        moe.expert_ffn(dims, d["x"], dev(offsets), dev(perm_src), d["wu"], d["wd"], None, y, ws)
        assert moe.check_device_error_status() == moe.MOE_ETIMEOUT
    finally:
        moe.debug_set(2, 0)
        moe.debug_set(1, 0)
    moe.expert_ffn(dims, d["x"], dev(offsets), dev(perm_src), d["wu"], d["wd"], None, y, ws)
    moe.check_device_error()
    xf = oracle.bf16_to_f64(h["x"])
    ref = oracle.expert_rows_bf16(xf[perm_src // w.K], ridx.reshape(-1)[perm_src], h["wu"], h["wd"],
                                  oracle.identity_slot(w.E))
    assert rel_err(host_f64(y), ref) <= BF16_TOL


# --------------------------------------------------------------------------- CTA-pair GEMM

@pytest.mark.parametrize("fp8", [False, True])
def test_cta_pair_gemm_matches_oracle(moe, fp8):
    """The cta_group::2 grouped GEMM (switched on by debug hook 3) on a batch whose
    tiles exceed 64 tokens, including a ragged expert tail: same parity bar."""
    w = W.Workload("pair_T600_ragged", 600, 512, 16, 4, 320, seed=21)
    h = inputs(w)
    moe.debug_set(3, 1)
    try:
        if fp8:
            assert fp8_case(moe, w, h["x"], h["wr"], h["bias"], h["wu"], h["wd"]) <= FP8_TOL
        else:
            d = device_inputs(h)
            dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
            ws = moe.alloc_workspace(dims)
            out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            moe.forward(dims, d["x"], d["wr"], None, d["wu"], d["wd"], out, ws)
            moe.check_device_error()
            r = oracle.moe_layer_bf16(h["x"], h["wr"], None, h["wu"], h["wd"], w.K)
            assert rel_err(host_f64(out), r["out"]) <= BF16_TOL
    finally:
        moe.debug_set(3, 0)


# --------------------------------------------------------------------------- one-launch expert FFN

@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("w", [W.WORKLOADS[1], W.WORKLOADS[3], W.WORKLOADS[2],
                               W.Workload("ffn_T700_E16_K4", 700, 512, 16, 4, 320, seed=23),
                               W.Workload("ffn_T37_H272_E8_K3_F208", 37, 272, 8, 3, 208, seed=24)],
                         ids=lambda w: w.name if hasattr(w, "name") else str(w))
@pytest.mark.parametrize("with_residual", [False, True], ids=["no_residual", "residual_aliased_to_out"])
def test_one_launch_ffn_equals_two_launches_bitwise(moe, w, fp8, with_residual):
    """Both projections in one launch compute exactly the products of the two launches (same
    tiles, same accumulation order), so the layer output is the same bit for bit, also with
    the residual in `out`."""
    h = inputs(w)
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, fp8=fp8)
    ws = moe.alloc_workspace(dims)
    scales = None
    wu, wd = d["wu"], d["wd"]
    if fp8:
        cu = torch.empty(wu.shape, dtype=torch.uint8, device="cuda")
        cd = torch.empty(wd.shape, dtype=torch.uint8, device="cuda")
        su = torch.empty(w.E, dtype=torch.float32, device="cuda")
        sd = torch.empty(w.E, dtype=torch.float32, device="cuda")
        moe.quantize_fp8(wu, cu, su)
        moe.quantize_fp8(wd, cd, sd)
        sx, sh = oracle.calibrate_fp8(h["x"][:64], h["wr"], h["bias"], h["wu"], w.K)
        scales = moe.fp8_scales(su, sd, float(sx), float(sh))
        wu, wd = cu, cd
    g = torch.Generator().manual_seed(w.seed + 1000)
    res = torch.randn(w.T, w.H, generator=g).to(torch.bfloat16).cuda() if with_residual else None
    outs = []
    for one in (1, 0):
        moe.debug_set(8, one)
        try:
            out = res.clone() if with_residual else torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            moe.forward(dims, d["x"], d["wr"], d["bias"], wu, wd, out, ws, scales=scales,
                        residual=out if with_residual else None)
            moe.check_device_error()
            outs.append(out)
        finally:
            moe.debug_set(8, 1)
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("w", [W.WORKLOADS[0], W.WORKLOADS[1]], ids=lambda w: w.name)
def test_router_l2_prefetch_changes_no_result(moe, w):
    """The decode router's L2 prefetch of the up bank's leading bytes is a hint: off, a ragged
    size (48 bytes, one 32 KB piece and 16 bytes), the default and a size past the bank's end
    (clamped to it) give the same routing and layer output bit for bit."""
    h = inputs(w)
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    runs = []
    for warm in (0, 48, 32 * 1024 + 16, -1, 1 << 40):
        moe.debug_set(9, warm)
        try:
            out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
            wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
            moe.forward(dims, d["x"], d["wr"], d["bias"], d["wu"], d["wd"], out, ws, topk_idx=idx, topk_w=wt)
            moe.check_device_error()
            runs.append((out, idx, wt))
        finally:
            moe.debug_set(9, -1)
    for out, idx, wt in runs[1:]:
        assert torch.equal(out, runs[0][0]) and torch.equal(idx, runs[0][1]) and torch.equal(wt, runs[0][2])


@pytest.mark.parametrize("fill", [0x00, 0x7F, 0xFF], ids=["zeros", "0x7F", "0xFF"])
def test_one_launch_ffn_ignores_stale_workspace(moe, fill):
    """The one-launch FFN's per-entry counters live in the workspace and are zeroed by the row
    gather of every call: a workspace full of stale bytes (or the previous call's counts) gives
    the same output bit for bit, call after call."""
    w = W.WORKLOADS[1]
    h = inputs(w)
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    ref = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    moe.debug_set(8, 0)
    try:
        moe.forward(dims, d["x"], d["wr"], d["bias"], d["wu"], d["wd"], ref, ws)
    finally:
        moe.debug_set(8, 1)
    ws.fill_(fill)
    for _ in range(3):
        out = torch.full((w.T, w.H), 7.0, dtype=torch.bfloat16, device="cuda")
        moe.forward(dims, d["x"], d["wr"], d["bias"], d["wu"], d["wd"], out, ws)
        moe.check_device_error()
        assert torch.equal(out, ref)
