"""GPU parity: every entry point of the C ABI against the oracle.

Expert indices and the permutation must be bit-exact; outputs must satisfy
max|err| / max|ref| <= 1e-2 (BF16).  Inputs are the seeded workloads of
``synth.workloads``; the oracle never sees a value the GPU produced.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import workloads as W

from _gpu import BF16_TOL, dev, dev_bf16, device_inputs, host_bits, host_f64, inputs, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def small_workloads():
    return [W.WORKLOADS[0], W.WORKLOADS[1], W.WORKLOADS[3],
            W.Workload("ragged_T37_E16_K4", 37, 512, 16, 4, 192, seed=11),
            W.Workload("T1", 1, 2688, 128, 6, 1856, seed=12),
            W.Workload("E_equals_K", 9, 256, 4, 4, 128, seed=13),
            W.Workload("odd_F_tail_H272_F208", 21, 272, 8, 3, 208, seed=14)]


WL_IDS = [w.name for w in small_workloads()]


def run_route(moe, w, d):
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    moe.route(dims, d["x"], d["wr"], d["bias"], idx, wt, ws)
    moe.check_device_error()
    return idx.cpu().numpy(), wt.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("w", small_workloads(), ids=WL_IDS)
def test_route_bit_exact_indices(moe, w):
    h = inputs(w)
    d = device_inputs(h)
    idx, wt = run_route(moe, w, d)
    L, ridx, rw = oracle.route(h["x"], h["wr"], h["bias"], w.K)
    assert np.array_equal(idx, ridx)
    assert np.max(np.abs(wt - rw)) <= 1e-5
    assert np.allclose(wt.sum(1), 1.0, atol=1e-5)


def test_route_ties_and_planted_bias(moe):
    w = W.WORKLOADS[0]
    h = inputs(w)
    wr = h["wr"].copy()
    wr[5] = wr[1]
    wr[6] = wr[1]
    bias = np.zeros(w.E, np.float32)
    bias[[1, 5, 6]] = 50.0
    dims = moe.dims(w.T, w.H, w.E, 3, w.F)
    ws = moe.alloc_workspace(dims)
    idx = torch.empty(w.T, 3, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, 3, dtype=torch.float32, device="cuda")
    moe.route(dims, dev_bf16(h["x"]), dev_bf16(wr), dev(bias), idx, wt, ws)
    moe.check_device_error()
    _, ridx, rw = oracle.route(h["x"], wr, bias, 3)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.all(ridx == np.array([1, 5, 6]))


@pytest.mark.parametrize("w", small_workloads(), ids=WL_IDS)
def test_permute_bit_exact(moe, w):
    h = inputs(w)
    _, ridx, _ = oracle.route(h["x"], h["wr"], h["bias"], w.K)
    counts, offsets, perm_src, inv_row = oracle.permute(ridx, w.E)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    g = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (w.E, w.E + 1, w.T * w.K, w.T * w.K)]
    moe.permute(dims, dev(ridx), *g)
    moe.check_device_error()
    for got, ref in zip(g, (counts, offsets, perm_src, inv_row)):
        assert np.array_equal(got.cpu().numpy(), ref)


def oracle_y_perm(h, w, perm_src):
    xf = oracle.bf16_to_f64(h["x"])
    _, ridx, _ = oracle.route(h["x"], h["wr"], h["bias"], w.K)
    src = perm_src
    rows_x = xf[src // w.K]
    ex = ridx.reshape(-1)[src]
    return oracle.expert_rows_bf16(rows_x, ex, h["wu"], h["wd"], oracle.identity_slot(w.E))


@pytest.mark.parametrize("w", small_workloads(), ids=WL_IDS)
def test_expert_ffn_parity(moe, w):
    h = inputs(w)
    d = device_inputs(h)
    _, ridx, _ = oracle.route(h["x"], h["wr"], h["bias"], w.K)
    counts, offsets, perm_src, inv_row = oracle.permute(ridx, w.E)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    y = torch.empty(w.T * w.K, w.H, dtype=torch.bfloat16, device="cuda")
    moe.expert_ffn(dims, d["x"], dev(offsets), dev(perm_src), d["wu"], d["wd"], None, y, ws)
    moe.check_device_error()
    ref = oracle_y_perm(h, w, perm_src)
    assert rel_err(host_f64(y), ref) <= BF16_TOL


@pytest.mark.parametrize("w", small_workloads(), ids=WL_IDS)
def test_combine_parity(moe, w):
    import synth
    h = inputs(w)
    _, ridx, rw = oracle.route(h["x"], h["wr"], h["bias"], w.K)
    _, _, perm_src, inv_row = oracle.permute(ridx, w.E)
    yb = synth.normal_bf16(synth.key(w.seed, 40, 0), w.T * w.K * w.H, 1.0).reshape(w.T * w.K, w.H)
    res = synth.normal_bf16(synth.key(w.seed, 41, 0), w.T * w.H, 1.0).reshape(w.T, w.H)
    w32 = rw.astype(np.float32)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    for residual in (None, res):
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        moe.combine(dims, dev_bf16(yb), dev(inv_row), dev(w32),
                    None if residual is None else dev_bf16(residual), out)
        moe.check_device_error()
        y_tk = oracle.bf16_to_f64(yb)[inv_row].reshape(w.T, w.K, w.H)
        ref = oracle.combine(y_tk, w32.astype(np.float64), residual)
        got = host_f64(out)
        # one rounding to bf16 of an fp32 sum: within 2^-8 relative (+ fp32 sum error)
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(ref)))


@pytest.mark.parametrize("w", small_workloads(), ids=WL_IDS)
def test_forward_parity(moe, w):
    h = inputs(w)
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    moe.forward(dims, d["x"], d["wr"], d["bias"], d["wu"], d["wd"], out, ws, topk_idx=idx, topk_w=wt)
    moe.check_device_error()
    r = oracle.moe_layer_bf16(h["x"], h["wr"], h["bias"], h["wu"], h["wd"], w.K)
    assert np.array_equal(idx.cpu().numpy(), r["idx"])
    assert rel_err(host_f64(out), r["out"]) <= BF16_TOL


def test_forward_hot_experts_split_into_token_blocks(moe):
    """Every token routed to the same K experts: segments of 600 rows > 256."""
    w = W.Workload("hot", 600, 512, 16, 3, 256, seed=15)
    h = inputs(w)
    bias = np.zeros(w.E, np.float32)
    bias[[2, 9, 14]] = [60.0, 50.0, 40.0]   # gaps far above the logit spread
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    moe.forward(dims, d["x"], d["wr"], dev(bias), d["wu"], d["wd"], out, ws)
    moe.check_device_error()
    r = oracle.moe_layer_bf16(h["x"], h["wr"], bias, h["wu"], h["wd"], w.K)
    assert np.all(r["idx"] == np.array([2, 9, 14]))
    assert rel_err(host_f64(out), r["out"]) <= BF16_TOL


def test_forward_is_deterministic_and_empty_batch_is_a_no_op(moe):
    w = W.WORKLOADS[3]
    h = inputs(w)
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    outs = []
    for _ in range(2):
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        moe.forward(dims, d["x"], d["wr"], d["bias"], d["wu"], d["wd"], out, ws)
        outs.append(host_bits(out))
    moe.check_device_error()
    assert np.array_equal(outs[0], outs[1])
    d0 = moe.dims(0, w.H, w.E, w.K, w.F)
    moe.forward(d0, d["x"], d["wr"], None, d["wu"], d["wd"], d["x"], ws)


def test_forward_residual_is_added(moe):
    w = W.WORKLOADS[0]
    h = inputs(w)
    d = device_inputs(h)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    out = d["x"].clone()
    moe.forward(dims, d["x"], d["wr"], None, d["wu"], d["wd"], out, ws, residual=out)
    moe.check_device_error()
    r = oracle.moe_layer_bf16(h["x"], h["wr"], None, h["wu"], h["wd"], w.K, residual=h["x"])
    assert rel_err(host_f64(out), r["out"]) <= BF16_TOL


def test_permute_reports_out_of_range_index(moe):
    dims = moe.dims(4, 256, 8, 2, 128)
    idx = dev(np.array([[0, 1], [2, 9], [3, 4], [5, 6]], np.int32))
    g = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (8, 9, 8, 8)]
    moe.permute(dims, idx, *g)
    assert moe.check_device_error_status() == moe.MOE_EINDEX
    moe.check_device_error()   # the word was cleared


def test_route_reports_magnitudes_beyond_the_exact_range(moe):
    w = W.WORKLOADS[0]
    h = inputs(w)
    x = np.full((w.T, w.H), 0x4700, np.uint16)   # bf16 32768.0 everywhere
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    wt = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    wr = np.full((w.E, w.H), 0x4700, np.uint16)
    moe.route(dims, dev_bf16(x), dev_bf16(wr), None, idx, wt, ws)
    assert moe.check_device_error_status() == moe.MOE_ERANGE


def test_host_rejects_bad_arguments(moe):
    w = W.WORKLOADS[0]
    d = device_inputs(inputs(w))
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.forward(dims, d["x"], d["wr"], None, d["wu"], d["wd"], out, ws[:100])
    assert e.value.status == moe.MOE_EWORKSPACE
    with pytest.raises(moe.MoeError) as e:
        moe.forward(moe.dims(w.T, w.H, w.E, w.E + 1, w.F), d["x"], d["wr"], None, d["wu"], d["wd"], out, ws)
    assert e.value.status == moe.MOE_EINVAL
    with pytest.raises(moe.MoeError) as e:
        moe.forward(dims, d["x"][:, 1:], d["wr"], None, d["wu"], d["wd"], out, ws)   # misaligned
    assert e.value.status == moe.MOE_EINVAL


@pytest.mark.parametrize("T,E,K,zipf", [(1000, 16, 5, True), (4096, 128, 6, False), (683, 256, 6, True)])
def test_permute_multi_block_bit_exact(moe, T, E, K, zipf):
    """More than 4096 assignments: the chunked multi-block sort (ragged last chunk, empty experts)."""
    w = W.Workload(f"perm_T{T}_E{E}", T, 256, E, K, 128, seed=19)
    x = W.host_x(w)
    wr = W.host_router(w)
    bias = W.zipf_bias(19, E) if zipf else None
    _, ridx, _ = oracle.route(x, wr, bias, K)
    ref = oracle.permute(ridx, E)
    dims = moe.dims(T, 256, E, K, 128)
    ws = moe.alloc_workspace(dims)
    g = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, T * K, T * K)]
    with pytest.raises(moe.MoeError) as err:
        moe.permute(dims, dev(ridx), *g)        # needs scratch above 4096 assignments
    assert err.value.status == moe.MOE_EWORKSPACE
    moe.permute(dims, dev(ridx), *g, ws=ws)
    moe.check_device_error()
    for got, r in zip(g, ref):
        assert np.array_equal(got.cpu().numpy(), r)
