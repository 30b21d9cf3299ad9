"""GPU parity of every router shape against the oracle's fixed-point ranking.

Small batches run as one launch of 8-CTA clusters split over the experts;
larger ones as int8 slices multiplied exactly on the tensor cores (E <= 128),
as one launch of clusters split over the hidden dimension (E <= 128), or as
the tiled logits kernel plus the top-K kernel.  Debug hooks 4 and 5 choose
the path, so every case here runs through all four (a case with E > 128 sent
to the tensor cores or the split clusters takes the two-kernel router).
Indices must be bit-exact and weights within 1e-5 (fp32 softmax over exact
selections).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

from _gpu import dev, dev_bf16

pytestmark = pytest.mark.gpu

# path: (largest batch of the expert-split clusters, router of larger batches: 1 two kernels,
# 2 hidden-split clusters, 3 tensor cores)
PATHS = {"cluster": (1 << 40, 0), "split": (0, 2), "tiled": (0, 1), "tensor": (0, 3)}


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    yield m
    restore(m)


def choose(moe, path):
    small_max, two_kernel = PATHS[path]
    moe.debug_set(4, small_max)
    moe.debug_set(5, two_kernel)


def restore(moe):
    moe.debug_set(4, -1)
    moe.debug_set(5, 0)


def route_case(moe, path, x, wr, bias, K):
    T, H = x.shape
    E = wr.shape[0]
    dims = moe.dims(T, H, E, K, 16)
    ws = moe.alloc_workspace(dims)
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, K, dtype=torch.float32, device="cuda")
    choose(moe, path)
    try:
        moe.route(dims, dev_bf16(x), dev_bf16(wr), None if bias is None else dev(bias), idx, wt, ws)
        moe.check_device_error()
    finally:
        restore(moe)
    _, ridx, rw = oracle.route(x, wr, bias, K)
    got = idx.cpu().numpy()
    assert np.array_equal(got, ridx)
    assert np.max(np.abs(wt.cpu().numpy().astype(np.float64) - rw)) <= 1e-5
    return got


SHAPES = [  # T, H, E, K, bias
    (1, 2688, 128, 6, False), (5, 2688, 128, 6, True), (64, 2688, 128, 6, False),
    (128, 2688, 128, 6, True), (129, 2688, 128, 6, False), (300, 1024, 256, 16, True),
    (512, 2688, 128, 6, False), (513, 512, 100, 1, True), (37, 8192, 8, 2, False),
    (70, 272, 256, 8, False), (17, 256, 9, 9, True), (1000, 2688, 128, 6, True),
    (300, 16, 128, 4, False), (4096, 2688, 128, 6, False),
]


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("T,H,E,K,with_bias", SHAPES, ids=[f"T{s[0]}_H{s[1]}_E{s[2]}_K{s[3]}" for s in SHAPES])
def test_router_shapes(moe, path, T, H, E, K, with_bias):
    seed = 1000 + T + H + E + K
    x = synth.normal_bf16(synth.key(seed, synth.T_X, 0), T * H, W.SIGMA_X).reshape(T, H)
    wr = synth.normal_bf16(synth.key(seed, synth.T_WR, 0), E * H, W.SIGMA_W).reshape(E, H)
    bias = W.zipf_bias(seed, E) if with_bias else None
    route_case(moe, path, x, wr, bias, K)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_router_exact_fallback_on_ties(moe, path):
    """Duplicated router rows give exactly equal logits: the certificate must fail and
    the exact pass must break the ties toward the lower index, in every token."""
    T, H, E, K = 40, 2688, 128, 6
    x = synth.normal_bf16(synth.key(77, synth.T_X, 0), T * H, W.SIGMA_X).reshape(T, H)
    wr = synth.normal_bf16(synth.key(77, synth.T_WR, 0), E * H, W.SIGMA_W).reshape(E, H).copy()
    for dup in (17, 90, 127):
        wr[dup] = wr[3]
    bias = np.zeros(E, np.float32)
    bias[[3, 17, 90, 127]] = 30.0
    got = route_case(moe, path, x, wr, bias, K)
    assert np.all(got[:, :4] == np.array([3, 17, 90, 127]))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_router_near_ties_below_the_bound(moe, path):
    """Rows that differ in the last mantissa bit of one weight: logit gaps of the
    size of the fp32 bound, which the exact fixed-point sums must decide."""
    T, H, E, K = 24, 2688, 128, 6
    x = synth.normal_bf16(synth.key(78, synth.T_X, 0), T * H, W.SIGMA_X).reshape(T, H)
    wr = synth.normal_bf16(synth.key(78, synth.T_WR, 0), E * H, W.SIGMA_W).reshape(E, H).copy()
    for j, dup in enumerate((40, 41, 42)):
        wr[dup] = wr[7]
        wr[dup, 11 + j] ^= 1            # flip the last mantissa bit of one weight
    bias = np.zeros(E, np.float32)
    bias[[7, 40, 41, 42]] = 30.0
    route_case(moe, path, x, wr, bias, K)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_router_reports_the_range_error(moe, path):
    T, H, E, K = 16, 256, 8, 2
    x = np.full((T, H), 0x4700, np.uint16)   # bf16 32768.0
    wr = np.full((E, H), 0x4700, np.uint16)
    dims = moe.dims(T, H, E, K, 16)
    ws = moe.alloc_workspace(dims)
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, K, dtype=torch.float32, device="cuda")
    choose(moe, path)
    try:
        moe.route(dims, dev_bf16(x), dev_bf16(wr), None, idx, wt, ws)
        assert moe.check_device_error_status() == moe.MOE_ERANGE
    finally:
        restore(moe)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_router_wide_dynamic_range(moe, path):
    """Rows whose values span many binades (a few values near 2^6, the rest down to 2^-20 and
    subnormal-sized, zeros and a zero row): the tensor-core router's int8 slices drop the small
    values' low bits, so its bound is wide and many tokens go to the exact pass; the ranking
    must still be the oracle's."""
    T, H, E, K = 300, 2688, 128, 6
    rng = np.random.default_rng(5)
    x = synth.normal_bf16(synth.key(79, synth.T_X, 0), T * H, W.SIGMA_X).reshape(T, H).copy()
    wr = synth.normal_bf16(synth.key(79, synth.T_WR, 0), E * H, W.SIGMA_W).reshape(E, H).copy()
    xf = oracle.bf16_to_f64(x) * np.exp2(rng.integers(-20, 1, size=(T, H)))
    xf[:, :3] = 64.0 * np.sign(xf[:, :3] + 1e-30)
    xf[7] = 0.0
    xf[:, 100:110] = 0.0
    x = oracle.round_bf16(xf)
    wf = oracle.bf16_to_f64(wr) * np.exp2(rng.integers(-12, 1, size=(E, H)))
    wr = oracle.round_bf16(wf)
    route_case(moe, path, x, wr, W.zipf_bias(80, E), K)


@pytest.mark.parametrize("fill", [0x00, 0xFF])
def test_tensor_core_router_ignores_stale_workspace(moe, fill):
    """The tensor-core router writes every slice, scale and partial it reads: a workspace full of
    stale bytes gives the oracle's ranking, call after call."""
    T, H, E, K = 2100, 2688, 128, 6
    x = synth.normal_bf16(synth.key(81, synth.T_X, 0), T * H, W.SIGMA_X).reshape(T, H)
    wr = synth.normal_bf16(synth.key(81, synth.T_WR, 0), E * H, W.SIGMA_W).reshape(E, H)
    bias = W.zipf_bias(81, E)
    dims = moe.dims(T, H, E, K, 16)
    ws = moe.alloc_workspace(dims)
    _, ridx, rw = oracle.route(x, wr, bias, K)
    for _ in range(2):
        ws.fill_(fill)
        idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
        wt = torch.empty(T, K, dtype=torch.float32, device="cuda")
        moe.route(dims, dev_bf16(x), dev_bf16(wr), dev(bias), idx, wt, ws)   # T >= 2048: the tensor cores
        moe.check_device_error()
        assert np.array_equal(idx.cpu().numpy(), ridx)
        assert np.max(np.abs(wt.cpu().numpy().astype(np.float64) - rw)) <= 1e-5
