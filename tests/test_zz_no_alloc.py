"""The router entry point that allocates nothing (moe_route_static).

It exists for callers that cannot allocate device memory for a workspace,
for example code inside a host framework whose pool allocator owns all
device memory, or a decode loop that must not call cudaMalloc because that
call can synchronise the device.  Its scratch is a fixed 8 MiB array that
the library holds on every GPU that loads it.

These tests call it through the C ABI and check that two calls in a row give
the same routing as moe_route (which takes a caller workspace): indices bit
for bit and weights within the tolerance of the router parity tests.  The
file sorts last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from synth import workloads as W

from _gpu import dev, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def _route_with_workspace(moe, dims, x, wr, bias, T, K):
    ws = moe.alloc_workspace(dims)
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, K, dtype=torch.float32, device="cuda")
    moe.route(dims, x, wr, bias, idx, wt, ws)
    moe.check_device_error()
    return idx.cpu().numpy(), wt.cpu().numpy()


def _route_static_abi(moe, dims, x, wr, bias, T, K):
    idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
    wt = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.raw_library().moe_route_static(ctypes.byref(dims), ctypes.c_void_p(x.data_ptr()),
                                            ctypes.c_void_p(wr.data_ptr()),
                                            None if bias is None else ctypes.c_void_p(bias.data_ptr()),
                                            ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(wt.data_ptr()),
                                            stream)
    assert rc == moe.MOE_OK, moe.status_string(rc)
    moe.check_device_error()
    return idx.cpu().numpy(), wt.cpu().numpy()


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
def test_static_scratch_router_matches_the_workspace_router_twice(moe, cfg):
    w = W.WORKLOADS[cfg]
    x = dev_bf16(W.host_x(w))
    wr = dev_bf16(W.host_router(w))
    b = W.host_bias(w)
    bias = None if b is None else dev(b)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
    ref_idx, ref_w = _route_with_workspace(moe, dims, x, wr, bias, w.T, w.K)
    for _ in range(2):
        idx, wt = _route_static_abi(moe, dims, x, wr, bias, w.T, w.K)
        assert np.array_equal(idx, ref_idx)
        assert np.max(np.abs(wt - ref_w)) <= 1e-5


def test_static_scratch_router_rejects_batches_beyond_its_array(moe):
    dims = moe.dims(8128, 2688, 128, 6, 1856)
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(16, dtype=torch.int32, device="cuda")
    rc = moe.raw_library().moe_route_static(ctypes.byref(dims), ctypes.c_void_p(x.data_ptr()),
                                            ctypes.c_void_p(x.data_ptr()), None, ctypes.c_void_p(out.data_ptr()),
                                            ctypes.c_void_p(out.data_ptr()), None)
    assert rc == moe.MOE_EWORKSPACE


@pytest.mark.parametrize("T,split", [(1200, 0), (8000, 1)])
def test_static_scratch_router_at_large_batches(moe, T, split):
    """Batches whose usual split of the hidden dimension does not fit the array.

    T = 1200 takes the two-kernel router, whose usual plan (7 splits, 8.6 MB of
    partial logits) is cut down until it fits; T = 8000, near the 8127 limit,
    is forced onto the two-kernel router so that one split's partials fill
    most of the array.  Indices bit for bit against moe_route under the same
    router shape, weights within 1e-5, two calls in a row."""
    import synth
    H, E, K, F = 2688, 128, 6, 1856
    stream = torch.cuda.current_stream().cuda_stream
    x = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    wr = torch.empty(E, H, dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(synth.key(11, synth.T_X, 0), x.numel(), W.SIGMA_X, x.data_ptr(), stream)
    synth.normal_bf16_device(synth.key(11, synth.T_WR, 0), wr.numel(), W.SIGMA_W, wr.data_ptr(), stream)
    dims = moe.dims(T, H, E, K, F)
    moe.debug_set(5, split)
    try:
        ref_idx, ref_w = _route_with_workspace(moe, dims, x, wr, None, T, K)
        for _ in range(2):
            idx, wt = _route_static_abi(moe, dims, x, wr, None, T, K)
            assert np.array_equal(idx, ref_idx)
            assert np.max(np.abs(wt - ref_w)) <= 1e-5
    finally:
        moe.debug_set(5, 0)


def test_static_scratch_takes_the_tensor_core_router_when_its_slices_fit(moe):
    """With the tensor-core router forced (debug hooks 4 = 0, 5 = 3), a batch whose int8 slices
    and partials fit the 8 MiB array (T = 100) takes it from the static scratch too: indices bit
    for bit against the workspace router under the same hooks, weights within 1e-5."""
    import synth
    T, H, E, K, F = 100, 2688, 128, 6, 1856
    stream = torch.cuda.current_stream().cuda_stream
    x = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    wr = torch.empty(E, H, dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(synth.key(12, synth.T_X, 0), x.numel(), W.SIGMA_X, x.data_ptr(), stream)
    synth.normal_bf16_device(synth.key(12, synth.T_WR, 0), wr.numel(), W.SIGMA_W, wr.data_ptr(), stream)
    dims = moe.dims(T, H, E, K, F)
    moe.debug_set(4, 0)
    moe.debug_set(5, 3)
    try:
        ref_idx, ref_w = _route_with_workspace(moe, dims, x, wr, None, T, K)
        for _ in range(2):
            idx, wt = _route_static_abi(moe, dims, x, wr, None, T, K)
            assert np.array_equal(idx, ref_idx)
            assert np.max(np.abs(wt - ref_w)) <= 1e-5
    finally:
        moe.debug_set(4, -1)
        moe.debug_set(5, 0)
