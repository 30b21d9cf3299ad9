"""The expert-parallel layer on one GPU (world size 1, NCCL): the library's
kernels behind ``routed_expert_moe_b200.ep.CudaOps`` with the row exchange as
NCCL all-to-alls to itself.  It must give the routing of ``forward`` bit for
bit and its output (the grouped GEMM then runs one expert's rows in wider
tiles) within rounding, and match the oracle within the BF16 tolerance.  The
exchange between several ranks is tested on CPU (gloo)."""
import socket

import numpy as np
import pytest
import torch

import oracle
from synth import workloads as W

from _gpu import BF16_TOL, device_inputs, host_f64, inputs, rel_err

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_gather_rows_matches_indexing():
    import routed_expert_moe_b200 as moe
    x = torch.randn(50, 264, device="cuda").to(torch.bfloat16)
    perm = torch.tensor(np.random.default_rng(1).integers(0, 150, 77), dtype=torch.int32, device="cuda")
    out = torch.empty(77, 264, dtype=torch.bfloat16, device="cuda")
    moe.gather_rows(x, perm, out, K=3)
    moe.check_device_error()
    assert torch.equal(out, x[perm.long() // 3])


@pytest.mark.parametrize("w", [W.Workload("ep_ragged_T37_E16_K4", 37, 512, 16, 4, 192, seed=41),
                               W.WORKLOADS[1]], ids=lambda w: w.name)
def test_expert_parallel_world_one_matches_forward(w):
    import torch.distributed as dist
    import routed_expert_moe_b200 as moe
    from routed_expert_moe_b200.ep import ExpertParallelLayer
    dist.init_process_group("nccl", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{_free_port()}")
    try:
        h = inputs(w)
        d = device_inputs(h)
        layer = ExpertParallelLayer(w.H, w.E, w.K, w.F)
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        idx, _ = layer.forward(d["x"], d["wr"], d["bias"], d["wu"], d["wd"], out)
        moe.check_device_error()
        dims = moe.dims(w.T, w.H, w.E, w.K, w.F)
        ref_out = torch.empty_like(out)
        ref_idx = torch.empty_like(idx)
        moe.forward(dims, d["x"], d["wr"], d["bias"], d["wu"], d["wd"], ref_out, moe.alloc_workspace(dims),
                    topk_idx=ref_idx)
        moe.check_device_error()
        assert torch.equal(idx, ref_idx)
        assert rel_err(host_f64(out), host_f64(ref_out)) <= 1e-2
        tok = np.arange(0, w.T, 5)
        r = oracle.moe_layer_bf16(h["x"], h["wr"], h["bias"], h["wu"], h["wd"], w.K, tokens=tok)
        assert rel_err(host_f64(out)[tok], r["out"]) <= BF16_TOL
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("W_,E_loc", [(1, 128), (2, 64), (8, 16), (4, 5), (16, 16)])
def test_device_regroup_orders_rows_by_expert_then_source(W_, E_loc):
    """moe_ep_regroup against a brute-force labelling of the received rows: every received row
    is (source p, local expert e, i-th of its block) in arrival order, and the grouped layout
    sorts them by (e, p, i)."""
    import routed_expert_moe_b200 as moe
    rng = np.random.default_rng(W_ * 100 + E_loc)
    counts = rng.integers(0, 7, size=(W_, E_loc))
    counts[0, 0] = 0
    counts[-1, :] = 0                         # a source that sends nothing
    labels = [(p, e, i) for p in range(W_) for e in range(E_loc) for i in range(counts[p, e])]
    want = sorted(range(len(labels)), key=lambda r: (labels[r][1], labels[r][0], labels[r][2]))
    R = len(labels)
    rc = torch.from_numpy(counts.astype(np.int64)).cuda()
    off = torch.empty(E_loc + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(R, dtype=torch.int32, device="cuda")
    inv = torch.empty(R, dtype=torch.int32, device="cuda")
    moe.ep_regroup(rc, off, perm, inv)
    moe.check_device_error()
    assert perm.cpu().tolist() == want
    assert np.array_equal(inv.cpu().numpy()[np.array(want, dtype=np.int64)], np.arange(R))
    assert off.cpu().tolist() == [0] + np.cumsum(counts.sum(0)).tolist()


def test_device_regroup_rejects_counts_that_do_not_sum_to_the_rows():
    import routed_expert_moe_b200 as moe
    rc = torch.tensor([[3, 1], [2, 2]], dtype=torch.int64, device="cuda")
    off = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    perm = torch.empty(7, dtype=torch.int32, device="cuda")    # 8 rows were announced
    inv = torch.empty(7, dtype=torch.int32, device="cuda")
    moe.ep_regroup(rc, off, perm, inv)
    assert moe.check_device_error_status() == moe.MOE_EINDEX
    assert off.cpu().tolist() == [-1, -1, -1]
