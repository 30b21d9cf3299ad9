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
