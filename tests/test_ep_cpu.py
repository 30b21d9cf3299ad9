"""Expert parallelism (routed_expert_moe_b200.ep) across gloo ranks on CPU.

Rank p owns experts [p*E/W, (p+1)*E/W) and routes its own tokens; the token
rows travel to the experts' owners and back in two all-to-alls.  The layer's
kernels are replaced here by oracle-backed steps (test infrastructure), so
what is checked is the exchange itself: the split sizes, the regrouping by
local expert and the return order.  Every rank's output must equal the
one-process oracle layer on its tokens exactly (same fp64 expert function,
same combine order).  On GPUs the same code runs the library's kernels and
NCCL; that path is exercised on one GPU by the world-size-1 GPU test.
"""
import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleOps:
    """The layer's steps on CPU from the oracle (bf16 rows travel as int16 bit patterns, expert
    outputs as float64)."""

    def __init__(self, E, K, H):
        import oracle
        self.o, self.E, self.K, self.H = oracle, E, K, H

    def route(self, x, w_router, bias):
        _, idx, w = self.o.route(x.numpy().view(np.uint16), w_router, bias, self.K)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def permute(self, idx):
        counts, offsets, perm_src, inv_row = self.o.permute(idx.numpy(), self.E)
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in (counts, offsets, perm_src, inv_row))

    def gather(self, x, perm, K):
        return x[perm.long() // K]

    def expert_ffn(self, rows, offsets, perm, w_up, w_down, scales=None):
        R = rows.shape[0]
        if R == 0:
            return torch.zeros(0, self.H, dtype=torch.float64)
        bits = rows.numpy().view(np.uint16)[perm.numpy()]
        ex = (np.searchsorted(offsets.numpy(), np.arange(R), side="right") - 1).astype(np.int32)
        slot = self.o.identity_slot(w_up[0].shape[0] if scales is not None else w_up.shape[0])
        if scales is None:
            y = self.o.expert_rows_bf16(self.o.bf16_to_f64(bits), ex, w_up, w_down, slot)
        else:                              # W8A8: banks (codes, tensor scales), scales (x, h)
            (qu, su), (qd, sd), (sx, sh) = w_up, w_down, scales
            y = self.o.expert_rows_fp8(self.o.quantize_act_fp8(bits, sx), ex, qu, su, qd, sd, slot, sx, sh)
        return torch.from_numpy(y)

    def combine(self, y_perm, inv_row, w, residual, out):
        T = out.shape[0]
        y_tk = y_perm.numpy()[inv_row.numpy()].reshape(T, self.K, self.H)
        out[:] = torch.from_numpy(self.o.combine(y_tk, w.numpy().astype(np.float64), residual))
        return out


def _worker(rank, world, port, T, q, fp8=False):
    try:
        _run(rank, world, port, T, q, fp8)
    except BaseException:                                 # report, so the parent fails at once
        import traceback
        q.put((rank, None, traceback.format_exc()))
        raise


def _run(rank, world, port, T, q, fp8):
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    from synth import workloads as W
    from routed_expert_moe_b200.ep import ExpertParallelLayer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.Workload("ep", T, 256, 8, 2, 128, seed=31)
        x = W.host_x(w, layer=rank)                       # each rank its own tokens
        wr, wu, wd = W.host_router(w), W.host_w_up(w), W.host_w_down(w)
        layer = ExpertParallelLayer(w.H, w.E, w.K, w.F, ops=OracleOps(w.E, w.K, w.H))
        mine = list(layer.experts())
        out = torch.empty(T, w.H, dtype=torch.float64)
        if fp8:
            import oracle
            qu, su = oracle.quantize_bank_fp8(wu)
            qd, sd = oracle.quantize_bank_fp8(wd)
            sc = oracle.calibrate_fp8(W.host_x(w)[:16], wr, None, wu, w.K)
            idx, _ = layer.forward(torch.from_numpy(x.view(np.int16)), wr, None, (qu[mine], su[mine]),
                                   (qd[mine], sd[mine]), out, scales=sc)
        else:
            idx, _ = layer.forward(torch.from_numpy(x.view(np.int16)), wr, None, np.ascontiguousarray(wu[mine]),
                                   np.ascontiguousarray(wd[mine]), out)
        q.put((rank, out.numpy(), idx.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,fp8", [(2, 16, False), (4, 9, False), (2, 1, False), (2, 12, True)])
def test_expert_parallel_layer_equals_the_one_process_layer(world, T, fp8):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q, fp8)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, o, i = q.get(timeout=180)
        if o is None:
            for p in procs:
                p.kill()
            pytest.fail(f"rank {r} failed:\n{i}")
        res[r] = (o, i)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from synth import workloads as W
    w = W.Workload("ep", T, 256, 8, 2, 128, seed=31)
    wr, wu, wd = W.host_router(w), W.host_w_up(w), W.host_w_down(w)
    if fp8:
        qu, su = oracle.quantize_bank_fp8(wu)
        qd, sd = oracle.quantize_bank_fp8(wd)
        sx, sh = oracle.calibrate_fp8(W.host_x(w)[:16], wr, None, wu, w.K)
    for rank in range(world):
        ref = (oracle.moe_layer_fp8(W.host_x(w, layer=rank), wr, None, qu, su, qd, sd, sx, sh, w.K) if fp8 else
               oracle.moe_layer_bf16(W.host_x(w, layer=rank), wr, None, wu, wd, w.K))
        out, idx = res[rank]
        assert np.array_equal(idx, ref["idx"])
        assert np.array_equal(out, ref["out"])


def test_regroup_orders_rows_by_expert_then_source():
    from routed_expert_moe_b200.ep import regroup
    rng = np.random.default_rng(3)
    for W_, E_loc in ((1, 4), (3, 2), (4, 5)):
        counts = rng.integers(0, 4, size=(W_, E_loc))
        counts[0, 0] = 0
        off, perm, inv = regroup(counts)
        # brute force: label every received row (source p, expert e, i) in arrival order
        labels = [(p, e, i) for p in range(W_) for e in range(E_loc) for i in range(counts[p, e])]
        want = sorted(range(len(labels)), key=lambda r: (labels[r][1], labels[r][0], labels[r][2]))
        assert perm.tolist() == want
        assert np.array_equal(inv[perm], np.arange(len(labels)))
        assert off.tolist() == [0] + np.cumsum(counts.sum(0)).tolist()
