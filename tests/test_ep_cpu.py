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


def host_regroup(recv_counts: np.ndarray):
    """The grouped layout of received rows, stated on the host: rows arrive source-major
    ([source][local expert] blocks); grouped row r holds the received row given by the
    expert-major, then source, then arrival order.  Returns (offsets, perm, inv)."""
    W, E_loc = recv_counts.shape
    src_base = np.concatenate([[0], np.cumsum(recv_counts.sum(1))])[:-1]
    within = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(recv_counts, axis=1)[:, :-1]], axis=1)
    perm = [np.arange(src_base[p] + within[p, e], src_base[p] + within[p, e] + recv_counts[p, e])
            for e in range(E_loc) for p in range(W)]
    perm = np.concatenate(perm).astype(np.int32) if perm else np.zeros(0, np.int32)
    offsets = np.concatenate([[0], np.cumsum(recv_counts.sum(0))]).astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return offsets, perm, inv


class OracleOps:
    """The layer's steps on CPU from the oracle (bf16 rows travel as int16 bit patterns, expert
    outputs as float64).  fmt: the experts' format; the banks and scales are the oracle's."""

    def __init__(self, E, K, H, F=None, fmt="bf16"):
        import oracle
        self.o, self.E, self.K, self.H, self.F, self.fmt = oracle, E, K, H, F, fmt

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
        o = self.o
        bits = rows.numpy().view(np.uint16)[perm.numpy()]
        ex = (np.searchsorted(offsets.numpy(), np.arange(R), side="right") - 1).astype(np.int32)
        slot = o.identity_slot(len(w_up[0]) if scales is not None else w_up.shape[0])
        if self.fmt == "bf16":
            y = o.expert_rows_bf16(o.bf16_to_f64(bits), ex, w_up, w_down, slot)
        elif self.fmt == "fp8":            # banks (codes, tensor scales); scales (x, h)
            (qu, su), (qd, sd), (sx, sh) = w_up, w_down, scales
            y = o.expert_rows_fp8(o.quantize_act_fp8(bits, sx), ex, qu, su, qd, sd, slot, sx, sh)
        elif self.fmt == "nvfp4":          # banks (codes, block scales, tensor scales)
            tx, th = scales
            cx, sx_ = o.quantize_nvfp4(bits, tx)
            y = o.expert_rows_nvfp4(cx, sx_, ex, w_up, w_down, slot, tx, th)
        else:                              # fp8_b128: banks (codes, block scales)
            sx, sh = scales
            y = o.expert_rows_fp8_b128(o.quantize_act_fp8_b128(bits, sx), ex, w_up, w_down, slot, sx, sh,
                                       self.H, self.F)
        return torch.from_numpy(y)

    def regroup(self, recv_counts, R):
        off, perm, inv = host_regroup(recv_counts.numpy())
        assert perm.size == R
        return tuple(torch.from_numpy(a) for a in (off, perm, inv))

    def combine(self, y_perm, inv_row, w, residual, out):
        T = out.shape[0]
        y_tk = y_perm.numpy()[inv_row.numpy()].reshape(T, self.K, self.H)
        out[:] = torch.from_numpy(self.o.combine(y_tk, w.numpy().astype(np.float64), residual))
        return out


def _worker(rank, world, port, T, q, fmt="bf16"):
    try:
        _run(rank, world, port, T, q, fmt)
    except BaseException:                                 # report, so the parent fails at once
        import traceback
        q.put((rank, None, traceback.format_exc()))
        raise


def local_banks(o, fmt, wu, wd, mine):
    """This rank's experts in the layer's format (the oracle quantises every bank)."""
    if fmt == "bf16":
        return np.ascontiguousarray(wu[mine]), np.ascontiguousarray(wd[mine])
    q = {"fp8": o.quantize_bank_fp8, "nvfp4": o.quantize_bank_nvfp4, "fp8_b128": o.quantize_fp8_b128}[fmt]
    bu, bd = q(wu), q(wd)
    return tuple(np.ascontiguousarray(a[mine]) for a in bu), tuple(np.ascontiguousarray(a[mine]) for a in bd)


def act_scales(o, fmt, w, wr, wu):
    if fmt == "nvfp4":
        return o.calibrate_nvfp4(_x(w, 0)[:16], wr, None, wu, w.K)
    return o.calibrate_fp8(_x(w, 0)[:16], wr, None, wu, w.K)


def _x(w, rank):
    from synth import workloads as W
    return W.host_x(w, layer=rank)


def reference(o, fmt, w, x, wr, wu, wd):
    if fmt == "bf16":
        return o.moe_layer_bf16(x, wr, None, wu, wd, w.K)
    s1, s2 = act_scales(o, fmt, w, wr, wu)
    if fmt == "fp8":
        qu, su = o.quantize_bank_fp8(wu)
        qd, sd = o.quantize_bank_fp8(wd)
        return o.moe_layer_fp8(x, wr, None, qu, su, qd, sd, s1, s2, w.K)
    if fmt == "nvfp4":
        return o.moe_layer_nvfp4(x, wr, None, o.quantize_bank_nvfp4(wu), o.quantize_bank_nvfp4(wd), s1, s2, w.K)
    return o.moe_layer_fp8_b128(x, wr, None, o.quantize_fp8_b128(wu), o.quantize_fp8_b128(wd), s1, s2, w.K,
                                w.H, w.F)


def _run(rank, world, port, T, q, fmt):
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
        import oracle
        layer = ExpertParallelLayer(w.H, w.E, w.K, w.F, ops=OracleOps(w.E, w.K, w.H, w.F, fmt))
        mine = list(layer.experts())
        out = torch.empty(T, w.H, dtype=torch.float64)
        bu, bd = local_banks(oracle, fmt, wu, wd, mine)
        sc = None if fmt == "bf16" else act_scales(oracle, fmt, w, wr, wu)
        idx, _ = layer.forward(torch.from_numpy(x.view(np.int16)), wr, None, bu, bd, out, scales=sc)
        q.put((rank, out.numpy(), idx.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,fmt", [(2, 16, "bf16"), (4, 9, "bf16"), (2, 1, "bf16"), (2, 12, "fp8"),
                                         (2, 12, "nvfp4"), (2, 12, "fp8_b128")])
def test_expert_parallel_layer_equals_the_one_process_layer(world, T, fmt):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, q, fmt)) for r in range(world)]
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
    for rank in range(world):
        ref = reference(oracle, fmt, w, W.host_x(w, layer=rank), wr, wu, wd)
        out, idx = res[rank]
        assert np.array_equal(idx, ref["idx"])
        assert np.array_equal(out, ref["out"])


def test_regroup_orders_rows_by_expert_then_source():
    rng = np.random.default_rng(3)
    for W_, E_loc in ((1, 4), (3, 2), (4, 5)):
        counts = rng.integers(0, 4, size=(W_, E_loc))
        counts[0, 0] = 0
        off, perm, inv = host_regroup(counts)
        # brute force: label every received row (source p, expert e, i) in arrival order
        labels = [(p, e, i) for p in range(W_) for e in range(E_loc) for i in range(counts[p, e])]
        want = sorted(range(len(labels)), key=lambda r: (labels[r][1], labels[r][0], labels[r][2]))
        assert perm.tolist() == want
        assert np.array_equal(inv[perm], np.arange(len(labels)))
        assert off.tolist() == [0] + np.cumsum(counts.sum(0)).tolist()


def _failing_worker(rank, world, port, q):
    """Rank 1 leaves before the layer's first exchange; rank 0 must get an error from its
    collective (the group's short timeout, or the peer's closed connection), not hang."""
    import datetime
    import time
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    from synth import workloads as W
    from routed_expert_moe_b200.ep import ExpertParallelLayer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=3))
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()                                 # the message is sent before the process goes
        os._exit(0)                                     # gone, with no collective in flight
    w = W.Workload("ep", 8, 256, 8, 2, 128, seed=31)
    layer = ExpertParallelLayer(w.H, w.E, w.K, w.F, ops=OracleOps(w.E, w.K, w.H))
    mine = list(layer.experts())
    out = torch.empty(w.T, w.H, dtype=torch.float64)
    t0 = time.monotonic()
    try:
        layer.forward(torch.from_numpy(W.host_x(w).view(np.int16)), W.host_router(w), None,
                      np.ascontiguousarray(W.host_w_up(w)[mine]), np.ascontiguousarray(W.host_w_down(w)[mine]), out)
        q.put((rank, "no error"))
    except Exception as e:                              # the failure reaches this rank as an error
        q.put((rank, f"error after {time.monotonic() - t0:.1f} s: {type(e).__name__}"))
    q.close()
    q.join_thread()
    os._exit(0)


def test_a_rank_that_leaves_ends_the_exchange_with_an_error():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    assert res[1] == "left"
    assert res[0].startswith("error after"), res[0]
    assert float(res[0].split()[2]) < 60

