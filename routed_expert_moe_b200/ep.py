"""Expert parallelism for the routed MoE layer over a torch.distributed group.

Rank p of W owns the experts [p*E/W, (p+1)*E/W) and its own tokens.  One
layer pass on every rank:

1. route its tokens (full router, replicated) and permute the assignments into
   expert order, which is also the order of the experts' owners;
2. gather the token rows in that order and send each owner its rows (one
   all-to-all for the per-expert counts, one for the rows);
3. regroup the received rows by local expert (source rank, then the source's
   order, inside each expert; a kernel, from the received counts on the
   device) and run the local grouped FFN;
4. put the outputs back in the order they arrived and return them (one
   all-to-all);
5. combine the returned rows with the routing weights, as the one-device layer.

Tokens never interact and each assignment's expert output depends only on its
token row, so the result equals the one-device layer.  The split sizes cross
to the host once per pass (one read): NCCL's all-to-all needs them there.  The
row exchange moves raw bytes, so any row dtype travels unchanged.

The kernels come from an ``ops`` object (``CudaOps``: the library's calls on
the current CUDA device); the collectives from ``torch.distributed`` (NCCL on
GPUs).  The expert banks a rank passes hold its own experts only, in any of
the library's expert formats (bf16, FP8 E4M3, NVFP4, FP8_B128): the rows
travel in bf16 and the owner's grouped FFN quantises them, with the scales of
its own experts.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


FORMATS = ("bf16", "fp8", "nvfp4", "fp8_b128")


class CudaOps:
    """The layer's steps on the current CUDA device, through the library's C ABI.  Workspaces
    are kept per problem size and reused across passes (no allocation once warm)."""

    def __init__(self, H: int, E: int, K: int, F: int, experts: str = "bf16"):
        from . import dims as _dims
        import routed_expert_moe_b200 as moe
        if experts not in FORMATS:
            raise ValueError(f"expert format {experts!r} is not one of {FORMATS}")
        self.moe, self._dims = moe, _dims
        self.H, self.E, self.K, self.F = H, E, K, F
        self.fmt = {k: experts == k for k in ("fp8", "nvfp4", "fp8_b128")}
        self._wss = {}

    def _ws(self, d):
        need = self.moe.workspace_size(d)
        ws = self._wss.get(d.expert_dtype)
        if ws is None or ws.numel() < need:
            ws = self.moe.alloc_workspace(d)
            self._wss[d.expert_dtype] = ws
        return ws

    def route(self, x, w_router, bias):
        T = x.shape[0]
        d = self._dims(T, self.H, self.E, self.K, self.F)
        idx = torch.empty(T, self.K, dtype=torch.int32, device=x.device)
        w = torch.empty(T, self.K, dtype=torch.float32, device=x.device)
        self.moe.route(d, x, w_router, bias, idx, w, self._ws(d))
        return idx, w

    def permute(self, idx):
        T = idx.shape[0]
        d = self._dims(T, self.H, self.E, self.K, self.F)
        dev = idx.device
        counts = torch.empty(self.E, dtype=torch.int32, device=dev)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        perm_src = torch.empty(T * self.K, dtype=torch.int32, device=dev)
        inv_row = torch.empty(T * self.K, dtype=torch.int32, device=dev)
        self.moe.permute(d, idx, counts, offsets, perm_src, inv_row, ws=self._ws(d))
        return counts, offsets, perm_src, inv_row

    def gather(self, x, perm_src, K):
        out = torch.empty(perm_src.shape[0], x.shape[1], dtype=x.dtype, device=x.device)
        if out.shape[0]:
            self.moe.gather_rows(x, perm_src, out, K=K)
        return out

    def regroup(self, recv_counts, R):
        """recv_counts [W, E_loc] int64 on the device -> (offsets, perm, inv) on the device (a kernel)."""
        dev = recv_counts.device
        E_loc = recv_counts.shape[1]
        offsets = torch.empty(E_loc + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(R, dtype=torch.int32, device=dev)
        inv = torch.empty(R, dtype=torch.int32, device=dev)
        self.moe.ep_regroup(recv_counts, offsets, perm, inv)
        return offsets, perm, inv

    def expert_ffn(self, rows, offsets, perm, w_up, w_down, scales=None):
        R, E_loc = rows.shape[0], w_up.shape[0]
        y = torch.empty(R, self.H, dtype=torch.bfloat16, device=rows.device)
        d = self._dims(R, self.H, E_loc, 1, self.F, **self.fmt)
        self.moe.expert_ffn(d, rows, offsets, perm, w_up, w_down, scales, y, self._ws(d))
        return y

    def combine(self, y_perm, inv_row, w, residual, out):
        T = out.shape[0]
        d = self._dims(T, self.H, self.E, self.K, self.F)
        self.moe.combine(d, y_perm, inv_row, w, residual, out)
        return out


def _bytes(t: torch.Tensor) -> torch.Tensor:
    """Rows [rows, n] as raw bytes [rows, n * itemsize] (a view; empty tensors included)."""
    return t.contiguous().view(torch.uint8)


class ExpertParallelLayer:
    """One MoE layer split over the ranks of ``group`` by expert."""

    def __init__(self, H: int, E: int, K: int, F: int, group=None, ops=None, experts: str = "bf16"):
        self.group = group
        self.W = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.W:
            raise ValueError(f"{E} experts do not split evenly over {self.W} ranks")
        self.H, self.E, self.K, self.F = H, E, K, F
        self.E_loc = E // self.W
        self.ops = ops if ops is not None else CudaOps(H, E, K, F, experts)

    def experts(self, rank=None):
        r = self.rank if rank is None else rank
        return range(r * self.E_loc, (r + 1) * self.E_loc)

    def forward(self, x, w_router, bias, w_up_local, w_down_local, out, residual=None, scales=None):
        """x [T, H] (this rank's tokens); w_up_local, w_down_local: this rank's E/W experts in the
        layer's expert format, with ``scales`` (moe_quant_scales of those experts; None for bf16);
        out [T, H].  Returns (topk_idx, topk_w)."""
        ops, W, E_loc, K = self.ops, self.W, self.E_loc, self.K
        idx, w = ops.route(x, w_router, bias)
        counts, offsets, perm_src, inv_row = ops.permute(idx)
        send_rows = ops.gather(x, perm_src, K)                       # expert order = owner order

        send_counts = counts.reshape(W, E_loc).to(torch.int64).contiguous()
        recv_counts = torch.empty_like(send_counts)
        dist.all_to_all_single(recv_counts, send_counts, group=self.group)
        # the split sizes of the row exchange: one device-to-host read per pass
        both = torch.stack([send_counts.sum(1), recv_counts.sum(1)]).cpu()
        sc, rc = both[0].tolist(), both[1].tolist()

        recv_rows = torch.empty(sum(rc), x.shape[1], dtype=x.dtype, device=x.device)
        dist.all_to_all_single(_bytes(recv_rows), _bytes(send_rows), output_split_sizes=rc, input_split_sizes=sc,
                               group=self.group)

        loc_off, perm, inv = ops.regroup(recv_counts, sum(rc))
        y_loc = ops.expert_ffn(recv_rows, loc_off, perm, w_up_local, w_down_local, scales)
        y_back = ops.gather(y_loc, inv, 1)                           # arrival order
        dev = x.device

        y_perm = torch.empty((sum(sc),) + tuple(y_back.shape[1:]), dtype=y_back.dtype, device=dev)
        dist.all_to_all_single(_bytes(y_perm), _bytes(y_back), output_split_sizes=sc, input_split_sizes=rc,
                               group=self.group)
        ops.combine(y_perm, inv_row, w, residual, out)
        return idx, w
