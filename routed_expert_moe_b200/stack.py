"""A stack of routed-MoE layers over one residual stream, through the C ABI.

Each layer l applies, to the residual stream x (bf16, [T, H]):
    u = rmsnorm(x)                      (moe_rmsnorm, unit gain)
    x = x + MoE_l(u)                    (moe_forward with residual = x)
with the expert banks in bf16 or in E4M3 codes with scalar scales (W8A8).
The normalisation before each layer follows the pre-norm blocks of the hybrid
decoder: the audio.cpp model page ("Q4_K, Q3_K and Q2_K expert profiles")
names a normalisation among the model's steps; without one, a stack of
these layers grows without bound.

Marshalling only: every step runs in the library's kernels.
"""
from __future__ import annotations

import torch

from . import alloc_workspace, dims, forward, fp8_scales, quantize_fp8, rmsnorm


class MoeStack:
    def __init__(self, T, H, E, K, F, fp8=True, eps=1e-5, device="cuda"):
        self.T, self.H, self.E, self.K, self.F = T, H, E, K, F
        self.fp8 = fp8
        self.eps = eps
        self.device = torch.device(device)
        self.layers = []
        self.dims = dims(T, H, E, K, F, fp8=fp8)
        self.ws = alloc_workspace(self.dims, self.device)
        self.u = torch.empty(T, H, dtype=torch.bfloat16, device=self.device)
        self.x = [torch.empty(T, H, dtype=torch.bfloat16, device=self.device) for _ in range(2)]

    def add_layer(self, w_router, w_up, w_down, x_scale=None, h_scale=None, bias=None):
        """w_up [E,F,H], w_down [E,H,F] as bf16 masters; quantised here when the stack is W8A8."""
        layer = {"wr": w_router, "bias": bias}
        if self.fp8:
            cu = torch.empty(w_up.shape, dtype=torch.uint8, device=self.device)
            cd = torch.empty(w_down.shape, dtype=torch.uint8, device=self.device)
            su = torch.empty(self.E, dtype=torch.float32, device=self.device)
            sd = torch.empty(self.E, dtype=torch.float32, device=self.device)
            quantize_fp8(w_up, cu, su)
            quantize_fp8(w_down, cd, sd)
            layer.update(wu=cu, wd=cd, su=su, sd=sd, scales=fp8_scales(su, sd, x_scale, h_scale))
        else:
            layer.update(wu=w_up, wd=w_down, scales=None)
        self.layers.append(layer)
        return layer

    def run_layer(self, l, x_in, x_out, topk_idx=None, topk_w=None):
        L = self.layers[l]
        rmsnorm(x_in, self.u, self.eps)
        forward(self.dims, self.u, L["wr"], L["bias"], L["wu"], L["wd"], x_out, self.ws, scales=L["scales"],
                residual=x_in, topk_idx=topk_idx, topk_w=topk_w)

    def forward(self, x):
        """Run every layer on x (bf16 [T, H]); returns the final residual stream (an internal buffer)."""
        src = x
        for l in range(len(self.layers)):
            dst = self.x[l % 2]
            self.run_layer(l, src, dst)
            src = dst
        return src
