"""Helpers of the GPU tests: moving seeded inputs to the device and the
tolerance checks.  Inputs always come from ``synth``; expected values always
come from ``oracle``; nothing here computes a step of the layer."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from synth import workloads as W

BF16_TOL = 1e-2   # max|err| / max|ref| for BF16 outputs
FP8_TOL = 3e-2    # max|err| / max|ref| for FP8 E4M3 W8A8 outputs


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / den if den > 0 else float(np.max(np.abs(got)))


def inputs(w: W.Workload, layer: int = 0):
    """Host bits of x, router, banks and bias of a workload."""
    return dict(x=W.host_x(w, layer), wr=W.host_router(w, layer), wu=W.host_w_up(w, layer),
                wd=W.host_w_down(w, layer), bias=W.host_bias(w))


def device_inputs(h):
    d = dict(x=dev_bf16(h["x"]), wr=dev_bf16(h["wr"]), wu=dev_bf16(h["wu"]), wd=dev_bf16(h["wd"]))
    d["bias"] = dev(h["bias"]) if h["bias"] is not None else None
    return d
