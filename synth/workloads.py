"""The seeded workloads of the routed mixture-of-experts layer.

Shapes follow the Nemotron 3.5 Transcribe decoder as the bloomery issue page
states them ("2. Checkpoint facts": hidden width 2688, top-6 routing over 128
experts, ungated ReLU^2 experts of width 1856, 23 MoE layers); the serving
shapes follow the SGLang-Omni cookbook page (64 running requests, 4096-token
chunked prefill).  Activations are ~N(0,1), router and expert weights
~N(0,0.02), all rounded to bf16; the router bias of the skewed workload gives
softmax(b) = Zipf(1.1) over a seeded expert ranking.

Nothing here computes any part of the layer: these are inputs only.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import (T_BIAS, T_WDOWN, T_WDOWN_S, T_WR, T_WUP, T_WUP_S, T_X, key, normal_bf16, u64)

SIGMA_X = 1.0
SIGMA_W = 0.02


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    K: int
    F: int
    seed: int
    zipf_bias: bool = False
    layers: int = 1
    fp8: bool = False
    nvfp4: bool = False
    shared: int = 0          # shared expert width Fs (0: none)
    fp8_b128: bool = False   # E4M3 experts with one scale per 128 values along K

    @property
    def assignments(self) -> int:
        return self.T * self.K


WORKLOADS = {
    0: Workload("tiny_T16_H256_E8_K2_F128", 16, 256, 8, 2, 128, seed=0),
    1: Workload("decode_T64", 64, 2688, 128, 6, 1856, seed=1),
    2: Workload("prefill_T4096", 4096, 2688, 128, 6, 1856, seed=2),
    3: Workload("skewed_zipf_T576", 576, 2688, 128, 6, 1856, seed=3, zipf_bias=True),
    4: Workload("chain23_fp8_T4096", 4096, 2688, 128, 6, 1856, seed=4, layers=23, fp8=True),
    # the NVFP4 (W4A4) release's experts on the decode and prefill shapes (same seeds and bf16 masters)
    5: Workload("decode_nvfp4_T64", 64, 2688, 128, 6, 1856, seed=1, nvfp4=True),
    6: Workload("prefill_nvfp4_T4096", 4096, 2688, 128, 6, 1856, seed=2, nvfp4=True),
    # the MoE block with its shared expert (the pages give no width: one expert of the routed shape)
    7: Workload("decode_shared_T64", 64, 2688, 128, 6, 1856, seed=1, shared=1856),
    8: Workload("prefill_shared_T4096", 4096, 2688, 128, 6, 1856, seed=2, shared=1856),
    # the FP8 release's block-scaled experts (FP8_B128) on the decode and prefill shapes
    9: Workload("decode_fp8_b128_T64", 64, 2688, 128, 6, 1856, seed=1, fp8_b128=True),
    10: Workload("prefill_fp8_b128_T4096", 4096, 2688, 128, 6, 1856, seed=2, fp8_b128=True),
}


def zipf_bias(seed: int, E: int, s: float = 1.1) -> np.ndarray:
    """Router bias b_e = ln(r_e^-s / sum_j j^-s), r_e = pi(e)+1 for a seeded permutation pi.

    softmax(b) is then exactly the Zipf(s) law over the ranking; the bias is an
    input of the layer, computed once on the host in float64 and stored fp32.
    """
    k = key(seed, T_BIAS, 0)
    perm = list(range(E))
    for i in range(E - 1, 0, -1):          # Fisher-Yates, draws from the counter stream
        j = u64(k, i) % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    ranks = np.array(perm, dtype=np.float64) + 1.0
    z = np.sum(np.arange(1, E + 1, dtype=np.float64) ** (-s))
    return (np.log(ranks ** (-s) / z)).astype(np.float32)


def host_x(w: Workload, layer: int = 0, tensor: int = T_X) -> np.ndarray:
    return normal_bf16(key(w.seed, tensor, layer), w.T * w.H, SIGMA_X).reshape(w.T, w.H)


def host_router(w: Workload, layer: int = 0) -> np.ndarray:
    return normal_bf16(key(w.seed, T_WR, layer), w.E * w.H, SIGMA_W).reshape(w.E, w.H)


def host_w_up(w: Workload, layer: int = 0, experts=None) -> np.ndarray:
    """W_up bits, [E, F, H] (or [len(experts), F, H] for a subset)."""
    k = key(w.seed, T_WUP, layer)
    n = w.F * w.H
    if experts is None:
        return normal_bf16(k, w.E * n, SIGMA_W).reshape(w.E, w.F, w.H)
    out = np.empty((len(experts), w.F, w.H), dtype=np.uint16)
    for i, e in enumerate(experts):
        out[i] = normal_bf16(k, n, SIGMA_W, offset=int(e) * n).reshape(w.F, w.H)
    return out


def host_w_down(w: Workload, layer: int = 0, experts=None) -> np.ndarray:
    """W_down bits, [E, H, F] (or a subset)."""
    k = key(w.seed, T_WDOWN, layer)
    n = w.H * w.F
    if experts is None:
        return normal_bf16(k, w.E * n, SIGMA_W).reshape(w.E, w.H, w.F)
    out = np.empty((len(experts), w.H, w.F), dtype=np.uint16)
    for i, e in enumerate(experts):
        out[i] = normal_bf16(k, n, SIGMA_W, offset=int(e) * n).reshape(w.H, w.F)
    return out


def host_w_up_shared(w: Workload, layer: int = 0) -> np.ndarray:
    """Shared expert W_up bits, [Fs, H]."""
    return normal_bf16(key(w.seed, T_WUP_S, layer), w.shared * w.H, SIGMA_W).reshape(w.shared, w.H)


def host_w_down_shared(w: Workload, layer: int = 0) -> np.ndarray:
    """Shared expert W_down bits, [H, Fs]."""
    return normal_bf16(key(w.seed, T_WDOWN_S, layer), w.H * w.shared, SIGMA_W).reshape(w.H, w.shared)


def host_bias(w: Workload):
    return zipf_bias(w.seed, w.E) if w.zipf_bias else None


def chain_scales():
    """Static W8A8 activation scales of the chain workload, per layer (x_scale, h_scale) as fp32.

    Written by tests/golden/make_fp8_chain_scales.py from a calibration pass of the oracle.
    """
    import json
    import struct
    from pathlib import Path
    p = Path(__file__).resolve().parents[1] / "tests" / "golden" / "fp8_chain_scales.json"
    d = json.loads(p.read_text())
    f32 = lambda h: np.float32(struct.unpack(">f", bytes.fromhex(h))[0])
    return [(f32(l["x_scale_f32"]), f32(l["h_scale_f32"])) for l in d["layers"]]


def nvfp4_scales(w: Workload):
    """Static NVFP4 activation tensor scales (x, H) of an NVFP4 workload, as fp32.

    Written by tests/golden/make_nvfp4_scales.py from a calibration pass of the oracle.
    """
    import json
    import struct
    from pathlib import Path
    p = Path(__file__).resolve().parents[1] / "tests" / "golden" / "nvfp4_scales.json"
    d = json.loads(p.read_text())[w.name]
    f32 = lambda h: np.float32(struct.unpack(">f", bytes.fromhex(h))[0])
    return f32(d["x_scale_f32"]), f32(d["h_scale_f32"])


def fp8_b128_scales(w: Workload):
    """Static W8A8 activation scales (x, H) of an FP8_B128 workload, as fp32.
    Written by tests/golden/make_fp8_b128_scales.py from a calibration pass of the oracle.
    """
    import json
    import struct
    from pathlib import Path
    p = Path(__file__).resolve().parents[1] / "tests" / "golden" / "fp8_b128_scales.json"
    d = json.loads(p.read_text())[w.name]
    f32 = lambda h: np.float32(struct.unpack(">f", bytes.fromhex(h))[0])
    return f32(d["x_scale_f32"]), f32(d["h_scale_f32"])
