"""Write fp8_chain_scales.json: the static W8A8 activation scales of the
23-layer FP8 chain workload (T=4096, hidden 2688, 128 experts, top-6,
width 1856, seed 4).

The scales are inputs of the layer, like its weights ("scalar-scale E4M3
W8A8", bloomery issue page, s.2).  They come from a calibration pass of the
oracle over the bf16 model on a seeded calibration batch of 64 tokens:
for each layer l, with u = rmsnorm(x_l) the layer's normalised input,
    x_scale[l] = amax|u| / 448
    h_scale[l] = amax relu(W_up[e] u)^2 / 448   over the routed experts e
and then x_{l+1} = bf16(x_l + MoE_l(u)).  Only ``oracle`` and ``synth`` are
used.  Run from the repository root:

    python tests/golden/make_fp8_chain_scales.py
"""
from __future__ import annotations

import json
import struct
import sys
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

EPS = 1e-5
N_CAL = 64


def f32_hex(v) -> str:
    return struct.pack(">f", float(np.float32(v))).hex()


def main():
    w = W.WORKLOADS[4]
    x = synth.normal_bf16(synth.key(w.seed, synth.T_CALIB, 0), N_CAL * w.H, W.SIGMA_X).reshape(N_CAL, w.H)
    layers = []
    for l in range(w.layers):
        t0 = time.time()
        wr = W.host_router(w, l)
        u = oracle.rmsnorm_bf16(x, EPS)
        _, idx, _ = oracle.route(u, wr, None, w.K)
        used = sorted(set(idx.reshape(-1).tolist()))
        slot = -np.ones(w.E, np.int32)
        slot[used] = np.arange(len(used))
        wu = W.host_w_up(w, l, experts=used)
        wd = W.host_w_down(w, l, experts=used)
        uf = oracle.bf16_to_f64(u)
        sx = np.float32(np.float32(np.max(np.abs(uf))) / np.float32(448.0))
        ah = oracle.hidden_amax_bf16(np.repeat(uf, w.K, axis=0), idx.reshape(-1), wu, slot)
        sh = np.float32(np.float32(ah) / np.float32(448.0))
        r = oracle.moe_layer_bf16(u, wr, None, wu, wd, w.K, slot=slot, residual=x)
        x = oracle.round_bf16(r["out"])
        rms = float(np.sqrt(np.mean(oracle.bf16_to_f64(x) ** 2)))
        layers.append({"layer": l, "x_scale": float(sx), "x_scale_f32": f32_hex(sx), "h_scale": float(sh),
                       "h_scale_f32": f32_hex(sh), "experts_used": len(used), "residual_rms_after": rms})
        print(f"layer {l:2d}: x_scale {float(sx):.6g} h_scale {float(sh):.6g} rms {rms:.3f} "
              f"({time.time() - t0:.1f} s)", flush=True)
    out = {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "K": w.K, "F": w.F, "seed": w.seed,
           "calibration_tokens": N_CAL, "rmsnorm_eps": EPS, "layers": layers,
           "made_by": "python tests/golden/make_fp8_chain_scales.py (oracle + synth only)"}
    (Path(__file__).resolve().parent / "fp8_chain_scales.json").write_text(json.dumps(out, indent=1) + "\n")


if __name__ == "__main__":
    main()
