"""Write fp8_b128_scales.json: the static activation scales of the FP8_B128
workloads (decode T=64 and prefill T=4096 shapes: hidden 2688, 128 experts,
top-6, width 1856; the bf16 masters of seeds 1 and 2).

The FP8 release keeps static scalar activation scales next to its
block-scaled weights (bloomery issue page, s.3: FP8_B128; s.2: scalar-scale
W8A8 activations).  They are inputs of the layer, like its weights, and come
from a calibration pass of the oracle over the bf16 model on a seeded
calibration batch of 64 tokens:
    x_scale = amax|x| / 448        h_scale = amax relu(W_up[e] x)^2 / 448
Only ``oracle`` and ``synth`` are used.  Run from the repository root:

    python tests/golden/make_fp8_b128_scales.py
"""
from __future__ import annotations

import json
import struct
import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

N_CAL = 64


def f32_hex(v) -> str:
    return struct.pack(">f", float(np.float32(v))).hex()


def main():
    out = {"_made_by": "python tests/golden/make_fp8_b128_scales.py (oracle + synth only)",
           "_calibration_tokens": N_CAL}
    for cfg in (9, 10):
        w = W.WORKLOADS[cfg]
        x = synth.normal_bf16(synth.key(w.seed, synth.T_CALIB, 0), N_CAL * w.H, W.SIGMA_X).reshape(N_CAL, w.H)
        wr = W.host_router(w)
        _, idx, _ = oracle.route(x, wr, W.host_bias(w), w.K)
        used = sorted(set(idx.reshape(-1).tolist()))
        slot = -np.ones(w.E, np.int32)
        slot[used] = np.arange(len(used))
        tx, th = oracle.calibrate_fp8(x, wr, W.host_bias(w), W.host_w_up(w, experts=used), w.K, slot=slot)
        out[w.name] = {"x_scale": float(tx), "x_scale_f32": f32_hex(tx), "h_scale": float(th),
                       "h_scale_f32": f32_hex(th), "experts_used": len(used), "seed": w.seed}
        print(w.name, out[w.name], flush=True)
    p = Path(__file__).with_name("fp8_b128_scales.json")
    p.write_text(json.dumps(out, indent=1) + "\n")


if __name__ == "__main__":
    main()
