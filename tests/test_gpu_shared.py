"""GPU parity of the MoE block with its shared expert (bloomery issue page,
section 4: the model's shared experts stay on the card).  Reading: an ungated
ReLU^2 FFN of width Fs that every token passes through, added with weight 1.
The library runs it as Fs/F chunks of width F inside the routed grouped GEMMs
and adds the chunks in the combine; the oracle computes it as one FFN of width
Fs.  Indices are compared bit for bit, outputs within BF16_TOL of max|ref|.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

from _gpu import BF16_TOL, dev, dev_bf16, host_f64, inputs, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def with_shared(w: W.Workload, Fs: int) -> W.Workload:
    return W.Workload(w.name + f"_Fs{Fs}", w.T, w.H, w.E, w.K, w.F, seed=w.seed, zipf_bias=w.zipf_bias, shared=Fs)


SMALL = [with_shared(W.WORKLOADS[0], 128), with_shared(W.WORKLOADS[0], 256),
         with_shared(W.Workload("ragged_T37_E16_K4", 37, 512, 16, 4, 192, seed=11), 576),
         with_shared(W.Workload("T1", 1, 2688, 128, 6, 1856, seed=12), 1856),
         with_shared(W.Workload("odd_F_tail_H272_F208", 21, 272, 8, 3, 208, seed=14), 416),
         with_shared(W.Workload("K10_three_chunks", 40, 256, 16, 10, 64, seed=15), 192),
         with_shared(W.Workload("K12_four_chunks", 33, 256, 16, 12, 64, seed=16), 256)]   # K + Fs/F = 16


def run_forward(moe, w, h, su, sd, residual=None):
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, Fs=w.shared)
    ws = moe.alloc_workspace(dims)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    moe.forward(dims, dev_bf16(h["x"]), dev_bf16(h["wr"]), None if h["bias"] is None else dev(h["bias"]),
                h["wu_d"], h["wd_d"], out, ws, residual=None if residual is None else dev_bf16(residual),
                topk_idx=idx, shared=(su, sd))
    moe.check_device_error()
    return out, idx


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_shared_forward_parity_small(moe, w):
    h = inputs(w)
    h["wu_d"], h["wd_d"] = dev_bf16(h["wu"]), dev_bf16(h["wd"])
    su, sd = W.host_w_up_shared(w), W.host_w_down_shared(w)
    res = W.host_x(w, tensor=7) if w.T == 37 else None
    out, idx = run_forward(moe, w, h, dev_bf16(su), dev_bf16(sd), residual=res)
    r = oracle.moe_layer_bf16(h["x"], h["wr"], h["bias"], h["wu"], h["wd"], w.K, residual=res, shared=(su, sd))
    assert np.array_equal(idx.cpu().numpy(), r["idx"])
    assert rel_err(host_f64(out), r["out"]) <= BF16_TOL
    if res is None:   # the shared expert is not negligible here: the check would fail without it
        assert rel_err(r["out"] - r["y_shared"], r["out"]) > 5 * BF16_TOL


@pytest.mark.parametrize("w", [SMALL[1], SMALL[4], SMALL[5]], ids=lambda w: w.name)
def test_shared_down_weight_through_the_fallback_map(moe, w):
    """The plain [H][Fs] map, chunk j from column j*F: a K tail (F = 208) reads the next chunk's
    weights against activation columns that read as zero."""
    h = inputs(w)
    h["wu_d"], h["wd_d"] = dev_bf16(h["wu"]), dev_bf16(h["wd"])
    su, sd = W.host_w_up_shared(w), W.host_w_down_shared(w)
    moe.debug_set(7, 1)
    try:
        out, idx = run_forward(moe, w, h, dev_bf16(su), dev_bf16(sd))
    finally:
        moe.debug_set(7, 0)
    r = oracle.moe_layer_bf16(h["x"], h["wr"], h["bias"], h["wu"], h["wd"], w.K, shared=(su, sd))
    assert np.array_equal(idx.cpu().numpy(), r["idx"])
    assert rel_err(host_f64(out), r["out"]) <= BF16_TOL


def test_expert_ffn_writes_each_shared_chunk_to_its_rows(moe):
    w = with_shared(W.WORKLOADS[0], 3 * 128)
    h = inputs(w)
    su, sd = W.host_w_up_shared(w), W.host_w_down_shared(w)
    _, ridx, _ = oracle.route(h["x"], h["wr"], None, w.K)
    _, offsets, perm_src, _ = oracle.permute(ridx, w.E)
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, Fs=w.shared)
    ws = moe.alloc_workspace(dims)
    ns = w.shared // w.F
    y = torch.empty(w.T * (w.K + ns), w.H, dtype=torch.bfloat16, device="cuda")
    moe.expert_ffn(dims, dev_bf16(h["x"]), dev(offsets), dev(perm_src), dev_bf16(h["wu"]), dev_bf16(h["wd"]),
                   None, y, ws, shared=(dev_bf16(su), dev_bf16(sd)))
    moe.check_device_error()
    got = host_f64(y)
    X = oracle.bf16_to_f64(h["x"])
    routed = oracle.expert_rows_bf16(X[perm_src // w.K], ridx.reshape(-1)[perm_src], h["wu"], h["wd"],
                                     oracle.identity_slot(w.E))
    assert rel_err(got[:w.T * w.K], routed) <= BF16_TOL
    for j in range(ns):
        ref = oracle.shared_expert_bf16(X, np.ascontiguousarray(su[j * w.F:(j + 1) * w.F]),
                                        np.ascontiguousarray(sd[:, j * w.F:(j + 1) * w.F]))
        rows = got[w.T * w.K + j * w.T: w.T * w.K + (j + 1) * w.T]
        assert rel_err(rows, ref) <= BF16_TOL


@pytest.mark.parametrize("cfg", [7, 8])
def test_shared_full_size_sampled_outputs(moe, cfg):
    """Decode (one 64-row tile per chunk) and prefill (16 tiles of 256 rows) with Fs = F."""
    w = W.WORKLOADS[cfg]
    x, wr = W.host_x(w), W.host_router(w)

    def bank(tid, n, shape):
        t = torch.empty(*shape, dtype=torch.bfloat16, device="cuda")
        synth.normal_bf16_device(synth.key(w.seed, tid, 0), n, W.SIGMA_W, t.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
        return t

    h = dict(x=x, wr=wr, bias=None,
             wu_d=bank(synth.T_WUP, w.E * w.F * w.H, (w.E, w.F, w.H)),
             wd_d=bank(synth.T_WDOWN, w.E * w.H * w.F, (w.E, w.H, w.F)))
    su_d = bank(synth.T_WUP_S, w.shared * w.H, (w.shared, w.H))
    sd_d = bank(synth.T_WDOWN_S, w.H * w.shared, (w.H, w.shared))
    out, idx = run_forward(moe, w, h, su_d, sd_d)
    _, ridx, _ = oracle.route(x, wr, None, w.K)
    assert np.array_equal(idx.cpu().numpy(), ridx)
    rng = np.random.default_rng(cfg)
    tok = np.unique(np.concatenate([[0, w.T - 1], rng.choice(w.T, size=min(w.T, 24), replace=False)]))
    used = sorted(set(ridx[tok].reshape(-1).tolist()))
    slot = -np.ones(w.E, np.int32)
    slot[used] = np.arange(len(used))
    r = oracle.moe_layer_bf16(x, wr, None, W.host_w_up(w, experts=used), W.host_w_down(w, experts=used), w.K,
                              tokens=tok, slot=slot, shared=(W.host_w_up_shared(w), W.host_w_down_shared(w)))
    assert rel_err(host_f64(out)[tok], r["out"]) <= BF16_TOL


@pytest.mark.parametrize("w", [SMALL[2], SMALL[4], SMALL[6],
                               with_shared(W.Workload("T300_E32_K6", 300, 512, 32, 6, 192, seed=17), 384)],
                         ids=lambda w: w.name)
def test_shared_one_launch_ffn_equals_two_launches_bitwise(moe, w):
    """The shared expert's chunks are entries of the one-launch FFN's unit list: the layer output
    is the same bit for bit as with the two projections in two launches (T = 300: several tiles
    per chunk)."""
    h = inputs(w)
    wu_d, wd_d = dev_bf16(h["wu"]), dev_bf16(h["wd"])
    su_d, sd_d = dev_bf16(W.host_w_up_shared(w)), dev_bf16(W.host_w_down_shared(w))
    dims = moe.dims(w.T, w.H, w.E, w.K, w.F, Fs=w.shared)
    ws = moe.alloc_workspace(dims)
    x, wr = dev_bf16(h["x"]), dev_bf16(h["wr"])
    bias = None if h["bias"] is None else dev(h["bias"])
    outs = []
    for one in (1, 0):
        moe.debug_set(8, one)
        try:
            out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            moe.forward(dims, x, wr, bias, wu_d, wd_d, out, ws, shared=(su_d, sd_d))
            moe.check_device_error()
            outs.append(out)
        finally:
            moe.debug_set(8, 1)
    assert torch.equal(outs[0], outs[1])
