"""Pins of the oracle's shared expert (the bloomery issue page, section 4
"Placement on card, host RAM and NVMe": the model's shared experts stay on
the card beside the routed ones).  Reading: an ungated ReLU^2 FFN of width Fs
that every token passes through, added to the routed sum with weight 1.

The pins: an identity-like shared expert has a closed form; with all routed
experts zero the layer is the shared expert alone; zero shared weights leave
the routed layer bitwise unchanged; a dense torch fp64 statement of the block
agrees; and the hidden dimension splits exactly (ReLU^2 is elementwise), which
is what lets a kernel run a shared expert of width n*F as n experts of width F.
"""
import numpy as np
import torch

import oracle
from synth import workloads as W

TINY = W.WORKLOADS[0]


def to_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
    return (bits >> 16).astype(np.uint16)


def shared_weights(w: W.Workload, Fs: int):
    ws = W.Workload(w.name, w.T, w.H, w.E, w.K, w.F, seed=w.seed + 100, shared=Fs)
    return W.host_w_up_shared(ws), W.host_w_down_shared(ws)


def test_identity_shared_expert_closed_form():
    """W_up_s = c [I | 0], W_down_s = [I ; 0]: y_s[i] = c^2 relu(x_i)^2 for i < Fs, 0 beyond."""
    H, Fs, c = 64, 32, 2.0
    wu = np.zeros((Fs, H), np.float32)
    wu[:, :Fs] = c * np.eye(Fs)
    wd = np.zeros((H, Fs), np.float32)
    wd[:Fs, :] = np.eye(Fs)
    rng = np.random.default_rng(11)
    x = to_bits(np.round(rng.standard_normal((5, H)) * 16) / 16)
    xf = oracle.bf16_to_f64(x)
    ys = oracle.shared_expert_bf16(xf, to_bits(wu), to_bits(wd))
    assert np.array_equal(ys[:, :Fs], c * c * np.maximum(xf[:, :Fs], 0.0) ** 2)
    assert not ys[:, Fs:].any()


def test_layer_with_zero_routed_experts_is_the_shared_expert():
    x, wr = W.host_x(TINY), W.host_router(TINY)
    zu = np.zeros((TINY.E, TINY.F, TINY.H), np.uint16)
    zd = np.zeros((TINY.E, TINY.H, TINY.F), np.uint16)
    su, sd = shared_weights(TINY, 2 * TINY.F)
    r = oracle.moe_layer_bf16(x, wr, None, zu, zd, TINY.K, shared=(su, sd))
    U, D = oracle.bf16_to_f64(su), oracle.bf16_to_f64(sd)
    X = oracle.bf16_to_f64(x)
    ref = (np.maximum(X @ U.T, 0.0) ** 2) @ D.T
    assert np.max(np.abs(r["out"] - ref)) <= 1e-12 * np.max(np.abs(ref))
    res = W.host_x(TINY, tensor=7)
    rr = oracle.moe_layer_bf16(x, wr, None, zu, zd, TINY.K, residual=res, shared=(su, sd))
    assert np.max(np.abs(rr["out"] - (oracle.bf16_to_f64(res) + ref))) <= 1e-12 * np.max(np.abs(ref))


def test_zero_shared_weights_change_nothing():
    x, wr, wu, wd = W.host_x(TINY), W.host_router(TINY), W.host_w_up(TINY), W.host_w_down(TINY)
    base = oracle.moe_layer_bf16(x, wr, None, wu, wd, TINY.K)
    z = oracle.moe_layer_bf16(x, wr, None, wu, wd, TINY.K,
                              shared=(np.zeros((TINY.F, TINY.H), np.uint16), np.zeros((TINY.H, TINY.F), np.uint16)))
    assert np.array_equal(z["out"], base["out"]) and np.array_equal(z["idx"], base["idx"])


def test_dense_torch_fp64_block_with_shared_expert():
    for wl, Fs in ((TINY, TINY.F), (W.Workload("mid", 12, 512, 16, 4, 192, seed=9), 384)):
        x, wr, wu, wd = W.host_x(wl), W.host_router(wl), W.host_w_up(wl), W.host_w_down(wl)
        su, sd = shared_weights(wl, Fs)
        r = oracle.moe_layer_bf16(x, wr, None, wu, wd, wl.K, shared=(su, sd))
        X = torch.from_numpy(oracle.bf16_to_f64(x))
        R = torch.from_numpy(oracle.bf16_to_f64(wr))
        U = torch.from_numpy(oracle.bf16_to_f64(wu))
        D = torch.from_numpy(oracle.bf16_to_f64(wd))
        logits = X @ R.T
        top = torch.topk(logits, wl.K, dim=-1)
        assert np.array_equal(top.indices.numpy(), r["idx"])
        p = torch.softmax(logits, dim=-1)
        gate = torch.zeros_like(p).scatter(1, top.indices, p.gather(1, top.indices))
        gate = gate / gate.sum(1, keepdim=True)
        dense = torch.zeros_like(X)
        for e in range(wl.E):
            dense += gate[:, e:e + 1] * (torch.relu(X @ U[e].T) ** 2 @ D[e].T)
        Us = torch.from_numpy(oracle.bf16_to_f64(su))
        Ds = torch.from_numpy(oracle.bf16_to_f64(sd))
        dense += torch.relu(X @ Us.T) ** 2 @ Ds.T
        ref = dense.numpy()
        assert np.max(np.abs(r["out"] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_hidden_dimension_splits_into_chunks_of_width_F():
    """y_s of width n*F = sum over j of the FFN with rows jF..(j+1)F of W_up_s and the same
    columns of W_down_s."""
    wl = W.Workload("split", 7, 256, 8, 2, 64, seed=13)
    n = 3
    su, sd = shared_weights(wl, n * wl.F)
    X = oracle.bf16_to_f64(W.host_x(wl))
    whole = oracle.shared_expert_bf16(X, su, sd)
    parts = sum(oracle.shared_expert_bf16(X, np.ascontiguousarray(su[j * wl.F:(j + 1) * wl.F]),
                                          np.ascontiguousarray(sd[:, j * wl.F:(j + 1) * wl.F]))
                for j in range(n))
    assert np.max(np.abs(whole - parts)) <= 1e-12 * np.max(np.abs(whole))
