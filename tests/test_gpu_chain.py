"""The 23-layer W8A8 chain workload (T=4096, hidden 2688, 128 experts,
top-6, width 1856): per-layer parity at full size.

A layer of the chain is u = rmsnorm(x); x' = x + MoE_l(u) with E4M3 experts
and the calibrated static scales of tests/golden/fp8_chain_scales.json.
Every one of the 23 layers is checked on its own seeded input (never a
value the GPU produced): the norm and the routing bit for bit on all 4096
tokens, the layer's MoE term on sampled tokens within 3e-2, and the chained
output within that tolerance plus one bf16 rounding of the sum.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

from _gpu import FP8_TOL, dev_bf16, host_bits, host_f64, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def device_bank(key, shape):
    t = torch.empty(*shape, dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(key, t.numel(), W.SIGMA_W, t.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return t


@pytest.mark.parametrize("layer", range(23))
def test_chain_layer_parity_full_size(moe, layer):
    """Layer l of the chain, teacher-forced on its own seeded input x_l (4096 tokens).

    - u = rmsnorm(x_l): bit for bit on every token.
    - routing on u: bit for bit on every token.
    - the layer's own term MoE_l(u), run without the residual: within
      max|err| / max|ref| <= 3e-2 (the FP8 W8A8 tolerance) on sampled tokens.
    - the chained output x_l + MoE_l(u), rounded once to bf16: per element within
      3e-2 * max|MoE_l(u)| + 2^-8 * |x_l + MoE_l(u)|, i.e. the same tolerance on the
      layer's term plus one bf16 rounding of the sum (bf16 keeps 8 significant bits,
      so round-to-nearest moves a value by at most 2^-8 of its magnitude).
    """
    from routed_expert_moe_b200.stack import MoeStack
    w = W.WORKLOADS[4]
    sx, sh = W.chain_scales()[layer]
    x = synth.normal_bf16(synth.key(w.seed, synth.T_XLAYER, layer), w.T * w.H, W.SIGMA_X).reshape(w.T, w.H)
    wr = W.host_router(w, layer)

    stack = MoeStack(w.T, w.H, w.E, w.K, w.F, fp8=True)
    L = stack.add_layer(dev_bf16(wr), device_bank(synth.key(w.seed, synth.T_WUP, layer), (w.E, w.F, w.H)),
                        device_bank(synth.key(w.seed, synth.T_WDOWN, layer), (w.E, w.H, w.F)), float(sx), float(sh))
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    stack.run_layer(0, dev_bf16(x), out, topk_idx=idx)
    moe.check_device_error()
    u_gpu = host_bits(stack.u)
    term = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
    moe.forward(stack.dims, stack.u, L["wr"], None, L["wu"], L["wd"], term, stack.ws, scales=L["scales"])
    moe.check_device_error()

    u = oracle.rmsnorm_bf16(x)
    assert np.array_equal(u_gpu, u)
    _, ridx, _ = oracle.route(u, wr, None, w.K)
    assert np.array_equal(idx.cpu().numpy(), ridx)

    rng = np.random.default_rng(100 + layer)
    tok = np.unique(np.concatenate([[0, w.T - 1], rng.choice(w.T, size=4, replace=False)]))
    used = sorted(set(ridx[tok].reshape(-1).tolist()))
    slot = -np.ones(w.E, np.int32)
    slot[used] = np.arange(len(used))
    qu, su = oracle.quantize_bank_fp8(W.host_w_up(w, layer, experts=used))
    qd, sd = oracle.quantize_bank_fp8(W.host_w_down(w, layer, experts=used))
    r = oracle.moe_layer_fp8(u, wr, None, qu, su, qd, sd, sx, sh, w.K, tokens=tok, slot=slot)
    assert np.array_equal(r["idx"], ridx[tok])
    ref_term = r["out"]
    assert rel_err(host_f64(term)[tok], ref_term) <= FP8_TOL

    ref_out = oracle.bf16_to_f64(x)[tok] + ref_term
    bound = FP8_TOL * np.max(np.abs(ref_term)) + 2.0 ** -8 * np.abs(ref_out)
    assert np.all(np.abs(host_f64(out)[tok] - ref_out) <= bound)


def test_stack_runs_every_layer_in_order(moe):
    """Small bf16 stack: running it equals applying its layers one by one (same kernels, same order)."""
    from routed_expert_moe_b200.stack import MoeStack
    w = W.WORKLOADS[0]
    stack = MoeStack(w.T, w.H, w.E, w.K, w.F, fp8=False)
    for l in range(3):
        stack.add_layer(dev_bf16(W.host_router(w, l)), dev_bf16(W.host_w_up(w, l)), dev_bf16(W.host_w_down(w, l)))
    x0 = dev_bf16(W.host_x(w))
    y = stack.forward(x0).clone()
    a = torch.empty_like(x0)
    b = torch.empty_like(x0)
    stack.run_layer(0, x0, a)
    stack.run_layer(1, a, b)
    stack.run_layer(2, b, a)
    torch.cuda.synchronize()
    assert torch.equal(y, a)
