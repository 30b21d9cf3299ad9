"""Pins of the oracle's calibration functions: the static activation scales of
the quantised workloads come from them.

Reading (bloomery issue page, s.2: "FP8 uses scalar-scale E4M3 W8A8", and the
NVFP4 release's W4A4 experts): one static scale per activation tensor, taken
from a calibration pass of the bf16 model,
    x_scale = amax|x| / Q,   h_scale = amax over tokens t and their routed
    experts e of relu(W_up[e] x_t)^2 / Q,
with Q = 448 (the largest E4M3 value) for FP8 and Q = 2688 = 6 * 448 (the
largest E2M1 value times the largest E4M3 block scale) for NVFP4, each
quotient an fp32 division.

Every expected value here is a brute-force numpy statement: the logits as an
fp64 matrix product, the top-K by a full sort with ties to the lower index,
and relu(z)^2 formed explicitly for every (token, routed expert) pair.  A
mistake such as taking the maximum before squaring, squaring without the
ReLU, or taking the maximum over experts the tokens were not routed to fails
one of these tests.
"""
import numpy as np
import pytest

import oracle
from synth import workloads as W


def _route_brute(x_bits, wr_bits, bias, K):
    x = oracle.bf16_to_f64(x_bits)
    wr = oracle.bf16_to_f64(wr_bits)
    L = x @ wr.T
    if bias is not None:
        L = L + np.asarray(bias, np.float64)
    idx = np.empty((L.shape[0], K), np.int64)
    for t in range(L.shape[0]):
        order = sorted(range(L.shape[1]), key=lambda e: (-L[t, e], e))
        # the brute force is only trusted where no two of the K+1 best logits are near ties
        gaps = np.diff(-L[t, order[:K + 1]])
        assert np.all(gaps > 1e-9)
        idx[t] = order[:K]
    return idx


def _hidden_brute(x_bits, idx, wup_bits):
    """relu(W_up[e] x_t)^2 for every token t and each of its routed experts e: [T, K, F]."""
    x = oracle.bf16_to_f64(x_bits)
    wup = oracle.bf16_to_f64(wup_bits)
    T, K = idx.shape
    h = np.empty((T, K, wup.shape[1]))
    for t in range(T):
        for k in range(K):
            z = wup[idx[t, k]] @ x[t]
            h[t, k] = np.maximum(z, 0.0) ** 2
    return h


def _tiny():
    w = W.WORKLOADS[0]
    return w, W.host_x(w), W.host_router(w), W.host_w_up(w)


def _times4(bits):
    """bf16 bits of 4 * v, exactly: the exponent field + 2 (values here are normal or zero)."""
    b = np.asarray(bits, np.uint16)
    return np.where((b & 0x7FFF) == 0, b, b + np.uint16(0x100)).astype(np.uint16)


@pytest.mark.parametrize("scale_up", [False, True])
def test_hidden_amax_is_the_largest_relu_square_over_routed_pairs(scale_up):
    w, x, wr, wu = _tiny()
    if scale_up:
        wu = _times4(wu)   # pre-activations x4, so squaring visibly changes the maximum
    idx = _route_brute(x, wr, None, w.K)
    h = _hidden_brute(x, idx, wu)
    xf = oracle.bf16_to_f64(x)
    got = oracle.hidden_amax_bf16(np.repeat(xf, w.K, axis=0), idx.reshape(-1).astype(np.int32), wu,
                                  oracle.identity_slot(w.E))
    assert got == pytest.approx(float(h.max()), rel=1e-12)
    # the plausible mistakes give other numbers on these inputs
    wf = oracle.bf16_to_f64(wu)
    z_routed = np.stack([[wf[idx[t, k]] @ xf[t] for k in range(w.K)] for t in range(w.T)])
    z_all = np.einsum("efh,th->tef", wf, xf)
    wrong = {"no square": np.maximum(z_routed, 0).max(), "no ReLU": (z_routed ** 2).max(),
             "all experts": (np.maximum(z_all, 0) ** 2).max()}
    for name, v in wrong.items():
        assert abs(v - got) > 1e-3 * got, name


def test_hidden_amax_ignores_experts_no_token_uses():
    w, x, wr, wu = _tiny()
    idx = _route_brute(x, wr, None, w.K)
    unused = sorted(set(range(w.E)) - set(idx.reshape(-1).tolist()))
    xf = oracle.bf16_to_f64(x)
    rows, ex = np.repeat(xf, w.K, axis=0), idx.reshape(-1).astype(np.int32)
    base = oracle.hidden_amax_bf16(rows, ex, wu, oracle.identity_slot(w.E))
    if not unused:
        # route every token away from one expert with a bias, so one bank is unused
        bias = np.zeros(w.E, np.float32)
        bias[w.E - 1] = -1e3
        idx = _route_brute(x, wr, bias, w.K)
        ex = idx.reshape(-1).astype(np.int32)
        base = oracle.hidden_amax_bf16(rows, ex, wu, oracle.identity_slot(w.E))
        unused = [w.E - 1]
    planted = wu.copy()
    planted[unused[0]] = 0x4200   # bf16 32.0 everywhere: a huge activation, were the expert used
    assert oracle.hidden_amax_bf16(rows, ex, planted, oracle.identity_slot(w.E)) == base


@pytest.mark.parametrize("Q,fn", [(448.0, "calibrate_fp8"), (2688.0, "calibrate_nvfp4")])
def test_calibration_scales_are_amax_over_the_format_maximum(Q, fn):
    w, x, wr, wu = _tiny()
    idx = _route_brute(x, wr, None, w.K)
    h = _hidden_brute(x, idx, wu)
    ax = np.float32(np.max(np.abs(oracle.bf16_to_f64(x))))
    want_x = np.float32(ax / np.float32(Q))
    want_h = np.float32(np.float32(h.max()) / np.float32(Q))
    sx, sh = getattr(oracle, fn)(x, wr, None, wu, w.K)
    assert sx.dtype == np.float32 and sh.dtype == np.float32
    assert sx == want_x
    # the hidden maximum is an fp64 sum in a different order: at most one fp32 step apart
    assert abs(int(sh.view(np.int32)) - int(want_h.view(np.int32))) <= 1


def test_calibration_follows_the_router_bias():
    """With a bias that forces every token onto experts {0, 1}, the hidden maximum is the
    maximum over those two experts only."""
    w, x, wr, wu = _tiny()
    bias = np.full(w.E, -1e3, np.float32)
    bias[:2] = 0.0
    idx = _route_brute(x, wr, bias, w.K)
    assert set(idx.reshape(-1).tolist()) == {0, 1}
    h = _hidden_brute(x, idx, wu)
    _, sh = oracle.calibrate_fp8(x, wr, bias, wu, w.K)
    want = np.float32(np.float32(h.max()) / np.float32(448.0))
    assert abs(int(sh.view(np.int32)) - int(want.view(np.int32))) <= 1


def test_stored_chain_scales_are_positive_and_follow_their_definition_at_layer_0():
    """tests/golden/fp8_chain_scales.json, layer 0: x_scale = amax|rmsnorm(x_cal)| / 448 over the
    64-token calibration batch, recomputed here from the synth batch with numpy."""
    import synth
    w = W.WORKLOADS[4]
    scales = W.chain_scales()
    assert len(scales) == w.layers
    assert all(sx > 0 and sh > 0 for sx, sh in scales)
    x = synth.normal_bf16(synth.key(w.seed, synth.T_CALIB, 0), 64 * w.H, W.SIGMA_X).reshape(64, w.H)
    xf = oracle.bf16_to_f64(x)
    u = xf / np.sqrt(np.mean(xf ** 2, axis=1, keepdims=True) + 1e-5)
    ax = np.float32(np.max(np.abs(u)))
    # u is rounded to bf16 before its maximum is taken: within one bf16 step (2^-8 relative)
    assert abs(float(scales[0][0]) * 448.0 - float(ax)) <= 2.0 ** -8 * float(ax) + 1e-6
