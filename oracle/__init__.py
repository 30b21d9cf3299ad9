"""ORACLE — test infrastructure only.

numpy front end of ``oracle.c``: the plain fp64 CPU statement of the routed
mixture-of-experts layer that the CUDA path is checked against.  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package; the product path never does.  It shares no code with
the CUDA path; the two meet only in the seeded input generators of
``synth``.

bf16 tensors travel as their uint16 bit patterns; everything the oracle
computes is float64 unless the function says otherwise.
"""
from __future__ import annotations

import ctypes
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
_SRC = HERE / "oracle.c"
_LIB = HERE / "liboracle.so"

FX_SHIFT = 40

_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_f = ctypes.c_float


def build(force: bool = False) -> Path:
    if force or (not _LIB.exists()) or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        subprocess.check_call([
            "gcc", "-O3", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
            "-fPIC", "-shared", str(_SRC), "-o", str(_LIB), "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(str(build()))
        sig = {
            "oracle_router_logits_fx": (None, [_i64, _i64, _i64, _p, _p, _p, _p]),
            "oracle_topk": (None, [_i64, _i64, _i64, _p, _p, _p]),
            "oracle_permute": (None, [_i64, _i64, _i64, _p, _p, _p, _p, _p]),
            "oracle_expert_bf16": (None, [_i64, _i64, _p, _p, _p, _p]),
            "oracle_expert_rows_bf16": (ctypes.c_int, [_i64, _i64, _i64, _p, _p, _p, _p, _p, _p]),
            "oracle_combine": (None, [_i64, _i64, _i64, _p, _p, _p, _p]),
            "oracle_shared_expert_bf16": (None, [_i64, _i64, _i64, _p, _p, _p, _p]),
            "oracle_e4m3_encode": (ctypes.c_uint8, [_f]),
            "oracle_e4m3_decode": (_f, [ctypes.c_uint8]),
            "oracle_e4m3_encode_n": (None, [_i64, _p, _p]),
            "oracle_e4m3_decode_n": (None, [_i64, _p, _p]),
            "oracle_quantize_tensor_fp8": (_f, [_i64, _p, _p]),
            "oracle_quantize_act_fp8": (None, [_i64, _p, _f, _p]),
            "oracle_expert_fp8": (None, [_i64, _i64, _p, _f, _p, _f, _p, _f, _f, _p]),
            "oracle_expert_rows_fp8": (ctypes.c_int, [_i64, _i64, _i64, _p, _p, _p, _p, _p, _p,
                                                      _p, _f, _f, _p]),
            "oracle_rmsnorm_bf16": (None, [_i64, _i64, _p, _f, _p]),
            "oracle_round_bf16": (None, [_i64, _p, _p]),
            "oracle_hidden_amax_bf16": (ctypes.c_double, [_i64, _i64, _i64, _p, _p, _p, _p]),
            "oracle_b128_kp": (_i64, [_i64]),
            "oracle_quantize_fp8_b128": (None, [_i64, _i64, _p, _p, _p]),
            "oracle_expert_fp8_b128": (None, [_i64, _i64, _p, _p, _p, _p, _p, _f, _f, _p]),
            "oracle_expert_rows_fp8_b128": (ctypes.c_int, [_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p,
                                                           _f, _f, _p]),
            "oracle_e2m1_encode": (ctypes.c_uint8, [_f]),
            "oracle_e2m1_decode": (_f, [ctypes.c_uint8]),
            "oracle_e2m1_encode_n": (None, [_i64, _p, _p]),
            "oracle_e2m1_decode_n": (None, [_i64, _p, _p]),
            "oracle_nvfp4_tensor_scale": (_f, [_i64, _p]),
            "oracle_quantize_nvfp4": (None, [_i64, _i64, _p, _f, _p, _p]),
            "oracle_dequantize_nvfp4": (None, [_i64, _i64, _p, _p, _f, _p]),
            "oracle_expert_nvfp4": (None, [_i64, _i64, _p, _p, _f, _p, _p, _f, _p, _p, _f, _f, _p]),
            "oracle_expert_rows_nvfp4": (ctypes.c_int, [_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                                                        _p, _f, _f, _p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- routing

def router_logits_fx(x, wr, bias=None) -> np.ndarray:
    """Fixed-point router logits, int64 in units of 2^-40, shape [T, E]."""
    x, px = _c(x, np.uint16)
    wr, pw = _c(wr, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.float32)
    L = np.empty((T, E), dtype=np.int64)
    lib().oracle_router_logits_fx(T, H, E, px, pw, pb, L.ctypes.data)
    return L


def topk(L: np.ndarray, K: int):
    L, pl = _c(L, np.int64)
    T, E = L.shape
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float64)
    lib().oracle_topk(T, E, K, pl, idx.ctypes.data, w.ctypes.data)
    return idx, w


def route(x, wr, bias, K):
    L = router_logits_fx(x, wr, bias)
    idx, w = topk(L, K)
    return L, idx, w


def permute(idx: np.ndarray, E: int):
    idx, pi = _c(idx, np.int32)
    T, K = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm_src = np.empty(T * K, dtype=np.int32)
    inv_row = np.empty(T * K, dtype=np.int32)
    lib().oracle_permute(T, K, E, pi, counts.ctypes.data, offsets.ctypes.data,
                         perm_src.ctypes.data, inv_row.ctypes.data)
    return counts, offsets, perm_src, inv_row


# --------------------------------------------------------------------------- experts

def expert_rows_bf16(xrows, ex, wup, wdown, slot) -> np.ndarray:
    """y[r] = expert_{ex[r]}(xrows[r]) for float64 rows; banks given for a set of experts."""
    xrows, px = _c(xrows, np.float64)
    ex, pe = _c(ex, np.int32)
    wup, pu = _c(wup, np.uint16)
    wdown, pd = _c(wdown, np.uint16)
    slot, ps = _c(slot, np.int32)
    R, H = xrows.shape
    F = wup.shape[1]
    y = np.empty((R, H), dtype=np.float64)
    if lib().oracle_expert_rows_bf16(R, H, F, px, pe, pu, pd, ps, y.ctypes.data) != 0:
        raise ValueError("a routed expert's bank was not supplied")
    return y


def combine(y_tk, w, residual=None) -> np.ndarray:
    y_tk, py = _c(y_tk, np.float64)
    w, pw = _c(w, np.float64)
    T, K, H = y_tk.shape
    pr = None
    if residual is not None:
        residual, pr = _c(residual, np.uint16)
    out = np.empty((T, H), dtype=np.float64)
    lib().oracle_combine(T, K, H, py, pw, pr, out.ctypes.data)
    return out


def shared_expert_bf16(xrows, wup_s, wdown_s) -> np.ndarray:
    """y_s[t] = W_down_s relu(W_up_s x_t)^2 for float64 rows x_t; W_up_s [Fs][H], W_down_s [H][Fs] bf16."""
    xrows, px = _c(xrows, np.float64)
    wup_s, pu = _c(wup_s, np.uint16)
    wdown_s, pd = _c(wdown_s, np.uint16)
    T, H = xrows.shape
    Fs = wup_s.shape[0]
    if wup_s.shape != (Fs, H) or wdown_s.shape != (H, Fs):
        raise ValueError("shared expert weights must be [Fs][H] and [H][Fs]")
    y = np.empty((T, H), dtype=np.float64)
    lib().oracle_shared_expert_bf16(T, H, Fs, px, pu, pd, y.ctypes.data)
    return y


def identity_slot(E: int) -> np.ndarray:
    return np.arange(E, dtype=np.int32)


def moe_layer_bf16(x, wr, bias, wup, wdown, K, tokens=None, slot=None, residual=None, shared=None):
    """The whole layer for the rows ``tokens`` of x (all rows if None).

    Tokens do not interact (no capacity limit), so any subset is exact.
    Returns a dict with logits, idx, w, the per-assignment expert outputs
    y [n, K, H] and out [n, H] (float64, before bf16 rounding).  With
    ``shared = (W_up_s, W_down_s)`` the shared expert's output y_s [n, H]
    is added to out with weight 1 (and returned as y_shared).
    """
    x = np.asarray(x, dtype=np.uint16)
    if tokens is not None:
        x = x[np.asarray(tokens)]
        if residual is not None:
            residual = np.asarray(residual)[np.asarray(tokens)]
    E = wr.shape[0]
    if slot is None:
        slot = identity_slot(E)
    L, idx, w = route(x, wr, bias, K)
    n, H = x.shape
    xr = np.repeat(bf16_to_f64(x), K, axis=0)
    y = expert_rows_bf16(xr, idx.reshape(-1), wup, wdown, slot).reshape(n, K, H)
    out = combine(y, w, residual)
    res = dict(logits=L, idx=idx, w=w, y=y, out=out)
    if shared is not None:
        ys = shared_expert_bf16(bf16_to_f64(x), *shared)
        res["y_shared"] = ys
        res["out"] = out + ys
    return res


# --------------------------------------------------------------------------- FP8

def e4m3_encode(v) -> np.ndarray:
    v, pv = _c(v, np.float32)
    q = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_n(v.size, pv, q.ctypes.data)
    return q


def e4m3_decode(q) -> np.ndarray:
    q, pq = _c(q, np.uint8)
    v = np.empty(q.shape, dtype=np.float32)
    lib().oracle_e4m3_decode_n(q.size, pq, v.ctypes.data)
    return v


def quantize_tensor_fp8(w):
    """Per-tensor E4M3 quantisation of a bf16 tensor: returns (codes, scale)."""
    w, pw = _c(w, np.uint16)
    q = np.empty(w.shape, dtype=np.uint8)
    s = lib().oracle_quantize_tensor_fp8(w.size, pw, q.ctypes.data)
    return q, np.float32(s)


def quantize_bank_fp8(bank):
    """Quantise each expert tensor of a bank [S, rows, cols] with its own scale."""
    q = np.empty(bank.shape, dtype=np.uint8)
    s = np.empty(bank.shape[0], dtype=np.float32)
    for i in range(bank.shape[0]):
        q[i], s[i] = quantize_tensor_fp8(bank[i])
    return q, s


def quantize_act_fp8(x, s: float) -> np.ndarray:
    x, px = _c(x, np.uint16)
    q = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_quantize_act_fp8(x.size, px, np.float32(s), q.ctypes.data)
    return q


def expert_rows_fp8(qx, ex, qup, sup, qdown, sdown, slot, sx, sh) -> np.ndarray:
    qx, px = _c(qx, np.uint8)
    ex, pe = _c(ex, np.int32)
    qup, pu = _c(qup, np.uint8)
    sup, psu = _c(sup, np.float32)
    qdown, pd = _c(qdown, np.uint8)
    sdown, psd = _c(sdown, np.float32)
    slot, ps = _c(slot, np.int32)
    R, H = qx.shape
    F = qup.shape[1]
    y = np.empty((R, H), dtype=np.float64)
    rc = lib().oracle_expert_rows_fp8(R, H, F, px, pe, pu, psu, pd, psd, ps,
                                      np.float32(sx), np.float32(sh), y.ctypes.data)
    if rc != 0:
        raise ValueError("a routed expert's bank was not supplied")
    return y


def moe_layer_fp8(x, wr, bias, qup, sup, qdown, sdown, sx, sh, K, tokens=None, slot=None,
                  residual=None):
    """W8A8 layer: bf16 router on x; experts on e4m3 codes with scalar scales."""
    x = np.asarray(x, dtype=np.uint16)
    if tokens is not None:
        x = x[np.asarray(tokens)]
        if residual is not None:
            residual = np.asarray(residual)[np.asarray(tokens)]
    E = wr.shape[0]
    if slot is None:
        slot = identity_slot(E)
    L, idx, w = route(x, wr, bias, K)
    n, H = x.shape
    qx = quantize_act_fp8(x, sx)
    qxr = np.repeat(qx, K, axis=0)
    y = expert_rows_fp8(qxr, idx.reshape(-1), qup, sup, qdown, sdown, slot, sx, sh).reshape(n, K, H)
    out = combine(y, w, residual)
    return dict(logits=L, idx=idx, w=w, y=y, out=out, qx=qx)


# --------------------------------------------------------------------------- FP8_B128

def b128_kp(K: int) -> int:
    """K padded to whole blocks of 128 (1856 -> 1920)."""
    return int(lib().oracle_b128_kp(K))


def quantize_fp8_b128(w):
    """W [..., rows, K] bf16 bits -> (codes [..., rows, Kp], scales [..., rows, Kp/128] fp32)."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    *lead, rows, K = w.shape
    n = int(np.prod(lead)) if lead else 1
    Kp = b128_kp(K)
    q = np.empty((n * rows, Kp), dtype=np.uint8)
    s = np.empty((n * rows, Kp // 128), dtype=np.float32)
    lib().oracle_quantize_fp8_b128(n * rows, K, w.ctypes.data, q.ctypes.data, s.ctypes.data)
    return q.reshape(*lead, rows, Kp), s.reshape(*lead, rows, Kp // 128)


def scalar_to_fp8_b128(q, s, K: int):
    """Per-tensor E4M3 codes q [..., rows, K] with tensor scales s [...] as FP8_B128: codes padded
    with zeros to Kp, every block scale = the tensor scale."""
    q = np.asarray(q, dtype=np.uint8)
    Kp = b128_kp(K)
    qp = np.zeros(q.shape[:-1] + (Kp,), dtype=np.uint8)
    qp[..., :K] = q
    s = np.asarray(s, dtype=np.float32)
    sb = np.broadcast_to(s.reshape(s.shape + (1, 1)), q.shape[:-1] + (Kp // 128,)).astype(np.float32)
    return qp, np.ascontiguousarray(sb)


def quantize_act_fp8_b128(x, s: float) -> np.ndarray:
    """Static-scale activation codes of x [rows, K], zero-padded to Kp."""
    q = quantize_act_fp8(x, s)
    K = q.shape[-1]
    qp = np.zeros(q.shape[:-1] + (b128_kp(K),), dtype=np.uint8)
    qp[..., :K] = q
    return qp


def expert_rows_fp8_b128(qx, ex, bank_up, bank_down, slot, sx, sh, H: int, F: int) -> np.ndarray:
    """y[r] = W8A8 expert ex[r] with FP8_B128 banks ((codes, scales) for up [n][F][Hp] and down
    [n][H][Fp]) on the zero-padded activation codes qx [R][Hp]."""
    qx, px = _c(qx, np.uint8)
    ex, pe = _c(ex, np.int32)
    qu, pqu = _c(bank_up[0], np.uint8)
    su, psu = _c(bank_up[1], np.float32)
    qd, pqd = _c(bank_down[0], np.uint8)
    sd, psd = _c(bank_down[1], np.float32)
    slot, ps = _c(slot, np.int32)
    R = qx.shape[0]
    if qu.shape[1:] != (F, b128_kp(H)) or qd.shape[1:] != (H, b128_kp(F)) or qx.shape[1] != b128_kp(H):
        raise ValueError("FP8_B128 shapes do not match H and F")
    y = np.empty((R, H), dtype=np.float64)
    if lib().oracle_expert_rows_fp8_b128(R, H, F, px, pe, pqu, psu, pqd, psd, ps, np.float32(sx),
                                         np.float32(sh), y.ctypes.data) != 0:
        raise ValueError("a routed expert's bank was not supplied")
    return y


def moe_layer_fp8_b128(x, wr, bias, bank_up, bank_down, sx, sh, K, H, F, tokens=None, slot=None,
                       residual=None):
    """W8A8 layer with FP8_B128 expert banks: bf16 router on x; x and H quantised with static scales."""
    x = np.asarray(x, dtype=np.uint16)
    if tokens is not None:
        x = x[np.asarray(tokens)]
        if residual is not None:
            residual = np.asarray(residual)[np.asarray(tokens)]
    E = wr.shape[0]
    if slot is None:
        slot = identity_slot(E)
    L, idx, w = route(x, wr, bias, K)
    n = x.shape[0]
    qx = quantize_act_fp8_b128(x, sx)
    y = expert_rows_fp8_b128(np.repeat(qx, K, axis=0), idx.reshape(-1), bank_up, bank_down, slot, sx, sh,
                             H, F).reshape(n, K, H)
    out = combine(y, w, residual)
    return dict(logits=L, idx=idx, w=w, y=y, out=out, qx=qx)


# --------------------------------------------------------------------------- NVFP4

def e2m1_encode(v) -> np.ndarray:
    v, pv = _c(v, np.float32)
    q = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e2m1_encode_n(v.size, pv, q.ctypes.data)
    return q


def e2m1_decode(q) -> np.ndarray:
    q, pq = _c(q, np.uint8)
    v = np.empty(q.shape, dtype=np.float32)
    lib().oracle_e2m1_decode_n(q.size, pq, v.ctypes.data)
    return v


def nvfp4_tensor_scale(x) -> np.float32:
    x, px = _c(x, np.uint16)
    return np.float32(lib().oracle_nvfp4_tensor_scale(x.size, px))


def quantize_nvfp4(x, s_t):
    """NVFP4 codes of a bf16 tensor [rows, K] with tensor scale s_t:
    (packed codes [rows, K/2] uint8, block scale codes [rows, K/16] uint8)."""
    x, px = _c(x, np.uint16)
    rows, K = x.shape
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    scales = np.empty((rows, K // 16), dtype=np.uint8)
    lib().oracle_quantize_nvfp4(rows, K, px, np.float32(s_t), codes.ctypes.data, scales.ctypes.data)
    return codes, scales


def dequantize_nvfp4(codes, scales, s_t) -> np.ndarray:
    codes, pc = _c(codes, np.uint8)
    scales, ps = _c(scales, np.uint8)
    rows = codes.shape[0]
    K = codes.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    lib().oracle_dequantize_nvfp4(rows, K, pc, ps, np.float32(s_t), out.ctypes.data)
    return out


def quantize_bank_nvfp4(bank):
    """Each expert tensor of a bank [S, rows, K] with its own tensor scale amax / 2688:
    (codes [S, rows, K/2], block scales [S, rows, K/16], tensor scales [S] fp32)."""
    S, rows, K = bank.shape
    c = np.empty((S, rows, K // 2), dtype=np.uint8)
    sc = np.empty((S, rows, K // 16), dtype=np.uint8)
    t = np.empty(S, dtype=np.float32)
    for i in range(S):
        t[i] = nvfp4_tensor_scale(bank[i])
        c[i], sc[i] = quantize_nvfp4(bank[i], t[i])
    return c, sc, t


def expert_rows_nvfp4(cx, sx, ex, bank_up, bank_down, slot, tx, th) -> np.ndarray:
    """W4A4 experts on NVFP4 rows (cx [R, H/2], sx [R, H/16]); banks from quantize_bank_nvfp4."""
    cx, pcx = _c(cx, np.uint8)
    sx, psx = _c(sx, np.uint8)
    ex, pe = _c(ex, np.int32)
    cu, pcu = _c(bank_up[0], np.uint8)
    su, psu = _c(bank_up[1], np.uint8)
    tu, ptu = _c(bank_up[2], np.float32)
    cd, pcd = _c(bank_down[0], np.uint8)
    sd, psd = _c(bank_down[1], np.uint8)
    td, ptd = _c(bank_down[2], np.float32)
    slot, ps = _c(slot, np.int32)
    R = cx.shape[0]
    H = cx.shape[1] * 2
    F = cu.shape[1]
    y = np.empty((R, H), dtype=np.float64)
    rc = lib().oracle_expert_rows_nvfp4(R, H, F, pcx, psx, pe, pcu, psu, ptu, pcd, psd, ptd, ps,
                                        np.float32(tx), np.float32(th), y.ctypes.data)
    if rc != 0:
        raise ValueError("a routed expert's bank was not supplied")
    return y


def moe_layer_nvfp4(x, wr, bias, bank_up, bank_down, tx, th, K, tokens=None, slot=None, residual=None):
    """W4A4 layer: bf16 router on x; x and H quantised to NVFP4 with static tensor scales."""
    x = np.asarray(x, dtype=np.uint16)
    if tokens is not None:
        x = x[np.asarray(tokens)]
        if residual is not None:
            residual = np.asarray(residual)[np.asarray(tokens)]
    E = wr.shape[0]
    if slot is None:
        slot = identity_slot(E)
    L, idx, w = route(x, wr, bias, K)
    n, H = x.shape
    cx, sx = quantize_nvfp4(x, tx)
    y = expert_rows_nvfp4(np.repeat(cx, K, axis=0), np.repeat(sx, K, axis=0), idx.reshape(-1), bank_up,
                          bank_down, slot, tx, th).reshape(n, K, H)
    out = combine(y, w, residual)
    return dict(logits=L, idx=idx, w=w, y=y, out=out, cx=cx, sx=sx)


def calibrate_nvfp4(x_cal, wr, bias, wup, K, slot=None):
    """Static NVFP4 activation tensor scales from a calibration batch of the bf16 model:
    amax|x| / 2688 and amax(relu(z)^2) / 2688, both fp32 (6 x 448 = 2688)."""
    x_cal = np.asarray(x_cal, dtype=np.uint16)
    E = wr.shape[0]
    if slot is None:
        slot = identity_slot(E)
    _, idx, _ = route(x_cal, wr, bias, K)
    xf = bf16_to_f64(x_cal)
    ax = np.float32(np.max(np.abs(xf)))
    ah = hidden_amax_bf16(np.repeat(xf, K, axis=0), idx.reshape(-1), wup, slot)
    return np.float32(ax / np.float32(2688.0)), np.float32(np.float32(ah) / np.float32(2688.0))


def rmsnorm_bf16(x, eps: float = 1e-5) -> np.ndarray:
    x, px = _c(x, np.uint16)
    T, H = x.shape
    u = np.empty_like(x)
    lib().oracle_rmsnorm_bf16(T, H, px, np.float32(eps), u.ctypes.data)
    return u


def round_bf16(v) -> np.ndarray:
    v, pv = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_round_bf16(v.size, pv, out.ctypes.data)
    return out


def hidden_amax_bf16(xrows, ex, wup, slot) -> float:
    """Largest ReLU^2 activation of the bf16 model over the given rows (calibration)."""
    xrows, px = _c(xrows, np.float64)
    ex, pe = _c(ex, np.int32)
    wup, pu = _c(wup, np.uint16)
    slot, ps = _c(slot, np.int32)
    R, H = xrows.shape
    F = wup.shape[1]
    a = lib().oracle_hidden_amax_bf16(R, H, F, px, pe, pu, ps)
    if a < 0:
        raise ValueError("a routed expert's bank was not supplied")
    return float(a)


def calibrate_fp8(x_cal, wr, bias, wup, K, slot=None):
    """Static W8A8 activation scales from a calibration batch of the bf16 model:
    x_scale = amax|x| / 448 and h_scale = amax(relu(z)^2) / 448, both fp32."""
    x_cal = np.asarray(x_cal, dtype=np.uint16)
    E = wr.shape[0]
    if slot is None:
        slot = identity_slot(E)
    _, idx, _ = route(x_cal, wr, bias, K)
    xf = bf16_to_f64(x_cal)
    ax = np.float32(np.max(np.abs(xf)))
    ah = hidden_amax_bf16(np.repeat(xf, K, axis=0), idx.reshape(-1), wup, slot)
    return np.float32(ax / np.float32(448.0)), np.float32(np.float32(ah) / np.float32(448.0))
