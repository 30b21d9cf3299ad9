"""routed_expert_moe_b200 — Python binding of the sm_100a routed-MoE library.

Argument marshalling only: every step of the layer runs in the CUDA kernels
of ``libmoe_b200.so`` (built in-tree by ``routed_expert_moe_b200.build``).
Tensors are torch CUDA tensors (bf16 as ``torch.bfloat16``, E4M3 codes as
``torch.uint8``); the stream is torch's current stream unless one is given.
There is no CPU fallback: importing the package fails if the library is
missing, and every call raises ``MoeError`` on a non-OK status.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_LIB_PATH = Path(__file__).resolve().parent / "_lib" / "libmoe_b200.so"

MOE_OK, MOE_EINVAL, MOE_EUNSUPPORTED, MOE_ECUDA, MOE_ETIMEOUT, MOE_EWORKSPACE, MOE_ERANGE, MOE_EINDEX = range(8)
MOE_BF16, MOE_FP8_E4M3, MOE_NVFP4, MOE_FP8_B128 = 0, 1, 2, 3

if not _LIB_PATH.exists():
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python routed_expert_moe_b200/build.py` "
        "(the routed-MoE layer has no CPU implementation)")

_lib = ctypes.CDLL(str(_LIB_PATH))


class MoeDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("F", ctypes.c_int32), ("expert_dtype", ctypes.c_int32),
                ("Fs", ctypes.c_int32)]


class MoeFp8Scales(ctypes.Structure):
    """moe_quant_scales: tensor scales (both formats) and the NVFP4 block-scale banks."""
    _fields_ = [("w_up_scale", ctypes.c_void_p), ("w_down_scale", ctypes.c_void_p),
                ("x_scale", ctypes.c_float), ("h_scale", ctypes.c_float),
                ("w_up_block", ctypes.c_void_p), ("w_down_block", ctypes.c_void_p)]


_P = ctypes.c_void_p
_S = ctypes.c_size_t
_DIMS = ctypes.POINTER(MoeDims)
_SIG = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_abi_version": (ctypes.c_int, []),
    "moe_workspace_size": (ctypes.c_int, [_DIMS, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_forward_launches": (ctypes.c_int, [_DIMS, ctypes.POINTER(ctypes.c_int32)]),
    "moe_route": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_route_static": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P]),
    "moe_permute": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_expert_ffn": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(MoeFp8Scales), _P,
                                      _P, _S, _P]),
    "moe_combine": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(MoeFp8Scales), _P, _P,
                                   _P, _P, _P, _S, _P]),
    "moe_gather_rows": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                       _P, _P]),
    "moe_ep_regroup": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, _P, _P, _P, _P, _P]),
    "moe_quantize_fp8": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, _P, _P, _P, _P]),
    "moe_quantize_nvfp4": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _P, _P, _P, _P, _P]),
    "moe_quantize_fp8_b128": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _P, _P, _P, _P]),
    "moe_rmsnorm": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int32, ctypes.c_float, _P, _P, _P]),
    "moe_quantize_act_fp8": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int32, ctypes.c_float, _P, _P, _P]),
    "moe_quantize_act_nvfp4": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int32, ctypes.c_float, _P, _P, _P, _P]),
    "moe_check_device_error": (ctypes.c_int, [_P]),
    "moe_set_stage_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]),
    "moe_debug_set": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int64]),
}
for _name, (_res, _args) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

_ABI = 3   # the struct layouts and signatures above
if _lib.moe_abi_version() != _ABI:
    raise ImportError(f"libmoe_b200 ABI {_lib.moe_abi_version()} does not match this binding ({_ABI}); rebuild")

# every symbol include/moe.h declares (checked by the ABI test)
EXPORTS = tuple(_SIG)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(s: int) -> str:
    return _lib.moe_status_string(s).decode()


def abi_version() -> int:
    return _lib.moe_abi_version()


def _check(s: int, where: str):
    if s != MOE_OK:
        raise MoeError(s, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def dims(T, H, E, K, F, fp8=False, nvfp4=False, Fs=0, fp8_b128=False) -> MoeDims:
    """Problem size; Fs is the width of the shared expert (0: none, else a multiple of F)."""
    dt = MOE_NVFP4 if nvfp4 else MOE_FP8_B128 if fp8_b128 else (MOE_FP8_E4M3 if fp8 else MOE_BF16)
    return MoeDims(int(T), int(H), int(E), int(K), int(F), dt, int(Fs))


def workspace_size(d: MoeDims) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_workspace_size(ctypes.byref(d), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def forward_launches(d: MoeDims) -> int:
    """Kernels one forward() with these dims launches (host only)."""
    n = ctypes.c_int32(0)
    _check(_lib.moe_forward_launches(ctypes.byref(d), ctypes.byref(n)), "moe_forward_launches")
    return n.value


def alloc_workspace(d: MoeDims, device=None):
    import torch
    return torch.empty(max(workspace_size(d), 256), dtype=torch.uint8, device=device or "cuda")


def fp8_scales(w_up_scale, w_down_scale, x_scale: float, h_scale: float) -> MoeFp8Scales:
    return MoeFp8Scales(w_up_scale.data_ptr(), w_down_scale.data_ptr(), float(x_scale), float(h_scale), None, None)


def nvfp4_scales(w_up_tscale, w_down_tscale, x_scale: float, h_scale: float, w_up_block, w_down_block) -> MoeFp8Scales:
    """Tensor scales [E] (fp32), static activation tensor scales, block-scale banks (uint8)."""
    return MoeFp8Scales(w_up_tscale.data_ptr(), w_down_tscale.data_ptr(), float(x_scale), float(h_scale),
                        w_up_block.data_ptr(), w_down_block.data_ptr())


def nvfp4_scale_row(K: int) -> int:
    """Bytes of one block-scale row: K/16 rounded up to a multiple of 16."""
    return (K // 16 + 15) // 16 * 16


def b128_kp(K: int) -> int:
    """K padded to whole blocks of 128 (the FP8_B128 banks' row length)."""
    return (K + 127) // 128 * 128


def quantize_fp8_b128(src, codes, scales, stream=None):
    """FP8_B128 quantisation of a bank src [n, rows, K] (bf16): codes [n, rows, b128_kp(K)] (uint8),
    scales [n, rows, b128_kp(K) / 128] (fp32)."""
    n, rows, K = src.shape
    _check(_lib.moe_quantize_fp8_b128(n, rows, K, _ptr(src), _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_quantize_fp8_b128")


def quantize_nvfp4(src, codes, block, tscale, stream=None):
    """NVFP4 quantisation of a bank src [n, rows, K] (bf16): codes [n, rows, K/2], block scales
    [n, rows, nvfp4_scale_row(K)], tensor scales [n]."""
    n, rows, K = src.shape
    _check(_lib.moe_quantize_nvfp4(n, rows, K, _ptr(src), _ptr(codes), _ptr(block), _ptr(tscale), _stream(stream)),
           "moe_quantize_nvfp4")


def route(d, x, w_router, bias, topk_idx, topk_w, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(d), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(topk_idx), _ptr(topk_w),
                          _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_route")


def route_static(d, x, w_router, bias, topk_idx, topk_w, stream=None):
    """The router with its scratch in the library's fixed device array (no workspace)."""
    _check(_lib.moe_route_static(ctypes.byref(d), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(topk_idx),
                                 _ptr(topk_w), _stream(stream)), "moe_route_static")


def permute(d, topk_idx, counts, offsets, perm_src, inv_row, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_permute(ctypes.byref(d), _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(perm_src),
                            _ptr(inv_row), _ptr(ws), nbytes, _stream(stream)), "moe_permute")


def expert_ffn(d, x, offsets, perm_src, w_up, w_down, scales, y_perm, ws, stream=None, shared=None):
    """shared = (w_up_shared [Fs, H], w_down_shared [H, Fs]) when d.Fs > 0; y_perm then has
    T*K + T*Fs/F rows."""
    sp = ctypes.byref(scales) if scales is not None else None
    su, sd = shared if shared is not None else (None, None)
    _check(_lib.moe_expert_ffn(ctypes.byref(d), _ptr(x), _ptr(offsets), _ptr(perm_src), _ptr(w_up),
                               _ptr(w_down), _ptr(su), _ptr(sd), sp, _ptr(y_perm), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "moe_expert_ffn")


def combine(d, y_perm, inv_row, topk_w, residual, out, stream=None):
    _check(_lib.moe_combine(ctypes.byref(d), _ptr(y_perm), _ptr(inv_row), _ptr(topk_w), _ptr(residual),
                            _ptr(out), _stream(stream)), "moe_combine")


def forward(d, x, w_router, bias, w_up, w_down, out, ws, scales=None, residual=None, topk_idx=None,
            topk_w=None, stream=None, shared=None):
    """The whole layer; shared = (w_up_shared [Fs, H], w_down_shared [H, Fs]) when d.Fs > 0."""
    sp = ctypes.byref(scales) if scales is not None else None
    su, sd = shared if shared is not None else (None, None)
    _check(_lib.moe_forward(ctypes.byref(d), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_up), _ptr(w_down),
                            _ptr(su), _ptr(sd), sp, _ptr(residual), _ptr(out), _ptr(topk_idx), _ptr(topk_w),
                            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_forward")


def gather_rows(x, perm_src, out, K=1, stream=None):
    """out[r] = x[perm_src[r] // K] for the rows of out (bf16 rows of x [src_rows, H])."""
    rows, H = out.shape[0], x.shape[1]
    _check(_lib.moe_gather_rows(rows, x.shape[0], H, int(K), _ptr(x), _ptr(perm_src), _ptr(out), _stream(stream)),
           "moe_gather_rows")


def ep_regroup(recv_counts, offsets, perm, inv, stream=None):
    """Grouped layout of the rows an expert's owner received: recv_counts [W, E_loc] int64 (device),
    offsets [E_loc + 1], perm [R], inv [R] int32 out (R = recv_counts.sum())."""
    W, E_loc = recv_counts.shape
    _check(_lib.moe_ep_regroup(int(W), int(E_loc), perm.numel(), _ptr(recv_counts), _ptr(offsets), _ptr(perm),
                               _ptr(inv), _stream(stream)), "moe_ep_regroup")


def quantize_fp8(src, codes, scales, stream=None):
    """Per-tensor E4M3 quantisation of src [n, ...] (bf16) into codes (uint8) and scales [n]."""
    n = src.shape[0]
    per = src.numel() // max(n, 1)
    _check(_lib.moe_quantize_fp8(n, per, _ptr(src), _ptr(codes), _ptr(scales), _stream(stream)),
           "moe_quantize_fp8")


def quantize_act_fp8(x, codes, x_scale, stream=None):
    """E4M3 codes of x [rows, H] (bf16) with the static scale x_scale: e4m3(fl32(x / x_scale))."""
    rows, H = x.shape
    _check(_lib.moe_quantize_act_fp8(rows, H, float(x_scale), _ptr(x), _ptr(codes), _stream(stream)),
           "moe_quantize_act_fp8")


def quantize_act_nvfp4(x, codes, block, x_scale, stream=None):
    """NVFP4 codes [rows, H/2] and block scales [rows, nvfp4_scale_row(H)] of x [rows, H] (bf16)."""
    rows, H = x.shape
    _check(_lib.moe_quantize_act_nvfp4(rows, H, float(x_scale), _ptr(x), _ptr(codes), _ptr(block), _stream(stream)),
           "moe_quantize_act_nvfp4")


def rmsnorm(x, u, eps=1e-5, stream=None):
    T, H = x.shape
    _check(_lib.moe_rmsnorm(T, H, float(eps), _ptr(x), _ptr(u), _stream(stream)), "moe_rmsnorm")


def check_device_error(stream=None):
    _check(_lib.moe_check_device_error(_stream(stream)), "moe_check_device_error")


def check_device_error_status(stream=None) -> int:
    return _lib.moe_check_device_error(_stream(stream))


STAGE_EVENTS = 8
STAGES = ("router_logits", "router_topk", "permute", "gather", "up_gemm", "down_gemm", "combine")


def set_stage_events(events):
    """events: a list of STAGE_EVENTS torch.cuda.Event(enable_timing=True), or None to stop."""
    if not events:
        _check(_lib.moe_set_stage_events(None, 0), "moe_set_stage_events")
        return
    for e in events:
        if not e.cuda_event:      # torch creates the CUDA event on its first record
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(_lib.moe_set_stage_events(arr, len(events)), "moe_set_stage_events")


def debug_set(what: int, value: int):
    _check(_lib.moe_debug_set(int(what), int(value)), "moe_debug_set")


def raw_library():
    """The ctypes handle (for tests of the C ABI itself)."""
    return _lib
