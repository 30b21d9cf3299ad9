"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This package holds no arithmetic of the routed mixture-of-experts method.  It
only turns (seed, tensor id, layer) into the activations, weights and router
bias of the workloads.  The definition of the generator is written once in
``synth.c``'s header comment; it is implemented three times (plain C on the
host, CUDA on the device, and a pure-Python loop used as a pin for small
sizes) and the three must agree bit for bit.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
_C_SRC = HERE / "synth.c"
_C_LIB = HERE / "libsynth.so"
_CU_SRC = HERE / "synth_cuda.cu"
_CU_LIB = HERE / "libsynth_cuda.so"

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15

# tensor ids of the key derivation
T_X = 1          # layer input activations [T, H]
T_WR = 2         # router weight [E, H]
T_WUP = 3        # expert up banks [E, F, H]
T_WDOWN = 4      # expert down banks [E, H, F]
T_BIAS = 5       # router-bias expert ranking (Zipf)
T_CALIB = 6      # calibration batch of the FP8 chain
T_XLAYER = 7     # per-layer seeded input of the FP8 chain parity cases
T_WUP_S = 8      # shared expert up weight [Fs, H]
T_WDOWN_S = 9    # shared expert down weight [H, Fs]


def _stale(lib: Path, src: Path) -> bool:
    return (not lib.exists()) or lib.stat().st_mtime < src.stat().st_mtime


def build_host(force: bool = False) -> Path:
    if force or _stale(_C_LIB, _C_SRC):
        subprocess.check_call([
            "gcc", "-O3", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
            "-std=c11", str(_C_SRC), "-o", str(_C_LIB)])
    return _C_LIB


def build_cuda(force: bool = False) -> Path:
    if force or _stale(_CU_LIB, _CU_SRC):
        subprocess.check_call([
            "nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC", "-shared", "-fmad=false", str(_CU_SRC), "-o", str(_CU_LIB)])
    return _CU_LIB


_host = None
_cuda = None


def _h():
    global _host
    if _host is None:
        lib = ctypes.CDLL(str(build_host()))
        lib.synth_key.restype = ctypes.c_uint64
        lib.synth_key.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32]
        lib.synth_u64.restype = ctypes.c_uint64
        lib.synth_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        for name in ("synth_normal_bf16", "synth_normal_f32"):
            f = getattr(lib, name)
            f.restype = None
            f.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float,
                          ctypes.c_void_p]
        _host = lib
    return _host


def _d():
    global _cuda
    if _cuda is None:
        lib = ctypes.CDLL(str(build_cuda()))
        for name in ("synth_normal_bf16_cuda", "synth_normal_f32_cuda"):
            f = getattr(lib, name)
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float,
                          ctypes.c_void_p, ctypes.c_void_p]
        _cuda = lib
    return _cuda


def key(seed: int, tensor_id: int, layer: int = 0) -> int:
    return int(_h().synth_key(seed, tensor_id, layer))


def u64(k: int, i: int) -> int:
    return int(_h().synth_u64(k, i))


def normal_bf16(k: int, n: int, sigma: float, offset: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of n generator draws starting at ``offset``."""
    out = np.empty(n, dtype=np.uint16)
    _h().synth_normal_bf16(k, offset, n, sigma, out.ctypes.data)
    return out


def normal_f32(k: int, n: int, sigma: float, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _h().synth_normal_f32(k, offset, n, sigma, out.ctypes.data)
    return out


def normal_bf16_device(k: int, n: int, sigma: float, out_ptr: int, stream: int = 0,
                       offset: int = 0) -> None:
    """Fill ``n`` bf16 values at device address ``out_ptr`` (same bits as the host)."""
    rc = _d().synth_normal_bf16_cuda(k, offset, n, sigma, out_ptr, stream)
    if rc != 0:
        raise RuntimeError(f"synth_normal_bf16_cuda failed with CUDA error {rc}")


# ---------------------------------------------------------------------------
# Pure-Python restatement of the same definition (pin for small sizes).
# ---------------------------------------------------------------------------

def py_mix64(z: int) -> int:
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def py_sm64(s: int, i: int) -> int:
    return py_mix64((s + (i + 1) * GAMMA) & MASK64)


def py_key(seed: int, tensor_id: int, layer: int = 0) -> int:
    return py_sm64(seed, (tensor_id << 32) | layer)


def py_normal_bf16(k: int, n: int, sigma: float, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    sig = np.float32(sigma)
    for i in range(n):
        j = offset + i
        s = 0
        for a in range(3):
            w = py_sm64(k, 3 * j + a)
            for q in range(4):
                s += (w >> (16 * q)) & 0xFFFF
        z = np.float32(s + 6 - 6 * 65536) / np.float32(65536.0)
        v = np.float32(z * sig)
        out[i] = _bf16_rne(v)
    return out


def _bf16_rne(v: np.float32) -> int:
    u = int(np.array([v], dtype=np.float32).view(np.uint32)[0])
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFFFFFF
    return u >> 16


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (b.astype(np.uint32) << 16).view(np.float32)
