"""The C ABI without a GPU: the library loads, exports every function the
header declares, and its host-side validation answers before any device
call (no compute is attempted here)."""
import ctypes
import re
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "moe.h"


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(moe_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def moe():
    import routed_expert_moe_b200 as m
    return m


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
                     "moe_workspace_size", "moe_check_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(moe):
    lib = moe.raw_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", str(moe._LIB_PATH)], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(moe_\w+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported
    assert set(moe.EXPORTS) == set(declared_functions())


def test_status_strings_and_version(moe):
    assert moe.abi_version() == 3   # moe_dims.Fs and the shared-expert weights of moe_expert_ffn / moe_forward
    for s in range(8):
        assert moe.status_string(s).startswith("MOE_")
    assert "unknown" in moe.status_string(99)


def bad(moe, **kw):
    base = dict(T=64, H=2688, E=128, K=6, F=1856)
    base.update(kw)
    return moe.dims(**base)


@pytest.mark.parametrize("kw", [dict(K=0), dict(K=17), dict(E=0), dict(E=257), dict(K=9, E=8),
                                dict(H=2690), dict(F=8), dict(H=0), dict(T=-1),
                                dict(T=2 ** 29, K=6)])
def test_invalid_dims_are_rejected_on_the_host(moe, kw):
    d = bad(moe, **kw)
    n = ctypes.c_size_t()
    assert moe.raw_library().moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == moe.MOE_EINVAL
    assert moe.raw_library().moe_forward(ctypes.byref(d), *([None] * 13), 0, None) == moe.MOE_EINVAL


def test_workspace_size_scales_with_tokens(moe):
    small = moe.workspace_size(moe.dims(64, 2688, 128, 6, 1856))
    big = moe.workspace_size(moe.dims(4096, 2688, 128, 6, 1856))
    assert 0 < small < big
    # X_perm, H and Y_perm of 24576 rows in bf16 dominate
    assert big >= 24576 * (2688 * 2 * 2 + 1856 * 2)
    fp8 = moe.workspace_size(moe.dims(4096, 2688, 128, 6, 1856, fp8=True))
    assert fp8 < big


def test_null_and_missing_arguments(moe):
    lib = moe.raw_library()
    d = bad(moe)
    assert lib.moe_workspace_size(ctypes.byref(d), None) == moe.MOE_EINVAL
    assert lib.moe_workspace_size(None, None) == moe.MOE_EINVAL
    assert lib.moe_route(ctypes.byref(d), None, None, None, None, None, None, 0, None) == moe.MOE_EINVAL
    assert lib.moe_permute(ctypes.byref(d), None, None, None, None, None, None, 0, None) == moe.MOE_EINVAL
    fp8 = moe.dims(64, 2688, 128, 6, 1856, fp8=True)
    assert lib.moe_expert_ffn(ctypes.byref(fp8), *([None] * 10), 0, None) == moe.MOE_EINVAL
    assert lib.moe_rmsnorm(4, 2690, 1e-5, None, None, None) == moe.MOE_EINVAL
    assert lib.moe_quantize_fp8(-1, 4, None, None, None, None) == moe.MOE_EINVAL
    assert lib.moe_debug_set(99, 0) == moe.MOE_EINVAL
    assert lib.moe_debug_set(9, 0) == moe.MOE_OK       # router L2 prefetch off
    assert lib.moe_debug_set(9, -1) == moe.MOE_OK      # its default
    assert lib.moe_gather_rows(-1, 4, 256, 1, None, None, None, None) == moe.MOE_EINVAL
    assert lib.moe_gather_rows(4, 4, 260, 1, None, None, None, None) == moe.MOE_EINVAL   # H % 8
    assert lib.moe_gather_rows(4, 4, 256, 0, None, None, None, None) == moe.MOE_EINVAL   # K < 1
    assert lib.moe_gather_rows(4, 4, 256, 1, None, None, None, None) == moe.MOE_EINVAL   # null buffers
    assert lib.moe_gather_rows(0, 0, 256, 1, None, None, None, None) == moe.MOE_OK
    assert lib.moe_quantize_fp8_b128(1, 4, 8, None, None, None, None) == moe.MOE_EINVAL      # K < 16
    assert lib.moe_quantize_fp8_b128(1, 4, 200, None, None, None, None) == moe.MOE_EINVAL    # K % 16
    assert lib.moe_quantize_fp8_b128(1, 4, 256, None, None, None, None) == moe.MOE_EINVAL    # null buffers
    assert lib.moe_quantize_fp8_b128(0, 4, 256, None, None, None, None) == moe.MOE_OK
    n = ctypes.c_size_t()
    b128 = moe.dims(64, 2688, 128, 6, 1856, fp8_b128=True)
    assert lib.moe_workspace_size(ctypes.byref(b128), ctypes.byref(n)) == moe.MOE_OK
    b128s = moe.dims(64, 2688, 128, 6, 1856, fp8_b128=True, Fs=1856)
    assert lib.moe_workspace_size(ctypes.byref(b128s), ctypes.byref(n)) == moe.MOE_EUNSUPPORTED
    assert lib.moe_set_stage_events(None, 3) == moe.MOE_EINVAL


def test_quantised_formats_need_their_scales(moe):
    """Every quantised format checks its scales on the host before any launch, even for an
    empty batch, where no other pointer is needed."""
    lib = moe.raw_library()
    fake = ctypes.c_void_p(4096)
    for kw in (dict(fp8=True), dict(fp8_b128=True), dict(nvfp4=True)):
        d = moe.dims(0, 2688, 128, 6, 1856, **kw)
        assert lib.moe_expert_ffn(ctypes.byref(d), *([None] * 7), None, None, None, 0, None) == moe.MOE_EINVAL
        sc = moe.MoeFp8Scales(None, fake, 1.0, 1.0, fake, fake)          # no up-projection scales
        assert lib.moe_expert_ffn(ctypes.byref(d), *([None] * 7), ctypes.byref(sc), None, None, 0,
                                  None) == moe.MOE_EINVAL
        sc = moe.MoeFp8Scales(fake, fake, 1.0, 0.0, fake, fake)          # h_scale must be > 0
        assert lib.moe_expert_ffn(ctypes.byref(d), *([None] * 7), ctypes.byref(sc), None, None, 0,
                                  None) == moe.MOE_EINVAL
        sc = moe.MoeFp8Scales(fake, fake, 1.0, 1.0, fake, fake)
        assert lib.moe_expert_ffn(ctypes.byref(d), *([None] * 7), ctypes.byref(sc), None, None, 0,
                                  None) == moe.MOE_OK
    d = moe.dims(0, 2688, 128, 6, 1856, nvfp4=True)                       # NVFP4 also needs its block scales
    sc = moe.MoeFp8Scales(fake, fake, 1.0, 1.0, None, fake)
    assert lib.moe_expert_ffn(ctypes.byref(d), *([None] * 7), ctypes.byref(sc), None, None, 0,
                              None) == moe.MOE_EINVAL


def test_empty_batch_is_ok_without_a_device(moe):
    lib = moe.raw_library()
    d = bad(moe, T=0)
    assert lib.moe_forward(ctypes.byref(d), *([None] * 13), 0, None) == moe.MOE_OK
    assert lib.moe_rmsnorm(0, 2688, 1e-5, None, None, None) == moe.MOE_OK
    assert lib.moe_quantize_fp8(0, 10, None, None, None, None) == moe.MOE_OK


def test_shared_expert_dims_and_pointers_are_checked_on_the_host(moe):
    lib = moe.raw_library()
    n = ctypes.c_size_t()
    ws = lambda d: lib.moe_workspace_size(ctypes.byref(d), ctypes.byref(n))
    assert ws(bad(moe, Fs=1000)) == moe.MOE_EINVAL                 # not a multiple of F
    assert ws(bad(moe, Fs=-1856)) == moe.MOE_EINVAL
    assert ws(bad(moe, Fs=11 * 1856)) == moe.MOE_EINVAL            # K + Fs/F > 16
    fp8 = moe.dims(64, 2688, 128, 6, 1856, fp8=True, Fs=1856)
    assert ws(fp8) == moe.MOE_EUNSUPPORTED                           # bf16 experts only
    plain = moe.workspace_size(bad(moe))
    shared = moe.workspace_size(bad(moe, Fs=2 * 1856))
    assert shared >= plain + 2 * 64 * (2688 * 2 * 2 + 1856 * 2)     # X, H and Y rows of two chunks
    fake = ctypes.c_void_p(4096)
    d0 = bad(moe, T=0)                                               # no device call before these checks
    assert lib.moe_forward(ctypes.byref(d0), *([None] * 5), fake, None, *([None] * 6), 0, None) == moe.MOE_EINVAL
    ds = bad(moe, T=0, Fs=1856)
    assert lib.moe_forward(ctypes.byref(ds), *([None] * 13), 0, None) == moe.MOE_OK
    ds = bad(moe, Fs=1856)
    assert lib.moe_forward(ctypes.byref(ds), *([None] * 13), 0, None) == moe.MOE_EINVAL
    odd = ctypes.c_void_p(4100)                                      # not 16-byte aligned
    assert lib.moe_forward(ctypes.byref(bad(moe, T=0, Fs=1856)), *([None] * 5), odd, fake,
                           *([None] * 6), 0, None) == moe.MOE_EINVAL


def test_forward_launch_count_follows_the_dispatch(moe):
    """Router: one launch up to 256 tokens (expert-split clusters), two up to 1023 (logits, top-K),
    three from 1024 (the tensor-core router); permutation: one block up to 4096 assignments, else three kernels;
    then the row gather, the expert FFN (both projections in one launch; two with the test hook
    off) and the combine."""
    count = lambda T, **kw: moe.forward_launches(moe.dims(T, 2688, 128, 6, 1856, **kw))
    assert [count(T) for T in (0, 1, 64, 256, 257, 682, 683, 1023, 1024, 4096)] == [0, 5, 5, 5, 6, 6, 8, 8, 9, 9]
    assert count(64, fp8=True) == count(64, nvfp4=True) == count(64, fp8_b128=True) == count(64, Fs=1856) == 5
    try:
        moe.debug_set(8, 0)             # the two projections as two launches
        assert count(64) == 6 and count(4096) == 10 and count(64, nvfp4=True) == count(64, fp8_b128=True) == 6
        assert count(64, Fs=1856) == 6
        moe.debug_set(8, 1)
        moe.debug_set(4, 0)             # never the expert-split clusters
        assert count(64) == 6
        moe.debug_set(5, 2)             # always the hidden-split clusters
        assert count(64) == 5 and count(576) == 5
        moe.debug_set(5, 1)             # always the two kernels
        assert count(4096) == 8
        moe.debug_set(5, 3)             # always the tensor-core router (slices, products, selection)
        assert count(576) == 7 and count(4096) == 9
    finally:
        moe.debug_set(8, 1)
        moe.debug_set(4, -1)
        moe.debug_set(5, 0)
    assert count(64) == 5


def test_package_has_no_cpu_path():
    src = (ROOT / "routed_expert_moe_b200" / "__init__.py").read_text()
    assert "oracle" not in src and "numpy" not in src
    for f in (ROOT / "routed_expert_moe_b200").rglob("*"):
        if f.suffix in (".py", ".cu", ".cuh", ".h"):
            assert "import oracle" not in f.read_text()
