"""The C-ABI library loads without a GPU, exports every function that
include/mxq.h declares, and rejects bad arguments on the host with the
documented status before touching CUDA (no call below launches anything)."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_sm_b200 as mxq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxq.h")

OK, NULL, SHAPE, DTYPE, ALIGN, WORKSPACE, CUDA, ARG = range(8)
A = 0x10000          # a 16-byte-aligned fake device address (never dereferenced)

# The argument checks below pass fake addresses: they only run where no GPU
# is visible, so a check that wrongly let a call through could never launch
# a kernel on real memory.
if __import__("torch").cuda.is_available():
    pytest.skip("host-validation tests with fake addresses run without a GPU only",
                allow_module_level=True)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z][a-z0-9_]*)\s*\(", text)) - {"sizeof"})


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for f in ("mxfp8_quantize", "mxfp8_dequantize", "mxfp8_quantize_grouped", "nvfp4_quantize",
              "nvfp4_dequantize", "nvfp4_amax", "mxq_abi_version", "mxq_status_string",
              "mxfp4_quantize", "mxfp4_dequantize", "mxfp4_quantize_grouped", "mx_fake_quantize",
              "nvfp4_quantize_sliced", "nvfp4_amax_sliced"):
        assert f in names


def test_library_exports_every_declared_symbol():
    raw = ctypes.CDLL(mxq.library_path)
    missing = [f for f in declared_functions() if not hasattr(raw, f)]
    assert not missing, missing


def test_bounded_wait_check_validation():
    """The bounded-wait self-check rejects limits outside [1 us, 1 s] and a
    NULL or misaligned result array before any launch."""
    f = mxq.lib.mxq_check_bounded_wait
    fake = ctypes.c_void_p(1 << 20)                  # never dereferenced: rejected first
    assert f(999, fake, None) == 7                   # MXQ_ERR_ARG
    assert f(10**9 + 1, fake, None) == 7
    assert f(-5, fake, None) == 7
    assert f(2_000_000, None, None) == 1             # MXQ_ERR_NULL
    assert f(2_000_000, ctypes.c_void_p((1 << 20) + 4), None) == 4   # MXQ_ERR_ALIGN


def test_version_and_strings():
    assert mxq.lib.mxq_abi_version() == 2
    for s in range(8):
        assert mxq.lib.mxq_status_string(s)
    assert mxq.lib.mxq_status_string(99) == b"unknown status"


def test_size_helpers():
    assert mxq.swizzled_scale_bytes(16384, 224) == 16384 * 224
    assert mxq.swizzled_scale_bytes(130, 7) == 256 * 8
    assert mxq.swizzled_scale_bytes(1, 1) == 128 * 4
    assert mxq.swizzled_scale_bytes(-1, 4) == -1
    assert mxq.nvfp4_workspace_bytes(8192, 8192) >= 4


def test_mxfp8_quantize_validation():
    L = mxq.lib
    assert L.mxfp8_quantize(A, 2, 4, 64, 64, A, A, None, None) == DTYPE
    assert L.mxfp8_quantize(A, 0, 4, 48, 48, A, A, None, None) == SHAPE
    assert L.mxfp8_quantize(A, 0, -1, 64, 64, A, A, None, None) == SHAPE
    assert L.mxfp8_quantize(A, 0, 4, 64, 32, A, A, None, None) == SHAPE
    assert L.mxfp8_quantize(None, 0, 4, 64, 64, A, A, None, None) == NULL
    assert L.mxfp8_quantize(A, 0, 4, 64, 64, None, A, None, None) == NULL
    assert L.mxfp8_quantize(A, 0, 4, 64, 64, A, None, None, None) == NULL
    assert L.mxfp8_quantize(A + 2, 0, 4, 64, 64, A, A, None, None) == ALIGN
    assert L.mxfp8_quantize(A, 0, 4, 64, 68, A, A, None, None) == ALIGN
    assert L.mxfp8_quantize(A, 0, 4, 64, 64, A + 8, A, None, None) == ALIGN
    big = 32 * ((1 << 27) - 3)        # swizzled scales take at most 2^27 - 4 columns
    assert L.mxfp8_quantize(A, 0, 1, big, big, A, A, A, None) == SHAPE
    assert L.mxfp4_quantize(A, 0, 1, big, big, A, A, A, None) == SHAPE
    # empty inputs succeed without touching any pointer
    assert L.mxfp8_quantize(None, 0, 0, 64, 64, None, None, None, None) == OK
    assert L.mxfp8_quantize(None, 1, 5, 0, 0, None, None, None, None) == OK


def test_mxfp8_dequantize_validation():
    L = mxq.lib
    assert L.mxfp8_dequantize(A, A, 4, 64, A, 7, None) == DTYPE
    assert L.mxfp8_dequantize(A, A, 4, 40, A, 0, None) == SHAPE
    assert L.mxfp8_dequantize(None, A, 4, 64, A, 0, None) == NULL
    assert L.mxfp8_dequantize(A, A, 4, 64, None, 0, None) == NULL
    assert L.mxfp8_dequantize(A + 4, A, 4, 64, A, 0, None) == ALIGN
    assert L.mxfp8_dequantize(A, A, 4, 64, A + 2, 1, None) == ALIGN
    assert L.mxfp8_dequantize(None, None, 0, 64, None, 0, None) == OK


def test_mxfp4_validation():
    L = mxq.lib
    assert L.mxfp4_quantize(A, 2, 4, 64, 64, A, A, None, None) == DTYPE
    assert L.mxfp4_quantize(A, 0, 4, 48, 48, A, A, None, None) == SHAPE
    assert L.mxfp4_quantize(A, 0, 4, 64, 32, A, A, None, None) == SHAPE
    assert L.mxfp4_quantize(None, 0, 4, 64, 64, A, A, None, None) == NULL
    assert L.mxfp4_quantize(A, 0, 4, 64, 64, None, A, None, None) == NULL
    assert L.mxfp4_quantize(A + 4, 0, 4, 64, 64, A, A, None, None) == ALIGN
    assert L.mxfp4_quantize(A, 0, 4, 64, 64, A + 8, A, None, None) == ALIGN
    assert L.mxfp4_quantize(None, 0, 0, 64, 64, None, None, None, None) == OK
    assert L.mxfp4_dequantize(A, A, 4, 64, A, 5, None) == DTYPE
    assert L.mxfp4_dequantize(A, A, 4, 80, A, 0, None) == SHAPE
    assert L.mxfp4_dequantize(A, None, 4, 64, A, 0, None) == NULL
    assert L.mxfp4_dequantize(A, A, 4, 64, A + 2, 0, None) == ALIGN
    rows = (ctypes.c_int64 * 2)(4, 0)
    ptrs = (ctypes.c_void_p * 2)(A, None)
    assert L.mxfp4_quantize_grouped_ptrs(0, ptrs, rows, 64, 0, A, A, None) == SHAPE
    assert L.mxfp4_quantize_grouped_ptrs(2, ptrs, rows, 40, 0, A, A, None) == SHAPE
    assert L.mxfp4_quantize_grouped_ptrs(2, ptrs, rows, 64, 0, None, A, None) == NULL


def test_fake_quantize_validation():
    L = mxq.lib
    assert L.mx_fake_quantize(2, A, 0, 4, 64, 64, A, 0, None) == ARG
    assert L.mx_fake_quantize(-1, A, 0, 4, 64, 64, A, 0, None) == ARG
    assert L.mx_fake_quantize(1, A, 3, 4, 64, 64, A, 0, None) == DTYPE
    assert L.mx_fake_quantize(1, A, 0, 4, 64, 64, A, 3, None) == DTYPE
    assert L.mx_fake_quantize(0, A, 0, 4, 40, 40, A, 0, None) == SHAPE
    assert L.mx_fake_quantize(0, A, 0, 4, 64, 32, A, 0, None) == SHAPE
    assert L.mx_fake_quantize(0, None, 0, 4, 64, 64, A, 0, None) == NULL
    assert L.mx_fake_quantize(1, A, 0, 4, 64, 64, None, 1, None) == NULL
    assert L.mx_fake_quantize(1, A + 2, 0, 4, 64, 64, A, 0, None) == ALIGN
    assert L.mx_fake_quantize(1, A, 0, 4, 64, 66, A, 0, None) == ALIGN
    assert L.mx_fake_quantize(1, A, 0, 4, 64, 64, A + 4, 1, None) == ALIGN
    assert L.mx_fake_quantize(0, None, 1, 0, 64, 64, None, 1, None) == OK


def test_grouped_ptrs_validation():
    L = mxq.lib
    ptrs = (ctypes.c_void_p * 3)(A, A, A)
    rows = (ctypes.c_int64 * 3)(4, 0, 2)
    P, R = ctypes.cast(ptrs, ctypes.c_void_p), ctypes.cast(rows, ctypes.c_void_p)
    assert L.mxfp8_quantize_grouped_ptrs(0, P, R, 64, 0, A, A, None) == SHAPE
    assert L.mxfp8_quantize_grouped_ptrs(1025, P, R, 64, 0, A, A, None) == SHAPE
    assert L.mxfp8_quantize_grouped_ptrs(3, P, R, 48, 0, A, A, None) == SHAPE
    assert L.mxfp8_quantize_grouped_ptrs(3, P, R, 64, 5, A, A, None) == DTYPE
    assert L.mxfp8_quantize_grouped_ptrs(3, None, R, 64, 0, A, A, None) == NULL
    assert L.mxfp8_quantize_grouped_ptrs(3, P, R, 64, 0, None, A, None) == NULL
    assert L.mxfp8_quantize_grouped_ptrs(3, P, R, 64, 0, A + 1, A, None) == ALIGN
    bad_rows = (ctypes.c_int64 * 3)(4, -1, 2)
    assert L.mxfp8_quantize_grouped_ptrs(3, P, ctypes.cast(bad_rows, ctypes.c_void_p), 64, 0, A, A,
                                    None) == SHAPE
    mis = (ctypes.c_void_p * 3)(A, A, A + 8)
    assert L.mxfp8_quantize_grouped_ptrs(3, ctypes.cast(mis, ctypes.c_void_p), R, 64, 0, A, A,
                                    None) == ALIGN
    zero_rows = (ctypes.c_int64 * 3)(0, 0, 0)
    assert L.mxfp8_quantize_grouped_ptrs(3, P, ctypes.cast(zero_rows, ctypes.c_void_p), 64, 0, None,
                                    None, None) == OK


def test_grouped_null_pointer_only_matters_for_nonempty_expert():
    L = mxq.lib
    rows = (ctypes.c_int64 * 2)(4, 0)
    ptrs = (ctypes.c_void_p * 2)(None, A)
    assert L.mxfp8_quantize_grouped_ptrs(2, ctypes.cast(ptrs, ctypes.c_void_p),
                                         ctypes.cast(rows, ctypes.c_void_p), 64, 0, A, A,
                                         None) == NULL


def test_grouped_stacked_validation():
    L = mxq.lib
    O = A + 0x100      # fake device row offsets (never read on the host)
    for G in (L.mxfp8_quantize_grouped, L.mxfp4_quantize_grouped):
        assert G(A, 0, 0, O, 64, 64, A, A, None) == SHAPE
        assert G(A, 0, 1025, O, 64, 64, A, A, None) == SHAPE
        assert G(A, 0, 4, O, -1, 64, A, A, None) == SHAPE
        assert G(A, 0, 4, O, 64, 48, A, A, None) == SHAPE
        assert G(A, 6, 4, O, 64, 64, A, A, None) == DTYPE
        assert G(A, 0, 4, None, 64, 64, A, A, None) == NULL
        assert G(A, 0, 4, O + 4, 64, 64, A, A, None) == ALIGN
        assert G(None, 0, 4, O, 64, 64, A, A, None) == NULL
        assert G(A, 0, 4, O, 64, 64, None, A, None) == NULL
        assert G(A, 0, 4, O, 64, 64, A, None, None) == NULL
        assert G(A + 2, 0, 4, O, 64, 64, A, A, None) == ALIGN
        assert G(A, 0, 4, O, 64, 64, A + 8, A, None) == ALIGN
        assert G(None, 0, 4, O, 0, 64, None, None, None) == OK
    for G in (L.mxfp8_quantize_grouped_swizzled, L.mxfp4_quantize_grouped_swizzled):
        assert G(A, 0, 4, O, 64, 64, A, A, None, 4096, None) == NULL
        assert G(A, 0, 4, O, 64, 64, A, A, A, -1, None) == SHAPE
        assert G(A, 0, 4, None, 64, 64, A, A, A, 4096, None) == NULL
        assert G(A, 0, 4, O, 64, 64, A, A, A + 8, 4096, None) == ALIGN
        assert G(A, 0, 4, O, 1, 32 * ((1 << 27) - 3), A, A, A, 1 << 40, None) == SHAPE
        assert G(None, 0, 4, O, 0, 64, None, None, A, 0, None) == OK


def test_swizzle_scales_validation():
    Z = mxq.lib.mxq_swizzle_scales
    assert Z(A, -1, 4, A, None) == SHAPE
    assert Z(A, 4, -1, A, None) == SHAPE
    assert Z(None, 4, 4, A, None) == NULL
    assert Z(A, 4, 4, None, None) == NULL
    assert Z(A, 4, 4, A + 4, None) == ALIGN
    assert Z(A, 4, (1 << 27) - 3, A, None) == SHAPE
    assert Z(A, 4, 1 << 27, A, None) == SHAPE     # 2^25 tiles: the word count would wrap
    assert Z(A, 4, (1 << 27) - 4, A, None) == CUDA  # the widest accepted: validation passes, the launch fails here
    assert Z(None, 0, 4, None, None) == OK
    assert Z(None, 4, 0, None, None) == OK


def test_grouped_swizzled_bound():
    B = mxq.lib.mxq_grouped_swizzled_scale_bytes_max
    assert B(1, 100, 7) == 128 * 8
    assert B(64, 64 * 2048, 224) == (64 * 2048 + 127 * 64) // 128 * 128 * 224
    assert B(3, 1, 4) == 256 * 4           # (1 + 381) // 128 = 2 tiles of rows
    assert B(-1, 4, 4) == -1 and B(1, -4, 4) == -1
    # the bound covers every split of M_total rows into E experts
    import itertools
    for E in (1, 2, 3):
        for rows in itertools.product(range(0, 300, 37), repeat=E):
            need = sum(mxq.swizzled_scale_bytes(r, 5) for r in rows)
            assert need <= B(E, sum(rows), 5)


def test_nvfp4_validation():
    L = mxq.lib
    ws = mxq.nvfp4_workspace_bytes()
    assert L.nvfp4_quantize(A, 0, 4, 64, 64, A, A, A, None, 2, A, ws, None) == ARG
    assert L.nvfp4_quantize(A, 0, 4, 64, 64, A, A, A, A, 1, A, ws, None) == ARG
    assert L.nvfp4_quantize(A, 3, 4, 64, 64, A, A, A, None, 0, A, ws, None) == DTYPE
    assert L.nvfp4_quantize(A, 0, 4, 40, 40, A, A, A, None, 0, A, ws, None) == SHAPE
    assert L.nvfp4_quantize(A, 0, 4, 64, 48, A, A, A, None, 0, A, ws, None) == SHAPE
    assert L.nvfp4_quantize(None, 0, 4, 64, 64, A, A, A, None, 0, A, ws, None) == NULL
    assert L.nvfp4_quantize(A, 0, 4, 64, 64, A, A, None, None, 0, A, ws, None) == NULL
    assert L.nvfp4_quantize(A, 0, 4, 64, 64, A + 4, A, A, None, 0, A, ws, None) == ALIGN
    assert L.nvfp4_quantize(A, 1, 4, 64, 66, A, A, A, None, 0, A, ws, None) == ALIGN
    assert L.nvfp4_quantize(A, 0, 4, 64, 64, A, A, A, None, 0, None, ws, None) == WORKSPACE
    assert L.nvfp4_quantize(A, 0, 4, 64, 64, A, A, A, None, 0, A, ws - 4, None) == WORKSPACE
    assert L.nvfp4_quantize(None, 0, 0, 64, 64, None, None, None, None, 0, None, 0, None) == OK
    assert L.nvfp4_amax(A, 0, 4, 64, 64, None, A, ws, None) == NULL
    assert L.nvfp4_amax(A, 0, 4, 64, 64, A, A, 16, None) == WORKSPACE
    assert L.nvfp4_dequantize(A, A, A, 4, 40, A, 0, None) == SHAPE
    assert L.nvfp4_dequantize(A, A, None, 4, 64, A, 0, None) == NULL
    assert L.nvfp4_dequantize(A, A, A, 4, 64, A + 2, 0, None) == ALIGN
    assert L.nvfp4_dequantize(A, A, A, 4, 64, A, 9, None) == DTYPE


def test_nvfp4_noalloc_validation():
    f = ctypes.CDLL(mxq.library_path).nvfp4_quantize_noalloc
    vp, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32
    f.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, u32, vp]
    f.restype = i32
    assert f(A, 0, 4, 64, 64, A, A, A, None, 2, None) == ARG
    assert f(A, 0, 4, 64, 64, A, A, A, A, 1, None) == ARG
    assert f(A, 0, 4, 40, 40, A, A, A, None, 0, None) == SHAPE
    assert f(None, 0, 4, 64, 64, A, A, A, None, 0, None) == NULL
    assert f(A, 0, 4, 64, 64, A, A, None, None, 0, None) == NULL
    assert f(A, 0, 4, 64, 64, A + 4, A, A, None, 0, None) == ALIGN
    assert f(None, 0, 0, 64, 64, None, None, None, None, 0, None) == OK


def test_nvfp4_sliced_validation():
    L = mxq.lib
    ws = mxq.lib.mxq_nvfp4_sliced_workspace_bytes(3)
    assert ws == 4 * (2048 + 3)
    assert mxq.lib.mxq_nvfp4_sliced_workspace_bytes(0) == 0
    assert mxq.lib.mxq_nvfp4_sliced_workspace_bytes(1025) == 0
    rows = (ctypes.c_int64 * 3)(4, 0, 12)
    bad_sum = (ctypes.c_int64 * 3)(4, 0, 11)
    neg = (ctypes.c_int64 * 3)(20, -4, 0)
    Q = L.nvfp4_quantize_sliced
    assert Q(A, 0, 16, 64, 64, 3, bad_sum, A, A, A, None, 0, A, ws, None) == SHAPE
    assert Q(A, 0, 16, 64, 64, 3, neg, A, A, A, None, 0, A, ws, None) == SHAPE
    assert Q(A, 0, 16, 64, 64, 0, rows, A, A, A, None, 0, A, ws, None) == SHAPE
    assert Q(A, 0, 16, 64, 64, 1025, rows, A, A, A, None, 0, A, ws, None) == SHAPE
    assert Q(A, 0, 16, 64, 64, 3, None, A, A, A, None, 0, A, ws, None) == NULL
    assert Q(A, 0, 16, 72, 72, 3, rows, A, A, A, None, 0, A, ws, None) == SHAPE
    assert Q(A, 0, 16, 64, 64, 3, rows, A, A, None, None, 0, A, ws, None) == NULL
    assert Q(A, 0, 16, 64, 64, 3, rows, A, A, A, None, 0, None, ws, None) == WORKSPACE
    assert Q(A, 0, 16, 64, 64, 3, rows, A, A, A, None, 0, A, ws - 4, None) == WORKSPACE
    assert Q(A, 0, 16, 64, 64, 3, rows, A, A, A, A, 1, None, 0, None) == ARG
    assert Q(A, 0, 16, 64, 64, 3, rows, A, A, A, None, 2, None, 0, None) == ARG
    assert Q(A, 0, 16, 64, 64, 3, rows, A + 8, A, A, None, 0, A, ws, None) == ALIGN
    assert Q(A, 5, 16, 64, 64, 3, rows, A, A, A, None, 0, A, ws, None) == DTYPE
    zero = (ctypes.c_int64 * 2)(0, 0)
    assert Q(None, 0, 0, 64, 64, 2, zero, None, None, None, None, 0, None, 0, None) == OK
    X = L.nvfp4_amax_sliced
    assert X(A, 0, 16, 64, 64, 3, bad_sum, A, A, ws, None) == SHAPE
    assert X(A, 0, 16, 64, 64, 3, rows, None, A, ws, None) == NULL
    assert X(A, 0, 16, 64, 64, 3, rows, A, A, 16, None) == WORKSPACE


def test_python_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        mxq.mxfp8_quantize(torch.zeros(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        mxq.nvfp4_quantize(torch.zeros(4, 64, dtype=torch.bfloat16))


def test_rows_view():
    import torch
    x = torch.zeros(6, 10, 64)
    assert mxq._rows_view(x) == (60, 64, 64)
    assert mxq._rows_view(torch.zeros(8, 96)[:, :64]) == (8, 64, 96)
    assert mxq._rows_view(torch.zeros(4, 1, 96)[:, :, :64]) == (4, 64, 96)
    with pytest.raises(ValueError):
        mxq._rows_view(torch.zeros(4, 6, 96)[:, :, :64].transpose(0, 1))
    with pytest.raises(ValueError):
        mxq._rows_view(torch.zeros(64, 4).t())


def test_c_program_against_header_and_library():
    """tests/c/abi_check.c, built with a C compiler against include/mxq.h
    (C11, warnings as errors) and linked with the library, runs its
    validation checks: the boundary is usable from plain C without Python."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    libdir = os.path.dirname(mxq.library_path)
    out_dir = os.path.join(here, "c", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_check")
    build = subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror",
                            "-I", os.path.join(root, "include"), os.path.join(here, "c", "abi_check.c"),
                            "-L", libdir, "-lmxq", f"-Wl,-rpath,{libdir}", "-o", exe],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "all" in run.stdout and "checks passed" in run.stdout
