"""The C-ABI library loads and exports every entry point include/moe.h
declares; host-side validation and size queries behave (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    import __graft_entry__
    __graft_entry__.build()          # builds before the package loads the library
    import block_scaled_fp8_permute_b200 as m
    return m


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = _declared_functions()
    for must in ("moe_transform_weights", "moe_plan", "moe_forward", "moe_workspace_bytes",
                 "moe_get_device_status", "moe_plan_export", "moe_forward_host"):
        assert must in names


def test_library_exports_every_declared_symbol(moe):
    lib = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_constants(moe):
    assert moe.moe_status_string(0) == "MOE_OK"
    assert moe.moe_status_string(6) == "MOE_ERR_BAD_EXPERT_ID"
    assert moe.moe_block_m() == 128


def test_sizes(moe):
    s = moe.shape(4096, 2048, 1024, 32, 4)
    n1, sf1 = moe.moe_transformed_bytes(s, 1)
    n2, sf2 = moe.moe_transformed_bytes(s, 2)
    assert n1 == 32 * 2048 * 2048 // 2 and sf1 == 32 * 2048 * 2048 // 32
    assert n2 == 32 * 2048 * 1024 // 2 and sf2 == 32 * 2048 * 1024 // 32
    R = 4096 * 4
    P_max = (R + 32 * 127 + 127) // 128 * 128
    assert moe.moe_plan_max_rows(s) == P_max
    ws = moe.moe_workspace_bytes(s)
    # at least the permuted rows, the intermediate and the bf16 partials
    assert ws >= P_max * (2048 + 1024 + 2 * 2048)
    assert moe.moe_workspace_bytes_host(s) > ws


@pytest.mark.parametrize("bad", [
    (64, 200, 512, 8, 2),      # H % 128
    (64, 256, 500, 8, 2),      # I % 128
    (64, 256, 512, 0, 2),      # E == 0
    (64, 256, 512, 8, 9),      # topk > E
    (64, 256, 512, 2000, 2),   # E too large
    (-1, 256, 512, 8, 2),      # negative T
])
def test_unsupported_shapes_rejected_without_launch(moe, bad):
    s = moe.shape(*bad)
    assert moe.moe_workspace_bytes(s) == 0
    assert moe.moe_transformed_bytes(s, 1)[0] == 0
    st = moe.lib().moe_plan(ctypes.byref(s), None, None, 0, None)
    assert st == 2


def test_invalid_arguments_rejected_without_launch(moe):
    s = moe.shape(64, 256, 512, 8, 2)
    lib = moe.lib()
    # null workspace
    assert lib.moe_plan(ctypes.byref(s), 16, None, 1 << 30, None) == 1
    # misaligned workspace
    assert lib.moe_plan(ctypes.byref(s), 16, 4096 + 8, 1 << 30, None) == 1
    # workspace too small
    assert lib.moe_plan(ctypes.byref(s), 16, 4096, 16, None) == 3
    ws = moe.moe_workspace_bytes(s)
    # null / misaligned forward operands
    args = [ctypes.byref(s), None, 256, 256, 256, 256, 256, 256, 256, 256, 4096, ws, None]
    assert lib.moe_forward(*args) == 1
    args[1] = 256 + 3
    assert lib.moe_forward(*args) == 1
    args[1] = 256
    args[5] = 256 + 16          # transformed weights need 256-byte alignment
    assert lib.moe_forward(*args) == 1
    # requant test hook: bad column count
    assert lib.moe_debug_requant(256, 4, 33, 256, 256, None) == 2


def test_pipelined_host_call_sizes_and_validation(moe):
    """Two staging slots after the regular workspace; every argument error is
    reported before anything is enqueued (these calls need no GPU)."""
    s = moe.shape(64, 256, 512, 8, 2)
    lib = moe.lib()
    one, two = moe.moe_workspace_bytes_host(s), moe.moe_workspace_bytes_host_pipelined(s)
    regular = moe.moe_workspace_bytes(s)
    assert two - one == one - regular > 0
    assert moe.moe_workspace_bytes_host_pipelined(moe.shape(64, 200, 512, 8, 2)) == 0
    vpa = ctypes.c_void_p * 2
    good, null = vpa(256, 256), vpa(256, None)
    w = [256] * 4

    def call(n, xs=good, ys=good, ws=4096, ws_bytes=two, shp=s):
        return lib.moe_forward_host_pipelined(ctypes.byref(shp), n, xs, good, good, good, *w,
                                              ys, ws, ws_bytes, None)
    assert call(-1) == 1                       # negative batch count
    assert call(2, ws=None) == 1               # null workspace
    assert call(2, ws=4096 + 64) == 1          # misaligned workspace
    assert call(2, ws_bytes=one) == 3          # room for one staging slot only
    assert call(2, xs=null) == 1               # a null host pointer in a list
    assert call(2, ys=null) == 1
    assert lib.moe_forward_host_pipelined(ctypes.byref(s), 2, None, good, good, good, *w, good,
                                          4096, two, None) == 1
    assert call(0) == 0                        # no batches: nothing to do
    assert call(2, shp=moe.shape(0, 256, 512, 8, 2),
                ws_bytes=moe.moe_workspace_bytes_host_pipelined(moe.shape(0, 256, 512, 8, 2))) == 0
    assert call(2, shp=moe.shape(64, 256, 500, 8, 2)) == 2


def test_zero_tokens_is_a_no_op(moe):
    s = moe.shape(0, 256, 512, 8, 2)
    ws = moe.moe_workspace_bytes(s)
    assert ws > 0
    # forward with T == 0 returns before touching the device
    st = moe.lib().moe_forward(ctypes.byref(s), None, None, None, None, 256, 256, 256, 256, None,
                               4096, ws, None)
    assert st == 0


def test_gemm_sizes_and_validation(moe):
    lib = moe.lib()
    assert moe.moe_gemm_b_bytes(2, 256, 512) == (2 * 256 * 512 // 2, 2 * 256 * 512 // 32)
    assert moe.moe_gemm_b_bytes(1, 100, 512)[0] == 0          # N % 128
    ws = moe.moe_gemm_workspace_bytes(1, 300, 256, 512)
    # at least A's scale chunks: 3 m-tiles x 4 K-blocks x 512 bytes
    assert ws >= 3 * 4 * 512
    assert moe.moe_gemm_workspace_bytes(1, 300, 256, 500) == 0  # K % 128
    assert moe.moe_gemm_workspace_bytes(0, 128, 256, 512) == 0  # no group
    ok = [256, 256, 256, 256, 256]                              # a, a_sf, b_t, b_sf_t, d
    # unsupported shapes
    assert lib.moe_gemm_fp8_fp4(300, 200, 512, *ok, 4096, ws, None) == 2
    assert lib.moe_gemm_fp8_fp4_masked(2, 100, 256, 512, 256, 256, 256, 256, 256, 256,
                                       4096, ws, None) == 2   # M_max % 128
    # masked form without counts
    assert lib.moe_gemm_fp8_fp4_masked(2, 128, 256, 512, 256, 256, None, 256, 256, 256,
                                       4096, ws, None) == 1
    # workspace: null, misaligned, too small
    assert lib.moe_gemm_fp8_fp4(300, 256, 512, *ok, None, ws, None) == 1
    assert lib.moe_gemm_fp8_fp4(300, 256, 512, *ok, 4096 + 64, ws, None) == 1
    assert lib.moe_gemm_fp8_fp4(300, 256, 512, *ok, 4096, 16, None) == 3
    # operands: null / misaligned A, B not 256-byte aligned
    assert lib.moe_gemm_fp8_fp4(300, 256, 512, None, 256, 256, 256, 256, 4096, ws, None) == 1
    assert lib.moe_gemm_fp8_fp4(300, 256, 512, 256 + 4, 256, 256, 256, 256, 4096, ws, None) == 1
    assert lib.moe_gemm_fp8_fp4(300, 256, 512, 256, 256, 256 + 16, 256, 256, 4096, ws, None) == 1
    # no rows: nothing to do
    ws0 = moe.moe_gemm_workspace_bytes(1, 0, 256, 512)
    assert lib.moe_gemm_fp8_fp4(0, 256, 512, None, None, None, None, None, 4096, ws0, None) == 0


def test_product_path_never_touches_the_oracle():
    """The library package and its CUDA sources name nothing under oracle/."""
    pkg = os.path.join(ROOT, "block_scaled_fp8_permute_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"\boracle\b", src), f


def test_binding_fails_loudly_without_the_library(tmp_path):
    """No CPU fallback: importing the binding where libmoe.so is absent raises."""
    import importlib.util
    import shutil
    pkg = tmp_path / "moe_pkg_copy"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "block_scaled_fp8_permute_b200", "__init__.py"),
                pkg / "__init__.py")
    spec = importlib.util.spec_from_file_location("moe_pkg_copy", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
