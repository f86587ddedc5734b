"""CPU checks of the C-ABI library: it builds for sm_100a, loads without a GPU,
exports every entry point include/moe.h declares, and the product path never
touches the oracle."""
import ctypes
import os
import re

import pytest
import torch

from fp4_block_scaled_route_b200 import build as moe_build
from fp4_block_scaled_route_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def libmoe():
    moe_build.build()
    return moe.lib()


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("moe_create", "moe_forward", "moe_destroy"):
        assert name in syms


def test_library_exports_every_declared_symbol(libmoe):
    for name in declared_symbols():
        assert hasattr(libmoe, name), name
    raw = ctypes.CDLL(moe.LIB_PATH)
    for name in declared_symbols():
        assert getattr(raw, name) is not None


def test_binding_covers_every_declared_symbol():
    assert sorted(moe.SIGNATURES) == declared_symbols()


def test_status_strings(libmoe):
    assert moe.status_string(0) == "ok"
    assert "range" in moe.status_string(moe.MOE_ERR_BAD_ROUTING)


def test_host_argument_checks_without_gpu(libmoe):
    ctx = ctypes.c_void_p()
    assert libmoe.moe_create(100, 128, 8, 2, 0, ctypes.byref(ctx)) == moe.MOE_ERR_UNSUPPORTED
    assert libmoe.moe_create_ex(256, 128, 8, 2, 7, 16, 0, ctypes.byref(ctx)) == moe.MOE_ERR_UNSUPPORTED
    assert libmoe.moe_create_ex(256, 128, 8, 2, 0, 0, 0, ctypes.byref(ctx)) == moe.MOE_ERR_INVALID_ARG
    assert libmoe.moe_create(256, 128, 8, 2, 0, None) == moe.MOE_ERR_INVALID_ARG
    # one past each documented limit: H, I <= 8192, E <= 1024, k <= 32, one shared expert
    for H, I, E, k, nsh in [(8320, 128, 4, 2, 0), (128, 8320, 4, 2, 0), (128, 128, 1025, 2, 0),
                            (128, 128, 64, 33, 0), (128, 128, 4, 2, 2)]:
        st = libmoe.moe_create_ex(H, I, E, k, 0, 16, nsh, ctypes.byref(ctx))
        assert st in (moe.MOE_ERR_UNSUPPORTED, moe.MOE_ERR_INVALID_ARG), (H, I, E, k, nsh, st)
    assert libmoe.moe_forward(None, 1, None, None, None, None, None, None, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert libmoe.moe_pack_mxfp4_scales(None, None, 128, 128, None) == moe.MOE_ERR_INVALID_ARG
    assert libmoe.moe_set_fault_injection(None, 1) == moe.MOE_ERR_INVALID_ARG
    if not torch.cuda.is_available():
        # valid arguments on a machine with no GPU: a CUDA error, no context, no crash
        ctx = ctypes.c_void_p(1)
        assert libmoe.moe_create(256, 128, 8, 2, 0, ctypes.byref(ctx)) == moe.MOE_ERR_CUDA and ctx.value is None
        ctx = ctypes.c_void_p(1)
        assert libmoe.moe_create_ex(256, 128, 8, 2, 1, 16, 1, ctypes.byref(ctx)) == moe.MOE_ERR_CUDA
        assert ctx.value is None


def test_product_path_does_not_use_the_oracle():
    pkg = os.path.join(ROOT, "fp4_block_scaled_route_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, flags=re.M), f
                assert "moe_oracle" not in text and "orc_" not in text, f


def test_sources_are_sm100a_only():
    src = open(os.path.join(ROOT, "fp4_block_scaled_route_b200", "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_every_entry_point_is_documented():
    """Each declaration in include/moe.h has its documentation comment
    (operation, arguments, layout, ownership, errors) right above it."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    decls = list(re.finditer(r"^(moe_status|void|const char\s*\*|int)\s+(moe_\w+)\s*\(", src, flags=re.M))
    assert len(decls) == len(declared_symbols())
    for m in decls:
        assert src[:m.start()].rstrip().endswith("*/"), m.group(2)


def test_declare_packed_scales_arguments():
    """Host-only bookkeeping: argument checks of moe_declare_packed_scales."""
    from fp4_block_scaled_route_b200 import moe
    assert moe.moe_declare_packed_scales(None, 64, 1) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_declare_packed_scales(4096, 0, 1) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_declare_packed_scales(4096, 64, 0) == moe.MOE_ERR_INVALID_ARG   # FP8 has no packed scales
    for fmt in (1, 2, 3):
        assert moe.moe_declare_packed_scales(4096 * (fmt + 1), 512, fmt) == moe.MOE_OK
