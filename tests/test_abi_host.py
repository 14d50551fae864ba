"""The C-ABI library loads, exports every entry point its header declares,
and rejects bad arguments on the host (no GPU needed, no compute calls)."""
import ctypes
import os
import re

import pytest

import moe_decode_block_b200 as mdb
from moe_decode_block_b200 import build as mbuild
from moe_decode_block_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_decode.h")


@pytest.fixture(scope="module")
def lib():
    mbuild.build_library()
    return mdb.load_library()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert sorted(header_functions()) == sorted(mdb.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a_only(lib):
    # the build flags name exactly one target: sm_100a
    flags = " ".join(mbuild.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def test_error_strings(lib):
    for code in range(0, -9, -1):
        s = lib.moe_decode_error_string(code).decode()
        assert s and s != "unknown error code"
    assert lib.moe_decode_error_string(-99).decode() == "unknown error code"


def _shapes(**kw):
    s = synth.FULL
    d = dict(hidden=s.hidden, n_experts=s.n_experts, top_k=s.top_k, inter=s.inter,
             shared_inter=s.shared_inter, n_shared=1, max_batch=64, router_bias=None, flags=0)
    d.update(kw)
    return mdb.Shapes(**d)


def test_workspace_bytes_and_shape_validation(lib):
    full = lib.moe_decode_workspace_bytes(ctypes.byref(_shapes()))
    assert 10 << 20 < full < 64 << 20
    tiny = lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(hidden=256, n_experts=16, top_k=2, inter=128,
                                                                shared_inter=128, max_batch=1)))
    assert 0 < tiny < full
    bad = [dict(hidden=7170), dict(hidden=0), dict(n_experts=12), dict(n_experts=2048), dict(top_k=0),
           dict(top_k=33), dict(top_k=9, n_experts=8), dict(inter=100), dict(n_shared=2),
           dict(shared_inter=12), dict(max_batch=0), dict(max_batch=65), dict(flags=32), dict(flags=33), dict(flags=1 << 31),
           dict(flags=8, hidden=7168 + 64), dict(flags=8, inter=2048 + 64), dict(flags=8 | 2)]
    for kw in bad:
        sh = _shapes(**kw)
        assert lib.moe_decode_workspace_bytes(ctypes.byref(sh)) == 0, kw
        h = ctypes.c_void_p()
        assert lib.moe_decode_init(ctypes.byref(sh), ctypes.byref(h)) == mdb.MOE_ERR_UNSUPPORTED_SHAPE, kw
        assert not h.value
    # the two-stream plan flag is accepted and needs the same workspace
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(flags=mdb.MOE_FLAG_TWO_STREAM))) == full
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(flags=mdb.MOE_FLAG_TCGEN05))) == full
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(flags=3))) == full
    # e4m3 expert weights: whole 128 x 128 scale blocks, not with tcgen05
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(flags=mdb.MOE_FLAG_FP8_WEIGHTS))) == full
    # the testing-only hold flag is accepted too (the handle's first forward
    # withholds one panel publication)
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(flags=mdb.MOE_FLAG_TEST_HOLD_PANEL))) == full
    # partial sums (one tensor-parallel rank's share) need no other workspace
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(flags=mdb.MOE_FLAG_PARTIAL_SUM))) == full
    # shared_inter is ignored when there is no shared expert
    assert lib.moe_decode_workspace_bytes(ctypes.byref(_shapes(n_shared=0, shared_inter=0))) > 0


def test_null_arguments_are_rejected_on_the_host(lib):
    assert lib.moe_decode_init(None, None) == mdb.MOE_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert lib.moe_decode_init(None, ctypes.byref(h)) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_destroy(None) == mdb.MOE_OK
    assert lib.moe_decode_get_status(None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_get_stats(None, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_forward(None, *([None] * 9), 1, None, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_forward_host(None, *([None] * 9), 1, None, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_set_wait_limit(None, 100) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_forward_fp8(None, *([None] * 13), 1, None, None) == mdb.MOE_ERR_INVALID_ARG
    # the reduce + residual step checks its arguments before touching a device
    buf = ctypes.create_string_buffer(64 + 16)
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    one = (ctypes.c_void_p * 1)(a16)
    assert lib.moe_decode_reduce_residual(None, 1, a16, a16, 1, 8, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_reduce_residual(one, 0, a16, a16, 1, 8, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_reduce_residual(one, mdb.MOE_REDUCE_MAX_PARTS + 1, a16, a16, 1, 8,
                                          None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_reduce_residual(one, 1, a16 + 4, a16, 1, 8, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_reduce_residual(one, 1, a16, a16, 1, 12, None) == mdb.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_reduce_residual(one, 1, a16, a16, 65, 8, None) == mdb.MOE_ERR_INVALID_ARG
    bad = (ctypes.c_void_p * 1)(a16 + 8)
    assert lib.moe_decode_reduce_residual(bad, 1, a16, a16, 1, 8, None) == mdb.MOE_ERR_INVALID_ARG


def test_init_without_a_gpu_reports_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    assert lib.moe_decode_init(ctypes.byref(_shapes()), ctypes.byref(h)) == mdb.MOE_ERR_NO_DEVICE
    assert not h.value
    with pytest.raises(mdb.MoEDecodeError):
        mdb.MoEDecode(256, 16, 2, 128, 128, max_batch=1)


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    monkeypatch.setattr(mdb, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mdb, "_lib", None)
    with pytest.raises(ImportError):
        mdb.load_library()
