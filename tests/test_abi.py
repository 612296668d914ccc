"""The C-ABI library loads, exports every entry point include/moe.h declares, and rejects bad
arguments on the host.  CPU only: no compute call is made."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.load_builder().build()
    import mixture_experts_layer_48_b200 as m
    return m


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("moe_create", "moe_destroy", "moe_route", "moe_forward", "moe_set_path",
                 "moe_workspace_bytes", "moe_sync_status", "moe_status_string", "moe_tune",
                 "moe_forward_mxfp4", "moe_workspace_bytes_mxfp4", "moe_route_static",
                 "moe_set_dispatch", "moe_get_dispatch"):
        assert name in syms


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(moe_\w+)$", out, flags=re.M))
    declared = set(declared_symbols())
    assert declared <= exported, f"missing: {sorted(declared - exported)}"
    assert set(lib.EXPORTED) == declared, "binding and header disagree"
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name)


def test_status_strings(lib):
    for s in range(7):
        assert lib.moe_status_string(s).decode() not in ("", "unknown status")
    assert lib.moe_status_string(99).decode() == "unknown status"
    names = [lib.moe_profile_kind_name(i).decode() for i in range(lib.MOE_PROFILE_KINDS)]
    assert names == ["router", "route_finalize", "gather", "gate_up_stream", "down_stream",
                     "to_f16", "gate_up_tile", "down_tile", "gate_up_gemm", "down_gemm"]
    assert lib.moe_profile_kind_name(-1).decode() == "unknown"
    assert lib.moe_profile_kind_name(lib.MOE_PROFILE_KINDS).decode() == "unknown"


@pytest.mark.parametrize("E,H,I,k", [
    (0, 256, 256, 1), (257, 256, 256, 4), (8, 256, 256, 0), (8, 256, 256, 9),
    (8, 2880 + 32, 2880, 4), (8, 2880, 100, 4), (8, 0, 256, 2), (8, 32768, 256, 2),
])
def test_create_rejects_bad_shapes(lib, E, H, I, k):
    h = ctypes.c_void_p()
    assert lib.moe_create(E, H, I, k, ctypes.byref(h)) == lib.MOE_ERR_ARG
    assert not h.value


def test_create_null_out(lib):
    assert lib.moe_create(8, 256, 256, 2, None) == lib.MOE_ERR_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU answer")
def test_create_without_gpu_reports_device(lib):
    h = ctypes.c_void_p()
    assert lib.moe_create(32, 2880, 2880, 4, ctypes.byref(h)) == lib.MOE_ERR_DEVICE
    with pytest.raises(lib.MoeError) as ei:
        lib.Moe(32, 2880, 2880, 4)
    assert ei.value.status == lib.MOE_ERR_DEVICE


def test_null_handle_calls(lib):
    assert lib.moe_destroy(None) == lib.MOE_OK
    assert lib.moe_workspace_bytes(None, 16) == 0
    assert lib.moe_route_workspace_bytes(None, 16) == 0
    assert lib.moe_launch_count(None) == 0
    assert lib.moe_forward(None, 1, None, None, None, None, None, None, None, 0, None) == lib.MOE_ERR_ARG
    assert lib.moe_route(None, 1, None, None, None, None, None, None, None, None, None, 0, None) == lib.MOE_ERR_ARG
    assert lib.moe_set_path(None, 0, -1) == lib.MOE_ERR_ARG
    assert lib.moe_set_dispatch(None, 16, 256, 0) == lib.MOE_ERR_ARG
    assert lib.moe_get_dispatch(None, None, None, None) == lib.MOE_ERR_ARG
    assert lib.moe_sync_status(None, None) == lib.MOE_ERR_ARG
    assert lib.moe_profile_begin(None, 4) == lib.MOE_ERR_ARG
    assert lib.moe_selftest_timeout(None, 10, None) == lib.MOE_ERR_ARG
    assert lib.moe_workspace_bytes_mxfp4(None, 16) == 0
    assert lib.moe_forward_mxfp4(None, 1, None, None, None, None, None, None, None, None, None,
                                 0, None) == lib.MOE_ERR_ARG


def test_no_closed_copy_calls_in_sources():
    # the batched memcpy family is closed on the test machines; none of the sources may name it
    pat = re.compile("cu" + "(da)?Memcpy(3D)?Batch" + "Async")
    for d, _, files in os.walk(os.path.join(ROOT, "mixture_experts_layer_48_b200")):
        for f in files:
            if f.endswith((".cu", ".cuh", ".h", ".py")):
                assert not pat.search(open(os.path.join(d, f)).read()), f
