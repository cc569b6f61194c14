"""The C ABI without a GPU: the library loads, exports every function the
public header declares, and its pure-host calls agree with the oracle's
statement of the pool layout.  No compute call is made here."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^LORA_API [^(]*?\b(lora_\w+)\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    import adapter_deltas_b200 as lib
    return lib


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("lora_pool_create", "lora_pool_load", "lora_pool_unload", "lora_pool_destroy",
                 "lora_pool_page_table", "lora_workspace_bytes", "lora_apply", "lora_apply_segments",
                 "lora_shrink", "lora_expand", "lora_get_error"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r" T (lora_\w+)$", out.stdout, flags=re.M))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(L._lib, n)
        assert hasattr(L, n), "binding must expose %s under the same name" % n


def test_header_compiles_as_plain_c(tmp_path):
    c = tmp_path / "t.c"
    c.write_text('#include "lora.h"\nint main(void){return lora_status_string(0)[0] == 0;}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I", os.path.dirname(HEADER), str(c)],
                   check=True)


def test_debug_library_exports_every_declared_symbol():
    # the LORA_DEBUG build (bounds checks in the kernels) has the same boundary
    import importlib.util
    spec = importlib.util.spec_from_file_location("_lora_build", os.path.join(ROOT, "adapter_deltas_b200", "_build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    lib = b.build(debug=True)  # (no-op when it is current)
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True, check=True)
    exported = set(re.findall(r" T (lora_\w+)$", out.stdout, flags=re.M))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing


def test_status_strings(L):
    assert L.lora_status_string(0) == "LORA_OK"
    assert L.lora_status_string(L.LORA_ERR_WORKSPACE) == "LORA_ERR_WORKSPACE"
    assert L.lora_status_string(L.LORA_ERR_BOUNDS) == "LORA_ERR_BOUNDS"
    assert L.lora_status_string(999) == "LORA_ERR_UNKNOWN"


@pytest.mark.parametrize("targets,r_max,page", [
    ([(4096, 4096)] * 128, 16, 1 << 20),
    ([(4096, 11008), (11008, 4096)], 64, 0),
    ([(256, 256)], 8, 4096),
    ([(24, 40)], 5, 0),
])
def test_pool_bytes_required_matches_layout(L, targets, r_max, page):
    _, _, slot = oracle.slot_layout(targets, r_max)
    n = 7
    got = L.lora_pool_bytes_required(targets, r_max, n, page)
    if page == 0:
        assert got == n * ((slot + 255) // 256 * 256)
    else:
        assert got == n * (-(-slot // page)) * page


def test_paged_workload_pool_is_31_25_gib(L):
    got = L.lora_pool_bytes_required([(4096, 4096)] * 128, 16, 1000, 1 << 20)
    assert got == 1000 * 32 * (1 << 20) and got / 2 ** 30 == 31.25


def test_pool_bytes_required_rejects_bad_shapes(L):
    assert L.lora_pool_bytes_required([(4096, 4100)], 16, 4, 0) == 0      # d_out not a multiple of 8
    assert L.lora_pool_bytes_required([(4096, 4096)], 65, 4, 0) == 0      # r_max above 64
    assert L.lora_pool_bytes_required([(4096, 4096)], 16, 4, 3000) == 0   # page not a power of two
    assert L.lora_pool_bytes_required([(4096, 4096)], 16, 0, 0) == 0


def test_workspace_and_plan_layout_need_no_device(L):
    lib = L._lib
    # a NULL pool is rejected before any device work
    assert lib.lora_workspace_bytes(None, 0, 64) == 0
    assert lib.lora_apply(None, 0, None, 0, None, 0, None, None, 4, None, 0, None) == L.LORA_ERR_INVALID_ARG
    assert L.lora_kernel_launches() == 0


def test_layer_and_routed_calls_reject_a_null_pool_without_device_work(L):
    lib = L._lib
    assert lib.lora_linear_workspace_bytes(None, 0, 64) == 0
    assert lib.lora_moe_workspace_bytes(None, 0, 64) == 0
    n0 = L.lora_kernel_launches()
    assert lib.lora_linear(None, 0, None, 0, None, 0, None, 0, None, None, 4, None, 0, None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_linear_expand(None, 0, None, 0, None, 0, None, 0, None, 0, None, None, 4,
                                  None) == L.LORA_ERR_INVALID_ARG
    assert lib.lora_apply_moe(None, 0, None, 0, None, 0, None, None, 4, 2, 8, None, None, 0,
                              None) == L.LORA_ERR_INVALID_ARG
    assert L.lora_kernel_launches() == n0
