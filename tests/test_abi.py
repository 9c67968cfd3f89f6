"""The C-ABI library builds, loads and exports every entry point that include/moe.h declares.

No compute call is made here (no GPU needed): only calls that must fail on their arguments
before touching the device.
"""
import ctypes
import os
import re

import pytest

import quantized_expert_ffn_02_b200 as qe
from quantized_expert_ffn_02_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qe.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_layer_create", "moe_pack_int4", "moe_route", "moe_forward"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names, "no declarations found"
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert sorted(qe.EXPORTS) == names


def test_status_strings(lib):
    for s in range(7):
        assert qe.status_str(s)
    assert qe.status_str(qe.MOE_ERR_TIMEOUT) == "device-side wait timed out"


def test_argument_errors_need_no_device(lib):
    h = ctypes.c_void_p()
    assert lib.moe_layer_create(None, None, ctypes.byref(h)) == qe.MOE_ERR_INVALID_ARG
    cfg = qe.moe_config(d=256, f=128, n_experts=8, top_k=9, n_shared=0, f_shared=0, max_tokens=4, router=0,
                        routed_scaling_factor=1.0, wkind=0, out_bf16=0)
    w = qe.moe_weights()
    assert lib.moe_layer_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == qe.MOE_ERR_INVALID_ARG
    assert lib.moe_pack_int4(None, 4, 7, None, None, None) == qe.MOE_ERR_INVALID_ARG      # odd cols
    assert lib.moe_pack_int4(None, 0, 8, None, None, None) == qe.MOE_OK                  # nothing to do
    assert lib.moe_forward(None, None, 1, None, None) == qe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host(None, None, 1, None, None) == qe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host_async(None, None, 1, None, None) == qe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(None, None, 1, None, None, None) == qe.MOE_ERR_INVALID_ARG
    assert lib.moe_last_error(None) == qe.MOE_ERR_INVALID_ARG
    lib.moe_layer_destroy(None)
    assert lib.moe_layer_workspace_bytes(None) == 0


def _header_enum_values():
    """name -> value for every `NAME = <int>` inside the header's enums."""
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return {n: int(v) for n, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(\d+)", text)}


def test_binding_constants_match_the_header():
    enums = _header_enum_values()
    for name, value in enums.items():
        if hasattr(qe, name):
            assert getattr(qe, name) == value, name
    # debug items and kernel names of the binding, in the header's numbering
    for item, value in qe.DEBUG_ITEMS.items():
        assert enums["MOE_DEBUG_" + item.upper()] == value
    assert len(qe.KERNELS) == enums["MOE_KERNEL_COUNT"]
    for i, name in enumerate(qe.KERNELS):
        key = "MOE_KERNEL_" + name.upper()
        assert enums[key] == i, key


def test_kernel_names_of_the_library(lib):
    for i, name in enumerate(qe.KERNELS):
        assert qe.moe_kernel_name(i) == name
