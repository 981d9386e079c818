"""The C-ABI library builds for sm_100a, loads, exports every declared symbol, and
rejects bad layer shapes on the host. No kernel is launched here (no GPU needed)."""
import ctypes
import os
import re

import pytest

from mixture_experts_ffn_expert_b200 import build as build_mod
from mixture_experts_ffn_expert_b200.binding import EXPORTED_SYMBOLS, MoEError, load_library

HEADER = os.path.join(build_mod.ROOT, "include", "moe_ffn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return load_library()


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a_only():
    # the build passes exactly one target to nvcc: real sm_100a code, no PTX for
    # other architectures
    flags = build_mod.NVCC_FLAGS
    i = flags.index("-gencode")
    assert flags[i + 1] == "arch=compute_100a,code=sm_100a"
    assert flags.count("-gencode") == 1
    assert not any(f.startswith("-arch") for f in flags)


@pytest.mark.parametrize("args", [
    (0, 64, 8, 2, 0, 1), (128, 0, 8, 2, 0, 1), (128, 64, 0, 2, 0, 1),
    (128, 64, 8, 0, 0, 1), (128, 64, 8, 2, -1, 1), (128, 64, 8, 9, 0, 1),
])
def test_plan_rejects_invalid_configuration(lib, args):
    # the budget rules of the cooking-agi page, checked before any CUDA call
    assert not lib.moe_plan_create(*args)
    assert lib.moe_last_status() == 1
    assert b"invalid" in lib.moe_last_error()


@pytest.mark.parametrize("args", [
    (100, 64, 8, 2, 0, 1),        # d not a multiple of 8
    (128, 60, 8, 2, 0, 1),        # f not a multiple of 8
    (128, 64, 2048, 2, 0, 1),     # too many routed experts
    (128, 64, 64, 33, 0, 1),      # top_k above 32
])
def test_plan_rejects_unsupported_shape(lib, args):
    assert not lib.moe_plan_create(*args)
    assert lib.moe_last_status() == 5


def test_status_strings(lib):
    assert lib.moe_strerror(0) == b"ok"
    assert lib.moe_strerror(3) == b"workspace too small"
    assert lib.moe_strerror(99) == b"unknown status"


def test_null_plan_is_rejected(lib):
    assert lib.moe_plan_set_workspace(None, None, 0) == 2
    assert lib.moe_forward(None, 1, *([None] * 10)) == 2
    assert lib.moe_workspace_bytes(None, 10) == 0
    lib.moe_plan_destroy(None)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(MoEError):
        load_library(str(tmp_path / "nope.so"))


def test_valid_plan_without_gpu_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert not lib.moe_plan_create(128, 64, 31, 7, 1, 1)
    assert lib.moe_last_status() == 4


def test_option_ids_match_the_header():
    import mixture_experts_ffn_expert_b200.binding as B
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "moe_ffn.h")).read()
    found = dict(re.findall(r"(MOE_OPTION_[A-Z_]+)\s*=\s*(\d+)", hdr))
    assert found, "no option ids in the header"
    for name, value in found.items():
        assert getattr(B, name) == int(value), name
