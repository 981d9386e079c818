"""GPU test of moe_forward_noalloc, the forward for callers that cannot allocate.

Some users of this library run inside a host application that owns every byte
of device memory through its own pool, or in a loop where a cudaMalloc would
stall the device; they cannot hand the layer a workspace. moe_forward_noalloc
serves them from a static device array inside the library. This test calls it
through the C ABI, twice in a row, and checks each result against the regular
workspace-based moe_forward on the same inputs, within the output tolerance
the parity tests use. The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_ffn_expert_b200.binding import load_library
from mixture_experts_ffn_expert_b200.inputs import WORKLOADS, make_layer_inputs
from mixture_experts_ffn_expert_b200.layer import MoELayer

from parity import check_output, to64

pytestmark = pytest.mark.gpu


def _ptrs(inp):
    return [inp[k].data_ptr() if inp[k] is not None else None
            for k in ("x", "W_g", "W1", "W3", "W2", "W1s", "W3s", "W2s")]


def test_noalloc_forward_matches_workspace_forward_twice():
    shape = WORKLOADS["decode_t128_d2048_f512_e512k10_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, bias=inp["bias"], device="cuda")
    ref = layer(inp["x"]).clone()                    # regular entry point, caller workspace
    torch.cuda.synchronize()
    lib = load_library()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(inp["x"], float("nan"))
        rc = lib.moe_forward_noalloc(layer.plan.handle, shape.T, *_ptrs(inp), out.data_ptr(),
                                     stream)
        assert rc == 0, (call, lib.moe_last_error())
        torch.cuda.synchronize()
        check_output(to64(out), to64(ref))
    assert layer.device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    shape = WORKLOADS["decode_t128_d2048_f512_e512k10_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, bias=inp["bias"], device="cuda")
    lib = load_library()
    out = torch.empty_like(inp["x"])
    big_T = 1 << 20                       # far beyond what 32 MiB of scratch can hold
    rc = lib.moe_forward_noalloc(layer.plan.handle, big_T, *_ptrs(inp), out.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == 3
    assert b"static scratch" in lib.moe_last_error()
    torch.cuda.synchronize()
