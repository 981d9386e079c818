"""GPU tests of moe_forward_noalloc, the forward for callers that cannot allocate.

Some users of this library run inside a host application that owns every byte
of device memory through its own pool, or in a loop where a cudaMalloc would
stall the device; they cannot hand the layer a workspace. moe_forward_noalloc
serves them from a static device array inside the library. These tests call it
through the C ABI, twice in a row, and check each result against the regular
workspace-based moe_forward on the same inputs. Both entry points launch the
same kernels with the same layout, so the outputs must agree bit for bit. The
file is named so that pytest collects it last.
"""
import time

import pytest
import torch

from mixture_experts_ffn_expert_b200.binding import MOE_OPTION_TEST_WAIT_TIMEOUT, load_library
from mixture_experts_ffn_expert_b200.inputs import WORKLOADS, make_layer_inputs
from mixture_experts_ffn_expert_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

MOE_WORKSPACE_TOO_SMALL = 3
MOE_DEVICE_TIMEOUT = 6


def _ptrs(inp):
    return [inp[k].data_ptr() if inp[k] is not None else None
            for k in ("x", "W_g", "W1", "W3", "W2", "W1s", "W3s", "W2s")]


def _layer(shape, inp, **options):
    return MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                    shape.renorm, inp, bias=inp["bias"], device="cuda", **options)


# the decode shape and the tiny one (a different routing kernel configuration):
# each with the split router (the default) and the fused one (whose scan ticket
# lives in the scratch), and with its small shared expert merged into the routed
# launches (the default) or forked onto the plan's side stream
@pytest.mark.parametrize("merge", [-1, 0], ids=["shared_merged", "shared_forked"])
@pytest.mark.parametrize("fused", [-1, 1], ids=["split_router", "fused_router"])
@pytest.mark.parametrize("name", ["decode_t128_d2048_f512_e512k10_s1",
                                  "tiny_t256_d128_f64_e31k7_s1"])
def test_noalloc_forward_matches_workspace_forward_twice(name, fused, merge):
    shape = WORKLOADS[name]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    layer = _layer(shape, inp, fused_router=fused, merge_shared=merge)
    ref = layer(inp["x"]).clone()                    # regular entry point, caller workspace
    routing_before = layer.routing()
    torch.cuda.synchronize()
    lib = load_library()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(inp["x"], float("nan"))
        rc = lib.moe_forward_noalloc(layer.plan.handle, shape.T, *_ptrs(inp), out.data_ptr(),
                                     stream)
        assert rc == 0, (call, lib.moe_last_error())
        torch.cuda.synchronize()
        assert torch.equal(out, ref), call
    # the plan's getters still describe the last workspace forward
    routing_after = layer.routing()
    torch.cuda.synchronize()
    for key, val in routing_before.items():
        assert torch.equal(val, routing_after[key]), key
    # no bounded wait gave up, in the workspace or in the static scratch
    assert layer.device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    shape = WORKLOADS["decode_t128_d2048_f512_e512k10_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    layer = _layer(shape, inp)
    lib = load_library()
    out = torch.empty_like(inp["x"])
    big_T = 1 << 20                       # far beyond what 32 MiB of scratch can hold
    rc = lib.moe_forward_noalloc(layer.plan.handle, big_T, *_ptrs(inp), out.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == MOE_WORKSPACE_TOO_SMALL
    assert b"static scratch" in lib.moe_last_error()
    torch.cuda.synchronize()


def test_noalloc_timeout_is_reported_by_device_status():
    # the failure path without a fault: the one-shot test hook makes one CTA of
    # the routed gate/up GEMM (one CTA per tile on this shape) withhold a stage's
    # loads, its MMA warp's bounded wait (2 s) expires and the kernel writes
    # MOE_DEVICE_TIMEOUT into the static scratch's status word, which the plan's
    # status read must report; the next call is bitwise equal to a clean forward
    shape = WORKLOADS["tiny_t256_d128_f64_e31k7_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    layer = _layer(shape, inp)
    ref = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    lib = load_library()
    stream = torch.cuda.current_stream().cuda_stream
    out = torch.empty_like(inp["x"])
    layer.plan.set_option(MOE_OPTION_TEST_WAIT_TIMEOUT, 1)
    t0 = time.perf_counter()
    rc = lib.moe_forward_noalloc(layer.plan.handle, shape.T, *_ptrs(inp), out.data_ptr(), stream)
    assert rc == 0, lib.moe_last_error()
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert 1.5 < waited < 30.0, waited          # one bounded wait, not a hang
    assert layer.device_status() == MOE_DEVICE_TIMEOUT
    assert layer.device_status() == 0           # reading clears it
    rc = lib.moe_forward_noalloc(layer.plan.handle, shape.T, *_ptrs(inp), out.data_ptr(), stream)
    assert rc == 0, lib.moe_last_error()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(out, ref)
