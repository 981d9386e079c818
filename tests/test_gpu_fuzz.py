"""Seeded randomized GPU parity: random layer shapes, each run with the default
kernel choices and with a random combination of the options that only change
how the same arithmetic is scheduled (tile shapes, CTAs per SM, row gather,
tile order, shared-expert placement, CTA-pair GEMMs). Those must give the default's bits exactly, and
both must pass the oracle parity check; the fused router (different score
summation order) is checked against the oracle only.
"""
import os

import numpy as np
import pytest
import torch

from mixture_experts_ffn_expert_b200.inputs import LayerShape, make_layer_inputs

from parity import full_parity

pytestmark = pytest.mark.gpu

N_LAYERS = int(os.environ.get("MOE_FUZZ_LAYERS", "40"))   # more for a longer soak


def _draw(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.choice([1, 7, 64, 129, 300, 777, 1500, 2600]))
    d = int(rng.choice([64, 136, 200, 256, 512, 1024]))
    f = int(rng.choice([8, 64, 72, 192, 328, 512]))
    n = int(rng.choice([1, 3, 8, 17, 64, 100, 257, 300]))
    k = int(rng.integers(1, min(n, 12) + 1))
    ns = int(rng.choice([0, 1, 2]))
    renorm = bool(rng.integers(0, 2))
    bias = str(rng.choice(["none", "normal_var0.5", "zipf1.1"]))
    shape = LayerShape(f"fuzz{seed}_t{T}_d{d}_f{f}_e{n}k{k}_s{ns}", T, d, f, n, k, ns, renorm, bias)
    opts = {}
    cols = int(rng.choice([0, 32, 64, 128]))
    if cols:
        opts["swiglu_tile_cols"] = cols
    rows = int(rng.choice([0, 64, 128]))
    if rows:
        opts["tile_rows"] = rows
    if rng.integers(0, 2):
        opts["down_tile_cols"] = int(rng.choice([128, 256]))
    if rng.integers(0, 2):
        opts["ctas_per_sm"] = 2
    opts["gather_rows"] = int(rng.choice([0, 1]))
    opts["interleave"] = int(rng.choice([-1, 0, 1]))
    opts["merge_shared"] = int(rng.choice([-1, 0, 1]))
    pair = int(rng.choice([0, 1 << 40]))
    fused = bool(rng.integers(0, 2)) and n <= 512 and k <= 32
    return shape, opts, pair, fused


@pytest.mark.parametrize("seed", range(N_LAYERS))
def test_random_layers_options_agree_bitwise_and_match_the_oracle(seed):
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape, opts, pair, fused = _draw(1000 + seed)
    inp = make_layer_inputs(shape, seed=seed, device="cuda")
    tokens = None
    if shape.T > 1024:
        tokens = np.sort(np.random.default_rng(seed).choice(shape.T, size=512, replace=False))
    # the default kernels, then the option combination, both against the oracle
    full_parity(inp, shape, tokens=tokens, pair_min_rows=1 << 40)
    full_parity(inp, shape, tokens=tokens, pair_min_rows=1 << 40, **opts)
    if fused:
        full_parity(inp, shape, tokens=tokens, fused_router=1)
    outs = []
    for kw in ({"pair_min_rows": 1 << 40}, dict(opts, pair_min_rows=1 << 40), {"pair_min_rows": pair}):
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                         shape.renorm, inp, bias=inp["bias"], device="cuda", **kw)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0, kw
    assert torch.equal(outs[0], outs[1]), opts
    assert torch.equal(outs[0], outs[2]), pair
