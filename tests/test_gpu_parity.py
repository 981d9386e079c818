"""GPU parity: the CUDA layer through the C ABI against the fp64 oracle.

Small layers are compared on every output element; the five page-shaped
workloads at full size are compared on every token's routing and permutation
and on a seeded sample of 1024 output rows (every row for the 128-token decode
batch; tokens are independent given the routing, so a sampled row is checked
exactly).
"""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_expert_b200.inputs import LayerShape, WORKLOADS, make_layer_inputs

from parity import check_output, check_routing, full_parity, oracle_out, to64

pytestmark = pytest.mark.gpu

SMALL = [
    # name, T, d, f, N_r, k, N_s, renorm, bias
    ("one_token", 1, 128, 64, 31, 7, 1, True, "none"),
    ("three_tokens", 3, 128, 64, 8, 2, 0, True, "none"),
    ("ragged_17", 17, 256, 128, 16, 4, 1, False, "normal_var0.5"),
    ("k_equals_n", 40, 128, 64, 12, 12, 0, False, "none"),
    ("top1_single_expert", 50, 128, 96, 1, 1, 0, True, "none"),
    ("top1_plus_shared", 70, 128, 64, 16, 1, 1, True, "none"),
    ("two_shared_raw", 129, 192, 64, 10, 3, 2, False, "none"),
    ("ragged_tiles", 600, 384, 320, 6, 2, 1, True, "none"),        # several m/n tiles + tails
    ("k_tail_not_64", 77, 136, 72, 9, 3, 1, True, "none"),         # K and N not multiples of 64
    ("wide_router", 96, 256, 64, 512, 10, 1, True, "zipf1.1"),      # 16 scores per lane, 2 n-tiles
    ("max_router", 64, 128, 32, 1024, 32, 0, True, "none"),         # N_r and k at their limits
    ("skewed_groups", 1000, 256, 128, 64, 6, 1, True, "zipf1.1"),
    ("sliced_row_copy", 40, 1024, 64, 12, 3, 1, True, "none"),      # few chunks: 4 column slices
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_layers_all_outputs(case):
    name, T, d, f, n, k, ns, renorm, bias = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=1, device="cuda")
    res = full_parity(inp, shape)
    assert res["near_ties"] <= max(2, T * k // 20)


ROUTER_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias: shapes that reach the fused router's
    # edges (clusters of 1..8 CTAs, one or two accumulators, CTAs without K blocks,
    # ragged token tiles and K tails, the chunk scan folded or separate)
    ("fr_one_token_512", 1, 256, 64, 512, 10, 1, True, "zipf1.1"),      # 4 K blocks, 8 CTAs
    ("fr_second_acc_one_expert", 129, 128, 64, 257, 9, 0, False, "none"),
    ("fr_eight_experts", 300, 512, 64, 8, 2, 0, True, "none"),          # 16-row W_g boxes
    ("fr_k_tail", 200, 200, 64, 100, 5, 1, True, "normal_var0.5"),     # d = 3*64 + 8
    ("fr_two_acc_ragged", 1000, 1024, 64, 384, 6, 1, True, "zipf1.1"),
    ("fr_scan_not_folded", 16384, 256, 64, 256, 8, 0, True, "normal_var0.5"),
]


@pytest.mark.parametrize("case", ROUTER_CASES, ids=[c[0] for c in ROUTER_CASES])
def test_fused_router_edges(case):
    name, T, d, f, n, k, ns, renorm, bias = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=21, device="cuda")
    tokens = None
    if T > 2048:
        tokens = np.sort(np.random.default_rng(3).choice(T, size=512, replace=False))
    res = full_parity(inp, shape, tokens=tokens, fused_router=1)
    names = res["layer"].plan.kernel_names()
    assert "route_fused" in names and "router_gemm" not in names, names
    assert ("route_scan" in names) == (name == "fr_scan_not_folded"), names


SPLIT_ROUTER_CASES = ["one_token", "ragged_17", "k_equals_n", "wide_router", "skewed_groups"]


@pytest.mark.parametrize("case", [c for c in SMALL if c[0] in SPLIT_ROUTER_CASES],
                         ids=[c[0] for c in SMALL if c[0] in SPLIT_ROUTER_CASES])
def test_split_router_kernels(case):
    # the two-kernel router (split-K scores GEMM, then softmax + top-k), the
    # default, asked for explicitly on shapes the fused one also covers
    name, T, d, f, n, k, ns, renorm, bias = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=1, device="cuda")
    res = full_parity(inp, shape, fused_router=0)
    names = res["layer"].plan.kernel_names()
    assert "router_gemm" in names and "route_fused" not in names, names


NARROW_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias: the 64-column SwiGLU tiles (N=128
    # accumulators, four in TMEM) against the 128-column ones
    LayerShape("narrow_decode_like", 128, 2048, 512, 512, 10, 1, True, "zipf1.1"),
    LayerShape("narrow_ragged", 600, 384, 328, 6, 2, 1, True, "none"),      # f tail of 8
    LayerShape("narrow_k_tail", 77, 136, 72, 9, 3, 0, True, "none"),
]


@pytest.mark.parametrize("shape", NARROW_CASES, ids=[c.name for c in NARROW_CASES])
def test_narrow_swiglu_tiles(shape):
    # 64- or 128-column gate/up tiles, 64- or 128-row tiles of both routed GEMMs
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    inp = make_layer_inputs(shape, seed=8, device="cuda")
    res = full_parity(inp, shape)        # default tile choice, against the oracle
    outs = {}
    for cols in (64, 128):
        for rows in (64, 128):
            layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                             shape.renorm, inp, bias=inp["bias"], device="cuda",
                             swiglu_tile_cols=cols, tile_rows=rows)
            outs[cols, rows] = layer(inp["x"]).clone()
            names = layer.plan.kernel_names()
            gu = [n for n in names if n.startswith("grouped_gate_up")][0]
            dn = [n for n in names if n.startswith("grouped_down")][0]
            assert ("n64" in gu) == (cols == 64), names
            assert ("m64" in gu) == (rows == 64) and ("m64" in dn) == (rows == 64), names
    torch.cuda.synchronize()
    # every output element is the same sum in the same k order on every tile shape
    for key, out in outs.items():
        assert torch.equal(out, outs[128, 128]), key
    del res


INTERLEAVE_CASES = [
    # skewed loads: a few experts with several 128-row m-blocks among many with one
    LayerShape("interleave_zipf", 3000, 512, 256, 64, 6, 1, True, "zipf1.1"),
    LayerShape("interleave_normal_bias", 2048, 256, 192, 32, 4, 0, False, "normal_var0.5"),
]


@pytest.mark.parametrize("shape", INTERLEAVE_CASES, ids=[c.name for c in INTERLEAVE_CASES])
def test_interleaved_tile_order(shape):
    # the same tiles in another order: the same bits, and parity with the oracle
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    inp = make_layer_inputs(shape, seed=17, device="cuda")
    full_parity(inp, shape)
    outs = []
    for il in (0, 1):
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                         shape.renorm, inp, bias=inp["bias"], device="cuda", interleave=il,
                         tile_rows=128)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0
    assert torch.equal(outs[0], outs[1])


OCC_CASES = [
    # weight streaming: few rows per expert, 64- and 128-row tiles
    LayerShape("occ_decode_like", 96, 256, 128, 64, 6, 1, True, "zipf1.1"),
    # several m-blocks per expert and a ragged tail
    LayerShape("occ_ragged", 1100, 256, 192, 8, 2, 0, False, "normal_var0.5"),
]


@pytest.mark.parametrize("tile_rows,cols,dcols", [(64, 32, 128), (64, 64, 256), (64, 128, 128),
                                                   (128, 32, 256), (128, 64, 128),
                                                   (128, 128, 256)])
@pytest.mark.parametrize("shape", OCC_CASES, ids=[c.name for c in OCC_CASES])
def test_two_ctas_per_sm_routed_gemms(shape, tile_rows, cols, dcols):
    # two resident CTAs per SM run the same tiles with half the ring each, and
    # tiles of 32..128 gate/up and 128 or 256 down output columns: the same bits
    # as one CTA per SM, and parity with the oracle
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    inp = make_layer_inputs(shape, seed=23, device="cuda")
    opts = dict(tile_rows=tile_rows, swiglu_tile_cols=cols, down_tile_cols=dcols,
                pair_min_rows=1 << 40)
    full_parity(inp, shape, ctas_per_sm=2, **opts)
    outs = []
    for occ in (1, 2):
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                         shape.renorm, inp, bias=inp["bias"], device="cuda", ctas_per_sm=occ,
                         **opts)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        names = layer.plan.kernel_names()
        assert any(n.startswith("grouped_gate_up") and ("x2" in n) == (occ == 2) for n in names)
    assert torch.equal(outs[0], outs[1])


GATHER_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias, options
    ("gather_default_tiles", 700, 256, 192, 8, 2, 1, True, "none", {}),
    ("gather_k_tail", 200, 200, 64, 100, 5, 1, True, "normal_var0.5", {}),           # d = 3*64 + 8
    ("gather_rows64", 600, 384, 328, 6, 2, 1, True, "none", {"tile_rows": 64}),     # f tail of 8
    ("gather_cols32", 96, 256, 128, 64, 6, 1, True, "zipf1.1",
     {"swiglu_tile_cols": 32, "tile_rows": 64}),
    ("gather_two_ctas", 1100, 256, 192, 8, 2, 0, False, "normal_var0.5", {"ctas_per_sm": 2}),
    ("gather_dropping", 512, 128, 64, 16, 4, 1, True, "zipf1.1", {"capacity": 40}),
]


@pytest.mark.parametrize("case", GATHER_CASES, ids=[c[0] for c in GATHER_CASES])
def test_gate_up_gathers_rows_from_x(case):
    # the gate/up GEMM's producer warps gather the grouped rows from x through
    # the permutation (no permuted copy): the same bits as the copy path, and
    # parity with the oracle
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    name, T, d, f, n, k, ns, renorm, bias, opts = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=29, device="cuda")
    opts = dict(opts, pair_min_rows=1 << 40)
    full_parity(inp, shape, gather_rows=1, **opts)
    outs = []
    for g in (0, 1):
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                         shape.renorm, inp, bias=inp["bias"], device="cuda", gather_rows=g,
                         **opts)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0
    assert torch.equal(outs[0], outs[1])


PAIR_CASES = ["three_tokens", "ragged_17", "two_shared_raw", "ragged_tiles", "k_tail_not_64",
              "skewed_groups"]


@pytest.mark.parametrize("wide", [0, 1], ids=["pair256", "pair512"])
@pytest.mark.parametrize("case", [c for c in SMALL if c[0] in PAIR_CASES],
                         ids=[c[0] for c in SMALL if c[0] in PAIR_CASES])
def test_small_layers_cta_pair_kernel(case, wide):
    # every GEMM (routed and shared) forced onto the cta_group::2 kernel, with
    # 256- or 512-column tiles
    name, T, d, f, n, k, ns, renorm, bias = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=4, device="cuda")
    full_parity(inp, shape, pair_min_rows=0, wide_tiles=wide)


@pytest.mark.parametrize("pair_min_rows,wide", [(0, 0), (0, 1), (1 << 40, -1)])
def test_pair_and_single_kernels_agree_bitwise(pair_min_rows, wide):
    # all GEMM kernels accumulate each output in the same k order, so results match exactly
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = LayerShape("agree", 700, 256, 192, 4, 2, 1, True, "none")
    inp = make_layer_inputs(shape, seed=5, device="cuda")
    ref = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared, True, inp,
                   device="cuda", pair_min_rows=1 << 40)(inp["x"]).clone()
    got = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared, True, inp,
                   device="cuda", pair_min_rows=pair_min_rows, wide_tiles=wide)(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


MERGE_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias, expected variant names; the
    # shared expert is too large for the side stream in the first three, small
    # (merged by default, else forked) in the last two, whose gate/up GEMMs also
    # gather their rows from x
    ("merged_both", 2048, 256, 640, 32, 2, 2, True, "none",
     ["grouped_gate_up[+shared]", "grouped_down[+shared]"]),
    ("merged_ragged", 2000, 320, 576, 40, 3, 3, False, "normal_var0.5",
     ["grouped_gate_up[+shared]", "grouped_down[+shared]"]),
    # 256 rows per expert: the routed down projection runs on CTA pairs, so
    # only the gate/up GEMM carries the shared tiles
    ("merged_gate_up_only", 2048, 256, 640, 16, 2, 2, True, "none",
     ["grouped_gate_up[+shared]", "grouped_down[pair]", "shared_down"]),
    ("merged_small_gathered", 200, 256, 320, 96, 6, 1, True, "zipf1.1",
     ["grouped_gate_up[+shared]", "grouped_down[+shared]"]),
    ("merged_small_two_shared", 77, 192, 72, 40, 4, 2, False, "none",
     ["grouped_gate_up[+shared]", "grouped_down[+shared]"]),
]


@pytest.mark.parametrize("case", MERGE_CASES, ids=[c[0] for c in MERGE_CASES])
def test_shared_expert_merged_into_routed_launches(case):
    name, T, d, f, n, k, ns, renorm, bias, expect = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=7, device="cuda")
    res = full_parity(inp, shape, merge_shared=1)
    names = res["layer"].plan.kernel_names()
    for e in expect:
        assert e in names, names
    assert "shared_gate_up" not in names, names


@pytest.mark.parametrize("case", MERGE_CASES, ids=[c[0] for c in MERGE_CASES])
def test_merged_and_separate_shared_expert_agree_bitwise(case):
    # a merged shared tile runs the same k loop and epilogue as a separate launch
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    name, T, d, f, n, k, ns, renorm, bias, _ = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=8, device="cuda")
    outs = []
    for merge in (0, 1):
        layer = MoELayer(d, f, n, k, ns, renorm, inp, bias=inp["bias"], device="cuda",
                         merge_shared=merge)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("options,merged", [({}, True), ({"merge_shared": 0}, False),
                                            ({"swiglu_tile_cols": 64}, False),
                                            ({"tile_rows": 64}, False)],
                         ids=["default", "never", "narrow_tiles", "short_tiles"])
def test_small_shared_expert_placement(options, merged):
    # automatic placement: a small shared expert rides in the routed launches
    # unless merging is switched off or the routed tile shape was chosen
    # explicitly; then it runs on the side stream. Same bits either way.
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = LayerShape("small_shared", 160, 256, 256, 64, 6, 1, True, "zipf1.1")
    inp = make_layer_inputs(shape, seed=10, device="cuda")
    outs, names = [], []
    for kw in ({"merge_shared": 0}, options):
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                         shape.renorm, inp, bias=inp["bias"], device="cuda", **kw)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        names.append(layer.plan.kernel_names())
    assert "shared_gate_up" in names[0], names[0]
    assert ("grouped_gate_up[+shared]" in names[1]) == merged, names[1]
    assert ("shared_gate_up" in names[1]) == (not merged), names[1]
    assert torch.equal(outs[0], outs[1])


CONCURRENT_CASES = [
    # a shared expert too large for the routing phase, beside weight-streaming
    # routed GEMMs (fewer than 192 rows per expert): forked onto a few SMs
    LayerShape("concurrent_prefill_like", 2048, 512, 256, 64, 4, 1, True, "normal_var0.5"),
    LayerShape("concurrent_two_shared", 1500, 384, 192, 48, 6, 2, False, "none"),
]


@pytest.mark.parametrize("shape", CONCURRENT_CASES, ids=[c.name for c in CONCURRENT_CASES])
def test_shared_expert_beside_the_routed_gemms(shape):
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    inp = make_layer_inputs(shape, seed=9, device="cuda")
    full_parity(inp, shape)                     # default policy, against the oracle
    outs = []
    for conc in (0, 1):
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                         shape.renorm, inp, bias=inp["bias"], device="cuda",
                         shared_concurrent=conc)
        outs.append(layer(inp["x"]).clone())
        torch.cuda.synchronize()
        assert layer.device_status() == 0
    # the same kernels on other SMs and streams: the same bits
    assert torch.equal(outs[0], outs[1])


def test_default_gemm_variants_on_coarse_shape():
    # defaults: SwiGLU GEMMs on the single-CTA kernel, the routed down projection
    # with many rows per expert and a long reduction on wide CTA pairs
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = LayerShape("variants", 8192, 2048, 4096, 8, 2, 0, True, "none")
    inp = make_layer_inputs(shape, seed=6, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared, True, inp,
                     device="cuda")
    layer(inp["x"])
    torch.cuda.synchronize()
    names = layer.plan.kernel_names()
    assert "grouped_gate_up" in names, names
    assert "grouped_down[pair512]" in names, names


def test_non_finite_tokens_keep_routing_in_range():
    # NaN / infinite activations give NaN router scores; the top-k must still pick
    # k distinct in-range experts for them (the permutation indexes with these),
    # and every other token is unaffected
    from oracle import route_permutation, router_scores, softmax_rows
    from parity import check_output, oracle_out, reconcile_routing, run_layer, to64
    T, k, n = 96, 4, 16
    shape = LayerShape("nonfinite", T, 128, 64, n, k, 1, True, "none")
    inp = make_layer_inputs(shape, seed=9, device="cuda")
    x = inp["x"].clone()
    x[3, 5] = float("nan")
    x[10, :] = float("inf")
    x[11, 7] = float("-inf")
    out, routing, _ = run_layer(dict(inp, x=x), shape)
    idx = routing["idx"].cpu().numpy().astype(np.int64)
    assert idx.min() >= 0 and idx.max() < n
    assert all(len(set(row.tolist())) == k for row in idx)
    counts, offsets, perm_src, inv_pos = route_permutation(idx, n)
    np.testing.assert_array_equal(routing["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(routing["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(routing["perm_src"].cpu().numpy(), perm_src)
    np.testing.assert_array_equal(routing["inv_pos"].cpu().numpy(), inv_pos)
    clean = np.array([t for t in range(T) if t not in (3, 10, 11)])
    sub = dict(inp, x=x[torch.as_tensor(clean, device=x.device)])
    p = softmax_rows(router_scores(to64(sub["x"]), to64(inp["W_g"]), None))
    idx_ref, _ = reconcile_routing(p, idx[clean], k)
    ref = oracle_out(sub, shape, idx_ref)
    check_output(to64(out)[clean], ref)


def test_tiny_workload_all_outputs():
    shape = WORKLOADS["tiny_t256_d128_f64_e31k7_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    full_parity(inp, shape)


# outputs on a seeded subset of 1024 tokens (all tokens for decode); routing,
# counts, offsets and the permutation on every token
@pytest.mark.parametrize("name,n_tokens", [
    ("coarse_t4096_d4096_f14336_e8k2_s0", 1024),
    ("dsmoe_small_t8192_d2048_f1408_e64k6_s2", 1024),
    ("dsv3_prefill_t4096_d7168_f2048_e256k8_s1", 1024),
    ("decode_t128_d2048_f512_e512k10_s1", 128),
])
def test_full_size_workloads(name, n_tokens):
    shape = WORKLOADS[name]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    rng = np.random.default_rng(1234)
    tokens = np.sort(rng.choice(shape.T, size=min(n_tokens, shape.T), replace=False))
    res = full_parity(inp, shape, tokens=tokens)
    print(f"{name}: near ties {res['near_ties']}, rel-L2 {res['rel_l2']:.2e}, "
          f"max-abs {res['max_abs']:.2e} of max|ref| {res['max_ref']:.2e}")
    del inp
    torch.cuda.empty_cache()


CAPACITY_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias, seats per expert, pair_min_rows
    ("cap_one_seat", 200, 128, 64, 16, 2, 1, True, "none", 1, None),
    ("cap_skewed", 1000, 256, 128, 64, 6, 1, True, "zipf1.1", 64, None),
    ("cap_all_overflow_raw", 600, 384, 320, 6, 2, 1, False, "none", 150, None),
    ("cap_pairs", 600, 384, 320, 6, 2, 1, True, "normal_var0.5", 170, 0),
    ("cap_no_drop", 300, 128, 64, 8, 2, 0, True, "none", 10000, None),
]


@pytest.mark.parametrize("case", CAPACITY_CASES, ids=[c[0] for c in CAPACITY_CASES])
def test_expert_capacity_drops_the_later_pairs(case):
    # "What is an expert, really?" glossary, capacity factor / token dropping
    name, T, d, f, n, k, ns, renorm, bias, cap, pmr = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=10, device="cuda")
    res = full_parity(inp, shape, capacity=cap, pair_min_rows=pmr)
    r = res["layer"].routing()
    counts = r["counts"].cpu().numpy()
    dropped = int((r["inv_pos"].cpu().numpy() < 0).sum())
    assert dropped == int(np.maximum(counts - cap, 0).sum())
    assert int(r["offsets"][-1]) == T * k - dropped


SELECTION_ONLY_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias
    ("selonly_normal_renorm", 600, 256, 128, 64, 6, 1, True, "normal_var0.5"),
    ("selonly_zipf_raw", 500, 256, 128, 128, 8, 1, False, "zipf1.1"),
    ("selonly_top1_raw", 300, 128, 64, 16, 1, 0, False, "normal_var0.5"),  # renormalised top-1 is always 1
]


@pytest.mark.parametrize("case", SELECTION_ONLY_CASES, ids=[c[0] for c in SELECTION_ONLY_CASES])
def test_selection_only_bias(case):
    name, T, d, f, n, k, ns, renorm, bias = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=14, device="cuda")
    res = full_parity(inp, shape, bias_selection_only=True)
    assert res["near_ties"] <= max(2, T * k // 20)
    # the same selections as the logit-bias layer, different gates
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    logit = MoELayer(d, f, n, k, ns, renorm, inp, bias=inp["bias"], device="cuda")
    logit(inp["x"])
    a, b = res["layer"].routing(), logit.routing()
    same_sel = (a["idx"] == b["idx"]).float().mean().item()
    assert same_sel > 0.99
    assert not torch.allclose(a["w"], b["w"])


def test_selection_only_bias_on_the_decode_shape():
    shape = WORKLOADS["decode_t128_d2048_f512_e512k10_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    full_parity(inp, shape, bias_selection_only=True)
    del inp
    torch.cuda.empty_cache()


def test_capacity_factor_seats_computed_by_the_library():
    # the glossary's capacity factor passed through the C ABI (thousandths); the
    # seats are ceil(cf * T * k / N_r), at least one, written out here by hand
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = LayerShape("cf", 8, 128, 64, 256, 8, 0, True, "none")
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    for cf, T, want in [(1.0, 4096, 128), (1.25, 4096, 160), (0.001, 10, 1), (0.5, 1000, 16)]:
        layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, 0, True, inp,
                         device="cuda", capacity_factor=cf)
        assert layer.capacity_seats(T) == want, (cf, T)
    shape7 = LayerShape("cf7", 8, 128, 64, 7, 3, 0, True, "none")
    inp7 = make_layer_inputs(shape7, seed=0, device="cuda")
    layer = MoELayer(128, 64, 7, 3, 0, True, inp7, device="cuda", capacity_factor=1.0)
    assert layer.capacity_seats(100) == 43            # 300 / 7 = 42.86, rounded up
    layer = MoELayer(128, 64, 7, 3, 0, True, inp7, device="cuda", capacity=5)
    assert layer.capacity_seats(100) == 5
    layer = MoELayer(128, 64, 7, 3, 0, True, inp7, device="cuda")
    assert layer.capacity_seats(100) == 0


def test_capacity_factor_on_the_deepseek_v3_shape():
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = WORKLOADS["dsv3_prefill_t4096_d7168_f2048_e256k8_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    cap = -(-shape.T * shape.top_k // shape.n_routed)        # factor 1.0: 128 seats
    assert cap == 128
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, bias=inp["bias"], device="cuda", capacity_factor=1.0)
    assert layer.capacity_seats(shape.T) == cap
    out = layer(inp["x"])
    routing = layer.routing()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _, idx_ref, _ = check_routing(inp, routing, shape, capacity=cap)
    tokens = np.sort(np.random.default_rng(77).choice(shape.T, size=24, replace=False))
    ref = oracle_out(inp, shape, idx_ref, tokens, capacity=cap)
    check_output(to64(out[torch.as_tensor(tokens, device=out.device)]), ref)
    assert (routing["inv_pos"].cpu().numpy() < 0).any()   # the skewed bias overflows some experts
    del inp, layer
    torch.cuda.empty_cache()


def test_many_tokens_routing_and_sampled_outputs():
    # 65536 tokens x 8 slots: 512 routing chunks, 524288 grouped rows (int32 row
    # indices well past 2^16, offsets past 2^18); routing is checked on every token
    shape = LayerShape("many_tokens", 65536, 256, 128, 64, 8, 1, True, "normal_var0.5")
    inp = make_layer_inputs(shape, seed=12, device="cuda")
    tokens = np.sort(np.random.default_rng(5).choice(shape.T, size=256, replace=False))
    res = full_parity(inp, shape, tokens=tokens)
    assert res["near_ties"] <= shape.T * shape.top_k // 50
    del inp
    torch.cuda.empty_cache()


POISON_CASES = [
    # name, T, d, f, N_r, k, N_s, renorm, bias, capacity, pair_min_rows
    ("poison_ragged", 600, 384, 320, 6, 2, 1, True, "none", None, None),
    ("poison_pairs", 600, 384, 320, 6, 2, 1, True, "none", None, 0),
    ("poison_capacity", 1000, 256, 128, 64, 6, 1, True, "zipf1.1", 40, None),
    ("poison_decode_like", 128, 2048, 512, 512, 10, 1, True, "zipf1.1", None, None),
]


@pytest.mark.parametrize("case", POISON_CASES, ids=[c[0] for c in POISON_CASES])
def test_poisoned_workspace_and_output_are_fully_overwritten(case):
    # every scratch byte 0xFF (NaN as bf16 / fp32, -1 as int32) and out NaN before
    # the forward: a kernel reading scratch that no kernel wrote, or leaving part
    # of out unwritten, shows up as NaN or a parity failure
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    from parity import check_output, check_routing, oracle_out, to64
    name, T, d, f, n, k, ns, renorm, bias, cap, pmr = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=13, device="cuda")
    layer = MoELayer(d, f, n, k, ns, renorm, inp, bias=inp["bias"], device="cuda",
                     capacity=cap, pair_min_rows=pmr)
    layer.ensure_workspace(T)
    layer.workspace[256:].fill_(0xFF)          # the first 256 bytes hold the status word
    out = torch.full_like(inp["x"], float("nan"))
    layer(inp["x"], out)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.isfinite(out).all()
    _, idx_ref, _ = check_routing(inp, layer.routing(), shape, capacity=cap)
    check_output(to64(out), oracle_out(inp, shape, idx_ref, capacity=cap))


def _random_cases(n=14, seed=2024):
    """Seeded random layer shapes within the library's limits (d, f multiples of
    8, N_r <= 1024, k <= 32), with random bias modes, capacities and kernels."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        n_r = int(rng.choice([1, 2, 5, 8, 17, 33, 64, 100, 257]))
        k = int(rng.integers(1, min(n_r, 16) + 1))
        T = int(rng.choice([1, 2, 7, 64, 129, 300, 777, 2000]))
        d = 8 * int(rng.integers(1, 97))
        f = 8 * int(rng.integers(1, 97))
        ns = int(rng.integers(0, 4))
        renorm = bool(rng.integers(0, 2))
        bias = str(rng.choice(["none", "normal_var0.5", "zipf1.1"]))
        sel_only = bias != "none" and bool(rng.integers(0, 2))
        cap = int(rng.integers(1, max(2, T * k // n_r + 2))) if rng.random() < 0.3 else None
        pmr = 0 if rng.random() < 0.3 else None
        cases.append((f"rand{i}_T{T}_d{d}_f{f}_e{n_r}k{k}_s{ns}", T, d, f, n_r, k, ns, renorm,
                      bias, sel_only, cap, pmr))
    return cases


RANDOM_CASES = _random_cases()


@pytest.mark.parametrize("case", RANDOM_CASES, ids=[c[0] for c in RANDOM_CASES])
def test_random_shapes_all_outputs(case):
    name, T, d, f, n, k, ns, renorm, bias, sel_only, cap, pmr = case
    shape = LayerShape(name, T, d, f, n, k, ns, renorm, bias)
    inp = make_layer_inputs(shape, seed=15, device="cuda")
    full_parity(inp, shape, capacity=cap, pair_min_rows=pmr, bias_selection_only=sel_only)


def test_zero_tokens_is_a_noop():
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = WORKLOADS["tiny_t256_d128_f64_e31k7_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda", T=0)
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared, True,
                     inp, device="cuda")
    out = layer(inp["x"])
    torch.cuda.synchronize()
    assert out.shape == (0, shape.d)
    assert layer.plan.last_launch_count() == 0


def test_repeated_forwards_are_deterministic():
    shape = LayerShape("det", 300, 256, 128, 16, 4, 1, True, "none")
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    inp = make_layer_inputs(shape, seed=3, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared, True,
                     inp, device="cuda")
    a = layer(inp["x"]).clone()
    b = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_error_paths_on_device():
    from mixture_experts_ffn_expert_b200.binding import MoEError, Plan
    shape = WORKLOADS["tiny_t256_d128_f64_e31k7_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    plan = Plan(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared, True)
    T = shape.T
    need = plan.workspace_bytes(T)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(inp["x"])
    p = {k: (v.data_ptr() if v is not None else None) for k, v in inp.items()}
    args = (p["x"], p["W_g"], p["W1"], p["W3"], p["W2"], p["W1s"], p["W3s"], p["W2s"],
            out.data_ptr())
    with pytest.raises(MoEError) as e:          # no workspace yet
        plan.forward(T, *args)
    assert e.value.status == 2
    plan.set_workspace(ws.data_ptr(), need - 256)
    with pytest.raises(MoEError) as e:
        plan.forward(T, *args)
    assert e.value.status == 3
    plan.set_workspace(ws.data_ptr(), need)
    with pytest.raises(MoEError) as e:          # shared weights missing while N_s = 1
        plan.forward(T, *args[:5], None, None, None, args[8])
    assert e.value.status == 2
    with pytest.raises(MoEError) as e:          # misaligned pointer
        plan.forward(T, args[0] + 2, *args[1:])
    assert e.value.status == 2
    with pytest.raises(MoEError) as e:
        plan.forward(-1, *args)
    assert e.value.status == 2
    from mixture_experts_ffn_expert_b200.binding import MOE_OPTION_EXPERT_CAPACITY
    with pytest.raises(MoEError) as e:          # negative seat limit
        plan.set_option(MOE_OPTION_EXPERT_CAPACITY, -1)
    assert e.value.status == 2
    plan.forward(T, *args)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    plan.close()


def test_bounded_wait_timeout_sets_status_and_context_recovers():
    # the failure path without a fault: the one-shot test hook makes one CTA of
    # the gate/up GEMM withhold a stage's loads, so its MMA warp's bounded wait
    # (2 s) expires; the kernel must report MOE_DEVICE_TIMEOUT and leave the
    # context usable
    import time
    from mixture_experts_ffn_expert_b200.binding import MOE_OPTION_TEST_WAIT_TIMEOUT
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = WORKLOADS["tiny_t256_d128_f64_e31k7_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, bias=inp["bias"], device="cuda")
    ref = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.plan.set_option(MOE_OPTION_TEST_WAIT_TIMEOUT, 1)
    t0 = time.perf_counter()
    layer(inp["x"])
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert layer.device_status() == 6          # MOE_DEVICE_TIMEOUT
    assert layer.device_status() == 0          # reading clears it
    assert 1.5 < waited < 30.0, waited         # one bounded wait, not a hang
    again = layer(inp["x"])                    # the hook was one-shot
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(again, ref)


def test_inconsistent_routing_state_is_reported_not_written_out_of_range():
    # a workspace overwritten during a forward: the fused router's ticket (byte 64
    # of the workspace, zero between forwards) is set to a value no forward
    # reaches, so no cluster scans the tile histogram; the permutation kernel
    # must find the totals inconsistent, drop every routed slot (the output is
    # the shared expert alone), report MOE_DEVICE_INCONSISTENT, and the next
    # forward must be clean again
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = LayerShape("one_tile", 100, 256, 128, 24, 4, 1, True, "none")
    inp = make_layer_inputs(shape, seed=31, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, device="cuda", fused_router=1)
    ref = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.workspace[64:68].view(torch.int32).fill_(1 << 20)
    out = layer(inp["x"]).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 7               # MOE_DEVICE_INCONSISTENT
    assert torch.isfinite(out).all()
    shared_only = oracle_out(inp, shape, None, capacity=0)     # every routed slot dropped
    check_output(to64(out), shared_only)
    again = layer(inp["x"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(again, ref)


@pytest.mark.parametrize("merge", [-1, 0], ids=["shared_merged", "shared_forked"])
@pytest.mark.parametrize("name", ["decode_t128_d2048_f512_e512k10_s1", "tiny_t256_d128_f64_e31k7_s1"])
def test_cuda_graph_replay_matches_stream_launch(name, merge):
    # the whole forward (with the small shared expert merged into the routed
    # launches, or on its forked stream) is captured once and replayed; replays
    # must reproduce the plain result
    from mixture_experts_ffn_expert_b200.layer import MoELayer
    shape = WORKLOADS[name]
    inp = make_layer_inputs(shape, seed=2, device="cuda")
    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, inp, bias=inp["bias"], device="cuda", merge_shared=merge)
    x = inp["x"]
    want = layer(x).clone()
    out = torch.empty_like(x)
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        layer(x, out)
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        layer(x, out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, want)
    assert layer.device_status() == 0
