"""The oracle's full layer against brute force, special cases and the shared-term rules."""
import numpy as np
import pytest

from oracle import (moe_layer, moe_layer_dense_bruteforce, select_topk, softmax_rows,
                    router_scores, swiglu_ffn)


def _tiny(rng, T, d, f, n, ns, bias=False):
    x = rng.normal(size=(T, d))
    W_g = rng.normal(size=(n, d)) / np.sqrt(d)
    W1 = rng.normal(size=(n, f, d)) / np.sqrt(d)
    W3 = rng.normal(size=(n, f, d)) / np.sqrt(d)
    W2 = rng.normal(size=(n, d, f)) / np.sqrt(f)
    shared = None
    if ns:
        shared = (rng.normal(size=(ns * f, d)) / np.sqrt(d),
                  rng.normal(size=(ns * f, d)) / np.sqrt(d),
                  rng.normal(size=(d, ns * f)) / np.sqrt(ns * f))
    b = rng.normal(size=n) if bias else None
    return x, W_g, b, (W1, W3, W2), shared


CASES = [
    # T, d, f, N_r, k, N_s, renorm, bias
    (5, 6, 4, 7, 2, 1, True, False),
    (4, 5, 3, 6, 3, 0, False, False),
    (3, 4, 2, 5, 5, 2, True, True),
    (6, 3, 5, 4, 1, 1, False, True),
    (2, 7, 3, 1, 1, 0, True, False),
]


@pytest.mark.parametrize("T,d,f,n,k,ns,renorm,bias", CASES)
def test_layer_equals_dense_bruteforce(T, d, f, n, k, ns, renorm, bias):
    rng = np.random.default_rng(T * 100 + d * 10 + n)
    x, W_g, b, experts, shared = _tiny(rng, T, d, f, n, ns, bias)
    got = moe_layer(x, W_g, b, experts, shared, k, renorm)["out"]
    want = moe_layer_dense_bruteforce(x, W_g, b, *experts, shared, k, renorm)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_token_subset_and_streamed_experts_match_full_run():
    rng = np.random.default_rng(11)
    x, W_g, b, experts, shared = _tiny(rng, 12, 8, 4, 9, 1, True)
    full = moe_layer(x, W_g, b, experts, shared, 3, True)
    W1, W3, W2 = experts
    sub = moe_layer(x, W_g, b, lambda e: (W1[e], W3[e], W2[e]), shared, 3, True,
                    tokens=[7, 2, 11])
    np.testing.assert_allclose(sub["out"], full["out"][[7, 2, 11]], rtol=1e-14)
    np.testing.assert_array_equal(sub["counts"], full["counts"])


def test_k_equals_n_raw_gates_is_dense_probability_mixture():
    # special case: every expert selected, raw gates, no shared -> sum_e p_e E_e(x)
    rng = np.random.default_rng(12)
    x, W_g, _, experts, _ = _tiny(rng, 6, 5, 3, 4, 0)
    W1, W3, W2 = experts
    p = softmax_rows(router_scores(x, W_g))
    want = sum(p[:, e:e + 1] * swiglu_ffn(x, W1[e], W3[e], W2[e]) for e in range(4))
    got = moe_layer(x, W_g, None, experts, None, 4, False)["out"]
    np.testing.assert_allclose(got, want, rtol=1e-12)


def test_single_expert_top1_is_plain_swiglu_mlp():
    # N_r = 1, k = 1, renormalised: the gate is exactly 1 and the layer is a dense FFN
    rng = np.random.default_rng(13)
    x, W_g, _, experts, _ = _tiny(rng, 5, 6, 4, 1, 0)
    W1, W3, W2 = experts
    r = moe_layer(x, W_g, None, experts, None, 1, True)
    np.testing.assert_array_equal(r["g"], np.ones((5, 1)))
    np.testing.assert_allclose(r["out"], swiglu_ffn(x, W1[0], W3[0], W2[0]), rtol=1e-14)


def test_shared_term_ignores_router_and_has_coefficient_one():
    rng = np.random.default_rng(14)
    x, W_g, b, experts, shared = _tiny(rng, 7, 6, 4, 5, 1, True)
    W1, W3, W2 = experts
    zero_routed = (W1, W3, np.zeros_like(W2))
    out_a = moe_layer(x, W_g, b, zero_routed, shared, 2, True)["out"]
    out_b = moe_layer(x, rng.normal(size=W_g.shape), None, zero_routed, shared, 2, False)["out"]
    want = swiglu_ffn(x, *shared)            # exactly the shared SwiGLU, no 1/N_s, no gate
    np.testing.assert_array_equal(out_a, want)
    np.testing.assert_array_equal(out_b, want)
    # shared + routed split: the routed part is what remains with the shared term removed
    full = moe_layer(x, W_g, b, experts, shared, 2, True)["out"]
    routed = moe_layer(x, W_g, b, experts, None, 2, True)["out"]
    np.testing.assert_allclose(full - routed, want, rtol=1e-12, atol=1e-14)


def test_shared_not_in_topk_pool():
    # the shared expert never takes a routed slot: the selection only sees W_g's rows
    rng = np.random.default_rng(15)
    x, W_g, b, experts, shared = _tiny(rng, 9, 5, 3, 6, 2, False)
    with_shared = moe_layer(x, W_g, b, experts, shared, 3, True)
    without = moe_layer(x, W_g, b, experts, None, 3, True)
    np.testing.assert_array_equal(with_shared["idx"], without["idx"])
    assert with_shared["idx"].max() < 6


def test_fused_two_shared_equals_sum_of_two_separate():
    rng = np.random.default_rng(16)
    d, f = 6, 3
    x = rng.normal(size=(5, d))
    A = [(rng.normal(size=(f, d)), rng.normal(size=(f, d)), rng.normal(size=(d, f)))
         for _ in range(2)]
    fused = (np.concatenate([A[0][0], A[1][0]]), np.concatenate([A[0][1], A[1][1]]),
             np.concatenate([A[0][2], A[1][2]], axis=1))
    separate = swiglu_ffn(x, *A[0]) + swiglu_ffn(x, *A[1])
    np.testing.assert_allclose(swiglu_ffn(x, *fused), separate, rtol=1e-12, atol=1e-14)


def test_forced_selection_rescores_with_oracle_probabilities():
    rng = np.random.default_rng(17)
    x, W_g, b, experts, shared = _tiny(rng, 4, 5, 3, 6, 0, False)
    base = moe_layer(x, W_g, b, experts, shared, 2, True)
    forced = base["idx"].copy()
    forced[0] = [5, 4] if list(forced[0]) != [5, 4] else [0, 1]
    r = moe_layer(x, W_g, b, experts, shared, 2, True, forced_idx=forced)
    np.testing.assert_array_equal(r["idx"], forced)
    np.testing.assert_allclose(r["out"][1:], base["out"][1:], rtol=1e-14)
    W1, W3, W2 = experts
    p = base["p"][0]
    e0, e1 = forced[0]
    g0, g1 = p[e0] / (p[e0] + p[e1]), p[e1] / (p[e0] + p[e1])
    want = g0 * swiglu_ffn(x[:1], W1[e0], W3[e0], W2[e0]) + g1 * swiglu_ffn(x[:1], W1[e1], W3[e1], W2[e1])
    np.testing.assert_allclose(r["out"][:1], want, rtol=1e-12)


def test_oracle_on_seeded_tiny_workload_inputs():
    # the shared input generator feeds the oracle on CPU; bf16 values widen exactly
    import torch
    from mixture_experts_ffn_expert_b200.inputs import WORKLOADS, make_layer_inputs
    shape = WORKLOADS["tiny_t256_d128_f64_e31k7_s1"]
    inp = make_layer_inputs(shape, seed=0, device="cpu", T=8)
    f64 = {k: (v.to(torch.float64).numpy() if v is not None else None) for k, v in inp.items()}
    r = moe_layer(f64["x"], f64["W_g"], f64["bias"], (f64["W1"], f64["W3"], f64["W2"]),
                  (f64["W1s"], f64["W3s"], f64["W2s"]), shape.top_k, shape.renorm)
    assert r["out"].shape == (8, 128)
    assert np.all(np.isfinite(r["out"]))
    np.testing.assert_allclose(r["g"].sum(1), 1.0, atol=1e-12)
    assert r["idx"].shape == (8, 7) and len(set(map(tuple, np.sort(r["idx"], 1)))) >= 1


@pytest.mark.parametrize("capacity", [0, 1, 2, 3])
def test_capacity_layer_equals_seat_by_seat_bruteforce(capacity):
    # [WIE] glossary "capacity factor / token dropping": a pair without a seat
    # is skipped; the brute force hands out seats in plain loops
    rng = np.random.default_rng(21)
    T, d, f, n, k, ns = 9, 5, 4, 4, 2, 1
    x, W_g, b, experts, shared = _tiny(rng, T, d, f, n, ns, bias=True)
    ref = moe_layer_dense_bruteforce(x, W_g, b, *experts, shared, k, True, capacity=capacity)
    got = moe_layer(x, W_g, b, experts, shared, k, True, capacity=capacity)["out"]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_zero_capacity_leaves_only_the_shared_expert():
    rng = np.random.default_rng(22)
    x, W_g, b, experts, shared = _tiny(rng, 7, 6, 4, 5, 2)
    got = moe_layer(x, W_g, b, experts, shared, 2, False, capacity=0)["out"]
    only_shared = moe_layer(x, W_g, b, tuple(np.zeros_like(a) for a in experts), shared, 2,
                            False)["out"]
    np.testing.assert_array_equal(got, only_shared)


@pytest.mark.parametrize("renorm", [True, False])
def test_selection_only_bias_layer_equals_bruteforce(renorm):
    rng = np.random.default_rng(23)
    T, d, f, n, k, ns = 8, 5, 4, 6, 2, 1
    x, W_g, b, experts, shared = _tiny(rng, T, d, f, n, ns, bias=True)
    b = b * 3.0                     # large enough to change some selections
    ref = moe_layer_dense_bruteforce(x, W_g, b, *experts, shared, k, renorm,
                                     bias_selection_only=True)
    got = moe_layer(x, W_g, b, experts, shared, k, renorm, bias_selection_only=True)["out"]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # and it differs from the logit-bias layer (the bias really left the gates)
    logit = moe_layer(x, W_g, b, experts, shared, k, renorm)["out"]
    assert np.abs(logit - got).max() > 1e-6
