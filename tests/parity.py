"""Shared GPU-vs-oracle parity checks (imported by the gpu tests and smoke()).

The acceptance rule: selected expert sets bit-exact wherever the oracle's k-th
and (k+1)-th probabilities (and, for the slot order, any two consecutive
selected ones) differ by more than 1e-5; counts and offsets bit-exact; the
output within relative-L2 1e-2 and max-abs 2e-2 * max|ref| (bf16 storage with
fp32 accumulation). Where several selections are correct (a near tie), the
GPU's choice is checked for validity and then scored by the oracle itself.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import (moe_layer, route_permutation, router_scores, routing_probabilities,
                    select_topk, softmax_rows)

TIE_TOL = 1e-5
REL_L2_TOL = 1e-2
MAX_ABS_TOL = 2e-2
GATE_TOL = 1e-4


def to64(t):
    return None if t is None else t.detach().to(torch.float64).cpu().numpy()


def reconcile_routing(p: np.ndarray, gpu_idx: np.ndarray, k: int, tol: float = TIE_TOL):
    """Oracle selection with near-tie tokens replaced by the GPU's (validated) choice.

    Returns (idx_ref, n_near_tie). Raises AssertionError on any mismatch that the
    tie rule does not excuse."""
    T, n = p.shape
    oracle_idx = select_topk(p, k)
    srt = -np.sort(-p, axis=1)
    m = min(k + 1, n)
    gaps = srt[:, :m - 1] - srt[:, 1:m] if m >= 2 else np.full((T, 0), np.inf)
    near = (gaps <= tol).any(axis=1) if gaps.shape[1] else np.zeros(T, bool)
    idx_ref = oracle_idx.copy()
    exact = ~near
    bad = np.nonzero(exact & (gpu_idx != oracle_idx).any(axis=1))[0]
    assert bad.size == 0, (f"{bad.size} tokens select different experts without a near tie; "
                           f"first t={bad[0]}: gpu={gpu_idx[bad[0]]} oracle={oracle_idx[bad[0]]}")
    for t in np.nonzero(near)[0]:
        row = gpu_idx[t]
        assert len(set(row.tolist())) == k and row.min() >= 0 and row.max() < n, \
            f"token {t}: invalid selection {row}"
        pk = srt[t, k - 1]
        assert np.all(p[t, row] >= pk - tol), f"token {t}: {row} is not a top-{k} set within {tol}"
        assert np.all(np.diff(p[t, row]) <= tol), f"token {t}: slots not in descending order"
        idx_ref[t] = row
    return idx_ref, int(near.sum())


def check_routing(inp, gpu, shape, T=None, capacity=None, bias_selection_only=False):
    """Routing parity on every token. Returns (p, idx_ref, n_near_tie). With an
    expert capacity only the kept rows of perm_src are defined. The near-tie rule
    applies to the probabilities the selection ranks; the gates are compared with
    the gate probabilities (different only for a selection-only bias)."""
    x = to64(inp["x"])
    p_sel, p = routing_probabilities(x, to64(inp["W_g"]), to64(inp["bias"]), bias_selection_only)
    gpu_idx = gpu["idx"].cpu().numpy().astype(np.int64)
    idx_ref, n_near = reconcile_routing(p_sel, gpu_idx, shape.top_k)
    counts, offsets, perm_src, inv_pos = route_permutation(idx_ref, shape.n_routed, capacity)
    np.testing.assert_array_equal(gpu["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(gpu["offsets"].cpu().numpy(), offsets)
    np.testing.assert_array_equal(gpu["perm_src"].cpu().numpy()[:perm_src.size], perm_src)
    np.testing.assert_array_equal(gpu["inv_pos"].cpu().numpy(), inv_pos)
    g = np.take_along_axis(p, idx_ref, 1)
    if shape.renorm:
        g = g / g.sum(1, keepdims=True)
    # fp32 scores summed over d bf16 products on the tensor core drift by ~1e-5;
    # a gate error of 1e-4 moves the output far less than its 1e-2 tolerance
    np.testing.assert_allclose(gpu["w"].cpu().numpy(), g, rtol=0, atol=GATE_TOL)
    return p, idx_ref, n_near


def oracle_out(inp, shape, idx_ref, tokens=None, capacity=None, bias_selection_only=False):
    """Oracle output for `tokens` (all when None), streaming one expert at a time."""
    W1, W3, W2 = inp["W1"], inp["W3"], inp["W2"]

    def expert(e):
        return to64(W1[e]), to64(W3[e]), to64(W2[e])

    shared = None
    if shape.n_shared > 0:
        shared = (to64(inp["W1s"]), to64(inp["W3s"]), to64(inp["W2s"]))
    r = moe_layer(to64(inp["x"]), to64(inp["W_g"]), to64(inp["bias"]), expert, shared,
                  shape.top_k, shape.renorm, tokens=tokens, forced_idx=idx_ref,
                  capacity=capacity, bias_selection_only=bias_selection_only)
    return r["out"]


def output_errors(gpu_out: np.ndarray, ref: np.ndarray):
    diff = gpu_out - ref
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    return rel_l2, max_abs, scale


def check_output(gpu_out: np.ndarray, ref: np.ndarray):
    rel_l2, max_abs, scale = output_errors(gpu_out, ref)
    assert np.all(np.isfinite(gpu_out)), "non-finite GPU output"
    assert rel_l2 <= REL_L2_TOL, f"relative L2 error {rel_l2:.3e} > {REL_L2_TOL}"
    assert max_abs <= MAX_ABS_TOL * scale, \
        f"max-abs error {max_abs:.3e} > {MAX_ABS_TOL} * max|ref| = {MAX_ABS_TOL * scale:.3e}"
    return rel_l2, max_abs, scale


def run_layer(inp, shape, device="cuda", pair_min_rows=None, wide_tiles=None, merge_shared=None,
              capacity=None, bias_selection_only=False, fused_router=None, **kernel_options):
    """Run the CUDA layer through the C ABI; returns (out (T,d) fp64 numpy, routing dict)."""
    from mixture_experts_ffn_expert_b200.layer import MoELayer

    layer = MoELayer(shape.d, shape.f, shape.n_routed, shape.top_k, shape.n_shared,
                     shape.renorm, {k: inp[k] for k in ("W_g", "W1", "W3", "W2", "W1s",
                                                        "W3s", "W2s")},
                     bias=inp["bias"], device=device, pair_min_rows=pair_min_rows,
                     wide_tiles=wide_tiles, merge_shared=merge_shared, capacity=capacity,
                     bias_selection_only=bias_selection_only, fused_router=fused_router,
                     **kernel_options)
    out = layer(inp["x"])
    routing = layer.routing()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return out, routing, layer


def full_parity(inp, shape, tokens=None, pair_min_rows=None, wide_tiles=None,
                merge_shared=None, capacity=None, bias_selection_only=False, fused_router=None,
                **kernel_options):
    """Routing on all tokens, output on `tokens` (all when None). Returns a summary dict.
    pair_min_rows forces (0) or forbids (huge) the CTA-pair GEMM kernel; wide_tiles
    forces (1) or forbids (0) its 512-column tiles; merge_shared forces (1) or
    forbids (0) the shared expert as extra tiles of the routed GEMM launches;
    capacity sets the seats per expert (token dropping); bias_selection_only keeps
    the bias out of the gates; fused_router 0 forces the two-kernel router; the
    other keyword arguments are MoELayer kernel options (tile_rows, ctas_per_sm, ...)."""
    out, routing, layer = run_layer(inp, shape, pair_min_rows=pair_min_rows,
                                    wide_tiles=wide_tiles, merge_shared=merge_shared,
                                    capacity=capacity, bias_selection_only=bias_selection_only,
                                    fused_router=fused_router, **kernel_options)
    _, idx_ref, n_near = check_routing(inp, routing, shape, capacity=capacity,
                                       bias_selection_only=bias_selection_only)
    ref = oracle_out(inp, shape, idx_ref, tokens, capacity=capacity,
                     bias_selection_only=bias_selection_only)
    got = to64(out if tokens is None else out[torch.as_tensor(tokens, device=out.device)])
    rel_l2, max_abs, scale = check_output(got, ref)
    return {"near_ties": n_near, "rel_l2": rel_l2, "max_abs": max_abs, "max_ref": scale,
            "layer": layer}
