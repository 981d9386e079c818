"""Plain fp64 CPU oracle of the MoE feed-forward layer with shared and fine-grained
routed experts.

TEST INFRASTRUCTURE ONLY. The test suite, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` are the only code allowed to import or run
this module. The product path (the CUDA library and its Python binding) never
touches it, and this module imports nothing from the product package. It is slow
on purpose: every step is the plain definition, written so that it can be checked
against the pages by eye.

Sources, cited by page title and section:

* [SFE]  "Shared and fine-grained experts" (learn.pranaymahendrakar.com):
  Developer "Counting the combinations", "Reading the output", the granularity
  table; Researcher "Why segmentation helps", "Why shared experts help".
* [CAGI] "MoE：细粒度专家与共享专家（shared expert）" (cooking-agi):
  the budget section "先把“预算一样”算明白" and the shared-expert section.
* [WIE]  "What is an “expert,” really?" (svac-llc): glossary entries
  router / gate, top-k, softmax; panel 2.
* [DSV3] "Shared Expert (DeepSeek-V3)" (ai-engineer-exhaustive): "How it works",
  eq. (12) and the SwiGLU definition; "Official code"; "Watch-outs".

The layer (DSV3 eq. (12) without its residual term; the residual is added by the
caller at block level, DSV3 "How it works"):

    out_t = sum_{s<N_s} FFN_s(u_t) + sum_{i<N_r} g_{i,t} FFN_i(u_t)
    FFN(u) = W2 ( SiLU(W1 u) * (W3 u) )

Readings taken where the pages leave a step open:

* Router order: softmax over all N_r scores, then top-k, then (optionally) the
  selected probabilities are renormalised to sum to one.
* Ties in top-k go to the lower expert index; the slots are written in
  descending probability, ties again toward the lower index.
* An optional per-expert logit bias is added to the scores before the softmax.
* N_s shared experts are one fused SwiGLU of inner width N_s*f, which equals the
  sum of the N_s separate experts (DSV3 "Official code", "Watch-outs").
* The routed rows are grouped by expert in ascending (token, slot) order.
* Bias placement: by default the per-expert bias is a logit bias (it moves both
  the selection and the gates). The selection-only variant (the survey's
  "selection-only load-balance bias"; DSV3 "How it works" names a load-balance
  bias on the routed centroids without defining it) adds the bias to the scores
  only to choose the top k; the gates are then the softmax of the unbiased
  scores over all N_r experts (raw), or those probabilities renormalised over
  the selected set. Ties in the biased scores go to the lower index.
* Capacity (token dropping, WIE glossary "capacity factor / token dropping":
  each expert has a seat limit per batch, overflow tokens are skipped): with a
  limit of C seats, an expert keeps the first C (token, slot) pairs routed to it
  in batch order, i.e. ascending (token, slot); a dropped pair adds nothing to
  its token's output, the kept gates are not renormalised, and the shared
  expert still applies to every token.

Every function below is pinned by tests under ``tests/`` against values the
pages print, closed forms, library routines, or brute force on tiny inputs; the
pin for each is named in its docstring. No function here is "parity unpinned".
"""
from __future__ import annotations

from math import comb
from typing import Callable, Optional, Sequence, Tuple, Union

import numpy as np

__all__ = [
    "expert_budget",
    "route_combinations",
    "granularity_rows",
    "layer_accounting",
    "silu",
    "swiglu_ffn",
    "router_scores",
    "softmax_rows",
    "select_topk",
    "gate_values",
    "routing_probabilities",
    "route_permutation",
    "topk_gap",
    "moe_layer",
    "moe_layer_dense_bruteforce",
]


# ---------------------------------------------------------------------------
# Budget and counting (the arithmetic the pages print)
# ---------------------------------------------------------------------------

def expert_budget(width: int, intermediate: int, routed: int, top_k: int,
                  shared: int = 0) -> Tuple[int, int]:
    """Parameter and per-token MAC budget of an expert layer.

    [CAGI] budget section: a SwiGLU expert with hidden size d and inner width f
    holds 3*d*f weights (gate, up, down; no bias) and costs as many MACs per token.
    All N_r routed + N_s shared experts are stored; k routed + N_s shared run per
    token. A configuration with any of d, f, N_r, k below 1, with N_s below 0 or
    with k above N_r is rejected with ValueError.

    Pinned by the page's equality of three budgets and the 221,184 figure
    (tests/golden/expert_budget.txt).
    """
    if min(width, intermediate, routed, top_k) < 1 or shared < 0 or top_k > routed:
        raise ValueError("Invalid expert configuration")
    per_expert = 3 * width * intermediate
    return per_expert * (routed + shared), per_expert * (top_k + shared)


def route_combinations(n_experts: int, top_k: int) -> int:
    """Number of distinct expert sets a top-k router can pick: C(N, K).

    [SFE] Researcher "Why segmentation helps": the reachable function class is
    indexed by the selected set, so its size is C(N, K). Pinned by the values the
    pages print (tests/golden/combinations.txt).
    """
    return comb(n_experts, top_k)


def granularity_rows(base_ff: int, n0: int, k0: int,
                     factors: Sequence[int]) -> list:
    """Fine-grained segmentation rows (m, N, K, expert ff, active ff, C(N,K)).

    [SFE] Developer "Counting the combinations" and Researcher "Why segmentation
    helps": splitting by m gives m*N experts, m*K active, expert width ff/m, so
    the active width K*ff stays fixed while C(mN, mK) grows. Pinned by the printed
    table and the m=16 width of 896 (tests/golden/granularity.txt).
    """
    rows = []
    for m in factors:
        n, k = n0 * m, k0 * m
        ff = base_ff // m
        rows.append((m, n, k, ff, k * ff, route_combinations(n, k)))
    return rows


def layer_accounting(hidden: int, moe_ff: int, n_routed: int, n_shared: int,
                     top_k: int) -> dict:
    """Per-layer parameter accounting of a shared + routed MoE layer.

    [SFE] Developer "DeepSeek-V3 feed-forward accounting": every expert is 3*h*f
    weights; the router adds h*N_r weights, counted both in the total and in the
    active set; active = (k + N_s) experts + router. Pinned by the printed
    DeepSeek-V3 figures (tests/golden/dsv3_accounting.txt).
    """
    per_expert = 3 * hidden * moe_ff
    router = hidden * n_routed
    total = (n_routed + n_shared) * per_expert + router
    active = (top_k + n_shared) * per_expert + router
    return {
        "per_expert": per_expert,
        "total": total,
        "active": active,
        "active_fraction": active / total,
        "shared_params": n_shared * per_expert,
        "shared_share_of_active_experts": n_shared / (top_k + n_shared),
    }


# ---------------------------------------------------------------------------
# The layer, step by step
# ---------------------------------------------------------------------------

def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def silu(z) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)).

    [DSV3] "How it works", the SwiGLU definition names SiLU as the gate
    activation. Pinned by scipy.special.expit and by the identity
    SiLU(-z) = SiLU(z) - z (tests/test_oracle_math.py).
    """
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_ffn(u, W1, W3, W2) -> np.ndarray:
    """FFN(u) = W2 (SiLU(W1 u) * (W3 u)) for a batch of rows u (n, d).

    [DSV3] "How it works", SwiGLU definition. Layouts: W1, W3 are (f, d) (gate and
    up projections), W2 is (d, f) (down projection); u is (n, d); result (n, d).
    Pinned by a hand-derived tiny example and by brute-force element loops
    (tests/test_oracle_math.py, tests/test_oracle_layer.py).
    """
    u, W1, W3, W2 = _f64(u), _f64(W1), _f64(W3), _f64(W2)
    gate = u @ W1.T            # (n, f)
    up = u @ W3.T              # (n, f)
    return (silu(gate) * up) @ W2.T   # (n, d)


def router_scores(x, W_g, bias=None) -> np.ndarray:
    """Router scores s[t, e] = x_t . W_g[e] (+ bias[e]).

    [WIE] glossary "router / gate" and panel 2: a linear layer scores every expert
    for the token; [DSV3] "How it works" calls the rows of W_g the routed experts'
    centroids. The optional per-expert bias is added to the score. Pinned through
    the routing tests (a dominant bias forces its expert; duplicate rows tie).
    """
    s = _f64(x) @ _f64(W_g).T
    if bias is not None:
        s = s + _f64(bias)[None, :]
    return s


def softmax_rows(s) -> np.ndarray:
    """Row-wise softmax, max-subtracted: p = exp(s - max) / sum exp(s - max).

    [WIE] glossary "softmax": raw scores become fractions that add to 1, the
    router's blend weights. Pinned by scipy.special.softmax, by uniform output for
    equal scores and by shift invariance (tests/test_oracle_math.py).
    """
    s = _f64(s)
    z = np.exp(s - s.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def select_topk(p, top_k: int) -> np.ndarray:
    """Indices of the top-k experts per token, ties toward the lower index.

    [WIE] glossary "top-k" and panel 2: the router keeps the k best-scoring
    experts. Slot j of row t holds the (j+1)-th largest probability; equal values
    are ordered by ascending expert index, so the lower index wins both the
    selection and the slot. Returns int64 (T, k).

    Pinned by brute force over all k-subsets (the top-k set maximises the sum of
    probabilities) and by constructed ties (tests/test_oracle_routing.py).
    """
    p = _f64(p)
    T, n = p.shape
    if not 1 <= top_k <= n:
        raise ValueError("top_k must lie in [1, N_r]")
    out = np.empty((T, top_k), dtype=np.int64)
    experts = np.arange(n)
    for t in range(T):
        # lexsort sorts by the last key first: descending p, then ascending index
        order = np.lexsort((experts, -p[t]))
        out[t] = order[:top_k]
    return out


def gate_values(p, idx, renorm: bool) -> np.ndarray:
    """Gate g_{i,t} for the selected experts, in slot order, shape (T, k).

    [WIE] panel 2: the selected experts' outputs are blended by the router's
    weights; [SFE] "Why segmentation helps": g_i is non-zero only inside the
    selected set. With renorm the selected probabilities are divided by their sum
    (equal to a softmax over the selected scores); without it the gate is the raw
    softmax probability. Pinned by "renormalised gates sum to 1" and by the raw
    gates equalling p (tests/test_oracle_routing.py).
    """
    p = _f64(p)
    idx = np.asarray(idx)
    g = np.take_along_axis(p, idx, axis=1)
    if renorm:
        g = g / g.sum(axis=1, keepdims=True)
    return g


def route_permutation(idx, n_routed: int, capacity: Optional[int] = None):
    """Group the (token, slot) pairs by expert in stable (token, slot) order.

    [DSV3] "How it works": routed outputs are scatter-summed back into the full
    packed batch, so each expert processes the rows of the tokens routed to it.
    Returns (counts (N_r,), offsets (N_r+1,), perm_src (R,), inv_pos (T, k)):
    counts[e] is the number of pairs routed to expert e; expert e owns rows
    offsets[e] .. offsets[e+1]-1 of the grouped batch, row r of it holds token
    perm_src[r], and slot j of token t lands in row inv_pos[t, j].

    ``capacity`` (None: unlimited) is the seat limit per expert of [WIE]
    glossary "capacity factor / token dropping": expert e keeps its first
    min(counts[e], capacity) pairs in (token, slot) order, the others are
    dropped (inv_pos -1, no row); offsets then count kept rows and R is their
    total.

    Pinned by a brute-force bucket sort, the bijection / sum invariants and a
    seat-by-seat loop for the capacity (tests/test_oracle_routing.py).
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=n_routed).astype(np.int64)
    # stable sort of the flat (t, j) entries by expert keeps (t, j) order inside a group
    order = np.argsort(flat, kind="stable")
    starts = np.zeros(n_routed, dtype=np.int64)
    starts[1:] = np.cumsum(counts)[:-1]
    rank = np.empty(T * k, dtype=np.int64)             # position inside its expert's group
    rank[order] = np.arange(T * k) - starts[flat[order]]
    kept = np.ones(T * k, dtype=bool) if capacity is None else rank < capacity
    kept_counts = counts if capacity is None else np.minimum(counts, capacity)
    offsets = np.zeros(n_routed + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept_counts)
    order_kept = order[kept[order]]
    perm_src = order_kept // k
    inv_flat = np.full(T * k, -1, dtype=np.int64)
    inv_flat[order_kept] = np.arange(order_kept.size)
    return counts, offsets, perm_src, inv_flat.reshape(T, k)


def topk_gap(p, top_k: int) -> np.ndarray:
    """Smallest gap between consecutive probabilities among the top k+1 of each token.

    Used to find tokens whose selection (or slot order) is not unique within a
    tolerance: a gap below the tolerance means two orders are equally correct.
    With k = N_r only the gaps inside the selection exist. Pinned by a direct
    small example (tests/test_oracle_routing.py).
    """
    p = _f64(p)
    n = p.shape[1]
    m = min(top_k + 1, n)
    srt = -np.sort(-p, axis=1)[:, :m]
    if m < 2:
        return np.full(p.shape[0], np.inf)
    return np.min(srt[:, :-1] - srt[:, 1:], axis=1)


ExpertSource = Union[Tuple[np.ndarray, np.ndarray, np.ndarray],
                     Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]]


def _expert_getter(experts: ExpertSource):
    if callable(experts):
        return experts
    W1, W3, W2 = experts
    return lambda e: (W1[e], W3[e], W2[e])


def routing_probabilities(x, W_g, bias, bias_selection_only: bool = False):
    """(p_select, p_gate): the probabilities the top-k ranks and the ones the gates
    take. With a logit bias (default) both are softmax(x W_g^T + b); with a
    selection-only bias p_select = softmax(x W_g^T + b) and p_gate = softmax(x W_g^T).
    Ranking by softmax(s + b) is ranking by s + b (softmax is increasing).
    Pinned by tests/test_oracle_routing.py (a forcing bias keeps the unbiased gate;
    no bias makes both modes equal) and by the scalar brute force.
    """
    p_sel = softmax_rows(router_scores(x, W_g, bias))
    if not bias_selection_only or bias is None:
        return p_sel, p_sel
    return p_sel, softmax_rows(router_scores(x, W_g, None))


def moe_layer(x, W_g, bias, experts: ExpertSource, shared, top_k: int, renorm: bool,
              tokens: Optional[Sequence[int]] = None,
              forced_idx: Optional[np.ndarray] = None,
              capacity: Optional[int] = None,
              bias_selection_only: bool = False) -> dict:
    """Forward pass of the layer: shared + sum of gated routed experts, no residual.

    [DSV3] eq. (12) without u_t, "Official code": route, run every expert on the
    rows routed to it, add the always-on shared SwiGLU (coefficient 1, outside the
    top-k pool) computed on the whole batch.

    Arguments: x (T, d); W_g (N_r, d); bias (N_r,) or None; ``experts`` either the
    stacked (W1 (N_r,f,d), W3 (N_r,f,d), W2 (N_r,d,f)) or a callable e -> the
    three matrices of expert e (so that large layers can be streamed one expert at
    a time); ``shared`` None or (W1s (N_s f, d), W3s (N_s f, d), W2s (d, N_s f)).
    ``tokens`` restricts the output rows computed (routing always covers all T).
    ``forced_idx`` (T, k) replaces the top-k selection (gates still come from the
    oracle's own probabilities); it is how a second correct selection is scored.
    ``capacity`` (None: unlimited) is the per-expert seat limit of
    ``route_permutation``: dropped (token, slot) pairs add nothing.
    ``bias_selection_only`` moves the bias out of the gates (see
    ``routing_probabilities``); the returned p is the gate probability.

    Returns a dict with p, idx, g, counts, offsets, perm_src, inv_pos, tokens and
    out (len(tokens), d) in fp64. Pinned by the dense brute force on tiny inputs,
    by the special cases k = N_r and N_r = 1, and by the shared-term invariants
    (tests/test_oracle_layer.py).
    """
    x = _f64(x)
    T, d = x.shape
    n_routed = np.asarray(W_g).shape[0]
    p_sel, p = routing_probabilities(x, W_g, bias, bias_selection_only)
    if forced_idx is None:
        idx = select_topk(p_sel, top_k)
    else:
        idx = np.asarray(forced_idx, dtype=np.int64)
        assert idx.shape == (T, top_k)
    g = gate_values(p, idx, renorm)
    counts, offsets, perm_src, inv_pos = route_permutation(idx, n_routed, capacity)
    kept = inv_pos >= 0

    rows = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    out = np.zeros((len(rows), d), dtype=np.float64)
    if shared is not None:
        W1s, W3s, W2s = shared
        out += swiglu_ffn(x[rows], W1s, W3s, W2s)

    get = _expert_getter(experts)
    # (row in out, slot) pairs per expert, restricted to the requested tokens
    sel_rows = idx[rows]                                   # (R, k)
    kept_rows = kept[rows]
    for e in range(n_routed):
        hit_r, hit_j = np.nonzero((sel_rows == e) & kept_rows)
        if hit_r.size == 0:
            continue
        W1e, W3e, W2e = get(e)
        y = swiglu_ffn(x[rows[hit_r]], W1e, W3e, W2e)     # (n_e, d)
        out[hit_r] += g[rows[hit_r], hit_j][:, None] * y
    return {"p": p, "idx": idx, "g": g, "counts": counts, "offsets": offsets,
            "perm_src": perm_src, "inv_pos": inv_pos, "tokens": rows, "out": out}


def moe_layer_dense_bruteforce(x, W_g, bias, W1, W3, W2, shared, top_k: int,
                               renorm: bool, capacity: Optional[int] = None,
                               bias_selection_only: bool = False) -> np.ndarray:
    """Brute-force evaluation for tiny inputs: every expert on every token.

    [SFE] "Why segmentation helps": the layer is sum_{i in S} g_i E_i(x), i.e. a
    dense sum over all experts weighted by a gate matrix that is zero outside the
    selected set. This version uses plain Python loops over scalars (no matrix
    products, no sorting routine) so that it shares no formulation with
    ``moe_layer``: the selection is found by repeatedly taking the first maximum,
    each expert's SwiGLU is summed element by element. With a ``capacity``, the
    seats are handed out pair by pair in (token, slot) order ([WIE] glossary
    "capacity factor / token dropping") and a pair without a seat is skipped.
    With ``bias_selection_only`` the biased scores choose the experts and the
    gates come from the unbiased scores.
    """
    import math

    x = [[float(v) for v in row] for row in np.asarray(x, dtype=np.float64)]
    Wg = np.asarray(W_g, dtype=np.float64)
    W1 = np.asarray(W1, dtype=np.float64)
    W3 = np.asarray(W3, dtype=np.float64)
    W2 = np.asarray(W2, dtype=np.float64)
    T, d = len(x), len(x[0])
    n_routed = W1.shape[0]

    def expert_out(u, A1, A3, A2):
        inner = len(A1)
        h = []
        for i in range(inner):
            a = sum(A1[i][c] * u[c] for c in range(d))
            b = sum(A3[i][c] * u[c] for c in range(d))
            h.append(a / (1.0 + math.exp(-a)) * b)
        return [sum(A2[c][i] * h[i] for i in range(inner)) for c in range(d)]

    out = np.zeros((T, d), dtype=np.float64)
    seats_used = [0] * n_routed
    for t in range(T):
        raw = [sum(Wg[e][c] * x[t][c] for c in range(d)) for e in range(n_routed)]
        scores = [raw[e] + (float(bias[e]) if bias is not None else 0.0)
                  for e in range(n_routed)]

        def probs(v):
            mx = max(v)
            ex = [math.exp(a - mx) for a in v]
            tot = sum(ex)
            return [a / tot for a in ex]

        prob_sel = probs(scores)
        prob = probs(raw) if bias_selection_only else prob_sel
        chosen = []
        for _ in range(top_k):
            best = None
            for e in range(n_routed):      # first maximum wins: lower index on ties
                if e in chosen:
                    continue
                if best is None or prob_sel[e] > prob_sel[best]:
                    best = e
            chosen.append(best)
        G = [0.0] * n_routed
        norm = sum(prob[e] for e in chosen) if renorm else 1.0
        for e in chosen:                   # slots in order; a full expert skips the pair
            if capacity is not None:
                if seats_used[e] >= capacity:
                    continue
                seats_used[e] += 1
            G[e] = prob[e] / norm
        acc = [0.0] * d
        for e in range(n_routed):          # dense over all experts
            y = expert_out(x[t], W1[e], W3[e], W2[e])
            for c in range(d):
                acc[c] += G[e] * y[c]
        if shared is not None:
            W1s, W3s, W2s = (np.asarray(a, dtype=np.float64) for a in shared)
            ys = expert_out(x[t], W1s, W3s, W2s)
            for c in range(d):
                acc[c] += ys[c]
        out[t] = acc
    return out
