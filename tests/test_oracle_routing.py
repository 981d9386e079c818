"""The oracle's router (scores, top-k, gates) and permutation against brute force."""
import itertools

import numpy as np
import pytest

from oracle import (gate_values, route_permutation, router_scores, select_topk,
                    softmax_rows, topk_gap)


@pytest.mark.parametrize("n,k", [(5, 1), (7, 3), (8, 2), (9, 9), (10, 4)])
def test_topk_set_is_the_max_sum_subset(n, k):
    # without ties, the top-k set is the unique k-subset with the largest sum of p
    rng = np.random.default_rng(n * 10 + k)
    p = softmax_rows(rng.normal(size=(12, n)) * 2)
    idx = select_topk(p, k)
    for t in range(p.shape[0]):
        best = max(itertools.combinations(range(n), k), key=lambda S: sum(p[t, list(S)]))
        assert sorted(idx[t]) == sorted(best)
        # slots are in descending probability
        assert np.all(np.diff(p[t, idx[t]]) <= 0)


def test_ties_go_to_lower_index():
    p = np.array([[0.1, 0.3, 0.3, 0.3],
                  [0.25, 0.25, 0.25, 0.25],
                  [0.4, 0.2, 0.2, 0.2]])
    np.testing.assert_array_equal(select_topk(p, 2), [[1, 2], [0, 1], [0, 1]])
    np.testing.assert_array_equal(select_topk(p, 3), [[1, 2, 3], [0, 1, 2], [0, 1, 2]])


def test_duplicate_router_rows_tie_exactly_and_lower_index_wins():
    rng = np.random.default_rng(5)
    d, n = 6, 5
    x = rng.normal(size=(20, d))
    W_g = rng.normal(size=(n, d))
    W_g[3] = W_g[1]                     # experts 1 and 3 always tie
    p = softmax_rows(router_scores(x, W_g))
    assert np.array_equal(p[:, 1], p[:, 3])
    idx = select_topk(p, 2)
    # expert 3 can only appear together with expert 1, in the slot after it
    for row in idx:
        if 3 in row:
            assert list(row).index(1) < list(row).index(3)


def test_bias_is_added_to_scores_and_can_force_an_expert():
    rng = np.random.default_rng(6)
    x = rng.normal(size=(9, 4))
    W_g = rng.normal(size=(6, 4))
    bias = np.zeros(6)
    bias[4] = 100.0
    s = router_scores(x, W_g, bias)
    np.testing.assert_allclose(s - router_scores(x, W_g), np.broadcast_to(bias, s.shape))
    idx = select_topk(softmax_rows(s), 3)
    assert np.all(idx[:, 0] == 4)


def test_gates_raw_and_renormalised():
    rng = np.random.default_rng(7)
    p = softmax_rows(rng.normal(size=(30, 16)))
    idx = select_topk(p, 4)
    raw = gate_values(p, idx, renorm=False)
    np.testing.assert_array_equal(raw, np.take_along_axis(p, idx, 1))
    assert np.all(raw.sum(1) < 1.0)
    ren = gate_values(p, idx, renorm=True)
    np.testing.assert_allclose(ren.sum(1), 1.0, rtol=0, atol=1e-12)
    # renormalising equals a softmax over the selected scores only
    s = np.log(p)
    sel = np.take_along_axis(s, idx, 1)
    np.testing.assert_allclose(ren, softmax_rows(sel), rtol=1e-12)


def test_k_equals_n_selects_every_expert():
    rng = np.random.default_rng(8)
    p = softmax_rows(rng.normal(size=(10, 7)))
    idx = select_topk(p, 7)
    for row in idx:
        assert sorted(row) == list(range(7))
    np.testing.assert_allclose(gate_values(p, idx, False).sum(1), 1.0, atol=1e-14)


@pytest.mark.parametrize("T,k,n", [(1, 1, 1), (5, 2, 3), (40, 3, 11), (64, 7, 31), (17, 4, 4)])
def test_permutation_against_bucket_sort(T, k, n):
    rng = np.random.default_rng(T + k + n)
    idx = np.stack([rng.choice(n, size=k, replace=False) for _ in range(T)])
    counts, offsets, perm_src, inv_pos = route_permutation(idx, n)
    # brute force: list the (expert, token, slot) triples and sort them
    triples = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k))
    assert list(perm_src) == [t for (_, t, _) in triples]
    for r, (e, t, j) in enumerate(triples):
        assert inv_pos[t, j] == r
        assert offsets[e] <= r < offsets[e + 1]
    assert counts.sum() == T * k and offsets[-1] == T * k and offsets[0] == 0
    np.testing.assert_array_equal(np.diff(offsets), counts)
    # bijection between (t, j) and rows
    assert sorted(inv_pos.reshape(-1)) == list(range(T * k))
    np.testing.assert_array_equal(perm_src[inv_pos], np.repeat(np.arange(T)[:, None], k, 1))


def test_topk_gap_small_example():
    p = np.array([[0.5, 0.3, 0.15, 0.05], [0.4, 0.3, 0.3, 0.0]])
    np.testing.assert_allclose(topk_gap(p, 2), [0.15, 0.0])
    np.testing.assert_allclose(topk_gap(p, 1), [0.2, 0.1])
    assert np.all(np.isinf(topk_gap(np.ones((2, 1)), 1)))


def _seat_loop(idx, n, capacity):
    """Seats handed out pair by pair in (token, slot) order ([WIE] glossary
    "capacity factor / token dropping"): returns kept mask and, per expert, the
    tokens of its kept pairs in order."""
    used = [0] * n
    rows = [[] for _ in range(n)]
    T, k = idx.shape
    kept = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if used[e] < capacity:
                used[e] += 1
                kept[t, j] = True
                rows[e].append(t)
    return kept, rows


@pytest.mark.parametrize("capacity", [0, 1, 2, 5, 1000])
def test_capacity_keeps_the_first_pairs_in_batch_order(capacity):
    rng = np.random.default_rng(11)
    T, k, n = 60, 3, 7
    # skewed routing so that some experts overflow
    p = rng.dirichlet(np.linspace(4.0, 0.3, n), size=T)
    idx = select_topk(p, k)
    counts, offsets, perm_src, inv_pos = route_permutation(idx, n, capacity)
    kept, rows = _seat_loop(idx, n, capacity)
    np.testing.assert_array_equal(counts, np.bincount(idx.reshape(-1), minlength=n))
    np.testing.assert_array_equal(inv_pos >= 0, kept)
    np.testing.assert_array_equal(np.diff(offsets), [len(r) for r in rows])
    np.testing.assert_array_equal(perm_src, [t for r in rows for t in r])
    assert offsets[-1] == min(T * k, sum(min(c, capacity) for c in counts))
    # kept pairs land on distinct rows of their expert's group, in (t, j) order
    for e in range(n):
        sel = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e and kept[t, j]]
        np.testing.assert_array_equal([inv_pos[t, j] for t, j in sel],
                                      np.arange(offsets[e], offsets[e + 1]))


def test_capacity_at_or_above_the_largest_load_drops_nothing():
    rng = np.random.default_rng(12)
    idx = select_topk(rng.random((40, 6)), 2)
    free = route_permutation(idx, 6)
    capped = route_permutation(idx, 6, int(np.bincount(idx.reshape(-1)).max()))
    for a, b in zip(free, capped):
        np.testing.assert_array_equal(a, b)


def test_selection_only_bias_keeps_the_unbiased_gate():
    # a bias that forces expert 3 into every selection: as a logit bias its gate is
    # ~1, as a selection-only bias the gate is expert 3's unbiased probability
    from oracle import routing_probabilities
    rng = np.random.default_rng(31)
    x = rng.normal(size=(20, 6))
    W_g = rng.normal(size=(5, 6))
    bias = np.array([0.0, 0.0, 0.0, 60.0, 0.0])
    p_sel, p_gate = routing_probabilities(x, W_g, bias, bias_selection_only=True)
    idx = select_topk(p_sel, 2)
    assert np.all(idx[:, 0] == 3)
    unbiased = softmax_rows(router_scores(x, W_g))
    np.testing.assert_array_equal(p_gate, unbiased)
    g = gate_values(p_gate, idx, False)
    np.testing.assert_allclose(g[:, 0], unbiased[:, 3], rtol=0, atol=0)
    assert np.all(g[:, 0] < 0.99)
    p_logit, p_logit_gate = routing_probabilities(x, W_g, bias)
    assert p_logit is p_logit_gate and np.all(p_logit[:, 3] > 0.999)


def test_selection_only_without_bias_is_the_plain_router():
    from oracle import routing_probabilities
    rng = np.random.default_rng(32)
    x, W_g = rng.normal(size=(7, 4)), rng.normal(size=(6, 4))
    a = routing_probabilities(x, W_g, None, bias_selection_only=True)
    b = routing_probabilities(x, W_g, None)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
