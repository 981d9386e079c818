"""The oracle's counting and budget helpers against the values the pages print.

Every expected number here is read from a fixture under tests/golden/, each of
which cites the page and section that prints it.
"""
import pytest

from oracle import expert_budget, granularity_rows, layer_accounting, route_combinations

from conftest import read_golden


def test_expert_budget_matches_printed_values():
    rows = read_golden("expert_budget.txt")
    assert len(rows) == 4
    for width, inter, routed, topk, shared, params, active in rows:
        got = expert_budget(int(width), int(inter), int(routed), int(topk), int(shared))
        if params != "-":
            assert got[0] == int(params)
        assert got[1] == int(active)


def test_equal_budget_configs_are_equal():
    # the three equal-budget shapes of the budget section give one identical pair
    rows = read_golden("expert_budget.txt")[:3]
    vals = {expert_budget(*(int(v) for v in r[:5])) for r in rows}
    assert vals == {(786432, 196608)}


@pytest.mark.parametrize("row", read_golden("invalid_budget.txt"))
def test_expert_budget_rejects_invalid(row):
    with pytest.raises(ValueError):
        expert_budget(*(int(v) for v in row))


@pytest.mark.parametrize("row", read_golden("combinations.txt"))
def test_route_combinations_match_printed(row):
    n, k, c = (int(v) for v in row)
    assert route_combinations(n, k) == c


def test_granularity_table_matches_printed():
    rows = read_golden("granularity.txt")
    got = granularity_rows(14336, 16, 2, [int(r[0]) for r in rows])
    for want, have in zip(rows, got):
        m, n, k, ff, active, comb = want
        assert have[0] == int(m) and have[1] == int(n) and have[2] == int(k)
        assert have[3] == int(ff)
        if active != "-":
            assert have[4] == int(active)
        if comb != "-":
            assert have[5] == int(comb)


def test_active_width_invariant_under_segmentation():
    # "Reading the output": 28,672 at every granularity of the printed table
    rows = granularity_rows(14336, 16, 2, [1, 2, 4, 8])
    assert {r[4] for r in rows} == {28672}


def test_dsv3_accounting_matches_printed():
    want = {r[0]: r[1] for r in read_golden("dsv3_accounting.txt")}
    acc = layer_accounting(7168, 2048, 256, 1, 8)
    assert acc["per_expert"] == int(want["per_expert"])
    assert acc["total"] == int(want["total"])
    assert acc["active"] == int(want["active"])
    assert f"{acc['active_fraction'] * 100:.2f}" == want["active_percent"]
    assert acc["shared_params"] == int(want["shared_params"])
    assert f"{acc['shared_share_of_active_experts'] * 100:.0f}" == want["shared_percent"]
