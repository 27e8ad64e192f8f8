"""Pins of the staircase cost reading and the asynchronous budget mode of
the prefix cut (oracle only).

- the staircase lookup on hand-picked token counts (an off-by-one in the
  ceiling lookup, a wrong extension past the table);
- a budget commits exactly the top candidates of the current survival order
  (numpy lexsort; a cut taken by request, by position or in the wrong
  order fails);
- the greedy's own N as budget reproduces the greedy cut, and the greedy
  output is unchanged by any budget (the budget only chooses the cut);
- budgets past both ends clamp; every cut is a prefix of each draft;
- on a staircase table the greedy stops exactly at a stair edge when the
  next stair costs more than the tokens it adds.
"""
import numpy as np
import pytest

from speculative_decoding_05_b200 import workloads as WL


def table():
    xs, ys = WL.cost_table()
    return xs.numpy(), ys.numpy()


def survivals(z, temps):
    c = 1.0 / (1.0 + np.exp(-z.astype(np.float64) / temps.astype(np.float64)))
    return np.cumprod(c, axis=1)


def test_staircase_lookup_hand_values(oracle_mod):
    xs = np.array([0, 512, 1024, 1536], np.float32)
    ys = np.array([20, 22, 24, 30], np.float32)
    f = lambda n: oracle_mod.cost_stair_ms(xs, ys, n)
    assert f(0) == 20 and f(-3) == 20
    assert f(1) == 22 and f(512) == 22 and f(512.5) == 24
    assert f(1024) == 24 and f(1025) == 30 and f(1536) == 30
    assert f(1536 + 256) == pytest.approx(30 + 6 * 256 / 512)  # last segment's slope
    # the linear reading on the same table differs inside a stair
    assert oracle_mod.cost_ms(xs, ys, 256) == pytest.approx(21.0)


@pytest.mark.parametrize("staircase", [False, True])
@pytest.mark.parametrize("seed", [0, 1])
def test_budget_commits_the_top_candidates(oracle_mod, staircase, seed):
    rng = np.random.default_rng(seed)
    B, K = 40, 6
    z = rng.normal(1.5, 1.0, (B, K)).astype(np.float32)
    temps = WL.seq_temps(K).numpy()
    xs, ys = table()
    S = survivals(z, temps)
    b_idx, k_idx = np.meshgrid(np.arange(B), np.arange(K), indexing="ij")
    order = np.lexsort((b_idx.ravel(), k_idx.ravel(), -S.ravel()))  # S desc, k asc, b asc
    for budget in (B, B + 1, B + 37, B + 111, B + B * K - 1):
        r = oracle_mod.prefix_async(z, temps, xs, ys, staircase=staircase, budget=budget)
        top = order[: budget - B]
        L = np.bincount(b_idx.ravel()[top], minlength=B)
        assert np.array_equal(r["L"], L)
        assert r["L"].sum() == budget - B
        # every cut is a prefix of each request's draft
        for b in range(B):
            kk = k_idx.ravel()[top][b_idx.ravel()[top] == b]
            assert np.array_equal(np.sort(kk), np.arange(len(kk)))


@pytest.mark.parametrize("staircase", [False, True])
def test_greedy_budget_reproduces_greedy(oracle_mod, staircase):
    rng = np.random.default_rng(7)
    B, K = 256, 6
    z = rng.normal(1.5, 1.0, (B, K)).astype(np.float32)
    temps = WL.seq_temps(K).numpy()
    xs, ys = table()
    g = oracle_mod.prefix_async(z, temps, xs, ys, staircase=staircase)
    r = oracle_mod.prefix_async(z, temps, xs, ys, staircase=staircase, budget=g["n_greedy"])
    assert np.array_equal(g["L"], r["L"]) and g["objective"] == r["objective"]
    assert g["n_greedy"] == B + g["L"].sum()
    other = oracle_mod.prefix_async(z, temps, xs, ys, staircase=staircase, budget=B + 5)
    assert other["n_greedy"] == g["n_greedy"]
    # the plain entry point is the linear, budget-free case
    if not staircase:
        p = oracle_mod.prefix(z, temps, xs, ys)
        assert np.array_equal(p["L"], g["L"]) and p["objective"] == g["objective"]


def test_budgets_clamp(oracle_mod):
    rng = np.random.default_rng(3)
    B, K = 10, 4
    z = rng.normal(1.5, 1.0, (B, K)).astype(np.float32)
    temps = WL.seq_temps(K).numpy()
    xs, ys = table()
    lo = oracle_mod.prefix_async(z, temps, xs, ys, budget=0)
    hi = oracle_mod.prefix_async(z, temps, xs, ys, budget=10 ** 6)
    assert np.all(lo["L"] == 0) and np.all(hi["L"] == K)


def test_staircase_greedy_stops_at_a_stair_edge(oracle_mod):
    # 8 requests with near-certain drafts; stairs of 16 tokens.  The second
    # stair costs 1.5x the first, so on the staircase E/t falls when the
    # 17th token is added (17 / 1.5 < 16), while the linear reading of the
    # same points charges the 17th token only 1/32 ms and keeps going.
    B, K = 8, 4
    z = np.full((B, K), 30.0, np.float32)  # c ~ 1, survival ~ 1
    temps = np.ones(K, np.float32)
    xs = np.array([0, 16, 32, 48], np.float32)
    ys = np.array([1, 1, 1.5, 3], np.float32)
    r = oracle_mod.prefix_async(z, temps, xs, ys, staircase=True)
    assert r["n_greedy"] == 16 and r["L"].sum() == 8
    # the linear reading of the same table has no such edge at 16
    lin = oracle_mod.prefix_async(z, temps, xs, ys, staircase=False)
    assert lin["n_greedy"] > 16
