"""The validity check of a prefix cut (tests.parity.cut_problems), pinned on
the CPU against the oracle before any GPU test relies on it.

The GPU tests fall back to this check when the oracle's own stopping
decision lies inside the 1e-6 margin, so it must accept every cut the
method could make and refuse the mistakes a broken sort or scan produces:
a cut far too short, the right number of candidates taken in the wrong
order, a cut that stops while the objective still rises, a budget cut of
the wrong size.
"""
import numpy as np
import pytest

from speculative_decoding_05_b200 import workloads as WL
from tests.parity import cut_problems


def case(seed, B=64, K=8):
    rng = np.random.default_rng(seed)
    z = (rng.standard_normal((B, K)) + 1.5).astype(np.float32)
    temps = WL.seq_temps(K).numpy()
    xs, ys = (t.numpy() for t in WL.cost_table())
    return z, temps, xs, ys


@pytest.mark.parametrize("staircase", [False, True])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_the_oracles_own_cuts_pass(oracle_mod, staircase, seed):
    z, temps, xs, ys = case(seed)
    r = oracle_mod.prefix_async(z, temps, xs, ys, staircase=staircase)
    assert cut_problems(oracle_mod, r["S"], xs, ys, r["L"], staircase=staircase) == []
    for budget in (0, z.shape[0] + 37, r["n_greedy"], 10 ** 6):
        rb = oracle_mod.prefix_async(z, temps, xs, ys, staircase=staircase, budget=budget)
        assert cut_problems(oracle_mod, rb["S"], xs, ys, rb["L"], staircase=staircase,
                            budget=budget) == []


def test_planted_mistakes_are_refused(oracle_mod):
    z, temps, xs, ys = case(4)
    B, K = z.shape
    r = oracle_mod.prefix_async(z, temps, xs, ys)
    S, L = r["S"], r["L"]
    N = int(L.sum())
    assert 4 < N < B * K - 4
    # far too short (what a sort that read stale survivals produced)
    tiny = np.zeros(B, np.int32)
    tiny[:2] = 1
    assert cut_problems(oracle_mod, S, xs, ys, tiny)
    # N candidates, but taken by position then request instead of by survival
    by_id = np.bincount(np.arange(N) % B, minlength=B).astype(np.int32)
    assert not np.array_equal(by_id, L)
    assert cut_problems(oracle_mod, S, xs, ys, by_id)
    # the first half of the same order: a valid order, but the scan stopped
    # while the objective still rose (near the optimum it is flat, so the
    # cut a few candidates early may still be inside the margin)
    kk, bb = np.meshgrid(np.arange(K), np.arange(B))
    order = np.lexsort((bb.ravel(), kk.ravel(), -S.ravel()))
    half = np.bincount(bb.ravel()[order[:N // 2]], minlength=B).astype(np.int32)
    assert cut_problems(oracle_mod, S, xs, ys, half)
    assert cut_problems(oracle_mod, S, xs, ys, half, budget=B + N // 2) == []
    # and past the oracle's cut by a quarter of the rest: it went on past a
    # clear fall
    more = np.bincount(bb.ravel()[order[:N + (B * K - N) // 4]], minlength=B).astype(np.int32)
    assert cut_problems(oracle_mod, S, xs, ys, more)
    # a budget cut of the wrong size
    assert cut_problems(oracle_mod, S, xs, ys, L, budget=B + N + 1)
    # lengths outside [0, K]
    bad = L.copy()
    bad[0] = K + 1
    assert cut_problems(oracle_mod, S, xs, ys, bad)
