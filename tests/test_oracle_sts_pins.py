"""Pins of the sequential-temperature-scaling oracle (fit and ECE).

What each test fixes, and which plausible mistake it catches:
- a large logistic sample recovers the temperatures that generated it
  (sign or reciprocal mix-ups of T, labels taken from the wrong position);
- a dense grid search of the likelihood itself (an independent method: the
  oracle bisects the likelihood's derivative) finds the same temperature
  (a wrong derivative, a wrong bracket update);
- scaling z by a scales every temperature by a exactly (theta used where T
  was meant);
- labels that separate perfectly put T on the bounds, a position nobody
  reached and a position with z = 0 only get T = 1 (bound handling);
- a position's fit ignores the scores of sequences that never reached it
  (the conditional set of "every earlier token accepted");
- the ECE of hand-worked samples (two bins; two confidences sharing one
  bin of width 1/15), and the ECE falls after the fit.
"""
import numpy as np
import pytest

T_MIN, T_MAX = 0.05, 20.0


def logistic_sample(rng, N, K, T, mu=1.5, sd=1.5):
    """Head scores z and accepted-prefix lengths drawn from the logistic
    model the fit assumes: position k is accepted with probability
    1 / (1 + exp(-z / T_k)) given every earlier one was."""
    z = rng.normal(mu, sd, (N, K)).astype(np.float32)
    p = 1.0 / (1.0 + np.exp(-z.astype(np.float64) / np.asarray(T)))
    acc = rng.random((N, K)) < p
    n_acc = np.where(acc.all(1), K, np.argmin(acc, 1)).astype(np.int32)
    return z, n_acc


def nll(z, y, T):
    """Bernoulli negative log-likelihood of labels y under sigmoid(z / T)."""
    x = z.astype(np.float64) / T
    return float(np.sum(np.logaddexp(0.0, x) - y * x))


def test_recovers_generating_temperatures(oracle_mod):
    rng = np.random.default_rng(11)
    T = np.array([1.3, 1.5, 0.8, 2.0, 1.1])
    z, n_acc = logistic_sample(rng, 200_000, 5, T)
    r = oracle_mod.sts_fit(z, n_acc)
    assert np.all(np.abs(r["temps"] - T) / T < 0.03), r["temps"]
    assert r["count"][0] == 200_000
    assert np.all(np.diff(r["count"]) <= 0)  # fewer sequences reach later positions


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_matches_dense_grid_search_of_the_likelihood(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    N, K = 3000, 3
    z, n_acc = logistic_sample(rng, N, K, [0.7, 1.6, 3.0])
    r = oracle_mod.sts_fit(z, n_acc)
    grid = np.exp(np.linspace(np.log(T_MIN), np.log(T_MAX), 6001))
    step = grid[1] / grid[0]
    for j in range(K):
        seen = n_acc >= j
        zz, y = z[seen, j], (n_acc[seen] > j).astype(np.float64)
        vals = np.array([nll(zz, y, t) for t in grid])
        best = grid[int(np.argmin(vals))]
        assert best / step <= r["temps"][j] <= best * step, (j, best, r["temps"][j])
        # and the fitted temperature is no worse than the grid's best point
        assert nll(zz, y, r["temps"][j]) <= vals.min() + 1e-9 * abs(vals.min())


def test_scaling_scores_scales_temperatures(oracle_mod):
    rng = np.random.default_rng(5)
    z, n_acc = logistic_sample(rng, 20_000, 4, [1.2, 1.4, 1.6, 1.8])
    a = 2.0  # exact in binary: z * a is exact in fp32
    r1 = oracle_mod.sts_fit(z, n_acc)
    r2 = oracle_mod.sts_fit(z * np.float32(a), n_acc)
    assert np.allclose(r2["temps"], a * r1["temps"], rtol=1e-9, atol=0)
    assert r2["ece_after"] == pytest.approx(r1["ece_after"], abs=1e-12)


def test_separable_labels_end_on_the_bounds(oracle_mod):
    z = np.array([[2.0], [1.0], [3.0]], np.float32)
    every = oracle_mod.sts_fit(z, np.array([1, 1, 1], np.int32))     # all accepted, z > 0
    assert every["temps"][0] == pytest.approx(T_MIN, rel=1e-12)
    none = oracle_mod.sts_fit(z, np.array([0, 0, 0], np.int32))      # all rejected, z > 0
    assert none["temps"][0] == pytest.approx(T_MAX, rel=1e-12)


def test_unreached_and_uninformative_positions_get_unit_temperature(oracle_mod):
    z = np.array([[1.0, 0.5, 0.0], [2.0, -1.0, 0.0]], np.float32)
    r = oracle_mod.sts_fit(z, np.array([0, 0, 0], np.int32)[:2])     # nobody reaches position 1
    assert r["temps"][1] == 1.0 and r["temps"][2] == 1.0 and r["count"][1] == 0
    r = oracle_mod.sts_fit(z, np.array([3, 2], np.int32))            # position 2: z = 0 only
    assert r["temps"][2] == 1.0 and r["count"][2] == 2


def test_unobserved_scores_do_not_move_the_fit(oracle_mod):
    rng = np.random.default_rng(9)
    z, n_acc = logistic_sample(rng, 5000, 4, [1.0, 1.5, 2.0, 2.5])
    r1 = oracle_mod.sts_fit(z, n_acc)
    z2 = z.copy()
    for j in range(4):
        z2[n_acc < j, j] = rng.normal(0, 50, int((n_acc < j).sum()))  # never reached
    r2 = oracle_mod.sts_fit(z2, n_acc)
    assert np.array_equal(r1["temps"], r2["temps"])
    assert r1["ece_before"] == r2["ece_before"] and r1["ece_after"] == r2["ece_after"]


def test_ece_hand_worked(oracle_mod):
    # K = 1; c = sigmoid(z) at T = 1: z = 0 -> 0.5 (bin 7 of 15), z = ln 3 -> 0.75 (bin 11).
    # bin 7: labels 1, 0 (sum 1), confidences 0.5 + 0.5 = 1   -> |1 - 1| = 0
    # bin 11: labels 1, 1 (sum 2), confidences 0.75 + 0.75    -> |2 - 1.5| = 0.5
    # ECE = 0.5 / 4 = 0.125
    z = np.array([[0.0], [0.0], [np.log(3.0)], [np.log(3.0)]], np.float32)
    n_acc = np.array([1, 0, 1, 1], np.int32)
    r = oracle_mod.sts_fit(z, n_acc)
    c = 1.0 / (1.0 + np.exp(-np.float64(np.float32(np.log(3.0)))))  # z is stored in fp32
    assert r["ece_before"] == pytest.approx(abs(2.0 - 2 * c) / 4.0, abs=1e-15)
    assert r["ece_before"] == pytest.approx(0.125, abs=1e-7)


def test_ece_shares_a_bin_one_fifteenth_wide(oracle_mod):
    # c = 0.62 and 0.66 (T = 1) share bin 9 of 15 ([0.6, 0.6667)), so their
    # label and confidence sums meet in one |sum y - sum c|; with any other
    # bin count near 15 they would fall apart (14 bins: bins 8 and 9)
    z = np.array([[np.log(0.62 / 0.38)], [np.log(0.66 / 0.34)]], np.float32)
    n_acc = np.array([1, 0], np.int32)  # the first accepted, the second rejected
    c = 1.0 / (1.0 + np.exp(-z[:, 0].astype(np.float64)))
    assert np.all(np.floor(c * 15) == 9) and np.floor(c[0] * 14) != np.floor(c[1] * 14)
    r = oracle_mod.sts_fit(z, n_acc)
    assert r["ece_before"] == pytest.approx(abs(1.0 - c.sum()) / 2.0, abs=1e-15)


def test_fit_lowers_ece_on_an_overconfident_head(oracle_mod):
    rng = np.random.default_rng(21)
    z, n_acc = logistic_sample(rng, 50_000, 6, np.linspace(1.3, 2.3, 6))
    r = oracle_mod.sts_fit(z, n_acc)
    assert r["ece_before"] > 0.03 and r["ece_after"] < 0.01, r


def test_accepted_lengths_are_clamped(oracle_mod):
    rng = np.random.default_rng(4)
    z, n_acc = logistic_sample(rng, 2000, 3, [1.0, 1.0, 1.0])
    big = n_acc.copy()
    big[big == 3] = 7  # beyond K reads as K
    neg = n_acc.copy()
    neg[neg == 0] = -2  # below 0 reads as 0
    for other in (big, neg):
        a, b = oracle_mod.sts_fit(z, n_acc), oracle_mod.sts_fit(z, other)
        assert np.array_equal(a["temps"], b["temps"])
