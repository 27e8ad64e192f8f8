"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a library
routine on a case the method reduces to, a closed form, an exact
enumeration, or a statistical law (chi-square at p > 0.01 on seeded draws).
A plausible slip in the oracle (a dropped bias term, U and W swapped, an
off-by-one in the inverse CDF, a wrong accept inequality, a residual that
is not clipped at zero, a scheduler that does not stop) fails one of them.

Sources: yage.ai "DSpark speculative decoding hardware scheduling" (Markov
head formula, rejection sampling needs exact p_d, SPS(B) scheduler);
freeaitool.com "DeepSeek DSpark complete guide" sections 3.1, 4.1, 4.2;
legalagi.cn "读懂 DSpark" sections 三 and 五 (lossless, latency identity,
early stop keeps it lossless).
"""
import itertools

import numpy as np
import pytest
from scipy import special, stats

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rng(seed):
    return np.random.Generator(np.random.Philox(seed))


def _softmax(l):
    l = np.asarray(l, np.float64)
    e = np.exp(l - l.max())
    return e / e.sum()


# ---------------------------------------------------------------- draft --

def test_hand_worked_inverse_cdf(oracle_mod):
    """V=4 with probabilities (1,2,3,4)/10: CDF 0.1, 0.3, 0.6, 1.0.

    The draw is the smallest i whose CDF exceeds u, so u=0.05 -> 0,
    u=0.1 -> 1 (0.1 is not > 0.1), u=0.35 -> 2, u=0.6 -> 3, u=0.99 -> 3.
    """
    base1 = np.log(np.array([1, 2, 3, 4], np.float64)).astype(np.float32)
    us = np.array([0.05, 0.1 + 1e-6, 0.35, 0.6 + 1e-6, 0.99], np.float32)
    B = len(us)
    base = np.tile(base1, (B, 1, 1))
    U = np.zeros((4, 2), np.float32)
    W = np.zeros((4, 2), np.float32)
    out = oracle_mod.draft(base, U, W, np.full(B, -1, np.int32), us[:, None])
    assert out["tokens"][:, 0].tolist() == [0, 1, 2, 3, 3]
    np.testing.assert_allclose(out["p_tok"][:, 0], [0.1, 0.2, 0.3, 0.4, 0.4], atol=2e-7)
    np.testing.assert_allclose(out["lse"][:, 0], np.log(10.0) * np.ones(B), atol=2e-7)


def test_w_zero_is_independent_categorical(oracle_mod):
    """W = 0: every position is an independent softmax draw (numpy searchsorted)."""
    g = _rng(1)
    B, K, V, r = 20, 3, 50, 4
    base = g.normal(0, 2, (B, K, V)).astype(np.float32)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = np.zeros((V, r), np.float32)
    prev = g.integers(0, V, B).astype(np.int32)
    it = (1.0 / g.choice([0.6, 1.0, 1.3], B)).astype(np.float32)
    ud = g.random((B, K)).astype(np.float32)
    out = oracle_mod.draft(base, U, W, prev, ud, inv_temp=it)
    for b in range(B):
        for k in range(K):
            l = base[b, k].astype(np.float64) * np.float64(it[b])
            p = _softmax(l)
            cdf = np.cumsum(p)
            x = int(np.searchsorted(cdf, np.float64(ud[b, k]), side="right"))
            assert out["tokens"][b, k] == x
            assert abs(out["p_tok"][b, k] - p[x]) < 1e-12
            assert abs(out["lse"][b, k] - special.logsumexp(l)) < 1e-10


def test_transition_lookup_orientation(oracle_mod):
    """Constructed transition: bias(x_prev -> v) = 60 iff v = x_prev + 1 (mod V).

    With U = I and W[v, i] = 60 [v == i+1], U[x_prev] . W[v] = W[v, x_prev],
    so the chain must step forward by one.  Swapping the factors (looking up
    W and projecting on U) would step backwards; dropping the bias would
    give an (almost) uniform draw.
    """
    V = 6
    U = np.eye(V, dtype=np.float32)
    W = np.zeros((V, V), np.float32)
    for i in range(V):
        W[(i + 1) % V, i] = 60.0
    B, K = 12, 5
    g = _rng(2)
    base = g.normal(0, 1, (B, K, V)).astype(np.float32)
    prev = (np.arange(B) % V).astype(np.int32)
    out = oracle_mod.draft(base, U, W, prev, g.random((B, K)).astype(np.float32))
    for b in range(B):
        x = prev[b]
        for k in range(K):
            x = (x + 1) % V
            assert out["tokens"][b, k] == x


def test_negative_prev_token_drops_first_bias(oracle_mod):
    """prev_token < 0: position 1 has no transition bias (pure base softmax)."""
    V = 6
    U = np.eye(V, dtype=np.float32)
    W = np.zeros((V, V), np.float32)
    for i in range(V):
        W[(i + 1) % V, i] = 60.0
    base = np.zeros((1, 2, V), np.float32)
    base[0, 0, 4] = 60.0  # position 1 decided by the base logits alone
    out = oracle_mod.draft(base, U, W, np.array([-1], np.int32),
                           np.array([[0.5, 0.5]], np.float32))
    assert out["tokens"][0].tolist() == [4, 5]


def test_markov_chain_enumeration_chi2(oracle_mod):
    """V=4, K=3: 10^6 sampled chains follow the exact joint law (chi-square)."""
    g = _rng(3)
    V, r, K, N = 4, 2, 3, 1_000_000
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    base1 = g.normal(0, 1, (K, V)).astype(np.float32)
    x0 = 2
    # exact joint probabilities by enumeration of all V^K sequences
    probs = {}
    for seq in itertools.product(range(V), repeat=K):
        p, x = 1.0, x0
        for k in range(K):
            l = base1[k].astype(np.float64) + W.astype(np.float64) @ U[x].astype(np.float64)
            p *= _softmax(l)[seq[k]]
            x = seq[k]
        probs[seq] = p
    base = np.broadcast_to(base1, (N, K, V))
    ud = g.random((N, K)).astype(np.float32)
    out = oracle_mod.draft(base, U, W, np.full(N, x0, np.int32), ud)
    codes = (out["tokens"] * np.array([V * V, V, 1])).sum(1)
    counts = np.bincount(codes, minlength=V ** K)
    expected = np.array([probs[s] for s in itertools.product(range(V), repeat=K)]) * N
    assert abs(expected.sum() - N) < 1e-6 * N
    _, pval = stats.chisquare(counts, expected)
    assert pval > 0.01


# ----------------------------------------------------------- scheduler --

def _table(kind):
    xs = np.arange(16, dtype=np.float32) * 512
    if kind == "flat":
        ys = np.full(16, 20.0, np.float32)
    elif kind == "steep":
        ys = (20.0 + 1e4 * xs).astype(np.float32)
    elif kind == "linear":
        ys = (20.0 + 0.004 * xs).astype(np.float32)
    else:  # knee at 4096
        ys = np.where(xs <= 4096, 20.0 + 0.004 * xs,
                      20.0 + 0.004 * 4096 + 0.016 * (xs - 4096)).astype(np.float32)
    return xs, ys


def test_cost_interpolation(oracle_mod):
    xs, ys = _table("knee")
    for n in [0, 1, 511.5, 512, 4096, 5000.25, 7680]:
        assert abs(oracle_mod.cost_ms(xs, ys, n) - np.interp(n, xs, ys)) < 1e-9
    # linear extension beyond the last point uses the last segment
    slope = (float(ys[-1]) - float(ys[-2])) / (float(xs[-1]) - float(xs[-2]))
    assert abs(oracle_mod.cost_ms(xs, ys, 9000) - (float(ys[-1]) + slope * (9000 - float(xs[-1])))) < 1e-9
    slope0 = (float(ys[1]) - float(ys[0])) / (float(xs[1]) - float(xs[0]))
    assert abs(oracle_mod.cost_ms(xs, ys, -100) - (float(ys[0]) - slope0 * 100)) < 1e-9


def test_sts_unit_temperature_is_logistic(oracle_mod):
    g = _rng(4)
    z = g.normal(1.5, 1.0, (7, 5)).astype(np.float32)
    xs, ys = _table("linear")
    out = oracle_mod.prefix(z, np.ones(5, np.float32), xs, ys, enable=False)
    np.testing.assert_allclose(out["c"], special.expit(z.astype(np.float64)), rtol=1e-14)
    np.testing.assert_allclose(out["S"], np.cumprod(special.expit(z.astype(np.float64)), axis=1),
                               rtol=1e-13)
    assert (out["L"] == 5).all()


def test_sts_temperatures_divide_logits(oracle_mod):
    g = _rng(5)
    z = g.normal(1.5, 1.0, (4, 6)).astype(np.float32)
    T = np.array([1.0 + 0.1 * k for k in range(1, 7)], np.float32)
    xs, ys = _table("linear")
    out = oracle_mod.prefix(z, T, xs, ys)
    np.testing.assert_allclose(out["c"], special.expit(z.astype(np.float64) / T.astype(np.float64)),
                               rtol=1e-14)


def test_flat_cost_takes_everything_steep_takes_nothing(oracle_mod):
    g = _rng(6)
    z = g.normal(1.5, 1.0, (32, 6)).astype(np.float32)
    T = np.ones(6, np.float32)
    out = oracle_mod.prefix(z, T, *_table("flat"))
    assert (out["L"] == 6).all()
    out = oracle_mod.prefix(z, T, *_table("steep"))
    assert (out["L"] == 0).all()


def _sorted_candidates(S):
    B, K = S.shape
    b, k = np.meshgrid(np.arange(B), np.arange(K), indexing="ij")
    order = np.lexsort((b.ravel(), k.ravel(), -S.ravel()))
    return S.ravel()[order], b.ravel()[order], k.ravel()[order]


@pytest.mark.parametrize("seed", [7, 8, 9])
def test_linear_cost_greedy_equals_argmax(oracle_mod, seed):
    """Linear cost, survival sorted descending: E/t(N) is unimodal in the
    number of committed candidates, so greedy-with-early-stop must land on
    the argmax over all prefix lengths; the committed set per request is a
    prefix of its positions."""
    g = _rng(seed)
    B, K = 64, 6
    z = g.normal(1.5, 1.0, (B, K)).astype(np.float32)
    T = np.array([1.0 + 0.1 * k for k in range(1, K + 1)], np.float32)
    xs, ys = _table("linear")
    a, slope = 20.0, 0.004
    out = oracle_mod.prefix(z, T, xs, ys)
    s, bb, kk = _sorted_candidates(out["S"])
    n = np.arange(0, len(s) + 1)
    E = B + np.concatenate([[0.0], np.cumsum(s)])
    t = np.array([oracle_mod.cost_ms(xs, ys, B + i) for i in n])
    assert np.allclose(t, a + np.float32(slope) * (B + n), rtol=1e-6)
    obj = E / t
    n_star = int(np.argmax(obj))
    assert out["L"].sum() == n_star
    assert abs(out["objective"] - obj[n_star]) < 1e-12 * obj[n_star]
    for b in range(B):
        committed = sorted(kk[:n_star][bb[:n_star] == b].tolist())
        assert committed == list(range(out["L"][b]))


def test_knee_cost_stops_at_first_non_improvement(oracle_mod):
    """With the knee table the greedy scan stops at the first candidate that
    does not raise E/t(N), even if a later one would (never resumes)."""
    g = _rng(10)
    B, K = 512, 16
    z = g.normal(1.5, 1.0, (B, K)).astype(np.float32)
    T = np.array([1.0 + 0.1 * k for k in range(1, K + 1)], np.float32)
    xs, ys = _table("knee")
    out = oracle_mod.prefix(z, T, xs, ys)
    s, bb, kk = _sorted_candidates(out["S"])
    E = B + np.concatenate([[0.0], np.cumsum(s)])
    t = np.array([oracle_mod.cost_ms(xs, ys, B + i) for i in range(len(s) + 1)])
    obj = E / t
    stop = np.nonzero(obj[1:] <= obj[:-1])[0]
    n_commit = int(stop[0]) if len(stop) else len(s)
    assert out["L"].sum() == n_commit
    assert 0 < n_commit < B * K


# --------------------------------------------------------------- verify --

def _verify_case(oracle_mod, base, target, U, W, prev, ud, ua, ur, L=None, it=None):
    B, K, V = base.shape
    d = oracle_mod.draft(base, U, W, prev, ud, inv_temp=it)
    rs = np.arange(B, dtype=np.int64) * (K + 1)
    L = np.full(B, K, np.int32) if L is None else L
    v = oracle_mod.verify(target.reshape(B * (K + 1), V), rs, L, base, U, W, prev,
                          d["tokens"], d["p_tok"], ua, ur, inv_temp=it)
    return d, v


def test_equal_distributions_accept_everything(oracle_mod):
    """p_d = p_t at every position: the ratio is 1 > u, every token is kept
    and the bonus token comes from the row after the verified block."""
    g = _rng(11)
    B, K, V, r = 200, 4, 16, 3
    base = g.normal(0, 2, (B, K, V)).astype(np.float32)
    bonus = g.normal(0, 2, (B, 1, V)).astype(np.float32)
    target = np.concatenate([base, bonus], axis=1)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = np.zeros((V, r), np.float32)
    L = g.integers(0, K + 1, B).astype(np.int32)
    ud = g.random((B, K)).astype(np.float32)
    ua = np.full((B, K), np.float32(1.0) - np.float32(2 ** -24), np.float32)
    ur = g.random(B).astype(np.float32)
    d, v = _verify_case(oracle_mod, base, target, U, W, np.zeros(B, np.int32), ud, ua, ur, L=L)
    assert (v["n_acc"] == L).all()
    for b in range(B):
        assert v["out_tokens"][b, :L[b]].tolist() == d["tokens"][b, :L[b]].tolist()
        p = _softmax(target[b, L[b]].astype(np.float64))
        x = int(np.searchsorted(np.cumsum(p), np.float64(ur[b]), side="right"))
        assert v["out_tokens"][b, L[b]] == x
        assert (v["out_tokens"][b, L[b] + 1:] == -1).all()


def test_certain_rejection_takes_residual(oracle_mod):
    """Draft puts all its mass on token 0, target on token 3: position 1 is
    rejected and the correction token is 3 (the residual max(0, p_t - p_d))."""
    B, K, V = 3, 2, 4
    base = np.zeros((B, K, V), np.float32)
    base[:, :, 0] = 60.0
    target = np.zeros((B, K + 1, V), np.float32)
    target[:, :, 3] = 60.0
    U = np.zeros((V, 1), np.float32)
    W = np.zeros((V, 1), np.float32)
    g = _rng(12)
    d, v = _verify_case(oracle_mod, base, target, U, W, np.full(B, -1, np.int32),
                        g.random((B, K)).astype(np.float32),
                        g.random((B, K)).astype(np.float32), g.random(B).astype(np.float32))
    assert (d["tokens"] == 0).all()
    assert (v["n_acc"] == 0).all()
    assert (v["out_tokens"][:, 0] == 3).all()
    assert (v["out_tokens"][:, 1:] == -1).all()


def test_expected_acceptance_is_one_minus_tv(oracle_mod):
    """Single position: P(accept) = sum_v min(p_t, p_d) = 1 - TV(p_t, p_d)."""
    g = _rng(13)
    V, N = 8, 400_000
    b1 = g.normal(0, 1.5, V).astype(np.float32)
    t1 = g.normal(0, 1.5, V).astype(np.float32)
    base = np.broadcast_to(b1, (N, 1, V))
    target = np.broadcast_to(np.stack([t1, t1]), (N, 2, V))
    U = np.zeros((V, 1), np.float32)
    W = np.zeros((V, 1), np.float32)
    d, v = _verify_case(oracle_mod, base, target, U, W, np.full(N, -1, np.int32),
                        g.random((N, 1)).astype(np.float32),
                        g.random((N, 1)).astype(np.float32), g.random(N).astype(np.float32))
    pd, pt = _softmax(b1), _softmax(t1)
    expect = np.minimum(pd, pt).sum()
    assert abs(expect - (1 - 0.5 * np.abs(pd - pt).sum())) < 1e-12
    mean = v["n_acc"].mean()
    sd = np.sqrt(expect * (1 - expect) / N)
    assert abs(mean - expect) < 5 * sd


def test_losslessness_chi2_positions_1_2_3(oracle_mod):
    """V=8, K=2, Markov head on, 10^6 trials: the emitted token at position 1
    follows p_t(row 1); given acceptance at 1, position 2 follows p_t(row 2);
    given acceptance at 1 and 2, the bonus follows p_t(row 3)."""
    g = _rng(14)
    V, r, K, N = 8, 3, 2, 1_000_000
    b1 = g.normal(0, 1.5, (K, V)).astype(np.float32)
    t1 = g.normal(0, 1.5, (K + 1, V)).astype(np.float32)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    base = np.broadcast_to(b1, (N, K, V))
    target = np.broadcast_to(t1, (N, K + 1, V))
    d, v = _verify_case(oracle_mod, base, target, U, W, np.full(N, 5, np.int32),
                        g.random((N, K)).astype(np.float32),
                        g.random((N, K)).astype(np.float32), g.random(N).astype(np.float32))
    out = v["out_tokens"]
    for pos, mask in [(0, np.ones(N, bool)), (1, v["n_acc"] >= 1), (2, v["n_acc"] >= 2)]:
        pt = _softmax(t1[pos])
        counts = np.bincount(out[mask, pos], minlength=V)
        n = int(mask.sum())
        assert n > 50_000
        _, pval = stats.chisquare(counts, pt * n)
        assert pval > 0.01, (pos, pval)


def test_expected_accepted_length_by_enumeration(oracle_mod):
    """V=4, K=2: E[n_acc] enumerated over every draft sequence equals the
    Monte-Carlo mean of the oracle's verify (draft chain + accept test)."""
    g = _rng(15)
    V, r, K, N = 4, 2, 2, 1_000_000
    b1 = g.normal(0, 1.0, (K, V)).astype(np.float32)
    t1 = g.normal(0, 1.0, (K + 1, V)).astype(np.float32)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    x0 = 1
    pt = [_softmax(t1[k]) for k in range(K)]

    def pdraft(k, xprev):
        return _softmax(b1[k].astype(np.float64) + W.astype(np.float64) @ U[xprev].astype(np.float64))

    exact = 0.0
    for x1 in range(V):
        p1 = pdraft(0, x0)[x1]
        a1 = min(1.0, pt[0][x1] / p1)
        inner = 0.0
        for x2 in range(V):
            p2 = pdraft(1, x1)[x2]
            inner += p2 * min(1.0, pt[1][x2] / p2)
        exact += p1 * a1 * (1.0 + inner)
    base = np.broadcast_to(b1, (N, K, V))
    target = np.broadcast_to(t1, (N, K + 1, V))
    d, v = _verify_case(oracle_mod, base, target, U, W, np.full(N, x0, np.int32),
                        g.random((N, K)).astype(np.float32),
                        g.random((N, K)).astype(np.float32), g.random(N).astype(np.float32))
    mean = v["n_acc"].mean()
    sd = v["n_acc"].std() / np.sqrt(N)
    assert abs(mean - exact) < 5 * sd
