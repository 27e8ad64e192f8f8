"""Pins of the oracle's RNN sequential head (draft and verify).

freeaitool.com "DeepSeek DSpark complete guide" 3.1 names an optional RNN
head that keeps a recurrent state; the pages give no formula.  The reading
pinned here: s_k = tanh(R s_{k-1} + U[x_{k-1}]) from h0, bias s_k . W^T,
then the Markov head's softmax and inverse CDF.  Each pin checks the oracle
against something other than itself:
  * R = 0, h0 = 0 reduces the head to the (pinned) Markov head on tanh(U);
  * at small amplitude tanh is the identity to third order, so the logits
    equal those of the linear recurrence s_k = R s_{k-1} + U[x_{k-1}],
    solved here with plain matrix products, to O(eps^3) -- a transposed R,
    a dropped input term or a token taken one position late differs at
    first order;
  * the state carries older tokens: with R != 0 position 2 depends on the
    token before position 1, with R = 0 it does not;
  * verify: p_t = p_d accepts everything, and 10^6 trials of the emitted
    tokens follow p_t (chi-square), which needs the residual to use the RNN
    head's own draft row at the rejected position.
"""
import numpy as np
import pytest
from scipy import special, stats

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rng(seed):
    return np.random.Generator(np.random.Philox(seed))


def _softmax(l):
    e = np.exp(l - l.max())
    return e / e.sum()


def test_zero_recurrence_is_markov_head_on_tanh_u(oracle_mod):
    g = _rng(41)
    B, K, V, r = 40, 5, 64, 8
    base = g.normal(0, 2, (B, K, V)).astype(np.float32)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    R = np.zeros((r, r), np.float32)
    prev = g.integers(-1, V, B).astype(np.int32)
    ud = g.random((B, K)).astype(np.float32)
    it = g.choice(np.array([0.6, 1.0, 1.3], np.float32), B)
    d = oracle_mod.draft_rnn(base, U, W, R, prev, ud, inv_temp=it)
    m = oracle_mod.draft(base, np.tanh(U.astype(np.float64)).astype(np.float32), W, prev, ud,
                         inv_temp=it)
    for b in range(B):
        for k in range(K):
            if d["tokens"][b, k] != m["tokens"][b, k]:
                assert m["margin"][b, k] < 1e-6
                break
            assert abs(d["p_tok"][b, k] - m["p_tok"][b, k]) < 1e-6
            assert abs(d["lse"][b, k] - m["lse"][b, k]) < 1e-6


@pytest.mark.parametrize("transposed_check", [False, True])
def test_small_amplitude_is_linear_recurrence(oracle_mod, transposed_check):
    g = _rng(42)
    B, K, V, r, eps = 16, 6, 32, 6, 1e-3
    base = g.normal(0, 1, (B, K, V)).astype(np.float32)
    U = (eps * g.normal(0, 1, (V, r))).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    R = (0.5 * g.normal(0, 1, (r, r)) / np.sqrt(r)).astype(np.float32)
    h0 = (eps * g.normal(0, 1, (B, r))).astype(np.float32)
    prev = g.integers(0, V, B).astype(np.int32)
    ud = g.random((B, K)).astype(np.float32)
    d = oracle_mod.draft_rnn(base, U, W, R, prev, ud, h0=h0, states=True)
    R64 = R.astype(np.float64).T if transposed_check else R.astype(np.float64)
    worst = 0.0
    for b in range(B):
        s = h0[b].astype(np.float64)
        x = prev[b]
        for k in range(K):
            s = R64 @ s + U[x].astype(np.float64)
            l = base[b, k].astype(np.float64) + W.astype(np.float64) @ s
            worst = max(worst, abs(special.logsumexp(l) - d["lse"][b, k]),
                        abs(np.exp(l[d["tokens"][b, k]] - special.logsumexp(l)) - d["p_tok"][b, k]))
            x = d["tokens"][b, k]
    if transposed_check:
        # the transposed recurrence is a different head: differs at first order
        assert worst > 1e-5
    else:
        assert worst < 1e-7


def test_state_carries_tokens_before_the_previous_one(oracle_mod):
    """Position 2's distribution, for a fixed first token, depends on the
    token before position 1 exactly when R != 0."""
    g = _rng(43)
    V, r, K = 16, 4, 2
    base1 = g.normal(0, 1, (K, V)).astype(np.float32)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    for R, differs in [(np.zeros((r, r), np.float32), False),
                       (g.normal(0, 0.8, (r, r)).astype(np.float32), True)]:
        B = 4 * V
        base = np.broadcast_to(base1, (B, K, V))
        prev = np.repeat(np.arange(4, dtype=np.int32), V)
        # u of position 1 chosen per request so that every first token occurs
        ud = np.zeros((B, K), np.float32)
        lse2 = {}
        for b in range(B):
            ud[b, 0] = np.float32(((b % V) + 0.5) / V)
            ud[b, 1] = 0.5
        d = oracle_mod.draft_rnn(base, U, W, R, prev, ud)
        for b in range(B):
            lse2.setdefault(int(d["tokens"][b, 0]), set()).add(round(float(d["lse"][b, 1]), 12))
        multi = [len(v) > 1 for v in lse2.values()]
        assert any(multi) == differs


def _rnn_case(oracle_mod, g, N, V, r, K):
    b1 = g.normal(0, 1.5, (K, V)).astype(np.float32)
    U = g.normal(0, 1, (V, r)).astype(np.float32)
    W = g.normal(0, 1, (V, r)).astype(np.float32)
    R = g.normal(0, 0.7, (r, r)).astype(np.float32)
    h0 = g.normal(0, 0.5, (1, r)).astype(np.float32)
    return b1, U, W, R, h0


def test_rnn_verify_equal_distributions_accept_everything(oracle_mod):
    g = _rng(44)
    B, V, r, K = 100, 12, 3, 4
    b1, U, W, R, h0 = _rnn_case(oracle_mod, g, B, V, r, K)
    base = g.normal(0, 2, (B, K, V)).astype(np.float32)
    hb = np.repeat(h0, B, axis=0)
    prev = g.integers(0, V, B).astype(np.int32)
    d = oracle_mod.draft_rnn(base, U, W, R, prev, g.random((B, K)).astype(np.float32), h0=hb,
                             states=True)
    # target rows = the draft's own logits (from its reported states), then a bonus row
    rows = base.astype(np.float64) + np.einsum("bkr,vr->bkv", d["states"], W.astype(np.float64))
    bonus = g.normal(0, 2, (B, 1, V))
    target = np.concatenate([rows, bonus], axis=1).astype(np.float32)
    L = g.integers(0, K + 1, B).astype(np.int32)
    # the fp32 target rows reproduce p_d to ~1e-7, so p_t / p_d is 1 to that
    # accuracy: every position passes u = 0.999, and none would if the rows,
    # the states or the accepted tokens were misplaced
    ua = np.full((B, K), 0.999, np.float32)
    ur = g.random(B).astype(np.float32)
    v = oracle_mod.verify_rnn(target.reshape(B * (K + 1), V), np.arange(B) * (K + 1), L, base, U,
                              W, R, prev, d["tokens"], d["p_tok"], ua, ur, h0=hb)
    assert (v["n_acc"] == L).all()
    for b in range(B):
        assert v["out_tokens"][b, :L[b]].tolist() == d["tokens"][b, :L[b]].tolist()


def test_rnn_verify_losslessness_chi2(oracle_mod):
    """V=8, K=2, RNN head with R != 0, 10^6 trials: the emitted token at
    position 1 follows p_t(row 1), given acceptance at 1 position 2 follows
    p_t(row 2).  Position 2's residual uses the RNN row (state s_2, which
    depends on the drafted first token and on h0); a Markov row there
    would bias the second histogram."""
    g = _rng(45)
    N, V, r, K = 1_000_000, 8, 3, 2
    b1, U, W, R, h0 = _rnn_case(oracle_mod, g, N, V, r, K)
    t1 = g.normal(0, 1.5, (K + 1, V)).astype(np.float32)
    base = np.broadcast_to(b1, (N, K, V))
    hb = np.broadcast_to(h0, (N, r))
    prev = np.full(N, 5, np.int32)
    d = oracle_mod.draft_rnn(base, U, W, R, prev, g.random((N, K)).astype(np.float32), h0=hb)
    target = np.broadcast_to(t1, (N, K + 1, V)).reshape(N * (K + 1), V)
    v = oracle_mod.verify_rnn(target, np.arange(N, dtype=np.int64) * (K + 1),
                              np.full(N, K, np.int32), base, U, W, R, prev, d["tokens"],
                              d["p_tok"], g.random((N, K)).astype(np.float32),
                              g.random(N).astype(np.float32), h0=hb)
    out = v["out_tokens"]
    for pos, mask in [(0, np.ones(N, bool)), (1, v["n_acc"] >= 1), (2, v["n_acc"] >= 2)]:
        pt = _softmax(t1[pos].astype(np.float64))
        counts = np.bincount(out[mask, pos], minlength=V)
        n = int(mask.sum())
        assert n > 50_000
        _, pval = stats.chisquare(counts, pt * n)
        assert pval > 0.01, (pos, pval)
