"""dspark_confidence_prefix_async (staircase cost reading, asynchronous
budget) against the oracle, and the two-steps-back loop replayed from a
CUDA graph with a two-slot device ring.

Decisions (the greedy stop, the budget cut, hence verify lengths and the
greedy N) are compared exactly unless the oracle's margin for that decision
is below 1e-6 (fp64 on both sides, but exp and fused multiply-adds may
differ by an ulp); c and survival within 1e-6 absolute (fp32 outputs),
the objective within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL
from tests.parity import cut_problems

pytestmark = pytest.mark.gpu
MARGIN = 1e-6


def run_gpu(z, temps, xs, ys, staircase, budget=None, enable=True, alias=False, ws=None):
    B, K = z.shape
    c = torch.empty(B, K, device="cuda")
    S = torch.empty(B, K, device="cuda")
    L = torch.empty(B, dtype=torch.int32, device="cuda")
    obj = torch.empty(1, device="cuda")
    if ws is None:
        ws = torch.zeros(D.dspark_prefix_workspace_size(B, K, xs.numel()), dtype=torch.uint8,
                         device="cuda")
    bin_ = None if budget is None else torch.tensor([budget], dtype=torch.int32, device="cuda")
    bout = bin_ if alias else torch.full((1,), -7, dtype=torch.int32, device="cuda")
    D.dspark_confidence_prefix_async(z, temps, xs, ys, enable, c, S, L, obj, ws,
                                     staircase=staircase, budget_in=bin_, budget_out=bout)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(ws, None) == 0
    return dict(c=c.cpu().numpy(), S=S.cpu().numpy(), L=L.cpu().numpy(),
                objective=float(obj.item()), n_greedy=int(bout.item()))


def compare(oracle_mod, g, z, temps, xs, ys, staircase, budget=None, enable=True):
    args = (z.cpu().numpy(), temps.cpu().numpy(), xs.cpu().numpy(), ys.cpu().numpy())
    r = oracle_mod.prefix_async(*args, staircase=staircase, enable=enable, budget=budget)
    greedy = oracle_mod.prefix_async(*args, staircase=staircase, enable=enable)
    np.testing.assert_allclose(g["c"], r["c"], atol=1e-6, rtol=0)
    np.testing.assert_allclose(g["S"], r["S"], atol=1e-6, rtol=0)
    if greedy["margin"] >= MARGIN:
        assert g["n_greedy"] == r["n_greedy"]
    if r["margin"] >= MARGIN:
        assert np.array_equal(g["L"], r["L"])
        assert g["objective"] == pytest.approx(r["objective"], rel=1e-5)
    elif enable:
        # a near-tie at the cut: the lengths must still be a cut of the same
        # order (for a budget, of the same size)
        why = cut_problems(oracle_mod, r["S"], args[2], args[3], g["L"], staircase=staircase,
                           budget=budget)
        assert not why, why
    if enable and budget is None:
        # the greedy N it returns is its own cut's
        assert g["n_greedy"] == z.shape[0] + int(g["L"].sum())
    return r


@pytest.mark.parametrize("staircase", [False, True])
@pytest.mark.parametrize("name", ["serving", "stress"])
def test_greedy_and_budgets(oracle_mod, name, staircase):
    w = WL.get(name)
    assert D.dspark_prefix_path(w.B, w.K, True) == "multi-cta"  # 1536 and 8192 candidates
    g = torch.Generator(device="cuda").manual_seed(5)
    z = torch.randn(w.B, w.K, generator=g, device="cuda").add_(1.5)
    temps = WL.seq_temps(w.K).cuda()
    xs, ys = (t.cuda() for t in WL.cost_table())
    greedy = compare(oracle_mod, run_gpu(z, temps, xs, ys, staircase), z, temps, xs, ys, staircase)
    n_star = greedy["n_greedy"]
    for budget in (0, w.B, n_star - 7, n_star, n_star + 13, w.B + w.B * w.K, 10 ** 6):
        compare(oracle_mod, run_gpu(z, temps, xs, ys, staircase, budget=budget), z, temps, xs, ys,
                staircase, budget=budget)


@pytest.mark.parametrize("B,K", [(1, 1), (3, 4), (37, 5), (130, 7)])
def test_small_and_ragged(oracle_mod, B, K):
    assert D.dspark_prefix_path(B, K, True) == "single-cta"
    g = torch.Generator(device="cuda").manual_seed(B * 31 + K)
    z = torch.randn(B, K, generator=g, device="cuda").add_(1.0)
    temps = WL.seq_temps(K).cuda()
    xs, ys = (t.cuda() for t in WL.cost_table())
    for staircase in (False, True):
        for budget in (None, B + (B * K) // 2):
            compare(oracle_mod, run_gpu(z, temps, xs, ys, staircase, budget=budget), z, temps, xs,
                    ys, staircase, budget=budget)
        compare(oracle_mod, run_gpu(z, temps, xs, ys, staircase, enable=False), z, temps, xs, ys,
                staircase, enable=False)


@pytest.mark.parametrize("B,K", [(512, 16), (256, 6), (129, 8), (100, 81), (1, 4096),
                                 (8192, 1)])
def test_one_workspace_many_calls(oracle_mod, B, K):
    """Calls in a row on one workspace that starts as garbage, each with new
    confidences.  Above 1024 candidates the cut runs as several CTAs that
    pass the survivals and the order through the workspace: a read of what
    an earlier call left there shows up as a wrong cut here."""
    assert D.dspark_prefix_path(B, K, True) == "multi-cta"
    temps = WL.seq_temps(K).cuda()
    xs, ys = (t.cuda() for t in WL.cost_table())
    ws = torch.full((D.dspark_prefix_workspace_size(B, K, xs.numel()),), 0xA5, dtype=torch.uint8,
                    device="cuda")
    g = torch.Generator(device="cuda").manual_seed(B + 7 * K)
    for t in range(4):
        z = torch.randn(B, K, generator=g, device="cuda").mul_(1.0 + 0.3 * t).add_(2.0 - 0.4 * t)
        staircase = t % 2 == 1
        budget = None if t < 3 else B + (B * K) // 3
        compare(oracle_mod, run_gpu(z, temps, xs, ys, staircase, budget=budget, ws=ws), z, temps,
                xs, ys, staircase, budget=budget)
    # the scheduler off: one CTA (of 1024 threads above 1024 candidates)
    assert D.dspark_prefix_path(B, K, False) == "single-cta"
    compare(oracle_mod, run_gpu(z, temps, xs, ys, False, enable=False, ws=ws), z, temps, xs, ys,
            False, enable=False)


def test_large_batch_bad_table_and_nan(oracle_mod):
    """The multi-CTA form (above 1024 candidates) raises the bad-table flag
    as the single CTA does, and the next call clears it.  A NaN confidence
    makes its request's survival NaN from that position on; such candidates
    are placed after every real one, so the cut equals the oracle's with
    those confidences at -inf (survival 0, which never raises the
    objective)."""
    B, K = 256, 6
    temps = WL.seq_temps(K).cuda()
    xs, ys = (t.cuda() for t in WL.cost_table())
    g = torch.Generator(device="cuda").manual_seed(77)
    z = torch.randn(B, K, generator=g, device="cuda").add_(1.5)
    ws = torch.full((D.dspark_prefix_workspace_size(B, K, xs.numel()),), 0x5A, dtype=torch.uint8,
                    device="cuda")
    c = torch.empty(B, K, device="cuda")
    S = torch.empty(B, K, device="cuda")
    L = torch.empty(B, dtype=torch.int32, device="cuda")
    obj = torch.empty(1, device="cuda")
    D.dspark_confidence_prefix(z, temps, xs.flip(0).contiguous(), ys, True, c, S, L, obj, ws)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(ws, None) & D.FLAG_BAD_TABLE
    D.dspark_confidence_prefix(z, temps, xs, ys, True, c, S, L, obj, ws)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(ws, None) == 0
    zn = z.clone()
    zn[3, 2] = float("nan")
    zn[7, 0] = float("nan")
    D.dspark_confidence_prefix(zn, temps, xs, ys, True, c, S, L, obj, ws)
    torch.cuda.synchronize()
    Lg = L.cpu().numpy()
    assert Lg[3] <= 2 and Lg[7] == 0 and np.isfinite(obj.item())
    zi = zn.cpu().numpy().copy()
    zi[np.isnan(zi)] = -np.inf
    r = oracle_mod.prefix_async(zi, temps.cpu().numpy(), xs.cpu().numpy(), ys.cpu().numpy())
    if r["margin"] >= MARGIN:
        assert np.array_equal(Lg, r["L"])
    else:
        assert not cut_problems(oracle_mod, r["S"], xs.cpu().numpy(), ys.cpu().numpy(), Lg)


def test_budget_word_may_be_shared(oracle_mod):
    w = WL.get("serving")
    z = torch.randn(w.B, w.K, device="cuda").add_(1.5)
    temps = WL.seq_temps(w.K).cuda()
    xs, ys = (t.cuda() for t in WL.cost_table())
    g = run_gpu(z, temps, xs, ys, True, budget=w.B + 100, alias=True)
    assert g["L"].sum() == 100  # the old budget was used ...
    r = oracle_mod.prefix_async(z.cpu().numpy(), temps.cpu().numpy(), xs.cpu().numpy(),
                                ys.cpu().numpy(), staircase=True)
    if r["margin"] >= MARGIN:
        assert g["n_greedy"] == r["n_greedy"]  # ... and the new one written in its place


def test_two_steps_back_loop_in_a_graph(oracle_mod):
    """Steps 0 and 1 take their own greedy cut; step t >= 2 verifies the
    greedy N of step t - 2, filled by its own confidences.  Step t reads and
    writes ring slot t % 2; the whole loop replays from one CUDA graph."""
    B, K, T = 256, 6, 6
    temps = WL.seq_temps(K).cuda()
    xs, ys = (t.cuda() for t in WL.cost_table())
    g = torch.Generator(device="cuda").manual_seed(11)
    zs = [torch.randn(B, K, generator=g, device="cuda").mul_(1.0 + 0.2 * t).add_(1.5 - 0.3 * t)
          for t in range(T)]
    ring = torch.zeros(2, dtype=torch.int32, device="cuda")
    c = torch.empty(B, K, device="cuda")
    S = torch.empty(B, K, device="cuda")
    Ls = [torch.empty(B, dtype=torch.int32, device="cuda") for _ in range(T)]
    obj = torch.empty(1, device="cuda")
    ws = torch.zeros(D.dspark_prefix_workspace_size(B, K, 16), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()

    def loop():
        for t in range(T):
            slot = ring[t % 2:t % 2 + 1]
            D.dspark_confidence_prefix_async(zs[t], temps, xs, ys, True, c, S, Ls[t], obj, ws,
                                             staircase=True, budget_in=slot if t >= 2 else None,
                                             budget_out=slot, stream=s)

    with torch.cuda.stream(s):
        loop()
    s.synchronize()
    first = [L.clone() for L in Ls]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        loop()
    ring.zero_()
    graph.replay()
    torch.cuda.synchronize()
    # oracle loop
    args = (temps.cpu().numpy(), xs.cpu().numpy(), ys.cpu().numpy())
    n_star, near = [], False  # after a near-tie, later budgets may differ: stop comparing
    for t in range(T):
        zt = zs[t].cpu().numpy()
        greedy = oracle_mod.prefix_async(zt, *args, staircase=True)
        near |= greedy["margin"] < MARGIN
        r = greedy if t < 2 else oracle_mod.prefix_async(zt, *args, staircase=True,
                                                         budget=n_star[t - 2])
        n_star.append(greedy["n_greedy"])
        near |= r["margin"] < MARGIN
        if not near:
            assert np.array_equal(Ls[t].cpu().numpy(), r["L"]), t
            assert np.array_equal(first[t].cpu().numpy(), r["L"]), t
