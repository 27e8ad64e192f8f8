"""Compare GPU steps with the oracle on the same seeded inputs.

Rules (the tolerances every comparison uses):
  * sampled / accepted tokens and prefix lengths bit-exact, except where the
    oracle's margin of that decision is below 1e-6; such cases are counted
    and reported, and the rest of that request's draft is not compared
    (later positions condition on a different token);
  * probabilities within 1e-5 absolute, log-probabilities within 1e-3
    relative.
The oracle receives host copies of the inputs only; nothing it reads comes
from the CUDA path's outputs.
"""
from __future__ import annotations

import numpy as np
import torch

from speculative_decoding_05_b200.workloads import host_uw

MARGIN = 1e-6
P_ATOL = 1e-5
LSE_RTOL = 1e-3


def host(t):
    return t.detach().cpu().numpy()


class Report:
    def __init__(self):
        self.checked = dict(draft=0, prefix=0, accept=0, residual=0)
        self.near = dict(draft=0, prefix=0, accept=0, residual=0)
        self.skipped = 0
        self.failures = []
        # request -> the token the oracle emitted last (its next prev_token),
        # for requests whose whole step was compared
        self.oracle_last = {}

    def fail(self, msg):
        self.failures.append(msg)

    def merge(self, other):
        for k in self.checked:
            self.checked[k] += other.checked[k]
            self.near[k] += other.near[k]
        self.skipped += other.skipped
        self.failures += other.failures

    def __repr__(self):
        return f"checked={self.checked} near_margin={self.near} skipped={self.skipped} failures={len(self.failures)}"


def host_inputs(inp, requests):
    """Host copies of one step's inputs for `requests`: the per-request
    logit rows (base [n,K,V], target rows [n][L+1 <= K+1, V] are taken from
    row_start), U, W, inverse temperatures, uniforms and prev_token."""
    requests = np.asarray(requests)
    dev = inp["base"].device
    idx = torch.as_tensor(requests, device=dev)
    K = inp["base"].shape[1]
    rs = host(inp["row_start"])
    rows = np.concatenate([np.arange(rs[b], rs[b] + K + 1) for b in requests]) if len(requests) \
        else np.zeros(0, np.int64)
    tgt = host(inp["target"].index_select(0, torch.as_tensor(rows, device=dev)))
    return dict(requests=requests, base=host(inp["base"].index_select(0, idx)),
                target=tgt.reshape(len(requests), K + 1, -1),
                U=host_uw(inp["U"]), W=host_uw(inp["W"]),
                inv_temp=host(inp["inv_temp"].index_select(0, idx)),
                prev_token=host(inp["prev_token"].index_select(0, idx)),
                u_draft=host(inp["u_draft"].index_select(0, idx)),
                u_accept=host(inp["u_accept"].index_select(0, idx)),
                u_res=host(inp["u_res"].index_select(0, idx)))


def gpu_outputs(step, requests):
    """Host copies of the outputs a DSparkStep holds, for `requests`."""
    idx = torch.as_tensor(np.asarray(requests), device=step.tokens.device)
    pick = lambda t: host(t.index_select(0, idx))
    return dict(tokens=pick(step.tokens), p_tok=pick(step.p_tok), lse=pick(step.lse),
                verify_len=pick(step.verify_len), n_accepted=pick(step.n_accepted),
                out_tokens=pick(step.out_tokens), last_token=pick(step.last_token))


def compare_requests(oracle, h, g, L_or, rep=None):
    """Oracle draft and verify of the requests in `h` (host inputs, see
    host_inputs) against the GPU outputs `g` (see gpu_outputs), both sides
    verifying the oracle's lengths L_or where the GPU's agree."""
    rep = rep or Report()
    requests = h["requests"]
    n = len(requests)
    if n == 0:
        return rep
    K = h["base"].shape[1]
    L_or = np.asarray(L_or, np.int32)
    L_gpu = g["verify_len"]
    d = oracle.draft(h["base"], h["U"], h["W"], h["prev_token"], h["u_draft"],
                     inv_temp=h["inv_temp"])
    tok_g, p_g, lse_g = g["tokens"], g["p_tok"], g["lse"]
    match_len = np.full(n, K)
    for i in range(n):
        for k in range(K):
            rep.checked["draft"] += 1
            if tok_g[i, k] != d["tokens"][i, k]:
                if d["margin"][i, k] < MARGIN:
                    rep.near["draft"] += 1
                else:
                    rep.fail(f"draft b={requests[i]} k={k}: token {tok_g[i, k]} != "
                             f"{d['tokens'][i, k]} (margin {d['margin'][i, k]:.3g})")
                match_len[i] = k
                break
            if abs(p_g[i, k] - d["p_tok"][i, k]) > P_ATOL:
                rep.fail(f"draft b={requests[i]} k={k}: p_tok {p_g[i, k]} vs {d['p_tok'][i, k]}")
            if abs(lse_g[i, k] - d["lse"][i, k]) > LSE_RTOL * max(1.0, abs(d["lse"][i, k])):
                rep.fail(f"draft b={requests[i]} k={k}: lse {lse_g[i, k]} vs {d['lse'][i, k]}")

    # verify: requests whose verified draft prefix and L agree
    keep = np.asarray([i for i in range(n) if match_len[i] >= L_or[i] and L_or[i] == L_gpu[i]],
                      dtype=np.int64)
    rep.skipped += n - len(keep)
    if len(keep) == 0:
        return rep
    Lk = L_or[keep]
    tgt = np.concatenate([h["target"][i, :L + 1] for i, L in zip(keep, Lk)])
    rs_sub = np.concatenate([[0], np.cumsum(Lk + 1)[:-1]]).astype(np.int64)
    v = oracle.verify(tgt, rs_sub, Lk, h["base"][keep], h["U"], h["W"], h["prev_token"][keep],
                      d["tokens"][keep], d["p_tok"][keep], h["u_accept"][keep],
                      h["u_res"][keep], inv_temp=h["inv_temp"][keep])
    na_g, out_g, last_g = g["n_accepted"][keep], g["out_tokens"][keep], g["last_token"][keep]
    for i, b in enumerate(requests[keep]):
        rep.checked["accept"] += 1
        if na_g[i] != v["n_acc"][i]:
            if v["accept_margin"][i] < MARGIN:
                rep.near["accept"] += 1
            else:
                rep.fail(f"verify b={b}: n_acc {na_g[i]} != {v['n_acc'][i]} "
                         f"(margin {v['accept_margin'][i]:.3g})")
            continue
        rep.checked["residual"] += 1
        if not np.array_equal(out_g[i], v["out_tokens"][i]):
            na = v["n_acc"][i]
            same_prefix = np.array_equal(out_g[i, :na], v["out_tokens"][i, :na]) and \
                np.all(out_g[i, na + 1:] == -1)
            if same_prefix and v["res_margin"][i] < MARGIN:
                rep.near["residual"] += 1
            else:
                rep.fail(f"verify b={b}: out {out_g[i].tolist()} != {v['out_tokens'][i].tolist()} "
                         f"(margin {v['res_margin'][i]:.3g})")
            continue
        if last_g[i] != v["out_tokens"][i, v["n_acc"][i]]:
            rep.fail(f"verify b={b}: last_token {last_g[i]}")
            continue
        rep.oracle_last[int(b)] = int(v["out_tokens"][i, v["n_acc"][i]])
    return rep


def cut_problems(oracle, S, cost_tokens, cost_ms, L_g, staircase=False, budget=None,
                 tol=MARGIN):
    """Why the verify lengths L_g are not a cut the method could have made:
    the empty list when they are one.  For where the oracle's own stopping
    decision lies inside the margin, so the GPU may stop elsewhere.

    The candidates in the oracle's order (survival S descending, then k,
    then b; S from the oracle, fp64) must give L_g as the per-request counts
    of the first N = sum(L_g) of them (a swap across the cut of two
    survivals equal to 1e-9 relative is allowed: the two sides' exp may
    differ by an ulp).  Greedy cut (budget None): the objective E/t(N) of
    the oracle's order may fall by at most tol (relative) at every step
    before N, and may rise by at most tol at the step after it.  Budget cut:
    N = the budget minus B, clamped to [0, B*K]."""
    B, K = S.shape
    n = B * K
    L_g = np.asarray(L_g)
    kk, bb = np.meshgrid(np.arange(K), np.arange(B))
    order = np.lexsort((bb.ravel(), kk.ravel(), -S.ravel()))
    s_sorted = S.ravel()[order]
    b_sorted = bb.ravel()[order]
    N = int(L_g.sum())
    if L_g.min(initial=0) < 0 or L_g.max(initial=0) > K or not 0 <= N <= n:
        return [f"lengths out of range (sum {N})"]
    problems = []
    counts = np.bincount(b_sorted[:N], minlength=B)
    if not np.array_equal(counts, L_g):
        d = L_g - counts
        swap = (0 < N < n and np.abs(d).sum() == 2 and d[b_sorted[N]] == 1
                and d[b_sorted[N - 1]] == -1
                and abs(s_sorted[N - 1] - s_sorted[N]) <= 1e-9 * s_sorted[N - 1])
        if not swap:
            problems.append(f"lengths are not the first {N} candidates of the order")
    if budget is not None:
        want = min(max(int(budget) - B, 0), n)
        if N != want:
            problems.append(f"budget cut of {want} candidates, got {N}")
        return problems
    cost = oracle.cost_stair_ms if staircase else oracle.cost_ms
    E = B + np.concatenate([[0.0], np.cumsum(s_sorted)])
    t = np.array([cost(cost_tokens, cost_ms, B + m) for m in range(n + 1)])
    obj = E / t
    falls = np.nonzero(obj[1:N + 1] < obj[:N] * (1.0 - tol))[0]
    if falls.size:
        problems.append(f"went on past a clear fall of the objective at {int(falls[0])} (cut {N})")
    if N < n and obj[N + 1] > obj[N] * (1.0 + tol):
        problems.append(f"stopped at {N} while the objective still rose")
    return problems


def compare_prefix(oracle, inp, step, enable_prefix, rep):
    """The prefix cut over the whole batch (it is global over requests);
    returns the oracle's verify lengths."""
    pr = oracle.prefix(host(inp["z"]), host(inp["temps"]), host(inp["cost_tokens"]),
                       host(inp["cost_ms"]), enable=enable_prefix)
    c_g, s_g = host(step.c), host(step.survival)
    if np.abs(c_g - pr["c"]).max() > P_ATOL or np.abs(s_g - pr["S"]).max() > P_ATOL:
        rep.fail("prefix: c / survival outside 1e-5")
    L_g = host(step.verify_len)
    rep.checked["prefix"] += 1
    if not np.array_equal(L_g, pr["L"]):
        if pr["margin"] < MARGIN:
            # the two sides may stop at different places, but each must
            # still be a greedy cut of the same order
            why = cut_problems(oracle, pr["S"], host(inp["cost_tokens"]), host(inp["cost_ms"]),
                               L_g) if enable_prefix else ["lengths differ with the cut off"]
            if why:
                rep.fail("prefix: " + "; ".join(why))
            else:
                rep.near["prefix"] += 1
        else:
            rep.fail(f"prefix: verify_len differs (margin {pr['margin']:.3g})")
    elif abs(float(host(step.objective)[0]) - pr["objective"]) > 1e-5 * abs(pr["objective"]):
        rep.fail("prefix: objective outside 1e-5 relative")
    return pr["L"]


def compare_step(oracle, inp, step, enable_prefix, requests=None, rep=None, verify_len=None):
    """Run the oracle on `requests` (default: all) and compare with the
    outputs held by `step` (a DSparkStep that has just run on `inp`).
    With `verify_len` (the lengths the caller set by hand) the prefix cut is
    not compared and both sides verify those lengths."""
    rep = rep or Report()
    B, K, V = inp["base"].shape
    if requests is None:
        requests = np.arange(B)
    requests = np.asarray(requests)
    if verify_len is not None:
        L_all = np.asarray(verify_len, np.int32)
    elif K > 0 and B > 0:
        L_all = compare_prefix(oracle, inp, step, enable_prefix, rep)
    else:
        L_all = np.zeros(B, np.int32)
    h = host_inputs(inp, requests)
    g = gpu_outputs(step, requests)
    return compare_requests(oracle, h, g, L_all[requests], rep)
