"""Compare one GPU step with the oracle on the same seeded inputs.

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

    def fail(self, msg):
        self.failures.append(msg)

    def __repr__(self):
        return f"checked={self.checked} near_margin={self.near} skipped={self.skipped} failures={len(self.failures)}"


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
    idx = torch.as_tensor(requests, device=inp["base"].device)

    # ---- prefix cut: on the whole batch (it is global over requests)
    if verify_len is not None:
        L_or = np.asarray(verify_len, np.int32)[requests]
    elif K > 0 and B > 0:
        pr = oracle.prefix(host(inp["z"]), host(inp["temps"]), host(inp["cost_tokens"]),
                           host(inp["cost_ms"]), enable=enable_prefix)
        c_g, s_g = host(step.c), host(step.survival)
        if np.abs(c_g - pr["c"]).max() > P_ATOL or np.abs(s_g - pr["S"]).max() > P_ATOL:
            rep.fail("prefix: c / survival outside 1e-5")
        L_g = host(step.verify_len)
        rep.checked["prefix"] += 1
        if not np.array_equal(L_g, pr["L"]):
            if pr["margin"] < MARGIN:
                rep.near["prefix"] += 1
            else:
                rep.fail(f"prefix: verify_len differs (margin {pr['margin']:.3g})")
        elif abs(float(host(step.objective)[0]) - pr["objective"]) > 1e-5 * abs(pr["objective"]):
            rep.fail("prefix: objective outside 1e-5 relative")
        L_or = pr["L"][requests]
    else:
        L_or = np.zeros(len(requests), np.int32)
    L_gpu = host(step.verify_len)[requests] if B > 0 else L_or

    # ---- draft on the sampled requests
    U, W = host_uw(inp["U"]), host_uw(inp["W"])
    base = host(inp["base"].index_select(0, idx))
    prev = host(inp["prev_token"].index_select(0, idx))
    it = host(inp["inv_temp"].index_select(0, idx))
    d = oracle.draft(base, U, W, prev, host(inp["u_draft"].index_select(0, idx)), inv_temp=it)
    tok_g = host(step.tokens.index_select(0, idx))
    p_g = host(step.p_tok.index_select(0, idx))
    lse_g = host(step.lse.index_select(0, idx))
    match_len = np.full(len(requests), K)
    for i in range(len(requests)):
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

    # ---- verify: requests whose verified draft prefix and L agree
    keep = [i for i in range(len(requests))
            if match_len[i] >= L_or[i] and L_or[i] == L_gpu[i]]
    rep.skipped += len(requests) - len(keep)
    if not keep:
        return rep
    keep = np.asarray(keep)
    sub = requests[keep]
    sidx = torch.as_tensor(sub, device=inp["base"].device)
    rows = []
    rs_all = host(inp["row_start"])
    for b, L in zip(sub, L_or[keep]):
        rows.append(np.arange(rs_all[b], rs_all[b] + L + 1))
    row_ids = np.concatenate(rows)
    tgt = host(inp["target"].index_select(0, torch.as_tensor(row_ids, device=inp["base"].device)))
    rs_sub = np.concatenate([[0], np.cumsum([len(x) for x in rows])[:-1]]).astype(np.int64)
    v = oracle.verify(tgt, rs_sub, L_or[keep].astype(np.int32), base[keep], U, W, prev[keep],
                      d["tokens"][keep], d["p_tok"][keep],
                      host(inp["u_accept"].index_select(0, sidx)),
                      host(inp["u_res"].index_select(0, sidx)), inv_temp=it[keep])
    na_g = host(step.n_accepted.index_select(0, sidx))
    out_g = host(step.out_tokens.index_select(0, sidx))
    last_g = host(step.last_token.index_select(0, sidx))
    for i, b in enumerate(sub):
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
            n = v["n_acc"][i]
            same_prefix = np.array_equal(out_g[i, :n], v["out_tokens"][i, :n]) and \
                np.all(out_g[i, n + 1:] == -1)
            if same_prefix and v["res_margin"][i] < MARGIN:
                rep.near["residual"] += 1
            else:
                rep.fail(f"verify b={b}: out {out_g[i].tolist()} != {v['out_tokens'][i].tolist()} "
                         f"(margin {v['res_margin'][i]:.3g})")
        elif last_g[i] != v["out_tokens"][i, v["n_acc"][i]]:
            rep.fail(f"verify b={b}: last_token {last_g[i]}")
    return rep
