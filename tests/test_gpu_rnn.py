"""The RNN-head draft (dspark_draft_rnn) and the verify of its drafts,
against the oracle's RNN head on the same seeded inputs.

State s_k = tanh(R s_{k-1} + U[x_{k-1}]) from h0, bias s_k . W^T, then the
Markov head's softmax and inverse CDF (freeaitool.com "DeepSeek DSpark
complete guide" 3.1 names the head; the recurrence is this library's
reading).  The verify takes the draft's bias rows (the RNN head's own rows
at a rejected position).  Rules as everywhere: tokens, accepted counts and
emitted tokens bit-exact unless the oracle's margin is below 1e-6;
probabilities within 1e-5; log-partitions within 1e-3 relative; the states
within 1e-5 (fp32 against fp64).
"""
import numpy as np
import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL

from tests.parity import LSE_RTOL, MARGIN, P_ATOL, host

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def run_case(oracle, name, over, with_h0=True):
    w = WL.get(name, **over)
    inp = WL.make_inputs(w, device="cuda")
    B, K, V, r = w.B, w.K, w.V, w.r
    g = torch.Generator(device="cuda").manual_seed(900 + V + B)
    R = (torch.randn(r, r, generator=g, device="cuda") * (0.8 / r ** 0.5)).to(torch.bfloat16)
    h0 = (torch.randn(B, r, generator=g, device="cuda") * 0.5) if with_h0 else None
    f32, i32 = torch.float32, torch.int32
    tokens = torch.full((B, K), -7, dtype=i32, device="cuda")
    p_tok, lse, rmax, rsum = (torch.empty(B, K, dtype=f32, device="cuda") for _ in range(4))
    states = torch.empty(B, K, r, dtype=f32, device="cuda")
    bias = torch.empty(B, K, V, dtype=f32, device="cuda")
    ws = D.workspace(D.dspark_draft_rnn_workspace_size(V, r, B, K), "cuda")
    D.dspark_draft_rnn(inp["base"], inp["U"], inp["W"], R, inp["prev_token"], h0, inp["inv_temp"],
                       inp["u_draft"], tokens, p_tok, lse, rmax, rsum, ws, states=states,
                       draft_bias=bias)
    # the verify of the RNN draft, with its bias rows (full block)
    vlen = torch.full((B,), K, dtype=i32, device="cuda")
    n_acc = torch.empty(B, dtype=i32, device="cuda")
    out = torch.empty(B, K + 1, dtype=i32, device="cuda")
    last = torch.empty(B, dtype=i32, device="cuda")
    wsv = D.workspace(D.dspark_verify_workspace_size(V, r, B, K), "cuda")
    D.dspark_verify(inp["target"], inp["row_start"], vlen, inp["base"], inp["U"], inp["W"],
                    inp["prev_token"], inp["inv_temp"], tokens, p_tok, rmax, rsum,
                    inp["u_accept"], inp["u_res"], n_acc, out, wsv, last_token=last,
                    draft_bias=bias)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(ws) == 0 and D.dspark_get_device_flags(wsv) == 0

    U, W, Rh = WL.host_uw(inp["U"]), WL.host_uw(inp["W"]), _bits(R)
    base, prev, it = host(inp["base"]), host(inp["prev_token"]), host(inp["inv_temp"])
    h0h = None if h0 is None else host(h0)
    d = oracle.draft_rnn(base, U, W, Rh, prev, host(inp["u_draft"]), h0=h0h, inv_temp=it,
                         states=True)
    tg, pg, lg, sg = host(tokens), host(p_tok), host(lse), host(states)
    near, keep = 0, []
    for b in range(B):
        ok = True
        for k in range(K):
            assert np.abs(sg[b, k] - d["states"][b, k]).max() < 1e-5, (b, k)
            if tg[b, k] != d["tokens"][b, k]:
                assert d["margin"][b, k] < MARGIN, (b, k, d["margin"][b, k])
                near += 1
                ok = False
                break
            assert abs(pg[b, k] - d["p_tok"][b, k]) <= P_ATOL, (b, k)
            assert abs(lg[b, k] - d["lse"][b, k]) <= LSE_RTOL * max(1.0, abs(d["lse"][b, k]))
        if ok:
            keep.append(b)
    keep = np.asarray(keep)
    rs = host(inp["row_start"])
    v = oracle.verify_rnn(host(inp["target"]), rs, np.full(B, K, np.int32), base, U, W, Rh, prev,
                          d["tokens"], d["p_tok"], host(inp["u_accept"]), host(inp["u_res"]),
                          h0=h0h, inv_temp=it)
    na, og, lg2 = host(n_acc), host(out), host(last)
    for b in keep:
        if na[b] != v["n_acc"][b]:
            assert v["accept_margin"][b] < MARGIN, b
            near += 1
            continue
        if not np.array_equal(og[b], v["out_tokens"][b]):
            assert v["res_margin"][b] < MARGIN, (b, og[b], v["out_tokens"][b])
            near += 1
            continue
        assert lg2[b] == v["out_tokens"][b, v["n_acc"][b]]
    assert near <= max(2, B * K // 200), near
    return d


@pytest.mark.parametrize("name,over,with_h0", [
    ("serving", dict(V=4096, r=64, B=5, K=6, seed=71), True),        # small batch
    ("stress", dict(V=8192, r=256, B=130, K=4, seed=72), True),      # two request blocks
    ("stress", dict(V=1000, r=128, B=17, K=3, seed=73), False),      # ragged tile, h0 = 0
    ("single", dict(B=2, K=8, seed=74), True),                       # V = 151936, r = 256
])
def test_rnn_draft_and_verify(oracle_mod, name, over, with_h0):
    run_case(oracle_mod, name, over, with_h0)

