"""The LM-head verify (dspark_verify_lmhead) against the oracle's LM-head
verify on the same seeded inputs.

The target logits are hidden [n_rows, dm] . lm_head [V, dm]^T, formed on the
GPU by tcgen05 MMAs and reduced on chip; the oracle forms them in fp64 from
the same bf16 values.  The verified rows are laid out flat and ragged (row
sets of lengths L_b + 1 back to back, as the variable-length verify lays
them out).  Accept uniforms near zero force accepted prefixes and bonus
draws on some requests, ordinary uniforms give early rejections on others.
Rules as for every verify comparison: accepted counts and emitted tokens
bit-exact unless the oracle's margin of that decision is below 1e-6.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL
from speculative_decoding_05_b200.step import DSparkStep

from tests.parity import MARGIN, P_ATOL, host

pytestmark = pytest.mark.gpu


def _bf16_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def run_case(oracle, name, over, dm, lens, keep_bias, tiny_accept):
    w = WL.get(name, **over)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype,
                      keep_bias=keep_bias)
    step.draft(inp)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(step.ws_draft) == 0
    L = np.asarray(lens, np.int32)
    n_rows = int((L + 1).sum())
    row_start = np.concatenate([[0], np.cumsum(L + 1)[:-1]]).astype(np.int64)
    g = torch.Generator(device="cuda").manual_seed(500 + dm + w.B)
    hidden = torch.randn(n_rows, dm, generator=g, device="cuda").to(torch.bfloat16)
    head = (torch.randn(w.V, dm, generator=g, device="cuda") * (3.0 / dm ** 0.5)).to(torch.bfloat16)
    ua = inp["u_accept"].clone()
    for b in tiny_accept:
        ua[b] = 1e-12  # every drafted token passes the ratio test
    vlen = torch.as_tensor(L, device="cuda")
    rs = torch.as_tensor(row_start, device="cuda")
    ws = D.workspace(D.dspark_verify_lmhead_workspace_size(w.V, w.r, w.B, w.K, dm, n_rows), "cuda")
    n_acc = torch.full((w.B,), -7, dtype=torch.int32, device="cuda")
    out = torch.full((w.B, w.K + 1), -7, dtype=torch.int32, device="cuda")
    last = torch.full((w.B,), -7, dtype=torch.int32, device="cuda")
    D.dspark_verify_lmhead(hidden, head, rs, vlen, inp["base"], inp["U"], inp["W"],
                           inp["prev_token"], inp["inv_temp"], step.tokens, step.p_tok,
                           step.ref_max, step.ref_sum, ua, inp["u_res"], n_acc, out, ws,
                           last_token=last, draft_bias=step.draft_bias)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(ws) == 0

    # the oracle: its own draft, then its LM-head verify on the same bf16 values
    U, W = WL.host_uw(inp["U"]), WL.host_uw(inp["W"])
    base, prev, it = host(inp["base"]), host(inp["prev_token"]), host(inp["inv_temp"])
    d = oracle.draft(base, U, W, prev, host(inp["u_draft"]), inv_temp=it)
    tok_g = host(step.tokens)
    near, checked = 0, 0
    ok_req = []
    for b in range(w.B):
        diverged = False
        for k in range(int(L[b])):  # the verified prefix must agree
            if tok_g[b, k] != d["tokens"][b, k]:
                assert d["margin"][b, k] < MARGIN, (b, k)
                near += 1
                diverged = True
                break
            assert abs(host(step.p_tok)[b, k] - d["p_tok"][b, k]) <= P_ATOL
        if not diverged:
            ok_req.append(b)
    v = oracle.verify_lmhead(_bf16_bits(hidden), _bf16_bits(head), row_start, L, base, U, W, prev,
                             d["tokens"], d["p_tok"], host(ua), host(inp["u_res"]), inv_temp=it)
    na_g, out_g, last_g = host(n_acc), host(out), host(last)
    for b in ok_req:
        checked += 1
        if na_g[b] != v["n_acc"][b]:
            assert v["accept_margin"][b] < MARGIN, (b, na_g[b], v["n_acc"][b])
            near += 1
            continue
        if not np.array_equal(out_g[b], v["out_tokens"][b]):
            assert v["res_margin"][b] < MARGIN, (b, out_g[b], v["out_tokens"][b])
            near += 1
            continue
        assert last_g[b] == v["out_tokens"][b, v["n_acc"][b]]
    assert checked >= w.B - 1 and near <= max(1, w.B // 8), (checked, near)
    return na_g, v


def test_lmhead_full_size_ragged(oracle_mod):
    """V = 151936, dm = 4096, three requests with L = 0, 2, 5 (one all-accepted)."""
    na, v = run_case(oracle_mod, "single", dict(B=3, K=5, seed=61), 4096, [0, 2, 5],
                     keep_bias=True, tiny_accept=[2])
    assert na[2] == 5  # the bonus draw from row L_b


def test_lmhead_several_row_blocks_tensor_core_residual(oracle_mod):
    """B = 24 > 16: the draft's tensor-core path, no bias rows (the residual
    re-projects on the tensor cores), about 200 hidden rows (two 128-row blocks)."""
    rng = np.random.default_rng(7)
    lens = rng.integers(0, 17, size=24)
    run_case(oracle_mod, "stress", dict(V=8192, B=24, K=16, seed=62), 256, lens,
             keep_bias=False, tiny_accept=[0, 5, 11])


def test_lmhead_ragged_vocabulary_fp32_draft(oracle_mod):
    """V = 1000 (a ragged last tile), fp32 U / W (CUDA-core draft and residual)."""
    run_case(oracle_mod, "tiny", dict(V=1000, B=5, K=4, seed=63), 128, [4, 0, 1, 3, 2],
             keep_bias=False, tiny_accept=[0])
