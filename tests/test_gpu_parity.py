"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Small shapes (several chunks, a ragged tail, every request) and the five
workloads at full size in the launch configuration the benchmark times
(sampled requests for the large batches).
"""
import numpy as np
import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL
from speculative_decoding_05_b200.step import DSparkStep

from tests.parity import compare_step, host

pytestmark = pytest.mark.gpu


def _run(w, enable=None, seed=None, requests=None, oracle=None, inp=None, keep_bias=None):
    inp = inp or WL.make_inputs(w, device="cuda", seed=seed)
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype,
                      keep_bias=keep_bias)
    en = w.scheduler if enable is None else enable
    step.run(inp, enable_prefix=en)
    torch.cuda.synchronize()
    flags = step.flags()
    assert all(f == 0 for f in flags.values()), flags
    rep = compare_step(oracle, inp, step, en, requests=requests)
    return rep, step, inp


def _assert_ok(rep):
    print(rep)
    assert not rep.failures, rep.failures[:10]
    # near-margin cases are allowed but must stay rare
    assert sum(rep.near.values()) <= max(2, sum(rep.checked.values()) // 200), rep


def test_tiny_full(oracle_mod):
    rep, _, _ = _run(WL.get("tiny"), oracle=oracle_mod)
    _assert_ok(rep)
    assert rep.checked["draft"] == 2 * 4


@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("V,r,B,K", [(1000, 64, 3, 5), (4096, 32, 7, 3), (2056, 256, 16, 4)])
def test_small_shapes(oracle_mod, bf16, V, r, B, K):
    w = WL.get("serving", V=V, r=r, B=B, K=K, uw_bf16=bf16, seed=11 + V + B)
    inp = WL.make_inputs(w, device="cuda")
    inp["prev_token"][0] = -1  # no bias at position 1 for request 0
    rep, _, _ = _run(w, oracle=oracle_mod, inp=inp)
    _assert_ok(rep)
    assert rep.checked["draft"] >= B


@pytest.mark.parametrize("V,r,B,K", [(4096, 64, 40, 3), (1000, 128, 130, 2), (3000, 256, 17, 4),
                                     (2048, 192, 257, 2)])
def test_tensor_core_path(oracle_mod, V, r, B, K):
    """B > 16 with bf16 U/W takes the tcgen05 projection (ragged last
    vocabulary tile, partial request blocks, several request blocks)."""
    w = WL.get("stress", V=V, r=r, B=B, K=K, seed=3 * V + B)
    assert D.dspark_draft_path(V, r, B, K, D.DSPARK_BF16) == "tcgen05"
    inp = WL.make_inputs(w, device="cuda")
    inp["prev_token"][1] = -1
    req = np.unique(np.r_[0, 1, B - 1, np.random.default_rng(V).choice(B, size=min(B, 12), replace=False)])
    rep, _, _ = _run(w, oracle=oracle_mod, inp=inp, requests=req)
    _assert_ok(rep)


@pytest.mark.parametrize("V,r,B,K,keep", [(4096, 64, 3, 5, True), (1000, 128, 1, 4, False),
                                          (20000, 256, 16, 6, True), (151936, 256, 2, 3, False),
                                          (8192, 192, 9, 16, False), (40000, 256, 4, 7, True),
                                          (30000, 128, 5, 5, True), (151936, 256, 1, 5, True),
                                          (9000, 256, 2, 9, False), (300, 256, 1, 3, True)])
def test_persistent_draft(oracle_mod, V, r, B, K, keep):
    """B <= 16 with bf16 U/W: all K positions in one persistent launch
    (resident + streamed W tiles, grid barrier, redundant sampler); the
    verify either reuses the draft's bias rows or re-projects."""
    w = WL.get("stress", V=V, r=r, B=B, K=K, seed=7 * V + B)
    assert D.dspark_draft_path(V, r, B, K, D.DSPARK_BF16) == (
        "persistent-cuda-core" if B <= 2 and r == 256 else "tcgen05-persistent")
    inp = WL.make_inputs(w, device="cuda")
    inp["prev_token"][0] = -1
    rep, step, _ = _run(w, oracle=oracle_mod, inp=inp, keep_bias=keep)
    _assert_ok(rep)
    assert rep.checked["draft"] >= B


def test_graph_capture_matches_eager():
    """A whole step captured in a CUDA graph replays to the same outputs as
    the eager calls (fixed launch shapes, no host synchronisation)."""
    for name, over in [("single", dict(V=16384, K=6, seed=12)), ("batched", dict(V=8192, B=40, K=3, seed=13))]:
        w = WL.get(name, **over)
        inp = WL.make_inputs(w, device="cuda")
        step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
        step.run(inp, enable_prefix=True)
        torch.cuda.synchronize()
        ref = [t.clone() for t in (step.tokens, step.p_tok, step.lse, step.verify_len,
                                    step.n_accepted, step.out_tokens, step.last_token)]
        for t in (step.tokens, step.p_tok, step.out_tokens):
            t.zero_()
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            step.run(inp, enable_prefix=True)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        got = (step.tokens, step.p_tok, step.lse, step.verify_len, step.n_accepted,
               step.out_tokens, step.last_token)
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        assert all(f == 0 for f in step.flags().values())
        del g


def test_temperatures_and_flat_peaked(oracle_mod):
    w = WL.get("stress", V=3072, r=64, B=24, K=6, seed=5)
    rep, _, _ = _run(w, oracle=oracle_mod)
    _assert_ok(rep)
    w = WL.get("batched", V=3072, r=64, B=12, K=5, seed=6)
    rep, _, _ = _run(w, oracle=oracle_mod)
    _assert_ok(rep)


def test_draft_logits_output(oracle_mod):
    w = WL.get("single", V=2048, r=64, B=2, K=3, seed=9)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    dl = torch.empty_like(inp["base"])
    step.draft(inp, draft_logits=dl)
    torch.cuda.synchronize()
    U, W = WL.host_uw(inp["U"]), WL.host_uw(inp["W"])
    tok = host(step.tokens)
    for b in range(w.B):
        x = int(host(inp["prev_token"])[b])
        for k in range(w.K):
            ref = oracle_mod.draft_row(host(inp["base"][b, k]), U, W, x, float(host(inp["inv_temp"])[b]))
            np.testing.assert_allclose(host(dl[b, k]), ref, atol=1e-5, rtol=1e-6)
            x = int(tok[b, k])


@pytest.mark.parametrize("name", ["single", "batched", "serving", "stress"])
def test_full_size(oracle_mod, name):
    w = WL.get(name)
    # every request up to 4; otherwise a seeded sample of 24 (the stress
    # workload's 512 requests are all compared by the 100-step chain test)
    requests = None if w.B <= 4 else np.random.default_rng(0).choice(w.B, size=24, replace=False)
    rep, _, _ = _run(w, oracle=oracle_mod, requests=requests)
    _assert_ok(rep)
    del rep
    torch.cuda.empty_cache()


EDGE_CASES = [
    # (V, r, B, K, verify lengths, prev_token fill or None)
    (512, 16, 1, 1, [0], None),               # one request, one position, nothing verified
    (512, 16, 1, 1, [1], None),               # ... and everything verified
    (516, 16, 2, 3, [3, 0], -1),              # ragged last chunk; no previous token
    (8196, 64, 17, 2, [0, 1, 2] * 5 + [2, 0], None),  # smallest tensor-core batch, ragged tile
    (4100, 256, 3, 4, [4, 0, 2], None),       # persistent tcgen05 draft, ragged vocabulary
]


@pytest.mark.parametrize("V,r,B,K,lens,prev", EDGE_CASES)
def test_edge_cases(oracle_mod, V, r, B, K, lens, prev):
    """Degenerate and ragged shapes, every output compared with the oracle."""
    w = WL.get("single", V=V, r=r, B=B, K=K, seed=30 + B + K + V % 7)
    inp = WL.make_inputs(w, device="cuda")
    if prev is not None:
        inp["prev_token"].fill_(prev)
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    step.draft(inp)
    step.verify_len.copy_(torch.tensor(lens, dtype=torch.int32))
    step.verify(inp)
    torch.cuda.synchronize()
    flags = step.flags()
    assert flags["draft"] == 0 and flags["verify"] == 0, flags
    rep = compare_step(oracle_mod, inp, step, False, verify_len=lens)
    print(step.path, rep)
    assert not rep.failures, rep.failures[:10]
    assert rep.checked["accept"] + rep.skipped == B
    assert sum(rep.near.values()) <= 1, rep


def test_empty_batch_is_noop():
    w = WL.get("single", V=512, r=16, B=1, K=2)
    inp = WL.make_inputs(w, device="cuda")
    ws = D.workspace(D.dspark_draft_workspace_size(512, 16, 0, 2), "cuda")
    e = torch.empty(0, 2, device="cuda")
    D.dspark_draft_markov(inp["base"][:0], inp["U"], inp["W"], inp["prev_token"][:0], None,
                          e, e.int(), e, e, e, e, ws)
    assert D.dspark_get_device_flags(ws) == 0


def test_device_flags_on_bad_data():
    w = WL.get("single", V=1024, r=16, B=4, K=3, seed=40)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    step.draft(inp)
    step.prefix(inp, enable=False)
    step.tokens[1, 0] = w.V + 7      # out-of-range token id
    step.verify_len[2] = w.K + 5     # out-of-range verify length
    step.verify(inp)
    f = D.dspark_get_device_flags(step.ws_verify)
    assert f & D.FLAG_BAD_TOKEN and f & D.FLAG_BAD_LENGTH
    assert D.dspark_get_device_status(step.ws_verify) == 5
    bad = inp["inv_temp"].clone()
    bad[0] = 0.0
    inp2 = dict(inp, inv_temp=bad)
    step.draft(inp2)
    assert D.dspark_get_device_flags(step.ws_draft) & D.FLAG_BAD_TEMP
    xs = inp["cost_tokens"].flip(0).contiguous()
    step.prefix(dict(inp, cost_tokens=xs), enable=True)
    assert D.dspark_get_device_flags(step.ws_prefix) & D.FLAG_BAD_TABLE
    # a clean call clears the status word again
    step.draft(inp)
    assert D.dspark_get_device_flags(step.ws_draft) == 0
