"""dspark_verify_noalloc against dspark_verify.

Some callers cannot call cudaMalloc: plugins whose host application owns
every device allocation and hands out no scratch, runtimes that run under a
fixed device-memory budget decided before the first step.  For them the
library offers dspark_verify_noalloc, whose scratch is a fixed 2 MiB array
inside the library image instead of a caller-provided workspace.

These tests check that it returns exactly what the regular verify returns
(integer outputs, so bit for bit), on two calls in a row with different
uniforms (the second call finds the first call's leftovers in the shared
scratch), that its status query reports the device's data checks, and that a
problem too large for the scratch is refused before anything is enqueued.
This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes

import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL
from speculative_decoding_05_b200.step import DSparkStep

pytestmark = pytest.mark.gpu


def _noalloc(inp, step, u_accept, u_res):
    na = torch.full_like(step.n_accepted, -7)
    out = torch.full_like(step.out_tokens, -7)
    last = torch.full_like(step.last_token, -7)
    D.dspark_verify_noalloc(inp["target"], inp["row_start"], step.verify_len, inp["base"],
                            inp["U"], inp["W"], inp["prev_token"], inp["inv_temp"], step.tokens,
                            step.p_tok, step.ref_max, step.ref_sum, u_accept, u_res, na, out,
                            last_token=last, draft_bias=step.draft_bias)
    return na, out, last


@pytest.mark.parametrize("name,over", [
    ("single", {}),                                      # B=1, K=16, reuses the draft's bias rows
    ("stress", dict(V=8192, B=24, K=4, seed=77)),        # B>16: tensor-core residual, scheduler on
    ("tiny", {}),                                        # fp32 U/W, CUDA-core residual
])
def test_noalloc_verify_matches_workspace_verify(name, over):
    w = WL.get(name, **over)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    step.draft(inp)
    step.prefix(inp, w.scheduler)
    for call in range(2):
        g = torch.Generator(device="cuda").manual_seed(1000 + call)
        ua = torch.rand(w.B, w.K, generator=g, device="cuda")
        ur = torch.rand(w.B, generator=g, device="cuda")
        step.verify(dict(inp, u_accept=ua, u_res=ur))
        torch.cuda.synchronize()
        ref = (step.n_accepted.clone(), step.out_tokens.clone(), step.last_token.clone())
        got = _noalloc(inp, step, ua, ur)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b), (name, call)
        assert D.dspark_verify_noalloc_status() == 0


def test_noalloc_status_reports_bad_data():
    """Out-of-range token ids and verify lengths are clamped on the device
    and reported through the status query; a clean call clears it again."""
    w = WL.get("single", V=1024, r=16, B=4, K=3, seed=40)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    step.draft(inp)
    step.prefix(inp, enable=False)
    good_tokens, good_len = step.tokens.clone(), step.verify_len.clone()
    step.tokens[1, 0] = w.V + 7
    step.verify_len[2] = w.K + 5
    _noalloc(inp, step, inp["u_accept"], inp["u_res"])
    assert D.dspark_verify_noalloc_status() == 5  # DSPARK_ERR_DEVICE_DATA
    step.tokens.copy_(good_tokens)
    step.verify_len.copy_(good_len)
    _noalloc(inp, step, inp["u_accept"], inp["u_res"])
    assert D.dspark_verify_noalloc_status() == 0


def test_noalloc_refuses_oversized_problems():
    """V=151936, B=64, K=8 needs about 2.5 MB of scratch: refused with
    DSPARK_ERR_UNSUPPORTED before any pointer is touched or work enqueued."""
    V, r, B, K = 151936, 256, 64, 8
    assert D.dspark_verify_workspace_size(V, r, B, K) > (2 << 20)
    lib = D.load()
    P = ctypes.c_void_p
    p = P(1 << 23)  # never dereferenced: the size check comes first
    rc = lib.dspark_verify_noalloc(p, 10, p, p, p, p, p, D.DSPARK_BF16, V, r, B, K, p, None, p, p,
                                   p, p, None, p, p, p, p, None, None)
    assert rc == 4
