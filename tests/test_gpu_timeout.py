"""Bounded device waits that run out, on the GPU, without a fault.

Every device wait of the library gives up after 2 s (and at least 4096
polls), raises DSPARK_FLAG_TIMEOUT and lets the kernel unwind: producers
wait for their copies in flight, tensor memory is freed, the call returns.
The test hook dspark_test_set_exchange_skew makes two real exchanges wait
for records that never arrive -- the persistent draft's first one and the
single-launch verify's -- so that path runs for real.  Each test checks
that the call comes back within seconds with the timeout in its status
word, and that the next call on the same device gives the results of a
call made before (the context is still usable).
"""
import time

import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL
from speculative_decoding_05_b200.step import DSparkStep

pytestmark = pytest.mark.gpu


def _timed_out_call(fn, ws):
    D.dspark_test_set_exchange_skew(1)
    try:
        t0 = time.time()
        fn()
        flags = D.dspark_get_device_flags(ws)  # synchronises
        dt = time.time() - t0
    finally:
        D.dspark_test_set_exchange_skew(0)
    return flags, dt


def test_persistent_draft_exchange_timeout():
    w = WL.get("single", V=16384, K=4, seed=91)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    assert step.path == "persistent-cuda-core"
    step.draft(inp)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(step.ws_draft) == 0
    ref = (step.tokens.clone(), step.p_tok.clone())
    flags, dt = _timed_out_call(lambda: step.draft(inp), step.ws_draft)
    assert flags & D.FLAG_TIMEOUT, flags
    assert D.dspark_get_device_status(step.ws_draft) == 3  # DSPARK_ERR_TIMEOUT
    assert dt < 60, dt
    step.draft(inp)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(step.ws_draft) == 0
    assert torch.equal(step.tokens, ref[0]) and torch.equal(step.p_tok, ref[1])


def test_single_launch_verify_exchange_timeout():
    w = WL.get("single", V=16384, B=2, K=4, seed=92)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype)
    assert D.dspark_verify_path(w.V, w.r, w.B, w.K, inp["U"].dtype, True) == "single-launch"
    step.run(inp, enable_prefix=False)
    torch.cuda.synchronize()
    assert all(f == 0 for f in step.flags().values())
    ref = (step.n_accepted.clone(), step.out_tokens.clone())
    flags, dt = _timed_out_call(lambda: step.verify(inp), step.ws_verify)
    assert flags & D.FLAG_TIMEOUT, flags
    assert D.dspark_get_device_status(step.ws_verify) == 3
    assert dt < 60, dt
    step.verify(inp)
    torch.cuda.synchronize()
    assert D.dspark_get_device_flags(step.ws_verify) == 0
    assert torch.equal(step.n_accepted, ref[0]) and torch.equal(step.out_tokens, ref[1])
