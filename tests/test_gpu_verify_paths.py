"""Verify of a few requests against the oracle, verify lengths set by hand.

Up to four requests with the draft's bias rows kept take the single-launch
verify; the same inputs without the bias rows take the staged kernels that
re-project the residual row from U and W.  Both are compared with the
oracle on zero, partial, full and mixed verify lengths, on the full
vocabulary of the single-request workload, on a ragged vocabulary and on the
largest single-launch case (B * (K + 1) = 72 verified rows).
"""
import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL
from speculative_decoding_05_b200.step import DSparkStep

from tests.parity import compare_step

pytestmark = pytest.mark.gpu

CASES = [
    (151936, 256, 1, 16, [16]),
    (151936, 256, 1, 16, [0]),
    (151936, 256, 1, 16, [7]),
    (9000, 256, 2, 9, [0, 9]),
    (1024, 16, 4, 3, [3, 1, 0, 2]),
    (300, 256, 3, 5, [5, 2, 4]),
    (4096, 64, 4, 17, [17, 0, 8, 16]),
]


@pytest.mark.parametrize("keep_bias", [True, False])
@pytest.mark.parametrize("V,r,B,K,lens", CASES)
def test_verify_with_given_lengths(oracle_mod, V, r, B, K, lens, keep_bias):
    w = WL.get("single", V=V, r=r, B=B, K=K, seed=60 + B + K)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype,
                      keep_bias=keep_bias)
    expect = "single-launch" if keep_bias else "staged-"
    assert D.dspark_verify_path(V, r, B, K, inp["U"].dtype, keep_bias).startswith(expect)
    step.draft(inp)
    step.verify_len.copy_(torch.tensor(lens, dtype=torch.int32))
    step.verify(inp)
    torch.cuda.synchronize()
    flags = step.flags()
    assert flags["draft"] == 0 and flags["verify"] == 0, flags  # the prefix is not run here
    rep = compare_step(oracle_mod, inp, step, False, verify_len=lens)
    print(rep)
    assert not rep.failures, rep.failures[:10]
    assert rep.checked["accept"] + rep.skipped == B
    assert sum(rep.near.values()) <= 1, rep


def test_single_launch_verify_twice_in_a_row(oracle_mod):
    """Second call on the same workspace: the records of the first call are
    cleared, not mistaken for the second call's."""
    w = WL.get("single", V=151936, r=256, B=2, K=8, seed=71)
    inp = WL.make_inputs(w, device="cuda")
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype, keep_bias=True)
    step.draft(inp)
    torch.cuda.synchronize()
    assert step.flags()["draft"] == 0, step.flags()  # a timed-out exchange would show here
    step.verify_len.fill_(w.K)
    outs = []
    for seed in (1, 2):
        g = torch.Generator(device="cuda").manual_seed(seed)
        inp2 = dict(inp, u_accept=torch.rand(w.B, w.K, generator=g, device="cuda"),
                    u_res=torch.rand(w.B, generator=g, device="cuda"))
        step.verify(inp2)
        torch.cuda.synchronize()
        rep = compare_step(oracle_mod, inp2, step, False, verify_len=[w.K] * w.B)
        assert not rep.failures, rep.failures[:10]
        outs.append(step.out_tokens.clone())
    assert step.flags()["verify"] == 0


PACKED = [
    (9000, 256, 2, 9, [0, 9], True),             # single-launch verify
    (4096, 64, 4, 17, [17, 0, 8, 16], False),    # staged, CUDA-core residual
    (8192, 256, 40, 5, None, False),             # staged, tcgen05 residual
]


@pytest.mark.parametrize("V,r,B,K,lens,keep_bias", PACKED)
def test_packed_target_rows_match_dense(V, r, B, K, lens, keep_bias):
    """The target rows may come packed: request b's L_b + 1 verified rows
    back to back, row_start holding their offsets (what a caller that only
    computes the verified rows passes).  The outputs equal those of the
    full (K + 1)-rows-per-request layout bit for bit."""
    w = WL.get("single", V=V, r=r, B=B, K=K, seed=90 + B + K)
    inp = WL.make_inputs(w, device="cuda")
    if lens is None:
        lens = torch.randint(0, K + 1, (B,), generator=torch.Generator().manual_seed(B)).tolist()
    step = DSparkStep(w.V, w.r, w.B, w.K, inp["target"].shape[0], inp["U"].dtype,
                      keep_bias=keep_bias)
    step.draft(inp)
    step.verify_len.copy_(torch.tensor(lens, dtype=torch.int32))
    step.verify(inp)
    torch.cuda.synchronize()
    dense = [t.clone() for t in (step.n_accepted, step.out_tokens, step.last_token)]
    rows = [L + 1 for L in lens]
    offs = [sum(rows[:b]) for b in range(B)]
    tgt = torch.cat([inp["target"][b * (K + 1):b * (K + 1) + rows[b]] for b in range(B)])
    rs = torch.tensor(offs, dtype=torch.int64, device="cuda")
    step.verify(dict(inp, target=tgt.contiguous(), row_start=rs))
    torch.cuda.synchronize()
    assert step.flags()["verify"] == 0
    for a, b in zip(dense, (step.n_accepted, step.out_tokens, step.last_token)):
        assert torch.equal(a, b)
