"""dspark_sts_fit (CUDA, through the C ABI) against the oracle.

Temperatures: the kernels search in fp64 and round T to fp32, the oracle
keeps fp64; the searches take the same steps except where a derivative
is within rounding of zero (the last bracket is then already far below
fp32 resolution), so T agrees to 3e-7 relative.  ECE: one pair whose
confidence lies within an ulp of a bin edge may fall in the neighbouring
bin on the other side (exp differs by an ulp), which moves the ECE by at
most 2 / pairs; fp32 output adds 1e-7 relative.
"""
import numpy as np
import pytest
import torch

from speculative_decoding_05_b200 import dspark as D
from speculative_decoding_05_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def fit_gpu(z, n_acc):
    N, K = z.shape
    ws = torch.zeros(D.dspark_sts_workspace_size(N, K), dtype=torch.uint8, device="cuda")
    temps = torch.empty(K, dtype=torch.float32, device="cuda")
    ece = torch.empty(2, dtype=torch.float32, device="cuda")
    D.dspark_sts_fit(z, n_acc, temps, ece, ws)
    torch.cuda.synchronize()
    return temps.cpu().numpy(), ece.cpu().numpy(), D.dspark_get_device_flags(ws, None)


def check(oracle_mod, z, n_acc, expect_flags=0):
    t_gpu, e_gpu, flags = fit_gpu(z, n_acc)
    r = oracle_mod.sts_fit(z.cpu().numpy(), n_acc.cpu().numpy())
    assert flags == expect_flags
    np.testing.assert_allclose(t_gpu, r["temps"], rtol=3e-7, atol=0)
    pairs = max(1, int(r["count"].sum()))
    tol = 2.0 / pairs + 1e-7
    assert abs(e_gpu[0] - r["ece_before"]) <= tol, (e_gpu, r)
    assert abs(e_gpu[1] - r["ece_after"]) <= tol, (e_gpu, r)
    return t_gpu, e_gpu, r


@pytest.mark.parametrize("name", ["calibration_small", "calibration"])
def test_calibration_sets(oracle_mod, name):
    c = WL.CALIBRATIONS[name]
    d = WL.make_calibration(c, device="cuda")
    t, e, r = check(oracle_mod, d["z"], d["n_acc"])
    assert e[1] < e[0]


def test_pass_count_is_reported():
    d = WL.make_calibration(WL.CALIBRATIONS["calibration_small"], device="cuda")
    N, K = d["z"].shape
    ws = torch.zeros(D.dspark_sts_workspace_size(N, K), dtype=torch.uint8, device="cuda")
    temps = torch.empty(K, device="cuda")
    ece = torch.empty(2, device="cuda")
    passes = torch.zeros(1, dtype=torch.int32, device="cuda")
    D.dspark_sts_fit(d["z"], d["n_acc"], temps, ece, ws, passes=passes)
    torch.cuda.synchronize()
    # two bound evaluations, a few Newton steps, two ECE passes; never the 44 maximum here
    assert 5 <= int(passes.item()) < 30, int(passes.item())


@pytest.mark.parametrize("N,K,seed", [(1, 1, 1), (7, 3, 2), (4096 + 13, 5, 3), (777, 32, 4),
                                      (75_000, 2, 5), (300, 16, 6)])
def test_ragged_sizes(oracle_mod, N, K, seed):
    d = WL.make_calibration(WL.Calibration("t", N=N, K=K, seed=seed), device="cuda")
    check(oracle_mod, d["z"], d["n_acc"])


def test_empty_set(oracle_mod):
    z = torch.zeros(0, 4, dtype=torch.float32, device="cuda")
    n_acc = torch.zeros(0, dtype=torch.int32, device="cuda")
    t, e, _ = check(oracle_mod, z, n_acc)
    assert np.all(t == 1.0) and np.all(e == 0.0)


def test_degenerate_positions(oracle_mod):
    g = torch.Generator(device="cuda").manual_seed(3)
    N, K = 5000, 4
    z = torch.rand(N, K, generator=g, device="cuda") + 0.5   # all scores > 0
    z[:, 3] = 0.0                                              # position 3: no information
    n_acc = torch.full((N,), 3, dtype=torch.int32, device="cuda")
    n_acc[: N // 2] = 4
    # position 0..2: always accepted with z > 0 -> T on the lower bound
    t, _, _ = check(oracle_mod, z, n_acc)
    assert np.all(np.abs(t[:3] - 0.05) < 1e-7) and t[3] == 1.0
    t, _, _ = check(oracle_mod, z, torch.zeros(N, dtype=torch.int32, device="cuda"))
    assert abs(t[0] - 20.0) < 1e-5 and np.all(t[1:] == 1.0)  # nobody reached 1..3


def test_bad_data_is_flagged_and_left_out(oracle_mod):
    d = WL.make_calibration(WL.Calibration("t", N=3000, K=6, seed=9), device="cuda")
    z, n_acc = d["z"].clone(), d["n_acc"].clone()
    z[10, 0] = float("nan")
    z[11, 0] = float("inf")
    check(oracle_mod, z, n_acc, expect_flags=D.FLAG_NONFINITE)
    n_acc[5] = 9
    n_acc[6] = -3
    check(oracle_mod, z, n_acc, expect_flags=D.FLAG_NONFINITE | D.FLAG_BAD_LENGTH)


def test_runs_are_bitwise_repeatable():
    d = WL.make_calibration(WL.CALIBRATIONS["calibration_small"], device="cuda")
    a = fit_gpu(d["z"], d["n_acc"])
    b = fit_gpu(d["z"], d["n_acc"])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fitted_temperatures_feed_the_prefix_cut():
    """The fit's output is the temps argument of dspark_confidence_prefix."""
    d = WL.make_calibration(WL.CALIBRATIONS["calibration_small"], device="cuda")
    t, _, _ = fit_gpu(d["z"], d["n_acc"])
    B, K = 8, 16
    z = torch.randn(B, K, device="cuda") + 1.5
    temps = torch.tensor(t, device="cuda")
    xs, ys = WL.cost_table()
    c = torch.empty(B, K, device="cuda")
    S = torch.empty(B, K, device="cuda")
    L = torch.empty(B, dtype=torch.int32, device="cuda")
    obj = torch.empty(1, device="cuda")
    ws = torch.zeros(D.dspark_prefix_workspace_size(B, K, 16), dtype=torch.uint8, device="cuda")
    D.dspark_confidence_prefix(z, temps, xs.cuda(), ys.cuda(), True, c, S, L, obj, ws)
    torch.cuda.synchronize()
    expect = torch.sigmoid(z.double() / temps.double()).float()
    assert torch.allclose(c, expect, rtol=1e-6, atol=1e-7)
