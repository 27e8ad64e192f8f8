"""Pins of the oracle's verify with target logits formed from hidden states
and the LM head (the first step of the fused LM-head verify).

- identity head (dm = V, E = I) gives exactly the verify on the hidden rows;
- small-integer hidden states and head make H E^T exact in fp32, so the
  LM-head verify equals the verify on that product, bit for bit, margins
  included (a transposed head, a wrong stride or a missing 1/T fails);
- the same integers stored in bf16 give the same result;
- scaling H by 2 and E by 1/2 (exact) changes nothing.
"""
import numpy as np
import pytest

from speculative_decoding_05_b200 import workloads as WL


def setup(seed, V=96, r=16, B=3, K=4):
    w = WL.get("tiny", V=V, r=r, B=B, K=K, seed=seed)
    inp = WL.make_inputs(w, device="cpu")
    h = {k: v.numpy() for k, v in inp.items()}
    # per-request temperatures other than 1, so the 1/T scaling is exercised
    h["inv_temp"] = np.array([0.8, 1.25, 1.5, 0.6][:B], np.float32)
    return w, h


def draft(oracle_mod, h):
    return oracle_mod.draft(h["base"], h["U"], h["W"], h["prev_token"], h["u_draft"],
                            inv_temp=h["inv_temp"])


def verify_both(oracle_mod, h, d, target, hidden, head, L):
    args = (h["row_start"], L, h["base"], h["U"], h["W"], h["prev_token"], d["tokens"],
            d["p_tok"], h["u_accept"], h["u_res"])
    a = oracle_mod.verify(target, *args, inv_temp=h["inv_temp"])
    b = oracle_mod.verify_lmhead(hidden, head, *args, inv_temp=h["inv_temp"])
    return a, b


def same(a, b):
    for k in ("n_acc", "out_tokens", "accept_margin", "res_margin"):
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("seed", [1, 2])
def test_identity_head(oracle_mod, seed):
    w, h = setup(seed)
    d = draft(oracle_mod, h)
    hidden = h["target"].astype(np.float32)
    head = np.eye(w.V, dtype=np.float32)
    L = np.full(w.B, w.K, np.int32)
    a, b = verify_both(oracle_mod, h, d, hidden, hidden, head, L)
    same(a, b)


@pytest.mark.parametrize("seed", [3, 4, 5])
def test_exact_integer_factorisation(oracle_mod, seed):
    w, h = setup(seed)
    d = draft(oracle_mod, h)
    rng = np.random.default_rng(seed)
    dm = 24
    n_rows = h["target"].shape[0]
    H = rng.integers(-3, 4, (n_rows, dm)).astype(np.float32)
    E = rng.integers(-2, 3, (w.V, dm)).astype(np.float32)
    T = (H.astype(np.float64) @ E.T.astype(np.float64)).astype(np.float32)
    assert np.array_equal(T.astype(np.float64), H.astype(np.float64) @ E.T)  # exact
    L = np.array([w.K, 1, 0][: w.B], np.int32)
    a, b = verify_both(oracle_mod, h, d, T, H, E, L)
    same(a, b)
    # bf16 storage of the same small integers (exact)
    import torch
    Hb = torch.from_numpy(H).to(torch.bfloat16)
    Eb = torch.from_numpy(E).to(torch.bfloat16)
    _, c = verify_both(oracle_mod, h, d, T, WL.host_uw(Hb), WL.host_uw(Eb), L)
    same(a, c)
    # scaling H by 2 and E by 1/2 leaves every product unchanged
    _, e = verify_both(oracle_mod, h, d, T, H * 2, E * 0.5, L)
    same(a, e)


def test_mismatched_widths_are_refused(oracle_mod):
    w, h = setup(6)
    d = draft(oracle_mod, h)
    H = np.zeros((h["target"].shape[0], 8), np.float32)
    E = np.zeros((w.V, 9), np.float32)
    with pytest.raises(ValueError):
        verify_both(oracle_mod, h, d, h["target"], H, E, np.full(w.B, w.K, np.int32))
