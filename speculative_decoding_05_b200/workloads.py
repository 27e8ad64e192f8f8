"""Seeded synthetic inputs for the five DSpark hot-path workloads.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic (no softmax, no sampling, no scheduling).  Both the
CUDA path and the CPU oracle are fed from it: tensors are drawn once (on the
requested device) and the oracle receives host copies of the same tensors.

The pages' own evaluation data (nine offline benchmark datasets and
production traffic) is not available; these seeded tensors stand in for it,
with peaked ("code-like") and flat ("chat-like") requests imitating the two
traffic kinds the pages contrast.

On CUDA the draws come from torch's CUDA generator (Philox4x32-10); on the
CPU from torch's CPU generator.  Draw order per workload: prev_token, U, W,
base (+ peak positions), target noise, z, u_draft, u_accept, u_res.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    V: int
    r: int
    B: int
    K: int
    uw_bf16: bool = True
    uw_var: float = 0.25          # U, W ~ N(0, uw_var / r)
    base_sigma: float = 3.0       # base ~ N(0, base_sigma^2)
    peak: float = 8.0             # one uniformly chosen token per position gets +peak
    split_peaked_flat: bool = False  # first half peaked (sigma 1, +10), second flat (sigma 4)
    target_mode: str = "scaled"   # "noise": base+N(0,.5^2); "scaled": .8 base+N(0,1); "rho"
    temps_per_request: bool = False  # T_b drawn from {0.6, 1.0, 1.3}
    scheduler: bool = False
    steps: int = 1                # sequential steps per run (stress: 100)
    seed: int = 0
    notes: dict = field(default_factory=dict)


WORKLOADS = {
    # V=1024, r=16, B=2, K=4; fp32 U,W ~ N(0,1/r); base ~ N(0,2^2);
    # target = base + N(0,0.5^2); prefix cut off.
    "tiny": Workload("tiny", V=1024, r=16, B=2, K=4, uw_bf16=False, uw_var=1.0,
                     base_sigma=2.0, peak=0.0, target_mode="noise", seed=0),
    # V=151936, r=256, B=1, K=16; bf16 W,U ~ N(0,0.25/r); base N(0,3^2) + one
    # peaked token (+8) per position; target = 0.8 base + N(0,1); full block.
    "single": Workload("single", V=151936, r=256, B=1, K=16, seed=1),
    # B=64, K=8: half peaked (sigma 1, +10), half flat (sigma 4); full block.
    "batched": Workload("batched", V=151936, r=256, B=64, K=8,
                        split_peaked_flat=True, seed=2),
    # V=129280, B=256, K=6, scheduler on (z ~ N(1.5,1), T_k = 1 + 0.1 k,
    # 16-point cost table, linear with a knee at 4096 tokens).
    "serving": Workload("serving", V=129280, r=256, B=256, K=6, scheduler=True,
                        seed=3),
    # B=512, K=16; per-request correlation rho ~ U(0.3,0.95); per-request
    # temperature in {0.6,1.0,1.3}; scheduler on; 100 sequential steps.
    "stress": Workload("stress", V=151936, r=256, B=512, K=16, peak=0.0,
                       target_mode="rho", temps_per_request=True, scheduler=True,
                       steps=100, seed=4),
}

ORDER = ["tiny", "single", "batched", "serving", "stress"]


def get(name: str, **overrides) -> Workload:
    """A named workload, optionally with shapes overridden (smaller parity cases)."""
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def cost_table(n_pts: int = 16, step: float = 512.0, knee: float = 4096.0,
               fixed_ms: float = 20.0, slope: float = 0.004, knee_factor: float = 4.0):
    """Profiled verify-cost table: tokens -> ms, linear with a knee.

    Stands in for the start-up SPS(B) profile: ``fixed_ms + slope*N`` up to
    the knee, slope multiplied by ``knee_factor`` after it.
    """
    xs = [i * step for i in range(n_pts)]
    ys = []
    for x in xs:
        if x <= knee:
            ys.append(fixed_ms + slope * x)
        else:
            ys.append(fixed_ms + slope * knee + slope * knee_factor * (x - knee))
    return (torch.tensor(xs, dtype=torch.float32), torch.tensor(ys, dtype=torch.float32))


def seq_temps(K: int):
    """Sequential temperature-scaling temperatures T_k = 1 + 0.1 k, k = 1..K."""
    return torch.tensor([1.0 + 0.1 * k for k in range(1, K + 1)], dtype=torch.float32)


def make_inputs(w: Workload, device="cpu", seed: int | None = None) -> dict:
    """Draw every input tensor of one step of workload ``w`` on ``device``.

    Returns a dict with
      base [B,K,V] f32, target [B*(K+1),V] f32, row_start [B] i64,
      U, W [V,r] (bf16 or f32), prev_token [B] i32, inv_temp [B] f32,
      z [B,K] f32, temps [K] f32, cost_tokens/cost_ms [16] f32,
      u_draft [B,K], u_accept [B,K], u_res [B] f32, verify_len [B] i32 (= K).
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    V, r, B, K = w.V, w.r, w.B, w.K
    f32 = torch.float32

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=f32)

    def rand(*shape):
        return torch.rand(*shape, generator=g, device=device, dtype=f32)

    prev = torch.randint(0, V, (B,), generator=g, device=device, dtype=torch.int64).to(torch.int32)
    std = math.sqrt(w.uw_var / r)
    U = randn(V, r).mul_(std)
    W = randn(V, r).mul_(std)
    if w.uw_bf16:
        U = U.to(torch.bfloat16)
        W = W.to(torch.bfloat16)

    # base logits for K draft positions plus the bonus position (K+1 rows)
    ext = randn(B, K + 1, V)
    if w.split_peaked_flat:
        half = B // 2
        ext[:half].mul_(1.0)
        ext[half:].mul_(4.0)
    else:
        ext.mul_(w.base_sigma)
    peak_pos = torch.randint(0, V, (B, K + 1), generator=g, device=device)
    if w.split_peaked_flat:
        half = B // 2
        if half > 0:
            ext[:half].scatter_add_(2, peak_pos[:half, :, None],
                                    torch.full((half, K + 1, 1), 10.0, device=device))
    elif w.peak != 0.0:
        ext.scatter_add_(2, peak_pos[:, :, None],
                         torch.full((B, K + 1, 1), w.peak, device=device))

    # target logits, rows laid out flat: request b, position p -> row b*(K+1)+p
    if w.target_mode == "noise":
        target = ext + randn(B, K + 1, V).mul_(0.5)
    elif w.target_mode == "scaled":
        target = ext.mul(0.8).add_(randn(B, K + 1, V))
    elif w.target_mode == "rho":
        rho = 0.3 + 0.65 * rand(B)
        target = ext.mul(rho[:, None, None])
        noise = randn(B, K + 1, V).mul_(3.0)
        target.add_(noise.mul_(torch.sqrt(1.0 - rho * rho)[:, None, None]))
        del noise
    else:
        raise ValueError(w.target_mode)
    base = ext[:, :K, :].contiguous()
    del ext
    target = target.reshape(B * (K + 1), V)
    row_start = torch.arange(B, device=device, dtype=torch.int64) * (K + 1)

    if w.temps_per_request:
        choice = torch.randint(0, 3, (B,), generator=g, device=device)
        T = torch.tensor([0.6, 1.0, 1.3], device=device, dtype=f32)[choice]
        inv_temp = (1.0 / T).to(f32)
    else:
        inv_temp = torch.ones(B, device=device, dtype=f32)

    z = randn(B, K).add_(1.5)
    u_draft = rand(B, K)
    u_accept = rand(B, K)
    u_res = rand(B)
    xs, ys = cost_table()
    return dict(base=base, target=target, row_start=row_start, U=U, W=W,
                prev_token=prev, inv_temp=inv_temp, z=z,
                temps=seq_temps(K).to(device), cost_tokens=xs.to(device),
                cost_ms=ys.to(device), u_draft=u_draft, u_accept=u_accept,
                u_res=u_res,
                verify_len=torch.full((B,), K, device=device, dtype=torch.int32))


def step_uniforms(w: Workload, step: int, device="cpu", seed: int | None = None):
    """Fresh uniforms for sequential step ``step`` (> 0) of a multi-step run."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed((w.seed if seed is None else seed) * 1_000_003 + step)
    B, K = w.B, w.K
    return dict(u_draft=torch.rand(B, K, generator=g, device=device),
                u_accept=torch.rand(B, K, generator=g, device=device),
                u_res=torch.rand(B, generator=g, device=device))


def host_uw(t: torch.Tensor):
    """U or W as a numpy array for the oracle: bf16 as uint16 bit patterns."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


# ---------------------------------------------------------------------------
# Calibration set for the sequential temperature fit
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Calibration:
    """An offline calibration set: N sequences of K head scores and the
    accepted-prefix length of a full-block verify of each."""
    name: str
    N: int
    K: int
    seed: int = 5


CALIBRATIONS = {
    # one million logged sequences at the Stress draft length
    "calibration": Calibration("calibration", N=1_000_000, K=16),
    # a smaller set that the oracle fits in well under a second per position
    "calibration_small": Calibration("calibration_small", N=50_003, K=16, seed=6),
}


def make_calibration(c: Calibration, device="cpu", seed: int | None = None) -> dict:
    """Head scores z [N,K] f32 ~ N(1.5, 1.5^2) and accepted lengths n_acc [N]
    i32 in [0, K].

    Ground truth of the synthetic head: given every earlier token was
    accepted, position k (1-based) is accepted with probability
    Phi(z * 0.588 / (1.2 + 0.05 k)), Phi the standard normal CDF.  This is a
    probit link, not the logistic form the fit assumes; 0.588 z is close to
    the logistic scale, so the raw scores read as over-confident by a factor
    of about 1.2 + 0.05 k, as the pages describe the head.  The first
    rejected position ends the prefix."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(c.seed if seed is None else seed)
    z = torch.randn(c.N, c.K, generator=g, device=device, dtype=torch.float32).mul_(1.5).add_(1.5)
    u = torch.rand(c.N, c.K, generator=g, device=device, dtype=torch.float32)
    k = torch.arange(1, c.K + 1, device=device, dtype=torch.float32)
    scale = 0.588 / (1.2 + 0.05 * k)
    accepted = u < torch.special.ndtr(z * scale)
    rejected = ~accepted
    first = rejected.to(torch.int32).argmax(dim=1).to(torch.int32)
    n_acc = torch.where(rejected.any(dim=1), first, torch.full_like(first, c.K))
    return dict(z=z, n_acc=n_acc.contiguous())
