"""Host-side checks of the C ABI that need no GPU: the library loads,
exports every symbol include/dspark.h declares, and rejects bad arguments
before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from speculative_decoding_05_b200 import build
from speculative_decoding_05_b200 import dspark as D

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return D.load()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(dspark_\w+)\s*\(", txt))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations found"
    out = subprocess.run(["nm", "-D", "--defined-only", D.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b(dspark_\w+)\b", out))
    assert declared <= exported, declared - exported
    assert set(D.SYMBOLS) <= declared
    for name in declared:
        assert hasattr(lib, name)


def test_status_strings_and_paths(lib):
    for code in range(7):
        assert D.status_string(code)
    assert D.dspark_version() >= 100
    assert D.dspark_draft_path(151936, 256, 1, 16, D.DSPARK_BF16) == "persistent-cuda-core"
    assert D.dspark_draft_path(151936, 256, 2, 16, D.DSPARK_BF16) == "persistent-cuda-core"
    assert D.dspark_draft_path(151936, 128, 1, 16, D.DSPARK_BF16) == "tcgen05-persistent"
    assert D.dspark_draft_path(151936, 256, 4, 16, D.DSPARK_BF16) == "tcgen05-persistent"
    assert D.dspark_draft_path(151936, 256, 5, 16, D.DSPARK_BF16) == "tcgen05-persistent"
    assert D.dspark_draft_path(151936, 256, 16, 16, D.DSPARK_BF16) == "tcgen05-persistent"
    assert D.dspark_draft_path(1024, 16, 2, 4, D.DSPARK_F32) == "cuda-core"
    assert D.dspark_draft_path(1024, 16, 64, 4, D.DSPARK_F32) == "cuda-core"
    assert D.dspark_draft_path(151936, 256, 64, 8, D.DSPARK_BF16) == "tcgen05"
    assert D.dspark_draft_path(151936, 256, 17, 8, D.DSPARK_BF16) == "tcgen05"
    assert D.dspark_draft_path(1000, 32, 4, 8, D.DSPARK_BF16) == "cuda-core"
    bf = D.DSPARK_BF16
    assert D.dspark_verify_path(151936, 256, 1, 16, bf, True) == "single-launch"
    assert D.dspark_verify_path(151936, 256, 4, 17, bf, True) == "single-launch"   # 72 rows
    assert D.dspark_verify_path(151936, 256, 4, 18, bf, True) == "staged-bias"     # 76 rows
    assert D.dspark_verify_path(151936, 256, 5, 8, bf, True) == "staged-bias"
    assert D.dspark_verify_path(1024, 16, 2, 4, D.DSPARK_F32, True) == "single-launch"
    assert D.dspark_verify_path(151936, 256, 1, 16, bf, False) == "staged-cuda-core"
    assert D.dspark_verify_path(151936, 256, 64, 8, bf, False) == "staged-tcgen05"


def test_workspace_sizes(lib):
    V, r, B, K = 151936, 256, 512, 16
    nch = (V + 31) // 32
    assert lib.dspark_draft_workspace_size(V, r, B, K) >= 256 + B * nch * 8
    assert lib.dspark_verify_workspace_size(V, r, B, K) >= 256 + B * nch * 8
    assert lib.dspark_prefix_workspace_size(B, K, 16) >= 4
    assert lib.dspark_draft_workspace_size(0, r, B, K) == 0
    # the prefix workspace: the 2 KB header, plus (for a valid batch) the
    # survivals and the order the multi-CTA form passes between its kernels,
    # 20 bytes per candidate; invalid or oversized batches get the header
    n = B * K
    assert lib.dspark_prefix_workspace_size(B, K, 16) >= 2048 + 20 * n
    assert lib.dspark_prefix_workspace_size(B, K, 16) < 2048 + 20 * n + 3 * 256
    assert lib.dspark_prefix_workspace_size(1024, 9, 16) == 2048
    assert lib.dspark_prefix_workspace_size(-1, 4, 16) == 2048


def _draft(lib, V=1024, r=16, B=2, K=3, base=1 << 20, U=1 << 21, W=1 << 22, ws=1 << 24,
           ws_bytes=None, dtype=D.DSPARK_BF16):
    if ws_bytes is None:
        ws_bytes = lib.dspark_draft_workspace_size(V, r, B, K)
    P = ctypes.c_void_p
    p = P(1 << 23)
    return lib.dspark_draft_markov(P(base), P(U), P(W), dtype, V, r, B, K, p, None, p, p, p, p, p,
                                   p, None, None, P(ws), ws_bytes, None)


def test_argument_validation_before_launch(lib):
    # every case below must be rejected on the host, before any CUDA call
    assert _draft(lib, V=1022) == 4            # V % 4 != 0 -> unsupported
    assert _draft(lib, r=12) == 4              # r % 8 != 0
    assert _draft(lib, r=2048) == 4            # r too large
    assert _draft(lib, K=65) == 4              # K too large
    assert _draft(lib, V=-4) == 1
    assert _draft(lib, dtype=7) == 1
    assert _draft(lib, ws_bytes=16) == 6       # workspace too small
    assert _draft(lib, ws=(1 << 24) + 8) == 6  # workspace misaligned
    assert _draft(lib, base=(1 << 20) + 4) == 1  # base not 16-byte aligned
    assert _draft(lib, U=0) == 1               # NULL required pointer
    P = ctypes.c_void_p
    p = P(1 << 23)
    ws = P(1 << 24)
    # prefix: too many candidates, bad table size
    assert lib.dspark_confidence_prefix(p, p, p, p, 16, 1024, 9, 1, p, p, p, p, ws, 256, None) == 4
    assert lib.dspark_confidence_prefix(p, p, p, p, 1, 4, 4, 1, p, p, p, p, ws, 256, None) == 1
    # asynchronous prefix: bad cost reading, too many candidates
    assert lib.dspark_confidence_prefix_async(p, p, p, p, 16, 2, 4, 4, 1, None, p, p, p, p, None,
                                              ws, 256, None) == 1
    assert lib.dspark_confidence_prefix_async(p, p, p, p, 16, 1, 1024, 9, 1, None, p, p, p, p,
                                              None, ws, 256, None) == 4
    # temperature fit: bad K, K past the limit, missing outputs, short or misaligned workspace
    sb = lib.dspark_sts_workspace_size(1000, 16)
    assert sb > 0 and lib.dspark_sts_workspace_size(1000, 33) == 0
    assert lib.dspark_sts_workspace_size(-1, 4) == 0
    assert lib.dspark_sts_fit(p, p, 1000, 0, p, p, None, ws, sb, None) == 1
    assert lib.dspark_sts_fit(p, p, 1000, 33, p, p, None, ws, sb, None) == 4
    assert lib.dspark_sts_fit(p, p, 1000, 16, None, p, None, ws, sb, None) == 1
    assert lib.dspark_sts_fit(None, p, 1000, 16, p, p, None, ws, sb, None) == 1
    assert lib.dspark_sts_fit(p, p, -5, 16, p, p, None, ws, sb, None) == 1
    assert lib.dspark_sts_fit(p, p, 1000, 16, p, p, None, ws, sb - 8, None) == 6
    assert lib.dspark_sts_fit(p, p, 1000, 16, p, p, None, P((1 << 24) + 8), sb, None) == 6
    # verify: missing target
    vb = lib.dspark_verify_workspace_size(1024, 16, 2, 3)
    assert lib.dspark_verify(None, 10, p, p, p, p, p, 1, 1024, 16, 2, 3, p, None, p, p, p, p, None,
                             p, p, p, p, None, ws, vb, None) == 1
    # LM-head verify: width not a multiple of 64 or too large, missing hidden
    # states, short workspace, misaligned head
    lb = lib.dspark_verify_lmhead_workspace_size(1024, 16, 2, 3, 256, 10)
    assert lb > 0 and lib.dspark_verify_lmhead_workspace_size(1024, 16, 2, 3, 0, 10) == 0

    def lm(hidden=p, head=p, dm=256, ws_bytes=lb):
        return lib.dspark_verify_lmhead(hidden, head, dm, 10, p, p, p, p, p, 1, 1024, 16, 2, 3, p,
                                        None, p, p, p, p, None, p, p, p, p, None, ws, ws_bytes,
                                        None)
    # RNN draft: fp32 factors, r not a multiple of 64, short workspace
    rb = lib.dspark_draft_rnn_workspace_size(1024, 64, 4, 3)
    assert rb > lib.dspark_draft_workspace_size(1024, 64, 4, 3)

    def rnn(dt=D.DSPARK_BF16, r=64, ws_bytes=rb):
        return lib.dspark_draft_rnn(p, p, p, p, dt, 1024, r, 4, 3, p, None, None, p, p, p, p, p,
                                    p, None, None, None, ws, ws_bytes, None)
    assert rnn(dt=D.DSPARK_F32) == 4 and rnn(r=72) == 4 and rnn(r=320) == 4
    assert rnn(ws_bytes=rb - 256) == 6
    assert lm(dm=100) == 4 and lm(dm=32768) == 4 and lm(dm=-64) == 1
    assert lm(hidden=None) == 1
    assert lm(ws_bytes=lb - 256) == 6
    assert lm(head=P((1 << 23) + 8)) == 1


def test_traffic_hash_covers_the_draft_kernels_sources():
    """The stored DRAM traffic of the persistent draft is keyed to the files
    that kernel is built from, not to every source of the library."""
    import os
    import bench
    names = {os.path.basename(f) for f in bench.source_closure("draft_persist.cuh")}
    assert {"draft_persist.cuh", "proj_tc.cuh", "tc_common.cuh", "common.cuh", "sample.cuh",
            "proj_simt.cuh", "dspark.h"} <= names
    assert not names & {"prefix.cuh", "sts.cuh", "verify.cuh", "verify_fused.cuh", "api.cu"}
    assert bench.source_digest("draft_persist.cuh") != bench.source_digest()


def test_bench_launch_count_follows_the_paths():
    """The bench's gpu_launches claim: three kernels per step on the single
    workload (persistent draft, prefix, single-launch verify), 2K + 5 on the
    tensor-core path with the staged verify."""
    import torch
    import bench
    d = D.dspark_draft_path(151936, 256, 1, 16, D.DSPARK_BF16)
    v = D.dspark_verify_path(151936, 256, 1, 16, torch.bfloat16, True)
    assert (d, v) == ("persistent-cuda-core", "single-launch")
    assert bench.launches_per_step(d, v, 16) == 3
    d = D.dspark_draft_path(129280, 256, 256, 6, D.DSPARK_BF16)
    v = D.dspark_verify_path(129280, 256, 256, 6, torch.bfloat16, False)
    assert (d, v) == ("tcgen05", "staged-tcgen05")
    assert bench.launches_per_step(d, v, 6) == 2 * 6 + 1 + 4
    # the prefix cut of more than 1024 candidates with the scheduler on is
    # two kernels
    p = D.dspark_prefix_path(256, 6, True)
    assert p == "multi-cta"
    assert bench.launches_per_step(d, v, 6, p) == 2 * 6 + 2 + 4
    assert D.dspark_prefix_path(256, 6, False) == "single-cta"
    assert D.dspark_prefix_path(64, 16, True) == "single-cta"   # exactly 1024
    assert D.dspark_prefix_path(1, 1025, True) == "multi-cta"


def test_temperature_fit_workspace_is_bounded(lib):
    """The fit's workspace does not grow with the calibration set past its
    grid cap: header, 32 search states, per-CTA partials (at most 1184 CTAs)."""
    small = lib.dspark_sts_workspace_size(1000, 16)
    big = lib.dspark_sts_workspace_size(10 ** 8, 16)
    assert 2048 < small <= big < 1.3e6
    assert lib.dspark_sts_workspace_size(10 ** 8, 32) > big  # partials grow with K
    assert lib.dspark_sts_workspace_size(10 ** 8, 32) % 256 == 0


def test_binding_raises_on_refused_calls(lib):
    """Argument errors come back from the library before any launch and the
    binding raises them (a stream handle is passed explicitly: without CUDA
    the binding cannot ask torch for the current stream)."""
    import types

    import torch
    s0 = types.SimpleNamespace(cuda_stream=0)
    z = torch.zeros(10, 33)
    n = torch.zeros(10, dtype=torch.int32)
    t = torch.zeros(33)
    e = torch.zeros(2)
    ws = torch.zeros(4096, dtype=torch.uint8)
    with pytest.raises(D.DSparkError) as err:
        D.dspark_sts_fit(z, n, t, e, ws, stream=s0)  # K = 33 > DSPARK_STS_MAX_K
    assert err.value.code == 4
    z = torch.zeros(10, 16)
    assert lib.dspark_sts_workspace_size(10, 16) > 1024
    with pytest.raises(D.DSparkError) as err:
        D.dspark_sts_fit(z, n, torch.zeros(16), e, ws[:1024], stream=s0)  # workspace too small
    assert err.value.code == 6
