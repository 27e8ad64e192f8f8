"""Python marshalling for the double-precision CPU oracle (dspark_oracle.c).

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT: only the test suite, the
package smoke check and the benchmark's CPU-baseline leg may import this
module.  It shares no code with the CUDA library and never imports it.

Every function here only converts numpy arrays to pointers and back; all of
the arithmetic is in dspark_oracle.c (see its header for the page citations
and for what pins each function).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dspark_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP).  Returns the .so path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99",
           "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, f64 = ctypes.c_int, ctypes.c_double
            lib.oracle_draft.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P,
                                         P, P, P, P]
            lib.oracle_draft.restype = i32
            lib.oracle_draft_row.argtypes = [P, P, P, i32, i32, i32, i32, f64, P]
            lib.oracle_draft_row.restype = None
            lib.oracle_prefix.argtypes = [P, P, P, P, i32, i32, i32, i32, P, P, P,
                                          P, P]
            lib.oracle_prefix.restype = i32
            lib.oracle_cost_ms.argtypes = [P, P, i32, f64]
            lib.oracle_cost_ms.restype = f64
            lib.oracle_cost_stair_ms.argtypes = [P, P, i32, f64]
            lib.oracle_cost_stair_ms.restype = f64
            lib.oracle_prefix_async.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, P, P, P,
                                                P, P, P]
            lib.oracle_prefix_async.restype = i32
            lib.oracle_verify.argtypes = [P, ctypes.c_int64, P, P, P, P, P, i32,
                                          i32, i32, i32, i32, P, P, P, P, P, P,
                                          P, P, P, P]
            lib.oracle_verify.restype = i32
            lib.oracle_verify_lmhead.argtypes = [P, P, i32, i32, ctypes.c_int64, P, P, P, P, P,
                                                 i32, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                                 P, P, P]
            lib.oracle_verify_lmhead.restype = i32
            lib.oracle_draft_rnn.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P,
                                             P, P, P, P]
            lib.oracle_draft_rnn.restype = i32
            lib.oracle_verify_rnn.argtypes = [P, ctypes.c_int64, P, P, P, P, P, P, i32, i32, i32,
                                              i32, i32, P, P, P, P, P, P, P, P, P, P, P]
            lib.oracle_verify_rnn.restype = i32
            lib.oracle_sts_fit.argtypes = [P, P, ctypes.c_long, i32, P, P, P]
            lib.oracle_sts_fit.restype = i32
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = i32
            _lib = lib
    return _lib


def _c(a, dtype):
    """Contiguous numpy array of the given dtype (copies only if needed)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _uw(m):
    """U/W as (array, is_bf16).  bf16 tensors arrive as uint16 bit patterns."""
    m = np.ascontiguousarray(m)
    if m.dtype == np.uint16:
        return m, 1
    return _c(m, np.float32), 0


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def draft_row(base_row, U, W, x_prev: int, inv_temp: float = 1.0):
    """Draft logits (fp64) of one position given the previous token."""
    lib = _load()
    base_row = _c(base_row, np.float32)
    Ua, bf = _uw(U)
    Wa, _ = _uw(W)
    V, r = Wa.shape
    out = np.empty(V, np.float64)
    lib.oracle_draft_row(_p(base_row), _p(Ua), _p(Wa), bf, V, r, int(x_prev),
                         float(inv_temp), _p(out))
    return out


def draft(base, U, W, prev_token, u_draft, inv_temp=None):
    """Markov-head draft.  base [B,K,V] fp32, U/W [V,r] fp32 or uint16 (bf16)."""
    lib = _load()
    base = _c(base, np.float32)
    B, K, V = base.shape
    Ua, bf = _uw(U)
    Wa, _ = _uw(W)
    r = Wa.shape[1]
    assert Wa.shape == (V, r) and Ua.shape == (V, r)
    prev = _c(prev_token, np.int32)
    ud = _c(u_draft, np.float32).reshape(B, K)
    it = None if inv_temp is None else _c(inv_temp, np.float32)
    tokens = np.empty((B, K), np.int32)
    p_tok = np.empty((B, K), np.float64)
    lse = np.empty((B, K), np.float64)
    margin = np.empty((B, K), np.float64)
    rc = lib.oracle_draft(_p(base), _p(Ua), _p(Wa), bf, V, r, B, K, _p(prev),
                          _p(it), _p(ud), _p(tokens), _p(p_tok), _p(lse),
                          _p(margin))
    if rc != 0:
        raise ValueError(f"oracle_draft rejected its arguments (rc={rc})")
    return dict(tokens=tokens, p_tok=p_tok, lse=lse, margin=margin)


def draft_rnn(base, U, W, R, prev_token, u_draft, h0=None, inv_temp=None, states=False):
    """RNN-head draft: state s_k = tanh(R s_{k-1} + U[x_{k-1}]) from h0
    (zeros if None), logits (base + s_k . W^T) / T.  U, W [V,r] and R [r,r]
    share one dtype (fp32, or uint16 bf16 bit patterns)."""
    lib = _load()
    base = _c(base, np.float32)
    B, K, V = base.shape
    Ua, bf = _uw(U)
    Wa, _ = _uw(W)
    Ra, rb = _uw(R)
    r = Wa.shape[1]
    assert Ra.shape == (r, r) and rb == bf and Ua.shape == (V, r)
    prev = _c(prev_token, np.int32)
    ud = _c(u_draft, np.float32).reshape(B, K)
    hh = None if h0 is None else _c(h0, np.float32).reshape(B, r)
    it = None if inv_temp is None else _c(inv_temp, np.float32)
    tokens = np.empty((B, K), np.int32)
    p_tok = np.empty((B, K), np.float64)
    lse = np.empty((B, K), np.float64)
    margin = np.empty((B, K), np.float64)
    st = np.empty((B, K, r), np.float64) if states else None
    rc = lib.oracle_draft_rnn(_p(base), _p(Ua), _p(Wa), _p(Ra), bf, V, r, B, K, _p(prev), _p(hh),
                              _p(it), _p(ud), _p(tokens), _p(p_tok), _p(lse), _p(margin), _p(st))
    if rc != 0:
        raise ValueError(f"oracle_draft_rnn rejected its arguments (rc={rc})")
    out = dict(tokens=tokens, p_tok=p_tok, lse=lse, margin=margin)
    if states:
        out["states"] = st
    return out


def verify_rnn(target, row_start, verify_len, base, U, W, R, prev_token, tokens, p_d, u_accept,
               u_res, h0=None, inv_temp=None):
    """The verify of an RNN-head draft (the rejected position's draft row
    is the RNN head's)."""
    lib = _load()
    target = _c(target, np.float32)
    n_rows, V = target.shape
    base = _c(base, np.float32)
    B, K, _ = base.shape
    Ua, bf = _uw(U)
    Wa, _ = _uw(W)
    Ra, _ = _uw(R)
    r = Wa.shape[1]
    rs = _c(row_start, np.int64)
    vl = _c(verify_len, np.int32)
    prev = _c(prev_token, np.int32)
    hh = None if h0 is None else _c(h0, np.float32).reshape(B, r)
    toks = _c(tokens, np.int32).reshape(B, K)
    pd = _c(p_d, np.float64).reshape(B, K)
    ua = _c(u_accept, np.float32).reshape(B, K)
    ur = _c(u_res, np.float32)
    it = None if inv_temp is None else _c(inv_temp, np.float32)
    n_acc = np.empty(B, np.int32)
    out = np.empty((B, K + 1), np.int32)
    am = np.empty(B, np.float64)
    rm = np.empty(B, np.float64)
    rc = lib.oracle_verify_rnn(_p(target), n_rows, _p(rs), _p(vl), _p(base), _p(Ua), _p(Wa),
                               _p(Ra), bf, V, r, B, K, _p(prev), _p(hh), _p(it), _p(toks), _p(pd),
                               _p(ua), _p(ur), _p(n_acc), _p(out), _p(am), _p(rm))
    if rc != 0:
        raise ValueError(f"oracle_verify_rnn rejected its arguments (rc={rc})")
    return dict(n_acc=n_acc, out_tokens=out, accept_margin=am, res_margin=rm)


def cost_ms(cost_tokens, cost_ms_, n_tokens: float) -> float:
    lib = _load()
    xs = _c(cost_tokens, np.float32)
    ys = _c(cost_ms_, np.float32)
    return float(lib.oracle_cost_ms(_p(xs), _p(ys), len(xs), float(n_tokens)))


def prefix(z, temps, cost_tokens, cost_ms_, enable: bool = True):
    """Sequential temperature scaling, survival, greedy prefix cut."""
    lib = _load()
    z = _c(z, np.float32)
    B, K = z.shape
    temps = _c(temps, np.float32)
    xs = _c(cost_tokens, np.float32)
    ys = _c(cost_ms_, np.float32)
    c = np.empty((B, K), np.float64)
    S = np.empty((B, K), np.float64)
    L = np.empty(B, np.int32)
    obj = np.empty(1, np.float64)
    mg = np.empty(1, np.float64)
    rc = lib.oracle_prefix(_p(z), _p(temps), _p(xs), _p(ys), len(xs), B, K,
                           int(bool(enable)), _p(c), _p(S), _p(L), _p(obj), _p(mg))
    if rc != 0:
        raise ValueError(f"oracle_prefix rejected its arguments (rc={rc})")
    return dict(c=c, S=S, L=L, objective=float(obj[0]), margin=float(mg[0]))


def verify(target, row_start, verify_len, base, U, W, prev_token, tokens, p_d,
           u_accept, u_res, inv_temp=None):
    """Rejection-sampling verify.  target [n_rows, V] fp32 (ragged rows)."""
    lib = _load()
    target = _c(target, np.float32)
    n_rows, V = target.shape
    base = _c(base, np.float32)
    B, K, _ = base.shape
    Ua, bf = _uw(U)
    Wa, _ = _uw(W)
    r = Wa.shape[1]
    rs = _c(row_start, np.int64)
    vl = _c(verify_len, np.int32)
    prev = _c(prev_token, np.int32)
    toks = _c(tokens, np.int32).reshape(B, K)
    pd = _c(p_d, np.float64).reshape(B, K)
    ua = _c(u_accept, np.float32).reshape(B, K)
    ur = _c(u_res, np.float32)
    it = None if inv_temp is None else _c(inv_temp, np.float32)
    n_acc = np.empty(B, np.int32)
    out = np.empty((B, K + 1), np.int32)
    am = np.empty(B, np.float64)
    rm = np.empty(B, np.float64)
    rc = lib.oracle_verify(_p(target), n_rows, _p(rs), _p(vl), _p(base), _p(Ua),
                           _p(Wa), bf, V, r, B, K, _p(prev), _p(it), _p(toks),
                           _p(pd), _p(ua), _p(ur), _p(n_acc), _p(out), _p(am),
                           _p(rm))
    if rc != 0:
        raise ValueError(f"oracle_verify rejected its arguments (rc={rc})")
    return dict(n_acc=n_acc, out_tokens=out, accept_margin=am, res_margin=rm)


def verify_lmhead(hidden, lm_head, row_start, verify_len, base, U, W, prev_token, tokens, p_d,
                  u_accept, u_res, inv_temp=None):
    """The verify with target logits formed as hidden [n_rows, dm] times
    lm_head [V, dm] transposed (both fp32, or both bf16 as uint16 bit
    patterns) instead of read from stored rows."""
    lib = _load()
    Ha, hb = _uw(hidden)
    Ea, eb = _uw(lm_head)
    if hb != eb or Ha.shape[1] != Ea.shape[1]:
        raise ValueError("hidden and lm_head must share dtype and width")
    n_rows, dm = Ha.shape
    V = Ea.shape[0]
    base = _c(base, np.float32)
    B, K, _ = base.shape
    Ua, bf = _uw(U)
    Wa, _ = _uw(W)
    r = Wa.shape[1]
    rs = _c(row_start, np.int64)
    vl = _c(verify_len, np.int32)
    prev = _c(prev_token, np.int32)
    toks = _c(tokens, np.int32).reshape(B, K)
    pd = _c(p_d, np.float64).reshape(B, K)
    ua = _c(u_accept, np.float32).reshape(B, K)
    ur = _c(u_res, np.float32)
    it = None if inv_temp is None else _c(inv_temp, np.float32)
    n_acc = np.empty(B, np.int32)
    out = np.empty((B, K + 1), np.int32)
    am = np.empty(B, np.float64)
    rm = np.empty(B, np.float64)
    rc = lib.oracle_verify_lmhead(_p(Ha), _p(Ea), dm, hb, n_rows, _p(rs), _p(vl), _p(base),
                                  _p(Ua), _p(Wa), bf, V, r, B, K, _p(prev), _p(it), _p(toks),
                                  _p(pd), _p(ua), _p(ur), _p(n_acc), _p(out), _p(am), _p(rm))
    if rc != 0:
        raise ValueError(f"oracle_verify_lmhead rejected its arguments (rc={rc})")
    return dict(n_acc=n_acc, out_tokens=out, accept_margin=am, res_margin=rm)


def sts_fit(z, n_accepted):
    """Sequential temperature scaling: per-position temperatures fitted by
    likelihood on the sequences that reached each position, and the pooled
    expected calibration error before and after."""
    lib = _load()
    z = _c(z, np.float32)
    N, K = z.shape
    n_acc = _c(n_accepted, np.int32)
    if n_acc.shape != (N,):
        raise ValueError("n_accepted must be [N]")
    temps = np.empty(K, np.float64)
    ece = np.empty(2, np.float64)
    count = np.empty(K, np.int64)
    rc = lib.oracle_sts_fit(_p(z), _p(n_acc), N, K, _p(temps), _p(ece), _p(count))
    if rc != 0:
        raise ValueError(f"oracle_sts_fit rejected its arguments (rc={rc})")
    return dict(temps=temps, ece_before=float(ece[0]), ece_after=float(ece[1]), count=count)


def cost_stair_ms(cost_tokens, cost_ms_, n_tokens: float) -> float:
    """Staircase reading of the cost table: the entry of the smallest
    profiled size that holds n_tokens."""
    lib = _load()
    xs = _c(cost_tokens, np.float32)
    ys = _c(cost_ms_, np.float32)
    return float(lib.oracle_cost_stair_ms(_p(xs), _p(ys), len(xs), float(n_tokens)))


def prefix_async(z, temps, cost_tokens, cost_ms_, staircase: bool = False, enable: bool = True,
                 budget: int | None = None):
    """Prefix cut with the cost table read as a staircase or piecewise
    linear, optionally against a budget of verify tokens decided earlier;
    also returns n_greedy, the greedy N of the current confidences."""
    lib = _load()
    z = _c(z, np.float32)
    B, K = z.shape
    temps = _c(temps, np.float32)
    xs = _c(cost_tokens, np.float32)
    ys = _c(cost_ms_, np.float32)
    c = np.empty((B, K), np.float64)
    S = np.empty((B, K), np.float64)
    L = np.empty(B, np.int32)
    obj = np.empty(1, np.float64)
    mg = np.empty(1, np.float64)
    ng = np.empty(1, np.int32)
    rc = lib.oracle_prefix_async(_p(z), _p(temps), _p(xs), _p(ys), len(xs), int(bool(staircase)),
                                 B, K, int(bool(enable)), -1 if budget is None else int(budget),
                                 _p(c), _p(S), _p(L), _p(obj), _p(mg), _p(ng))
    if rc != 0:
        raise ValueError(f"oracle_prefix_async rejected its arguments (rc={rc})")
    return dict(c=c, S=S, L=L, objective=float(obj[0]), margin=float(mg[0]),
                n_greedy=int(ng[0]))
