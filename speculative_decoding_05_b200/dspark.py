"""Thin Python binding of the C ABI in include/dspark.h (ctypes).

Argument marshalling only: tensors are turned into device pointers and
sizes, every step of the hot path runs in libdspark.so.  The functions carry
the C names.  Loading fails loudly if the CUDA library is missing; there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdspark.so")

DSPARK_F32 = 0
DSPARK_BF16 = 1

STATUS = {0: "DSPARK_OK", 1: "DSPARK_ERR_INVALID_ARG", 2: "DSPARK_ERR_CUDA",
          3: "DSPARK_ERR_TIMEOUT", 4: "DSPARK_ERR_UNSUPPORTED",
          5: "DSPARK_ERR_DEVICE_DATA", 6: "DSPARK_ERR_WORKSPACE"}

FLAG_BAD_TOKEN = 0x01
FLAG_BAD_LENGTH = 0x02
FLAG_NONFINITE = 0x04
FLAG_BAD_TEMP = 0x08
FLAG_TIMEOUT = 0x10
FLAG_BAD_TABLE = 0x20

# every symbol include/dspark.h declares
SYMBOLS = [
    "dspark_draft_workspace_size", "dspark_draft_markov",
    "dspark_prefix_workspace_size", "dspark_confidence_prefix",
    "dspark_verify_workspace_size", "dspark_verify",
    "dspark_get_device_status", "dspark_get_device_flags",
    "dspark_status_string", "dspark_draft_path", "dspark_verify_path", "dspark_prefix_path",
    "dspark_version",
    "dspark_verify_noalloc",
    "dspark_verify_noalloc_status",
    "dspark_verify_lmhead_workspace_size",
    "dspark_verify_lmhead",
    "dspark_draft_rnn_workspace_size",
    "dspark_draft_rnn",
    "dspark_test_set_exchange_skew",
    "dspark_sts_workspace_size",
    "dspark_sts_fit",
    "dspark_confidence_prefix_async",
]


class DSparkError(RuntimeError):
    def __init__(self, where: str, code: int):
        super().__init__(f"{where}: {STATUS.get(code, code)} ({status_string(code)})")
        self.code = code


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libdspark.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"CUDA library not built: {p} (run speculative_decoding_05_b200.build)")
    lib = ctypes.CDLL(p)
    P, I, L, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.dspark_draft_workspace_size.argtypes = [I, I, I, I]
    lib.dspark_draft_workspace_size.restype = S
    lib.dspark_verify_workspace_size.argtypes = [I, I, I, I]
    lib.dspark_verify_workspace_size.restype = S
    lib.dspark_prefix_workspace_size.argtypes = [I, I, I]
    lib.dspark_prefix_workspace_size.restype = S
    lib.dspark_draft_markov.argtypes = [P, P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P,
                                        S, P]
    lib.dspark_draft_markov.restype = I
    lib.dspark_verify.argtypes = [P, L, P, P, P, P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P,
                                  P, P, P, S, P]
    lib.dspark_verify.restype = I
    lib.dspark_verify_noalloc.argtypes = [P, L, P, P, P, P, P, I, I, I, I, I, P, P, P, P, P, P, P,
                                          P, P, P, P, P, P]
    lib.dspark_verify_noalloc.restype = I
    lib.dspark_verify_noalloc_status.argtypes = [P]
    lib.dspark_verify_noalloc_status.restype = I
    lib.dspark_verify_lmhead_workspace_size.argtypes = [I, I, I, I, I, L]
    lib.dspark_verify_lmhead_workspace_size.restype = S
    lib.dspark_verify_lmhead.argtypes = [P, P, I, L, P, P, P, P, P, I, I, I, I, I, P, P, P, P, P,
                                         P, P, P, P, P, P, P, P, S, P]
    lib.dspark_verify_lmhead.restype = I
    lib.dspark_draft_rnn_workspace_size.argtypes = [I, I, I, I]
    lib.dspark_draft_rnn_workspace_size.restype = S
    lib.dspark_draft_rnn.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P,
                                     P, P, S, P]
    lib.dspark_draft_rnn.restype = I
    lib.dspark_test_set_exchange_skew.argtypes = [I]
    lib.dspark_test_set_exchange_skew.restype = I
    lib.dspark_confidence_prefix.argtypes = [P, P, P, P, I, I, I, I, P, P, P, P, P, S, P]
    lib.dspark_confidence_prefix.restype = I
    lib.dspark_confidence_prefix_async.argtypes = [P, P, P, P, I, I, I, I, I, P, P, P, P, P, P, P,
                                                   S, P]
    lib.dspark_confidence_prefix_async.restype = I
    lib.dspark_sts_workspace_size.argtypes = [L, I]
    lib.dspark_sts_workspace_size.restype = S
    lib.dspark_sts_fit.argtypes = [P, P, L, I, P, P, P, P, S, P]
    lib.dspark_sts_fit.restype = I
    lib.dspark_get_device_status.argtypes = [P, P]
    lib.dspark_get_device_status.restype = I
    lib.dspark_get_device_flags.argtypes = [P, P]
    lib.dspark_get_device_flags.restype = I
    lib.dspark_status_string.argtypes = [I]
    lib.dspark_status_string.restype = ctypes.c_char_p
    lib.dspark_draft_path.argtypes = [I, I, I, I, I]
    lib.dspark_draft_path.restype = ctypes.c_char_p
    lib.dspark_verify_path.argtypes = [I, I, I, I, I, I]
    lib.dspark_verify_path.restype = ctypes.c_char_p
    lib.dspark_prefix_path.argtypes = [I, I, I]
    lib.dspark_prefix_path.restype = ctypes.c_char_p
    lib.dspark_version.argtypes = []
    lib.dspark_version.restype = I
    if path is None:
        _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(where, rc):
    if rc != 0:
        raise DSparkError(where, rc)


def _dtype_code(U):
    return DSPARK_BF16 if U.dtype == torch.bfloat16 else DSPARK_F32


def status_string(code: int) -> str:
    try:
        return load().dspark_status_string(int(code)).decode()
    except Exception:  # the library may be missing when formatting an error
        return STATUS.get(code, "unknown")


dspark_status_string = status_string


def dspark_version() -> int:
    return int(load().dspark_version())


def dspark_draft_path(V, r, B, K, uw_dtype) -> str:
    code = uw_dtype if isinstance(uw_dtype, int) else (
        DSPARK_BF16 if uw_dtype == torch.bfloat16 else DSPARK_F32)
    return load().dspark_draft_path(V, r, B, K, code).decode()


def dspark_verify_path(V, r, B, K, uw_dtype, have_bias) -> str:
    code = uw_dtype if isinstance(uw_dtype, int) else (
        DSPARK_BF16 if uw_dtype == torch.bfloat16 else DSPARK_F32)
    return load().dspark_verify_path(V, r, B, K, code, int(bool(have_bias))).decode()


def dspark_prefix_path(B, K, enable) -> str:
    return load().dspark_prefix_path(B, K, int(bool(enable))).decode()


def dspark_draft_workspace_size(V, r, B, K) -> int:
    return int(load().dspark_draft_workspace_size(V, r, B, K))


def dspark_verify_workspace_size(V, r, B, K) -> int:
    return int(load().dspark_verify_workspace_size(V, r, B, K))


def dspark_prefix_workspace_size(B, K, n_pts) -> int:
    return int(load().dspark_prefix_workspace_size(B, K, n_pts))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned device byte buffer (torch's allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def dspark_draft_markov(base_logits, U, W, prev_token, inv_temp, u_draft, tokens, p_tok, lse,
                        ref_max, ref_sum, workspace, draft_logits=None, draft_bias=None,
                        stream=None):
    B, K, V = base_logits.shape
    r = W.shape[1]
    rc = load().dspark_draft_markov(
        _ptr(base_logits), _ptr(U), _ptr(W), _dtype_code(U), V, r, B, K, _ptr(prev_token),
        _ptr(inv_temp), _ptr(u_draft), _ptr(tokens), _ptr(p_tok), _ptr(lse), _ptr(ref_max),
        _ptr(ref_sum), _ptr(draft_logits), _ptr(draft_bias), _ptr(workspace), workspace.numel(),
        _stream(stream))
    _check("dspark_draft_markov", rc)


def dspark_confidence_prefix(z, temps, cost_tokens, cost_ms, enable, c, survival, verify_len,
                             objective, workspace, stream=None):
    B, K = z.shape
    rc = load().dspark_confidence_prefix(
        _ptr(z), _ptr(temps), _ptr(cost_tokens), _ptr(cost_ms), cost_tokens.numel(), B, K,
        int(bool(enable)), _ptr(c), _ptr(survival), _ptr(verify_len), _ptr(objective),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check("dspark_confidence_prefix", rc)


def dspark_verify(target_logits, row_start, verify_len, base_logits, U, W, prev_token, inv_temp,
                  tokens, p_tok, ref_max, ref_sum, u_accept, u_resample, n_accepted, out_tokens,
                  workspace, last_token=None, draft_bias=None, stream=None):
    n_rows, V = target_logits.shape
    B, K = tokens.shape
    r = W.shape[1]
    rc = load().dspark_verify(
        _ptr(target_logits), n_rows, _ptr(row_start), _ptr(verify_len), _ptr(base_logits),
        _ptr(U), _ptr(W), _dtype_code(U), V, r, B, K, _ptr(prev_token), _ptr(inv_temp),
        _ptr(tokens), _ptr(p_tok), _ptr(ref_max), _ptr(ref_sum), _ptr(draft_bias), _ptr(u_accept),
        _ptr(u_resample), _ptr(n_accepted), _ptr(out_tokens), _ptr(last_token),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check("dspark_verify", rc)


def dspark_verify_noalloc(target_logits, row_start, verify_len, base_logits, U, W, prev_token,
                          inv_temp, tokens, p_tok, ref_max, ref_sum, u_accept, u_resample,
                          n_accepted, out_tokens, last_token=None, draft_bias=None, stream=None):
    """dspark_verify with the library's built-in scratch (no workspace)."""
    n_rows, V = target_logits.shape
    B, K = tokens.shape
    r = W.shape[1]
    rc = load().dspark_verify_noalloc(
        _ptr(target_logits), n_rows, _ptr(row_start), _ptr(verify_len), _ptr(base_logits),
        _ptr(U), _ptr(W), _dtype_code(U), V, r, B, K, _ptr(prev_token), _ptr(inv_temp),
        _ptr(tokens), _ptr(p_tok), _ptr(ref_max), _ptr(ref_sum), _ptr(draft_bias), _ptr(u_accept),
        _ptr(u_resample), _ptr(n_accepted), _ptr(out_tokens), _ptr(last_token), _stream(stream))
    _check("dspark_verify_noalloc", rc)


def dspark_draft_rnn_workspace_size(V, r, B, K) -> int:
    return int(load().dspark_draft_rnn_workspace_size(V, r, B, K))


def dspark_draft_rnn(base_logits, U, W, R, prev_token, h0, inv_temp, u_draft, tokens, p_tok, lse,
                     ref_max, ref_sum, workspace, states=None, draft_logits=None, draft_bias=None,
                     stream=None):
    """The draft with the RNN head: state s_k = tanh(R s_{k-1} + U[x_{k-1}])
    from h0 (None: zeros), bias s_k . W^T."""
    B, K, V = base_logits.shape
    r = W.shape[1]
    rc = load().dspark_draft_rnn(
        _ptr(base_logits), _ptr(U), _ptr(W), _ptr(R), _dtype_code(U), V, r, B, K,
        _ptr(prev_token), _ptr(h0), _ptr(inv_temp), _ptr(u_draft), _ptr(tokens), _ptr(p_tok),
        _ptr(lse), _ptr(ref_max), _ptr(ref_sum), _ptr(states), _ptr(draft_logits),
        _ptr(draft_bias), _ptr(workspace), workspace.numel(), _stream(stream))
    _check("dspark_draft_rnn", rc)


def dspark_verify_lmhead_workspace_size(V, r, B, K, dm, n_rows) -> int:
    return int(load().dspark_verify_lmhead_workspace_size(V, r, B, K, dm, int(n_rows)))


def dspark_verify_lmhead(hidden, lm_head, row_start, verify_len, base_logits, U, W, prev_token,
                         inv_temp, tokens, p_tok, ref_max, ref_sum, u_accept, u_resample,
                         n_accepted, out_tokens, workspace, last_token=None, draft_bias=None,
                         stream=None):
    """dspark_verify with target logits hidden [n_rows, dm] . lm_head [V, dm]^T
    (both bf16) formed on chip instead of read from stored rows."""
    n_rows, dm = hidden.shape
    V = lm_head.shape[0]
    B, K = tokens.shape
    r = W.shape[1]
    rc = load().dspark_verify_lmhead(
        _ptr(hidden), _ptr(lm_head), dm, n_rows, _ptr(row_start), _ptr(verify_len),
        _ptr(base_logits), _ptr(U), _ptr(W), _dtype_code(U), V, r, B, K, _ptr(prev_token),
        _ptr(inv_temp), _ptr(tokens), _ptr(p_tok), _ptr(ref_max), _ptr(ref_sum), _ptr(draft_bias),
        _ptr(u_accept), _ptr(u_resample), _ptr(n_accepted), _ptr(out_tokens), _ptr(last_token),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check("dspark_verify_lmhead", rc)


def dspark_test_set_exchange_skew(skew: int) -> None:
    """Test hook: non-zero makes the persistent draft's and the
    single-launch verify's record exchanges time out (see the header)."""
    _check("dspark_test_set_exchange_skew", load().dspark_test_set_exchange_skew(int(skew)))


def dspark_verify_noalloc_status(stream=None) -> int:
    """Status code of the last dspark_verify_noalloc call on this device
    (synchronises the stream)."""
    return int(load().dspark_verify_noalloc_status(_stream(stream)))


def dspark_get_device_flags(workspace, stream=None) -> int:
    f = int(load().dspark_get_device_flags(_ptr(workspace), _stream(stream)))
    if f < 0:
        raise DSparkError("dspark_get_device_flags", 2)
    return f


def dspark_get_device_status(workspace, stream=None) -> int:
    return int(load().dspark_get_device_status(_ptr(workspace), _stream(stream)))


def dspark_sts_workspace_size(N, K) -> int:
    return int(load().dspark_sts_workspace_size(int(N), int(K)))


def dspark_sts_fit(z, n_accepted, temps, ece, workspace, passes=None, stream=None):
    """Per-position temperatures of the confidence head fitted on a
    calibration set (z [N,K] fp32, n_accepted [N] int32); writes temps [K],
    ece [2] (before, after) and, if given, passes [1] int32."""
    N, K = z.shape
    rc = load().dspark_sts_fit(_ptr(z), _ptr(n_accepted), N, K, _ptr(temps), _ptr(ece),
                               _ptr(passes), _ptr(workspace), workspace.numel(), _stream(stream))
    _check("dspark_sts_fit", rc)


COST_LINEAR, COST_STAIRCASE = 0, 1


def dspark_confidence_prefix_async(z, temps, cost_tokens, cost_ms, enable, c, survival, verify_len,
                                   objective, workspace, staircase=False, budget_in=None,
                                   budget_out=None, stream=None):
    """The prefix cut with an optional budget decided earlier (budget_in
    [1] int32) and the greedy N of this step written to budget_out [1]
    (the two may be the same tensor); staircase selects the cost reading."""
    B, K = z.shape
    rc = load().dspark_confidence_prefix_async(
        _ptr(z), _ptr(temps), _ptr(cost_tokens), _ptr(cost_ms), cost_tokens.numel(),
        COST_STAIRCASE if staircase else COST_LINEAR, B, K, int(bool(enable)), _ptr(budget_in),
        _ptr(c), _ptr(survival), _ptr(verify_len), _ptr(objective), _ptr(budget_out),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check("dspark_confidence_prefix_async", rc)
