"""One DSpark decode step (draft -> prefix cut -> verify) through the C ABI.

DSparkStep owns the output tensors and workspaces of one problem size on
one device, so a step launches only library kernels (no allocation) and can
be captured in a CUDA graph.
"""
from __future__ import annotations

import torch

from . import dspark as D


class DSparkStep:
    def __init__(self, V: int, r: int, B: int, K: int, n_target_rows: int, uw_dtype,
                 device="cuda", n_pts: int = 16, keep_bias=None):
        self.V, self.r, self.B, self.K = V, r, B, K
        self.n_rows = n_target_rows
        self.device = torch.device(device)
        dev = self.device
        i32, f32 = torch.int32, torch.float32
        self.tokens = torch.empty(B, K, dtype=i32, device=dev)
        self.p_tok = torch.empty(B, K, dtype=f32, device=dev)
        self.lse = torch.empty(B, K, dtype=f32, device=dev)
        self.ref_max = torch.empty(B, K, dtype=f32, device=dev)
        self.ref_sum = torch.empty(B, K, dtype=f32, device=dev)
        self.c = torch.empty(B, K, dtype=f32, device=dev)
        self.survival = torch.empty(B, K, dtype=f32, device=dev)
        self.verify_len = torch.empty(B, dtype=i32, device=dev)
        self.objective = torch.empty(1, dtype=f32, device=dev)
        self.n_accepted = torch.empty(B, dtype=i32, device=dev)
        self.out_tokens = torch.empty(B, K + 1, dtype=i32, device=dev)
        self.last_token = torch.empty(B, dtype=i32, device=dev)
        self.ws_draft = D.workspace(D.dspark_draft_workspace_size(V, r, B, K), dev)
        self.ws_prefix = D.workspace(D.dspark_prefix_workspace_size(B, K, n_pts), dev)
        self.ws_verify = D.workspace(D.dspark_verify_workspace_size(V, r, B, K), dev)
        self.path = D.dspark_draft_path(V, r, B, K, uw_dtype)
        # Keep the draft's bias rows for the verify when B is small (saves a
        # pass over W in the verify); large batches re-project instead.
        if keep_bias is None:
            keep_bias = B <= 16
        self.draft_bias = (torch.empty(B, K, V, dtype=f32, device=dev) if keep_bias and B * K > 0
                           else None)

    def draft(self, inp, prev_token=None, stream=None, draft_logits=None):
        D.dspark_draft_markov(inp["base"], inp["U"], inp["W"],
                              inp["prev_token"] if prev_token is None else prev_token,
                              inp["inv_temp"], inp["u_draft"], self.tokens, self.p_tok, self.lse,
                              self.ref_max, self.ref_sum, self.ws_draft,
                              draft_logits=draft_logits, draft_bias=self.draft_bias,
                              stream=stream)

    def prefix(self, inp, enable: bool, stream=None):
        D.dspark_confidence_prefix(inp["z"], inp["temps"], inp["cost_tokens"], inp["cost_ms"],
                                   enable, self.c, self.survival, self.verify_len,
                                   self.objective, self.ws_prefix, stream=stream)

    def verify(self, inp, prev_token=None, stream=None):
        D.dspark_verify(inp["target"], inp["row_start"], self.verify_len, inp["base"], inp["U"],
                        inp["W"], inp["prev_token"] if prev_token is None else prev_token,
                        inp["inv_temp"], self.tokens, self.p_tok, self.ref_max, self.ref_sum,
                        inp["u_accept"], inp["u_res"], self.n_accepted, self.out_tokens,
                        self.ws_verify, last_token=self.last_token,
                        draft_bias=self.draft_bias, stream=stream)

    def run(self, inp, enable_prefix: bool, prev_token=None, stream=None):
        """One full step; the next step's prev_token is self.last_token."""
        self.draft(inp, prev_token=prev_token, stream=stream)
        self.prefix(inp, enable_prefix, stream=stream)
        self.verify(inp, prev_token=prev_token, stream=stream)

    def flags(self, stream=None):
        return {name: D.dspark_get_device_flags(ws, stream)
                for name, ws in [("draft", self.ws_draft), ("prefix", self.ws_prefix),
                                 ("verify", self.ws_verify)]}
