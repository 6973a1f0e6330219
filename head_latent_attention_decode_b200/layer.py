"""Device-memory plumbing around the C-ABI: upload a weight set, own the
repacked blob and a workspace, and call the entry points on torch tensors.

No arithmetic of the layer happens here; each method is one C-ABI call.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (MLA_ROW_LATENT_FIRST, make_config, mla_decode_attn, mla_decode_qkv, mla_destroy,
               mla_init_weights, mla_prefill, mla_rope_cos_sin, mla_rope_cos_sin_inv_freq, mla_v4_qkv,
               mla_weights_bytes, mla_workspace_bytes, mla_workspace_init)

ACT_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}


def upload_weights(weights, device) -> dict:
    """workloads.Weights -> dict of device tensors in the C-ABI's storage dtypes."""
    s = weights.shape
    out = {}
    for name, arr in weights.dense.items():
        t = torch.from_numpy(np.ascontiguousarray(arr))
        out[name] = t.to(ACT_TORCH[s.weight_dtype]).to(device)
    for name, codes in weights.codes.items():
        out[name] = torch.from_numpy(np.ascontiguousarray(codes)).to(device)
        out[name + "_scale"] = torch.from_numpy(np.ascontiguousarray(weights.scales[name])).to(device)
    if weights.q_norm_w is not None:
        out["q_norm_w"] = torch.from_numpy(weights.q_norm_w).to(device)
    out["kv_norm_w"] = torch.from_numpy(weights.kv_norm_w).to(device)
    return out


class MlaLayer:
    """One layer's repacked weights (device) and C-ABI handle."""

    def __init__(self, shape, weights, row_layout: int = MLA_ROW_LATENT_FIRST,
                 device: str = "cuda", softmax_scale: float = 0.0, attn_sink=None):
        self.shape = shape
        self.device = torch.device(device)
        self.act = ACT_TORCH[shape.act_dtype]
        self.row_layout = row_layout
        self.cfg = make_config(shape, row_layout, softmax_scale)
        nbytes = mla_weights_bytes(self.cfg)
        if nbytes == 0:
            raise ValueError(f"configuration not accepted by the library: {shape}")
        self.blob = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        src = upload_weights(weights, self.device) if not isinstance(weights, dict) else dict(weights)
        if attn_sink is not None:   # per-head sink logits, fp32 [n_heads]
            src["attn_sink"] = torch.as_tensor(attn_sink, dtype=torch.float32).to(self.device).contiguous()
        self.handle = mla_init_weights(self.cfg, src, self.blob)
        torch.cuda.current_stream(self.device).synchronize()
        del src
        self.ws = None

    def close(self) -> None:
        """Release the library handle (the weight blob is torch memory)."""
        h = getattr(self, "handle", None)
        if h:
            mla_destroy(h)
            self.handle = None

    def __del__(self):
        # at interpreter shutdown the module's globals may already be gone
        if mla_destroy is not None:
            self.close()

    def workspace(self, max_tokens: int, max_context_len: int = 1) -> torch.Tensor:
        need = mla_workspace_bytes(self.handle, max(1, max_tokens), max(1, max_context_len))
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            mla_workspace_init(self.ws)
        return self.ws

    def rope(self, positions: torch.Tensor, inv_freq: torch.Tensor | None = None):
        """cos/sin [n, qk_rope/2] fp32 of the positions; inv_freq (device fp32
        [qk_rope/2], e.g. a YaRN table) replaces theta^(-2i/qk_rope)."""
        n = positions.numel()
        half = self.shape.qk_rope // 2
        cos = torch.empty((n, half), dtype=torch.float32, device=self.device)
        sin = torch.empty((n, half), dtype=torch.float32, device=self.device)
        if inv_freq is None:
            mla_rope_cos_sin(positions, self.shape.qk_rope, self.shape.rope_theta, cos, sin)
        else:
            mla_rope_cos_sin_inv_freq(positions, self.shape.qk_rope, inv_freq, cos, sin)
        return cos, sin

    def decode_qkv(self, hidden, cos, sin, kv_cache, slot_mapping, q_abs=None, q_pe=None, input_norm_w=None):
        s = self.shape
        n = hidden.shape[0]
        if q_abs is None:
            q_abs = torch.empty((n, s.n_heads, s.kv_lora_rank), dtype=self.act, device=self.device)
        if q_pe is None:
            q_pe = torch.empty((n, s.n_heads, s.qk_rope), dtype=self.act, device=self.device)
        ws = self.ws if self.ws is not None and self.ws.numel() >= mla_workspace_bytes(
            self.handle, max(n, 1), 1) else self.workspace(n, 1)
        mla_decode_qkv(self.handle, hidden, cos, sin, kv_cache, slot_mapping, q_abs, q_pe, ws,
                       input_norm_w=input_norm_w)
        return q_abs, q_pe

    def decode_attn(self, q_abs, q_pe, kv_cache, block_table, context_lens, max_context_len,
                    out=None, head_out=None):
        s = self.shape
        n = q_abs.shape[0]
        if out is None:
            out = torch.empty((n, s.hidden), dtype=self.act, device=self.device)
        ws = self.ws if self.ws is not None and self.ws.numel() >= mla_workspace_bytes(
            self.handle, max(n, 1), max_context_len) else self.workspace(n, max_context_len)
        mla_decode_attn(self.handle, q_abs, q_pe, kv_cache, block_table, context_lens,
                        max_context_len, out, ws, head_out=head_out)
        return out

    def v4_qkv(self, hidden, cos, sin, kv_norm_w, q_out=None, kv_out=None):
        """DeepSeek-V4 QKV projection: (q [S, H, d_n + d_r], kv [S, r_kv + d_r])."""
        s = self.shape
        S = hidden.shape[0]
        if q_out is None:
            q_out = torch.empty((S, s.n_heads, s.qk_nope + s.qk_rope), dtype=self.act, device=self.device)
        if kv_out is None:
            kv_out = torch.empty((S, s.kv_lora_rank + s.qk_rope), dtype=self.act, device=self.device)
        ws = self.ws if self.ws is not None and self.ws.numel() >= mla_workspace_bytes(
            self.handle, max(S, 1), 1) else self.workspace(S, 1)
        mla_v4_qkv(self.handle, hidden, cos, sin, kv_norm_w, q_out, kv_out, ws)
        return q_out, kv_out

    def prefill(self, hidden, cos, sin, out=None, head_out=None, kv_cache=None, slot_mapping=None):
        s = self.shape
        S = hidden.shape[0]
        if out is None:
            out = torch.empty((S, s.hidden), dtype=self.act, device=self.device)
        ws = self.ws if self.ws is not None and self.ws.numel() >= mla_workspace_bytes(
            self.handle, max(S, 1), 1) else self.workspace(S, 1)
        mla_prefill(self.handle, hidden, cos, sin, out, ws, head_out=head_out, kv_cache=kv_cache,
                    slot_mapping=slot_mapping)
        return out
