"""Shared plumbing of the GPU parity tests: build a layer and its inputs on the
device from the seeded workloads, run the same case through the fp64 oracle,
and compare. The oracle never receives anything the CUDA path produced."""
from __future__ import annotations

import numpy as np
import torch

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import workloads as wl
from head_latent_attention_decode_b200.build import build
from head_latent_attention_decode_b200.layer import ACT_TORCH, MlaLayer
from oracle import mla_ref as ref

# |gpu - ref| <= TOL * max|ref| (per head for head_out)
TOL = {"f32": 1e-4, "bf16": 2e-2}


def ensure_built():
    build()
    mla.lib()


def to_dev(arr, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(arr)).to(dtype).to(device)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_rel_err(gpu, want):
    scale = np.max(np.abs(want))
    return float(np.max(np.abs(gpu - want)) / (scale if scale > 0 else 1.0))


def assert_close(gpu, want, tol, what):
    err = max_rel_err(gpu, want)
    assert err <= tol, f"{what}: max|gpu-ref|/max|ref| = {err:.3e} > {tol:.1e}"
    return err


def assert_close_per_head(gpu, want, tol, what):
    """gpu/want [n, H, d]: each (token, head) block within tol * its own max|ref|."""
    worst = 0.0
    for t in range(want.shape[0]):
        for h in range(want.shape[1]):
            worst = max(worst, max_rel_err(gpu[t, h], want[t, h]))
    assert worst <= tol, f"{what}: worst per-head error {worst:.3e} > {tol:.1e}"
    return worst


def compact(inp, seqs, shape):
    """Sub-problem of sequences `seqs`: their blocks copied, in order, into a
    small cache with remapped block tables, slots and fill slots (data
    movement only). Returns (cache, table, slots, fill_slots, blocks) where
    blocks[i] is the original id of compact block i."""
    bs = shape.block_size
    blocks = []
    for b in seqs:
        nb = (int(inp.context_lens[b]) + bs - 1) // bs
        blocks.extend(int(x) for x in inp.block_table[b, :nb])
    remap = np.full(inp.n_blocks, -1, np.int64)
    remap[blocks] = np.arange(len(blocks))
    cache = inp.cache[blocks]
    table = np.full((len(seqs), inp.block_table.shape[1]), -1, np.int32)
    for i, b in enumerate(seqs):
        nb = (int(inp.context_lens[b]) + bs - 1) // bs
        table[i, :nb] = remap[inp.block_table[b, :nb]]

    def rs(sl):
        sl = np.asarray(sl, np.int64)
        return (remap[sl // bs] * bs + sl % bs).astype(np.int32)
    slots = rs(inp.slot_mapping[list(seqs)])
    fill = None if inp.fill_slots is None else [rs(inp.fill_slots[b]) for b in seqs]
    return cache, table, slots, fill, np.array(blocks)


class DecodeCase:
    """A decode step on the GPU and its inputs, for one workload."""

    def __init__(self, workload, batch=None, ctx=None, row_layout=ref.LATENT_FIRST, device="cuda",
                 input_norm_w=None, inv_freq=None, attn_sink=None):
        """input_norm_w [hidden] / inv_freq [qk_rope/2] / attn_sink [n_heads]: optional fp32
        numpy arrays for this step's input RMSNorm, RoPE frequency table and per-head sink
        logits (both sides get the same values)."""
        ensure_built()
        self.attn_sink = None if attn_sink is None else np.asarray(attn_sink, np.float32)
        self.input_norm_w = None if input_norm_w is None else np.asarray(input_norm_w, np.float32)
        self.inv_freq = None if inv_freq is None else np.asarray(inv_freq, np.float32)
        self.w = workload
        self.shape = s = workload.shape
        self.row_layout = row_layout
        self.weights = wl.make_weights(s, workload.seed)
        self.inp = wl.make_decode_inputs(workload, batch=batch, ctx=ctx)
        self.layer = MlaLayer(s, self.weights, row_layout=row_layout, device=device, attn_sink=self.attn_sink)
        self.act = ACT_TORCH[s.act_dtype]
        self.device = device
        inp = self.inp
        self.cache = to_dev(inp.cache, self.act, device)
        if inp.fill_hidden is not None:
            self._fill_by_projection()
        self.hidden = to_dev(inp.hidden, self.act, device)
        self.positions = torch.from_numpy(inp.positions).to(device)
        self.g_in = None if self.input_norm_w is None else torch.from_numpy(self.input_norm_w).to(device)
        f = None if self.inv_freq is None else torch.from_numpy(self.inv_freq).to(device)
        self.cos, self.sin = self.layer.rope(self.positions, f)
        self.slot = torch.from_numpy(inp.slot_mapping).to(device)
        self.table = torch.from_numpy(inp.block_table).to(device)
        self.ctx = torch.from_numpy(inp.context_lens).to(device)
        self.max_ctx = int(inp.context_lens.max())

    def _fill_by_projection(self, chunk=4096):
        s = self.shape
        xs = np.concatenate(self.inp.fill_hidden, axis=0)
        slots = np.concatenate(self.inp.fill_slots, axis=0)
        pos = np.concatenate([np.arange(len(f), dtype=np.int32) for f in self.inp.fill_slots])
        for i in range(0, len(slots), chunk):
            x = to_dev(xs[i:i + chunk], self.act, self.device)
            p = torch.from_numpy(pos[i:i + chunk]).to(self.device)
            cos, sin = self.layer.rope(p)
            self.layer.decode_qkv(x, cos, sin, self.cache, torch.from_numpy(slots[i:i + chunk]).to(self.device))
        torch.cuda.synchronize()

    def run(self):
        s = self.shape
        self.q_abs, self.q_pe = self.layer.decode_qkv(self.hidden, self.cos, self.sin, self.cache, self.slot,
                                                      input_norm_w=self.g_in)
        n = self.hidden.shape[0]
        self.head_out = torch.empty((n, s.n_heads, s.v_dim), dtype=self.act, device=self.device)
        self.out = self.layer.decode_attn(self.q_abs, self.q_pe, self.cache, self.table, self.ctx,
                                          self.max_ctx, head_out=self.head_out)
        torch.cuda.synchronize()
        return self

    def flag(self):
        return mla.mla_read_device_flag(self.layer.ws)

    # ---------------- oracle side ----------------
    def oracle(self, seqs=None):
        """Oracle of this step for sequences `seqs` (default all), on a compact
        copy of their cache blocks. The returned 'blocks' maps compact block i
        to the original (GPU) block id."""
        s = self.shape
        inp = self.inp
        seqs = list(range(len(inp.hidden))) if seqs is None else list(seqs)
        cache, table, slots, fill_slots, blocks = compact(inp, seqs, s)
        W = ref.weights_fp64(self.weights)
        cache = np.asarray(cache, np.float64)
        if inp.fill_hidden is not None:
            cache = ref.fill_cache_by_projection(s, W, cache, [inp.fill_hidden[b] for b in seqs],
                                                 fill_slots, self.row_layout)
        cos, sin = ref.rope_cos_sin(inp.positions[seqs], s.qk_rope, s.rope_theta, inv_freq=self.inv_freq)
        q_abs, q_pe, new_cache = ref.decode_qkv(s, W, inp.hidden[seqs], cos, sin, cache, slots,
                                                self.row_layout, input_norm_w=self.input_norm_w)
        out, head_out = ref.decode_attn(s, W, q_abs, q_pe, new_cache, table,
                                        inp.context_lens[seqs], self.row_layout, attn_sink=self.attn_sink)
        return dict(q_abs=q_abs, q_pe=q_pe, cache=new_cache, out=out, head_out=head_out,
                    slots=slots, blocks=blocks, seqs=seqs)
