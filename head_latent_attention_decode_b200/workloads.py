"""Seeded synthetic workloads for the MLA layer step.

This module only draws random numbers and lays them out; it holds none of
the layer's arithmetic (no projection, norm, rotation or attention). Both the
CUDA path (tests, bench) and the fp64 oracle consume what it produces, so the
two sides see exactly the same inputs.

Shapes follow the pages:
  * DeepSeek-V3 dims (q_lora 1536, kv_lora 512, nope 128 + rope 64, v 128):
    "QKV CTE MLA Kernel API Reference", qkv_mla_mx, Dimensions.
  * Paged cache [n_blocks, 1, block_size, kv_row_dim] and int32 slot_mapping:
    "MLA Decode QKV Kernel API Reference", Parameters (kv_cache, slot_mapping).
  * Weight init N(0, 0.02): nemo_automodel ... deepseek_v3.layers, MLA.init_weights
    (init_std default).
  * FP8-E4M3 codes with 128x128 fp32 block scales: "Struct MlaWeights",
    field wq_a_fp8; scale tensor shape [ceil(K/128), ceil(N/128)]: "QKV CTE MLA
    Kernel API Reference", qkv_mla_mx parameters (*_scale_hbm).

Values that the CUDA path receives in bf16 are rounded to bf16 here (by torch's
round-to-nearest-even cast), and the same rounded values are what the oracle
sees, upcast to fp64.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class MlaShape:
    hidden: int
    n_heads: int
    q_lora_rank: int          # 0 = full query projection (no low-rank q path)
    kv_lora_rank: int
    qk_nope: int
    qk_rope: int
    v_dim: int
    block_size: int
    act_dtype: str            # "f32" | "bf16"
    weight_dtype: str         # "f32" | "bf16" | "fp8"
    norm_eps: float = 1e-6
    rope_theta: float = 10000.0
    o_groups: int = 0         # DeepSeek-V4 grouped low-rank O: head groups (0 = one dense wo)
    o_lora_rank: int = 0      # ... and each group's low rank

    @property
    def kv_row_dim(self) -> int:
        return self.kv_lora_rank + self.qk_rope

    @property
    def qk_head_dim(self) -> int:
        return self.qk_nope + self.qk_rope

    @property
    def q_out_dim(self) -> int:
        return self.n_heads * self.qk_head_dim


@dataclass(frozen=True)
class Workload:
    name: str
    shape: MlaShape
    mode: str                  # "decode" | "prefill" | "v4qkv" (the DeepSeek-V4 QKV projection)
    batch: int                 # decode tokens (one per sequence); 1 for prefill
    ctx_lo: int                # context length range (inclusive) per sequence
    ctx_hi: int
    cache_fill: str            # "project": earlier rows come from projecting
                               # N(0,1) hidden states; "random": N(0,1) rows
    seed: int
    seq_len: int = 0           # prefill only
    spare_blocks: int = 3      # cache blocks beyond what the sequences use
    description: str = ""


TINY = MlaShape(hidden=256, n_heads=4, q_lora_rank=64, kv_lora_rank=64, qk_nope=32,
                qk_rope=16, v_dim=32, block_size=16, act_dtype="f32", weight_dtype="f32")
V2LITE = MlaShape(hidden=2048, n_heads=16, q_lora_rank=0, kv_lora_rank=512, qk_nope=128,
                  qk_rope=64, v_dim=128, block_size=64, act_dtype="bf16", weight_dtype="bf16")
V3 = MlaShape(hidden=7168, n_heads=128, q_lora_rank=1536, kv_lora_rank=512, qk_nope=128,
              qk_rope=64, v_dim=128, block_size=64, act_dtype="bf16", weight_dtype="bf16")
V3_FP8 = dataclasses.replace(V3, weight_dtype="fp8")

WORKLOADS = {
    "tiny_fp32": Workload(
        "tiny_fp32", TINY, "decode", batch=2, ctx_lo=64, ctx_hi=64, cache_fill="project",
        seed=0, description="tiny MLA fp32 decode, batch 2, context 64, block 16, "
        "random block permutation"),
    "v2lite_bf16": Workload(
        "v2lite_bf16", V2LITE, "decode", batch=32, ctx_lo=4096, ctx_hi=4096,
        cache_fill="project", seed=1, description="DeepSeek-V2-Lite-shaped MLA bf16 decode, "
        "batch 32, context 4096, block 64, cache filled by projecting N(0,1) hidden states"),
    "v3_bf16": Workload(
        "v3_bf16", V3, "decode", batch=64, ctx_lo=1024, ctx_hi=16384, cache_fill="random",
        seed=2, description="DeepSeek-V3-shaped MLA bf16 decode, batch 64, context "
        "U[1024,16384], block 64, random block tables / slot_mapping"),
    "v3_fp8": Workload(
        "v3_fp8", V3_FP8, "decode", batch=128, ctx_lo=8192, ctx_hi=8192, cache_fill="random",
        seed=3, description="DeepSeek-V3-shaped MLA decode, FP8-E4M3 weights with 128x128 "
        "fp32 block scales, bf16 activations, batch 128, context 8192"),
    "v3_prefill_bf16": Workload(
        "v3_prefill_bf16", V3, "prefill", batch=1, ctx_lo=0, ctx_hi=0, cache_fill="none",
        seed=4, seq_len=8192, description="DeepSeek-V3-shaped MLA prefill bf16, seq 8192 "
        "causal, expanded K/V"),
    "v3_prefill_fp8": Workload(
        "v3_prefill_fp8", V3_FP8, "prefill", batch=1, ctx_lo=0, ctx_hi=0, cache_fill="none",
        seed=6, seq_len=8192, description="DeepSeek-V3-shaped MLA prefill, FP8-E4M3 weights with "
        "128x128 fp32 block scales, bf16 activations, seq 8192 causal, expanded K/V"),
    "v4_qkv_bf16": Workload(
        "v4_qkv_bf16", V3, "v4qkv", batch=1, ctx_lo=0, ctx_hi=0, cache_fill="none",
        seed=7, seq_len=8192, description="DeepSeek-V4 form of the QKV projection on "
        "DeepSeek-V3-sized matrices (hidden 7168, q_lora 1536, kv_dim 576, 128 heads of "
        "192), bf16, 8192 tokens"),
}


# ----------------------------------------------------------------------------
# rounding helpers (storage formats only)
# ----------------------------------------------------------------------------

def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64/fp32 values to what `dtype` can hold; returned as float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16).to(torch.float32).numpy()
    if dtype == "f32":
        return t.numpy()
    raise ValueError(dtype)


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Host tensor in the storage dtype the C-ABI takes for `dtype`."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def e4m3_encode(w_over_s: np.ndarray) -> np.ndarray:
    """Round to the nearest FP8-E4M3 code (saturating at +-448); uint8 codes.

    Input-generation only: the codes and scales are the weights both sides get.
    """
    t = torch.from_numpy(np.clip(np.asarray(w_over_s, np.float32), -448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------

WEIGHT_NAMES = ("wq_a", "wq_b", "wkv_a", "wkv_b", "wo", "wo_a", "wo_b")


def weight_shapes(s: MlaShape) -> dict:
    """[in, out] shapes (x @ W), as the pages give them."""
    d = {}
    if s.q_lora_rank:
        d["wq_a"] = (s.hidden, s.q_lora_rank)
        d["wq_b"] = (s.q_lora_rank, s.q_out_dim)
    else:
        d["wq_b"] = (s.hidden, s.q_out_dim)      # the full q_proj
    d["wkv_a"] = (s.hidden, s.kv_row_dim)
    d["wkv_b"] = (s.kv_lora_rank, s.n_heads * (s.qk_nope + s.v_dim))
    if s.o_lora_rank:
        # grouped low-rank O: wo_a holds each group's [(H/G) d_v, r_o] block, the
        # groups stacked along its input rows; wo_b [G r_o, D]
        d["wo_a"] = (s.n_heads * s.v_dim, s.o_lora_rank)
        d["wo_b"] = (s.o_groups * s.o_lora_rank, s.hidden)
    else:
        d["wo"] = (s.n_heads * s.v_dim, s.hidden)
    return d


@dataclass
class Weights:
    """Weights in the C-ABI's input format.

    dense[name]: float32 [in, out] holding values exactly representable in the
      weight storage dtype (f32 / bf16). For fp8: the dequantised values are not
      stored here; codes[name] (uint8 [in, out]) and scales[name] (float32
      [ceil(in/128), ceil(out/128)]) are.
    q_norm_w / kv_norm_w: float32 gammas.
    """
    shape: MlaShape
    dense: dict
    codes: dict
    scales: dict
    q_norm_w: np.ndarray | None
    kv_norm_w: np.ndarray


def make_weights(s: MlaShape, seed: int) -> Weights:
    rng = np.random.default_rng(seed)
    dense, codes, scales = {}, {}, {}
    for name, (k, n) in weight_shapes(s).items():
        w = rng.standard_normal((k, n), dtype=np.float32) * np.float32(0.02)
        if s.weight_dtype == "fp8":
            kb, nb = -(-k // 128), -(-n // 128)
            # log-uniform block scales in [2^-8, 2^-4]
            sc = np.exp2(rng.uniform(-8.0, -4.0, size=(kb, nb))).astype(np.float32)
            full = np.repeat(np.repeat(sc, 128, axis=0), 128, axis=1)[:k, :n]
            codes[name] = e4m3_encode(w / full)
            scales[name] = sc
        else:
            dense[name] = round_to(w, s.weight_dtype)
    q_norm_w = None
    if s.q_lora_rank:
        q_norm_w = (1.0 + rng.uniform(-0.1, 0.1, size=s.q_lora_rank)).astype(np.float32)
    kv_norm_w = (1.0 + rng.uniform(-0.1, 0.1, size=s.kv_lora_rank)).astype(np.float32)
    return Weights(s, dense, codes, scales, q_norm_w, kv_norm_w)


# ----------------------------------------------------------------------------
# decode inputs
# ----------------------------------------------------------------------------

@dataclass
class DecodeInputs:
    hidden: np.ndarray          # [n, hidden] float32 (act-dtype values)
    positions: np.ndarray       # [n] int32 = context_len - 1
    context_lens: np.ndarray    # [n] int32 (counts this step's token)
    block_table: np.ndarray     # [n, max_blocks_per_seq] int32 (unused entries = -1)
    slot_mapping: np.ndarray    # [n] int32 = physical row of position context_len-1
    n_blocks: int
    cache: np.ndarray           # [n_blocks, 1, block_size, R] float32 (act-dtype values);
                                # rows the fill step would write are zero here
    fill_hidden: list | None    # "project" fill: per sequence [ctx-1, hidden] float32
    fill_slots: list | None     #   and the physical rows they go to ([ctx-1] int32)


def _context_lens(w: Workload, rng) -> np.ndarray:
    if w.ctx_lo == w.ctx_hi:
        return np.full(w.batch, w.ctx_lo, np.int32)
    return rng.integers(w.ctx_lo, w.ctx_hi + 1, size=w.batch).astype(np.int32)


def make_decode_inputs(w: Workload, seed_offset: int = 100, batch: int | None = None,
                       ctx: tuple | None = None) -> DecodeInputs:
    """Decode-step inputs for workload `w` (optionally with a smaller batch / ctx range)."""
    s = w.shape
    if batch is not None or ctx is not None:
        w = dataclasses.replace(w, batch=batch or w.batch,
                                ctx_lo=(ctx or (w.ctx_lo, w.ctx_hi))[0],
                                ctx_hi=(ctx or (w.ctx_lo, w.ctx_hi))[1])
    rng = np.random.default_rng(w.seed + seed_offset)
    bs, R = s.block_size, s.kv_row_dim
    lens = _context_lens(w, rng)
    nb_per_seq = (lens + bs - 1) // bs
    n_blocks = int(nb_per_seq.sum()) + w.spare_blocks
    perm = rng.permutation(n_blocks).astype(np.int32)     # random physical blocks
    maxb = int(nb_per_seq.max())
    table = np.full((w.batch, maxb), -1, np.int32)
    off = 0
    for b in range(w.batch):
        table[b, :nb_per_seq[b]] = perm[off:off + nb_per_seq[b]]
        off += nb_per_seq[b]
    pos = (lens - 1).astype(np.int32)
    slot = np.array([table[b, pos[b] // bs] * bs + pos[b] % bs for b in range(w.batch)],
                    np.int32)
    hidden = round_to(rng.standard_normal((w.batch, s.hidden), dtype=np.float32), s.act_dtype)
    cache = np.zeros((n_blocks, 1, bs, R), np.float32)
    fill_hidden = fill_slots = None
    if w.cache_fill == "random":
        cache = round_to(rng.standard_normal(cache.shape, dtype=np.float32), s.act_dtype)
    elif w.cache_fill == "project":
        fill_hidden, fill_slots = [], []
        for b in range(w.batch):
            p = np.arange(lens[b] - 1)
            fill_slots.append((table[b, p // bs] * bs + p % bs).astype(np.int32))
            fill_hidden.append(round_to(
                rng.standard_normal((lens[b] - 1, s.hidden), dtype=np.float32), s.act_dtype))
    return DecodeInputs(hidden, pos, lens, table, slot, n_blocks, cache, fill_hidden, fill_slots)


def make_prefill_inputs(w: Workload, seq_len: int | None = None, seed_offset: int = 200):
    """hidden [S, hidden] float32 (act-dtype values) and positions 0..S-1."""
    s = w.shape
    S = seq_len or w.seq_len
    rng = np.random.default_rng(w.seed + seed_offset)
    hidden = round_to(rng.standard_normal((S, s.hidden), dtype=np.float32), s.act_dtype)
    return hidden, np.arange(S, dtype=np.int32)


def shrink(w: Workload, **shape_changes) -> Workload:
    """Same workload with a modified shape (smaller parity cases)."""
    return dataclasses.replace(w, shape=dataclasses.replace(w.shape, **shape_changes))
