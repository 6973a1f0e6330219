"""fp64 CPU oracle of the MLA layer step.  TEST INFRASTRUCTURE ONLY.

Plain, slow and meant to be read against the pages. Only tests/,
__graft_entry__.smoke() and bench.py's cpu_baseline / reference leg may import
this module; the library's product path never does, and this module imports
nothing from the library (it shares no code with the CUDA path: no kernels,
headers, helpers or table generators).

Every quantity is numpy float64; inputs that arrive in bf16 / e4m3 are upcast
exactly and nothing is rounded in between. Each function names the passage it
follows. Where a page is silent or ambiguous the reading adopted is stated in
the function's docstring.

Notation (the pages'): n tokens, H heads, hidden D, q_lora_rank r_q,
kv_lora_rank r_kv, qk_nope d_n, qk_rope d_r, v_dim d_v, block_size bs,
kv_row_dim R = r_kv + d_r.

Pins: every function here is pinned by tests/test_oracle_*.py against brute
force loops, closed forms, library routines (torch fp64 SDPA, torch's e4m3
cast) or identities the pages state. No function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

LATENT_FIRST = 0   # cache row [latent | k_pe]  (DeepSeek's order)
PE_FIRST = 1       # cache row [k_pe | latent]  (the NKI kernel's inverted order)


# ----------------------------------------------------------------------------
# primitive steps
# ----------------------------------------------------------------------------

def rms_norm(v, gamma, eps):
    """RMSNorm over the last axis: v / sqrt(mean(v^2) + eps) * gamma.

    "MLA Decode QKV Kernel API Reference", Parameters (q_norm_w, kv_norm_w:
    RMSNorm gammas; norm_eps, default 1e-6). eps sits inside the square root
    (the usual RMSNorm definition; the page does not spell it out).
    """
    v = np.asarray(v, np.float64)
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * np.asarray(gamma, np.float64)


def rope_inv_freq(rope_dim, theta):
    """inv_freq_i = theta^(-2i / d_r), i < d_r/2 (plain-theta RoPE; "Struct MlaWeights",
    field yarn_inv_freq: NULL selects the standard theta computation)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / rope_dim)


def rope_cos_sin(positions, rope_dim, theta, inv_freq=None):
    """Half-width tables [n, d_r/2] of cos/sin(pos * inv_freq_i).

    Half width as "MLA Decode QKV Kernel API Reference", Parameters (cos, sin:
    [n_tokens, qk_rope_dim // 2]). inv_freq, when given, is a precomputed
    [d_r/2] table used as is ("Struct MlaWeights", field yarn_inv_freq: a
    precomputed YaRN inv_freq table [rotary_dim/2]; NULL selects the standard
    theta computation), and theta is then unused.
    """
    f = rope_inv_freq(rope_dim, theta) if inv_freq is None else np.asarray(inv_freq, np.float64)
    phi = np.asarray(positions, np.float64)[:, None] * f[None, :]
    return np.cos(phi), np.sin(phi)


def rope_interleaved(v, cos, sin):
    """Interleaved RoPE: element 2i pairs with element 2i+1.

    "MLA Decode QKV Kernel API Reference", Notes ("RoPE here is interleaved:
    element 2i pairs with element 2i + 1", in contrast with the indexer's
    half-split pairing). The pair (a, b) is rotated by phi_i:
    (a cos - b sin, a sin + b cos), i.e. complex multiplication by e^{i phi}
    (the freqs_cis that the NeMo MLA.forward takes). cos/sin broadcast against
    v[..., ::2].
    """
    v = np.asarray(v, np.float64)
    a, b = v[..., 0::2], v[..., 1::2]
    out = np.empty(np.broadcast_shapes(v.shape), np.float64)
    out[..., 0::2] = a * cos - b * sin
    out[..., 1::2] = a * sin + b * cos
    return out


def softmax(s, axis=-1):
    """Max-subtracted softmax."""
    s = np.asarray(s, np.float64)
    e = np.exp(s - np.max(s, axis=axis, keepdims=True))
    return e / np.sum(e, axis=axis, keepdims=True)


def softmax_with_sink(s, sink):
    """Softmax over the last axis with one extra logit per row that carries no
    value: p_j = e^{s_j} / (sum_k e^{s_k} + e^{sink}).

    "Struct MlaWeights", attn_sink: a per-head attention sink logit (DeepSeek-V4
    s_aux). The page gives only that it is one logit per query head. Reading
    adopted: the sink is one more column of the softmax, in the units of the
    scaled scores, and its own probability is dropped, so a head's weights sum
    to less than one. Written as exactly that: the plain softmax of the row
    extended by the sink, without its last column.
    """
    s = np.asarray(s, np.float64)
    sink = np.broadcast_to(np.asarray(sink, np.float64), s.shape[:-1])
    full = np.concatenate([s, sink[..., None]], axis=-1)
    return softmax(full, axis=-1)[..., :-1]


def softmax_scale(qk_nope, qk_rope, mscale=1.0):
    """1/sqrt(qk_nope + qk_rope) * mscale^2.

    "struct Mla", field scale (YaRN's magnitude squared; mscale = 1 without
    YaRN); nemo_automodel deepseek_v3.layers MLA.softmax_scale = qk_head_dim**-0.5.
    The absorbed dot product is r_kv + d_r long, but the scale stays that of the
    expanded head dim d_n + d_r.
    """
    return (qk_nope + qk_rope) ** -0.5 * mscale * mscale


# ----------------------------------------------------------------------------
# FP8-E4M3 weights with 128x128 block scales
# ----------------------------------------------------------------------------

def e4m3_to_float(code):
    """Decode OCP FP8 E4M3 codes: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (m/8 * 2^-6); no infinities; S.1111.111 is NaN.

    Written from the OCP 8-bit floating point specification (E4M3 variant), the
    format "Struct MlaWeights" (field wq_a_fp8) names.
    """
    c = np.asarray(code).astype(np.int64)
    sign = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


def dequant_block128(codes, scales):
    """W[k, n] = e4m3(code[k, n]) * scale[k // 128, n // 128].

    "Struct MlaWeights", field wq_a_fp8 (FP8-E4M3 + 128x128 block scales,
    dequantised in fp32 before the MAC); scale tensor [ceil(K/128), ceil(N/128)]
    as "QKV CTE MLA Kernel API Reference", qkv_mla_mx (*_scale_hbm).
    """
    k, n = codes.shape
    s = np.asarray(scales, np.float64)
    full = np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)[:k, :n]
    return e4m3_to_float(codes) * full


# ----------------------------------------------------------------------------
# weight views
# ----------------------------------------------------------------------------

def split_wkv_b(wkv_b, n_heads, qk_nope, v_dim):
    """W_UK [H, d_n, r_kv] and W_UV [H, r_kv, d_v] from wkv_b [r_kv, H*(d_n+d_v)].

    wkv_b shape: "QKV CTE MLA Kernel API Reference", KV Path Stage 2 (split into
    k_nope and v). Per head the columns are contiguous [k_nope_h | v_h] (the
    plain reshape [H, d_n + d_v]; "struct Mla", field kv_b_split: one attn_kv_b
    of qk_nope + v_dim rows a head). W_UK is the nope half ("MLA Decode QKV
    Kernel API Reference", q_absorb_w [n_heads, qk_nope_dim, kv_lora_rank];
    "Struct MlaWeights", w_uk_t); W_UV the value half ("Struct MlaWeights", w_uv
    [n_heads, kv_lora, v_dim]).
    """
    w = np.asarray(wkv_b, np.float64)
    r_kv = w.shape[0]
    w = w.reshape(r_kv, n_heads, qk_nope + v_dim)
    w_uk = np.ascontiguousarray(w[:, :, :qk_nope].transpose(1, 2, 0))   # [H, d_n, r_kv]
    w_uv = np.ascontiguousarray(w[:, :, qk_nope:].transpose(1, 0, 2))   # [H, r_kv, d_v]
    return w_uk, w_uv


def fused_w_qk(wq_b, w_uk, n_heads, qk_nope, qk_rope):
    """W_QK[h, l, c] = sum_p wq_b_nope[h, p, l] * W_UK[h, p, c]  ("Struct MlaWeights",
    w_qk_absorbed). Used only as an identity check: q_abs = q_lat_n @ W_QK."""
    rq = wq_b.shape[0]
    wb = np.asarray(wq_b, np.float64).reshape(rq, n_heads, qk_nope + qk_rope)[:, :, :qk_nope]
    return np.einsum("lhp,hpc->hlc", wb, w_uk)


# ----------------------------------------------------------------------------
# the cache row and the paged cache
# ----------------------------------------------------------------------------

def cache_row(c_kv, k_pe, layout):
    """One cache row per token: LATENT_FIRST [c_kv | k_pe] or PE_FIRST [k_pe | c_kv].

    "MLA Decode QKV Kernel API Reference", Notes: the NKI kernel lays the row out
    [k_pe | kv_latent], inverting DeepSeek's [latent | k_pe]; both are offered.
    """
    if layout == LATENT_FIRST:
        return np.concatenate([c_kv, k_pe], axis=-1)
    if layout == PE_FIRST:
        return np.concatenate([k_pe, c_kv], axis=-1)
    raise ValueError(layout)


def split_row(rows, r_kv, layout):
    """Inverse of cache_row: (c_kv, k_pe)."""
    if layout == LATENT_FIRST:
        return rows[..., :r_kv], rows[..., r_kv:]
    return rows[..., rows.shape[-1] - r_kv:], rows[..., :rows.shape[-1] - r_kv]


def scatter_rows(kv_cache, slot_mapping, rows):
    """Write rows[t] to flat cache row slot_mapping[t] ("MLA Decode QKV Kernel API
    Reference", Parameters: kv_cache [n_blocks, 1, block_size, kv_row_dim] mutated
    in place; slot_mapping [n_tokens] int32, the destination row per token).
    A negative slot skips the token (padding). Returns a new array."""
    cache = np.array(kv_cache, np.float64, copy=True)
    flat = cache.reshape(-1, cache.shape[-1])
    for t, slot in enumerate(np.asarray(slot_mapping)):
        if slot >= 0:
            flat[int(slot)] = rows[t]
    return cache


def gather_context(kv_cache, block_table_row, context_len, block_size):
    """Rows of positions 0..L-1 of one sequence: position j lives in physical block
    block_table[j // bs] at offset j % bs (the flat slot block*bs + offset, as
    slot_mapping addresses it)."""
    flat = np.asarray(kv_cache, np.float64).reshape(-1, kv_cache.shape[-1])
    j = np.arange(context_len)
    slots = np.asarray(block_table_row)[j // block_size].astype(np.int64) * block_size + j % block_size
    return flat[slots]


# ----------------------------------------------------------------------------
# the decode step
# ----------------------------------------------------------------------------

def q_projection(cfg, W, hidden):
    """q [n, H, d_n + d_r] before RoPE.

    Low-rank path: q = rms_norm(x @ wq_a, q_norm_w) @ wq_b ("Struct MlaWeights":
    input x wq_a -> latent -> norm -> x wq_b; "MLA Decode QKV Kernel API
    Reference", wq_a, q_norm_w, wq_b). With q_lora_rank = 0 the query is one full
    projection x @ q_proj ("struct Mla": "The query is a full projection, or
    itself low-rank"); W['wq_b'] then holds q_proj [hidden, H*(d_n+d_r)].
    Per head the output is [q_nope | q_pe] ("... wq_b ... emitting every head's
    [q_nope | q_pe] concatenated").
    """
    x = np.asarray(hidden, np.float64)
    if cfg.q_lora_rank:
        q = rms_norm(x @ W["wq_a"], W["q_norm_w"], cfg.norm_eps) @ W["wq_b"]
    else:
        q = x @ W["wq_b"]
    return q.reshape(x.shape[0], cfg.n_heads, cfg.qk_nope + cfg.qk_rope)


def q_latent_normed(cfg, W, hidden):
    """rms_norm(x @ wq_a, q_norm_w) (low-rank query path only)."""
    return rms_norm(np.asarray(hidden, np.float64) @ W["wq_a"], W["q_norm_w"], cfg.norm_eps)


def kv_projection(cfg, W, hidden, cos, sin):
    """(c_kv normed [n, r_kv], k_pe rotated [n, d_r]).

    kv = x @ wkv_a, one cache row per token in DeepSeek's [latent | k_pe] output
    order ("MLA Decode QKV Kernel API Reference", wkv_a [hidden, kv_row_dim];
    "QKV CTE MLA Kernel API Reference", Split: kv, k_pe). Only the latent is
    RMS-normed, with kv_norm_w [1, kv_lora_rank]; k_pe is rotated, never normed.
    """
    kv = np.asarray(hidden, np.float64) @ W["wkv_a"]
    c = rms_norm(kv[:, :cfg.kv_lora_rank], W["kv_norm_w"], cfg.norm_eps)
    k_pe = rope_interleaved(kv[:, cfg.kv_lora_rank:], cos, sin)
    return c, k_pe


def decode_q(cfg, W, hidden, cos, sin):
    """(q_nope [n, H, d_n], q_pe rotated [n, H, d_r])."""
    q = q_projection(cfg, W, hidden)
    q_nope = q[..., :cfg.qk_nope]
    q_pe = rope_interleaved(q[..., cfg.qk_nope:], cos[:, None, :], sin[:, None, :])
    return q_nope, q_pe


def absorb(q_nope, w_uk):
    """q_abs[t, h, c] = sum_p q_nope[t, h, p] * W_UK[h, p, c]
    ("MLA Decode QKV Kernel API Reference", q_absorb_w; "Struct MlaWeights",
    w_uk_t: Q_absorbed = Q_nope @ W_UK_T)."""
    return np.einsum("thp,hpc->thc", q_nope, w_uk)


def input_norm(cfg, hidden, input_norm_w):
    """The layer's input RMSNorm, rms_norm(x, input_norm_w) with eps = norm_eps.

    "MLA Decode QKV Kernel API Reference", Parameters (input_norm_w: [1,
    hidden] fp32, optional; when given, the layer's input RMSNorm is folded into
    the hidden load). The page names no separate epsilon, so the reading is the
    kernel's norm_eps.
    """
    return rms_norm(hidden, input_norm_w, cfg.norm_eps)


def decode_qkv(cfg, W, hidden, cos, sin, kv_cache, slot_mapping, row_layout=LATENT_FIRST, input_norm_w=None):
    """The decode front-fold: (q_abs [n,H,r_kv], q_pe [n,H,d_r], new kv_cache).

    "MLA Decode QKV Kernel API Reference", mla_decode_qkv: query and KV
    projections, both RMSNorms, interleaved RoPE, absorption of the query into
    the latent space, and the scatter of this step's row into the paged cache.
    With input_norm_w the hidden states are first RMS-normalised (input_norm).
    """
    if input_norm_w is not None:
        hidden = input_norm(cfg, hidden, input_norm_w)
    q_nope, q_pe = decode_q(cfg, W, hidden, cos, sin)
    c, k_pe = kv_projection(cfg, W, hidden, cos, sin)
    w_uk, _ = split_wkv_b(W["wkv_b"], cfg.n_heads, cfg.qk_nope, cfg.v_dim)
    q_abs = absorb(q_nope, w_uk)
    cache = scatter_rows(kv_cache, slot_mapping, cache_row(c, k_pe, row_layout))
    return q_abs, q_pe, cache


def grouped_o_projection(head_out, wo_a, wo_b, o_groups):
    """DeepSeek-V4 grouped low-rank output projection ("Struct MlaWeights",
    wo_a / wo_b / o_lora_rank: wo_a -> wo_b replaces wo; wo_a is sliced per
    o_group, block-diagonal). The heads split into o_groups consecutive groups;
    group g's head outputs, flattened to [(H/G) d_v], go through its own block
    wo_a[g] [(H/G) d_v, r_o] (rows g (H/G) d_v .. of wo_a); the G low-rank
    vectors, concatenated in group order, go through wo_b [G r_o, D].
    head_out [n, H, d_v] -> out [n, D]."""
    n, H, dv = head_out.shape
    G = o_groups
    hg = H // G
    wo_a = np.asarray(wo_a, np.float64)
    z = [np.asarray(head_out[:, g * hg:(g + 1) * hg, :], np.float64).reshape(n, hg * dv)
         @ wo_a[g * hg * dv:(g + 1) * hg * dv] for g in range(G)]
    return np.concatenate(z, axis=1) @ np.asarray(wo_b, np.float64)


def o_projection(cfg, W, head_out):
    """out = concat_h(o[h]) @ wo, or the grouped low-rank wo_a -> wo_b when the
    shape has o_lora_rank > 0 (grouped_o_projection)."""
    if getattr(cfg, "o_lora_rank", 0):
        return grouped_o_projection(head_out, W["wo_a"], W["wo_b"], cfg.o_groups)
    return np.asarray(head_out, np.float64).reshape(head_out.shape[0], -1) @ np.asarray(W["wo"], np.float64)


def decode_attn(cfg, W, q_abs, q_pe, kv_cache, block_table, context_lens,
                row_layout=LATENT_FIRST, scale=None, attn_sink=None):
    """Absorbed attention over the latent cache, V extraction and o_proj.

    For token t (sequence t) with L = context_lens[t] rows:
      s[h, j] = (q_abs[h] . c_j + q_pe[h] . k_pe_j) * scale
      p = softmax_j(s);  o_lat[h] = sum_j p[h, j] c_j;  o[h] = o_lat[h] @ W_UV[h]
      out = concat_h(o[h]) @ wo
    "Struct MlaWeights": w_uk_t (absorption), w_uv (v_out = attn_latent @ W_UV),
    wo; "struct Mla": scale. attn_sink [H] (optional): each head's softmax
    takes the sink logit as one more column (softmax_with_sink).
    Returns (out [n, hidden], head_out [n, H, d_v]).
    """
    scale = softmax_scale(cfg.qk_nope, cfg.qk_rope) if scale is None else scale
    _, w_uv = split_wkv_b(W["wkv_b"], cfg.n_heads, cfg.qk_nope, cfg.v_dim)
    n = q_abs.shape[0]
    head_out = np.zeros((n, cfg.n_heads, cfg.v_dim))
    for t in range(n):
        rows = gather_context(kv_cache, block_table[t], int(context_lens[t]), cfg.block_size)
        c, k_pe = split_row(rows, cfg.kv_lora_rank, row_layout)
        s = (np.asarray(q_abs[t], np.float64) @ c.T
             + np.asarray(q_pe[t], np.float64) @ k_pe.T) * scale           # [H, L]
        p = softmax(s, axis=-1) if attn_sink is None else softmax_with_sink(s, attn_sink)
        o_lat = p @ c                                                      # [H, r_kv]
        head_out[t] = np.einsum("hc,hcd->hd", o_lat, w_uv)
    out = o_projection(cfg, W, head_out)
    return out, head_out


def decode_attn_expanded(cfg, W, q_nope, q_pe, kv_cache, block_table, context_lens,
                         row_layout=LATENT_FIRST, scale=None):
    """The same attention in the unabsorbed form: every head's K and V are
    rebuilt from the latent (k_nope_j[h] = W_UK[h] c_j, v_j[h] = c_j W_UV[h],
    K_h = [k_nope | k_pe] with k_pe shared by all heads). "struct Mla" (keys and
    values of every head expanded from one shared latent; the rotating key dims
    are shared by every head); "QKV CTE MLA Kernel API Reference", Final assembly.
    """
    scale = softmax_scale(cfg.qk_nope, cfg.qk_rope) if scale is None else scale
    w_uk, w_uv = split_wkv_b(W["wkv_b"], cfg.n_heads, cfg.qk_nope, cfg.v_dim)
    n = q_nope.shape[0]
    head_out = np.zeros((n, cfg.n_heads, cfg.v_dim))
    for t in range(n):
        rows = gather_context(kv_cache, block_table[t], int(context_lens[t]), cfg.block_size)
        c, k_pe = split_row(rows, cfg.kv_lora_rank, row_layout)
        k_nope = np.einsum("hpc,jc->hjp", w_uk, c)                         # [H, L, d_n]
        v = np.einsum("jc,hcd->hjd", c, w_uv)                              # [H, L, d_v]
        s = (np.einsum("hp,hjp->hj", q_nope[t], k_nope) + q_pe[t] @ k_pe.T) * scale
        p = softmax(s, axis=-1)
        head_out[t] = np.einsum("hj,hjd->hd", p, v)
    out = o_projection(cfg, W, head_out)
    return out, head_out


# ----------------------------------------------------------------------------
# prefill (context encoding): the expanded path
# ----------------------------------------------------------------------------

def prefill(cfg, W, hidden, cos, sin, rows=None, scale=None, row_layout=LATENT_FIRST, attn_sink=None):
    """Causal prefill of one sequence with K/V expanded from the latent.

    "QKV CTE MLA Kernel API Reference", qkv_mla_mx Notes: Stage 1 x @ [wq_a | wkv_a]
    split into q_lat, kv, k_pe; Q Stage 2 norm(q_lat) @ wq_b; KV Stage 2
    norm(kv) @ wkv_b split per head into k_nope, v; Final assembly: RoPE on q_pe
    and k_pe, k_pe broadcast to all heads and concatenated with k_nope. Then
    causal softmax(Q K^T * scale) V (query i sees keys j <= i) and o_proj.
    attn_sink [H] (optional): each head's softmax takes the sink logit as one
    more column (softmax_with_sink).

    rows: query rows to evaluate (default all). K/V are always built for all S
    tokens. Returns (out [len(rows), hidden], head_out [len(rows), H, d_v],
    cache_rows [S, R] in `row_layout`).
    """
    scale = softmax_scale(cfg.qk_nope, cfg.qk_rope) if scale is None else scale
    x = np.asarray(hidden, np.float64)
    S = x.shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows)
    H, dn, dv = cfg.n_heads, cfg.qk_nope, cfg.v_dim
    c, k_pe = kv_projection(cfg, W, x, cos, sin)                       # [S, r_kv], [S, d_r]
    kv_out = (c @ np.asarray(W["wkv_b"], np.float64)).reshape(S, H, dn + dv)
    k_nope, v = kv_out[..., :dn], kv_out[..., dn:]
    q_nope, q_pe = decode_q(cfg, W, x[rows], cos[rows], sin[rows])     # [m, H, *]
    head_out = np.zeros((len(rows), H, dv))
    for m, i in enumerate(rows):
        i = int(i)
        s = (np.einsum("hp,jhp->hj", q_nope[m], k_nope[:i + 1])
             + q_pe[m] @ k_pe[:i + 1].T) * scale                       # [H, i+1]
        p = softmax(s, axis=-1) if attn_sink is None else softmax_with_sink(s, attn_sink)
        head_out[m] = np.einsum("hj,jhd->hd", p, v[:i + 1])
    out = o_projection(cfg, W, head_out)
    return out, head_out, cache_row(c, k_pe, row_layout)


# ----------------------------------------------------------------------------
# DeepSeek-V4 QKV projection
# ----------------------------------------------------------------------------

def head_rms(q, eps):
    """Each head's vector divided by the root of its mean square (+ eps), no gain:
    the "per-head rsqrt norm" of "QKV CTE MLA Kernel API Reference",
    qkv_mla_mx_deepseek_v4, Final assembly. Reading adopted: the RMS form of
    the norm used everywhere else on the pages, with the kernel's norm_eps."""
    q = np.asarray(q, np.float64)
    return q / np.sqrt(np.mean(q * q, axis=-1, keepdims=True) + eps)


def v4_qkv(cfg, W, hidden, cos, sin, kv_norm_w):
    """(q [n, H, hd], kv [n, kv_dim]) of the DeepSeek-V4 QKV projection.

    "QKV CTE MLA Kernel API Reference", qkv_mla_mx_deepseek_v4, Notes:
      fused first projection x @ wqkv [H_in, qk_lora_rank + kv_dim], split into
      qr [qk_lora_rank] and kv [kv_dim] (kv_dim = kv_lora_rank + qk_rope);
      Q stage 2: norm(qr) @ wq_b [qk_lora_rank, n_heads * head_dim], with the
      q_norm gamma;
      final assembly: q -> per-head rsqrt norm -> RoPE on the last qk_rope dims
      of each head; kv -> RMSNorm with kv_norm_gamma [kv_dim] over all kv_dim
      columns -> RoPE on its last qk_rope columns (the kv latent is returned).
    Here wqkv is [wq_a | wkv_a] (the same fused first projection this library
    already uses), head_dim = qk_nope + qk_rope, and kv_norm_w has kv_dim
    entries. Readings: RoPE is the interleaved pairing of the decode page; the
    per-head norm is head_rms.
    """
    x = np.asarray(hidden, np.float64)
    eps = cfg.norm_eps
    H, hd, dr = cfg.n_heads, cfg.qk_nope + cfg.qk_rope, cfg.qk_rope
    qr = x @ np.asarray(W["wq_a"], np.float64)
    kv = x @ np.asarray(W["wkv_a"], np.float64)
    q = (rms_norm(qr, W["q_norm_w"], eps) @ np.asarray(W["wq_b"], np.float64)).reshape(x.shape[0], H, hd)
    q = head_rms(q, eps)
    q[..., hd - dr:] = rope_interleaved(q[..., hd - dr:], cos[:, None, :], sin[:, None, :])
    kv = rms_norm(kv, kv_norm_w, eps)
    R = kv.shape[1]
    kv[:, R - dr:] = rope_interleaved(kv[:, R - dr:], cos, sin)
    return q, kv


# ----------------------------------------------------------------------------
# glue: weights in the C-ABI input format -> fp64 dict
# ----------------------------------------------------------------------------

def weights_fp64(weights):
    """fp64 dict {wq_a?, wq_b, wkv_a, wkv_b, wo, q_norm_w?, kv_norm_w} from a
    workloads.Weights (dense values, or e4m3 codes + block scales)."""
    W = {}
    for name in ("wq_a", "wq_b", "wkv_a", "wkv_b", "wo", "wo_a", "wo_b"):
        if name in weights.dense:
            W[name] = np.asarray(weights.dense[name], np.float64)
        elif name in weights.codes:
            W[name] = dequant_block128(weights.codes[name], weights.scales[name])
    if weights.q_norm_w is not None:
        W["q_norm_w"] = np.asarray(weights.q_norm_w, np.float64)
    W["kv_norm_w"] = np.asarray(weights.kv_norm_w, np.float64)
    return W


def fill_cache_by_projection(cfg, W, cache, fill_hidden, fill_slots, row_layout=LATENT_FIRST):
    """Earlier cache rows of each sequence: the front-fold's (normed latent,
    rotated k_pe) row of that position's hidden state, at that position."""
    cache = np.array(cache, np.float64, copy=True)
    for xs, slots in zip(fill_hidden, fill_slots):
        if len(slots) == 0:
            continue
        cos, sin = rope_cos_sin(np.arange(len(slots)), cfg.qk_rope, cfg.rope_theta)
        c, k_pe = kv_projection(cfg, W, xs, cos, sin)
        cache = scatter_rows(cache, slots, cache_row(c, k_pe, row_layout))
    return cache
