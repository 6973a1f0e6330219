"""Pins of the fp64 oracle against things other than itself.

Brute-force loops (oracle/brute.py), closed forms, invariants the pages state
and library routines (torch fp64 scaled_dot_product_attention, torch's e4m3
cast). CPU only.
"""
import dataclasses
import json
import math
import os

import numpy as np
import pytest
import torch

from head_latent_attention_decode_b200 import workloads as wl
from oracle import brute
from oracle import mla_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

SMALL = wl.MlaShape(hidden=24, n_heads=2, q_lora_rank=12, kv_lora_rank=8, qk_nope=4,
                    qk_rope=4, v_dim=6, block_size=2, act_dtype="f32", weight_dtype="f32")
SMALL_NOQ = dataclasses.replace(SMALL, q_lora_rank=0)


def _weights(shape, seed):
    return ref.weights_fp64(wl.make_weights(shape, seed))


def _decode_case(shape, seed, batch=3, ctx=(1, 5), layout=ref.LATENT_FIRST):
    w = wl.Workload("t", shape, "decode", batch=batch, ctx_lo=ctx[0], ctx_hi=ctx[1],
                    cache_fill="random", seed=seed)
    inp = wl.make_decode_inputs(w)
    W = _weights(shape, seed)
    cos, sin = ref.rope_cos_sin(inp.positions, shape.qk_rope, shape.rope_theta)
    return W, inp, cos, sin


@pytest.mark.parametrize("shape", [SMALL, SMALL_NOQ])
@pytest.mark.parametrize("layout", [ref.LATENT_FIRST, ref.PE_FIRST])
def test_decode_matches_brute_force(shape, layout):
    W, inp, cos, sin = _decode_case(shape, 7)
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache,
                                        inp.slot_mapping, layout)
    out, head_out = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table,
                                    inp.context_lens, layout)
    flat_rows = inp.cache.reshape(-1, shape.kv_row_dim).tolist()
    b_out, b_head, b_qabs, b_qpe, b_rows = brute.decode_step(
        shape, W, inp.hidden, inp.positions, flat_rows, inp.block_table.tolist(),
        inp.context_lens, inp.slot_mapping, layout)
    np.testing.assert_allclose(q_abs, np.array(b_qabs), rtol=0, atol=1e-12)
    np.testing.assert_allclose(q_pe, np.array(b_qpe), rtol=0, atol=1e-12)
    np.testing.assert_allclose(cache.reshape(-1, shape.kv_row_dim), np.array(b_rows), rtol=0, atol=1e-12)
    np.testing.assert_allclose(head_out, np.array(b_head), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


def _yarn_like_inv_freq(rope_dim, theta=10000.0, factor=8.0):
    """A frequency table of the YaRN kind for the pins: the low frequencies
    divided by `factor`, the high ones kept, a linear ramp in between (any
    positive table serves; only its use as given is pinned)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    base = theta ** (-2.0 * i / rope_dim)
    ramp = np.clip((i - 0.25 * len(i)) / max(0.5 * len(i), 1.0), 0.0, 1.0)
    return base * (1.0 - ramp) + base / factor * ramp


@pytest.mark.parametrize("shape", [SMALL, SMALL_NOQ])
def test_decode_with_input_norm_and_inv_freq_matches_brute_force(shape):
    """The optional input RMSNorm ("MLA Decode QKV Kernel API Reference",
    input_norm_w) and a precomputed RoPE frequency table ("Struct MlaWeights",
    yarn_inv_freq) against the literal loops."""
    W, inp, _, _ = _decode_case(shape, 11)
    rng = np.random.default_rng(11)
    g_in = 1.0 + rng.uniform(-0.3, 0.3, shape.hidden)
    f = _yarn_like_inv_freq(shape.qk_rope)
    cos, sin = ref.rope_cos_sin(inp.positions, shape.qk_rope, shape.rope_theta, inv_freq=f)
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping,
                                        input_norm_w=g_in)
    out, head_out = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    b_out, b_head, b_qabs, b_qpe, b_rows = brute.decode_step(
        shape, W, inp.hidden, inp.positions, inp.cache.reshape(-1, shape.kv_row_dim).tolist(),
        inp.block_table.tolist(), inp.context_lens, inp.slot_mapping, input_norm_w=g_in, inv_freq=f)
    np.testing.assert_allclose(q_abs, np.array(b_qabs), rtol=0, atol=1e-12)
    np.testing.assert_allclose(q_pe, np.array(b_qpe), rtol=0, atol=1e-12)
    np.testing.assert_allclose(cache.reshape(-1, shape.kv_row_dim), np.array(b_rows), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


def test_input_norm_removes_the_input_scale():
    """RMSNorm makes the front-fold blind to a positive scale of x (up to eps):
    scaling the hidden states by 3.7 changes nothing, whereas without the
    norm the unnormed k_pe scales with x."""
    W, inp, cos, sin = _decode_case(SMALL, 12)
    g_in = 1.0 + np.random.default_rng(12).uniform(-0.3, 0.3, SMALL.hidden)
    a = ref.decode_qkv(SMALL, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping, input_norm_w=g_in)
    b = ref.decode_qkv(SMALL, W, 3.7 * inp.hidden, cos, sin, inp.cache, inp.slot_mapping, input_norm_w=g_in)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-6, atol=1e-9)
    c = ref.decode_qkv(SMALL, W, 3.7 * inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    d = ref.decode_qkv(SMALL, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    assert np.max(np.abs(c[2] - d[2])) > 1e-3


def test_inv_freq_table_of_plain_theta_reproduces_theta():
    pos = np.array([0, 1, 7, 4095])
    c0, s0 = ref.rope_cos_sin(pos, 64, 10000.0)
    i = np.arange(32)
    c1, s1 = ref.rope_cos_sin(pos, 64, 1.0, inv_freq=10000.0 ** (-i / 32.0))
    np.testing.assert_allclose(c0, c1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s0, s1, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape", [SMALL, SMALL_NOQ])
def test_prefill_matches_brute_force(shape):
    W = _weights(shape, 3)
    x = np.random.default_rng(3).standard_normal((5, shape.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(5), shape.qk_rope, shape.rope_theta)
    out, head_out, _ = ref.prefill(shape, W, x, cos, sin)
    b_out, b_head = brute.prefill(shape, W, x)
    np.testing.assert_allclose(head_out, np.array(b_head), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


def test_prefill_rows_subset_matches_full():
    W = _weights(SMALL, 4)
    x = np.random.default_rng(4).standard_normal((9, SMALL.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(9), SMALL.qk_rope, SMALL.rope_theta)
    full, hfull, _ = ref.prefill(SMALL, W, x, cos, sin)
    part, hpart, _ = ref.prefill(SMALL, W, x, cos, sin, rows=[0, 4, 8])
    np.testing.assert_allclose(part, full[[0, 4, 8]], atol=1e-13)


# ---------------------------------------------------------------------------
# identities the pages state
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("layout", [ref.LATENT_FIRST, ref.PE_FIRST])
def test_absorbed_equals_expanded(layout):
    shape = dataclasses.replace(SMALL, hidden=64, n_heads=3, kv_lora_rank=16, qk_nope=8,
                                qk_rope=6, v_dim=5, block_size=4)
    W, inp, cos, sin = _decode_case(shape, 11, batch=4, ctx=(1, 19))
    q_nope, q_pe = ref.decode_q(shape, W, inp.hidden, cos, sin)
    w_uk, _ = ref.split_wkv_b(W["wkv_b"], shape.n_heads, shape.qk_nope, shape.v_dim)
    q_abs = ref.absorb(q_nope, w_uk)
    a_out, a_head = ref.decode_attn(shape, W, q_abs, q_pe, inp.cache, inp.block_table,
                                    inp.context_lens, layout)
    e_out, e_head = ref.decode_attn_expanded(shape, W, q_nope, q_pe, inp.cache,
                                             inp.block_table, inp.context_lens, layout)
    np.testing.assert_allclose(a_head, e_head, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(a_out, e_out, rtol=1e-10, atol=1e-12)


def test_fused_w_qk_equals_two_stage():
    shape = SMALL
    W = _weights(shape, 5)
    x = np.random.default_rng(5).standard_normal((3, shape.hidden))
    ql = ref.q_latent_normed(shape, W, x)
    w_uk, _ = ref.split_wkv_b(W["wkv_b"], shape.n_heads, shape.qk_nope, shape.v_dim)
    w_qk = ref.fused_w_qk(W["wq_b"], w_uk, shape.n_heads, shape.qk_nope, shape.qk_rope)
    cos, sin = ref.rope_cos_sin(np.zeros(3), shape.qk_rope, shape.rope_theta)
    q_nope, _ = ref.decode_q(shape, W, x, cos, sin)
    two_stage = ref.absorb(q_nope, w_uk)
    fused = np.einsum("tl,hlc->thc", ql, w_qk)
    np.testing.assert_allclose(fused, two_stage, rtol=1e-11, atol=1e-13)


def test_merged_first_projection_equals_separate():
    W = _weights(SMALL, 6)
    x = np.random.default_rng(6).standard_normal((4, SMALL.hidden))
    merged = x @ np.concatenate([W["wq_a"], W["wkv_a"]], axis=1)
    np.testing.assert_allclose(merged[:, :SMALL.q_lora_rank], x @ W["wq_a"], atol=1e-13)
    np.testing.assert_allclose(merged[:, SMALL.q_lora_rank:], x @ W["wkv_a"], atol=1e-13)


def test_kv_b_split_checkpoint_form():
    """kv_b_split: attn_k_b holds per head kv_lora_rank rows of qk_nope, attn_v_b per
    head v_dim rows of kv_lora_rank, versus one attn_kv_b of qk_nope + v_dim rows a
    head ("struct Mla", field kv_b_split). Built here from a per-head [out, in]
    attn_kv_b by index; the oracle's W_UK / W_UV must be those halves."""
    H, dn, dv, rkv = 3, 4, 5, 7
    rng = np.random.default_rng(0)
    attn_kv_b = rng.standard_normal((H, dn + dv, rkv))          # rows a head, each kv_lora wide
    attn_k_b = np.zeros((H, rkv, dn))
    attn_v_b = np.zeros((H, dv, rkv))
    for h in range(H):
        for c in range(rkv):
            for p in range(dn):
                attn_k_b[h, c, p] = attn_kv_b[h, p, c]
        for d in range(dv):
            for c in range(rkv):
                attn_v_b[h, d, c] = attn_kv_b[h, dn + d, c]
    # wkv_b in [in, out] = [kv_lora, H*(dn+dv)] form: column h*(dn+dv)+i is row i of head h
    wkv_b = np.zeros((rkv, H * (dn + dv)))
    for h in range(H):
        for i in range(dn + dv):
            wkv_b[:, h * (dn + dv) + i] = attn_kv_b[h, i, :]
    w_uk, w_uv = ref.split_wkv_b(wkv_b, H, dn, dv)
    assert w_uk.shape == (H, dn, rkv) and w_uv.shape == (H, rkv, dv)
    np.testing.assert_array_equal(w_uk, attn_k_b.transpose(0, 2, 1))
    np.testing.assert_array_equal(w_uv, attn_v_b.transpose(0, 2, 1))


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def test_rope_position_zero_is_identity():
    v = np.random.default_rng(1).standard_normal((3, 16))
    cos, sin = ref.rope_cos_sin(np.zeros(3), 16, 10000.0)
    np.testing.assert_array_equal(ref.rope_interleaved(v, cos, sin), v)


def test_rope_hand_case():
    cos, sin = np.array([[math.cos(1.0)]]), np.array([[math.sin(1.0)]])
    out = ref.rope_interleaved(np.array([[1.0, 0.0]]), cos, sin)
    np.testing.assert_allclose(out, [[math.cos(1.0), math.sin(1.0)]], atol=1e-16)
    # position 1 with d_r = 2 has inv_freq theta^0 = 1, so phi = 1
    c1, s1 = ref.rope_cos_sin(np.array([1]), 2, 10000.0)
    np.testing.assert_allclose(ref.rope_interleaved(np.array([[1.0, 0.0]]), c1, s1),
                               [[math.cos(1.0), math.sin(1.0)]], atol=1e-16)


def test_rope_inv_freq_closed_form():
    f = ref.rope_inv_freq(8, 10000.0)
    np.testing.assert_allclose(f, [1.0, 10000 ** -0.25, 10000 ** -0.5, 10000 ** -0.75], rtol=1e-15)


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((5, 64))
    cos, sin = ref.rope_cos_sin(rng.integers(0, 20000, 5), 64, 10000.0)
    r = ref.rope_interleaved(v, cos, sin)
    np.testing.assert_allclose(r[:, 0::2] ** 2 + r[:, 1::2] ** 2,
                               v[:, 0::2] ** 2 + v[:, 1::2] ** 2, rtol=1e-12)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(64), rng.standard_normal(64)

    def score(m, n):
        cq, sq = ref.rope_cos_sin(np.array([m]), 64, 10000.0)
        ck, sk = ref.rope_cos_sin(np.array([n]), 64, 10000.0)
        return float(ref.rope_interleaved(q, cq[0], sq[0]) @ ref.rope_interleaved(k, ck[0], sk[0]))

    assert abs(score(10, 3) - score(1010, 1003)) < 1e-10
    assert abs(score(10, 3) - score(10, 4)) > 1e-6


def test_rope_is_interleaved_not_half_split():
    """Interleaved pairs (2i, 2i+1), not (i, i + d/2) ("MLA Decode QKV Kernel API
    Reference", Notes)."""
    v = np.arange(1.0, 9.0)
    cos, sin = ref.rope_cos_sin(np.array([3]), 8, 10000.0)
    inter = ref.rope_interleaved(v, cos[0], sin[0])
    a, b = v[:4], v[4:]
    half = np.concatenate([a * cos[0] - b * sin[0], a * sin[0] + b * cos[0]])
    assert np.max(np.abs(inter - half)) > 1e-3
    # complex-multiplication form of the same rotation (freqs_cis)
    z = (v[0::2] + 1j * v[1::2]) * np.exp(1j * 3 * ref.rope_inv_freq(8, 10000.0))
    np.testing.assert_allclose(inter[0::2], z.real, atol=1e-13)
    np.testing.assert_allclose(inter[1::2], z.imag, atol=1e-13)


# ---------------------------------------------------------------------------
# RMSNorm / softmax / scale
# ---------------------------------------------------------------------------

def test_rms_norm_constant_vector_closed_form():
    c, eps = 3.0, 1e-6
    g = np.linspace(0.9, 1.1, 16)
    out = ref.rms_norm(np.full(16, c), g, eps)
    np.testing.assert_allclose(out, g * c / math.sqrt(c * c + eps), rtol=1e-15)


def test_rms_norm_eps_matters_at_small_scale():
    v = np.full(4, 1e-3)
    out = ref.rms_norm(v, np.ones(4), 1e-6)
    np.testing.assert_allclose(out, 1e-3 / math.sqrt(1e-6 + 1e-6), rtol=1e-14)


def test_softmax_scale_reading():
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        g = json.load(f)
    v3 = g["deepseek_v3_dims"]
    assert ref.softmax_scale(v3["qk_nope_head_dim"], v3["qk_rope_head_dim"]) == pytest.approx(
        v3["qk_head_dim"] ** -0.5, rel=1e-15)
    assert v3["qk_nope_head_dim"] + v3["qk_rope_head_dim"] == v3["qk_head_dim"]


def test_context_of_one_returns_value_of_that_row():
    shape = SMALL
    W, inp, cos, sin = _decode_case(shape, 12, batch=2, ctx=(1, 1))
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    out, head_out = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    _, w_uv = ref.split_wkv_b(W["wkv_b"], shape.n_heads, shape.qk_nope, shape.v_dim)
    c, _ = ref.kv_projection(shape, W, inp.hidden, cos, sin)
    for t in range(2):
        np.testing.assert_allclose(head_out[t], np.einsum("c,hcd->hd", c[t], w_uv), atol=1e-13)


def test_identical_rows_give_row_value():
    shape = SMALL
    W, inp, cos, sin = _decode_case(shape, 13, batch=2, ctx=(4, 7))
    cache = np.array(inp.cache, np.float64)
    row = np.random.default_rng(0).standard_normal(shape.kv_row_dim)
    cache.reshape(-1, shape.kv_row_dim)[:] = row
    q_abs = np.random.default_rng(1).standard_normal((2, shape.n_heads, shape.kv_lora_rank))
    q_pe = np.random.default_rng(2).standard_normal((2, shape.n_heads, shape.qk_rope))
    _, head_out = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    _, w_uv = ref.split_wkv_b(W["wkv_b"], shape.n_heads, shape.qk_nope, shape.v_dim)
    want = np.einsum("c,hcd->hd", row[:shape.kv_lora_rank], w_uv)
    np.testing.assert_allclose(head_out, np.broadcast_to(want, head_out.shape), atol=1e-13)


# ---------------------------------------------------------------------------
# against torch's fp64 scaled_dot_product_attention (a textbook routine)
# ---------------------------------------------------------------------------

def test_expanded_decode_equals_torch_sdpa_default_scale():
    """SDPA's default scale is 1/sqrt(q.shape[-1]) = 1/sqrt(d_n + d_r): this pins the
    scale reading as well as the attention arithmetic."""
    shape = dataclasses.replace(SMALL, n_heads=3, kv_lora_rank=16, qk_nope=8, qk_rope=6, v_dim=5,
                                block_size=4)
    W, inp, cos, sin = _decode_case(shape, 14, batch=3, ctx=(2, 13))
    q_nope, q_pe = ref.decode_q(shape, W, inp.hidden, cos, sin)
    w_uk, w_uv = ref.split_wkv_b(W["wkv_b"], shape.n_heads, shape.qk_nope, shape.v_dim)
    _, head_out = ref.decode_attn(shape, W, ref.absorb(q_nope, w_uk), q_pe, inp.cache,
                                  inp.block_table, inp.context_lens)
    for t in range(3):
        rows = ref.gather_context(inp.cache, inp.block_table[t], int(inp.context_lens[t]),
                                  shape.block_size)
        c, kpe = rows[:, :shape.kv_lora_rank], rows[:, shape.kv_lora_rank:]
        K = torch.cat([torch.einsum("hpc,jc->hjp", torch.from_numpy(w_uk), torch.from_numpy(c)),
                       torch.from_numpy(kpe)[None].expand(shape.n_heads, -1, -1)], dim=-1)
        V = torch.einsum("jc,hcd->hjd", torch.from_numpy(c), torch.from_numpy(w_uv))
        Q = torch.cat([torch.from_numpy(q_nope[t]), torch.from_numpy(q_pe[t])], dim=-1)[:, None, :]
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V)[:, 0, :]
        np.testing.assert_allclose(head_out[t], o.numpy(), rtol=1e-10, atol=1e-12)


def test_prefill_equals_torch_sdpa_causal():
    shape = dataclasses.replace(SMALL, n_heads=3, kv_lora_rank=16, qk_nope=8, qk_rope=6, v_dim=5)
    W = _weights(shape, 15)
    S = 11
    x = np.random.default_rng(15).standard_normal((S, shape.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(S), shape.qk_rope, shape.rope_theta)
    _, head_out, rows = ref.prefill(shape, W, x, cos, sin)
    q_nope, q_pe = ref.decode_q(shape, W, x, cos, sin)
    c, kpe = rows[:, :shape.kv_lora_rank], rows[:, shape.kv_lora_rank:]
    kvo = (c @ W["wkv_b"]).reshape(S, shape.n_heads, shape.qk_nope + shape.v_dim)
    K = torch.cat([torch.from_numpy(kvo[..., :shape.qk_nope]),
                   torch.from_numpy(kpe)[:, None, :].expand(-1, shape.n_heads, -1)], -1)
    V = torch.from_numpy(kvo[..., shape.qk_nope:])
    Q = torch.cat([torch.from_numpy(q_nope), torch.from_numpy(q_pe)], -1)
    o = torch.nn.functional.scaled_dot_product_attention(
        Q.transpose(0, 1), K.transpose(0, 1), V.transpose(0, 1), is_causal=True).transpose(0, 1)
    np.testing.assert_allclose(head_out, o.numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------
# paged cache invariances
# ---------------------------------------------------------------------------

def test_block_permutation_and_layout_invariance():
    shape = dataclasses.replace(SMALL, block_size=3)
    W, inp, cos, sin = _decode_case(shape, 16, batch=3, ctx=(2, 14))
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    base, _ = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    # move every physical block to a new place and rewrite the tables accordingly
    nb = cache.shape[0]
    perm = np.random.default_rng(0).permutation(nb)
    moved = np.empty_like(cache)
    moved[perm] = cache
    table = np.where(inp.block_table >= 0, perm[np.maximum(inp.block_table, 0)], -1)
    out_p, _ = ref.decode_attn(shape, W, q_abs, q_pe, moved, table, inp.context_lens)
    np.testing.assert_allclose(out_p, base, atol=1e-14)
    # the inverted row layout with the same contents
    flipped = ref.cache_row(*ref.split_row(cache, shape.kv_lora_rank, ref.LATENT_FIRST),
                            ref.PE_FIRST)
    out_f, _ = ref.decode_attn(shape, W, q_abs, q_pe, flipped, inp.block_table, inp.context_lens,
                               ref.PE_FIRST)
    np.testing.assert_allclose(out_f, base, atol=1e-14)
    assert not np.allclose(flipped, cache)


def test_scatter_writes_only_mapped_rows():
    cache = np.arange(6 * 1 * 2 * 3, dtype=np.float64).reshape(6, 1, 2, 3)
    rows = np.array([[-1.0, -2, -3], [-4, -5, -6], [-7, -8, -9]])
    new = ref.scatter_rows(cache, np.array([5, -1, 0], np.int32), rows)
    flat_old, flat_new = cache.reshape(-1, 3), new.reshape(-1, 3)
    np.testing.assert_array_equal(flat_new[5], rows[0])
    np.testing.assert_array_equal(flat_new[0], rows[2])
    untouched = [i for i in range(12) if i not in (0, 5)]
    np.testing.assert_array_equal(flat_new[untouched], flat_old[untouched])


@pytest.mark.parametrize("shape", [SMALL, SMALL_NOQ])
@pytest.mark.parametrize("layout", [ref.LATENT_FIRST, ref.PE_FIRST])
def test_fill_cache_by_projection_matches_brute_force(shape, layout):
    """The earlier rows of each sequence (positions 0..L-2, the hidden state of
    position p projected, normed, rotated at p and written at its slot) against
    the literal loops, which take one token per position through the same
    front-fold and scatter; every other row keeps its value."""
    w = wl.Workload("t", shape, "decode", batch=3, ctx_lo=2, ctx_hi=7, cache_fill="project", seed=11)
    inp = wl.make_decode_inputs(w)
    W = _weights(shape, 11)
    got = ref.fill_cache_by_projection(shape, W, inp.cache, inp.fill_hidden, inp.fill_slots, layout)
    rows = inp.cache.reshape(-1, shape.kv_row_dim).tolist()
    shifted = [list(r) for r in rows]
    for xs, slots in zip(inp.fill_hidden, inp.fill_slots):
        m = len(slots)
        if m == 0:
            continue
        for pos0, dst in ((0, rows), (1, shifted)):   # pos0 = 1: the off-by-one reading
            _, _, _, _, new = brute.decode_step(shape, W, xs, np.arange(pos0, pos0 + m), dst,
                                                [[0]] * m, [1] * m, slots, layout)
            dst[:] = new
    got_flat = got.reshape(-1, shape.kv_row_dim)
    np.testing.assert_allclose(got_flat, np.array(rows), rtol=0, atol=1e-12)
    written = {int(s) for sl in inp.fill_slots for s in sl}
    assert written and len(written) == sum(len(s) for s in inp.fill_slots)
    old = inp.cache.reshape(-1, shape.kv_row_dim)
    for i in range(len(old)):
        if i not in written:
            np.testing.assert_array_equal(got_flat[i], old[i])
    # positions shifted by one would move every rotated k_pe: the pin sees it
    assert np.max(np.abs(got_flat - np.array(shifted))) > 1e-3


def test_cache_row_layouts():
    c, kpe = np.array([1.0, 2, 3]), np.array([8.0, 9])
    np.testing.assert_array_equal(ref.cache_row(c, kpe, ref.LATENT_FIRST), [1, 2, 3, 8, 9])
    np.testing.assert_array_equal(ref.cache_row(c, kpe, ref.PE_FIRST), [8, 9, 1, 2, 3])
    for lay in (ref.LATENT_FIRST, ref.PE_FIRST):
        c2, k2 = ref.split_row(ref.cache_row(c, kpe, lay), 3, lay)
        np.testing.assert_array_equal(c2, c)
        np.testing.assert_array_equal(k2, kpe)


# ---------------------------------------------------------------------------
# FP8-E4M3
# ---------------------------------------------------------------------------

def test_e4m3_decoder_all_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = ref.e4m3_to_float(codes)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(theirs)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    np.testing.assert_array_equal(mine[~nan], theirs[~nan])


def test_e4m3_special_values():
    with open(os.path.join(GOLDEN, "e4m3_values.json")) as f:
        g = json.load(f)
    for code_hex, value in g["values"].items():
        assert ref.e4m3_to_float(np.array([int(code_hex, 16)]))[0] == value, code_hex


def test_dequant_with_unit_scales_gives_exact_integer_gemm():
    rng = np.random.default_rng(0)
    vals = rng.integers(-8, 9, size=(200, 130))
    codes = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    W = ref.dequant_block128(codes, np.ones((2, 2)))
    np.testing.assert_array_equal(W, vals)
    x = rng.integers(-5, 6, size=(3, 200))
    np.testing.assert_array_equal(x @ W, x @ vals)


def test_dequant_block_scale_indexing():
    codes = np.full((130, 260), 0x38, np.uint8)     # 0x38 = 1.0
    scales = np.arange(1, 7, dtype=np.float64).reshape(2, 3)
    W = ref.dequant_block128(codes, scales)
    assert W[0, 0] == 1 and W[127, 127] == 1 and W[128, 0] == 4 and W[0, 128] == 2
    assert W[129, 259] == 6 and W[0, 256] == 3


# ---------------------------------------------------------------------------
# planted mistakes must be caught by the pins above
# ---------------------------------------------------------------------------

def _brute_decode_mismatch(shape, monkeypatch_target=None):
    W, inp, cos, sin = _decode_case(shape, 7)
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    out, _ = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    b_out = brute.decode_step(shape, W, inp.hidden, inp.positions,
                              inp.cache.reshape(-1, shape.kv_row_dim).tolist(),
                              inp.block_table.tolist(), inp.context_lens, inp.slot_mapping)[0]
    return np.max(np.abs(out - np.array(b_out)))


def test_planted_half_split_rope_is_caught(monkeypatch):
    def half_split(v, cos, sin):
        v = np.asarray(v, np.float64)
        d = v.shape[-1] // 2
        a, b = v[..., :d], v[..., d:]
        return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)
    assert _brute_decode_mismatch(SMALL) < 1e-12
    monkeypatch.setattr(ref, "rope_interleaved", half_split)
    assert _brute_decode_mismatch(SMALL) > 1e-6


def test_planted_wrong_scale_is_caught(monkeypatch):
    monkeypatch.setattr(ref, "softmax_scale", lambda dn, dr, mscale=1.0: (512 + dr) ** -0.5)
    assert _brute_decode_mismatch(SMALL) > 1e-6


def test_planted_wkv_b_grouping_is_caught(monkeypatch):
    def grouped_wrong(wkv_b, H, dn, dv):       # all heads' k_nope first, then all v
        w = np.asarray(wkv_b, np.float64)
        r = w.shape[0]
        k = w[:, :H * dn].reshape(r, H, dn).transpose(1, 2, 0)
        v = w[:, H * dn:].reshape(r, H, dv).transpose(1, 0, 2)
        return k, v
    monkeypatch.setattr(ref, "split_wkv_b", grouped_wrong)
    assert _brute_decode_mismatch(SMALL) > 1e-6


def test_planted_input_norm_without_gamma_is_caught(monkeypatch):
    W, inp, cos, sin = _decode_case(SMALL, 13)
    g_in = 1.0 + np.random.default_rng(13).uniform(-0.3, 0.3, SMALL.hidden)
    flat = inp.cache.reshape(-1, SMALL.kv_row_dim).tolist()

    def mismatch():
        _, q_pe, cache = ref.decode_qkv(SMALL, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping,
                                        input_norm_w=g_in)
        b = brute.decode_step(SMALL, W, inp.hidden, inp.positions, flat, inp.block_table.tolist(),
                              inp.context_lens, inp.slot_mapping, input_norm_w=g_in)
        return max(np.max(np.abs(q_pe - np.array(b[3]))),
                   np.max(np.abs(cache.reshape(-1, SMALL.kv_row_dim) - np.array(b[4]))))
    assert mismatch() < 1e-12
    monkeypatch.setattr(ref, "input_norm", lambda cfg, x, g: ref.rms_norm(x, np.ones_like(g), cfg.norm_eps))
    assert mismatch() > 1e-6


def test_planted_normed_k_pe_is_caught(monkeypatch):
    orig = ref.kv_projection

    def normed_all(cfg, W, hidden, cos, sin):
        c, k_pe = orig(cfg, W, hidden, cos, sin)
        return c, ref.rms_norm(k_pe, np.ones(k_pe.shape[-1]), cfg.norm_eps)
    monkeypatch.setattr(ref, "kv_projection", normed_all)
    assert _brute_decode_mismatch(SMALL) > 1e-6
