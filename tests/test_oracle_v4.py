"""Pins of the oracle's DeepSeek-V4 pieces: the attention sink logit and the V4
QKV projection, against brute-force loops (oracle/brute.py), closed forms and
torch's fp64 scaled_dot_product_attention. CPU only.
"""
import dataclasses

import numpy as np
import pytest
import torch

from head_latent_attention_decode_b200 import workloads as wl
from oracle import brute
from oracle import mla_ref as ref

SMALL = wl.MlaShape(hidden=24, n_heads=2, q_lora_rank=12, kv_lora_rank=8, qk_nope=4,
                    qk_rope=4, v_dim=6, block_size=2, act_dtype="f32", weight_dtype="f32")
SMALL_NOQ = dataclasses.replace(SMALL, q_lora_rank=0)


def _weights(shape, seed):
    return ref.weights_fp64(wl.make_weights(shape, seed))


def _decode_case(shape, seed, batch=3, ctx=(1, 5)):
    w = wl.Workload("t", shape, "decode", batch=batch, ctx_lo=ctx[0], ctx_hi=ctx[1],
                    cache_fill="random", seed=seed)
    inp = wl.make_decode_inputs(w)
    W = _weights(shape, seed)
    cos, sin = ref.rope_cos_sin(inp.positions, shape.qk_rope, shape.rope_theta)
    return W, inp, cos, sin


def _sink(shape, seed):
    return np.random.default_rng(seed).uniform(-2.0, 2.0, shape.n_heads)


# ---------------------------------------------------------------------------
# attention sink
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [SMALL, SMALL_NOQ])
def test_decode_with_sink_matches_brute_force(shape):
    W, inp, cos, sin = _decode_case(shape, 21)
    sink = _sink(shape, 21)
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    out, head_out = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens,
                                    attn_sink=sink)
    b_out, b_head = brute.decode_step(shape, W, inp.hidden, inp.positions,
                                      inp.cache.reshape(-1, shape.kv_row_dim).tolist(),
                                      inp.block_table.tolist(), inp.context_lens, inp.slot_mapping,
                                      attn_sink=sink)[:2]
    np.testing.assert_allclose(head_out, np.array(b_head), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape", [SMALL, SMALL_NOQ])
def test_prefill_with_sink_matches_brute_force(shape):
    W = _weights(shape, 22)
    sink = _sink(shape, 22)
    x = np.random.default_rng(22).standard_normal((5, shape.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(5), shape.qk_rope, shape.rope_theta)
    out, head_out, _ = ref.prefill(shape, W, x, cos, sin, attn_sink=sink)
    b_out, b_head = brute.prefill(shape, W, x, attn_sink=sink)
    np.testing.assert_allclose(head_out, np.array(b_head), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


def test_sink_equal_to_the_rows_log_mass_halves_the_output():
    """Every row identical, so every score is the same s0; a sink of s0 + ln L
    weighs as much as all L rows together, so each head keeps exactly half of
    the sink-free output (closed form; pins the sink's units and that it only
    enters the denominator)."""
    shape = SMALL
    W, inp, cos, sin = _decode_case(shape, 23, batch=2, ctx=(3, 6))
    cache = np.array(inp.cache, np.float64)
    row = np.random.default_rng(0).standard_normal(shape.kv_row_dim)
    cache.reshape(-1, shape.kv_row_dim)[:] = row
    q_abs = np.random.default_rng(1).standard_normal((2, shape.n_heads, shape.kv_lora_rank))
    q_pe = np.random.default_rng(2).standard_normal((2, shape.n_heads, shape.qk_rope))
    _, plain = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    scale = ref.softmax_scale(shape.qk_nope, shape.qk_rope)
    for t in range(2):
        L = int(inp.context_lens[t])
        s0 = (q_abs[t] @ row[:shape.kv_lora_rank] + q_pe[t] @ row[shape.kv_lora_rank:]) * scale   # [H]
        _, with_sink = ref.decode_attn(shape, W, q_abs[t:t + 1], q_pe[t:t + 1], cache, inp.block_table[t:t + 1],
                                       inp.context_lens[t:t + 1], attn_sink=s0 + np.log(L))
        np.testing.assert_allclose(with_sink[0], 0.5 * plain[t], rtol=1e-12, atol=1e-14)


def test_very_negative_sink_is_no_sink():
    shape = SMALL
    W, inp, cos, sin = _decode_case(shape, 24)
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    a = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)[1]
    b = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens,
                        attn_sink=np.full(shape.n_heads, -1e4))[1]
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_sink_equals_torch_sdpa_with_a_zero_value_column():
    """torch's fp64 SDPA over the keys plus one extra key whose value is zero
    and whose score the additive mask sets to the sink: the same weights."""
    shape = dataclasses.replace(SMALL, n_heads=3, kv_lora_rank=16, qk_nope=8, qk_rope=6, v_dim=5)
    W = _weights(shape, 25)
    S = 9
    sink = _sink(shape, 25)
    x = np.random.default_rng(25).standard_normal((S, shape.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(S), shape.qk_rope, shape.rope_theta)
    _, head_out, rows = ref.prefill(shape, W, x, cos, sin, attn_sink=sink)
    q_nope, q_pe = ref.decode_q(shape, W, x, cos, sin)
    c, kpe = rows[:, :shape.kv_lora_rank], rows[:, shape.kv_lora_rank:]
    kvo = (c @ W["wkv_b"]).reshape(S, shape.n_heads, shape.qk_nope + shape.v_dim)
    H, dq = shape.n_heads, shape.qk_nope + shape.qk_rope
    K = torch.cat([torch.from_numpy(kvo[..., :shape.qk_nope]),
                   torch.from_numpy(kpe)[:, None, :].expand(-1, H, -1)], -1).transpose(0, 1)   # [H, S, dq]
    V = torch.from_numpy(kvo[..., shape.qk_nope:]).transpose(0, 1)                          # [H, S, dv]
    Q = torch.cat([torch.from_numpy(q_nope), torch.from_numpy(q_pe)], -1).transpose(0, 1)   # [H, S, dq]
    K = torch.cat([K, torch.zeros(H, 1, dq, dtype=torch.float64)], 1)
    V = torch.cat([V, torch.zeros(H, 1, shape.v_dim, dtype=torch.float64)], 1)
    mask = torch.full((H, S, S + 1), float("-inf"), dtype=torch.float64)
    causal = torch.tril(torch.ones(S, S, dtype=torch.bool))
    mask[:, :, :S][:, causal] = 0.0
    mask[:, :, S] = torch.from_numpy(sink)[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask).transpose(0, 1)
    np.testing.assert_allclose(head_out, o.numpy(), rtol=1e-10, atol=1e-12)


def test_planted_sink_in_the_numerator_is_caught(monkeypatch):
    shape = SMALL
    W = _weights(shape, 26)
    sink = _sink(shape, 26)
    x = np.random.default_rng(26).standard_normal((4, shape.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(4), shape.qk_rope, shape.rope_theta)
    b_head = np.array(brute.prefill(shape, W, x, attn_sink=sink)[1])

    def mismatch():
        return np.max(np.abs(ref.prefill(shape, W, x, cos, sin, attn_sink=sink)[1] - b_head))
    assert mismatch() < 1e-12
    # a sink that is renormalised away (weights summing to one again) is not the reading
    monkeypatch.setattr(ref, "softmax_with_sink", lambda s, sink: ref.softmax(s, axis=-1))
    assert mismatch() > 1e-6


# ---------------------------------------------------------------------------
# V4 QKV projection
# ---------------------------------------------------------------------------

V4 = wl.MlaShape(hidden=24, n_heads=3, q_lora_rank=12, kv_lora_rank=8, qk_nope=6,
                 qk_rope=4, v_dim=6, block_size=2, act_dtype="f32", weight_dtype="f32")


def _v4_case(shape, seed, n=4, positions=None):
    W = _weights(shape, seed)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, shape.hidden))
    g = 1.0 + rng.uniform(-0.3, 0.3, shape.kv_row_dim)
    pos = np.arange(3, 3 + n) if positions is None else np.asarray(positions)
    cos, sin = ref.rope_cos_sin(pos, shape.qk_rope, shape.rope_theta)
    return W, x, g, pos, cos, sin


def test_v4_qkv_matches_brute_force():
    W, x, g, pos, cos, sin = _v4_case(V4, 31)
    q, kv = ref.v4_qkv(V4, W, x, cos, sin, g)
    bq, bkv = brute.v4_qkv(V4, W, x, pos, g)
    np.testing.assert_allclose(q, np.array(bq), rtol=0, atol=1e-12)
    np.testing.assert_allclose(kv, np.array(bkv), rtol=0, atol=1e-12)


def test_v4_q_heads_mean_square_closed_form():
    """RoPE preserves pair norms, so each output head keeps the mean square the
    gain-free norm gives it: ms / (ms + eps), ms that of the stage-2 head."""
    W, x, g, pos, cos, sin = _v4_case(V4, 32)
    q, _ = ref.v4_qkv(V4, W, x, cos, sin, g)
    hd = V4.qk_nope + V4.qk_rope
    raw = (ref.rms_norm(x @ W["wq_a"], W["q_norm_w"], V4.norm_eps) @ W["wq_b"]).reshape(4, V4.n_heads, hd)
    ms_raw = np.mean(raw * raw, axis=-1)
    np.testing.assert_allclose(np.mean(q * q, axis=-1), ms_raw / (ms_raw + V4.norm_eps), rtol=1e-12)


def test_v4_kv_at_position_zero_is_its_rmsnorm_over_all_columns():
    """At position 0 RoPE is the identity, so kv / gamma has mean square
    ms / (ms + eps) over all kv_dim columns (the norm spans the rope tail too)."""
    W, x, g, pos, cos, sin = _v4_case(V4, 33, positions=[0, 0, 0, 0])
    _, kv = ref.v4_qkv(V4, W, x, cos, sin, g)
    u = kv / g
    raw = x @ W["wkv_a"]
    ms_raw = np.mean(raw * raw, axis=-1)
    np.testing.assert_allclose(np.mean(u * u, axis=-1), ms_raw / (ms_raw + V4.norm_eps), rtol=1e-12)
    # and the rotated tail at a later position has the same pair norms
    _, kv5 = ref.v4_qkv(V4, W, x, *ref.rope_cos_sin(np.full(4, 5), V4.qk_rope, V4.rope_theta), g)
    d = V4.kv_row_dim - V4.qk_rope
    np.testing.assert_allclose(kv5[:, :d], kv[:, :d], atol=1e-14)
    pn = lambda a: a[:, d::2] ** 2 + a[:, d + 1::2] ** 2
    np.testing.assert_allclose(pn(kv5), pn(kv), rtol=1e-12)


def test_v4_q_nope_part_is_the_normed_projection():
    """The first head_dim - d_r entries of each head are not rotated: they are
    the gain-free RMS norm of the head (closed form from the stage-2 product)."""
    W, x, g, pos, cos, sin = _v4_case(V4, 34)
    q, _ = ref.v4_qkv(V4, W, x, cos, sin, g)
    hd = V4.qk_nope + V4.qk_rope
    raw = (ref.rms_norm(x @ W["wq_a"], W["q_norm_w"], V4.norm_eps) @ W["wq_b"]).reshape(4, V4.n_heads, hd)
    want = raw / np.sqrt(np.mean(raw * raw, axis=-1, keepdims=True) + V4.norm_eps)
    np.testing.assert_allclose(q[..., :V4.qk_nope], want[..., :V4.qk_nope], rtol=1e-12)


def test_planted_latent_only_kv_norm_is_caught(monkeypatch):
    W, x, g, pos, cos, sin = _v4_case(V4, 35)
    bq, bkv = brute.v4_qkv(V4, W, x, pos, g)

    def mismatch():
        _, kv = ref.v4_qkv(V4, W, x, cos, sin, g)
        return np.max(np.abs(kv - np.array(bkv)))
    assert mismatch() < 1e-12
    r = V4.kv_lora_rank
    orig = ref.rms_norm

    def latent_only(v, gamma, eps):
        v = np.asarray(v, np.float64)
        if v.shape[-1] != V4.kv_row_dim:
            return orig(v, gamma, eps)
        out = v.copy()
        out[..., :r] = orig(v[..., :r], np.asarray(gamma)[:r], eps)
        return out
    monkeypatch.setattr(ref, "rms_norm", latent_only)
    assert mismatch() > 1e-6


def test_planted_missing_head_norm_is_caught(monkeypatch):
    W, x, g, pos, cos, sin = _v4_case(V4, 36)
    bq, _ = brute.v4_qkv(V4, W, x, pos, g)

    def mismatch():
        q, _ = ref.v4_qkv(V4, W, x, cos, sin, g)
        return np.max(np.abs(q - np.array(bq)))
    assert mismatch() < 1e-12
    monkeypatch.setattr(ref, "head_rms", lambda q, eps: np.asarray(q, np.float64))
    assert mismatch() > 1e-6


# ---------------------------------------------------------------------------
# grouped low-rank output projection (wo_a -> wo_b)
# ---------------------------------------------------------------------------

GROUPED = dataclasses.replace(wl.MlaShape(hidden=24, n_heads=4, q_lora_rank=12, kv_lora_rank=8, qk_nope=4,
                                          qk_rope=4, v_dim=6, block_size=2, act_dtype="f32",
                                          weight_dtype="f32"), o_groups=2, o_lora_rank=3)


@pytest.mark.parametrize("shape", [GROUPED, dataclasses.replace(GROUPED, q_lora_rank=0, o_groups=4)])
def test_decode_with_grouped_o_matches_brute_force(shape):
    W, inp, cos, sin = _decode_case(shape, 31)
    assert "wo" not in W and W["wo_a"].shape == (shape.n_heads * shape.v_dim, shape.o_lora_rank)
    q_abs, q_pe, cache = ref.decode_qkv(shape, W, inp.hidden, cos, sin, inp.cache, inp.slot_mapping)
    out, head_out = ref.decode_attn(shape, W, q_abs, q_pe, cache, inp.block_table, inp.context_lens)
    b_out, b_head = brute.decode_step(shape, W, inp.hidden, inp.positions,
                                      inp.cache.reshape(-1, shape.kv_row_dim).tolist(),
                                      inp.block_table.tolist(), inp.context_lens, inp.slot_mapping)[:2]
    np.testing.assert_allclose(head_out, np.array(b_head), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


def test_prefill_with_grouped_o_matches_brute_force():
    shape = GROUPED
    W = _weights(shape, 32)
    x = np.random.default_rng(32).standard_normal((5, shape.hidden))
    cos, sin = ref.rope_cos_sin(np.arange(5), shape.qk_rope, shape.rope_theta)
    out, head_out, _ = ref.prefill(shape, W, x, cos, sin)
    b_out, b_head = brute.prefill(shape, W, x)
    np.testing.assert_allclose(head_out, np.array(b_head), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, np.array(b_out), rtol=0, atol=1e-12)


def test_grouped_o_equals_its_block_diagonal_matrix():
    """The grouped form is one block-diagonal [H d_v, G r_o] matrix (group g's
    block on rows g (H/G) d_v.., columns g r_o..) followed by wo_b."""
    rng = np.random.default_rng(33)
    n, H, dv, G, ro, D = 3, 8, 5, 4, 3, 7
    head = rng.standard_normal((n, H, dv))
    wo_a, wo_b = rng.standard_normal((H * dv, ro)), rng.standard_normal((G * ro, D))
    bd = np.zeros((H * dv, G * ro))
    kg = H * dv // G
    for g in range(G):
        bd[g * kg:(g + 1) * kg, g * ro:(g + 1) * ro] = wo_a[g * kg:(g + 1) * kg]
    want = head.reshape(n, -1) @ bd @ wo_b
    np.testing.assert_allclose(ref.grouped_o_projection(head, wo_a, wo_b, G), want, rtol=1e-13, atol=1e-13)


def test_one_group_is_the_low_rank_factorisation_of_wo():
    """With one group the projection is the dense wo = wo_a @ wo_b."""
    rng = np.random.default_rng(34)
    head = rng.standard_normal((4, 6, 5))
    wo_a, wo_b = rng.standard_normal((30, 2)), rng.standard_normal((2, 9))
    np.testing.assert_allclose(ref.grouped_o_projection(head, wo_a, wo_b, 1),
                               head.reshape(4, -1) @ (wo_a @ wo_b), rtol=1e-12, atol=1e-12)


def test_planted_strided_head_groups_are_caught(monkeypatch):
    """Groups of every G-th head instead of consecutive heads fail the pins."""
    def strided(head_out, wo_a, wo_b, o_groups):
        n, H, dv = head_out.shape
        hg = H // o_groups
        z = [np.asarray(head_out[:, g::o_groups, :], np.float64).reshape(n, hg * dv)
             @ np.asarray(wo_a, np.float64)[g * hg * dv:(g + 1) * hg * dv] for g in range(o_groups)]
        return np.concatenate(z, axis=1) @ np.asarray(wo_b, np.float64)
    monkeypatch.setattr(ref, "grouped_o_projection", strided)
    with pytest.raises(AssertionError):
        test_decode_with_grouped_o_matches_brute_force(GROUPED)
