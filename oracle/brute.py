"""Literal-loop MLA for tiny shapes.  TEST INFRASTRUCTURE ONLY.

Pure Python (lists and the math module, no numpy arithmetic) so that it shares
no vectorised code with oracle/mla_ref.py; tests use it to pin the oracle on
shapes of a few elements. Same readings as mla_ref (see its docstrings):
eps inside the root, interleaved pairs (2i, 2i+1), scale 1/sqrt(d_n + d_r),
per-head [k_nope | v] columns of wkv_b, cache row [latent | k_pe] or
[k_pe | latent].
"""
from __future__ import annotations

import math


def _mat(a):
    return [[float(v) for v in row] for row in a]


def _vecmat(v, m):
    """v [K] times m [K][N] -> [N]."""
    K, N = len(m), len(m[0])
    return [sum(v[k] * m[k][j] for k in range(K)) for j in range(N)]


def _rms(v, g, eps):
    ms = sum(x * x for x in v) / len(v)
    r = 1.0 / math.sqrt(ms + eps)
    return [v[i] * r * g[i] for i in range(len(v))]


def _rope(v, pos, theta, inv_freq=None):
    d = len(v)
    out = list(v)
    for i in range(d // 2):
        f = theta ** (-2.0 * i / d) if inv_freq is None else float(inv_freq[i])
        phi = pos * f
        a, b = v[2 * i], v[2 * i + 1]
        out[2 * i] = a * math.cos(phi) - b * math.sin(phi)
        out[2 * i + 1] = a * math.sin(phi) + b * math.cos(phi)
    return out


def _softmax_row(s, sink=None):
    """exp(s_j - m) / (sum_k exp(s_k - m) [+ exp(sink - m)]), m the largest of
    the row and the sink."""
    mx = max(s) if sink is None else max(max(s), sink)
    e = [math.exp(v - mx) for v in s]
    z = sum(e) + (0.0 if sink is None else math.exp(sink - mx))
    return [v / z for v in e]


def _o_proj(cfg, W, head_out_t):
    """One token's output projection from its head outputs [H][d_v]: wo, or the
    grouped low-rank wo_a (per group of consecutive heads, its own block of
    rows) then wo_b."""
    flat = [v for h in head_out_t for v in h]
    if not getattr(cfg, "o_lora_rank", 0):
        return _vecmat(flat, _mat(W["wo"]))
    G, ro = cfg.o_groups, cfg.o_lora_rank
    kg = len(flat) // G
    wo_a = _mat(W["wo_a"])
    z = []
    for g in range(G):
        for j in range(ro):
            z.append(sum(flat[g * kg + i] * wo_a[g * kg + i][j] for i in range(kg)))
    return _vecmat(z, _mat(W["wo_b"]))


def decode_step(cfg, W, hidden, positions, cache_rows, block_table, context_lens,
                slot_mapping, layout=0, input_norm_w=None, inv_freq=None, attn_sink=None):
    """One whole decode step, loops only.

    input_norm_w: optional input RMSNorm gamma [hidden] applied to each token
    first (eps = norm_eps); inv_freq: optional RoPE frequency table [d_r/2]
    replacing theta^(-2i/d_r); attn_sink: optional per-head logit that joins
    each head's softmax denominator and carries no value.
    cache_rows: list of flat cache rows (lists of R floats), mutated copy returned.
    Returns (out [n][hidden], head_out [n][H][d_v], q_abs [n][H][r_kv],
    q_pe [n][H][d_r], new cache_rows).
    """
    H, dn, dr, dv = cfg.n_heads, cfg.qk_nope, cfg.qk_rope, cfg.v_dim
    rkv, bs = cfg.kv_lora_rank, cfg.block_size
    wkv_b = _mat(W["wkv_b"])
    rows = [list(r) for r in cache_rows]
    q_abs_all, q_pe_all = [], []
    for t, x in enumerate(hidden):
        x = [float(v) for v in x]
        if input_norm_w is not None:
            x = _rms(x, [float(g) for g in input_norm_w], cfg.norm_eps)
        pos = int(positions[t])
        if cfg.q_lora_rank:
            ql = _rms(_vecmat(x, _mat(W["wq_a"])), [float(g) for g in W["q_norm_w"]], cfg.norm_eps)
            q = _vecmat(ql, _mat(W["wq_b"]))
        else:
            q = _vecmat(x, _mat(W["wq_b"]))
        kv = _vecmat(x, _mat(W["wkv_a"]))
        c = _rms(kv[:rkv], [float(g) for g in W["kv_norm_w"]], cfg.norm_eps)
        kpe = _rope(kv[rkv:], pos, cfg.rope_theta, inv_freq)
        q_abs_t, q_pe_t = [], []
        for h in range(H):
            qh = q[h * (dn + dr):(h + 1) * (dn + dr)]
            qn, qp = qh[:dn], _rope(qh[dn:], pos, cfg.rope_theta, inv_freq)
            # absorption through the nope columns of head h of wkv_b
            qa = [sum(qn[p] * wkv_b[cc][h * (dn + dv) + p] for p in range(dn)) for cc in range(rkv)]
            q_abs_t.append(qa)
            q_pe_t.append(qp)
        q_abs_all.append(q_abs_t)
        q_pe_all.append(q_pe_t)
        slot = int(slot_mapping[t])
        if slot >= 0:
            rows[slot] = (c + kpe) if layout == 0 else (kpe + c)
    scale = 1.0 / math.sqrt(dn + dr)
    head_out = []
    for t in range(len(hidden)):
        L = int(context_lens[t])
        ctx = []
        for j in range(L):
            r = rows[int(block_table[t][j // bs]) * bs + j % bs]
            ctx.append((r[:rkv], r[rkv:]) if layout == 0 else (r[dr:], r[:dr]))
        o_t = []
        for h in range(H):
            s = [(sum(q_abs_all[t][h][cc] * ctx[j][0][cc] for cc in range(rkv))
                  + sum(q_pe_all[t][h][i] * ctx[j][1][i] for i in range(dr))) * scale
                 for j in range(L)]
            p = _softmax_row(s, None if attn_sink is None else float(attn_sink[h]))
            o_lat = [sum(p[j] * ctx[j][0][cc] for j in range(L)) for cc in range(rkv)]
            o_t.append([sum(o_lat[cc] * wkv_b[cc][h * (dn + dv) + dn + d] for cc in range(rkv))
                        for d in range(dv)])
        head_out.append(o_t)
    out = [_o_proj(cfg, W, head_out[t]) for t in range(len(hidden))]
    return out, head_out, q_abs_all, q_pe_all, rows


def prefill(cfg, W, hidden, attn_sink=None):
    """Causal expanded prefill of one sequence at positions 0..S-1, loops only
    (attn_sink as in decode_step). Returns (out [S][hidden], head_out [S][H][d_v])."""
    H, dn, dr, dv = cfg.n_heads, cfg.qk_nope, cfg.qk_rope, cfg.v_dim
    rkv = cfg.kv_lora_rank
    S = len(hidden)
    wkv_b = _mat(W["wkv_b"])
    Q, K, V = [], [], []
    for i, x in enumerate(hidden):
        x = [float(v) for v in x]
        if cfg.q_lora_rank:
            ql = _rms(_vecmat(x, _mat(W["wq_a"])), [float(g) for g in W["q_norm_w"]], cfg.norm_eps)
            q = _vecmat(ql, _mat(W["wq_b"]))
        else:
            q = _vecmat(x, _mat(W["wq_b"]))
        kv = _vecmat(x, _mat(W["wkv_a"]))
        c = _rms(kv[:rkv], [float(g) for g in W["kv_norm_w"]], cfg.norm_eps)
        kpe = _rope(kv[rkv:], i, cfg.rope_theta)
        kvo = _vecmat(c, wkv_b)
        Qi, Ki, Vi = [], [], []
        for h in range(H):
            qh = q[h * (dn + dr):(h + 1) * (dn + dr)]
            Qi.append(qh[:dn] + _rope(qh[dn:], i, cfg.rope_theta))
            base = h * (dn + dv)
            Ki.append(kvo[base:base + dn] + kpe)
            Vi.append(kvo[base + dn:base + dn + dv])
        Q.append(Qi)
        K.append(Ki)
        V.append(Vi)
    scale = 1.0 / math.sqrt(dn + dr)
    head_out = []
    for i in range(S):
        o_i = []
        for h in range(H):
            s = [sum(Q[i][h][d] * K[j][h][d] for d in range(dn + dr)) * scale for j in range(i + 1)]
            p = _softmax_row(s, None if attn_sink is None else float(attn_sink[h]))
            o_i.append([sum(p[j] * V[j][h][d] for j in range(i + 1)) for d in range(dv)])
        head_out.append(o_i)
    out = [_o_proj(cfg, W, head_out[i]) for i in range(S)]
    return out, head_out


def v4_qkv(cfg, W, hidden, positions, kv_norm_w, inv_freq=None):
    """DeepSeek-V4 QKV projection, loops only (same reading as mla_ref.v4_qkv:
    per-head root-mean-square norm without gain, interleaved RoPE on the last
    d_r of each head and of the kv row, kv RMSNorm over all its columns).
    Returns (q [n][H][hd], kv [n][kv_dim])."""
    H, hd, dr = cfg.n_heads, cfg.qk_nope + cfg.qk_rope, cfg.qk_rope
    qs, kvs = [], []
    for t, x in enumerate(hidden):
        x = [float(v) for v in x]
        pos = int(positions[t])
        ql = _rms(_vecmat(x, _mat(W["wq_a"])), [float(g) for g in W["q_norm_w"]], cfg.norm_eps)
        q = _vecmat(ql, _mat(W["wq_b"]))
        q_t = []
        for h in range(H):
            qh = q[h * hd:(h + 1) * hd]
            qh = _rms(qh, [1.0] * hd, cfg.norm_eps)
            q_t.append(qh[:hd - dr] + _rope(qh[hd - dr:], pos, cfg.rope_theta, inv_freq))
        kv = _rms(_vecmat(x, _mat(W["wkv_a"])), [float(g) for g in kv_norm_w], cfg.norm_eps)
        R = len(kv)
        kvs.append(kv[:R - dr] + _rope(kv[R - dr:], pos, cfg.rope_theta, inv_freq))
        qs.append(q_t)
    return qs, kvs
