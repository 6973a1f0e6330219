"""GPU parity, through the C-ABI, of the DeepSeek-V4 pieces against the fp64
oracle: the per-head attention sink logit in decode attention (every attention
kernel family: CUDA-core, few-head pair, head-major) and in prefill (CUDA-core
and tensor-core), and the V4 QKV projection (mla_v4_qkv) for fp32, bf16 and
FP8 block-scaled weights with ragged token counts. Tolerances as everywhere:
1e-4 * max|ref| for fp32, 2e-2 * max|ref| (per head for head outputs) for
bf16 / FP8."""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import workloads as wl
from head_latent_attention_decode_b200.layer import ACT_TORCH, MlaLayer
from oracle import mla_ref as ref

from gpu_common import (TOL, DecodeCase, assert_close, assert_close_per_head, ensure_built, max_rel_err,
                        to_dev, to_np)
from test_gpu_decode import check_case
from test_gpu_prefill import run_prefill

pytestmark = pytest.mark.gpu


def sink_for(shape, seed, mean_ctx):
    """Sink logits around the log of the row count, so that the sink holds a
    large share of every head's softmax mass."""
    return (np.log(max(mean_ctx, 1.0)) + np.random.default_rng(seed).uniform(-1.0, 1.0, shape.n_heads)).astype(np.float32)


def _sink_matters(case, r):
    """The sink-free oracle output is far outside the tolerance of the one with
    the sink, so the parity check below really tests the sink."""
    s = case.shape
    inp = case.inp
    q_abs, q_pe = r["q_abs"], r["q_pe"]
    from gpu_common import compact
    cache, table, slots, fill, blocks = compact(inp, r["seqs"], s)
    _, plain = ref.decode_attn(s, ref.weights_fp64(case.weights), q_abs, q_pe, r["cache"], table,
                               inp.context_lens[r["seqs"]], case.row_layout)
    assert max_rel_err(plain, r["head_out"]) > 5 * TOL[s.act_dtype]


@pytest.mark.parametrize("name,batch,ctx", [
    ("tiny_fp32", None, None),
    ("v2lite_bf16", 3, (300, 1100)),
    ("v3_bf16", 2, (100, 700)),
    ("v3_fp8", 2, (200, 500)),
])
def test_decode_with_attn_sink(name, batch, ctx):
    w = wl.WORKLOADS[name]
    mean = (ctx[0] + ctx[1]) / 2 if ctx else (w.ctx_lo + w.ctx_hi) / 2
    case = DecodeCase(w, batch=batch, ctx=ctx, attn_sink=sink_for(w.shape, 41, mean)).run()
    r = check_case(case)
    _sink_matters(case, r)


def test_decode_sink_on_a_context_of_one():
    """One row and a sink: the head keeps e^s / (e^s + e^z) of that row's value."""
    w = dataclasses.replace(wl.WORKLOADS["v2lite_bf16"], seed=43)
    case = DecodeCase(w, batch=4, ctx=(1, 1), attn_sink=sink_for(w.shape, 43, 1.0)).run()
    check_case(case)


@pytest.mark.parametrize("name,S", [("tiny", 77), ("v3", 300)])
def test_prefill_with_attn_sink(name, S):
    base = wl.WORKLOADS["v3_prefill_bf16"]
    w = dataclasses.replace(base, shape=wl.TINY, seed=44) if name == "tiny" else dataclasses.replace(base, seed=45)
    run_prefill(w, S, attn_sink=sink_for(w.shape, 46, S / 2))


# ---------------------------------------------------------------------------
# V4 QKV projection
# ---------------------------------------------------------------------------

def run_v4(shape, seed, S, positions=None):
    ensure_built()
    weights = wl.make_weights(shape, seed)
    rng = np.random.default_rng(seed)
    x = wl.round_to(rng.standard_normal((S, shape.hidden)), shape.act_dtype)
    g = (1.0 + rng.uniform(-0.3, 0.3, shape.kv_row_dim)).astype(np.float32)
    pos = (rng.integers(0, 30000, S) if positions is None else np.asarray(positions)).astype(np.int32)
    layer = MlaLayer(shape, weights)
    act = ACT_TORCH[shape.act_dtype]
    cos, sin = layer.rope(torch.from_numpy(pos).cuda())
    q, kv = layer.v4_qkv(to_dev(x, act), cos, sin, torch.from_numpy(g).cuda())
    torch.cuda.synchronize()
    assert mla.mla_read_device_flag(layer.ws) == 0
    rcos, rsin = ref.rope_cos_sin(pos, shape.qk_rope, shape.rope_theta)
    rq, rkv = ref.v4_qkv(shape, ref.weights_fp64(weights), x, rcos, rsin, g.astype(np.float64))
    tol = TOL[shape.act_dtype]
    assert_close_per_head(to_np(q), rq, tol, "q")
    assert_close(to_np(kv), rkv, tol, "kv")
    return layer


def test_v4_qkv_tiny_fp32():
    run_v4(wl.TINY, 51, S=9)


@pytest.mark.parametrize("S", [1, 129, 200])
def test_v4_qkv_v3_bf16(S):
    run_v4(wl.V3, 52, S=S)


@pytest.mark.parametrize("S", [3, 150])
def test_v4_qkv_v3_fp8_weights(S):
    run_v4(wl.WORKLOADS["v3_fp8"].shape, 53, S=S)


def test_v4_qkv_needs_a_low_rank_query():
    ensure_built()
    s = wl.V2LITE
    layer = MlaLayer(s, wl.make_weights(s, 54))
    x = torch.zeros((2, s.hidden), dtype=torch.bfloat16, device="cuda")
    cos, sin = layer.rope(torch.zeros(2, dtype=torch.int32, device="cuda"))
    g = torch.ones(s.kv_row_dim, dtype=torch.float32, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        layer.v4_qkv(x, cos, sin, g)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED


# ---------------------------------------------------------------------------
# grouped low-rank output projection (wo_a -> wo_b)
# ---------------------------------------------------------------------------

def grouped(name, o_groups, o_lora_rank):
    """The workload `name` with the grouped output projection in place of wo."""
    w = wl.WORKLOADS[name]
    return dataclasses.replace(w, shape=dataclasses.replace(w.shape, o_groups=o_groups, o_lora_rank=o_lora_rank))


@pytest.mark.parametrize("name,groups,rank,batch,ctx", [
    ("tiny_fp32", 2, 64, None, None),          # CUDA-core GEMVs
    ("v2lite_bf16", 4, 128, 3, (100, 700)),    # tensor-core decode, few-head attention
    ("v3_bf16", 16, 256, 5, (1, 900)),         # tensor-core decode, head-major attention
])
def test_grouped_output_projection_decode(name, groups, rank, batch, ctx):
    case = DecodeCase(grouped(name, groups, rank), batch=batch, ctx=ctx).run()
    check_case(case)


@pytest.mark.parametrize("name,groups,rank,S", [
    ("tiny_fp32", 2, 64, 40),
    ("v3_prefill_bf16", 16, 256, 200),
    ("v3_prefill_bf16", 8, 512, 129),
])
def test_grouped_output_projection_prefill(name, groups, rank, S):
    run_prefill(grouped(name, groups, rank), S)
