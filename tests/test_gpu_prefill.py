"""GPU parity of the causal expanded prefill (mla_prefill) against the fp64
oracle through the C-ABI: small sequences with ragged tails checked in full,
the 8192-token DeepSeek-V3-shaped case on sampled query rows."""
import dataclasses

import numpy as np
import pytest
import torch

from head_latent_attention_decode_b200 import workloads as wl
from head_latent_attention_decode_b200.layer import ACT_TORCH, MlaLayer
from oracle import mla_ref as ref

from gpu_common import TOL, assert_close, assert_close_per_head, ensure_built, to_dev, to_np

pytestmark = pytest.mark.gpu

TINY_PREFILL = dataclasses.replace(wl.WORKLOADS["v3_prefill_bf16"], shape=wl.TINY, seed=9)
V2LITE_PREFILL = dataclasses.replace(wl.WORKLOADS["v3_prefill_bf16"], shape=wl.V2LITE, seed=10)
V3_FP8_PREFILL = dataclasses.replace(wl.WORKLOADS["v3_prefill_bf16"], shape=wl.WORKLOADS["v3_fp8"].shape, seed=12)


def run_prefill(workload, S, rows=None, with_cache=False, attn_sink=None):
    """attn_sink: optional fp32 [n_heads] sink logits, given to both sides."""
    ensure_built()
    s = workload.shape
    weights = wl.make_weights(s, workload.seed)
    x, pos = wl.make_prefill_inputs(workload, seq_len=S)
    layer = MlaLayer(s, weights, attn_sink=attn_sink)
    act = ACT_TORCH[s.act_dtype]
    xd = to_dev(x, act)
    cos, sin = layer.rope(torch.from_numpy(pos).cuda())
    head = torch.empty((S, s.n_heads, s.v_dim), dtype=act, device="cuda")
    cache = slots = None
    if with_cache:
        nb = (S + s.block_size - 1) // s.block_size + 2
        cache = torch.zeros((nb, 1, s.block_size, s.kv_row_dim), dtype=act, device="cuda")
        perm = np.random.default_rng(1).permutation(nb)
        slots = torch.from_numpy((perm[np.arange(S) // s.block_size] * s.block_size
                                  + np.arange(S) % s.block_size).astype(np.int32)).cuda()
    out = layer.prefill(xd, cos, sin, head_out=head, kv_cache=cache, slot_mapping=slots)
    torch.cuda.synchronize()
    W = ref.weights_fp64(weights)
    rcos, rsin = ref.rope_cos_sin(pos, s.qk_rope, s.rope_theta)
    r_out, r_head, r_rows = ref.prefill(s, W, x, rcos, rsin, rows=rows, attn_sink=attn_sink)
    sel = np.arange(S) if rows is None else np.asarray(rows)
    tol = TOL[s.act_dtype]
    assert_close_per_head(to_np(head)[sel], r_head, tol, "head_out")
    assert_close(to_np(out)[sel], r_out, tol, "out")
    if with_cache:
        got = to_np(cache.reshape(-1, s.kv_row_dim))[slots.cpu().numpy()]
        assert_close(got, r_rows, tol, "cache rows")
    import head_latent_attention_decode_b200 as mla
    assert mla.mla_read_device_flag(layer.ws) == 0


def test_tiny_fp32_prefill_ragged():
    run_prefill(TINY_PREFILL, S=77, with_cache=True)


def test_tiny_fp32_prefill_single_token():
    run_prefill(TINY_PREFILL, S=1)


def test_v2lite_bf16_prefill_small():
    run_prefill(V2LITE_PREFILL, S=200)


@pytest.mark.parametrize("S", [1, 128, 129, 256])
def test_v2lite_bf16_prefill_tile_edges(S):
    """The tensor-core attention's degenerate sizes: one token (a single
    diagonal tile with one key), exactly one query tile, one row into a second
    tile, and an exact multiple of the tile."""
    run_prefill(V2LITE_PREFILL, S=S, with_cache=True)


def test_v3_bf16_prefill_small():
    run_prefill(wl.WORKLOADS["v3_prefill_bf16"], S=300, with_cache=True)


@pytest.mark.parametrize("S", [129, 300])
def test_v3_fp8_weights_prefill(S):
    """FP8-E4M3 weights with 128 x 128 block scales on the tensor-core prefill:
    each weight dequantised into the workspace just before its GEMM."""
    run_prefill(V3_FP8_PREFILL, S=S, with_cache=True)


def test_v3_bf16_prefill_full_sampled():
    rng = np.random.default_rng(0)
    rows = sorted(set([0, 127, 128, 8191] + rng.integers(0, 8192, 60).tolist()))
    run_prefill(wl.WORKLOADS["v3_prefill_bf16"], S=8192, rows=rows)
