"""GPU parity of the decode step with the layer's input RMSNorm folded into
the front-fold ("MLA Decode QKV Kernel API Reference", input_norm_w) and RoPE
tables built from a precomputed frequency table ("Struct MlaWeights",
yarn_inv_freq), against the fp64 oracle given the same gamma and table, at the
decode tolerances (1e-4 * max|ref| fp32, 2e-2 bf16)."""
import numpy as np
import pytest
import torch

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import workloads as wl
from oracle import mla_ref as ref

from gpu_common import DecodeCase, ensure_built
from test_gpu_decode import check_case

pytestmark = pytest.mark.gpu


def _yarn_like(rope_dim, theta=10000.0, factor=40.0):
    # low frequencies divided by `factor`, high ones kept, a linear ramp between
    i = np.arange(rope_dim // 2, dtype=np.float64)
    base = theta ** (-2.0 * i / rope_dim)
    ramp = np.clip((i - 0.25 * len(i)) / max(0.5 * len(i), 1.0), 0.0, 1.0)
    return (base * (1.0 - ramp) + base / factor * ramp).astype(np.float32)


@pytest.mark.parametrize("name,batch,ctx", [
    ("tiny_fp32", 3, (1, 40)),
    ("v2lite_bf16", 4, (1, 300)),
    ("v3_bf16", 3, (100, 600)),
    ("v3_fp8", 2, (64, 200)),
])
def test_decode_with_input_norm_and_yarn_table(name, batch, ctx):
    w = wl.WORKLOADS[name]
    g = (1.0 + np.random.default_rng(5).uniform(-0.3, 0.3, w.shape.hidden)).astype(np.float32)
    case = DecodeCase(w, batch=batch, ctx=ctx, input_norm_w=g, inv_freq=_yarn_like(w.shape.qk_rope)).run()
    check_case(case)


def test_rope_tables_from_a_frequency_table():
    ensure_built()
    pos = torch.tensor([0, 1, 5, 4095, 163839], dtype=torch.int32, device="cuda")
    f = _yarn_like(64)
    cos = torch.empty((5, 32), dtype=torch.float32, device="cuda")
    sin = torch.empty_like(cos)
    mla.mla_rope_cos_sin_inv_freq(pos, 64, torch.from_numpy(f).cuda(), cos, sin)
    rc, rs = ref.rope_cos_sin(pos.cpu().numpy(), 64, 1.0, inv_freq=f.astype(np.float64))
    # fp64 on both sides from the same fp32 table, one rounding to fp32
    np.testing.assert_allclose(cos.cpu().numpy(), rc, rtol=0, atol=2e-7)
    np.testing.assert_allclose(sin.cpu().numpy(), rs, rtol=0, atol=2e-7)
