"""GPU parity of the decode step (mla_decode_qkv + mla_decode_attn) against the
fp64 oracle, through the C-ABI, for every decode workload shape: small cases
the oracle finishes in seconds (ragged lengths, several tiles, both cache row
layouts) and the full sizes on sampled sequences. Tolerances: 1e-4 * max|ref|
for fp32, 2e-2 * max|ref| (per head for head_out) for bf16 / FP8 weights."""
import dataclasses

import numpy as np
import pytest
import torch

from head_latent_attention_decode_b200 import workloads as wl
from oracle import mla_ref as ref

from gpu_common import (TOL, DecodeCase, assert_close, assert_close_per_head, ensure_built,
                        to_dev, to_np)

pytestmark = pytest.mark.gpu


def check_case(case, seqs=None, check_cache=True):
    r = case.oracle(seqs)
    s = case.shape
    tol = TOL[s.act_dtype]
    idx = r["seqs"]
    assert_close(to_np(case.q_abs)[idx], r["q_abs"], tol, "q_abs")
    assert_close(to_np(case.q_pe)[idx], r["q_pe"], tol, "q_pe")
    assert_close_per_head(to_np(case.head_out)[idx], r["head_out"], tol, "head_out")
    assert_close(to_np(case.out)[idx], r["out"], tol, "out")
    if check_cache:
        bs, R = s.block_size, s.kv_row_dim
        gpu_rows = to_np(case.cache.reshape(-1, R))
        want = r["cache"].reshape(-1, R)
        for i, slot in enumerate(r["slots"]):
            g = int(r["blocks"][slot // bs]) * bs + slot % bs
            assert g == int(case.inp.slot_mapping[idx[i]])
            assert_close(gpu_rows[g], want[slot], tol, f"cache row {g}")
    assert case.flag() == 0
    return r


def test_tiny_fp32_full():
    case = DecodeCase(wl.WORKLOADS["tiny_fp32"]).run()
    check_case(case)


def test_tiny_fp32_pe_first_layout():
    case = DecodeCase(wl.WORKLOADS["tiny_fp32"], row_layout=ref.PE_FIRST).run()
    check_case(case)


def test_tiny_fp32_ragged_contexts():
    w = dataclasses.replace(wl.WORKLOADS["tiny_fp32"], batch=5, ctx_lo=1, ctx_hi=300)
    case = DecodeCase(w).run()
    check_case(case)


def test_v2lite_bf16_small():
    case = DecodeCase(wl.WORKLOADS["v2lite_bf16"], batch=3, ctx=(300, 1100)).run()
    check_case(case)


def test_v2lite_bf16_ragged_single_tiles():
    # contexts of 1 to 300 rows: units of one, two and three 128-row tiles, so
    # the rotary block falls on either CTA of the pair and tails are ragged
    case = DecodeCase(wl.WORKLOADS["v2lite_bf16"], batch=7, ctx=(1, 300)).run()
    check_case(case)


def test_v2lite_bf16_24_heads():
    # 17..32 heads take the 32-column variant of the few-head attention kernel
    w = dataclasses.replace(wl.WORKLOADS["v2lite_bf16"],
                            shape=dataclasses.replace(wl.V2LITE, n_heads=24))
    case = DecodeCase(w, batch=3, ctx=(200, 900)).run()
    check_case(case)


def test_v3_bf16_small_ragged():
    case = DecodeCase(wl.WORKLOADS["v3_bf16"], batch=5, ctx=(1, 2500)).run()
    check_case(case)


def test_v3_bf16_pe_first_small():
    case = DecodeCase(wl.WORKLOADS["v3_bf16"], batch=2, ctx=(60, 200), row_layout=ref.PE_FIRST).run()
    check_case(case)


def test_v3_fp8_small():
    case = DecodeCase(wl.WORKLOADS["v3_fp8"], batch=4, ctx=(100, 1500)).run()
    check_case(case)


# ---------------------------------------------------------------------------
# full sizes (sampled sequences where the oracle would take too long)
# ---------------------------------------------------------------------------

def test_v2lite_bf16_full():
    case = DecodeCase(wl.WORKLOADS["v2lite_bf16"]).run()
    check_case(case, seqs=[0, 7, 31])


def test_v3_bf16_full_sampled():
    case = DecodeCase(wl.WORKLOADS["v3_bf16"]).run()
    lens = case.inp.context_lens
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, 63, 17})
    check_case(case, seqs=seqs)


@pytest.mark.parametrize("batch", [129, 200])
def test_v3_fp8_more_tokens_than_the_fp8_gemm(batch):
    """FP8 weights with 129..256 tokens per call: each weight dequantised to
    bf16 in the workspace, then the bf16 tensor-core GEMMs (the FP8 GEMM takes
    up to 128 tokens); sampled sequences against the oracle."""
    case = DecodeCase(wl.WORKLOADS["v3_fp8"], batch=batch, ctx=(64, 300)).run()
    check_case(case, seqs=[0, 77, batch - 1])


def test_v3_fp8_full_sampled():
    case = DecodeCase(wl.WORKLOADS["v3_fp8"]).run()
    check_case(case, seqs=[0, 64, 127])


@pytest.mark.parametrize("batch", [3, 128])
def test_v3_fp8_without_head_out(batch):
    """Without a head_out buffer the FP8-weight step keeps its internal
    activations (o_lat, the head outputs) in f16, the FP8 GEMM's token type;
    `out` still matches the oracle, and the call that also returns head_out
    (bf16) to within the same tolerance."""
    case = DecodeCase(wl.WORKLOADS["v3_fp8"], batch=batch, ctx=(64, 700)).run()
    out_with_head = to_np(case.out).copy()
    out = case.layer.decode_attn(case.q_abs, case.q_pe, case.cache, case.table, case.ctx, case.max_ctx)
    torch.cuda.synchronize()
    seqs = [0, 1, 2] if batch == 3 else [0, 77, 127]
    r = case.oracle(seqs)
    tol = TOL[case.shape.act_dtype]
    assert_close(to_np(out)[r["seqs"]], r["out"], tol, "out without head_out")
    assert_close(to_np(out), out_with_head, tol, "out with and without head_out")
    assert case.flag() == 0


# ---------------------------------------------------------------------------
# scatter exactness and device-side checks
# ---------------------------------------------------------------------------

def test_scatter_touches_only_mapped_rows_bit_exact():
    """Arbitrary distinct slots (and -1 = skip): every other cache row keeps its
    bytes; written rows match the oracle's (normed latent, rotated k_pe)."""
    ensure_built()
    w = wl.WORKLOADS["tiny_fp32"]
    case = DecodeCase(w, batch=6, ctx=(5, 40))
    s = case.shape
    n_rows = case.cache.shape[0] * s.block_size
    rng = np.random.default_rng(5)
    slots = rng.choice(n_rows, size=6, replace=False).astype(np.int32)
    slots[2] = -1
    sentinel = torch.from_numpy(rng.integers(-2**31, 2**31 - 1, size=case.cache.numel(),
                                             dtype=np.int64).astype(np.int32))
    cache = sentinel.view(torch.float32).reshape(case.cache.shape).cuda()
    before = cache.clone()
    case.layer.decode_qkv(case.hidden, case.cos, case.sin, cache, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    flat_b = before.view(torch.int32).reshape(n_rows, -1).cpu().numpy()
    flat_a = cache.view(torch.int32).reshape(n_rows, -1).cpu().numpy()
    written = set(int(x) for x in slots if x >= 0)
    for r in range(n_rows):
        if r not in written:
            assert np.array_equal(flat_a[r], flat_b[r]), r
        else:
            assert not np.array_equal(flat_a[r], flat_b[r]), r
    W = ref.weights_fp64(case.weights)
    cos, sin = ref.rope_cos_sin(case.inp.positions, s.qk_rope, s.rope_theta)
    c, k_pe = ref.kv_projection(s, W, case.inp.hidden, cos, sin)
    rows = ref.cache_row(c, k_pe, ref.LATENT_FIRST)
    with np.errstate(invalid="ignore"):             # sentinel rows may hold NaN patterns
        got = cache.reshape(n_rows, -1).cpu().numpy().astype(np.float64)
    for t, slot in enumerate(slots):
        if slot >= 0:
            assert_close(got[slot], rows[t], TOL["f32"], f"row {slot}")
    assert case.flag() == 0


def test_out_of_range_slot_sets_flag_and_writes_nothing():
    case = DecodeCase(wl.WORKLOADS["tiny_fp32"], batch=2, ctx=(10, 20))
    n_rows = case.cache.shape[0] * case.shape.block_size
    before = case.cache.clone()
    slots = torch.tensor([n_rows, n_rows + 1000], dtype=torch.int32, device="cuda")
    case.layer.decode_qkv(case.hidden, case.cos, case.sin, case.cache, slots)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int32), case.cache.view(torch.int32))
    import head_latent_attention_decode_b200 as mla
    assert case.flag() & mla.MLA_FLAG_BAD_SLOT
    mla.mla_clear_device_flag(case.layer.ws)
    assert case.flag() == 0


def test_bad_block_and_context_set_flags():
    import head_latent_attention_decode_b200 as mla
    case = DecodeCase(wl.WORKLOADS["tiny_fp32"], batch=2, ctx=(30, 40)).run()
    assert case.flag() == 0
    table = case.table.clone()
    table[0, 0] = case.cache.shape[0] + 5          # out of range block id
    case.layer.decode_attn(case.q_abs, case.q_pe, case.cache, table, case.ctx, case.max_ctx)
    torch.cuda.synchronize()
    assert case.flag() & mla.MLA_FLAG_BAD_BLOCK
    mla.mla_clear_device_flag(case.layer.ws)
    ctx = case.ctx.clone()
    ctx[1] = case.max_ctx + 1                      # beyond the stated maximum
    case.layer.decode_attn(case.q_abs, case.q_pe, case.cache, case.table, ctx, case.max_ctx)
    torch.cuda.synchronize()
    assert case.flag() & mla.MLA_FLAG_BAD_CONTEXT
    mla.mla_clear_device_flag(case.layer.ws)


def test_bad_block_on_tensor_core_path_sets_flag():
    import head_latent_attention_decode_b200 as mla
    for name in ("v2lite_bf16", "v3_bf16"):
        case = DecodeCase(wl.WORKLOADS[name], batch=2, ctx=(150, 300)).run()
        assert case.flag() == 0
        table = case.table.clone()
        table[1, 1] = case.cache.shape[0] + 7      # out of range block id: rows read as zeros, flag set
        table[0, 0] = -3
        case.layer.decode_attn(case.q_abs, case.q_pe, case.cache, table, case.ctx, case.max_ctx)
        torch.cuda.synchronize()
        assert case.flag() & mla.MLA_FLAG_BAD_BLOCK
        mla.mla_clear_device_flag(case.layer.ws)


def test_context_of_one():
    case = DecodeCase(wl.WORKLOADS["v3_bf16"], batch=3, ctx=(1, 1)).run()
    check_case(case)


def test_empty_batch_is_a_no_op():
    import head_latent_attention_decode_b200 as mla
    case = DecodeCase(wl.WORKLOADS["tiny_fp32"], batch=1, ctx=(4, 4))
    before = mla.mla_kernel_launch_count()
    empty = case.hidden[:0]
    case.layer.decode_qkv(empty, case.cos[:0], case.sin[:0], case.cache, case.slot[:0])
    assert mla.mla_kernel_launch_count() == before
