"""GPU checks of the decode step's exact parts and of its rarely taken branches,
through the C-ABI, against the fp64 oracle:

- the slot scatter of the tensor-core front-fold (bf16 and FP8 weights, both
  cache row orders): exactly the mapped rows change, every other byte of the
  cache is kept, and the written rows match the oracle's rows;
- out-of-range slots on that path: the device flag is set and nothing is written;
- the lazily moved reference max of both tensor-core attention kernels, on
  inputs built so that the two CTAs of a pair see one cache row's score on
  opposite sides of the rescale threshold;
- the [k_pe | latent] row order on the few-head attention kernel.
"""
import math

import numpy as np
import pytest
import torch

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import workloads as wl
from head_latent_attention_decode_b200.layer import MlaLayer
from oracle import mla_ref as ref

from gpu_common import TOL, DecodeCase, assert_close, assert_close_per_head, to_dev, to_np
from test_gpu_decode import check_case

pytestmark = pytest.mark.gpu

TC_WORKLOADS = ["v2lite_bf16", "v3_bf16", "v3_fp8"]


@pytest.mark.parametrize("name", TC_WORKLOADS)
@pytest.mark.parametrize("layout", [ref.LATENT_FIRST, ref.PE_FIRST])
def test_tensor_core_scatter_touches_only_mapped_rows(name, layout):
    """Distinct random slots (one -1 = skip) into a cache filled with random
    16-bit patterns: every row not mapped keeps its bytes, every mapped row
    changes, and the mapped rows hold the oracle's (normed latent, rotated
    k_pe) row in the handle's row order, within the bf16 tolerance."""
    case = DecodeCase(wl.WORKLOADS[name], batch=6, ctx=(5, 40), row_layout=layout)
    s = case.shape
    n_rows = case.cache.shape[0] * s.block_size
    R = s.kv_row_dim
    rng = np.random.default_rng(17)
    slots = rng.choice(n_rows, size=6, replace=False).astype(np.int32)
    slots[3] = -1
    bits = rng.integers(-2**15, 2**15 - 1, size=case.cache.numel(), dtype=np.int64).astype(np.int16)
    cache = torch.from_numpy(bits).view(torch.bfloat16).reshape(case.cache.shape).cuda()
    before = cache.view(torch.int16).reshape(n_rows, R).cpu().numpy().copy()
    case.layer.decode_qkv(case.hidden, case.cos, case.sin, cache, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    after = cache.view(torch.int16).reshape(n_rows, R).cpu().numpy()
    written = sorted(int(x) for x in slots if x >= 0)
    changed = np.nonzero(np.any(after != before, axis=1))[0].tolist()
    assert changed == written
    W = ref.weights_fp64(case.weights)
    cos, sin = ref.rope_cos_sin(case.inp.positions, s.qk_rope, s.rope_theta)
    c, k_pe = ref.kv_projection(s, W, case.inp.hidden, cos, sin)
    rows = ref.cache_row(c, k_pe, layout)
    got = cache.reshape(n_rows, R)
    for t, slot in enumerate(slots):
        if slot >= 0:
            assert_close(to_np(got[int(slot)]), rows[t], TOL["bf16"], f"{name} row {slot}")
    assert case.flag() == 0


@pytest.mark.parametrize("name", TC_WORKLOADS)
def test_tensor_core_out_of_range_slot_sets_flag_and_writes_nothing(name):
    case = DecodeCase(wl.WORKLOADS[name], batch=3, ctx=(10, 20))
    n_rows = case.cache.shape[0] * case.shape.block_size
    before = case.cache.clone()
    slots = torch.tensor([n_rows, -1, n_rows + 1000], dtype=torch.int32, device="cuda")
    case.layer.decode_qkv(case.hidden, case.cos, case.sin, case.cache, slots)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), case.cache.view(torch.int16))
    assert case.flag() & mla.MLA_FLAG_BAD_SLOT
    mla.mla_clear_device_flag(case.layer.ws)
    assert case.flag() == 0


def test_v2lite_bf16_pe_first_ragged():
    # [k_pe | latent] rows on the few-head kernel, with contexts of 1 to 300 rows
    case = DecodeCase(wl.WORKLOADS["v2lite_bf16"], batch=7, ctx=(1, 300), row_layout=ref.PE_FIRST).run()
    check_case(case)


# ---------------------------------------------------------------------------
# the lazily moved reference max
# ---------------------------------------------------------------------------

def _bf16(x):
    return float(torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).float())


def _threshold_combos(scale):
    """Triples (a, A, B) of bf16 values for which the two roundings the pair of
    CTAs applies to one score land on opposite sides of the rescale threshold.

    With q_abs[h] = a at latent column c0 (first CTA's half) and 1 at column c1
    (second CTA's half), and a cache row holding A at c0 and B at c1, the
    partial scores are S0 = a*A and S1 = B (each exact in fp32). One CTA adds
    its own S0 to the peer's f16(S1) (= S1, exact), the other f16(S0) to its
    own S1. After a first tile whose scores are all 0 (reference max 0), a row
    moves the reference when its score times scale*log2(e) exceeds 8. Each
    triple puts that threshold at least 0.003 inside the gap between the two
    sums. The partials stay near the threshold's own size (S0 about 77), so the
    gap (the f16 rounding of S0, at most 1/32) changes the row's weight by
    under 0.3%: the divergence is exercised without an f16 error beyond the
    tolerance. Returns (combos with the first CTA above, with the second)."""
    c = np.float32(scale) * np.float32(1.4426950408889634)
    tr = 8.0 / float(c)
    first, second = [], []
    for k in range(1, 24):
        a = 1.0 + k / 128.0
        for A in np.arange(40.0, 80.0, 0.25):
            if _bf16(A) != A:
                continue
            s0 = a * float(A)
            f = float(np.float16(s0))
            if f == s0:
                continue
            mid = tr - (s0 + f) / 2
            for B in {_bf16(mid), _bf16(mid + 0.004), _bf16(mid - 0.004)}:
                if B == 0.0:
                    continue
                v_first, v_second = s0 + B, f + B
                if min(v_first, v_second) < tr - 0.003 and max(v_first, v_second) > tr + 0.003:
                    (first if v_first > v_second else second).append((a, float(A), B))
    return first, second


def lazy_max_case(s, n, L, special):
    """Inputs of the lazy-max test (numpy, all bf16 values): q_abs [n, H, r_kv],
    q_pe [n, H, d_r] (zeros), cache rows [n_blocks * bs, R], block table and
    context lengths; row `special` of every sequence holds the straddling
    score, every other row scores exactly 0."""
    H, rkv, dr, bs, R = s.n_heads, s.kv_lora_rank, s.qk_rope, s.block_size, s.kv_row_dim
    first, second = _threshold_combos(1.0 / math.sqrt(s.qk_nope + s.qk_rope))
    assert len(first) >= 8 and len(second) >= 8
    combos = [(first if h % 2 else second)[(h * 7) % 8] for h in range(H)]
    rng = np.random.default_rng(23)
    nb = n * L // bs
    n_blocks = nb + 3
    table = rng.permutation(n_blocks)[:nb].reshape(n, L // bs).astype(np.int32)
    cache = wl.round_to(rng.standard_normal((n_blocks * bs, R)), "bf16")
    q_abs = np.zeros((n, H, rkv), np.float32)
    for h in range(H):
        cache[:, h] = 0.0
        cache[:, 256 + h] = 0.0
        q_abs[:, h, h] = combos[h][0]
        q_abs[:, h, 256 + h] = 1.0
    for b in range(n):
        row = table[b, special // bs] * bs + special % bs
        for h in range(H):
            cache[row, h] = combos[h][1]
            cache[row, 256 + h] = combos[h][2]
    assert np.array_equal(wl.round_to(cache, "bf16"), cache)
    assert np.array_equal(wl.round_to(q_abs, "bf16"), q_abs)
    q_pe = np.zeros((n, H, dr), np.float32)
    lens = np.full(n, L, np.int32)
    return q_abs, q_pe, cache, table, lens


@pytest.mark.parametrize("name,special", [("v2lite_bf16", 130), ("v3_bf16", 70)])
def test_lazy_max_diverging_between_the_pair(name, special):
    """Every sequence has one cache row, in the second tile of its first KV
    split (128-row tiles and splits of at least two tiles on the few-head
    kernel, 64-row tiles and splits of at least four on the head-major one),
    whose score sits, per head, within a few hundredths of a score unit of
    the rescale threshold, on the far side of it for one CTA of the pair and
    on the near side for the other; all other rows score 0. The two CTAs then keep
    different reference maxima, and each half of the latent must be
    normalised with its own CTA's statistics."""
    w = wl.WORKLOADS[name]
    s = w.shape
    n, L = 4, 2048
    q_abs, q_pe, cache, table, lens = lazy_max_case(s, n, L, special)
    n_blocks, bs, R, H = cache.shape[0] // s.block_size, s.block_size, s.kv_row_dim, s.n_heads
    weights = wl.make_weights(s, w.seed)
    layer = MlaLayer(s, weights)
    act = layer.act
    d_cache = to_dev(cache.reshape(n_blocks, 1, bs, R), act)
    head = torch.empty((n, H, s.v_dim), dtype=act, device="cuda")
    ws = layer.workspace(n, L)
    mla.mla_clear_device_flag(ws)
    out = layer.decode_attn(to_dev(q_abs, act), to_dev(q_pe, act), d_cache, torch.from_numpy(table).cuda(),
                            torch.from_numpy(lens).cuda(), L, head_out=head)
    torch.cuda.synchronize()
    W = ref.weights_fp64(weights)
    r_out, r_head = ref.decode_attn(s, W, q_abs.astype(np.float64), q_pe.astype(np.float64),
                                    cache.reshape(n_blocks, 1, bs, R).astype(np.float64), table, lens)
    tol = TOL["bf16"]
    assert_close_per_head(to_np(head), r_head, tol, "head_out")
    assert_close(to_np(out), r_out, tol, "out")
    assert mla.mla_read_device_flag(ws) == 0
