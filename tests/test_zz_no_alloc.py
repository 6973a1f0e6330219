"""The allocation-free front-fold (mla_decode_qkv_noalloc) against the regular
entry point. It exists for callers that cannot allocate device memory (a
process whose memory is all reserved by its own pool, or a serving loop that
must not call cudaMalloc); its scratch is a fixed device array inside the
library. Two calls in a row must both match mla_decode_qkv, since every call
reuses the same array, and neither may take device memory. Collected last on
purpose."""
import gc

import pytest
import torch

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import workloads as wl

from gpu_common import TOL, DecodeCase, assert_close, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,batch,ctx", [("v3_bf16", 8, (100, 600)), ("tiny_fp32", 2, (64, 64))])
def test_noalloc_front_fold_matches_regular_entry(name, batch, ctx):
    case = DecodeCase(wl.WORKLOADS[name], batch=batch, ctx=ctx)
    s = case.shape
    ref_cache = case.cache.clone()
    q_abs_ref, q_pe_ref = case.layer.decode_qkv(case.hidden, case.cos, case.sin, ref_cache, case.slot)
    torch.cuda.synchronize()
    tol = TOL[s.act_dtype]
    caches = [case.cache.clone() for _ in range(2)]
    outs = [(torch.full_like(q_abs_ref, float("nan")), torch.full_like(q_pe_ref, float("nan"))) for _ in range(2)]
    free_before, used_before = None, None
    for call in range(2):
        if call == 1:   # the first call has run: nothing more may be taken from the device
            # tensors left unreachable by earlier tests are freed now, not by a
            # collection in the middle of the measured call
            gc.collect()
            gc.disable()
            torch.cuda.synchronize()
            free_before, used_before = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        q_abs, q_pe = outs[call]
        mla.mla_decode_qkv_noalloc(case.layer.handle, case.hidden, case.cos, case.sin, caches[call], case.slot,
                                   q_abs, q_pe)
        torch.cuda.synchronize()
        if call == 1:
            gc.enable()
            assert torch.cuda.mem_get_info()[0] == free_before
            assert torch.cuda.memory_allocated() == used_before
        assert mla.mla_noalloc_read_device_flag() == 0
        assert_close(to_np(q_abs), to_np(q_abs_ref), tol, f"q_abs (call {call})")
        assert_close(to_np(q_pe), to_np(q_pe_ref), tol, f"q_pe (call {call})")
        assert_close(to_np(caches[call].reshape(-1, s.kv_row_dim)), to_np(ref_cache.reshape(-1, s.kv_row_dim)),
                     tol, f"cache (call {call})")


def test_noalloc_reports_bad_slot_through_its_flag():
    case = DecodeCase(wl.WORKLOADS["v3_bf16"], batch=2, ctx=(10, 20))
    n_rows = case.cache.shape[0] * case.shape.block_size
    before = case.cache.clone()
    bad = torch.tensor([n_rows, n_rows + 5], dtype=torch.int32, device="cuda")
    q_abs = torch.empty((2, case.shape.n_heads, case.shape.kv_lora_rank), dtype=case.act, device="cuda")
    q_pe = torch.empty((2, case.shape.n_heads, case.shape.qk_rope), dtype=case.act, device="cuda")
    mla.mla_decode_qkv_noalloc(case.layer.handle, case.hidden, case.cos, case.sin, case.cache, bad, q_abs, q_pe)
    assert mla.mla_noalloc_read_device_flag() & mla.MLA_FLAG_BAD_SLOT
    assert torch.equal(before.view(torch.int16), case.cache.view(torch.int16))
    # the next call clears the flag before it runs
    mla.mla_decode_qkv_noalloc(case.layer.handle, case.hidden, case.cos, case.sin, case.cache, case.slot,
                               q_abs, q_pe)
    assert mla.mla_noalloc_read_device_flag() == 0


def test_noalloc_rejects_batches_beyond_the_array():
    """The first batch the array cannot hold is exactly the first batch a
    regular call given a workspace of the array's size rejects too."""
    case = DecodeCase(wl.WORKLOADS["v3_bf16"], batch=1, ctx=(10, 10))
    s = case.shape
    ws = torch.zeros(mla.MLA_NOALLOC_SCRATCH_BYTES, dtype=torch.uint8, device="cuda")

    def tensors(n):
        half = s.qk_rope // 2
        return (torch.zeros((n, s.hidden), dtype=case.act, device="cuda"),
                torch.zeros((n, half), dtype=torch.float32, device="cuda"),
                torch.zeros((n, half), dtype=torch.float32, device="cuda"),
                torch.full((n,), -1, dtype=torch.int32, device="cuda"),
                torch.empty((n, s.n_heads, s.kv_lora_rank), dtype=case.act, device="cuda"),
                torch.empty((n, s.n_heads, s.qk_rope), dtype=case.act, device="cuda"))

    def status(fn, n):
        x, c, sn, sl, qa, qp = tensors(n)
        try:
            fn(x, c, sn, sl, qa, qp)
            torch.cuda.synchronize()
            return mla.MLA_OK
        except mla.MlaError as e:
            return e.status

    noalloc = lambda x, c, sn, sl, qa, qp: mla.mla_decode_qkv_noalloc(case.layer.handle, x, c, sn, case.cache,
                                                                      sl, qa, qp)
    regular = lambda x, c, sn, sl, qa, qp: mla.mla_decode_qkv(case.layer.handle, x, c, sn, case.cache, sl,
                                                              qa, qp, ws)
    lo, hi = 1, 1
    while status(noalloc, hi) == mla.MLA_OK:
        lo, hi = hi, hi * 2
        assert hi <= 4096
    while hi - lo > 1:   # first rejected batch
        mid = (lo + hi) // 2
        if status(noalloc, mid) == mla.MLA_OK:
            lo = mid
        else:
            hi = mid
    assert status(noalloc, hi) == mla.MLA_ERR_WORKSPACE
    assert status(regular, hi) == mla.MLA_ERR_WORKSPACE
    assert status(regular, lo) == mla.MLA_OK
