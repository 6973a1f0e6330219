"""The allocation-free front-fold (mla_decode_qkv_noalloc) against the regular
entry point. It exists for callers that cannot allocate device memory (a
process whose memory is all reserved by its own pool, or a serving loop that
must not call cudaMalloc); its scratch is a fixed device array inside the
library. Two calls in a row must both match mla_decode_qkv, since every call
reuses the same array. Collected last on purpose."""
import numpy as np
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
    n = case.hidden.shape[0]
    ref_cache = case.cache.clone()
    q_abs_ref, q_pe_ref = case.layer.decode_qkv(case.hidden, case.cos, case.sin, ref_cache, case.slot)
    torch.cuda.synchronize()
    tol = TOL[s.act_dtype]
    for call in range(2):
        cache = case.cache.clone()
        q_abs = torch.full_like(q_abs_ref, float("nan"))
        q_pe = torch.full_like(q_pe_ref, float("nan"))
        mla.mla_decode_qkv_noalloc(case.layer.handle, case.hidden, case.cos, case.sin, cache, case.slot,
                                   q_abs, q_pe)
        torch.cuda.synchronize()
        assert_close(to_np(q_abs), to_np(q_abs_ref), tol, f"q_abs (call {call})")
        assert_close(to_np(q_pe), to_np(q_pe_ref), tol, f"q_pe (call {call})")
        assert_close(to_np(cache.reshape(-1, s.kv_row_dim)), to_np(ref_cache.reshape(-1, s.kv_row_dim)),
                     tol, f"cache (call {call})")


def test_noalloc_rejects_batches_beyond_the_array():
    case = DecodeCase(wl.WORKLOADS["v3_bf16"], batch=1, ctx=(10, 10))
    n = 1
    while mla.mla_workspace_bytes(case.layer.handle, n, 1) <= mla.MLA_NOALLOC_SCRATCH_BYTES:
        n *= 2
    hidden = torch.zeros((n, case.shape.hidden), dtype=case.act, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_qkv_noalloc(case.layer.handle, hidden, case.cos, case.sin, case.cache,
                                   case.slot, case.cache, case.cache)
    assert e.value.status == mla.MLA_ERR_WORKSPACE
