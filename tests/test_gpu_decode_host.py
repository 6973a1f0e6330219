"""The whole decode step from host buffers (mla_decode_step_host) against the
device-buffer calls and the fp64 oracle. It runs the same kernels as
mla_rope_cos_sin + mla_decode_qkv + mla_decode_attn on the same inputs, so its
output and its cache writes are bit-identical to theirs; the output is also
checked against the oracle at the decode tolerances."""
import pytest
import torch

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import workloads as wl

from gpu_common import TOL, DecodeCase, assert_close, to_np

pytestmark = pytest.mark.gpu


def _pin(t):
    return t.detach().cpu().contiguous().pin_memory()


@pytest.mark.parametrize("name,batch,ctx", [
    ("tiny_fp32", 2, (1, 40)),
    ("v2lite_bf16", 5, (1, 300)),
    ("v3_bf16", 3, (100, 700)),
])
def test_decode_step_host_matches_device_calls_and_oracle(name, batch, ctx):
    """Three calls on the same host buffers: the first captures the step's
    graph, the second replays it, the third replays it on new contents of the
    host buffers. Each must equal the device-buffer calls on the same data."""
    w = wl.WORKLOADS[name]
    case = DecodeCase(w, batch=batch, ctx=ctx)
    cache_host_path = case.cache.clone()
    h = case.layer.handle
    n, mbps = batch, case.table.shape[1]
    hid, pos, slot, table, ctxl = (_pin(t) for t in (case.hidden, case.positions, case.slot, case.table, case.ctx))
    out_h = torch.empty((n, w.shape.hidden), dtype=case.hidden.dtype).pin_memory()
    stage = torch.empty(mla.mla_decode_step_host_bytes(h, n, mbps), dtype=torch.uint8, device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(h, n, case.max_ctx), dtype=torch.uint8, device="cuda")
    mla.mla_workspace_init(ws)
    for call in range(3):
        if call == 2:                           # new inputs in the same host buffers
            case.hidden = case.hidden * 0.5
            hid.copy_(case.hidden.cpu())
        if call != 1:
            case.run()                          # device-buffer calls, on case.cache
        out_h.zero_()
        mla.mla_decode_step_host(h, hid, pos, slot, table, ctxl, case.max_ctx, w.shape.rope_theta,
                                 cache_host_path, out_h, stage, ws)
        torch.cuda.synchronize()
        assert torch.equal(out_h, case.out.cpu()), f"call {call}"
        assert torch.equal(cache_host_path, case.cache), f"call {call}"
        if call == 0:                           # the oracle knows the original inputs only
            r = case.oracle()
            assert_close(to_np(out_h)[r["seqs"]], r["out"], TOL[w.shape.act_dtype], "out")
    assert mla.mla_read_device_flag(ws) == 0


def test_decode_step_host_counts_replayed_launches():
    w = wl.WORKLOADS["v2lite_bf16"]
    case = DecodeCase(w, batch=2, ctx=(5, 70))
    h = case.layer.handle
    hid, pos, slot, table, ctxl = (_pin(t) for t in (case.hidden, case.positions, case.slot, case.table, case.ctx))
    out_h = torch.empty((2, w.shape.hidden), dtype=case.hidden.dtype).pin_memory()
    stage = torch.empty(mla.mla_decode_step_host_bytes(h, 2, case.table.shape[1]), dtype=torch.uint8,
                        device="cuda")
    ws = torch.zeros(mla.mla_workspace_bytes(h, 2, case.max_ctx), dtype=torch.uint8, device="cuda")
    counts = []
    for _ in range(3):
        c0 = mla.mla_kernel_launch_count()
        mla.mla_decode_step_host(h, hid, pos, slot, table, ctxl, case.max_ctx, w.shape.rope_theta, case.cache,
                                 out_h, stage, ws)
        counts.append(mla.mla_kernel_launch_count() - c0)
    torch.cuda.synchronize()
    assert counts[0] > 0 and counts == [counts[0]] * 3


def test_decode_step_host_rejects_small_stage_and_device_inputs():
    w = wl.WORKLOADS["tiny_fp32"]
    case = DecodeCase(w, batch=2, ctx=(4, 9))
    h = case.layer.handle
    mbps = case.table.shape[1]
    need = mla.mla_decode_step_host_bytes(h, 2, mbps)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    ws = torch.empty(mla.mla_workspace_bytes(h, 2, case.max_ctx), dtype=torch.uint8, device="cuda")
    out_h = torch.empty(tuple(case.hidden.shape), dtype=case.hidden.dtype).pin_memory()
    with pytest.raises(mla.MlaError):
        mla.mla_decode_step_host(h, _pin(case.hidden), _pin(case.positions), _pin(case.slot), _pin(case.table),
                                 _pin(case.ctx), case.max_ctx, w.shape.rope_theta, case.cache, out_h, small, ws)
    with pytest.raises(ValueError):
        mla.mla_decode_step_host(h, case.hidden, _pin(case.positions), _pin(case.slot), _pin(case.table),
                                 _pin(case.ctx), case.max_ctx, w.shape.rope_theta, case.cache, out_h,
                                 small, ws)
