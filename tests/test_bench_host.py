"""Host-side logic of bench.py that needs no GPU: the profiling-slice options,
which kernel a workload's roofline names, and how the DRAM traffic of that
kernel is read from the committed ncu summary (null when there is none, or when
the kernel's source changed since the capture)."""
import hashlib
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from head_latent_attention_decode_b200 import workloads as wl  # noqa: E402


def _args(**kw):
    base = dict(workload="v3_fp8", batch=0, context=0)
    base.update(kw)
    return types.SimpleNamespace(**base)


def test_slice_options_change_only_what_they_name():
    w = bench.selected_workload(_args())
    assert w == wl.WORKLOADS["v3_fp8"]
    s = bench.selected_workload(_args(batch=16))
    assert s.batch == 16 and s.name == "v3_fp8[batch=16]"
    assert (s.shape, s.ctx_lo, s.ctx_hi, s.seed) == (w.shape, w.ctx_lo, w.ctx_hi, w.seed)
    c = bench.selected_workload(_args(context=256))
    assert (c.ctx_lo, c.ctx_hi, c.batch) == (256, 256, w.batch)
    # prefill and projection workloads have no decode batch to slice
    p = bench.selected_workload(_args(workload="v3_prefill_bf16", batch=16))
    assert p == wl.WORKLOADS["v3_prefill_bf16"]
    # argument objects without the options (as other callers build them) select the workload as named
    assert bench.selected_workload(types.SimpleNamespace(workload="tiny_fp32")) == wl.WORKLOADS["tiny_fp32"]


def test_dominant_kernel_follows_mode_and_heads():
    assert bench.dominant_kernel(wl.WORKLOADS["v3_fp8"]) == "tc_attn_decode_kernel"
    assert bench.dominant_kernel(wl.WORKLOADS["v2lite_bf16"]) == "tc_attn_pair_kernel"
    assert bench.dominant_kernel(wl.WORKLOADS["v3_prefill_bf16"]) == "tc_prefill_attn_kernel"
    assert bench.dominant_kernel(wl.WORKLOADS["v4_qkv_bf16"]) == "tc_gemm_kernel"


def test_traffic_comes_from_a_summary_of_the_current_source():
    # every committed summary that names a kernel source either matches it (traffic read) or not (null)
    for name in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        if not name.startswith("ncu_") or not name.endswith(".md"):
            continue
        text = open(os.path.join(ROOT, "profiles", name)).read()
        kernel = next((k for k in bench.KERNEL_SOURCES if name.startswith(f"ncu_{k}_")), None)
        if kernel is None:
            continue
        workload = name[len(f"ncu_{kernel}_"):-3]
        src = os.path.join(ROOT, "head_latent_attention_decode_b200", "csrc", bench.KERNEL_SOURCES[kernel])
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
        t = bench.measured_traffic(kernel, workload)
        if f"kernel source sha256: {digest}" in text:
            assert isinstance(t, int) and t > 0, name
        else:
            assert t is None, name
    # the default workload's dominant kernel has a summary of its current source
    assert bench.measured_traffic("tc_attn_decode_kernel", "v3_fp8") is not None
    # a profiling slice names no summary, so it claims no traffic
    assert bench.measured_traffic("tc_attn_decode_kernel", "v3_fp8[batch=16]") is None
