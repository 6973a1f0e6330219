"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every entry point include/mla.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import dataclasses
import os
import re

import pytest

import head_latent_attention_decode_b200 as mla
from head_latent_attention_decode_b200 import build as mla_build
from head_latent_attention_decode_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mla_build.build()
    return mla.lib()


def header_symbols():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    for name in ("mla_init_weights", "mla_decode_qkv", "mla_decode_attn", "mla_prefill"):
        assert name in syms
    assert set(syms) == set(mla.SYMBOLS)


def test_library_exports_every_header_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_strerror(lib):
    assert mla.mla_strerror(0) == "ok"
    assert "invalid" in mla.mla_strerror(mla.MLA_ERR_INVALID_ARG)
    assert mla.mla_strerror(12345) == "unknown status"


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_weights_bytes_for_every_workload(lib, name):
    s = wl.WORKLOADS[name].shape
    n = mla.mla_weights_bytes(mla.make_config(s))
    esz = {"f32": 4, "bf16": 2, "fp8": 1}[s.weight_dtype]
    params = sum(k * v for k, v in wl.weight_shapes(s).values())
    # the blob holds every weight once, plus W_UK / W_UV / Wkvb slices of wkv_b
    assert n >= params * esz
    assert n < 2 * params * esz + (1 << 24)


def _cfg(**kw):
    c = mla.make_config(wl.TINY)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("bad", [
    dict(qk_rope=15), dict(n_heads=0), dict(hidden=-1), dict(act_dtype=7), dict(row_layout=2),
    dict(weight_dtype=9), dict(norm_eps=-1.0)])
def test_invalid_configs_rejected(lib, bad):
    assert mla.mla_weights_bytes(_cfg(**bad)) == 0
    h = ctypes.c_void_p()
    d = mla.mla_weights_desc()
    assert lib.mla_init_weights(ctypes.byref(_cfg(**bad)), ctypes.byref(d), 256, 1 << 30, None,
                                ctypes.byref(h)) == mla.MLA_ERR_INVALID_ARG


def test_unsupported_combinations(lib):
    # fp8 weights need bf16 activations; mixed f32/bf16 is not offered
    c = _cfg(weight_dtype=mla.MLA_FP8_E4M3_B128)
    h = ctypes.c_void_p()
    d = mla.mla_weights_desc()
    assert lib.mla_init_weights(ctypes.byref(c), ctypes.byref(d), 256, 1 << 30, None,
                                ctypes.byref(h)) == mla.MLA_ERR_UNSUPPORTED
    c = _cfg(act_dtype=mla.MLA_BF16)
    assert lib.mla_init_weights(ctypes.byref(c), ctypes.byref(d), 256, 1 << 30, None,
                                ctypes.byref(h)) == mla.MLA_ERR_UNSUPPORTED


def test_init_rejects_missing_weights_and_small_blob(lib):
    c = _cfg()
    h = ctypes.c_void_p()
    d = mla.mla_weights_desc()            # all NULL
    assert lib.mla_init_weights(ctypes.byref(c), ctypes.byref(d), 256, 1 << 30, None,
                                ctypes.byref(h)) == mla.MLA_ERR_INVALID_ARG
    d = mla.mla_weights_desc(*([4096] * 7 + [None] * 5))
    assert lib.mla_init_weights(ctypes.byref(c), ctypes.byref(d), 256, 16, None,
                                ctypes.byref(h)) == mla.MLA_ERR_WORKSPACE
    assert lib.mla_init_weights(ctypes.byref(c), ctypes.byref(d), 257, 1 << 30, None,
                                ctypes.byref(h)) == mla.MLA_ERR_INVALID_ARG   # misaligned blob


def test_calls_reject_null_handle_and_bad_sizes(lib):
    P = 4096
    assert lib.mla_decode_qkv(None, P, 1, P, P, P, 1, P, P, P, None, P, 1 << 20, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_attn(None, P, P, P, 1, P, 1, P, 1, 1, P, None, P, 1 << 20, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_prefill(None, P, 1, P, P, P, None, None, 0, None, P, 1 << 20, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_workspace_bytes(None, 1, 1) == 0
    assert lib.mla_decode_step_host_bytes(None, 1, 1) == 0
    assert lib.mla_decode_step_host(None, P, P, P, P, 1, P, 1, 1, 10000.0, P, 1, P, P, 1 << 20, P, 1 << 20,
                                    None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_rope_cos_sin(P, 4, 15, 10000.0, P, P, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_rope_cos_sin(P, -1, 16, 10000.0, P, P, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_rope_cos_sin(P, 4, 16, -1.0, P, P, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_rope_cos_sin(None, 0, 16, 10000.0, None, None, None) == mla.MLA_OK  # empty
    assert lib.mla_rope_cos_sin_inv_freq(P, 4, 15, P, P, P, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_rope_cos_sin_inv_freq(P, 4, 16, None, P, P, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_rope_cos_sin_inv_freq(None, 0, 16, None, None, None, None) == mla.MLA_OK  # empty
    assert lib.mla_workspace_init(None, 1024, None) == mla.MLA_ERR_INVALID_ARG
    v = ctypes.c_int()
    assert lib.mla_read_device_flag(None, ctypes.byref(v), None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_clear_device_flag(None, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_v4_qkv(None, P, 1, P, P, P, P, P, P, 1 << 20, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_v4_qkv(None, P, -1, P, P, P, P, P, P, 1 << 20, None) == mla.MLA_ERR_INVALID_ARG


def test_weights_descriptor_field_order_matches_the_header():
    """The C struct's field order: twelve weight / gamma / scale pointers, the
    optional attn_sink pointer, then the grouped output projection's wo_a and
    wo_b (a zero-initialised descriptor has neither)."""
    names = [f[0] for f in mla.mla_weights_desc._fields_]
    assert names[-3:] == ["attn_sink", "wo_a", "wo_b"] and len(names) == 15
    assert ctypes.sizeof(mla.mla_weights_desc) == 15 * ctypes.sizeof(ctypes.c_void_p)
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "mla.h")).read()
    body = hdr[hdr.index("typedef struct {\n  const void* wq_a;"):hdr.index("} mla_weights_desc;")]
    fields = [ln.strip().rstrip(";").split()[-1].lstrip("*") for ln in body.splitlines()[1:] if ln.strip()]
    assert fields == names


def test_launch_counter_starts_at_zero_without_gpu_work(lib):
    assert mla.mla_kernel_launch_count() == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No silent fallback: without the built library every entry point raises."""
    from head_latent_attention_decode_b200.layer import MlaLayer
    monkeypatch.setattr(mla, "LIB_PATH", str(tmp_path / "libmla_b200.so"))
    monkeypatch.setattr(mla, "_lib", None)
    with pytest.raises(ImportError):
        mla.lib()
    with pytest.raises(ImportError):
        mla.mla_weights_bytes(mla.make_config(wl.TINY))
    with pytest.raises(ImportError):
        MlaLayer(wl.TINY, wl.make_weights(wl.TINY, 0), device="cpu")


def test_config_field_order_matches_the_header():
    names = [f[0] for f in mla.mla_config._fields_]
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "mla.h")).read()
    body = hdr[hdr.index("typedef struct {\n  int hidden;"):hdr.index("} mla_config;")]
    fields = [ln.split(";")[0].split()[-1] for ln in body.splitlines()[1:] if ln.strip().startswith(("int ", "float "))]
    assert fields == names and names[-2:] == ["o_groups", "o_lora_rank"]


def test_grouped_output_projection_config_checks(lib):
    """o_lora_rank > 0 needs o_groups dividing H, 64-multiple sizes, and no FP8."""
    base = wl.MlaShape(hidden=256, n_heads=4, q_lora_rank=64, kv_lora_rank=64, qk_nope=32, qk_rope=16,
                       v_dim=32, block_size=16, act_dtype="f32", weight_dtype="f32")
    ok = dataclasses.replace(base, o_groups=2, o_lora_rank=64)
    assert mla.mla_weights_bytes(mla.make_config(ok)) > 0
    for bad in (dataclasses.replace(base, o_groups=3, o_lora_rank=64),     # 3 does not divide 4 heads
                dataclasses.replace(base, o_groups=0, o_lora_rank=64),
                dataclasses.replace(base, o_groups=4, o_lora_rank=64),     # 32 inputs per group
                dataclasses.replace(base, o_groups=2, o_lora_rank=48)):
        assert mla.mla_weights_bytes(mla.make_config(bad)) == 0, bad
