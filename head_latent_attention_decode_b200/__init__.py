"""Python binding of libmla_b200 (include/mla.h): a B200 (sm_100a) MLA layer step.

Argument marshalling only. Every function below has the C entry point's name
and passes torch tensors' device pointers, sizes and the current CUDA stream
to it; every step of the computation runs in the library's CUDA kernels.
torch is used for device memory and streams. Loading fails loudly when the
built library is missing: there is no other implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_b200.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_DEVICE_FLAG = -4
MLA_ERR_WORKSPACE = -5

MLA_FLAG_BAD_SLOT = 1
MLA_FLAG_BAD_BLOCK = 2
MLA_FLAG_BAD_CONTEXT = 4
MLA_FLAG_WAIT_TIMEOUT = 8

MLA_F32, MLA_BF16, MLA_FP8_E4M3_B128 = 0, 1, 2
MLA_ROW_LATENT_FIRST, MLA_ROW_PE_FIRST = 0, 1

SYMBOLS = (
    "mla_weights_bytes", "mla_init_weights", "mla_destroy", "mla_workspace_bytes",
    "mla_workspace_init", "mla_read_device_flag", "mla_clear_device_flag", "mla_rope_cos_sin",
    "mla_decode_qkv", "mla_decode_attn", "mla_prefill", "mla_strerror",
    "mla_kernel_launch_count", "mla_set_kernel_timer", "mla_decode_qkv_noalloc",
    "mla_decode_step_host_bytes", "mla_decode_step_host", "mla_rope_cos_sin_inv_freq",
    "mla_v4_qkv", "mla_noalloc_read_device_flag",
)

MLA_NOALLOC_SCRATCH_BYTES = 64 << 20


class mla_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "hidden", "n_heads", "q_lora_rank", "kv_lora_rank", "qk_nope", "qk_rope", "v_dim",
        "block_size")] + [("norm_eps", ctypes.c_float), ("softmax_scale", ctypes.c_float)] + [
        (n, ctypes.c_int) for n in ("act_dtype", "weight_dtype", "row_layout", "o_groups", "o_lora_rank")]


class mla_weights_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "wq_a", "wq_b", "wkv_a", "wkv_b", "wo", "q_norm_w", "kv_norm_w", "wq_a_scale",
        "wq_b_scale", "wkv_a_scale", "wkv_b_scale", "wo_scale", "attn_sink", "wo_a", "wo_b")]


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {mla_strerror(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m head_latent_attention_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.mla_weights_bytes.restype = sz
        L.mla_weights_bytes.argtypes = [ctypes.POINTER(mla_config)]
        L.mla_init_weights.restype = i
        L.mla_init_weights.argtypes = [ctypes.POINTER(mla_config), ctypes.POINTER(mla_weights_desc),
                                       vp, sz, vp, ctypes.POINTER(vp)]
        L.mla_destroy.restype = None
        L.mla_destroy.argtypes = [vp]
        L.mla_workspace_bytes.restype = sz
        L.mla_workspace_bytes.argtypes = [vp, i, i]
        L.mla_workspace_init.restype = i
        L.mla_workspace_init.argtypes = [vp, sz, vp]
        L.mla_read_device_flag.restype = i
        L.mla_read_device_flag.argtypes = [vp, ctypes.POINTER(i), vp]
        L.mla_clear_device_flag.restype = i
        L.mla_clear_device_flag.argtypes = [vp, vp]
        L.mla_rope_cos_sin.restype = i
        L.mla_rope_cos_sin.argtypes = [vp, i, i, ctypes.c_double, vp, vp, vp]
        L.mla_decode_qkv.restype = i
        L.mla_decode_qkv.argtypes = [vp, vp, i, vp, vp, vp, i, vp, vp, vp, vp, vp, sz, vp]
        L.mla_decode_attn.restype = i
        L.mla_decode_attn.argtypes = [vp, vp, vp, vp, i, vp, i, vp, i, i, vp, vp, vp, sz, vp]
        L.mla_prefill.restype = i
        L.mla_prefill.argtypes = [vp, vp, i, vp, vp, vp, vp, vp, i, vp, vp, sz, vp]
        L.mla_v4_qkv.restype = i
        L.mla_v4_qkv.argtypes = [vp, vp, i, vp, vp, vp, vp, vp, vp, sz, vp]
        L.mla_strerror.restype = ctypes.c_char_p
        L.mla_strerror.argtypes = [i]
        L.mla_kernel_launch_count.restype = ctypes.c_uint64
        L.mla_kernel_launch_count.argtypes = []
        L.mla_set_kernel_timer.restype = i
        L.mla_decode_qkv_noalloc.restype = i
        L.mla_decode_qkv_noalloc.argtypes = [vp, vp, i, vp, vp, vp, i, vp, vp, vp, vp]
        L.mla_noalloc_read_device_flag.restype = i
        L.mla_noalloc_read_device_flag.argtypes = [ctypes.POINTER(i), vp]
        L.mla_set_kernel_timer.argtypes = [ctypes.c_char_p, vp, vp]
        L.mla_rope_cos_sin_inv_freq.restype = i
        L.mla_rope_cos_sin_inv_freq.argtypes = [vp, i, i, vp, vp, vp, vp]
        L.mla_decode_step_host_bytes.restype = sz
        L.mla_decode_step_host_bytes.argtypes = [vp, i, i]
        L.mla_decode_step_host.restype = i
        L.mla_decode_step_host.argtypes = [vp, vp, vp, vp, vp, i, vp, i, i, ctypes.c_double, vp, i, vp, vp, sz,
                                           vp, sz, vp]
        _lib = L
    return _lib


def mla_strerror(status: int) -> str:
    return lib().mla_strerror(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def make_config(shape, row_layout: int = MLA_ROW_LATENT_FIRST, softmax_scale: float = 0.0) -> mla_config:
    """mla_config from a workloads.MlaShape-like object."""
    dt = {"f32": MLA_F32, "bf16": MLA_BF16, "fp8": MLA_FP8_E4M3_B128}
    return mla_config(shape.hidden, shape.n_heads, shape.q_lora_rank, shape.kv_lora_rank,
                      shape.qk_nope, shape.qk_rope, shape.v_dim, shape.block_size,
                      shape.norm_eps, softmax_scale, dt[shape.act_dtype], dt[shape.weight_dtype],
                      row_layout, getattr(shape, "o_groups", 0), getattr(shape, "o_lora_rank", 0))


def mla_weights_bytes(cfg: mla_config) -> int:
    return int(lib().mla_weights_bytes(ctypes.byref(cfg)))


def mla_init_weights(cfg: mla_config, weights: dict, dst: torch.Tensor, stream=None) -> int:
    """weights: name -> device tensor (wq_a, wq_b, wkv_a, wkv_b, wo or wo_a + wo_b, q_norm_w,
    kv_norm_w, *_scale for FP8, optional attn_sink [H] fp32). Returns the opaque handle (int)."""
    d = mla_weights_desc(*[_ptr(weights.get(n)) for n in (
        "wq_a", "wq_b", "wkv_a", "wkv_b", "wo", "q_norm_w", "kv_norm_w", "wq_a_scale",
        "wq_b_scale", "wkv_a_scale", "wkv_b_scale", "wo_scale", "attn_sink", "wo_a", "wo_b")])
    h = ctypes.c_void_p()
    _check(lib().mla_init_weights(ctypes.byref(cfg), ctypes.byref(d), _ptr(dst), _nbytes(dst),
                                  _stream(stream), ctypes.byref(h)), "mla_init_weights")
    return h.value


def mla_destroy(handle: int) -> None:
    lib().mla_destroy(handle)


def mla_workspace_bytes(handle: int, max_tokens: int, max_context_len: int) -> int:
    return int(lib().mla_workspace_bytes(handle, int(max_tokens), int(max_context_len)))


def mla_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib().mla_workspace_init(_ptr(ws), _nbytes(ws), _stream(stream)), "mla_workspace_init")


def mla_read_device_flag(ws: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int(0)
    st = lib().mla_read_device_flag(_ptr(ws), ctypes.byref(v), _stream(stream))
    if st not in (MLA_OK, MLA_ERR_DEVICE_FLAG):
        _check(st, "mla_read_device_flag")
    return v.value


def mla_clear_device_flag(ws: torch.Tensor, stream=None) -> None:
    _check(lib().mla_clear_device_flag(_ptr(ws), _stream(stream)), "mla_clear_device_flag")


def mla_rope_cos_sin(positions: torch.Tensor, qk_rope: int, theta: float, cos: torch.Tensor,
                     sin: torch.Tensor, stream=None) -> None:
    _check(lib().mla_rope_cos_sin(_ptr(positions), positions.numel(), qk_rope, float(theta),
                                  _ptr(cos), _ptr(sin), _stream(stream)), "mla_rope_cos_sin")


def mla_rope_cos_sin_inv_freq(positions: torch.Tensor, qk_rope: int, inv_freq: torch.Tensor, cos: torch.Tensor,
                              sin: torch.Tensor, stream=None) -> None:
    """RoPE tables from a precomputed frequency table (e.g. YaRN's) [qk_rope/2] fp32."""
    _check(lib().mla_rope_cos_sin_inv_freq(_ptr(positions), positions.numel(), qk_rope, _ptr(inv_freq),
                                           _ptr(cos), _ptr(sin), _stream(stream)), "mla_rope_cos_sin_inv_freq")


def mla_decode_qkv(handle, hidden, cos, sin, kv_cache, slot_mapping, q_abs, q_pe, ws,
                   input_norm_w=None, stream=None) -> None:
    n = hidden.shape[0]
    _check(lib().mla_decode_qkv(handle, _ptr(hidden), n, _ptr(cos), _ptr(sin), _ptr(kv_cache),
                                kv_cache.shape[0], _ptr(slot_mapping), _ptr(q_abs), _ptr(q_pe),
                                _ptr(input_norm_w), _ptr(ws), _nbytes(ws), _stream(stream)),
           "mla_decode_qkv")


def mla_decode_qkv_noalloc(handle, hidden, cos, sin, kv_cache, slot_mapping, q_abs, q_pe,
                           stream=None) -> None:
    """mla_decode_qkv with the library's own fixed device scratch instead of a
    caller workspace (for callers that cannot allocate)."""
    n = hidden.shape[0]
    _check(lib().mla_decode_qkv_noalloc(handle, _ptr(hidden), n, _ptr(cos), _ptr(sin), _ptr(kv_cache),
                                        kv_cache.shape[0], _ptr(slot_mapping), _ptr(q_abs), _ptr(q_pe),
                                        _stream(stream)), "mla_decode_qkv_noalloc")


def mla_noalloc_read_device_flag(stream=None) -> int:
    """Device flag of the last mla_decode_qkv_noalloc call on the current device
    (synchronises the stream); 0 when that call met no bad slot or timeout."""
    v = ctypes.c_int(0)
    st = lib().mla_noalloc_read_device_flag(ctypes.byref(v), _stream(stream))
    if st not in (MLA_OK, MLA_ERR_DEVICE_FLAG):
        _check(st, "mla_noalloc_read_device_flag")
    return v.value


def mla_decode_attn(handle, q_abs, q_pe, kv_cache, block_table, context_lens, max_context_len,
                    out, ws, head_out=None, stream=None) -> None:
    n = q_abs.shape[0]
    _check(lib().mla_decode_attn(handle, _ptr(q_abs), _ptr(q_pe), _ptr(kv_cache), kv_cache.shape[0],
                                 _ptr(block_table), block_table.shape[1], _ptr(context_lens),
                                 int(max_context_len), n, _ptr(out), _ptr(head_out), _ptr(ws),
                                 _nbytes(ws), _stream(stream)), "mla_decode_attn")


def mla_decode_step_host_bytes(handle, n: int, max_blocks_per_seq: int) -> int:
    return int(lib().mla_decode_step_host_bytes(handle, int(n), int(max_blocks_per_seq)))


def mla_decode_step_host(handle, hidden, positions, slot_mapping, block_table, context_lens,
                         max_context_len, rope_theta, kv_cache, out, stage, ws, stream=None) -> None:
    """One decode step whose inputs (hidden, positions, slot_mapping,
    block_table, context_lens) and result (out) are host tensors, pinned for
    asynchronous copies; kv_cache, stage and ws are device tensors. Enqueued on
    the stream: synchronise it before reading out."""
    for t in (hidden, positions, slot_mapping, block_table, context_lens, out):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("mla_decode_step_host: inputs and out must be contiguous host tensors")
    n = hidden.shape[0]
    _check(lib().mla_decode_step_host(handle, _ptr(hidden), _ptr(positions), _ptr(slot_mapping),
                                      _ptr(block_table), block_table.shape[1], _ptr(context_lens),
                                      int(max_context_len), n, float(rope_theta), _ptr(kv_cache),
                                      kv_cache.shape[0], _ptr(out), _ptr(stage), _nbytes(stage), _ptr(ws),
                                      _nbytes(ws), _stream(stream)), "mla_decode_step_host")


def mla_prefill(handle, hidden, cos, sin, out, ws, head_out=None, kv_cache=None,
                slot_mapping=None, stream=None) -> None:
    S = hidden.shape[0]
    _check(lib().mla_prefill(handle, _ptr(hidden), S, _ptr(cos), _ptr(sin), _ptr(out),
                             _ptr(head_out), _ptr(kv_cache),
                             kv_cache.shape[0] if kv_cache is not None else 0,
                             _ptr(slot_mapping), _ptr(ws), _nbytes(ws), _stream(stream)),
           "mla_prefill")


def mla_v4_qkv(handle, hidden, cos, sin, kv_norm_w, q_out, kv_out, ws, stream=None) -> None:
    """DeepSeek-V4 QKV projection (see include/mla.h): q_out [S, H, d_n + d_r],
    kv_out [S, r_kv + d_r]."""
    S = hidden.shape[0]
    _check(lib().mla_v4_qkv(handle, _ptr(hidden), S, _ptr(cos), _ptr(sin), _ptr(kv_norm_w), _ptr(q_out),
                            _ptr(kv_out), _ptr(ws), _nbytes(ws), _stream(stream)), "mla_v4_qkv")


def mla_kernel_launch_count() -> int:
    return int(lib().mla_kernel_launch_count())


def mla_set_kernel_timer(kernel: str | None, start=None, stop=None) -> None:
    """Bracket every launch of `kernel` with records of two torch.cuda.Event
    (enable_timing=True); None clears the timer."""
    if kernel is None:
        _check(lib().mla_set_kernel_timer(None, None, None), "mla_set_kernel_timer")
        return
    _check(lib().mla_set_kernel_timer(kernel.encode(), start.cuda_event, stop.cuda_event),
           "mla_set_kernel_timer")
