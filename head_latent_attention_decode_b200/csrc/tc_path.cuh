// Tensor-core (tcgen05 / TMEM / TMA) path of the MLA layer step for bf16
// activations with bf16 or FP8 weights.
#pragma once

#include "handle.cuh"

static inline size_t tc_decode_ws_bytes(const mla_handle*, long long, int) { return 0; }
static inline int tc_init(mla_handle* h) { h->tc.enabled = 0; return MLA_OK; }
static inline bool tc_decode_qkv_supported(const mla_handle*, int) { return false; }
static inline bool tc_decode_attn_supported(const mla_handle*, int, int) { return false; }
static inline bool tc_prefill_supported(const mla_handle*, int) { return false; }
static inline int tc_decode_qkv(const mla_handle*, const void*, int, const float*, const float*, void*, int,
                                const int32_t*, void*, void*, char*, size_t, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
static inline int tc_decode_attn(const mla_handle*, const void*, const void*, const void*, int, const int32_t*,
                                 int, const int32_t*, int, int, void*, void*, char*, size_t, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
static inline int tc_prefill(const mla_handle*, const void*, int, const float*, const float*, void*, void*, void*,
                             int, const int32_t*, char*, size_t, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
