/*
 * mla.h -- C-ABI of a B200 (sm_100a) implementation of one DeepSeek-style
 * Multi-head Latent Attention (MLA) layer step: the decode front-fold, the
 * absorbed decode attention over a paged latent cache, and the expanded
 * causal prefill.
 *
 * Conventions shared by every entry point
 *   - Every call returns int: MLA_OK (0) or a negative MLA_ERR_* code;
 *     mla_strerror() names it. On an error return nothing was launched.
 *   - Pointers named "device" must be device memory on the current device;
 *     "host" pointers are host memory. All device work is enqueued,
 *     asynchronously, on `stream` (a cudaStream_t; NULL = legacy default).
 *   - The library never allocates device memory. The caller owns every
 *     buffer: weights blob, workspace, KV cache, inputs and outputs.
 *     mla_init_weights() allocates one small host-side handle.
 *   - Matrices are row-major. Weights are given in [in, out] form (y = x @ W),
 *     as the pages give them ("MLA Decode QKV Kernel API Reference",
 *     Parameters; "QKV CTE MLA Kernel API Reference", qkv_mla_mx parameters).
 *   - Activation dtype (MLA_F32 or MLA_BF16) applies to hidden states,
 *     q_abs / q_pe, the KV cache, head_out and out. RoPE tables and RMSNorm
 *     gammas are always fp32.
 *   - Content errors that only the device can see (a slot or block id out of
 *     range, a context length out of range) set bits of a sticky int32 flag in
 *     the workspace; the offending write or row is skipped. Read the flag with
 *     mla_read_device_flag() and clear it with mla_clear_device_flag().
 *
 * Notation: n tokens, H heads, hidden D, q_lora_rank r_q, kv_lora_rank r_kv,
 * qk_nope d_n, qk_rope d_r, v_dim d_v, R = r_kv + d_r (cache row width).
 */
#ifndef MLA_B200_MLA_H_
#define MLA_B200_MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define MLA_OK 0
#define MLA_ERR_INVALID_ARG (-1)   /* bad pointer, size, shape or enum value */
#define MLA_ERR_UNSUPPORTED (-2)   /* valid request this library does not implement */
#define MLA_ERR_CUDA (-3)          /* a CUDA runtime call or launch failed */
#define MLA_ERR_DEVICE_FLAG (-4)   /* the device flag is non-zero (see below) */
#define MLA_ERR_WORKSPACE (-5)     /* workspace / weights buffer too small */

/* Device flag bits (sticky, OR-ed by kernels). */
#define MLA_FLAG_BAD_SLOT 1        /* slot_mapping[t] >= n_blocks * block_size */
#define MLA_FLAG_BAD_BLOCK 2       /* block_table entry outside [0, n_blocks) */
#define MLA_FLAG_BAD_CONTEXT 4     /* context_lens[t] < 1 or > max_context_len */
#define MLA_FLAG_WAIT_TIMEOUT 8    /* a bounded device-side wait gave up */

/* ---- configuration ----------------------------------------------------- */
typedef enum {
  MLA_F32 = 0,
  MLA_BF16 = 1,
  /* FP8-E4M3 (OCP) codes, one byte per weight, with fp32 scales per 128x128
   * block: W[k][n] = e4m3(code[k][n]) * scale[k/128][n/128], scale tensor
   * [ceil(in/128), ceil(out/128)] row-major. "Struct MlaWeights", field
   * wq_a_fp8 (128x128 block scales, dequantised in fp32 before the MAC with
   * bf16 activations); scale shape as "QKV CTE MLA Kernel API Reference",
   * *_scale_hbm. Weights only; needs act_dtype MLA_BF16. */
  MLA_FP8_E4M3_B128 = 2
} mla_dtype;

typedef enum {
  /* cache row = [latent (r_kv) | k_pe (d_r)], DeepSeek's order */
  MLA_ROW_LATENT_FIRST = 0,
  /* cache row = [k_pe (d_r) | latent (r_kv)], the inverted order of
   * "MLA Decode QKV Kernel API Reference", Notes */
  MLA_ROW_PE_FIRST = 1
} mla_row_layout;

/* Layer shape ("struct Mla" fields; "MLA Decode QKV Kernel API Reference",
 * Dimensions). Limits of this library: d_r even; r_kv, d_n, d_v, d_r, D and
 * H*(d_n+d_r) multiples of 8 (16-byte rows); for MLA_FP8_E4M3_B128 also
 * r_q, d_n, d_v, H*(d_n+d_r) multiples of 128. */
typedef struct {
  int hidden;          /* D */
  int n_heads;         /* H */
  int q_lora_rank;     /* r_q; 0 = one full query projection x @ q_proj */
  int kv_lora_rank;    /* r_kv */
  int qk_nope;         /* d_n: per-head query/key dims RoPE does not rotate */
  int qk_rope;         /* d_r: per-head dims RoPE rotates (the trailing ones) */
  int v_dim;           /* d_v */
  int block_size;      /* rows per paged-cache block */
  float norm_eps;      /* RMSNorm epsilon ("... norm_eps", default 1e-6) */
  float softmax_scale; /* 0 => 1/sqrt(d_n + d_r) ("struct Mla", field scale) */
  int act_dtype;       /* mla_dtype: MLA_F32 or MLA_BF16 */
  int weight_dtype;    /* mla_dtype: must equal act_dtype, or MLA_FP8_E4M3_B128 */
  int row_layout;      /* mla_row_layout */
  /* DeepSeek-V4 grouped low-rank output projection ("Struct MlaWeights",
   * wo_a / wo_b / o_lora_rank: when o_lora_rank > 0 the decode and prefill
   * paths use wo_a -> wo_b instead of wo; wo_a is sliced per o_group,
   * block-diagonal). 0 / 0 = the dense wo. With o_lora_rank > 0: o_groups >= 1
   * divides H; o_lora_rank and (H / o_groups) * d_v are multiples of 64; the
   * weights are MLA_F32 or MLA_BF16. */
  int o_groups;        /* G: consecutive head groups */
  int o_lora_rank;     /* r_o: each group's low rank */
} mla_config;

/* Weights in [in, out] row-major form, device pointers, element type
 * weight_dtype (uint8 codes for FP8). Only read during mla_init_weights().
 *   wq_a  [D, r_q]                  (NULL when q_lora_rank == 0)
 *   wq_b  [r_q, H*(d_n+d_r)]        or, when q_lora_rank == 0, the full
 *                                   q_proj [D, H*(d_n+d_r)]
 *   wkv_a [D, r_kv + d_r]           output order [latent | k_pe]
 *   wkv_b [r_kv, H*(d_n+d_v)]       per head [k_nope_h | v_h] columns
 *   wo    [H*d_v, D]                (NULL when o_lora_rank > 0)
 *   wo_a  [H*d_v, r_o]              o_lora_rank > 0 only: group g's block
 *                                   [(H/G) d_v, r_o] in rows g (H/G) d_v ..;
 *                                   it takes heads g (H/G) .. (g+1) (H/G) - 1
 *   wo_b  [G*r_o, D]                o_lora_rank > 0 only: the groups' low-rank
 *                                   outputs, concatenated in group order, -> D
 *   q_norm_w [r_q] fp32 (NULL when q_lora_rank == 0), kv_norm_w [r_kv] fp32
 *   *_scale: FP8 only, fp32 [ceil(in/128), ceil(out/128)], else NULL.
 *   attn_sink [H] fp32 or NULL: a per-head attention sink logit ("Struct
 *            MlaWeights", attn_sink, DeepSeek-V4 s_aux; a bf16 checkpoint
 *            value converts to fp32 exactly). When set, every softmax of
 *            mla_decode_attn and mla_prefill takes it as one more column in
 *            the units of the scaled scores that carries no value:
 *            p_j = e^{s_j} / (sum_k e^{s_k} + e^{attn_sink[h]}). */
typedef struct {
  const void* wq_a;
  const void* wq_b;
  const void* wkv_a;
  const void* wkv_b;
  const void* wo;
  const float* q_norm_w;
  const float* kv_norm_w;
  const float* wq_a_scale;
  const float* wq_b_scale;
  const float* wkv_a_scale;
  const float* wkv_b_scale;
  const float* wo_scale;
  const float* attn_sink;
  const void* wo_a;
  const void* wo_b;
} mla_weights_desc;

typedef struct mla_handle mla_handle;

/* ---- weights ------------------------------------------------------------ */

/* Bytes of the library's repacked weight blob for `cfg` (0 if cfg is invalid). */
size_t mla_weights_bytes(const mla_config* cfg);

/* Validate cfg, repack the weights into `dst` (device, >= mla_weights_bytes,
 * 256-byte aligned, owned by the caller and kept alive while the handle is
 * used), enqueue the repack on `stream`, and return a host handle in *out.
 * The repack merges [wq_a | wkv_a] into one first projection ("Struct
 * MlaWeights", wkv_a_merged; "QKV CTE MLA Kernel API Reference", Combined Q/KV
 * Path Stage 1) and slices wkv_b into W_UK [H, d_n, r_kv] and W_UV
 * [H, r_kv, d_v] ("Struct MlaWeights", w_uk_t and w_uv). The source weights
 * may be freed once the stream has passed the repack. */
int mla_init_weights(const mla_config* cfg, const mla_weights_desc* w, void* dst,
                     size_t dst_bytes, void* stream, mla_handle** out);

/* Release the host handle (not `dst`). NULL is ignored. */
void mla_destroy(mla_handle* h);

/* ---- workspace ------------------------------------------------------------ */

/* Bytes of device workspace the calls below need for up to `max_tokens`
 * decode tokens (or prefill sequence length) and contexts of up to
 * `max_context_len` rows. For FP8 weights this includes one bf16 buffer of
 * the largest weight, into which mla_prefill dequantises each weight in turn
 * (the decode calls never use it and accept a workspace without it). */
size_t mla_workspace_bytes(const mla_handle* h, int max_tokens, int max_context_len);

/* Zero the workspace (device flag and internal counters). Call once on a new
 * workspace before its first use; the library keeps it consistent afterwards. */
int mla_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Copy the device flag to *flag_out (synchronises `stream`). Returns
 * MLA_ERR_DEVICE_FLAG when it is non-zero, MLA_OK otherwise. */
int mla_read_device_flag(const void* ws, int* flag_out, void* stream);
int mla_clear_device_flag(void* ws, void* stream);

/* ---- RoPE tables ---------------------------------------------------------- */

/* cos/sin [n, d_r/2] fp32 (device) of positions[n] (device int32):
 * angle_i = pos * theta^(-2i/d_r), evaluated in fp64 on the device and
 * rounded once to fp32. Half width as "MLA Decode QKV Kernel API Reference",
 * Parameters (cos, sin: [n_tokens, qk_rope_dim // 2]). */
int mla_rope_cos_sin(const int32_t* positions, int n, int qk_rope, double theta,
                     float* cos_out, float* sin_out, void* stream);

/* The same tables from a precomputed frequency table: angle_i = pos *
 * inv_freq[i], evaluated in fp64 and rounded once to fp32. This is how a YaRN
 * (or any other) frequency scaling enters ("Struct MlaWeights", yarn_inv_freq:
 * a precomputed [rotary_dim/2] fp32 table; NULL there selects the plain theta
 * computation, mla_rope_cos_sin here). YaRN's magnitude correction enters the
 * score scale, mla_config.softmax_scale ("struct Mla", scale).
 * inv_freq device [qk_rope/2] fp32; positions, cos_out, sin_out as above. */
int mla_rope_cos_sin_inv_freq(const int32_t* positions, int n, int qk_rope, const float* inv_freq,
                              float* cos_out, float* sin_out, void* stream);

/* ---- decode ----------------------------------------------------------------- */

/* The decode front-fold ("MLA Decode QKV Kernel API Reference",
 * mla_decode_qkv): for each of n tokens (one per sequence)
 *   q_lat = x @ wq_a; q = rms_norm(q_lat, q_norm_w) @ wq_b  (or x @ q_proj)
 *   q_pe  = RoPE(q[h, d_n:]) per head, interleaved pairs (2i, 2i+1)
 *   q_abs[h] = q[h, :d_n] @ W_UK[h]
 *   kv = x @ wkv_a; c = rms_norm(kv[:r_kv], kv_norm_w); k_pe = RoPE(kv[r_kv:])
 *   kv_cache row slot_mapping[t] = [c | k_pe] (or [k_pe | c], per row_layout)
 * hidden      device [n, D] act dtype
 * cos, sin    device [n, d_r/2] fp32, the token's position (mla_rope_cos_sin)
 * kv_cache    device [n_blocks, 1, block_size, R] act dtype, mutated in place
 * slot_mapping device [n] int32 flat row (block * block_size + offset);
 *             negative = skip the token's write; >= n_blocks*block_size sets
 *             MLA_FLAG_BAD_SLOT and skips. Slots must be distinct.
 * q_abs       device [n, H, r_kv] act dtype (output)
 * q_pe        device [n, H, d_r] act dtype (output)
 * input_norm_w device [D] fp32, or NULL. When given, the layer's input
 *             RMSNorm is applied first: x <- x * rsqrt(mean(x^2) + norm_eps) *
 *             input_norm_w, rounded to the activation dtype ("MLA Decode QKV
 *             Kernel API Reference", input_norm_w: folded into the hidden load).
 * ws          device workspace (mla_workspace_bytes with max_tokens >= n). */
int mla_decode_qkv(mla_handle* h, const void* hidden, int n, const float* cos,
                   const float* sin, void* kv_cache, int n_blocks,
                   const int32_t* slot_mapping, void* q_abs, void* q_pe,
                   const float* input_norm_w, void* ws, size_t ws_bytes, void* stream);

/* Absorbed decode attention, V extraction and o_proj ("Struct MlaWeights",
 * w_uk_t / w_uv / wo; "struct Mla", scale): for token t (sequence t) with
 * L = context_lens[t] cached rows at positions 0..L-1,
 *   s[h, j] = (q_abs[h] . c_j + q_pe[h] . k_pe_j) * softmax_scale
 *   o_lat[h] = softmax_j(s[h]) @ c;  head_out[h] = o_lat[h] @ W_UV[h]
 *   out = concat_h(head_out[h]) @ wo
 * Row j of sequence t is flat cache row block_table[t][j / bs] * bs + j % bs.
 * q_abs, q_pe    device, as written by mla_decode_qkv
 * kv_cache       device [n_blocks, 1, bs, R] act dtype (read only)
 * block_table    device [n, max_blocks_per_seq] int32
 * context_lens   device [n] int32, 1 <= L <= max_context_len (includes this
 *                step's token, which mla_decode_qkv wrote at position L-1)
 * max_context_len host int, an upper bound on every context_lens[t]
 * out            device [n, D] act dtype
 * head_out       device [n, H, d_v] act dtype, or NULL
 * Must follow mla_decode_qkv on the same stream when both are used for one
 * step (the scatter writes the row attention reads). */
int mla_decode_attn(mla_handle* h, const void* q_abs, const void* q_pe,
                    const void* kv_cache, int n_blocks, const int32_t* block_table,
                    int max_blocks_per_seq, const int32_t* context_lens,
                    int max_context_len, int n, void* out, void* head_out, void* ws,
                    size_t ws_bytes, void* stream);

/* Size of the device array mla_decode_qkv_noalloc() uses as its workspace. */
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* mla_decode_qkv without a workspace argument and without allocating: for
 * callers that cannot allocate device memory -- a process whose device memory
 * is entirely reserved up front by its own pool allocator, or a serving loop
 * that must not call cudaMalloc because it synchronises the device and stalls
 * every stream. (The pages have no counterpart; this is a library convenience.)
 * Same computation, arguments and results as mla_decode_qkv (input_norm_w is
 * taken as NULL); the scratch is a static device array of
 * MLA_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the
 * process exits. The array's device memory is taken when the library first
 * looks up its address (cudaGetSymbolAddress) on a device, with that device
 * current: mla_init_weights does so for its device, so the memory is committed
 * when the first handle is created; if that lookup failed, the first call
 * here repeats it, so make that first call before any stream capture.
 * Returns MLA_ERR_WORKSPACE when the front-fold's workspace for n tokens
 * exceeds the array (for the DeepSeek-V3 shape that allows about 64 tokens
 * per call). All calls share the one array, whose contents persist between
 * calls: each call clears the device flag it holds before its kernels run
 * (read it with mla_noalloc_read_device_flag), and calls that overlap on the
 * GPU, on any streams, race. Calls no cudaMalloc, cudaFree or allocating
 * routine. */
int mla_decode_qkv_noalloc(mla_handle* h, const void* hidden, int n, const float* cos,
                           const float* sin, void* kv_cache, int n_blocks,
                           const int32_t* slot_mapping, void* q_abs, void* q_pe, void* stream);

/* The device flag of the last mla_decode_qkv_noalloc call on the current
 * device (bad slot: that row was not written; wait timeout: q_abs / q_pe are
 * incomplete), copied to *flag_out after synchronising `stream`. Returns
 * MLA_ERR_DEVICE_FLAG when it is non-zero, MLA_OK otherwise. */
int mla_noalloc_read_device_flag(int* flag_out, void* stream);

/* ---- one decode step from host memory ------------------------------------------ */

/* Device bytes of the `stage` buffer mla_decode_step_host() needs for n tokens
 * and block tables of max_blocks_per_seq entries: the step's inputs copied in,
 * the cos/sin tables, q_abs, q_pe and out. 0 on invalid arguments. */
size_t mla_decode_step_host_bytes(const mla_handle* h, int n, int max_blocks_per_seq);

/* One whole decode step with its inputs and result in host memory: copies
 * hidden, positions, slot_mapping, block_table and context_lens to the
 * device, then runs mla_rope_cos_sin, mla_decode_qkv and mla_decode_attn (the
 * same computation, arguments and results as those calls) and copies out back,
 * all enqueued on `stream`. Returns once enqueued: synchronise `stream` before
 * reading out_host. Host buffers should be page-locked (cudaHostAlloc, or
 * torch's pin_memory) for the copies to run asynchronously; pageable memory
 * gives the same results with blocking copies.
 * hidden_host        host [n, D] act dtype
 * positions_host     host [n] int32 (the position each token's RoPE uses)
 * slot_mapping_host  host [n] int32, as in mla_decode_qkv
 * block_table_host   host [n, max_blocks_per_seq] int32, as in mla_decode_attn
 * context_lens_host  host [n] int32, as in mla_decode_attn
 * rope_theta         RoPE base, as in mla_rope_cos_sin
 * kv_cache           device, as in mla_decode_qkv (mutated in place)
 * out_host           host [n, D] act dtype (written when the stream reaches it)
 * stage              device buffer of mla_decode_step_host_bytes(h, n,
 *                    max_blocks_per_seq) bytes, owned by the caller
 * ws                 device workspace of mla_workspace_bytes(h, n, max_context_len)
 * The four int32 arrays are packed on the host into one page-locked buffer
 * the handle owns (allocated on the first call, regrown when a call needs
 * more, freed by mla_destroy) and copied in one transfer; a call first waits
 * for the previous call's transfer out of that buffer. */
int mla_decode_step_host(mla_handle* h, const void* hidden_host, const int32_t* positions_host,
                         const int32_t* slot_mapping_host, const int32_t* block_table_host,
                         int max_blocks_per_seq, const int32_t* context_lens_host,
                         int max_context_len, int n, double rope_theta, void* kv_cache,
                         int n_blocks, void* out_host, void* stage, size_t stage_bytes, void* ws,
                         size_t ws_bytes, void* stream);

/* ---- prefill ------------------------------------------------------------------ */

/* Causal prefill (context encoding) of one sequence of S tokens at positions
 * 0..S-1 with K/V expanded from the latent ("QKV CTE MLA Kernel API
 * Reference", qkv_mla_mx: Stage 1 x @ [wq_a | wkv_a]; Q Stage 2; KV Stage 2
 * norm(kv) @ wkv_b split into k_nope, v; RoPE on q_pe and k_pe, k_pe
 * broadcast to every head), then softmax(Q K^T * scale) V with query i seeing
 * keys j <= i, and o_proj.
 * hidden   device [S, D] act dtype; cos, sin device [S, d_r/2] fp32
 * out      device [S, D] act dtype; head_out device [S, H, d_v] or NULL
 * kv_cache / slot_mapping: optional (both NULL or both set): the sequence's
 *          cache rows are scattered as in mla_decode_qkv. */
int mla_prefill(mla_handle* h, const void* hidden, int S, const float* cos,
                const float* sin, void* out, void* head_out, void* kv_cache,
                int n_blocks, const int32_t* slot_mapping, void* ws, size_t ws_bytes,
                void* stream);

/* ---- DeepSeek-V4 QKV projection ---------------------------------------------------- */

/* The DeepSeek-V4 form of the QKV projection ("QKV CTE MLA Kernel API
 * Reference", qkv_mla_mx_deepseek_v4), on the handle's [wq_a | wkv_a] (the
 * fused first projection wqkv [D, r_q + kv_dim], kv_dim = r_kv + d_r),
 * q_norm_w and wq_b (wkv_b and wo are not used):
 *   qr, kv = split(x @ wqkv)
 *   q      = RMSNorm(qr, q_norm_w) @ wq_b, viewed [S, H, hd] (hd = d_n + d_r)
 *   q_h    = q_h / sqrt(mean(q_h^2) + norm_eps)       (per head, no gain)
 *   q_h[hd - d_r:]   rotated by interleaved RoPE at the token's position
 *   kv     = RMSNorm(kv, kv_norm_w) over all kv_dim columns
 *   kv[kv_dim - d_r:] rotated by interleaved RoPE
 * for S tokens with their own cos/sin rows (any positions).
 * hidden     device [S, D] act dtype; cos, sin device [S, d_r/2] fp32
 * kv_norm_w  device [r_kv + d_r] fp32 (the V4 kv gamma covers the whole row)
 * q_out      device [S, H, hd] act dtype; kv_out device [S, r_kv + d_r] act
 *            dtype ([latent | rotated tail], the form of a cache row)
 * ws         device workspace of mla_workspace_bytes(h, S, 1)
 * Needs q_lora_rank > 0 (MLA_ERR_UNSUPPORTED otherwise). Readings where the
 * page is brief: the per-head norm is the RMS form with norm_eps; RoPE is the
 * interleaved pairing of the decode kernel. */
int mla_v4_qkv(mla_handle* h, const void* hidden, int S, const float* cos, const float* sin,
               const float* kv_norm_w, void* q_out, void* kv_out, void* ws, size_t ws_bytes,
               void* stream);

/* ---- misc ------------------------------------------------------------------------ */

const char* mla_strerror(int status);

/* Launches of the library's own kernels since load (all entry points). */
uint64_t mla_kernel_launch_count(void);

/* Kernel timer (tracing). While set, every launch of the library kernel named
 * `kernel` is bracketed by records of the two events (cudaEvent_t, created by
 * the caller with timing enabled) on the launch stream, so that
 * cudaEventElapsedTime(start, stop) is that kernel's device time. Names:
 * "attn" (decode attention), "prefill_attn", and the decode weight GEMMs
 * "gemm_w1" (down-projection), "gemm_qb" (wq_b), "gemm_uk" (absorption),
 * "gemm_uv" (V extraction), "gemm_o" (o_proj), each including the operand
 * conversion or weight dequantisation it launches, and "v4_qb" (the wq_b GEMM
 * of mla_v4_qkv on tensor cores). NULL clears the timer. Inside a
 * stream capture the records become external event-record nodes of the graph.
 * Process-wide; not thread-safe against concurrent launches. */
int mla_set_kernel_timer(const char* kernel, void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_MLA_H_ */
