// C-ABI of the MLA layer step (include/mla.h): argument validation, the
// repacked weight layout, workspace layout, and the launch sequence of each
// entry point. Every step of the path runs in this library's kernels.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "common.cuh"
#include "simt_kernels.cuh"
#include "handle.cuh"
#include "tc_path.cuh"

using namespace mla;

static std::atomic<unsigned long long> g_launches{0};
void mla_count_launch(int k) { g_launches.fetch_add((unsigned long long)k); }
static inline void count_launch(int k = 1) { mla_count_launch(k); }

static char g_timer_kernel[32] = {0};
static cudaEvent_t g_timer_start = nullptr, g_timer_stop = nullptr;

static void timer_record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  if (cs == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  else cudaEventRecord(ev, s);
}
void mla_timer_begin(const char* k, cudaStream_t s) {
  if (g_timer_kernel[0] && strcmp(k, g_timer_kernel) == 0) timer_record(g_timer_start, s);
}
void mla_timer_end(const char* k, cudaStream_t s) {
  if (g_timer_kernel[0] && strcmp(k, g_timer_kernel) == 0) timer_record(g_timer_stop, s);
}


static int validate_config(const mla_config* c) {
  if (!c) return MLA_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->n_heads <= 0 || c->q_lora_rank < 0 || c->kv_lora_rank <= 0 ||
      c->qk_nope <= 0 || c->qk_rope <= 0 || c->v_dim <= 0 || c->block_size <= 0)
    return MLA_ERR_INVALID_ARG;
  if (c->qk_rope % 2) return MLA_ERR_INVALID_ARG;  // RoPE pairs ("qk_rope_dim ... Must be even")
  if (!(c->norm_eps >= 0.f) || !(c->softmax_scale >= 0.f)) return MLA_ERR_INVALID_ARG;
  if (c->act_dtype != MLA_F32 && c->act_dtype != MLA_BF16) return MLA_ERR_INVALID_ARG;
  if (c->weight_dtype != MLA_F32 && c->weight_dtype != MLA_BF16 && c->weight_dtype != MLA_FP8_E4M3_B128)
    return MLA_ERR_INVALID_ARG;
  if (c->row_layout != MLA_ROW_LATENT_FIRST && c->row_layout != MLA_ROW_PE_FIRST) return MLA_ERR_INVALID_ARG;
  if (c->weight_dtype == MLA_FP8_E4M3_B128) {
    if (c->act_dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  } else if (c->weight_dtype != c->act_dtype) {
    return MLA_ERR_UNSUPPORTED;
  }
  // the library's limits
  const long long Hq = (long long)c->n_heads * (c->qk_nope + c->qk_rope);
  if (c->kv_lora_rank % 32 || c->kv_lora_rank > 512) return MLA_ERR_UNSUPPORTED;
  if (c->v_dim % 32 || c->v_dim > 128) return MLA_ERR_UNSUPPORTED;
  if (c->qk_nope % 8 || c->qk_rope % 8 || c->hidden % 8 || c->q_lora_rank % 8) return MLA_ERR_UNSUPPORTED;
  if (c->qk_nope + c->qk_rope > 256) return MLA_ERR_UNSUPPORTED;
  if (c->weight_dtype == MLA_FP8_E4M3_B128) {
    if (c->q_lora_rank % 128 || c->qk_nope % 128 || c->v_dim % 128 || Hq % 128)
      return MLA_ERR_UNSUPPORTED;
  }
  // grouped low-rank output projection
  if (c->o_lora_rank < 0 || c->o_groups < 0) return MLA_ERR_INVALID_ARG;
  if (c->o_lora_rank > 0) {
    if (c->o_groups < 1 || c->n_heads % c->o_groups) return MLA_ERR_INVALID_ARG;
    if (c->weight_dtype == MLA_FP8_E4M3_B128) return MLA_ERR_UNSUPPORTED;
    if (c->o_lora_rank % 64 || ((long long)(c->n_heads / c->o_groups) * c->v_dim) % 64) return MLA_ERR_UNSUPPORTED;
  }
  return MLA_OK;
}

static size_t dtype_size(int dt) { return dt == MLA_F32 ? 4 : (dt == MLA_BF16 ? 2 : 1); }

static WeightLayout make_layout(const mla_config* c) {
  WeightLayout L{};
  const int H = c->n_heads, dn = c->qk_nope, dr = c->qk_rope, dv = c->v_dim, rkv = c->kv_lora_rank;
  const int D = c->hidden, rq = c->q_lora_rank;
  L.R = rkv + dr;
  L.Hq = H * (dn + dr);
  L.Hkv = H * (dn + dv);
  L.Nq1 = rq ? rq : L.Hq;
  L.N1 = L.Nq1 + L.R;
  L.esz = dtype_size(c->weight_dtype);
  const bool fp8 = c->weight_dtype == MLA_FP8_E4M3_B128;
  size_t off = 0;
  auto put = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  auto sblocks = [](long long n, long long k) { return (size_t)(cdiv(n, 128) * cdiv(k, 128)) * 4; };
  L.W1 = put((size_t)L.N1 * D * L.esz);
  L.Wqb = rq ? put((size_t)L.Hq * rq * L.esz) : 0;
  L.Wuk = put((size_t)H * rkv * dn * L.esz);
  L.Wuv = put((size_t)H * dv * rkv * L.esz);
  L.Wkvb = put((size_t)L.Hkv * rkv * L.esz);
  if (c->o_lora_rank > 0) {
    L.G = c->o_groups;
    L.ro = c->o_lora_rank;
    L.Kg = H / L.G * dv;
    L.Woa = put((size_t)L.G * L.ro * L.Kg * L.esz);
    L.Wob = put((size_t)D * L.G * L.ro * L.esz);
  } else {
    L.Wo = put((size_t)D * H * dv * L.esz);
  }
  L.gq = rq ? put((size_t)rq * 4) : 0;
  L.gkv = put((size_t)rkv * 4);
  L.sink = put((size_t)H * 4);
  if (fp8) {
    L.sW1 = put(sblocks(L.N1, D));
    L.sWqb = rq ? put(sblocks(L.Hq, rq)) : 0;
    L.sWuk = put(H * sblocks(rkv, dn));
    L.sWuv = put(H * sblocks(dv, rkv));
    L.sWkvb = put(sblocks(L.Hkv, rkv));
    L.sWo = put(sblocks(D, (long long)H * dv));
  }
  L.total = off;
  return L;
}

// ---------------------------------------------------------------------------
// workspace
// ---------------------------------------------------------------------------
// [0, 256): device flag (int32 at 0) and counters. Then decode and prefill
// scratch share one region (calls on one workspace are stream-ordered).
struct WsLayout {
  size_t Y1, qn, Q, part_o, part_ml, nseg, o_lat, head, xn, oy;   // decode
  size_t pY1, pqn, pQ, pcn, pkpe, pKV, phead, pDQ, poy;            // prefill
  size_t tc;                                                   // tensor-core path scratch
  size_t dec_total;                                            // what the decode calls need
  size_t total;                                                // what every call needs
  int splits;
};

static int decode_splits(int max_ctx) {
  const int c = (int)cdiv(max_ctx, 256);
  return c < 2 ? 2 : (c > 16 ? 16 : c);
}

static WsLayout make_ws(const mla_handle* h, long long n, int max_ctx) {
  const mla_config* c = &h->cfg;
  const WeightLayout& L = h->L;
  const size_t a = dtype_size(c->act_dtype);
  const int H = c->n_heads, rkv = c->kv_lora_rank, dv = c->v_dim, dr = c->qk_rope;
  WsLayout W{};
  W.splits = decode_splits(max_ctx);
  size_t off = 256;
  auto put = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  W.Y1 = put((size_t)n * L.N1 * 4);
  W.qn = put((size_t)n * (c->q_lora_rank ? c->q_lora_rank : 1) * a);
  W.Q = put((size_t)n * L.Hq * 4);
  W.part_o = put((size_t)n * W.splits * H * rkv * 4);
  W.part_ml = put((size_t)n * W.splits * H * 2 * 4 * 2);   // one (m, l) copy per CTA of a pair
  W.nseg = put((size_t)n * 4);                                // split partials per sequence
  W.o_lat = put((size_t)n * H * rkv * a);
  W.head = put((size_t)n * H * dv * a);
  W.xn = put((size_t)n * c->hidden * a);
  W.oy = put((size_t)n * (L.G ? L.G * L.ro : 1) * a);   // grouped output projection: the low-rank rows
  W.tc = put(tc_decode_ws_bytes(h, n, max_ctx));
  const size_t dec_end = off;
  W.dec_total = dec_end;
  off = 256;
  W.pY1 = put((size_t)n * L.N1 * 4);
  W.pqn = put((size_t)n * (c->q_lora_rank ? c->q_lora_rank : 1) * a);
  W.pQ = put((size_t)n * L.Hq * a);
  W.pcn = put((size_t)n * rkv * a);
  W.pkpe = put((size_t)n * dr * a);
  W.pKV = put((size_t)n * L.Hkv * a);
  W.phead = put((size_t)n * H * dv * a);
  W.poy = put((size_t)n * (L.G ? L.G * L.ro : 1) * a);
  W.pDQ = put(tc_prefill_dequant_bytes(h));   // FP8 weights: one dequantised weight at a time
  W.total = dec_end > off ? dec_end : off;
  return W;
}

// A runtime call returned an error: report it and clear the sticky copy.
static int cuda_fail() {
  cudaError_t e = cudaGetLastError();
  fprintf(stderr, "mla: CUDA error %s\n", cudaGetErrorString(e));
  return MLA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------
static int cuda_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "mla: CUDA error %s\n", cudaGetErrorString(e));
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

template <typename TA, typename TW, typename TC>
static void launch_linear_t(const LinearArgs& a, int batch, cudaStream_t st) {
  dim3 grid((unsigned)cdiv(a.N, LIN_BN), (unsigned)cdiv(a.M, LIN_BM), (unsigned)batch);
  linear_simt_kernel<TA, TW, TC><<<grid, 256, 0, st>>>(a);
  count_launch();
}

// dtype codes: 0 f32, 1 bf16, 2 fp8 (weights only)
static void launch_linear(int ta, int tw, int tc, const LinearArgs& a, int batch, cudaStream_t st) {
  if (a.M <= 0 || a.N <= 0) return;
#define MLA_LIN(TA_, TW_, TC_) launch_linear_t<TA_, TW_, TC_>(a, batch, st)
  if (ta == 0) {
    if (tw == 0) { if (tc == 0) MLA_LIN(float, float, float); else MLA_LIN(float, float, bf16); }
    else if (tw == 1) { if (tc == 0) MLA_LIN(float, bf16, float); else MLA_LIN(float, bf16, bf16); }
    else { if (tc == 0) MLA_LIN(float, uint8_t, float); else MLA_LIN(float, uint8_t, bf16); }
  } else {
    if (tw == 0) { if (tc == 0) MLA_LIN(bf16, float, float); else MLA_LIN(bf16, float, bf16); }
    else if (tw == 1) { if (tc == 0) MLA_LIN(bf16, bf16, float); else MLA_LIN(bf16, bf16, bf16); }
    else { if (tc == 0) MLA_LIN(bf16, uint8_t, float); else MLA_LIN(bf16, uint8_t, bf16); }
  }
#undef MLA_LIN
}

static LinearArgs lin(const void* A, long long lda, const void* W, long long ldw, const float* s,
                      long long lds, void* C, long long ldc, int M, int N, int K) {
  LinearArgs a{};
  a.A = A; a.lda = lda; a.W = W; a.ldw = ldw; a.scale = s; a.lds = lds; a.C = C; a.ldc = ldc;
  a.M = M; a.N = N; a.K = K;
  return a;
}

static void launch_o_proj_simt(const mla_handle* h, const void* head, void* out, void* y, long long n, cudaStream_t s) {
  const WeightLayout& L = h->L;
  const mla_config* c = &h->cfg;
  const int H = c->n_heads, dv = c->v_dim, D = c->hidden;
  const int ta = h->cfg.act_dtype == MLA_F32 ? 0 : 1;
  const int tw = h->cfg.weight_dtype == MLA_F32 ? 0 : (h->cfg.weight_dtype == MLA_BF16 ? 1 : 2);
  if (!L.G) {
    const float* sc = L.sWo ? (const float*)(h->base + L.sWo) : nullptr;
    launch_linear(ta, tw, ta, lin(head, (long long)H * dv, h->base + L.Wo, (long long)H * dv, sc,
                                  cdiv((long long)H * dv, 128), out, D, (int)n, D, H * dv), 1, s);
    return;
  }
  // y[:, g*r_o + j] = head[:, g*Kg .. (g+1)*Kg) @ wo_a block g; then out = y @ wo_b
  LinearArgs a = lin(head, (long long)H * dv, h->base + L.Woa, L.Kg, nullptr, 0, y, (long long)L.G * L.ro,
                     (int)n, L.ro, L.Kg);
  a.a_batch = L.Kg; a.w_batch = (long long)L.ro * L.Kg; a.c_batch = L.ro; a.s_batch = 0;
  launch_linear(ta, tw, ta, a, L.G, s);
  launch_linear(ta, tw, ta, lin(y, (long long)L.G * L.ro, h->base + L.Wob, (long long)L.G * L.ro, nullptr, 0, out, D,
                                (int)n, D, L.G * L.ro), 1, s);
}

template <typename K>
static void set_smem(K kernel, size_t bytes) {
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

static const float* wscale(const mla_handle* h, size_t off) {
  return h->cfg.weight_dtype == MLA_FP8_E4M3_B128 ? (const float*)(h->base + off) : nullptr;
}
static int wcode(const mla_handle* h) {
  return h->cfg.weight_dtype == MLA_F32 ? 0 : (h->cfg.weight_dtype == MLA_BF16 ? 1 : 2);
}
static int acode(const mla_handle* h) { return h->cfg.act_dtype == MLA_F32 ? 0 : 1; }

// out [n, D] = the output projection of head [n, H*d_v] on CUDA cores: the dense
// wo, or the grouped low-rank wo_a (one batched product per group of heads, into
// y [n, G*r_o] in act dtype) then wo_b ("Struct MlaWeights", wo_a / wo_b).
static void launch_o_proj_simt(const mla_handle* h, const void* head, void* out, void* y, long long n, cudaStream_t s);

// ---------------------------------------------------------------------------
// entry points
// ---------------------------------------------------------------------------
// The decode calls' own requirement (mla_workspace_bytes also covers prefill,
// whose FP8 weight dequantisation buffer decode never touches).
size_t mla_decode_workspace_bytes_internal(const mla_handle* h, int n) {
  if (!h || n < 1) return 0;
  return make_ws(h, n, 1).dec_total;
}

// Commits mla_decode_qkv_noalloc's device array on the current device (mla_noalloc.cu).
void mla_noalloc_prepare_device();

extern "C" {

const char* mla_strerror(int s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported by this library";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE_FLAG: return "device flag set (bad slot, block id or context length)";
    case MLA_ERR_WORKSPACE: return "buffer too small";
    default: return "unknown status";
  }
}

uint64_t mla_kernel_launch_count(void) { return (uint64_t)g_launches.load(); }

int mla_set_kernel_timer(const char* kernel, void* start_event, void* stop_event) {
  if (!kernel) { g_timer_kernel[0] = 0; g_timer_start = g_timer_stop = nullptr; return MLA_OK; }
  if (!start_event || !stop_event || strlen(kernel) >= sizeof(g_timer_kernel)) return MLA_ERR_INVALID_ARG;
  strcpy(g_timer_kernel, kernel);
  g_timer_start = (cudaEvent_t)start_event;
  g_timer_stop = (cudaEvent_t)stop_event;
  return MLA_OK;
}

size_t mla_weights_bytes(const mla_config* cfg) {
  if (validate_config(cfg) != MLA_OK) return 0;
  return make_layout(cfg).total;
}

int mla_init_weights(const mla_config* cfg, const mla_weights_desc* w, void* dst, size_t dst_bytes,
                     void* stream, mla_handle** out) {
  int st = validate_config(cfg);
  if (st != MLA_OK) return st;
  if (!w || !dst || !out) return MLA_ERR_INVALID_ARG;
  if (((uintptr_t)dst) % 256) return MLA_ERR_INVALID_ARG;
  const bool fp8 = cfg->weight_dtype == MLA_FP8_E4M3_B128;
  const int rq = cfg->q_lora_rank;
  if (!w->wq_b || !w->wkv_a || !w->wkv_b || !w->kv_norm_w) return MLA_ERR_INVALID_ARG;
  if (cfg->o_lora_rank > 0 ? (!w->wo_a || !w->wo_b) : !w->wo) return MLA_ERR_INVALID_ARG;
  if (rq && (!w->wq_a || !w->q_norm_w)) return MLA_ERR_INVALID_ARG;
  if (fp8 && (!w->wq_b_scale || !w->wkv_a_scale || !w->wkv_b_scale || !w->wo_scale || (rq && !w->wq_a_scale)))
    return MLA_ERR_INVALID_ARG;
  WeightLayout L = make_layout(cfg);
  if (dst_bytes < L.total) return MLA_ERR_WORKSPACE;
  mla_handle* h = new (std::nothrow) mla_handle();
  if (!h) return MLA_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->L = L;
  h->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)(cfg->qk_nope + cfg->qk_rope));
  h->base = (char*)dst;
  cudaGetDevice(&h->device);
  cudaStream_t s = (cudaStream_t)stream;
  const int H = cfg->n_heads, dn = cfg->qk_nope, dv = cfg->v_dim, rkv = cfg->kv_lora_rank, D = cfg->hidden;
  const int dr = cfg->qk_rope;
  const long long ldkvb = L.Hkv;  // row stride of wkv_b [r_kv, H*(dn+dv)]
  auto gather = [&](size_t dst_off, const void* src, long long off, long long sb, long long sn,
                    long long sk, int B, int N, int K, int esz) {
    const long long total = (long long)B * N * K;
    const int blocks = (int)((total + 255) / 256 > 65535 ? 65535 : (total + 255) / 256);
    if (esz == 4) gather3_kernel<uint32_t><<<blocks, 256, 0, s>>>((uint32_t*)(h->base + dst_off), (const uint32_t*)src, off, sb, sn, sk, B, N, K);
    else if (esz == 2) gather3_kernel<uint16_t><<<blocks, 256, 0, s>>>((uint16_t*)(h->base + dst_off), (const uint16_t*)src, off, sb, sn, sk, B, N, K);
    else gather3_kernel<uint8_t><<<blocks, 256, 0, s>>>((uint8_t*)(h->base + dst_off), (const uint8_t*)src, off, sb, sn, sk, B, N, K);
    count_launch();
  };
  const int e = (int)L.esz;
  // W1 = [wq_a | wkv_a]^T (or [q_proj | wkv_a]^T)
  if (rq) gather(L.W1, w->wq_a, 0, 0, 1, rq, 1, rq, D, e);
  else gather(L.W1, w->wq_b, 0, 0, 1, L.Hq, 1, L.Hq, D, e);
  gather(L.W1 + (size_t)L.Nq1 * D * L.esz, w->wkv_a, 0, 0, 1, L.R, 1, L.R, D, e);
  if (rq) gather(L.Wqb, w->wq_b, 0, 0, 1, L.Hq, 1, L.Hq, rq, e);
  gather(L.Wuk, w->wkv_b, 0, dn + dv, ldkvb, 1, H, rkv, dn, e);
  gather(L.Wuv, w->wkv_b, dn, dn + dv, 1, ldkvb, H, dv, rkv, e);
  gather(L.Wkvb, w->wkv_b, 0, 0, 1, ldkvb, 1, L.Hkv, rkv, e);
  if (L.G) {
    // Woa[g][j][i] = wo_a[g*Kg + i][j]; Wob[d][k] = wo_b[k][d]
    gather(L.Woa, w->wo_a, 0, (long long)L.Kg * L.ro, 1, L.ro, L.G, L.ro, L.Kg, e);
    gather(L.Wob, w->wo_b, 0, 0, 1, D, 1, D, L.G * L.ro, e);
  } else {
    gather(L.Wo, w->wo, 0, 0, 1, D, 1, D, H * dv, e);
  }
  if (rq) cudaMemcpyAsync(h->base + L.gq, w->q_norm_w, (size_t)rq * 4, cudaMemcpyDeviceToDevice, s);
  cudaMemcpyAsync(h->base + L.gkv, w->kv_norm_w, (size_t)rkv * 4, cudaMemcpyDeviceToDevice, s);
  h->has_sink = w->attn_sink != nullptr;
  if (w->attn_sink) cudaMemcpyAsync(h->base + L.sink, w->attn_sink, (size_t)H * 4, cudaMemcpyDeviceToDevice, s);
  if (fp8) {
    // scale tensors [ceil(in/128), ceil(out/128)] -> per K-major matrix [N/128][K/128]
    const long long Db = cdiv(D, 128), Rb = cdiv(L.R, 128), Hqb = L.Hq / 128, rqb = rq / 128;
    const long long rkvb = cdiv(rkv, 128), Hkvb = cdiv(L.Hkv, 128), Hvb = (long long)H * dv / 128;
    if (rq) gather(L.sW1, w->wq_a_scale, 0, 0, 1, rqb, 1, (int)rqb, (int)Db, 4);
    else gather(L.sW1, w->wq_b_scale, 0, 0, 1, Hqb, 1, (int)Hqb, (int)Db, 4);
    gather(L.sW1 + (size_t)(L.Nq1 / 128) * Db * 4, w->wkv_a_scale, 0, 0, 1, Rb, 1, (int)Rb, (int)Db, 4);
    if (rq) gather(L.sWqb, w->wq_b_scale, 0, 0, 1, Hqb, 1, (int)Hqb, (int)rqb, 4);
    // Wuk[h] = N r_kv (blocks of wkv_b rows), K d_n (blocks of head h's nope columns)
    gather(L.sWuk, w->wkv_b_scale, 0, (dn + dv) / 128, Hkvb, 1, H, (int)rkvb, dn / 128, 4);
    gather(L.sWuv, w->wkv_b_scale, dn / 128, (dn + dv) / 128, 1, Hkvb, H, dv / 128, (int)rkvb, 4);
    gather(L.sWkvb, w->wkv_b_scale, 0, 0, 1, Hkvb, 1, (int)Hkvb, (int)rkvb, 4);
    gather(L.sWo, w->wo_scale, 0, 0, 1, Db, 1, (int)Db, (int)Hvb, 4);
  }
  (void)dr;
  st = cuda_status();
  if (st == MLA_OK) st = tc_init(h);
  if (st != MLA_OK) { delete h; return st; }
  mla_noalloc_prepare_device();
  *out = h;
  return MLA_OK;
}

void mla_destroy(mla_handle* h) { delete h; }

size_t mla_workspace_bytes(const mla_handle* h, int max_tokens, int max_context_len) {
  if (!h || max_tokens < 1 || max_context_len < 1) return 0;
  return make_ws(h, max_tokens, max_context_len).total;
}


int mla_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) return MLA_ERR_INVALID_ARG;
  if (cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_read_device_flag(const void* ws, int* flag_out, void* stream) {
  if (!ws || !flag_out) return MLA_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  *flag_out = v;
  return v ? MLA_ERR_DEVICE_FLAG : MLA_OK;
}

int mla_clear_device_flag(void* ws, void* stream) {
  if (!ws) return MLA_ERR_INVALID_ARG;
  if (cudaMemsetAsync(ws, 0, 4, (cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_rope_cos_sin(const int32_t* positions, int n, int qk_rope, double theta, float* cos_out,
                     float* sin_out, void* stream) {
  if (n < 0 || qk_rope <= 0 || qk_rope % 2 || !(theta > 0.0)) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!positions || !cos_out || !sin_out) return MLA_ERR_INVALID_ARG;
  const long long total = (long long)n * (qk_rope / 2);
  const int blocks = (int)(cdiv(total, 256) > 4096 ? 4096 : cdiv(total, 256));
  rope_table_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(positions, n, qk_rope, theta, cos_out, sin_out);
  count_launch();
  return cuda_status();
}

int mla_rope_cos_sin_inv_freq(const int32_t* positions, int n, int qk_rope, const float* inv_freq,
                              float* cos_out, float* sin_out, void* stream) {
  if (n < 0 || qk_rope <= 0 || qk_rope % 2) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!positions || !inv_freq || !cos_out || !sin_out) return MLA_ERR_INVALID_ARG;
  const long long total = (long long)n * (qk_rope / 2);
  const int blocks = (int)(cdiv(total, 256) > 4096 ? 4096 : cdiv(total, 256));
  rope_table_freq_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(positions, n, qk_rope, inv_freq, cos_out, sin_out);
  count_launch();
  return cuda_status();
}

int mla_decode_qkv(mla_handle* h, const void* hidden, int n, const float* cos, const float* sin,
                   void* kv_cache, int n_blocks, const int32_t* slot_mapping, void* q_abs, void* q_pe,
                   const float* input_norm_w, void* ws, size_t ws_bytes, void* stream) {
  if (!h || n < 0 || n_blocks < 0) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!hidden || !cos || !sin || !kv_cache || !slot_mapping || !q_abs || !q_pe || !ws)
    return MLA_ERR_INVALID_ARG;
  const mla_config* c = &h->cfg;
  const WsLayout W = make_ws(h, n, 1);
  if (ws_bytes < W.dec_total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* wsb = (char*)ws;
  int* flag = (int*)wsb;
  const WeightLayout& L = h->L;
  const int H = c->n_heads, dn = c->qk_nope, dr = c->qk_rope, rkv = c->kv_lora_rank, D = c->hidden;
  const int rq = c->q_lora_rank;
  const int ta = acode(h), tw = wcode(h);
  if (input_norm_w) {
    // 0. the layer's input RMSNorm into the workspace; the path reads that instead
    void* xn = wsb + W.xn;
    if (ta == 0) input_rmsnorm_kernel<float><<<n, 256, 0, s>>>((const float*)hidden, input_norm_w, D, c->norm_eps, (float*)xn);
    else input_rmsnorm_kernel<bf16><<<n, 256, 0, s>>>((const bf16*)hidden, input_norm_w, D, c->norm_eps, (bf16*)xn);
    count_launch();
    hidden = xn;
  }
  if (tc_decode_qkv_supported(h, n)) {
    const int r = tc_decode_qkv(h, hidden, n, cos, sin, kv_cache, n_blocks, slot_mapping, q_abs, q_pe,
                                wsb, W.tc, s);
    return r != MLA_OK ? r : cuda_status();
  }
  // 1. merged first projection Y1 = x @ [wq_a | wkv_a]  (fp32)
  float* Y1 = (float*)(wsb + W.Y1);
  launch_linear(ta, tw, 0, lin(hidden, D, h->base + L.W1, D, wscale(h, L.sW1), cdiv(D, 128), Y1, L.N1, n, L.N1, D), 1, s);
  // 2. norms, k_pe RoPE, cache scatter
  FrontFoldArgs f{};
  f.Y = Y1; f.ldy = L.N1; f.r_q = rq; f.kv0 = L.Nq1; f.r_kv = rkv; f.d_r = dr;
  f.q_norm_w = rq ? (const float*)(h->base + L.gq) : nullptr;
  f.kv_norm_w = (const float*)(h->base + L.gkv); f.eps = c->norm_eps;
  f.cos = cos; f.sin = sin;
  f.qn = rq ? wsb + W.qn : nullptr; f.ldqn = rq;
  f.cache = kv_cache; f.n_rows = (long long)n_blocks * c->block_size;
  f.slot = slot_mapping; f.layout = c->row_layout; f.flag = flag;
  if (ta == 0) frontfold_epilogue_kernel<float><<<n, 256, 0, s>>>(f);
  else frontfold_epilogue_kernel<bf16><<<n, 256, 0, s>>>(f);
  count_launch();
  // 3. q = qn @ wq_b (fp32)
  const float* Qp = Y1;
  long long ldq = L.N1;
  if (rq) {
    float* Q = (float*)(wsb + W.Q);
    launch_linear(ta, tw, 0, lin(wsb + W.qn, rq, h->base + L.Wqb, rq, wscale(h, L.sWqb), rq / 128, Q, L.Hq, n, L.Hq, rq), 1, s);
    Qp = Q;
    ldq = L.Hq;
  }
  // 4. q_pe = RoPE(q[h, d_n:])
  if (ta == 0) q_rope_kernel<float, float><<<n, 256, 0, s>>>(Qp, ldq, H, dn, dr, cos, sin, (float*)q_pe, (long long)H * dr, dr, 0);
  else q_rope_kernel<float, bf16><<<n, 256, 0, s>>>(Qp, ldq, H, dn, dr, cos, sin, (bf16*)q_pe, (long long)H * dr, dr, 0);
  count_launch();
  // 5. q_abs[h] = q_nope[h] @ W_UK[h]   (batched over heads)
  LinearArgs a = lin(Qp, ldq, h->base + L.Wuk, dn, wscale(h, L.sWuk), 1, q_abs, (long long)H * rkv, n, rkv, dn);
  a.a_batch = dn + dr; a.w_batch = (long long)rkv * dn; a.c_batch = rkv;
  a.s_batch = cdiv(rkv, 128) * cdiv(dn, 128);
  launch_linear(0, tw, ta, a, H, s);
  return cuda_status();
}

int mla_decode_attn(mla_handle* h, const void* q_abs, const void* q_pe, const void* kv_cache, int n_blocks,
                    const int32_t* block_table, int max_blocks_per_seq, const int32_t* context_lens,
                    int max_context_len, int n, void* out, void* head_out, void* ws, size_t ws_bytes,
                    void* stream) {
  if (!h || n < 0 || n_blocks < 0 || max_blocks_per_seq < 0) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!q_abs || !q_pe || !kv_cache || !block_table || !context_lens || !out || !ws) return MLA_ERR_INVALID_ARG;
  if (max_context_len < 1 || max_blocks_per_seq < 1) return MLA_ERR_INVALID_ARG;
  const mla_config* c = &h->cfg;
  const WsLayout W = make_ws(h, n, max_context_len);
  if (ws_bytes < W.dec_total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* wsb = (char*)ws;
  int* flag = (int*)wsb;
  const WeightLayout& L = h->L;
  const int H = c->n_heads, dr = c->qk_rope, rkv = c->kv_lora_rank, dv = c->v_dim;
  const int ta = acode(h), tw = wcode(h);
  void* head = head_out ? head_out : (void*)(wsb + W.head);
  if (tc_decode_attn_supported(h, n, max_context_len)) {
    const int r = tc_decode_attn(h, q_abs, q_pe, kv_cache, n_blocks, block_table, max_blocks_per_seq,
                                 context_lens, max_context_len, n, out, head, wsb, W.tc, s,
                                 (float*)(wsb + W.part_o), (float*)(wsb + W.part_ml), W.splits,
                                 (bf16*)(wsb + W.o_lat), (int*)(wsb + W.nseg), head_out == nullptr);
    return r != MLA_OK ? r : cuda_status();
  }
  void* o_lat = wsb + W.o_lat;
  if (tc_attention_supported(h)) {
    // tensor-core attention (bf16 activations) ahead of CUDA-core W_UV / o_proj
    const int r = tc_attention_core(h, q_abs, q_pe, kv_cache, n_blocks, block_table, max_blocks_per_seq,
                                    context_lens, max_context_len, n, (float*)(wsb + W.part_o),
                                    (float*)(wsb + W.part_ml), W.splits, (bf16*)o_lat, flag,
                                    (int*)(wsb + W.nseg), s);
    if (r != MLA_OK) return r;
  } else {
    AttnArgs p{};
    p.q_abs = q_abs; p.q_pe = q_pe; p.cache = kv_cache; p.n_blocks = n_blocks; p.bs = c->block_size;
    p.block_table = block_table; p.mbps = max_blocks_per_seq; p.ctx = context_lens; p.max_ctx = max_context_len;
    p.H = H; p.r_kv = rkv; p.d_r = dr; p.layout = c->row_layout; p.scale = h->scale;
    p.n_splits = W.splits;
    p.chunk = (int)cdiv(cdiv(max_context_len, W.splits), ATT_TR) * ATT_TR;
    p.part_o = (float*)(wsb + W.part_o); p.part_ml = (float*)(wsb + W.part_ml); p.flag = flag;
    const int R = rkv + dr;
    const size_t smem = (size_t)(ATT_TR * (R + 1) + ATT_HPB * R) * 4;
    dim3 grid(W.splits, n, (unsigned)cdiv(H, ATT_HPB));
    mla_timer_begin("attn", s);
    if (ta == 0) { set_smem(attn_decode_simt_kernel<float>, smem); attn_decode_simt_kernel<float><<<grid, 256, smem, s>>>(p); }
    else { set_smem(attn_decode_simt_kernel<bf16>, smem); attn_decode_simt_kernel<bf16><<<grid, 256, smem, s>>>(p); }
    mla_timer_end("attn", s);
    count_launch();
    dim3 cg(n, H);
    const float* sink = h->has_sink ? (const float*)(h->base + L.sink) : nullptr;
    if (ta == 0) attn_combine_kernel<float><<<cg, 128, 0, s>>>(p.part_o, p.part_ml, W.splits, H, rkv, (float*)o_lat, sink, 0, 0, nullptr);
    else attn_combine_kernel<bf16><<<cg, 128, 0, s>>>(p.part_o, p.part_ml, W.splits, H, rkv, (bf16*)o_lat, sink, 0, 0, nullptr);
    count_launch();
  }
  // head_out[h] = o_lat[h] @ W_UV[h]
  LinearArgs a = lin(o_lat, (long long)H * rkv, h->base + L.Wuv, rkv, wscale(h, L.sWuv), cdiv(rkv, 128), head,
                     (long long)H * dv, n, dv, rkv);
  a.a_batch = rkv; a.w_batch = (long long)dv * rkv; a.c_batch = dv; a.s_batch = cdiv(dv, 128) * cdiv(rkv, 128);
  launch_linear(ta, tw, ta, a, H, s);
  // out = head_out @ wo (or wo_a -> wo_b)
  launch_o_proj_simt(h, head, out, wsb + W.oy, n, s);
  return cuda_status();
}

// Stage buffer of mla_decode_step_host: staged inputs, then the step's own
// device tensors.
struct StepStage {
  size_t hidden, ints, cos, sin, q_abs, q_pe, out, total;
  size_t ints_bytes;
};

static StepStage make_stage(const mla_handle* h, long long n, long long mbps) {
  const mla_config* c = &h->cfg;
  const size_t a = dtype_size(c->act_dtype);
  StepStage P{};
  size_t off = 0;
  auto put = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  P.hidden = put((size_t)n * c->hidden * a);
  P.ints_bytes = (size_t)(3 * n + n * mbps) * 4;   // positions, slot_mapping, context_lens, block_table
  P.ints = put(P.ints_bytes);
  P.cos = put((size_t)n * (c->qk_rope / 2) * 4);
  P.sin = put((size_t)n * (c->qk_rope / 2) * 4);
  P.q_abs = put((size_t)n * c->n_heads * c->kv_lora_rank * a);
  P.q_pe = put((size_t)n * c->n_heads * c->qk_rope * a);
  P.out = put((size_t)n * c->hidden * a);
  P.total = off;
  return P;
}

size_t mla_decode_step_host_bytes(const mla_handle* h, int n, int max_blocks_per_seq) {
  if (!h || n < 1 || max_blocks_per_seq < 1) return 0;
  return make_stage(h, n, max_blocks_per_seq).total;
}

// The device work of one host step, enqueued on `s`: inputs in, RoPE tables,
// front-fold, attention, output out.
static int enqueue_host_step(mla_handle* h, const StepStage& P, const void* hidden_host, int mbps, int max_ctx,
                             int n, double rope_theta, void* kv_cache, int n_blocks, void* out_host, char* st,
                             void* ws, size_t ws_bytes, cudaStream_t s) {
  const mla_config* c = &h->cfg;
  const size_t act_bytes = (size_t)n * c->hidden * dtype_size(c->act_dtype);
  const int32_t* d_ints = (const int32_t*)(st + P.ints);
  if (cudaMemcpyAsync(st + P.hidden, hidden_host, act_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(st + P.ints, h->host_pack, P.ints_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaEventRecordWithFlags(h->pack_done, s, cudaEventRecordExternal) != cudaSuccess)
    return cuda_fail();
  float* cos = (float*)(st + P.cos);
  float* sin = (float*)(st + P.sin);
  int r = mla_rope_cos_sin(d_ints, n, c->qk_rope, rope_theta, cos, sin, s);
  if (r != MLA_OK) return r;
  r = mla_decode_qkv(h, st + P.hidden, n, cos, sin, kv_cache, n_blocks, d_ints + n, st + P.q_abs, st + P.q_pe,
                     nullptr, ws, ws_bytes, s);
  if (r != MLA_OK) return r;
  r = mla_decode_attn(h, st + P.q_abs, st + P.q_pe, kv_cache, n_blocks, d_ints + 3 * n, mbps, d_ints + 2 * n,
                      max_ctx, n, st + P.out, nullptr, ws, ws_bytes, s);
  if (r != MLA_OK) return r;
  if (cudaMemcpyAsync(out_host, st + P.out, act_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return cuda_fail();
  return cuda_status();
}

int mla_decode_step_host(mla_handle* h, const void* hidden_host, const int32_t* positions_host,
                         const int32_t* slot_mapping_host, const int32_t* block_table_host,
                         int max_blocks_per_seq, const int32_t* context_lens_host, int max_context_len,
                         int n, double rope_theta, void* kv_cache, int n_blocks, void* out_host, void* stage,
                         size_t stage_bytes, void* ws, size_t ws_bytes, void* stream) {
  if (!h || n < 0 || n_blocks < 0) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  if (!hidden_host || !positions_host || !slot_mapping_host || !block_table_host || !context_lens_host ||
      !kv_cache || !out_host || !stage || !ws)
    return MLA_ERR_INVALID_ARG;
  if (max_blocks_per_seq < 1 || max_context_len < 1 || !(rope_theta > 0.0)) return MLA_ERR_INVALID_ARG;
  const StepStage P = make_stage(h, n, max_blocks_per_seq);
  if (stage_bytes < P.total) return MLA_ERR_WORKSPACE;
  if (ws_bytes < make_ws(h, n, max_context_len).dec_total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  // pack the int32 inputs into the handle's page-locked buffer: one transfer
  if (h->pack_done && cudaEventSynchronize(h->pack_done) != cudaSuccess) return cuda_fail();
  if (h->host_pack_bytes < P.ints_bytes) {
    if (h->host_pack) cudaFreeHost(h->host_pack);
    h->host_pack = nullptr;
    h->host_pack_bytes = 0;
    if (cudaHostAlloc(&h->host_pack, P.ints_bytes, cudaHostAllocDefault) != cudaSuccess) {
      h->host_pack = nullptr;
      return cuda_fail();
    }
    h->host_pack_bytes = P.ints_bytes;
  }
  if (!h->pack_done && cudaEventCreateWithFlags(&h->pack_done, cudaEventDisableTiming) != cudaSuccess) {
    h->pack_done = nullptr;
    return cuda_fail();
  }
  int32_t* pk = (int32_t*)h->host_pack;
  memcpy(pk, positions_host, (size_t)n * 4);
  memcpy(pk + n, slot_mapping_host, (size_t)n * 4);
  memcpy(pk + 2 * n, context_lens_host, (size_t)n * 4);
  memcpy(pk + 3 * n, block_table_host, (size_t)n * max_blocks_per_seq * 4);
  char* st = (char*)stage;
  // with a kernel timer set, run eagerly so that its events bracket this call's launch
  if (g_timer_kernel[0])
    return enqueue_host_step(h, P, hidden_host, max_blocks_per_seq, max_context_len, n, rope_theta, kv_cache,
                             n_blocks, out_host, st, ws, ws_bytes, s);
  // otherwise replay the step's CUDA graph, captured again whenever a buffer or a size changes
  double theta = rope_theta;
  unsigned long long theta_bits = 0;
  memcpy(&theta_bits, &theta, sizeof theta_bits);
  const unsigned long long key[14] = {
      (unsigned long long)(uintptr_t)hidden_host, (unsigned long long)(uintptr_t)out_host,
      (unsigned long long)(uintptr_t)kv_cache,    (unsigned long long)(uintptr_t)stage,
      (unsigned long long)(uintptr_t)ws,          (unsigned long long)ws_bytes,
      (unsigned long long)stage_bytes,            (unsigned long long)n,
      (unsigned long long)max_blocks_per_seq,     (unsigned long long)max_context_len,
      (unsigned long long)n_blocks,               theta_bits,
      (unsigned long long)(uintptr_t)h->host_pack, 1ull};
  if (!h->step_exec || memcmp(key, h->step_key, sizeof key) != 0) {
    if (!h->capture_stream && cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking) != cudaSuccess) {
      h->capture_stream = nullptr;
      return cuda_fail();
    }
    const unsigned long long before = mla_kernel_launch_count();
    if (cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
      return cuda_fail();
    const int r = enqueue_host_step(h, P, hidden_host, max_blocks_per_seq, max_context_len, n, rope_theta,
                                    kv_cache, n_blocks, out_host, st, ws, ws_bytes, h->capture_stream);
    cudaGraph_t g = nullptr;
    const cudaError_t e = cudaStreamEndCapture(h->capture_stream, &g);
    // the launches counted while capturing run at each replay instead
    const long long captured = (long long)(mla_kernel_launch_count() - before);
    mla_count_launch((int)-captured);
    if (r != MLA_OK || e != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      cudaGetLastError();
      return r != MLA_OK ? r : MLA_ERR_CUDA;
    }
    cudaGraphExec_t ex = nullptr;
    const cudaError_t ei = cudaGraphInstantiate(&ex, g, 0);
    cudaGraphDestroy(g);
    if (ei != cudaSuccess) return cuda_fail();
    if (h->step_exec) cudaGraphExecDestroy(h->step_exec);
    h->step_exec = ex;
    h->step_launches = (int)captured;
    memcpy(h->step_key, key, sizeof key);
  }
  if (cudaGraphLaunch(h->step_exec, s) != cudaSuccess) return cuda_fail();
  count_launch(h->step_launches);
  return MLA_OK;
}

int mla_prefill(mla_handle* h, const void* hidden, int S, const float* cos, const float* sin, void* out,
                void* head_out, void* kv_cache, int n_blocks, const int32_t* slot_mapping, void* ws,
                size_t ws_bytes, void* stream) {
  if (!h || S < 0 || n_blocks < 0) return MLA_ERR_INVALID_ARG;
  if (S == 0) return MLA_OK;
  if (!hidden || !cos || !sin || !out || !ws) return MLA_ERR_INVALID_ARG;
  if ((kv_cache == nullptr) != (slot_mapping == nullptr)) return MLA_ERR_INVALID_ARG;
  const mla_config* c = &h->cfg;
  const WsLayout W = make_ws(h, S, 1);
  if (ws_bytes < W.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* wsb = (char*)ws;
  int* flag = (int*)wsb;
  const WeightLayout& L = h->L;
  const int H = c->n_heads, dn = c->qk_nope, dr = c->qk_rope, rkv = c->kv_lora_rank, dv = c->v_dim;
  const int D = c->hidden, rq = c->q_lora_rank;
  const int ta = acode(h), tw = wcode(h);
  void* head = head_out ? head_out : (void*)(wsb + W.phead);
  if (tc_prefill_supported(h, S)) {
    const int r = tc_prefill(h, hidden, S, cos, sin, out, head, kv_cache, n_blocks, slot_mapping, wsb,
                             W.pY1, W.pqn, W.pQ, W.pcn, W.pkpe, W.pKV, W.pDQ, W.poy, s);
    return r != MLA_OK ? r : cuda_status();
  }
  float* Y1 = (float*)(wsb + W.pY1);
  void* Q = wsb + W.pQ;
  FrontFoldArgs f{};
  if (rq) {
    launch_linear(ta, tw, 0, lin(hidden, D, h->base + L.W1, D, wscale(h, L.sW1), cdiv(D, 128), Y1, L.N1, S, L.N1, D), 1, s);
    f.Y = Y1; f.ldy = L.N1; f.kv0 = L.Nq1;
  } else {
    // q = x @ q_proj straight to act dtype; kv part to fp32
    launch_linear(ta, tw, ta, lin(hidden, D, h->base + L.W1, D, wscale(h, L.sW1), cdiv(D, 128), Q, L.Hq, S, L.Hq, D), 1, s);
    const float* sc = wscale(h, L.sW1);
    launch_linear(ta, tw, 0, lin(hidden, D, h->base + L.W1 + (size_t)L.Nq1 * D * L.esz, D,
                                 sc ? sc + (size_t)(L.Nq1 / 128) * cdiv(D, 128) : nullptr, cdiv(D, 128), Y1, L.R, S, L.R, D), 1, s);
    f.Y = Y1; f.ldy = L.R; f.kv0 = 0;
  }
  f.r_q = rq; f.r_kv = rkv; f.d_r = dr;
  f.q_norm_w = rq ? (const float*)(h->base + L.gq) : nullptr;
  f.kv_norm_w = (const float*)(h->base + L.gkv); f.eps = c->norm_eps;
  f.cos = cos; f.sin = sin;
  f.qn = rq ? wsb + W.pqn : nullptr; f.ldqn = rq;
  f.cache = kv_cache; f.n_rows = (long long)n_blocks * c->block_size;
  f.slot = slot_mapping; f.layout = c->row_layout; f.flag = flag;
  f.cn = wsb + W.pcn; f.kpe = wsb + W.pkpe;
  if (ta == 0) frontfold_epilogue_kernel<float><<<S, 256, 0, s>>>(f);
  else frontfold_epilogue_kernel<bf16><<<S, 256, 0, s>>>(f);
  count_launch();
  if (rq) launch_linear(ta, tw, ta, lin(wsb + W.pqn, rq, h->base + L.Wqb, rq, wscale(h, L.sWqb), rq / 128, Q, L.Hq, S, L.Hq, rq), 1, s);
  // RoPE q_pe in place
  if (ta == 0) q_rope_kernel<float, float><<<S, 256, 0, s>>>((const float*)Q, L.Hq, H, dn, dr, cos, sin, (float*)Q, L.Hq, dn + dr, dn);
  else q_rope_kernel<bf16, bf16><<<S, 256, 0, s>>>((const bf16*)Q, L.Hq, H, dn, dr, cos, sin, (bf16*)Q, L.Hq, dn + dr, dn);
  count_launch();
  // kv_out = c @ wkv_b
  void* KV = wsb + W.pKV;
  launch_linear(ta, tw, ta, lin(wsb + W.pcn, rkv, h->base + L.Wkvb, rkv, wscale(h, L.sWkvb), cdiv(rkv, 128), KV, L.Hkv, S, L.Hkv, rkv), 1, s);
  PrefillAttnArgs pa{};
  pa.Q = Q; pa.ldq = L.Hq; pa.KV = KV; pa.ldkv = L.Hkv; pa.kpe = wsb + W.pkpe;
  pa.O = head; pa.ldo = (long long)H * dv; pa.S = S; pa.H = H; pa.d_n = dn; pa.d_r = dr; pa.d_v = dv;
  pa.scale = h->scale;
  pa.sink = h->has_sink ? (const float*)(h->base + L.sink) : nullptr;
  const size_t smem = (size_t)(PA_BQ * (dn + dr) + PA_BK * (dn + dr + 1) + PA_BK * dv) * 4;
  dim3 grid((unsigned)cdiv(S, PA_BQ), H);
  mla_timer_begin("prefill_attn", s);
  if (ta == 0) { set_smem(prefill_attn_simt_kernel<float>, smem); prefill_attn_simt_kernel<float><<<grid, 128, smem, s>>>(pa); }
  else { set_smem(prefill_attn_simt_kernel<bf16>, smem); prefill_attn_simt_kernel<bf16><<<grid, 128, smem, s>>>(pa); }
  mla_timer_end("prefill_attn", s);
  count_launch();
  launch_o_proj_simt(h, head, out, wsb + W.poy, S, s);
  return cuda_status();
}

int mla_v4_qkv(mla_handle* h, const void* hidden, int S, const float* cos, const float* sin,
               const float* kv_norm_w, void* q_out, void* kv_out, void* ws, size_t ws_bytes, void* stream) {
  if (!h || S < 0) return MLA_ERR_INVALID_ARG;
  if (S == 0) return MLA_OK;
  if (!hidden || !cos || !sin || !kv_norm_w || !q_out || !kv_out || !ws) return MLA_ERR_INVALID_ARG;
  const mla_config* c = &h->cfg;
  if (c->q_lora_rank == 0) return MLA_ERR_UNSUPPORTED;   // the V4 query path is low-rank
  const WsLayout W = make_ws(h, S, 1);
  if (ws_bytes < W.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  char* wsb = (char*)ws;
  int* flag = (int*)wsb;
  const WeightLayout& L = h->L;
  const int H = c->n_heads, dn = c->qk_nope, dr = c->qk_rope, rkv = c->kv_lora_rank;
  const int D = c->hidden, rq = c->q_lora_rank;
  const int ta = acode(h), tw = wcode(h);
  if (tc_prefill_supported(h, S)) {
    const int r = tc_v4_qkv(h, hidden, S, cos, sin, kv_norm_w, q_out, kv_out, wsb, W.pY1, W.pqn, W.pDQ, s);
    return r != MLA_OK ? r : cuda_status();
  }
  float* Y1 = (float*)(wsb + W.pY1);
  launch_linear(ta, tw, 0, lin(hidden, D, h->base + L.W1, D, wscale(h, L.sW1), cdiv(D, 128), Y1, L.N1, S, L.N1, D), 1, s);
  FrontFoldArgs f{};
  f.Y = Y1; f.ldy = L.N1; f.kv0 = L.Nq1;
  f.r_q = rq; f.r_kv = rkv; f.d_r = dr;
  f.q_norm_w = (const float*)(h->base + L.gq);
  f.kv_norm_w = kv_norm_w; f.eps = c->norm_eps;
  f.cos = cos; f.sin = sin;
  f.qn = wsb + W.pqn; f.ldqn = rq;
  f.cache = kv_out; f.n_rows = S; f.slot = nullptr; f.layout = MLA_ROW_LATENT_FIRST; f.flag = flag;
  f.v4 = 1;
  if (ta == 0) frontfold_epilogue_kernel<float><<<S, 256, 0, s>>>(f);
  else frontfold_epilogue_kernel<bf16><<<S, 256, 0, s>>>(f);
  count_launch();
  launch_linear(ta, tw, ta, lin(wsb + W.pqn, rq, h->base + L.Wqb, rq, wscale(h, L.sWqb), rq / 128, q_out, L.Hq, S, L.Hq, rq), 1, s);
  if (ta == 0) q_headnorm_rope_kernel<float><<<S, 256, 0, s>>>((float*)q_out, L.Hq, H, dn + dr, dr, cos, sin, c->norm_eps);
  else q_headnorm_rope_kernel<bf16><<<S, 256, 0, s>>>((bf16*)q_out, L.Hq, H, dn + dr, dr, cos, sin, c->norm_eps);
  count_launch();
  return cuda_status();
}

}  // extern "C"
