// Tensor-core (tcgen05 / TMEM / TMA) path of the MLA layer step for bf16
// activations with bf16 weights: every weight contraction runs on the
// persistent tcgen05 GEMM (tc_gemm.cuh); the norms, RoPE and the cache scatter
// run in the GEMM epilogues or in one per-token front-fold kernel.
#pragma once

#include <atomic>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "handle.cuh"
#include "simt_kernels.cuh"
#include "tc_gemm.cuh"
#include "tc_gemm_fp8.cuh"
#include "tc_attn.cuh"
#include "tc_attn_pair.cuh"
#include "tc_prefill_attn.cuh"

namespace mla {
namespace tc {

// Raises a kernel's dynamic shared memory limit once per device. The flags are
// atomic, so host threads launching at the same time are safe; two of them may
// both make the (idempotent) call. Devices past the table set it on every call.
template <typename K>
static void set_smem_once(std::atomic<bool>* done, K kernel, int bytes) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && done[dev].load(std::memory_order_acquire)) return;
  cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (dev < 64) done[dev].store(true, std::memory_order_release);
}

// ---------------------------------------------------------------------------
// TMA tensor maps (cuTensorMapEncodeTiled, resolved through the runtime so the
// library needs no link-time libcuda)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

// bf16 3-D map {K, d1, d2} (K contiguous) with 128-byte swizzle and a box of
// 64 K-elements x `box_rows` rows; the rows are dimension 1 (rows_dim2 = 0) or
// dimension 2 (rows_dim2 = 1). Strides in bytes. Out-of-range elements read 0.
static int make_map(CUtensorMap* m, const void* base, long long K, long long d1, long long d2, long long s1,
                    long long s2, int box_rows, int rows_dim2, bool u8 = false) {
  auto fn = encode_fn();
  if (!fn) return MLA_ERR_CUDA;
  if (((uintptr_t)base) & 15 || s1 % 16 || s2 % 16) return MLA_ERR_UNSUPPORTED;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)d1, (cuuint64_t)d2};
  cuuint64_t strides[2] = {(cuuint64_t)s1, (cuuint64_t)s2};
  // 128-byte rows: 64 bf16 or 128 FP8 codes
  cuuint32_t box[3] = {(cuuint32_t)(u8 ? 128 : 64), (cuuint32_t)(rows_dim2 ? 1 : box_rows),
                       (cuuint32_t)(rows_dim2 ? box_rows : 1)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// 2-D row-major [rows, K] bf16 matrix with row stride ld (elements).
static int make_map2(CUtensorMap* m, const void* base, long long K, long long rows, long long ld, int box_rows) {
  return make_map(m, base, K, rows, 1, ld * 2, ld * 2 * rows, box_rows, 0);
}

// The paged cache [rows, R] bf16 (R a multiple of 64, rows a multiple of 8)
// as a 4-D map {64 columns, 8 rows, R / 64 column groups, rows / 8 octets}, so
// that one box brings `groups` adjacent 64-column k-blocks of 64 rows: in
// shared memory [octet][group][8 rows][128 B], a 128-byte-swizzle operand
// whose 8-row groups lie groups x 1024 B apart. Few large boxes stream faster
// than many [64 x 64] ones.
static int make_map_cache_groups(CUtensorMap* m, const void* base, long long R, long long rows, int groups) {
  auto fn = encode_fn();
  if (!fn) return MLA_ERR_CUDA;
  if (((uintptr_t)base) & 15 || R % 64 || rows % 8) return MLA_ERR_UNSUPPORTED;
  cuuint64_t dims[4] = {64, 8, (cuuint64_t)(R / 64), (cuuint64_t)(rows / 8)};
  cuuint64_t strides[3] = {(cuuint64_t)(R * 2), 128, (cuuint64_t)(8 * R * 2)};
  cuuint32_t box[4] = {64, 8, (cuuint32_t)groups, 8};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel's CTAs may start
// while the previous kernel of the stream drains (its launch latency and
// set-up overlap that kernel); each kernel of this library calls griddep_wait
// before it touches memory an earlier kernel writes.
template <typename... KArgs, typename... Args>
static void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <int BN>
static int launch_gemm_bn(const CUtensorMap& A, const CUtensorMap& B, const GemmArgs& g, int num_sms,
                          cudaStream_t s) {
  using C = GemmCfg<BN>;
  static std::atomic<bool> attr_set[64];
  set_smem_once(attr_set, tc_gemm_kernel<BN>, C::SMEM);
  const int grid = g.total_units < num_sms ? g.total_units : num_sms;
  launch_pdl(tc_gemm_kernel<BN>, grid, 192, C::SMEM, s, A, B, g);
  mla_count_launch(1);
  return MLA_OK;
}

static int pick_bn(int n) {
  if (n <= 16) return 16;
  if (n <= 32) return 32;
  if (n <= 64) return 64;
  if (n <= 128) return 128;
  return 256;
}

// Fill the tiling fields of g and launch with an N tile of `bn`.
static int launch_gemm(const CUtensorMap& A, const CUtensorMap& B, GemmArgs g, int bn, int splits, int num_sms,
                       cudaStream_t s) {
  g.m_tiles = (int)cdiv(g.M, 128);
  g.n_tiles = (int)cdiv(g.N, bn);
  g.k_blocks = (int)cdiv(g.K, 64);
  if (splits < 1) splits = 1;
  if (splits > g.k_blocks) splits = g.k_blocks;
  g.kb_per_split = (int)cdiv(g.k_blocks, splits);
  g.splits = (int)cdiv(g.k_blocks, g.kb_per_split);   // no empty split
  g.total_units = g.m_tiles * g.n_tiles * g.batches * g.splits;
  if (g.total_units <= 0) return MLA_OK;
  switch (bn) {
    case 16: return launch_gemm_bn<16>(A, B, g, num_sms, s);
    case 32: return launch_gemm_bn<32>(A, B, g, num_sms, s);
    case 64: return launch_gemm_bn<64>(A, B, g, num_sms, s);
    case 128: return launch_gemm_bn<128>(A, B, g, num_sms, s);
    default: return launch_gemm_bn<256>(A, B, g, num_sms, s);
  }
}

template <int BN>
static int launch_gemm_fp8_bn(const CUtensorMap& A, const CUtensorMap& B, const Fp8GemmArgs& fa, int num_sms,
                              cudaStream_t s) {
  using C = Fp8Cfg<BN>;
  static std::atomic<bool> attr_set[64];
  set_smem_once(attr_set, tc_gemm_fp8_kernel<BN>, C::SMEM);
  const int grid = fa.g.total_units < num_sms ? fa.g.total_units : num_sms;
  launch_pdl(tc_gemm_fp8_kernel<BN>, grid, FP8_THREADS, C::SMEM, s, A, B, fa);
  mla_count_launch(1);
  return MLA_OK;
}

// FP8-weight GEMM (A = codes, K blocks of 128 = one scale column each).
static int launch_gemm_fp8(const CUtensorMap& A, const CUtensorMap& B, GemmArgs g, int bn, int splits,
                           const float* scale, long long scale_ld, long long scale_batch, int num_sms,
                           cudaStream_t s) {
  g.m_tiles = (int)cdiv(g.M, 128);
  g.n_tiles = (int)cdiv(g.N, bn);
  g.k_blocks = (int)cdiv(g.K, 128);
  if (splits < 1) splits = 1;
  if (splits > g.k_blocks) splits = g.k_blocks;
  g.kb_per_split = (int)cdiv(g.k_blocks, splits);
  g.splits = (int)cdiv(g.k_blocks, g.kb_per_split);
  g.total_units = g.m_tiles * g.n_tiles * g.batches * g.splits;
  if (g.total_units <= 0) return MLA_OK;
  Fp8GemmArgs fa{};
  fa.g = g; fa.scale = scale; fa.scale_ld = scale_ld; fa.scale_batch = scale_batch;
  switch (bn) {
    case 16: return launch_gemm_fp8_bn<16>(A, B, fa, num_sms, s);
    case 32: return launch_gemm_fp8_bn<32>(A, B, fa, num_sms, s);
    case 64: return launch_gemm_fp8_bn<64>(A, B, fa, num_sms, s);
    default: return launch_gemm_fp8_bn<128>(A, B, fa, num_sms, s);
  }
}

// Splits of the K loop for a persistent grid of num_sms CTAs: minimise the
// work of the busiest CTA, ceil(m_tiles * s / num_sms) units of 1/s of K each,
// a unit costing its K blocks plus epi_blocks for storing its fp32 partial
// (ties to fewer splits: fewer partial sums to add up afterwards).
static int decode_splits_for(int m_tiles, int k_blocks, int num_sms, int epi_blocks = 0) {
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 16 && s <= k_blocks; ++s) {
    const int per = (int)cdiv(k_blocks, s);
    const int real = (int)cdiv(k_blocks, per);          // the launcher drops empty splits
    const double cost = (double)cdiv((long long)m_tiles * real, num_sms) * (per + epi_blocks);
    if (cost < best_cost - 1e-9) { best_cost = cost; best = real; }
  }
  return best;
}

// ---------------------------------------------------------------------------
// small kernels of the tensor-core decode path
// ---------------------------------------------------------------------------
struct FrontFoldTcArgs {
  const float* Yp;  long long split_stride; int splits; int N1;
  int rq, Nq1, rkv, dr, H, dn;
  const float* q_norm_w; const float* kv_norm_w; float eps;
  const float* cos; const float* sin;
  bf16* qn; bf16* q_nope; bf16* q_pe;
  int act_f16;   // qn and q_nope in f16 (their only reader is an FP8-weight GEMM)
  bf16* cache; long long n_rows; const int* slot; int layout;
  int* flag;
  int q_cols;   // columns of the q part per CTA: all r_q, or whole heads of d_n + d_r
};

// Sum the K-split partials of columns [c0, c0 + w) of token t's row of x @ W1
// into y[0, w) (16-byte loads when aligned, the first eight splits' loads all
// in flight before the sum).
__device__ __forceinline__ void frontfold_sum(const FrontFoldTcArgs& p, int t, int c0, int w, float* y) {
  const float* yp = p.Yp + (long long)t * p.N1 + c0;
  if (w % 4 == 0 && c0 % 4 == 0 && p.N1 % 4 == 0 && p.split_stride % 4 == 0 && ((uintptr_t)p.Yp & 15) == 0) {
    const float4* yp4 = reinterpret_cast<const float4*>(yp);
    const long long st4 = p.split_stride >> 2;
    for (int c = threadIdx.x; c < (w >> 2); c += blockDim.x) {
      float4 v[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) v[s] = s < p.splits ? yp4[s * st4 + c] : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 acc = v[0];
#pragma unroll
      for (int s = 1; s < 8; ++s) { acc.x += v[s].x; acc.y += v[s].y; acc.z += v[s].z; acc.w += v[s].w; }
      for (int s = 8; s < p.splits; ++s) {
        const float4 u = yp4[s * st4 + c];
        acc.x += u.x; acc.y += u.y; acc.z += u.z; acc.w += u.w;
      }
      reinterpret_cast<float4*>(y)[c] = acc;
    }
  } else {
    for (int c = threadIdx.x; c < w; c += blockDim.x) {
      float acc = 0.f;
      for (int s = 0; s < p.splits; ++s) acc += yp[s * p.split_stride + c];
      y[c] = acc;
    }
  }
}

// grid (tokens, 1 + q slices). For token t, CTA 0 sums the kv part of the
// K-split partials of x @ W1 and does
//   kv latent -> RMSNorm * kv_norm_w, k_pe -> RoPE, row -> cache[slot];
// CTA g >= 1 sums its slice of the q part and does
//   q latent -> RMSNorm * q_norm_w -> qn (bf16)            (r_q > 0: one slice, all r_q)
//   or q -> q_nope (bf16) and RoPE(q_pe) (bf16)            (r_q = 0: slices of whole heads)
__global__ void __launch_bounds__(512) frontfold_tc_kernel(FrontFoldTcArgs p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float y[];   // [max(q_cols, r_kv + d_r)]
  __shared__ float red[32];
  const int t = blockIdx.x, g = blockIdx.y;
  const int half = p.dr / 2;
  if (g > 0) {
    const int c0 = (g - 1) * p.q_cols;
    const int w = min(p.Nq1, c0 + p.q_cols) - c0;
    if (w <= 0) return;
    frontfold_sum(p, t, c0, w, y);
    __syncthreads();
    if (p.rq) {
      float ss = 0.f;
      for (int i = threadIdx.x; i < p.rq; i += blockDim.x) ss += y[i] * y[i];
      const float r = rsqrtf(block_sum(ss, red) / (float)p.rq + p.eps);
      for (int i = threadIdx.x; i < p.rq; i += blockDim.x) {
        const float v = y[i] * r * p.q_norm_w[i];
        if (p.act_f16) ((__half*)p.qn)[(long long)t * p.rq + i] = __float2half_rn(v);
        else p.qn[(long long)t * p.rq + i] = __float2bfloat16_rn(v);
      }
    } else {
      const int hd = p.dn + p.dr, h0 = c0 / hd, nh = w / hd;
      for (int idx = threadIdx.x; idx < nh * p.dn; idx += blockDim.x) {
        const int h = idx / p.dn, j = idx % p.dn;
        const long long o = ((long long)t * p.H + h0 + h) * p.dn + j;
        if (p.act_f16) ((__half*)p.q_nope)[o] = __float2half_rn(y[h * hd + j]);
        else p.q_nope[o] = __float2bfloat16_rn(y[h * hd + j]);
      }
      for (int idx = threadIdx.x; idx < nh * half; idx += blockDim.x) {
        const int h = idx / half, i = idx % half;
        float o0, o1;
        rope_pair(y[h * hd + p.dn + 2 * i], y[h * hd + p.dn + 2 * i + 1], p.cos[(long long)t * half + i],
                  p.sin[(long long)t * half + i], &o0, &o1);
        p.q_pe[((long long)t * p.H + h0 + h) * p.dr + 2 * i] = __float2bfloat16_rn(o0);
        p.q_pe[((long long)t * p.H + h0 + h) * p.dr + 2 * i + 1] = __float2bfloat16_rn(o1);
      }
    }
    return;
  }
  frontfold_sum(p, t, p.Nq1, p.rkv + p.dr, y);
  __syncthreads();
  const float* kv = y;
  float ss = 0.f;
  for (int i = threadIdx.x; i < p.rkv; i += blockDim.x) ss += kv[i] * kv[i];
  const float r = rsqrtf(block_sum(ss, red) / (float)p.rkv + p.eps);
  const int slot = p.slot[t];
  if (slot < 0) return;
  if ((long long)slot >= p.n_rows) {
    if (threadIdx.x == 0) set_flag(p.flag, MLA_FLAG_BAD_SLOT);
    return;
  }
  bf16* row = p.cache + (long long)slot * (p.rkv + p.dr);
  const int lat_off = (p.layout == MLA_ROW_LATENT_FIRST) ? 0 : p.dr;
  const int pe_off = (p.layout == MLA_ROW_LATENT_FIRST) ? p.rkv : 0;
  for (int i = threadIdx.x; i < p.rkv; i += blockDim.x)
    row[lat_off + i] = __float2bfloat16_rn(kv[i] * r * p.kv_norm_w[i]);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    float o0, o1;
    rope_pair(kv[p.rkv + 2 * i], kv[p.rkv + 2 * i + 1], p.cos[(long long)t * half + i],
              p.sin[(long long)t * half + i], &o0, &o1);
    row[pe_off + 2 * i] = __float2bfloat16_rn(o0);
    row[pe_off + 2 * i + 1] = __float2bfloat16_rn(o1);
  }
}

// bf16 -> f16 copy (the FP8 GEMM's token operand), 8 elements per thread.
__global__ void cvt_bf16_f16_kernel(const uint4* src, uint4* dst, long long n8) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 v = src[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
      const __half2 hh = __floats2half2_rn(f.x, f.y);
      o[k] = *reinterpret_cast<const uint32_t*>(&hh);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// out[n][m] = bf16(sum_s part[s][n][m])
__global__ void splitk_reduce_bf16_kernel(const float* part, int splits, long long count, bf16* out) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += part[s * count + i];
    out[i] = __float2bfloat16_rn(acc);
  }
}

}  // namespace tc
}  // namespace mla

// ---------------------------------------------------------------------------
// entry points used by mla_abi.cu
// ---------------------------------------------------------------------------
using namespace mla;
using namespace mla::tc;

struct TcDecodeWs {
  size_t Yp, qn, q_nope, wo_part, oy, bf16c, dq, total;
  int s1, s5;
  bool deq;   // FP8 weights beyond the FP8 GEMM's 128 tokens: dequantise each weight into dq, bf16 GEMMs
};

static inline size_t tc_prefill_dequant_bytes(const mla_handle* h);

static TcDecodeWs tc_decode_ws(const mla_handle* h, long long n) {
  TcDecodeWs w{};
  const mla_config& c = h->cfg;
  const WeightLayout& L = h->L;
  const int sms = h->tc.num_sms > 0 ? h->tc.num_sms : 148;
  w.deq = h->tc.fp8 && n > 128;
  const int ku = h->tc.fp8 && !w.deq ? 128 : 64;   // K block of the GEMM kernel in use
  // The FP8 kernel's fold warps store a finished unit themselves, behind the code stream: about
  // six K blocks of time for a 128-token fp32 partial (the bf16 kernel's epilogue warps overlap it).
  const int epi = h->tc.fp8 && !w.deq ? FP8_EPI_BLOCKS : 0;
  w.s1 = decode_splits_for((int)cdiv(L.N1, 128), (int)cdiv(c.hidden, ku), sms, epi);
  const long long ko = L.G ? (long long)L.G * L.ro : (long long)c.n_heads * c.v_dim;   // K of the last projection
  w.s5 = decode_splits_for((int)cdiv(c.hidden, 128), (int)cdiv(ko, ku), sms, epi);
  size_t off = 0;
  auto put = [&](size_t b) { size_t o = off; off = align_up(off + b, 256); return o; };
  w.Yp = put((size_t)w.s1 * n * L.N1 * 4);
  w.qn = put((size_t)n * (c.q_lora_rank ? c.q_lora_rank : 8) * 2);
  w.q_nope = put((size_t)n * c.n_heads * c.qk_nope * 2);
  w.wo_part = put((size_t)w.s5 * n * c.hidden * 4);
  if (L.G) w.oy = put((size_t)n * L.G * L.ro * 2);   // grouped output projection: the low-rank rows (bf16)
  if (w.deq) w.dq = put(tc_prefill_dequant_bytes(h));   // one dequantised weight at a time
  if (h->tc.fp8 && !w.deq) {   // f16 copy of the largest token operand of an FP8 GEMM
    long long e = c.hidden;
    if (c.q_lora_rank > e) e = c.q_lora_rank;
    if ((long long)c.n_heads * c.qk_nope > e) e = (long long)c.n_heads * c.qk_nope;
    if ((long long)c.n_heads * c.kv_lora_rank > e) e = (long long)c.n_heads * c.kv_lora_rank;
    if ((long long)c.n_heads * c.v_dim > e) e = (long long)c.n_heads * c.v_dim;
    w.bf16c = put((size_t)n * e * 2 + 16);
  }
  w.total = off;
  return w;
}

static inline size_t tc_decode_ws_bytes(const mla_handle* h, long long n, int) {
  if (!h->tc.enabled && !h->tc.fp8) return 0;
  return tc_decode_ws(h, n).total;
}

static inline int tc_init(mla_handle* h) {
  TcState& T = h->tc;
  T.enabled = 0;
  T.attn = 0;
  T.fp8 = 0;
  T.pf8 = 0;
  int dev = 0, major = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&T.num_sms, cudaDevAttrMultiProcessorCount, dev);
  const mla_config& c = h->cfg;
  T.attn = (major == 10 && c.act_dtype == MLA_BF16) ? 1 : 0;
  if (major == 10 && c.act_dtype == MLA_BF16 && c.weight_dtype == MLA_FP8_E4M3_B128 && c.hidden % 128 == 0 &&
      c.kv_lora_rank % 128 == 0 && ((long long)c.n_heads * c.v_dim) % 128 == 0 && (c.qk_nope + c.qk_rope) % 2 == 0) {
    const WeightLayout& L = h->L;
    const char* b = h->base;
    const long long H = c.n_heads, dn = c.qk_nope, dv = c.v_dim, rkv = c.kv_lora_rank, D = c.hidden;
    const long long rq = c.q_lora_rank;
    int st = MLA_OK;
    st |= make_map(&T.a8_W1, b + L.W1, D, L.N1, 1, D, D * L.N1, 128, 0, true);
    if (rq) st |= make_map(&T.a8_Wqb, b + L.Wqb, rq, L.Hq, 1, rq, rq * L.Hq, 128, 0, true);
    st |= make_map(&T.a8_Wuk, b + L.Wuk, dn, rkv, H, dn, rkv * dn, 128, 0, true);
    st |= make_map(&T.a8_Wuv, b + L.Wuv, rkv, dv, H, rkv, dv * rkv, 128, 0, true);
    st |= make_map(&T.a8_Wo, b + L.Wo, H * dv, D, 1, H * dv, H * dv * D, 128, 0, true);
    if (st == MLA_OK) T.fp8 = 1;
    // prefill: the same shape limits as the bf16 tensor-core prefill
    if (c.hidden % 64 == 0 && c.kv_lora_rank % 64 == 0 && c.qk_nope % 64 == 0 && c.q_lora_rank % 64 == 0 &&
        ((long long)c.n_heads * c.v_dim) % 64 == 0)
      T.pf8 = 1;
    return MLA_OK;
  }
  if (major != 10 || c.act_dtype != MLA_BF16 || c.weight_dtype != MLA_BF16) return MLA_OK;
  if (c.hidden % 64 || c.kv_lora_rank % 64 || c.qk_nope % 64 || c.q_lora_rank % 64 ||
      ((long long)c.n_heads * c.v_dim) % 64 || (c.qk_nope + c.qk_rope) % 2)
    return MLA_OK;
  const WeightLayout& L = h->L;
  const char* b = h->base;
  const int H = c.n_heads, dn = c.qk_nope, dv = c.v_dim, rkv = c.kv_lora_rank, D = c.hidden, rq = c.q_lora_rank;
  int st = MLA_OK;
  st |= make_map2(&T.a_W1, b + L.W1, D, L.N1, D, 128);
  if (rq) st |= make_map2(&T.a_Wqb, b + L.Wqb, rq, L.Hq, rq, 128);
  st |= make_map(&T.a_Wuk, b + L.Wuk, dn, rkv, H, (long long)dn * 2, (long long)rkv * dn * 2, 128, 0);
  st |= make_map(&T.a_Wuv, b + L.Wuv, rkv, dv, H, (long long)rkv * 2, (long long)dv * rkv * 2, 128, 0);
  if (L.G) {
    st |= make_map(&T.a_Woa, b + L.Woa, L.Kg, L.ro, L.G, (long long)L.Kg * 2, (long long)L.ro * L.Kg * 2, 128, 0);
    st |= make_map2(&T.a_Wob, b + L.Wob, (long long)L.G * L.ro, D, (long long)L.G * L.ro, 128);
  } else {
    st |= make_map2(&T.a_Wo, b + L.Wo, (long long)H * dv, D, (long long)H * dv, 128);
  }
  st |= make_map2(&T.b_W1, b + L.W1, D, L.N1, D, 256);
  st |= make_map2(&T.b_W1q, b + L.W1, D, L.Nq1, D, 256);
  st |= make_map2(&T.b_W1kv, b + L.W1 + (size_t)L.Nq1 * D * 2, D, L.R, D, 256);
  if (rq) st |= make_map2(&T.b_Wqb, b + L.Wqb, rq, L.Hq, rq, 256);
  st |= make_map2(&T.b_Wkvb, b + L.Wkvb, rkv, L.Hkv, rkv, 256);
  if (L.G) {
    T.bn_oa = L.ro % 256 == 0 ? 256 : (L.ro % 128 == 0 ? 128 : 64);
    st |= make_map(&T.b_Woa, b + L.Woa, L.Kg, L.ro, L.G, (long long)L.Kg * 2, (long long)L.ro * L.Kg * 2, T.bn_oa, 0);
    st |= make_map2(&T.b_Wob, b + L.Wob, (long long)L.G * L.ro, D, (long long)L.G * L.ro, 256);
  } else {
    st |= make_map2(&T.b_Wo, b + L.Wo, (long long)H * dv, D, (long long)H * dv, 256);
  }
  if (st != MLA_OK) return MLA_OK;   // stay on the CUDA-core path
  T.enabled = 1;
  return MLA_OK;
}

// FP8 weights take the FP8 GEMMs up to 128 tokens and, up to 256, the bf16
// GEMMs on weights dequantised per call (flattening the per-head W_UK / W_UV
// scale blocks needs r_kv and d_v to be multiples of 128).
static inline bool tc_decode_fp8_dequant_ok(const mla_handle* h) {
  return h->tc.pf8 && h->cfg.v_dim % 128 == 0 && h->cfg.kv_lora_rank % 128 == 0;
}
static inline bool tc_decode_qkv_supported(const mla_handle* h, int n) {
  return (h->tc.enabled && n <= 256) || (h->tc.fp8 && n <= 128) || (tc_decode_fp8_dequant_ok(h) && n <= 256);
}
static inline bool tc_decode_attn_supported(const mla_handle* h, int n, int) {
  return (h->tc.enabled && n <= 256) || (h->tc.fp8 && n <= 128) || (tc_decode_fp8_dequant_ok(h) && n <= 256);
}

static inline bool tc_attention_supported(const mla_handle* h) { return h->tc.attn != 0; }
static inline bool tc_prefill_supported(const mla_handle* h, int) { return h->tc.enabled || h->tc.pf8; }

// Bytes of the bf16 buffer FP8 handles dequantise each prefill weight into (the largest of them).
static inline size_t tc_prefill_dequant_bytes(const mla_handle* h) {
  if (!h->tc.pf8) return 0;
  const WeightLayout& L = h->L;
  const mla_config& c = h->cfg;
  long long m = (long long)L.N1 * c.hidden;
  if (c.q_lora_rank) m = m > (long long)L.Hq * c.q_lora_rank ? m : (long long)L.Hq * c.q_lora_rank;
  m = m > (long long)L.Hkv * c.kv_lora_rank ? m : (long long)L.Hkv * c.kv_lora_rank;
  m = m > (long long)c.hidden * c.n_heads * c.v_dim ? m : (long long)c.hidden * c.n_heads * c.v_dim;
  return (size_t)m * 2;
}

// The B-operand map (256-row boxes) of prefill weight [N, K] starting at row
// `row0`: the resident bf16 weights, or, for FP8 handles, the weight just
// dequantised into `dq` (rows [0, N) of it; launched here, on `s`).
static inline int prefill_weight_map(const mla_handle* h, CUtensorMap* m, const CUtensorMap& bf16_map,
                                     size_t codes_off, size_t scales_off, long long N, long long K, long long row0,
                                     long long rows, char* dq, bool dequant, cudaStream_t s) {
  if (!h->tc.pf8) { *m = bf16_map; return MLA_OK; }
  if (dequant) {
    const long long total = N * (K / 16);
    const int blocks = (int)(cdiv(total, 256) > 8 * 148 ? 8 * 148 : cdiv(total, 256));
    dequant_fp8_bf16_kernel<<<blocks, 256, 0, s>>>((const uint8_t*)(h->base + codes_off),
                                                   (const float*)(h->base + scales_off), N, K, (bf16*)dq);
    mla_count_launch(1);
  }
  return make_map2(m, dq + (size_t)row0 * K * 2, K, rows, K, 256);
}

enum WSel { W_1, W_QB, W_UK, W_UV, W_O, W_OA, W_OB };

// Token operand of a decode GEMM: a bf16 3-D view {K, d1, d2} (strides in
// elements) over `elems` contiguous elements, rows in dimension rows_dim2 + 1.
struct BView {
  const void* p;
  long long K, d1, d2, s1, s2, elems;
  int rows_dim2;
  int f16;   // the tokens are f16 already (an FP8-weight GEMM then reads them as they are)
};

static BView bview2(const void* p, long long K, long long rows, int f16 = 0) {
  return BView{p, K, rows, 1, K, K * rows, K * rows, 0, f16};
}

// Weight GEMM of the decode path: bf16 weights on tc_gemm_kernel, FP8 weights
// on tc_gemm_fp8_kernel (bf16 tokens converted to f16 into `f16buf` first,
// f16 tokens read as they are) with the matrix's block scales, or, given `dq`,
// on tc_gemm_kernel after dequantising the weight into it.
static int wgemm_body(const mla_handle* h, WSel w, const BView& bv, GemmArgs g, int bn, int splits, void* f16buf,
                      char* dq, cudaStream_t s);

// Kernel-timer names of the decode weight GEMMs (mla_set_kernel_timer).
static const char* wgemm_name(WSel w) {
  return w == W_1 ? "gemm_w1" : w == W_QB ? "gemm_qb" : w == W_UK ? "gemm_uk" : w == W_UV ? "gemm_uv"
         : w == W_OA ? "gemm_oa" : w == W_OB ? "gemm_ob" : "gemm_o";
}

static int wgemm(const mla_handle* h, WSel w, const BView& bv, GemmArgs g, int bn, int splits, void* f16buf,
                 char* dq, cudaStream_t s) {
  mla_timer_begin(wgemm_name(w), s);
  const int st = wgemm_body(h, w, bv, g, bn, splits, f16buf, dq, s);
  mla_timer_end(wgemm_name(w), s);
  return st;
}

static int wgemm_body(const mla_handle* h, WSel w, const BView& bv, GemmArgs g, int bn, int splits, void* f16buf,
                      char* dq, cudaStream_t s) {
  const TcState& T = h->tc;
  CUtensorMap B;
  int st;
  g.b_rows_dim2 = bv.rows_dim2;
  if (!T.fp8) {
    if ((st = make_map(&B, bv.p, bv.K, bv.d1, bv.d2, bv.s1 * 2, bv.s2 * 2, bn, bv.rows_dim2)) != MLA_OK) return st;
    const CUtensorMap* A = w == W_1 ? &T.a_W1 : w == W_QB ? &T.a_Wqb : w == W_UK ? &T.a_Wuk : w == W_UV ? &T.a_Wuv
                           : w == W_OA ? &T.a_Woa : w == W_OB ? &T.a_Wob : &T.a_Wo;
    return launch_gemm(*A, B, g, bn, splits, T.num_sms, s);
  }
  if (dq) {
    // FP8 weights, more tokens than the FP8 GEMM takes: dequantise the weight to bf16
    // [N, K] (per-head blocks stacked) and run the bf16 GEMM on it; the GEMM must not
    // load the weight ahead of its dependency wait
    const WeightLayout& L = h->L;
    const mla_config& c = h->cfg;
    const long long D = c.hidden, rq = c.q_lora_rank, dn = c.qk_nope, dv = c.v_dim, rkv = c.kv_lora_rank;
    const long long H = c.n_heads;
    size_t co, so;
    long long N, K;
    switch (w) {
      case W_1: co = L.W1; so = L.sW1; N = L.N1; K = D; break;
      case W_QB: co = L.Wqb; so = L.sWqb; N = L.Hq; K = rq; break;
      case W_UK: co = L.Wuk; so = L.sWuk; N = H * rkv; K = dn; break;
      case W_UV: co = L.Wuv; so = L.sWuv; N = H * dv; K = rkv; break;
      default: co = L.Wo; so = L.sWo; N = D; K = H * dv; break;
    }
    const long long total = N * (K / 16);
    const int blocks = (int)(cdiv(total, 256) > 8 * 148 ? 8 * 148 : cdiv(total, 256));
    dequant_fp8_bf16_kernel<<<blocks, 256, 0, s>>>((const uint8_t*)(h->base + co), (const float*)(h->base + so), N,
                                                   K, (bf16*)dq);
    mla_count_launch(1);
    CUtensorMap A;
    if (w == W_UK) st = make_map(&A, dq, dn, rkv, H, dn * 2, rkv * dn * 2, 128, 0);
    else if (w == W_UV) st = make_map(&A, dq, rkv, dv, H, rkv * 2, dv * rkv * 2, 128, 0);
    else st = make_map2(&A, dq, K, N, K, 128);
    if (st != MLA_OK) return st;
    if ((st = make_map(&B, bv.p, bv.K, bv.d1, bv.d2, bv.s1 * 2, bv.s2 * 2, bn, bv.rows_dim2)) != MLA_OK) return st;
    g.static_op = 0;
    return launch_gemm(A, B, g, bn, splits, T.num_sms, s);
  }
  const void* tok = bv.p;
  if (!bv.f16) {
    if ((((uintptr_t)bv.p) & 15) || (bv.elems % 8)) return MLA_ERR_UNSUPPORTED;
    const long long n8 = bv.elems / 8;
    const unsigned blocks = (unsigned)(cdiv(n8, 256) < 2048 ? cdiv(n8, 256) : 2048);
    launch_pdl(cvt_bf16_f16_kernel, blocks, 256, 0, s, (const uint4*)bv.p, (uint4*)f16buf, n8);
    mla_count_launch(1);
    tok = f16buf;
  }
  if ((st = make_map(&B, tok, bv.K, bv.d1, bv.d2, bv.s1 * 2, bv.s2 * 2, bn, bv.rows_dim2)) != MLA_OK) return st;
  const WeightLayout& L = h->L;
  const mla_config& c = h->cfg;
  const char* base = h->base;
  const long long D = c.hidden, rq = c.q_lora_rank, dn = c.qk_nope, dv = c.v_dim, rkv = c.kv_lora_rank;
  const long long H = c.n_heads;
  const CUtensorMap* A;
  const float* sc;
  long long ld, bs = 0;
  switch (w) {
    case W_1: A = &T.a8_W1; sc = (const float*)(base + L.sW1); ld = cdiv(D, 128); break;
    case W_QB: A = &T.a8_Wqb; sc = (const float*)(base + L.sWqb); ld = cdiv(rq, 128); break;
    case W_UK: A = &T.a8_Wuk; sc = (const float*)(base + L.sWuk); ld = cdiv(dn, 128); bs = cdiv(rkv, 128) * ld; break;
    case W_UV: A = &T.a8_Wuv; sc = (const float*)(base + L.sWuv); ld = cdiv(rkv, 128); bs = cdiv(dv, 128) * ld; break;
    default: A = &T.a8_Wo; sc = (const float*)(base + L.sWo); ld = cdiv(H * dv, 128); break;
  }
  return launch_gemm_fp8(*A, B, g, bn, splits, sc, ld, bs, T.num_sms, s);
}

static GemmArgs gemm_args(int M, int N, int K, int batches, int mode, void* out, long long ldo, long long bstride,
                          int* flag) {
  GemmArgs g{};
  g.M = M; g.N = N; g.K = K; g.batches = batches; g.mode = mode; g.out = out; g.ldo = ldo; g.bstride = bstride;
  g.flag = flag;
  // decode GEMMs run swap-AB (A = the weights), prefill GEMMs with B = the weights
  g.static_op = (mode == EPI_F32_T || mode == EPI_BF16_T || mode == EPI_QROPE_T) ? 1 : 2;
  return g;
}

static inline int tc_decode_qkv(const mla_handle* h, const void* hidden, int n, const float* cos, const float* sin,
                                void* kv_cache, int n_blocks, const int32_t* slot_mapping, void* q_abs, void* q_pe,
                                char* ws, size_t tc_off, cudaStream_t s) {
  const mla_config& c = h->cfg;
  const WeightLayout& L = h->L;
  const TcDecodeWs W = tc_decode_ws(h, n);
  char* tw = ws + tc_off;
  int* flag = (int*)ws;
  const int H = c.n_heads, dn = c.qk_nope, dr = c.qk_rope, rkv = c.kv_lora_rank, D = c.hidden, rq = c.q_lora_rank;
  const int bn = pick_bn(n);
  int st;
  // 1. Yp[split] = x @ W1 (swap-AB: A = W1 [N1, D], B = x [n, D])
  void* f16buf = tw + W.bf16c;
  char* dq = W.deq ? tw + W.dq : nullptr;
  // with the FP8-weight GEMM, the activations only it reads are written in f16
  const int af16 = h->tc.fp8 && !W.deq;
  GemmArgs g = gemm_args(L.N1, n, D, 1, EPI_F32_T, tw + W.Yp, L.N1, 0, flag);
  if ((st = wgemm(h, W_1, bview2(hidden, D, n), g, bn, W.s1, f16buf, dq, s)) != MLA_OK) return st;
  // 2. split sum, norms, RoPE, scatter (and, without q_lora, q_nope / q_pe)
  FrontFoldTcArgs f{};
  f.Yp = (const float*)(tw + W.Yp); f.split_stride = (long long)n * L.N1; f.splits = W.s1; f.N1 = L.N1;
  f.rq = rq; f.Nq1 = L.Nq1; f.rkv = rkv; f.dr = dr; f.H = H; f.dn = dn;
  f.q_norm_w = rq ? (const float*)(h->base + L.gq) : nullptr;
  f.kv_norm_w = (const float*)(h->base + L.gkv); f.eps = c.norm_eps;
  f.cos = cos; f.sin = sin;
  f.qn = (bf16*)(tw + W.qn); f.q_nope = (bf16*)(tw + W.q_nope); f.q_pe = (bf16*)q_pe; f.act_f16 = af16;
  f.cache = (bf16*)kv_cache; f.n_rows = (long long)n_blocks * c.block_size; f.slot = slot_mapping;
  f.layout = c.row_layout; f.flag = flag;
  // the q part in slices: all of r_q (its RMSNorm spans it), or about a third
  // of the heads each without q_lora; the kv part in CTA 0
  const int hd = dn + dr;
  f.q_cols = rq ? rq : (int)cdiv(H, 3) * hd;
  const int q_slices = (int)cdiv(L.Nq1, f.q_cols);
  const size_t ff_smem = (size_t)(f.q_cols > L.R ? f.q_cols : L.R) * 4;
  if (ff_smem > 48 * 1024) cudaFuncSetAttribute(frontfold_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ff_smem);
  launch_pdl(frontfold_tc_kernel, dim3(n, 1 + q_slices), 512, ff_smem, s, f);
  mla_count_launch(1);
  // 3. q = qn @ wq_b with q_nope out and RoPE(q_pe) out (swap-AB)
  if (rq) {

    GemmArgs g2 = gemm_args(L.Hq, n, rq, 1, EPI_QROPE_T, tw + W.q_nope, 0, 0, flag);
    g2.out2 = q_pe; g2.cos = cos; g2.sin = sin; g2.H = H; g2.dn = dn; g2.dr = dr; g2.out_f16 = af16;
    if ((st = wgemm(h, W_QB, bview2(tw + W.qn, rq, n, af16), g2, bn, 1, f16buf, dq, s)) != MLA_OK) return st;
  }
  // 4. q_abs[h] = q_nope[h] @ W_UK[h]  (batched over heads: A = Wuk[h] [r_kv, d_n], B = q_nope[:, h, :])
  const BView vn{tw + W.q_nope, dn, H, n, dn, (long long)H * dn, (long long)n * H * dn, 1, af16};
  GemmArgs g3 = gemm_args(rkv, n, dn, H, EPI_BF16_T, q_abs, (long long)H * rkv, rkv, flag);
  g3.b_rows_dim2 = 1;
  return wgemm(h, W_UK, vn, g3, bn, 1, f16buf, dq, s);
}

// Split-KV absorbed attention and the LSE merge of the splits -> o_lat (bf16).
// tcgen05 kernel for the DeepSeek latent dims, CUDA-core kernel otherwise.
static inline int tc_attention_core(const mla_handle* h, const void* q_abs, const void* q_pe, const void* kv_cache,
                                    int n_blocks, const int32_t* block_table, int mbps, const int32_t* ctx,
                                    int max_ctx, int n, float* part_o, float* part_ml, int splits, bf16* o_lat,
                                    int* flag, int* nseg, cudaStream_t s, int olat_f16 = 0) {
  const mla_config& c = h->cfg;
  const TcState& T = h->tc;
  const int H = c.n_heads, dr = c.qk_rope, rkv = c.kv_lora_rank;
  int st;
  // 1. split-KV absorbed attention and the LSE merge -> o_lat (bf16)
  const int R = rkv + dr;
  const float* sink = h->has_sink ? (const float*)(h->base + h->L.sink) : nullptr;
  long long ml_r = 0;         // offset of the second CTA's (m, l) copy (tensor-core kernels)
  int half_cols = 0;          // latent columns per (m, l) copy (0: one copy)
  int* seg_counts = nullptr;  // split partials per sequence, when a kernel reports them
  const bool latent_ok = rkv == 512 && dr == 64 && c.block_size % 64 == 0 && (((uintptr_t)q_abs) & 15) == 0 &&
                         (((uintptr_t)q_pe) & 15) == 0;
  if (latent_ok && H <= 32) {
    // few heads: transposed tiles, one 2-CTA cluster per (sequence, split).
    // Pick the split length (whole 128-row tiles) that minimises waves x tiles
    // per cluster.
    const int sms = T.num_sms > 0 ? T.num_sms : 148;
    const int tiles = (int)cdiv(max_ctx, 128);
    int best_ct = tiles, best_cost = 1 << 30;
    for (int ct = 1; ct <= tiles; ++ct) {
      const int spl = (int)cdiv(tiles, ct);
      if (spl > splits) continue;
      const int waves = (int)cdiv(2LL * n * spl, sms);
      const int cost = waves * (ct + 2);   // + per-cluster set-up, in tiles
      if (cost < best_cost) { best_cost = cost; best_ct = ct; }
    }
    const int chunk = best_ct * 128;
    const int sp = (int)cdiv(max_ctx, chunk);
    splits = sp;
    const int NH = H <= 16 ? 16 : 32;
    CUtensorMap mqa, mqp, mc, ml;
    if ((st = make_map2(&mqa, q_abs, rkv, (long long)n * H, rkv, NH)) != MLA_OK) return st;
    if ((st = make_map2(&mqp, q_pe, dr, (long long)n * H, dr, NH)) != MLA_OK) return st;
    if ((st = make_map2(&mc, kv_cache, R, (long long)n_blocks * c.block_size, R, 64)) != MLA_OK) return st;
    if ((st = make_map_cache_groups(&ml, kv_cache, R, (long long)n_blocks * c.block_size, 2)) != MLA_OK) return st;
    TcAttnArgs ta{};
    ta.n = n; ta.H = H; ta.splits = sp; ta.chunk = chunk;
    ta.bs = c.block_size; ta.n_blocks = n_blocks; ta.mbps = mbps; ta.max_ctx = max_ctx;
    ta.block_table = block_table; ta.ctx = ctx; ta.q_abs = (const bf16*)q_abs;
    ta.lat_col0 = c.row_layout == MLA_ROW_LATENT_FIRST ? 0 : dr;
    ta.rope_col0 = c.row_layout == MLA_ROW_LATENT_FIRST ? rkv : 0;
    ta.scale_log2 = h->scale * 1.4426950408889634f;
    ta.part_o = part_o; ta.part_ml = part_ml; ta.flag = flag;
    ta.ml_r = ml_r = (long long)n * sp * H * 2;   // CTA r's (m, l) copy, one per latent half
    half_cols = 256;
    static std::atomic<bool> attr16[64], attr32[64];
    mla_timer_begin("attn", s);
    if (NH == 16) {
      set_smem_once(attr16, tc_attn_pair_kernel<16>, AttnPairSmem<16>::SIZE);
      launch_pdl(tc_attn_pair_kernel<16>, 2 * n * sp, 224, AttnPairSmem<16>::SIZE, s, mqa, mqp, mc, ml, ta);
    } else {
      set_smem_once(attr32, tc_attn_pair_kernel<32>, AttnPairSmem<32>::SIZE);
      launch_pdl(tc_attn_pair_kernel<32>, 2 * n * sp, 224, AttnPairSmem<32>::SIZE, s, mqa, mqp, mc, ml, ta);
    }
    mla_timer_end("attn", s);
    mla_count_launch(1);
  } else if (latent_ok && H <= 128 && n <= ATT_MAX_SEQ && splits >= 2) {
    // persistent and balanced: one 2-CTA cluster per SM pair, each an equal
    // slice of the batch's 64-row tiles; a slice holds at least `min_per` tiles
    // so that no sequence spreads over more segments than the workspace holds
    const int pairs = T.num_sms / 2 > 0 ? T.num_sms / 2 : 74;
    const int max_tiles = (int)cdiv(max_ctx, 64);
    CUtensorMap mc, ml;
    if ((st = make_map2(&mc, kv_cache, R, (long long)n_blocks * c.block_size, R, 64)) != MLA_OK) return st;
    if ((st = make_map_cache_groups(&ml, kv_cache, R, (long long)n_blocks * c.block_size, 4)) != MLA_OK) return st;
    TcAttnArgs ta{};
    ta.n = n; ta.H = H; ta.splits = splits; ta.chunk = 0;
    ta.bs = c.block_size; ta.n_blocks = n_blocks; ta.mbps = mbps; ta.max_ctx = max_ctx;
    ta.block_table = block_table; ta.ctx = ctx; ta.q_abs = (const bf16*)q_abs; ta.q_pe = (const bf16*)q_pe;
    ta.lat_col0 = c.row_layout == MLA_ROW_LATENT_FIRST ? 0 : dr;
    ta.rope_col0 = c.row_layout == MLA_ROW_LATENT_FIRST ? rkv : 0;
    ta.scale_log2 = h->scale * 1.4426950408889634f;
    ta.part_o = part_o; ta.part_ml = part_ml; ta.flag = flag;
    ta.ml_r = ml_r = (long long)n * splits * H * 2;
    ta.units = pairs;
    ta.min_per = (int)cdiv(max_tiles, splits - 1);
    ta.nseg = nseg;
    half_cols = 256;
    seg_counts = nseg;
    static std::atomic<bool> attr[64];
    set_smem_once(attr, tc_attn_decode_kernel, AttnSmem::SIZE);
    mla_timer_begin("attn", s);
    launch_pdl(tc_attn_decode_kernel, 2 * pairs, ATT_THREADS, AttnSmem::SIZE, s, mc, ml, ta);
    mla_timer_end("attn", s);
    mla_count_launch(1);
  } else {
    AttnArgs p{};
    p.q_abs = q_abs; p.q_pe = q_pe; p.cache = kv_cache; p.n_blocks = n_blocks; p.bs = c.block_size;
    p.block_table = block_table; p.mbps = mbps; p.ctx = ctx; p.max_ctx = max_ctx;
    p.H = H; p.r_kv = rkv; p.d_r = dr; p.layout = c.row_layout; p.scale = h->scale;
    p.n_splits = splits; p.chunk = (int)cdiv(cdiv(max_ctx, splits), ATT_TR) * ATT_TR;
    p.part_o = part_o; p.part_ml = part_ml; p.flag = flag;
    const size_t smem = (size_t)(ATT_TR * (R + 1) + ATT_HPB * R) * 4;
    cudaFuncSetAttribute(attn_decode_simt_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    mla_timer_begin("attn", s);
    attn_decode_simt_kernel<bf16><<<dim3(splits, n, (unsigned)cdiv(H, ATT_HPB)), 256, smem, s>>>(p);
    mla_timer_end("attn", s);
    mla_count_launch(1);
  }
  if (olat_f16)   // its only reader is an FP8-weight GEMM
    launch_pdl(attn_combine_kernel<__half>, dim3(n, H), 128, 0, s, (const float*)part_o, (const float*)part_ml, splits,
               H, rkv, (__half*)o_lat, sink, ml_r, half_cols, (const int*)seg_counts);
  else
    launch_pdl(attn_combine_kernel<bf16>, dim3(n, H), 128, 0, s, (const float*)part_o, (const float*)part_ml, splits,
               H, rkv, o_lat, sink, ml_r, half_cols, (const int*)seg_counts);
  mla_count_launch(1);
  return MLA_OK;
}

static inline int tc_decode_attn(const mla_handle* h, const void* q_abs, const void* q_pe, const void* kv_cache,
                                 int n_blocks, const int32_t* block_table, int mbps, const int32_t* ctx,
                                 int max_ctx, int n, void* out, void* head, char* ws, size_t tc_off,
                                 cudaStream_t s, float* part_o, float* part_ml, int splits, bf16* o_lat,
                                 int* nseg, bool head_internal) {
  const mla_config& c = h->cfg;
  const TcDecodeWs W = tc_decode_ws(h, n);
  char* tw = ws + tc_off;
  int* flag = (int*)ws;
  const int H = c.n_heads, rkv = c.kv_lora_rank, dv = c.v_dim, D = c.hidden;
  const int bn = pick_bn(n);
  // with the FP8-weight GEMM, o_lat, the head outputs (unless the caller asked for
  // them) and the grouped low-rank rows are written in f16: only those GEMMs read them
  const int af16 = h->tc.fp8 && !W.deq, hf16 = af16 && head_internal;
  int st = tc_attention_core(h, q_abs, q_pe, kv_cache, n_blocks, block_table, mbps, ctx, max_ctx, n, part_o,
                             part_ml, splits, o_lat, flag, nseg, s, af16);
  if (st != MLA_OK) return st;
  // 2. head_out[h] = o_lat[h] @ W_UV[h]  (A = Wuv[h] [d_v, r_kv], B = o_lat[:, h, :])
  void* f16buf = tw + W.bf16c;
  char* dq = W.deq ? tw + W.dq : nullptr;
  const BView vo{o_lat, rkv, H, n, rkv, (long long)H * rkv, (long long)n * H * rkv, 1, af16};
  GemmArgs g4 = gemm_args(dv, n, rkv, H, EPI_BF16_T, head, (long long)H * dv, dv, flag);
  g4.b_rows_dim2 = 1;
  g4.out_f16 = hf16;
  if ((st = wgemm(h, W_UV, vo, g4, bn, 1, f16buf, dq, s)) != MLA_OK) return st;
  // 3. out = head_out @ wo  (swap-AB, K split, then reduce to bf16); or, grouped,
  //    y[:, g] = head_out[:, group g] @ wo_a block g (batched over the groups:
  //    A = Woa[g] [r_o, Kg], B = the group's head outputs), then out = y @ wo_b
  const WeightLayout& L = h->L;
  if (L.G) {
    const BView vg{head, L.Kg, L.G, n, L.Kg, (long long)H * dv, (long long)n * H * dv, 1, hf16};
    GemmArgs ga = gemm_args(L.ro, n, L.Kg, L.G, EPI_BF16_T, tw + W.oy, (long long)L.G * L.ro, L.ro, flag);
    ga.b_rows_dim2 = 1;
    ga.out_f16 = af16;
    if ((st = wgemm(h, W_OA, vg, ga, bn, 1, f16buf, dq, s)) != MLA_OK) return st;
    GemmArgs gb = gemm_args(D, n, L.G * L.ro, 1, EPI_F32_T, tw + W.wo_part, D, 0, flag);
    if ((st = wgemm(h, W_OB, bview2(tw + W.oy, (long long)L.G * L.ro, n, af16), gb, bn, W.s5, f16buf, dq, s)) !=
        MLA_OK)
      return st;
  } else {
    GemmArgs g5 = gemm_args(D, n, H * dv, 1, EPI_F32_T, tw + W.wo_part, D, 0, flag);
    if ((st = wgemm(h, W_O, bview2(head, (long long)H * dv, n, hf16), g5, bn, W.s5, f16buf, dq, s)) != MLA_OK)
      return st;
  }
  const long long cnt = (long long)n * D;
  launch_pdl(splitk_reduce_bf16_kernel, (unsigned)cdiv(cnt, 256) < 4096 ? (unsigned)cdiv(cnt, 256) : 4096, 256, 0, s,
             (const float*)(tw + W.wo_part), W.s5, cnt, (bf16*)out);
  mla_count_launch(1);
  return MLA_OK;
}

// DeepSeek-V4 QKV projection on the prefill tensor-core GEMMs ("QKV CTE MLA
// Kernel API Reference", qkv_mla_mx_deepseek_v4): Y1 = x @ [wq_a | wkv_a]
// (fp32), the front-fold in its V4 form (q latent RMSNorm -> qn; the whole kv
// row RMS-normed with kv_norm_w [r_kv + d_r], its tail rotated -> kv_out),
// q = qn @ wq_b written as bf16 into q_out, then each head normalised without
// gain and its tail rotated in place. FP8 handles dequantise each weight first.
static inline int tc_v4_qkv(const mla_handle* h, const void* hidden, int S, const float* cos, const float* sin,
                            const float* kv_norm_w, void* q_out, void* kv_out, char* ws, size_t pY1, size_t pqn,
                            size_t pDQ, cudaStream_t s) {
  const mla_config& c = h->cfg;
  const WeightLayout& L = h->L;
  const TcState& T = h->tc;
  int* flag = (int*)ws;
  const int H = c.n_heads, dn = c.qk_nope, dr = c.qk_rope, rkv = c.kv_lora_rank, D = c.hidden;
  const int rq = c.q_lora_rank;
  int st;
  char* dq = T.pf8 ? ws + pDQ : nullptr;
  const int sop = T.pf8 ? 0 : 2;
  CUtensorMap mx;
  if ((st = make_map2(&mx, hidden, D, S, D, 128)) != MLA_OK) return st;
  float* Y1 = (float*)(ws + pY1);
  GemmArgs g = gemm_args(S, L.N1, D, 1, EPI_F32_N, Y1, L.N1, 0, flag);
  CUtensorMap bw;
  if ((st = prefill_weight_map(h, &bw, T.b_W1, L.W1, L.sW1, L.N1, D, 0, L.N1, dq, true, s)) != MLA_OK) return st;
  g.static_op = sop;
  if ((st = launch_gemm(mx, bw, g, 256, 1, T.num_sms, s)) != MLA_OK) return st;
  FrontFoldArgs f{};
  f.Y = Y1; f.ldy = L.N1; f.kv0 = L.Nq1;
  f.r_q = rq; f.r_kv = rkv; f.d_r = dr;
  f.q_norm_w = (const float*)(h->base + L.gq);
  f.kv_norm_w = kv_norm_w; f.eps = c.norm_eps;
  f.cos = cos; f.sin = sin;
  f.qn = ws + pqn; f.ldqn = rq;
  f.cache = kv_out; f.n_rows = S; f.slot = nullptr; f.layout = MLA_ROW_LATENT_FIRST; f.flag = flag;
  f.v4 = 1;
  launch_pdl(frontfold_epilogue_kernel<bf16>, S, 256, 0, s, f);
  mla_count_launch(1);
  CUtensorMap mq;
  if ((st = make_map2(&mq, ws + pqn, rq, S, rq, 128)) != MLA_OK) return st;
  GemmArgs g2 = gemm_args(S, L.Hq, rq, 1, EPI_BF16_N, q_out, L.Hq, 0, flag);
  CUtensorMap bq;
  if ((st = prefill_weight_map(h, &bq, T.b_Wqb, L.Wqb, L.sWqb, L.Hq, rq, 0, L.Hq, dq, true, s)) != MLA_OK) return st;
  g2.static_op = sop;
  mla_timer_begin("v4_qb", s);
  st = launch_gemm(mq, bq, g2, 256, 1, T.num_sms, s);
  mla_timer_end("v4_qb", s);
  if (st != MLA_OK) return st;
  const int hd = dn + dr;
  if (hd % 8 == 0 && dr % 8 == 0 && hd <= 512 && ((uintptr_t)q_out & 15) == 0)
    launch_pdl(q_headnorm_rope_bf16x8_kernel, dim3(S, (unsigned)cdiv(H, 32)), 256, 0, s, (bf16*)q_out,
               (long long)L.Hq, H, hd, dr, cos, sin, c.norm_eps);
  else
    launch_pdl(q_headnorm_rope_kernel<bf16>, S, 256, 0, s, (bf16*)q_out, (long long)L.Hq, H, hd, dr, cos, sin,
               c.norm_eps);
  mla_count_launch(1);
  return MLA_OK;
}

static inline int tc_prefill(const mla_handle* h, const void* hidden, int S, const float* cos, const float* sin,
                             void* out, void* head, void* kv_cache, int n_blocks, const int32_t* slot_mapping,
                             char* ws, size_t pY1, size_t pqn, size_t pQ, size_t pcn, size_t pkpe, size_t pKV,
                             size_t pDQ, size_t pOY, cudaStream_t s) {
  const mla_config& c = h->cfg;
  const WeightLayout& L = h->L;
  const TcState& T = h->tc;
  int* flag = (int*)ws;
  const int H = c.n_heads, dn = c.qk_nope, dr = c.qk_rope, rkv = c.kv_lora_rank, dv = c.v_dim, D = c.hidden;
  const int rq = c.q_lora_rank;
  int st;
  // FP8 handles dequantise each weight into `dq` just before its GEMM; that GEMM then
  // must not load its weights ahead of its dependency wait (static_op 0)
  char* dq = T.pf8 ? ws + pDQ : nullptr;
  const int sop = T.pf8 ? 0 : 2;
  CUtensorMap mx;
  if ((st = make_map2(&mx, hidden, D, S, D, 128)) != MLA_OK) return st;
  float* Y1 = (float*)(ws + pY1);
  bf16* Q = (bf16*)(ws + pQ);
  FrontFoldArgs f{};
  if (rq) {
    GemmArgs g = gemm_args(S, L.N1, D, 1, EPI_F32_N, Y1, L.N1, 0, flag);
    CUtensorMap bw;
    if ((st = prefill_weight_map(h, &bw, T.b_W1, L.W1, L.sW1, L.N1, D, 0, L.N1, dq, true, s)) != MLA_OK) return st;
    g.static_op = sop;
    if ((st = launch_gemm(mx, bw, g, 256, 1, T.num_sms, s)) != MLA_OK) return st;
    f.Y = Y1; f.ldy = L.N1; f.kv0 = L.Nq1;
  } else {
    GemmArgs gq = gemm_args(S, L.Hq, D, 1, EPI_QROPE_N, Q, L.Hq, 0, flag);
    gq.cos = cos; gq.sin = sin; gq.H = H; gq.dn = dn; gq.dr = dr;
    CUtensorMap bq, bk;
    if ((st = prefill_weight_map(h, &bq, T.b_W1q, L.W1, L.sW1, L.N1, D, 0, L.Nq1, dq, true, s)) != MLA_OK) return st;
    if ((st = prefill_weight_map(h, &bk, T.b_W1kv, L.W1, L.sW1, L.N1, D, L.Nq1, L.R, dq, false, s)) != MLA_OK)
      return st;
    gq.static_op = sop;
    if ((st = launch_gemm(mx, bq, gq, 256, 1, T.num_sms, s)) != MLA_OK) return st;
    GemmArgs gk = gemm_args(S, L.R, D, 1, EPI_F32_N, Y1, L.R, 0, flag);
    gk.static_op = sop;
    if ((st = launch_gemm(mx, bk, gk, 256, 1, T.num_sms, s)) != MLA_OK) return st;
    f.Y = Y1; f.ldy = L.R; f.kv0 = 0;
  }
  f.r_q = rq; f.r_kv = rkv; f.d_r = dr;
  f.q_norm_w = rq ? (const float*)(h->base + L.gq) : nullptr;
  f.kv_norm_w = (const float*)(h->base + L.gkv); f.eps = c.norm_eps;
  f.cos = cos; f.sin = sin;
  f.qn = rq ? ws + pqn : nullptr; f.ldqn = rq;
  f.cache = kv_cache; f.n_rows = (long long)n_blocks * c.block_size;
  f.slot = slot_mapping; f.layout = c.row_layout; f.flag = flag;
  f.cn = ws + pcn; f.kpe = ws + pkpe;
  launch_pdl(frontfold_epilogue_kernel<bf16>, S, 256, 0, s, f);
  mla_count_launch(1);
  if (rq) {
    CUtensorMap mq;
    if ((st = make_map2(&mq, ws + pqn, rq, S, rq, 128)) != MLA_OK) return st;
    GemmArgs g2 = gemm_args(S, L.Hq, rq, 1, EPI_QROPE_N, Q, L.Hq, 0, flag);
    g2.cos = cos; g2.sin = sin; g2.H = H; g2.dn = dn; g2.dr = dr;
    CUtensorMap bw;
    if ((st = prefill_weight_map(h, &bw, T.b_Wqb, L.Wqb, L.sWqb, L.Hq, rq, 0, L.Hq, dq, true, s)) != MLA_OK) return st;
    g2.static_op = sop;
    if ((st = launch_gemm(mq, bw, g2, 256, 1, T.num_sms, s)) != MLA_OK) return st;
  }
  CUtensorMap mc;
  if ((st = make_map2(&mc, ws + pcn, rkv, S, rkv, 128)) != MLA_OK) return st;
  bf16* KV = (bf16*)(ws + pKV);
  GemmArgs g3 = gemm_args(S, L.Hkv, rkv, 1, EPI_BF16_N, KV, L.Hkv, 0, flag);
  CUtensorMap bkv;
  if ((st = prefill_weight_map(h, &bkv, T.b_Wkvb, L.Wkvb, L.sWkvb, L.Hkv, rkv, 0, L.Hkv, dq, true, s)) != MLA_OK)
    return st;
  g3.static_op = sop;
  if ((st = launch_gemm(mc, bkv, g3, 256, 1, T.num_sms, s)) != MLA_OK) return st;
  if (dn == 128 && dr == 64 && dv == 128) {
    CUtensorMap mq, mkv, mkpe;
    if ((st = make_map2(&mq, Q, L.Hq, S, L.Hq, 128)) != MLA_OK) return st;
    if ((st = make_map2(&mkv, KV, L.Hkv, S, L.Hkv, 128)) != MLA_OK) return st;
    if ((st = make_map2(&mkpe, ws + pkpe, dr, S, dr, 128)) != MLA_OK) return st;
    TcPrefillAttnArgs pa{};
    pa.S = S; pa.H = H; pa.q_tiles = (int)cdiv(S, 128);
    pa.scale_log2 = h->scale * 1.4426950408889634f;
    pa.out = (bf16*)head; pa.flag = flag;
    pa.sink = h->has_sink ? (const float*)(h->base + L.sink) : nullptr;
    static std::atomic<bool> attr[64];
    set_smem_once(attr, tc_prefill_attn_kernel, PaSmem::SIZE);
    mla_timer_begin("prefill_attn", s);
    launch_pdl(tc_prefill_attn_kernel, pa.q_tiles * H, 320, PaSmem::SIZE, s, mq, mkv, mkpe, pa);
    mla_timer_end("prefill_attn", s);
    mla_count_launch(1);
  } else {
    PrefillAttnArgs pa{};
    pa.Q = Q; pa.ldq = L.Hq; pa.KV = KV; pa.ldkv = L.Hkv; pa.kpe = ws + pkpe;
    pa.O = head; pa.ldo = (long long)H * dv; pa.S = S; pa.H = H; pa.d_n = dn; pa.d_r = dr; pa.d_v = dv;
    pa.scale = h->scale;
    pa.sink = h->has_sink ? (const float*)(h->base + L.sink) : nullptr;
    const size_t smem = (size_t)(PA_BQ * (dn + dr) + PA_BK * (dn + dr + 1) + PA_BK * dv) * 4;
    cudaFuncSetAttribute(prefill_attn_simt_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    mla_timer_begin("prefill_attn", s);
    prefill_attn_simt_kernel<bf16><<<dim3((unsigned)cdiv(S, PA_BQ), H), 128, smem, s>>>(pa);
    mla_timer_end("prefill_attn", s);
    mla_count_launch(1);
  }
  if (L.G) {
    // grouped output projection: y[t][g r_o + j] = head[t, group g] @ wo_a block g
    // (batched over the groups: A = the group's head outputs {Kg, S, G}, B = Woa),
    // then out = y @ wo_b
    CUtensorMap mg, my;
    if ((st = make_map(&mg, head, L.Kg, S, L.G, (long long)H * dv * 2, (long long)L.Kg * 2, 128, 0)) != MLA_OK)
      return st;
    GemmArgs ga = gemm_args(S, L.ro, L.Kg, L.G, EPI_BF16_N, ws + pOY, (long long)L.G * L.ro, L.ro, flag);
    ga.static_op = sop;
    if ((st = launch_gemm(mg, T.b_Woa, ga, T.bn_oa, 1, T.num_sms, s)) != MLA_OK) return st;
    if ((st = make_map2(&my, ws + pOY, (long long)L.G * L.ro, S, (long long)L.G * L.ro, 128)) != MLA_OK) return st;
    GemmArgs gb = gemm_args(S, D, L.G * L.ro, 1, EPI_BF16_N, out, D, 0, flag);
    gb.static_op = sop;
    return launch_gemm(my, T.b_Wob, gb, 256, 1, T.num_sms, s);
  }
  CUtensorMap mh;
  if ((st = make_map2(&mh, head, (long long)H * dv, S, (long long)H * dv, 128)) != MLA_OK) return st;
  GemmArgs g5 = gemm_args(S, D, H * dv, 1, EPI_BF16_N, out, D, 0, flag);
  CUtensorMap bo;
  if ((st = prefill_weight_map(h, &bo, T.b_Wo, L.Wo, L.sWo, D, (long long)H * dv, 0, D, dq, true, s)) != MLA_OK)
    return st;
  g5.static_op = sop;
  return launch_gemm(mh, bo, g5, 256, 1, T.num_sms, s);
}
