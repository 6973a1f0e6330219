// CUDA-core (SIMT) kernels of the MLA layer step. They carry every dtype the
// library takes (fp32 activations and weights, bf16, FP8-E4M3 block-scaled
// weights) and are the path of the fp32 configuration, whose 1e-4 tolerance
// no tensor-core input format meets. The bf16 / FP8 hot path runs on the
// tcgen05 kernels; these stay as the general-shape path.
#pragma once

#include <math.h>

#include "common.cuh"

namespace mla {

// ---------------------------------------------------------------------------
// Batched linear: C[b][m][n] = sum_k A[b][m][k] * W[b][n][k]   (fp32 accumulate)
// A: activations, K contiguous (row stride lda). W: weights in the library's
// K-major layout [N, K] (row stride ldw). FP8 weights carry fp32 scales per
// 128x128 block of W, [ceil(N/128)][ceil(K/128)] with row stride lds; the
// scale multiplies each dequantised element in fp32 before the MAC ("Struct
// MlaWeights", field wq_a_fp8).
// ---------------------------------------------------------------------------
struct LinearArgs {
  const void* A; long long lda, a_batch;
  const void* W; long long ldw, w_batch;
  const float* scale; long long lds, s_batch;
  void* C; long long ldc, c_batch;
  int M, N, K;
};

constexpr int LIN_BM = 64, LIN_BN = 64, LIN_BK = 32;

template <typename TA, typename TW, typename TC>
__global__ void __launch_bounds__(256) linear_simt_kernel(LinearArgs p) {
  __shared__ float As[LIN_BK][LIN_BM + 4];
  __shared__ float Ws[LIN_BK][LIN_BN + 4];
  const int b = blockIdx.z;
  const TA* A = (const TA*)p.A + (long long)b * p.a_batch;
  const TW* W = (const TW*)p.W + (long long)b * p.w_batch;
  const float* S = p.scale ? p.scale + (long long)b * p.s_batch : nullptr;
  TC* C = (TC*)p.C + (long long)b * p.c_batch;
  const int m0 = blockIdx.y * LIN_BM, n0 = blockIdx.x * LIN_BN;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int lk = tid & 31, lr = tid >> 5;  // loader: k lane, row group
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += LIN_BK) {
    const int k = k0 + lk;
#pragma unroll
    for (int i = 0; i < LIN_BM / 8; ++i) {
      const int r = lr + 8 * i;
      const int m = m0 + r, n = n0 + r;
      float av = 0.f, wv = 0.f;
      if (k < p.K) {
        if (m < p.M) av = to_f32(A[(long long)m * p.lda + k]);
        if (n < p.N) {
          wv = to_f32(W[(long long)n * p.ldw + k]);
          if (S) wv *= S[(long long)(n >> 7) * p.lds + (k >> 7)];
        }
      }
      As[lk][r] = av;
      Ws[lk][r] = wv;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < LIN_BK; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < p.N) C[(long long)m * p.ldc + n] = from_f32<TC>(acc[i][j]);
    }
  }
}

// ---------------------------------------------------------------------------
// Interleaved RoPE of one pair: (a, b) -> (a cos - b sin, a sin + b cos);
// element 2i pairs with 2i+1 ("MLA Decode QKV Kernel API Reference", Notes).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float* o0, float* o1) {
  *o0 = a * c - b * s;
  *o1 = a * s + b * c;
}

// ---------------------------------------------------------------------------
// Front-fold epilogue, one CTA per token. Y is the fp32 output of the merged
// first projection [n, ldy]: columns [0, r_q) = q latent (when r_q > 0),
// [kv0, kv0 + r_kv) = kv latent, [kv0 + r_kv, kv0 + R) = k_pe.
//   q latent -> rms_norm * q_norm_w -> qn (act dtype)              (if qn)
//   kv latent -> rms_norm * kv_norm_w; k_pe -> RoPE; row -> cache   (if cache)
//   and (prefill) the normed latent / rotated k_pe to cn / kpe      (if cn)
// RMSNorm: v * rsqrt(mean(v^2) + eps) * gamma ("MLA Decode QKV Kernel API
// Reference", Parameters q_norm_w, kv_norm_w, norm_eps).
// ---------------------------------------------------------------------------
struct FrontFoldArgs {
  const float* Y; long long ldy;
  int r_q, kv0, r_kv, d_r;
  const float* q_norm_w; const float* kv_norm_w; float eps;
  const float* cos; const float* sin;     // [n, d_r/2]
  void* qn; long long ldqn;               // [n, r_q] act
  void* cache; long long n_rows;          // flat rows [n_rows, R] act
  const int* slot; int layout;
  void* cn; void* kpe;                    // prefill: [n, r_kv], [n, d_r] act
  int* flag;
  // DeepSeek-V4 form ("QKV CTE MLA Kernel API Reference", qkv_mla_mx_deepseek_v4):
  // the whole kv row [r_kv + d_r] is RMS-normed with a gamma of that length and
  // its normed tail is rotated; with slot == NULL row t goes to cache row t
  int v4;
};

template <typename TACT>
__global__ void __launch_bounds__(256) frontfold_epilogue_kernel(FrontFoldArgs p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* y = p.Y + (long long)t * p.ldy;
  if (p.qn) {
    float ss = 0.f;
    for (int i = threadIdx.x; i < p.r_q; i += blockDim.x) ss += y[i] * y[i];
    const float r = rsqrtf(block_sum(ss, red) / (float)p.r_q + p.eps);
    TACT* q = (TACT*)p.qn + (long long)t * p.ldqn;
    for (int i = threadIdx.x; i < p.r_q; i += blockDim.x) q[i] = from_f32<TACT>(y[i] * r * p.q_norm_w[i]);
  }
  const float* kv = y + p.kv0;
  const int R = p.r_kv + p.d_r;
  const int nn = p.v4 ? R : p.r_kv;       // the normed width
  float ss = 0.f;
  for (int i = threadIdx.x; i < nn; i += blockDim.x) ss += kv[i] * kv[i];
  const float r = rsqrtf(block_sum(ss, red) / (float)nn + p.eps);
  TACT* row = nullptr;
  if (p.cache) {
    const int s = p.slot ? p.slot[t] : t;
    if (s >= 0 && (long long)s < p.n_rows) {
      row = (TACT*)p.cache + (long long)s * R;
    } else if (s >= 0) {
      if (threadIdx.x == 0) set_flag(p.flag, MLA_FLAG_BAD_SLOT);
    }
  }
  const int lat_off = (p.layout == MLA_ROW_LATENT_FIRST) ? 0 : p.d_r;
  const int pe_off = (p.layout == MLA_ROW_LATENT_FIRST) ? p.r_kv : 0;
  for (int i = threadIdx.x; i < p.r_kv; i += blockDim.x) {
    const TACT v = from_f32<TACT>(kv[i] * r * p.kv_norm_w[i]);
    if (row) row[lat_off + i] = v;
    if (p.cn) ((TACT*)p.cn)[(long long)t * p.r_kv + i] = v;
  }
  const float* pe = kv + p.r_kv;
  const int half = p.d_r / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    float e0 = pe[2 * i], e1 = pe[2 * i + 1];
    if (p.v4) {
      e0 *= r * p.kv_norm_w[p.r_kv + 2 * i];
      e1 *= r * p.kv_norm_w[p.r_kv + 2 * i + 1];
    }
    float o0, o1;
    rope_pair(e0, e1, p.cos[(long long)t * half + i], p.sin[(long long)t * half + i], &o0, &o1);
    const TACT a = from_f32<TACT>(o0), b = from_f32<TACT>(o1);
    if (row) { row[pe_off + 2 * i] = a; row[pe_off + 2 * i + 1] = b; }
    if (p.kpe) {
      ((TACT*)p.kpe)[(long long)t * p.d_r + 2 * i] = a;
      ((TACT*)p.kpe)[(long long)t * p.d_r + 2 * i + 1] = b;
    }
  }
}

// q_pe of every head: RoPE of Q[t, h*(d_n+d_r) + d_n + ...] -> out[t, h, d_r]
// (out may alias Q's storage when TQ == TOUT and strides match: in place).
template <typename TQ, typename TOUT>
__global__ void q_rope_kernel(const TQ* Q, long long ldq, int H, int d_n, int d_r,
                              const float* cos, const float* sin, TOUT* out, long long ldo,
                              long long out_head_stride, int out_off) {
  const int t = blockIdx.x;
  const int half = d_r / 2;
  for (int idx = threadIdx.x; idx < H * half; idx += blockDim.x) {
    const int h = idx / half, i = idx % half;
    const TQ* q = Q + (long long)t * ldq + (long long)h * (d_n + d_r) + d_n;
    float o0, o1;
    rope_pair(to_f32(q[2 * i]), to_f32(q[2 * i + 1]), cos[(long long)t * half + i],
              sin[(long long)t * half + i], &o0, &o1);
    TOUT* o = out + (long long)t * ldo + (long long)h * out_head_stride + out_off;
    o[2 * i] = from_f32<TOUT>(o0);
    o[2 * i + 1] = from_f32<TOUT>(o1);
  }
}

// ---------------------------------------------------------------------------
// DeepSeek-V4 query heads, in place: each head of q [n, H, hd] (row stride ldq)
// is divided by the root of its mean square (+ eps, no gain), then its last
// d_r entries are rotated by interleaved RoPE at the token's position
// ("QKV CTE MLA Kernel API Reference", qkv_mla_mx_deepseek_v4, Final assembly:
// per-head rsqrt norm, then RoPE on the last rope dims). grid n, 256 threads:
// warp w handles heads w, w + 8, ...
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) q_headnorm_rope_kernel(T* q, long long ldq, int H, int hd, int d_r,
                                                              const float* cos, const float* sin, float eps) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = d_r / 2, base = hd - d_r;
  for (int h = warp; h < H; h += (int)(blockDim.x >> 5)) {
    T* qh = q + (long long)t * ldq + (long long)h * hd;
    float ss = 0.f;
    for (int j = lane; j < hd; j += 32) {
      const float v = to_f32(qh[j]);
      ss += v * v;
    }
    const float r = rsqrtf(warp_sum(ss) / (float)hd + eps);   // every lane has read its entries
    for (int j = lane; j < base; j += 32) qh[j] = from_f32<T>(to_f32(qh[j]) * r);
    for (int i = lane; i < half; i += 32) {
      float o0, o1;
      rope_pair(to_f32(qh[base + 2 * i]) * r, to_f32(qh[base + 2 * i + 1]) * r, cos[(long long)t * half + i],
                sin[(long long)t * half + i], &o0, &o1);
      qh[base + 2 * i] = from_f32<T>(o0);
      qh[base + 2 * i + 1] = from_f32<T>(o1);
    }
  }
}

// The same for bf16 heads with hd and d_r multiples of 8 and 16-byte aligned
// rows: 8 lanes per head, each moving 16-byte chunks (chunk c of the head on
// lane c % 8), so a warp streams four heads with full 128-byte accesses.
// grid (n, ceil(H / 32)), 256 threads; hd <= 512.
__global__ void __launch_bounds__(256) q_headnorm_rope_bf16x8_kernel(bf16* q, long long ldq, int H, int hd, int d_r,
                                                                     const float* cos, const float* sin, float eps) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x, lane = threadIdx.x & 31;
  const int h = blockIdx.y * 32 + (threadIdx.x >> 3);   // 4 heads per warp, 8 lanes per head
  const int i = lane & 7;
  const int nc = hd / 8, base = hd - d_r, half = d_r / 2;
  uint4* qh = reinterpret_cast<uint4*>(q + (long long)t * ldq + (long long)(h < H ? h : 0) * hd);
  uint4 v[8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c = i + 8 * k;
    v[k] = (h < H && c < nc) ? qh[c] : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p2[j]);
      ss += f.x * f.x + f.y * f.y;
    }
  }
  // the head's sum over its 8 lanes (the xor partners stay inside the group)
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  ss += __shfl_xor_sync(0xffffffffu, ss, 4);
  if (h >= H) return;
  const float r = rsqrtf(ss / (float)hd + eps);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c = i + 8 * k;
    if (c >= nc) break;
    __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&v[k]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(p2[j]);
      f.x *= r;
      f.y *= r;
      const int e = 8 * c + 2 * j;   // even element index within the head
      if (e >= base) {
        const int pi = (e - base) / 2;
        float o0, o1;
        rope_pair(f.x, f.y, cos[(long long)t * half + pi], sin[(long long)t * half + pi], &o0, &o1);
        f.x = o0;
        f.y = o1;
      }
      p2[j] = __floats2bfloat162_rn(f.x, f.y);
    }
    qh[c] = v[k];
  }
}

// ---------------------------------------------------------------------------
// Absorbed split-KV decode attention (CUDA cores). grid (n_splits, n, head
// groups of 8), 256 threads: warp w owns head g*8 + w; lane = cache row of the
// current 32-row tile. For its rows [s*chunk, min(L, (s+1)*chunk)) a CTA keeps
// the running max m, sum l and unnormalised o_lat[h] (r_kv) of every head,
//   s_hj = (q_abs[h] . c_j + q_pe[h] . k_pe_j) * scale,
// and writes them as one split partial (merged by attn_combine_kernel).
// ---------------------------------------------------------------------------
struct AttnArgs {
  const void* q_abs; const void* q_pe;    // [n, H, r_kv], [n, H, d_r]
  const void* cache; int n_blocks, bs;    // [n_blocks*bs, R]
  const int* block_table; int mbps;
  const int* ctx; int max_ctx;
  int H, r_kv, d_r, layout;
  float scale;
  int chunk, n_splits;
  float* part_o;                           // [n, n_splits, H, r_kv]
  float* part_ml;                          // [n, n_splits, H, 2]
  int* flag;
};

constexpr int ATT_HPB = 8, ATT_TR = 32;

template <typename T>
__global__ void __launch_bounds__(256) attn_decode_simt_kernel(AttnArgs p) {
  extern __shared__ float smem[];
  const int R = p.r_kv + p.d_r, RP = R + 1;
  float* rows = smem;                       // [ATT_TR][RP]
  float* qf = rows + ATT_TR * RP;           // [ATT_HPB][R], in cache-row order
  __shared__ int valid_row[ATT_TR];
  const int s = blockIdx.x, t = blockIdx.y, g = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = g * ATT_HPB + warp;
  int L = p.ctx[t];
  if (L < 1 || L > p.max_ctx || L > p.mbps * p.bs) {
    if (threadIdx.x == 0 && s == 0 && g == 0) set_flag(p.flag, MLA_FLAG_BAD_CONTEXT);
    L = 0;
  }
  const int j0 = s * p.chunk, j1 = min(L, j0 + p.chunk);
  const int lat_off = (p.layout == MLA_ROW_LATENT_FIRST) ? 0 : p.d_r;
  const int pe_off = (p.layout == MLA_ROW_LATENT_FIRST) ? p.r_kv : 0;
  // query in cache-row order
  for (int idx = threadIdx.x; idx < ATT_HPB * R; idx += blockDim.x) {
    const int hh = g * ATT_HPB + idx / R, k = idx % R;
    float v = 0.f;
    if (hh < p.H) {
      if (k >= lat_off && k < lat_off + p.r_kv)
        v = to_f32(((const T*)p.q_abs)[((long long)t * p.H + hh) * p.r_kv + (k - lat_off)]);
      else
        v = to_f32(((const T*)p.q_pe)[((long long)t * p.H + hh) * p.d_r + (k - pe_off)]);
    }
    qf[idx] = v;
  }
  const int per_lane = p.r_kv / 32;        // r_kv % 32 == 0
  float o[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int jt = j0; jt < j1; jt += ATT_TR) {
    __syncthreads();
    for (int r = warp; r < ATT_TR; r += 8) {
      const int j = jt + r;
      int ok = 0;
      long long row = 0;
      if (j < j1) {
        const int blk = p.block_table[(long long)t * p.mbps + j / p.bs];
        if (blk >= 0 && blk < p.n_blocks) { ok = 1; row = (long long)blk * p.bs + j % p.bs; }
        else if (lane == 0) set_flag(p.flag, MLA_FLAG_BAD_BLOCK);
      }
      const T* src = (const T*)p.cache + row * R;
      for (int k = lane; k < R; k += 32) rows[r * RP + k] = ok ? to_f32(src[k]) : 0.f;
      if (lane == 0) valid_row[r] = ok;
    }
    __syncthreads();
    if (h < p.H) {
      float sc = -INFINITY;
      if (valid_row[lane]) {
        const float* q = qf + warp * R;
        const float* rw = rows + lane * RP;
        float acc = 0.f;
        for (int k = 0; k < R; ++k) acc = fmaf(q[k], rw[k], acc);
        sc = acc * p.scale;
      }
      const float mt = warp_max(sc);
      const float m_new = fmaxf(m, mt);
      const float alpha = (m_new == -INFINITY) ? 1.f : __expf(m - m_new);
      const float pj = (sc == -INFINITY) ? 0.f : __expf(sc - m_new);
      l = l * alpha + warp_sum(pj);
      m = m_new;
#pragma unroll
      for (int i = 0; i < 16; ++i) if (i < per_lane) o[i] *= alpha;
      for (int r = 0; r < ATT_TR; ++r) {
        const float pr = __shfl_sync(0xffffffffu, pj, r);
        if (pr == 0.f) continue;
        const float* rw = rows + r * RP + lat_off;
#pragma unroll
        for (int i = 0; i < 16; ++i) if (i < per_lane) o[i] = fmaf(pr, rw[lane + 32 * i], o[i]);
      }
    }
  }
  if (h < p.H) {
    const long long base = ((long long)t * p.n_splits + s) * p.H + h;
#pragma unroll
    for (int i = 0; i < 16; ++i) if (i < per_lane) p.part_o[base * p.r_kv + lane + 32 * i] = o[i];
    if (lane == 0) { p.part_ml[base * 2] = m; p.part_ml[base * 2 + 1] = l; }
  }
}

// Merge split partials: o_lat = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s.
// With a per-head sink logit z_h ("Struct MlaWeights", attn_sink) the softmax
// has one more column that carries no value: M also covers z_h and the
// denominator gains e^{z_h - M}. Kernels that split the latent columns over a
// CTA pair store one (m, l) copy per CTA: columns c >= half_cols then use the
// copy ml_r floats further on (half_cols = 0: one copy for all columns).
// nseg (optional): sequence t has nseg[t] partials, in its first split slots;
// otherwise all n_splits slots are read and empty ones carry l = 0.
// grid (n, H), 128 threads x 4 consecutive columns (r_kv <= 512, r_kv % 4 == 0).
// Writes o_lat [n, H, r_kv] in act dtype.
template <typename T>
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* part_o, const float* part_ml, int n_splits,
                                                           int H, int r_kv, T* o_lat, const float* sink,
                                                           long long ml_r, int half_cols, const int* nseg) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float wsh[2][64];
  __shared__ float inv_sh[2];
  const int t = blockIdx.x, h = blockIdx.y;
  const int used = nseg ? min(nseg[t], n_splits) : n_splits;   // slots holding this sequence's partials
  const int warp = threadIdx.x >> 5;
  if (warp < (half_cols > 0 ? 2 : 1)) {   // warp w: the weights of stats copy w
    const float* ml = part_ml + warp * ml_r;
    float M = -INFINITY;
    for (int s = threadIdx.x & 31; s < used; s += 32) {
      const long long base = ((long long)t * n_splits + s) * H + h;
      if (ml[base * 2 + 1] > 0.f) M = fmaxf(M, ml[base * 2]);
    }
    M = warp_max(M);
    const float z = sink ? sink[h] : -INFINITY;
    M = fmaxf(M, z);
    float den = ((threadIdx.x & 31) == 0 && z > -INFINITY) ? __expf(z - M) : 0.f;
    for (int s = threadIdx.x & 31; s < used; s += 32) {
      const long long base = ((long long)t * n_splits + s) * H + h;
      const float l = ml[base * 2 + 1];
      const float w = (l > 0.f) ? __expf(ml[base * 2] - M) : 0.f;
      if (s < 64) wsh[warp][s] = w;
      den += w * l;
    }
    den = warp_sum(den);
    if ((threadIdx.x & 31) == 0) inv_sh[warp] = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  const int c = threadIdx.x * 4;
  if (c >= r_kv) return;
  const int cp = (half_cols > 0 && c >= half_cols) ? 1 : 0;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int ns = used < 64 ? used : 64;
#pragma unroll 4
  for (int s = 0; s < ns; ++s) {
    const float w = wsh[cp][s];
    if (w == 0.f) continue;
    const long long base = ((long long)t * n_splits + s) * H + h;
    const float4 v = *reinterpret_cast<const float4*>(part_o + base * r_kv + c);
    acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
  }
  const float inv = inv_sh[cp];
  T* o = o_lat + ((long long)t * H + h) * r_kv + c;
  o[0] = from_f32<T>(acc.x * inv); o[1] = from_f32<T>(acc.y * inv);
  o[2] = from_f32<T>(acc.z * inv); o[3] = from_f32<T>(acc.w * inv);
}

// ---------------------------------------------------------------------------
// Causal expanded prefill attention (CUDA cores). grid (ceil(S/32), H),
// 128 threads (4 warps x 8 queries). Per head h:
//   Q_h[i] = Q[i, h*(d_n+d_r) + ...]                 (q_pe already rotated)
//   K_h[j] = [KV[j, h*(d_n+d_v) + 0..d_n) | kpe[j]]   (k_pe shared by heads)
//   V_h[j] = KV[j, h*(d_n+d_v) + d_n + 0..d_v)
//   O_h[i] = softmax_{j<=i}(Q_h[i] . K_h[j] * scale) V_h
// ("QKV CTE MLA Kernel API Reference", qkv_mla_mx, Final assembly.)
// ---------------------------------------------------------------------------
struct PrefillAttnArgs {
  const void* Q; long long ldq;
  const void* KV; long long ldkv;
  const void* kpe;                       // [S, d_r]
  void* O; long long ldo;                // [S, H*d_v]
  int S, H, d_n, d_r, d_v;
  float scale;
  const float* sink;                     // [H] sink logits (one more softmax column, no value), or NULL
};

constexpr int PA_BQ = 32, PA_BK = 32;

template <typename T>
__global__ void __launch_bounds__(128) prefill_attn_simt_kernel(PrefillAttnArgs p) {
  extern __shared__ float smem[];
  const int dq = p.d_n + p.d_r, DP = dq + 1;
  float* Qs = smem;                      // [PA_BQ][dq]
  float* Ks = Qs + PA_BQ * dq;           // [PA_BK][DP]
  float* Vs = Ks + PA_BK * DP;           // [PA_BK][d_v]
  const int qt = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = qt * PA_BQ;
  const T* Q = (const T*)p.Q;
  const T* KV = (const T*)p.KV;
  const T* KPE = (const T*)p.kpe;
  for (int idx = threadIdx.x; idx < PA_BQ * dq; idx += blockDim.x) {
    const int r = idx / dq, k = idx % dq, i = i0 + r;
    Qs[idx] = (i < p.S) ? to_f32(Q[(long long)i * p.ldq + (long long)h * dq + k]) : 0.f;
  }
  const int per_lane = p.d_v / 32;      // d_v % 32 == 0, <= 128
  float o[8][4];
  float m[8], l[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    m[q] = -INFINITY; l[q] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) o[q][c] = 0.f;
  }
  const int i_last = min(p.S - 1, i0 + PA_BQ - 1);
  for (int j0 = 0; j0 <= i_last; j0 += PA_BK) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < PA_BK * dq; idx += blockDim.x) {
      const int r = idx / dq, k = idx % dq, j = j0 + r;
      float v = 0.f;
      if (j < p.S) {
        if (k < p.d_n) v = to_f32(KV[(long long)j * p.ldkv + (long long)h * (p.d_n + p.d_v) + k]);
        else v = to_f32(KPE[(long long)j * p.d_r + (k - p.d_n)]);
      }
      Ks[r * DP + k] = v;
    }
    for (int idx = threadIdx.x; idx < PA_BK * p.d_v; idx += blockDim.x) {
      const int r = idx / p.d_v, c = idx % p.d_v, j = j0 + r;
      Vs[idx] = (j < p.S) ? to_f32(KV[(long long)j * p.ldkv + (long long)h * (p.d_n + p.d_v) + p.d_n + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = warp * 8 + q, i = i0 + r;
      const int j = j0 + lane;
      float sc = -INFINITY;
      if (i < p.S && j <= i) {
        const float* qq = Qs + r * dq;
        const float* kk = Ks + lane * DP;
        float acc = 0.f;
        for (int k = 0; k < dq; ++k) acc = fmaf(qq[k], kk[k], acc);
        sc = acc * p.scale;
      }
      const float mt = warp_max(sc);
      const float m_new = fmaxf(m[q], mt);
      const float alpha = (m_new == -INFINITY) ? 1.f : __expf(m[q] - m_new);
      const float pj = (sc == -INFINITY) ? 0.f : __expf(sc - m_new);
      l[q] = l[q] * alpha + warp_sum(pj);
      m[q] = m_new;
#pragma unroll
      for (int c = 0; c < 4; ++c) o[q][c] *= alpha;
      for (int rr = 0; rr < PA_BK; ++rr) {
        const float pr = __shfl_sync(0xffffffffu, pj, rr);
        if (pr == 0.f) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c < per_lane) o[q][c] = fmaf(pr, Vs[rr * p.d_v + lane + 32 * c], o[q][c]);
      }
    }
  }
  T* O = (T*)p.O;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int i = i0 + warp * 8 + q;
    if (i >= p.S) continue;
    const float den = l[q] + ((p.sink && l[q] > 0.f) ? __expf(p.sink[h] - m[q]) : 0.f);
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (c < per_lane) O[(long long)i * p.ldo + (long long)h * p.d_v + lane + 32 * c] = from_f32<T>(o[q][c] * inv);
  }
}

// ---------------------------------------------------------------------------
// Weight repack: dst[b][n][k] = src[off + b*sb + n*sn + k*sk] (element copy).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void gather3_kernel(T* dst, const T* src, long long off, long long sb, long long sn,
                               long long sk, int B, int N, int K) {
  const long long total = (long long)B * N * K;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long k = idx % K, n = (idx / K) % N, b = idx / ((long long)K * N);
    dst[idx] = src[off + b * sb + n * sn + k * sk];
  }
}

// cos/sin(pos * theta^(-2i/d_r)) in fp64, rounded once to fp32.
__global__ void rope_table_kernel(const int* pos, int n, int d_r, double theta, float* cs, float* sn) {
  const int half = d_r / 2;
  const long long total = (long long)n * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(idx / half), i = (int)(idx % half);
    const double inv_freq = pow(theta, -2.0 * (double)i / (double)d_r);
    const double phi = (double)pos[t] * inv_freq;
    double sv, cv;
    sincos(phi, &sv, &cv);
    cs[idx] = (float)cv;
    sn[idx] = (float)sv;
  }
}

// RoPE tables from a given frequency table: angle = pos * inv_freq[i], the
// product and the cosine / sine in fp64, rounded once to fp32 ("Struct
// MlaWeights", yarn_inv_freq: a precomputed [rotary_dim/2] table).
__global__ void rope_table_freq_kernel(const int* pos, int n, int d_r, const float* inv_freq, float* cs, float* sn) {
  const int half = d_r / 2;
  const long long total = (long long)n * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(idx / half), i = (int)(idx % half);
    const double phi = (double)pos[t] * (double)inv_freq[i];
    double sv, cv;
    sincos(phi, &sv, &cv);
    cs[idx] = (float)cv;
    sn[idx] = (float)sv;
  }
}

// FP8-E4M3 weight codes with 128 x 128 block scales to bf16, for the prefill
// GEMMs: out[n][k] = bf16(e4m3(code[n][k]) * scale[n / 128][k / 128]) over a
// K-major [N, K] matrix whose scales are [ceil(N/128)][ceil(K/128)] ("Struct
// MlaWeights", wq_a_fp8: dequantised in fp32 before the MAC with bf16
// activations). 16 codes per thread; K a multiple of 16.
__global__ void dequant_fp8_bf16_kernel(const uint8_t* codes, const float* scales, long long N, long long K,
                                        bf16* out) {
  const long long kb = (K + 127) / 128;
  const long long total = N * (K / 16);
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long n = idx / (K / 16), k0 = (idx % (K / 16)) * 16;
    const float sc = scales[(n / 128) * kb + k0 / 128];
    const uint4 c = *reinterpret_cast<const uint4*>(codes + n * K + k0);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const float lo = e4m3_to_f32((uint8_t)(w[j] >> (16 * b))) * sc;
        const float hi = e4m3_to_f32((uint8_t)(w[j] >> (16 * b + 8))) * sc;
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        o[2 * j + b] = *reinterpret_cast<uint32_t*>(&v);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + n * K + k0);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// The layer's input RMSNorm, one CTA per token: xn = x * rsqrt(mean(x^2) + eps)
// * gamma in the activation dtype ("MLA Decode QKV Kernel API Reference",
// input_norm_w: the input RMSNorm folded into the hidden load).
template <typename T>
__global__ void __launch_bounds__(256) input_rmsnorm_kernel(const T* x, const float* gamma, int D, float eps, T* xn) {
  __shared__ float red[32];
  const T* xr = x + (long long)blockIdx.x * D;
  T* yr = xn + (long long)blockIdx.x * D;
  float ss = 0.f;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const float v = to_f32(xr[i]);
    ss += v * v;
  }
  const float r = rsqrtf(block_sum(ss, red) / (float)D + eps);
  for (int i = threadIdx.x; i < D; i += blockDim.x) yr[i] = from_f32<T>(to_f32(xr[i]) * r * gamma[i]);
}

}  // namespace mla
