// Persistent, warp-specialised tcgen05 GEMM for the layer's weight contractions:
//   D[b][m][n] = sum_k A[b][m][k] * B[b][n][k]      (bf16 in, fp32 accumulate)
// A and B are K-major and arrive by TMA (128-byte swizzle) into a STAGES-deep
// shared-memory ring; one thread issues tcgen05.mma (M = 128, N = BN, K = 16)
// into one of two TMEM accumulators; four epilogue warps drain the other
// accumulator (tcgen05.ld) while the next tile accumulates. Work units are
// (m tile, n tile, batch, K split), taken round-robin by a grid of at most one
// CTA per SM.
//
// Decode uses it "swap-AB": A = weights (M = output features), B = the few
// tokens (N = tokens), so that no tensor-core row is padding; prefill uses it
// with A = tokens. The epilogue modes write fp32 split partials, bf16 rows, or
// the query with interleaved RoPE applied to its q_pe columns.
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

enum EpiMode : int {
  EPI_F32_T = 0,    // out_f32[(split*N + n)*ldo + m]                  (A = weights)
  EPI_BF16_T = 1,   // out_bf16[n*ldo + b*bstride + m]
  EPI_QROPE_T = 2,  // m = h*(dn+dr)+j, n = token: j < dn -> out_bf16 q_nope[n][h][j];
                    //   else RoPE pair -> out2_bf16 q_pe[n][h][j-dn]
  EPI_BF16_N = 3,   // out_bf16[m*ldo + b*bstride + n]                 (A = tokens)
  EPI_F32_N = 4,    // out_f32[(split*M + m)*ldo + n]
  EPI_QROPE_N = 5,  // m = token, n = h*(dn+dr)+j: out_bf16[m*ldo + n], q_pe columns rotated
};

struct GemmArgs {
  int M, N, K;
  int m_tiles, n_tiles, batches, splits, kb_per_split, k_blocks, total_units;
  int a_rows_dim2, b_rows_dim2;   // tensor-map dim holding the rows: 0 -> dim 1, 1 -> dim 2
  int mode;
  void* out;
  long long ldo, bstride;
  void* out2;
  const float* cos;
  const float* sin;
  int H, dn, dr;
  int* flag;
  // operand read from memory no earlier kernel of the stream writes (the
  // weights): 1 = A, 2 = B, 0 = neither. Its first pipeline stages are loaded
  // before waiting for the previous kernel.
  int static_op;
  // EPI_BF16_T and the q_nope part of EPI_QROPE_T write f16 instead of bf16
  // (activations whose only reader is an FP8-weight GEMM, which takes f16 tokens)
  int out_f16;
};

constexpr int EPI_STG_BYTES = 2 * 8192;   // the transposed epilogue's staging (gemm_store_t16)

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (196608 / STAGE_BYTES) > 8 ? 8 : (196608 / STAGE_BYTES);
  static constexpr int TMEM_COLS = (2 * BN) < 32 ? 32 : 2 * BN;   // two accumulators
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int STG_OFF = BAR_OFF + 256;   // the transposed epilogue's staging
  static constexpr int SMEM = 1024 + STG_OFF + EPI_STG_BYTES;
};

__device__ __forceinline__ void gemm_store(const GemmArgs& g, int m, int n0, int split, int b, const uint32_t* r) {
  const bool m_ok = m < g.M;
  switch (g.mode) {
    case EPI_F32_T: {
      if (!m_ok) break;
      float* o = (float*)g.out;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n0 + j;
        if (n < g.N) o[((long long)split * g.N + n) * g.ldo + m] = __uint_as_float(r[j]);
      }
      break;
    }
    case EPI_BF16_T: {
      if (!m_ok) break;
      const long long base = (long long)b * g.bstride + m;
      if (g.out_f16) {
        __half* o = (__half*)g.out;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = n0 + j;
          if (n < g.N) o[(long long)n * g.ldo + base] = __float2half_rn(__uint_as_float(r[j]));
        }
      } else {
        bf16* o = (bf16*)g.out;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = n0 + j;
          if (n < g.N) o[(long long)n * g.ldo + base] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
      }
      break;
    }
    case EPI_QROPE_T: {
      const int hd = g.dn + g.dr;
      const int h = m / hd, jj = m % hd;
      const bool odd = (m & 1) != 0;
      const bool rot = m_ok && jj >= g.dn;
      // The 16 tokens' cos / sin first: a load placed after a store to q (which may alias the
      // tables, as far as the compiler knows) waits for it, and under a saturated memory system
      // that wait is long.
      float cs[16], sn[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int n = n0 + j;
        cs[j] = sn[j] = 0.f;
        if (rot && n < g.N) {
          const long long t = (long long)n * (g.dr >> 1) + ((jj - g.dn) >> 1);
          cs[j] = g.cos[t];
          sn[j] = g.sin[t];
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v = __uint_as_float(r[j]);
        const float partner = __shfl_xor_sync(0xffffffffu, v, 1);   // all lanes take part
        const int n = n0 + j;
        if (!m_ok || n >= g.N) continue;
        if (!rot) {
          const long long o = ((long long)n * g.H + h) * g.dn + jj;
          if (g.out_f16) ((__half*)g.out)[o] = __float2half_rn(v);
          else ((bf16*)g.out)[o] = __float2bfloat16_rn(v);
        } else {
          const float o = odd ? (partner * sn[j] + v * cs[j]) : (v * cs[j] - partner * sn[j]);
          ((bf16*)g.out2)[((long long)n * g.H + h) * g.dr + (jj - g.dn)] = __float2bfloat16_rn(o);
        }
      }
      break;
    }
    case EPI_BF16_N: {
      if (!m_ok) break;
      bf16* o = (bf16*)g.out + (long long)m * g.ldo + (long long)b * g.bstride;
      if (n0 + 16 <= g.N && ((((uintptr_t)(o + n0)) & 15) == 0)) {
        uint4 v0, v1;
        v0.x = pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1]));
        v0.y = pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3]));
        v0.z = pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5]));
        v0.w = pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]));
        v1.x = pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9]));
        v1.y = pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11]));
        v1.z = pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13]));
        v1.w = pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15]));
        *reinterpret_cast<uint4*>(o + n0) = v0;
        *reinterpret_cast<uint4*>(o + n0 + 8) = v1;
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (n0 + j < g.N) o[n0 + j] = __float2bfloat16_rn(__uint_as_float(r[j]));
      }
      break;
    }
    case EPI_F32_N: {
      if (!m_ok) break;
      float* o = (float*)g.out + ((long long)split * g.M + m) * g.ldo;
      if (n0 + 16 <= g.N && ((((uintptr_t)(o + n0)) & 15) == 0)) {
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4*>(o + n0 + j) =
              make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                          __uint_as_float(r[j + 3]));
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (n0 + j < g.N) o[n0 + j] = __uint_as_float(r[j]);
      }
      break;
    }
    case EPI_QROPE_N: {
      if (!m_ok) break;
      const int hd = g.dn + g.dr;
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const int jj = (n0 + j) % hd;      // n0 + j even, so (jj, jj+1) is one RoPE pair
        if (jj >= g.dn) {
          const int i = (jj - g.dn) >> 1;
          const float c = g.cos[(long long)m * (g.dr >> 1) + i], s = g.sin[(long long)m * (g.dr >> 1) + i];
          const float a = v[j], bb = v[j + 1];
          v[j] = a * c - bb * s;
          v[j + 1] = a * s + bb * c;
        }
      }
      bf16* o = (bf16*)g.out + (long long)m * g.ldo;
      if (n0 + 16 <= g.N && ((((uintptr_t)(o + n0)) & 15) == 0)) {
        uint4 v0, v1;
        v0.x = pack_bf16x2(v[0], v[1]); v0.y = pack_bf16x2(v[2], v[3]);
        v0.z = pack_bf16x2(v[4], v[5]); v0.w = pack_bf16x2(v[6], v[7]);
        v1.x = pack_bf16x2(v[8], v[9]); v1.y = pack_bf16x2(v[10], v[11]);
        v1.z = pack_bf16x2(v[12], v[13]); v1.w = pack_bf16x2(v[14], v[15]);
        *reinterpret_cast<uint4*>(o + n0) = v0;
        *reinterpret_cast<uint4*>(o + n0 + 8) = v1;
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (n0 + j < g.N) o[n0 + j] = __float2bfloat16_rn(v[j]);
      }
      break;
    }
    default:
      break;
  }
}

// The transposed (swap-AB) epilogue modes through shared memory. The 128
// epilogue threads (et = the tile row = TMEM lane) each hold their row's 16
// columns n0 .. n0 + 15; those go into stg as [16 columns][128 rows] and leave
// as 16-byte stores along m, so a warp's store instruction covers 512 contiguous
// bytes instead of 32 scattered 2- or 4-byte values (under a saturated read
// stream, such narrow stores took microseconds per tile). stg: two 8 KB
// buffers, used by these 128 threads only; `chunk` counts the calls and picks
// the buffer, and stg_bars[chunk & 1] (mbarriers of 4 arrivals, one per warp)
// tell that all four warps have written it. Returns false if that wait gave up.
__device__ __forceinline__ bool gemm_store_t16(const GemmArgs& g, int mt, int et, int n0, int split, int b,
                                               uint32_t* v, uint8_t* stg_base, int chunk, uint32_t stg_bars,
                                               volatile int* abort_word) {
  const int m0 = mt * 128, m = m0 + et;
  uint8_t* stg = stg_base + (chunk & 1) * 8192;
  const int hd = g.dn + g.dr;
  bool half_out = g.out_f16 != 0;   // 2-byte rows written as f16 (else bf16)
  if (g.mode == EPI_QROPE_T) {
    // rotate the q_pe rows (pairs of adjacent rows, i.e. lanes)
    const int jj = m % hd;
    const bool rot = m < g.M && jj >= g.dn;
    const bool odd = (m & 1) != 0;
    float cs[16], sn[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int n = n0 + j;
      cs[j] = 1.f;
      sn[j] = 0.f;
      if (rot && n < g.N) {
        const long long t = (long long)n * (g.dr >> 1) + ((jj - g.dn) >> 1);
        cs[j] = g.cos[t];
        sn[j] = g.sin[t];
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float x = __uint_as_float(v[j]);
      const float partner = __shfl_xor_sync(0xffffffffu, x, 1);   // all lanes take part
      v[j] = __float_as_uint(odd ? (partner * sn[j] + x * cs[j]) : (x * cs[j] - partner * sn[j]));
    }
    half_out = half_out && !rot;   // q_pe stays bf16
  }
  // chunk - 1's writes are behind every thread, so chunk - 2's copy-out (same buffer) is done
  if (g.mode == EPI_F32_T) {
    float* st = (float*)stg;
#pragma unroll
    for (int j = 0; j < 16; ++j) st[j * 128 + et] = __uint_as_float(v[j]);
  } else {
    __half* sh = (__half*)stg;
    bf16* sb = (bf16*)stg;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (half_out) sh[j * 128 + et] = __float2half_rn(__uint_as_float(v[j]));
      else sb[j * 128 + et] = __float2bfloat16_rn(__uint_as_float(v[j]));
    }
  }
  __syncwarp();
  const uint32_t sb_bar = stg_bars + 8 * (chunk & 1);
  if ((et & 31) == 0) mbar_arrive(sb_bar);
  if (!mbar_wait_warp(sb_bar, (chunk >> 1) & 1, abort_word, g.flag)) return false;
  if (g.mode == EPI_F32_T) {
#pragma unroll
    for (int c = et; c < 512; c += 128) {   // [16 columns][32 groups of 4 rows]
      const int j = c >> 5, mm = m0 + 4 * (c & 31), n = n0 + j;
      if (n >= g.N || mm >= g.M) continue;
      const float4 val = reinterpret_cast<const float4*>(stg)[c];
      float* dst = (float*)g.out + ((long long)split * g.N + n) * g.ldo + mm;
      if (mm + 4 <= g.M && (((uintptr_t)dst) & 15) == 0) {
        *reinterpret_cast<float4*>(dst) = val;
      } else {
        const float e[4] = {val.x, val.y, val.z, val.w};
        for (int k = 0; k < 4 && mm + k < g.M; ++k) dst[k] = e[k];
      }
    }
  } else {
#pragma unroll
    for (int c = et; c < 256; c += 128) {   // [16 columns][16 groups of 8 rows]
      const int j = c >> 4, mm = m0 + 8 * (c & 15), n = n0 + j;
      if (n >= g.N || mm >= g.M) continue;
      const uint4 val = reinterpret_cast<const uint4*>(stg)[c];
      uint16_t* dst;
      if (g.mode == EPI_BF16_T) {
        dst = (uint16_t*)g.out + (long long)n * g.ldo + (long long)b * g.bstride + mm;
      } else {   // QROPE: 8-row groups never straddle a head or its nope / rope boundary (d_n, d_r % 8 == 0)
        const int h = mm / hd, jj = mm % hd;
        dst = jj < g.dn ? (uint16_t*)g.out + ((long long)n * g.H + h) * g.dn + jj
                        : (uint16_t*)g.out2 + ((long long)n * g.H + h) * g.dr + (jj - g.dn);
      }
      if (mm + 8 <= g.M && (((uintptr_t)dst) & 15) == 0) {
        *reinterpret_cast<uint4*>(dst) = val;
      } else {
        const uint16_t* e = reinterpret_cast<const uint16_t*>(&val);
        for (int k = 0; k < 8 && mm + k < g.M; ++k) dst[k] = e[k];
      }
    }
  }
  return true;
}

__device__ __forceinline__ void decode_unit(const GemmArgs& g, int u, int& mt, int& nt, int& b, int& s) {
  mt = u % g.m_tiles;
  u /= g.m_tiles;
  nt = u % g.n_tiles;
  u /= g.n_tiles;
  b = u % g.batches;
  s = u / g.batches;
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmArgs g) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t a_base = sbase;                                  // [STAGES][A]
  const uint32_t b_base = sbase + C::STAGES * C::A_BYTES;          // [STAGES][B]
  const uint32_t bar = sbase + C::BAR_OFF;
  auto full_bar = [&](int s) { return bar + 8 * s; };
  auto empty_bar = [&](int s) { return bar + 8 * (C::STAGES + s); };
  auto tfull_bar = [&](int a) { return bar + 8 * (2 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return bar + 8 * (2 * C::STAGES + 2 + a); };
  const uint32_t final_bar = bar + 8 * (2 * C::STAGES + 4);
  uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + 8 * (2 * C::STAGES + 5));
  volatile int* abort_word = (volatile int*)(tmem_slot + 1);
  const uint32_t stg_bars = bar + 192;   // [2] the transposed epilogue's staging written (4 warps)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull_bar(a), 1); mbar_init(tempty_bar(a), 128); }
    mbar_init(final_bar, 1);
    mbar_init(stg_bars, 4);
    mbar_init(stg_bars + 8, 4);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) { prefetch_tmap(&tmA); prefetch_tmap(&tmB); }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      auto load_a = [&](int st, int kb, int mt, int b) {
        const int ar = mt * C::BM;
        if (g.a_rows_dim2) tma_load_3d(a_base + st * C::A_BYTES, &tmA, full_bar(st), kb * C::BK, b, ar);
        else tma_load_3d(a_base + st * C::A_BYTES, &tmA, full_bar(st), kb * C::BK, ar, b);
      };
      auto load_b = [&](int st, int kb, int nt, int b) {
        const int br = nt * BN;
        if (g.b_rows_dim2) tma_load_3d(b_base + st * C::B_BYTES, &tmB, full_bar(st), kb * C::BK, b, br);
        else tma_load_3d(b_base + st * C::B_BYTES, &tmB, full_bar(st), kb * C::BK, br, b);
      };
      // the static operand of the first STAGES k-blocks goes out before the wait
      const int npre = g.static_op ? C::STAGES : 0;
      {
        int it = 0;
        for (int u = blockIdx.x; u < g.total_units && it < npre; u += gridDim.x) {
          int mt, nt, b, s;
          decode_unit(g, u, mt, nt, b, s);
          const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
          for (int kb = kb0; kb < kb1 && it < npre; ++kb, ++it) {
            mbar_arrive_expect_tx(full_bar(it), C::STAGE_BYTES);
            if (g.static_op == 1) load_a(it, kb, mt, b);
            else load_b(it, kb, nt, b);
          }
        }
      }
      griddep_wait();
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x) {
        int mt, nt, b, s;
        decode_unit(g, u, mt, nt, b, s);
        const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int st = it % C::STAGES, round = it / C::STAGES;
          if (it < npre) {   // the stage is armed and its static operand is on its way
            if (g.static_op == 1) load_b(st, kb, nt, b);
            else load_a(st, kb, mt, b);
            continue;
          }
          if (!mbar_wait(empty_bar(st), (round & 1) ^ 1, abort_word, g.flag)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(st), C::STAGE_BYTES);
          load_a(st, kb, mt, b);
          load_b(st, kb, nt, b);
        }
      }
      // drain: every load issued has landed before the CTA can exit
      const int first = it > C::STAGES ? it - C::STAGES : 0;
      for (int j = first; j < it; ++j) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(full_bar(j % C::STAGES), (j / C::STAGES) & 1)) {
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
        }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN);
      // descriptors built once; stages and k-steps add their byte offset >> 4
      const uint64_t da0 = sdesc_sw128(a_base), db0 = sdesc_sw128(b_base);
      int it = 0, tile = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x, ++tile) {
        int mt, nt, b, s;
        decode_unit(g, u, mt, nt, b, s);
        const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
        const int acc = tile & 1, use = tile >> 1;
        if (!mbar_wait(tempty_bar(acc), (use & 1) ^ 1, abort_word, g.flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int st = it % C::STAGES, round = it / C::STAGES;
          if (!mbar_wait(full_bar(st), round & 1, abort_word, g.flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = da0 + (uint64_t)(st * (C::A_BYTES / 16)), db = db0 + (uint64_t)(st * (C::B_BYTES / 16));
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) mma_bf16(d, da + 2 * k, db + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          mma_commit(empty_bar(st));
        }
        if (!ok) break;
        mma_commit(tfull_bar(acc));
      }
      // all MMAs complete before teardown
      mma_commit(final_bar);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(final_bar, 0)) {
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else {
    // ---------------- epilogue: warps 0..3 <-> TMEM lanes 32w..32w+31 ----------------
    griddep_wait();   // the output and the RoPE tables belong to the stream's earlier kernels
    int tile = 0, chunk = 0;
    for (int u = blockIdx.x; u < g.total_units; u += gridDim.x, ++tile) {
      int mt, nt, b, s;
      decode_unit(g, u, mt, nt, b, s);
      const int acc = tile & 1, use = tile >> 1;
      if (!mbar_wait_warp(tfull_bar(acc), use & 1, abort_word, g.flag)) break;
      tc_fence_after();
      const int m = mt * C::BM + warp * 32 + lane;
      const uint32_t row_addr = tmem + ((uint32_t)(warp * 32) << 16) + acc * BN;
      // narrow tiles (few tokens) store directly: their staging round trip costs more than it saves
      const bool staged = BN >= 64 && (g.mode == EPI_F32_T || g.mode == EPI_BF16_T || g.mode == EPI_QROPE_T);
      bool ok = true;
#pragma unroll 1
      for (int c = 0; c < BN / 16 && ok; ++c) {
        uint32_t r[16];
        tmem_ld16(row_addr + c * 16, r);
        tmem_ld_wait();
        if (staged)
          ok = gemm_store_t16(g, mt, warp * 32 + lane, nt * BN + c * 16, s, b, r, smem + C::STG_OFF, chunk++,
                              stg_bars, abort_word);
        else
          gemm_store(g, m, nt * BN + c * 16, s, b, r);
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace mla
