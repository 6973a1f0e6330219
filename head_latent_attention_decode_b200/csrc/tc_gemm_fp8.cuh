// Decode GEMM with FP8-E4M3 weights and fp32 128 x 128 block scales on tcgen05
// ("Struct MlaWeights", field wq_a_fp8: one byte per weight, dequantised in
// fp32 before the MAC with bf16 activations).
//   D[b][m][n] = sum_kb scale[b][m/128][kb] * sum_{k in kb} e4m3(A[b][m][k]) * B[b][n][k]
// A = the FP8 weight matrix (M = output features, 128 per tile = one scale row),
// B = the tokens converted to f16 (N = BN; exact for |x| in f16's normal range,
// which holds every activation of this layer). Per 128-wide K block:
//   TMA brings the 128 x 128 code tile into a deep ring of its own (the codes
//   are the HBM stream) and the BN x 128 f16 token tile into a shorter one
//   (the tokens come from L2);
//   warps 0-3 decode the codes to f16 with cvt.rn.f16x2.e4m3x2 (exact: every
//   E4M3 value is an f16 value) straight into TMEM, one weight row per thread,
//   so the code stage is free again as soon as it is read;
//   tcgen05 (kind::f16, A from TMEM, f16 x f16 -> fp32) multiplies that block
//   alone into one of three TMEM partials;
//   warps 4-11 add scale * partial to fp32 registers (two column halves) and,
//   once a unit's K blocks are all folded, hand the tile to TMEM;
//   warps 14-17 store it (the epilogue), so a store that waits behind the code
//   stream holds up neither the fold nor the MMAs;
//   warp 12 issues the TMA loads, warp 13 the MMAs.
// So the scale multiplies each block's exact fp32 partial sum, the same value
// as dequantising every weight in fp32 before the MAC, up to fp32 rounding.
// The epilogue modes are those of tc_gemm.cuh.
#pragma once

#include "tc_gemm.cuh"

namespace mla {
namespace tc {

struct Fp8GemmArgs {
  GemmArgs g;                 // shape, tiling (k_blocks count 128-wide blocks here) and epilogue
  const float* scale;         // [batches][ceil(M/128)][ceil(K/128)]
  long long scale_ld, scale_batch;
};

template <int BN>
struct Fp8Cfg {
  static constexpr int A8 = 128 * 128;             // one FP8 code tile
  static constexpr int BB = BN * 64 * 2;           // one [BN x 64] f16 token tile
  static constexpr int TOK = 2 * BB;               // the tokens of one 128-wide K block
  static constexpr int TS = 3;                     // token stages
  static constexpr int CS_RAW = (227 * 1024 - 1536 - EPI_STG_BYTES - TS * TOK) / A8;
  static constexpr int CS = CS_RAW > 10 ? 10 : CS_RAW;   // code stages
  static constexpr int TOK_OFF = CS * A8;
  static constexpr int BAR_OFF = TOK_OFF + TS * TOK;
  static constexpr int STG_OFF = BAR_OFF + 512;   // the transposed epilogue's staging
  static constexpr int SMEM = 1024 + STG_OFF + EPI_STG_BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // TMEM columns: decoded A buffers [0,64) [64,128) (f16 pairs), partials [128, 128 + NP BN),
  // the finished tile on its way out [128 + NP BN, 128 + (NP + 1) BN)
  static constexpr int NP = BN >= 128 ? 2 : 3;
  static constexpr uint32_t TM_A = 0, TM_P = 128, TM_OUT = 128 + NP * BN;
  static constexpr int TMEM_COLS = (128 + (NP + 1) * BN) <= 256 ? 256 : 512;
  static_assert(128 + (NP + 1) * BN <= 512, "TMEM columns");
  static constexpr int FOLD_WARPS = BN >= 32 ? 8 : 4;
};
constexpr int FP8_THREADS = 576;   // 4 decode, 8 fold, TMA, MMA, 4 epilogue warps
constexpr int FP8_EPI_BLOCKS = 6;  // a unit's partial store, in K blocks of time (split choice)

// Two E4M3 codes (low byte -> low half) to two f16 values.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes16) {
  uint32_t d;
  const uint16_t a = (uint16_t)codes16;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(a));
  return d;
}
// kind::f16 with f16 A and B, fp32 accumulator, K-major operands.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int BN>
__global__ void __launch_bounds__(FP8_THREADS, 1)
    tc_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       Fp8GemmArgs fa) {
  using C = Fp8Cfg<BN>;
  const GemmArgs& g = fa.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + C::BAR_OFF;
  const uint32_t code_full = bar, code_empty = bar + 8 * C::CS;          // [CS]
  const uint32_t tok_full = bar + 16 * C::CS, tok_empty = tok_full + 8 * C::TS;   // [TS]
  const uint32_t a_full = tok_empty + 8 * C::TS, a_free = a_full + 16;   // [2] decoded A in TMEM / consumed
  const uint32_t part_full = a_free + 16, part_free = part_full + 8 * C::NP;   // [NP]
  const uint32_t fin = part_free + 8 * C::NP;
  const uint32_t out_full = fin + 8, out_free = out_full + 8;                  // the finished tile in TMEM
  const uint32_t stg_bars = out_free + 8;                                      // [2] epilogue staging written
  uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + 480);
  volatile int* abort_word = (volatile int*)(smem + C::BAR_OFF + 484);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::CS; ++s) { mbar_init(code_full + 8 * s, 1); mbar_init(code_empty + 8 * s, 4); }
    for (int s = 0; s < C::TS; ++s) { mbar_init(tok_full + 8 * s, 1); mbar_init(tok_empty + 8 * s, 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(a_full + 8 * i, 4);
      mbar_init(a_free + 8 * i, 1);
    }
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(part_full + 8 * i, 1);
      mbar_init(part_free + 8 * i, C::FOLD_WARPS);
    }
    mbar_init(fin, 1);
    mbar_init(out_full, C::FOLD_WARPS);
    mbar_init(out_free, 4);
    mbar_init(stg_bars, 4);
    mbar_init(stg_bars + 8, 4);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 12 && lane == 0) { prefetch_tmap(&tmA); prefetch_tmap(&tmB); }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 12) {
    // ---------------- TMA producer: the codes (the first CS ahead of the dependency wait: no
    // earlier kernel writes the weights), and the tokens CS - TS K blocks behind them ----------------
    if (lane == 0) {
      constexpr int LAG = C::CS - C::TS;
      // the (unit, K block) of the j-th K block of this CTA, walked twice: codes and tokens
      struct Cursor {
        int u, kb, kb1, mt, nt, b;
        __device__ bool valid(const GemmArgs& g) const { return u < g.total_units; }
        __device__ void enter(const GemmArgs& g) {
          int s;
          if (u < g.total_units) {
            decode_unit(g, u, mt, nt, b, s);
            kb = s * g.kb_per_split;
            kb1 = min(g.k_blocks, kb + g.kb_per_split);
          }
        }
        __device__ void next(const GemmArgs& g) {
          if (++kb >= kb1) {
            u += gridDim.x;
            enter(g);
          }
        }
      };
      Cursor cc{(int)blockIdx.x, 0, 0, 0, 0, 0}, tc{(int)blockIdx.x, 0, 0, 0, 0, 0};
      cc.enter(g);
      tc.enter(g);
      int jc = 0, jt = 0;
      bool ok = true;
      auto issue_codes = [&]() -> bool {
        const int cs = jc % C::CS;
        if (!mbar_wait(code_empty + 8 * cs, ((jc / C::CS) & 1) ^ 1, abort_word, g.flag)) return false;
        mbar_arrive_expect_tx(code_full + 8 * cs, C::A8);
        tma_load_3d(sbase + cs * C::A8, &tmA, code_full + 8 * cs, cc.kb * 128, cc.mt * 128, cc.b);
        ++jc;
        cc.next(g);
        return true;
      };
      auto issue_tokens = [&]() -> bool {
        const int ts = jt % C::TS;
        if (!mbar_wait(tok_empty + 8 * ts, ((jt / C::TS) & 1) ^ 1, abort_word, g.flag)) return false;
        const uint32_t dst = sbase + C::TOK_OFF + ts * C::TOK;
        const int br = tc.nt * BN;
        mbar_arrive_expect_tx(tok_full + 8 * ts, C::TOK);
        if (g.b_rows_dim2) {
          tma_load_3d(dst, &tmB, tok_full + 8 * ts, tc.kb * 128, tc.b, br);
          tma_load_3d(dst + C::BB, &tmB, tok_full + 8 * ts, tc.kb * 128 + 64, tc.b, br);
        } else {
          tma_load_3d(dst, &tmB, tok_full + 8 * ts, tc.kb * 128, br, tc.b);
          tma_load_3d(dst + C::BB, &tmB, tok_full + 8 * ts, tc.kb * 128 + 64, br, tc.b);
        }
        ++jt;
        tc.next(g);
        return true;
      };
      while (ok && jc < C::CS && cc.valid(g)) ok = issue_codes();
      griddep_wait();
      while (ok && (cc.valid(g) || tc.valid(g))) {
        if (tc.valid(g) && (jt + LAG <= jc || !cc.valid(g))) ok = issue_tokens();
        else ok = issue_codes();
      }
      for (int u = (jc > C::CS ? jc - C::CS : 0); u < jc; ++u) {   // loads still in flight land before exit
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(code_full + 8 * (u % C::CS), (u / C::CS) & 1))
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
      for (int u = (jt > C::TS ? jt - C::TS : 0); u < jt; ++u) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(tok_full + 8 * (u % C::TS), (u / C::TS) & 1))
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 13) {
    // ---------------- MMA issuer: one 128-wide K block into one TMEM partial ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, BN);
      const uint64_t db0 = sdesc_sw128(sbase + C::TOK_OFF);
      int j = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x) {
        int mt, nt, b, s;
        decode_unit(g, u, mt, nt, b, s);
        const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++j) {
          const int ts = j % C::TS, pb = j & 1, pp = j % C::NP;
          if (!mbar_wait(a_full + 8 * pb, (j >> 1) & 1, abort_word, g.flag) ||
              !mbar_wait(tok_full + 8 * ts, (j / C::TS) & 1, abort_word, g.flag) ||
              !mbar_wait(part_free + 8 * pp, ((j / C::NP) & 1) ^ 1, abort_word, g.flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = db0 + (uint64_t)(ts * (C::TOK / 16));
          const uint32_t ta = tmem + C::TM_A + 64 * pb, td = tmem + C::TM_P + BN * pp;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16_ts(td, ta + 32 * kk + 8 * k, db + (kk * C::BB + 32 * k) / 16, idesc, (kk > 0 || k > 0) ? 1u : 0u);
          mma_commit(part_full + 8 * pp);
          mma_commit(a_free + 8 * pb);
          mma_commit(tok_empty + 8 * ts);
        }
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else if (warp < 4) {
    // ---------------- decode: thread = weight row m of the tile = TMEM lane ----------------
    const int m = threadIdx.x;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int j = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x) {
      int mt, nt, b, s;
      decode_unit(g, u, mt, nt, b, s);
      const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
      for (int kb = kb0; kb < kb1; ++kb, ++j) {
        const int cs = j % C::CS, pb = j & 1;
        if (!mbar_wait_warp(code_full + 8 * cs, (j / C::CS) & 1, abort_word, g.flag) ||
            !mbar_wait_warp(a_free + 8 * pb, ((j >> 1) & 1) ^ 1, abort_word, g.flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* arow = smem + cs * C::A8 + m * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {   // 32 codes = elements 32 q4 .. 32 q4 + 31 -> 16 TMEM columns
          uint32_t outw[16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int q = 2 * q4 + h;
            const uint4 v = *reinterpret_cast<const uint4*>(arow + ((q ^ (m & 7)) << 4));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              outw[8 * h + 2 * k] = e4m3x2_to_f16x2(w[k] & 0xFFFF);
              outw[8 * h + 2 * k + 1] = e4m3x2_to_f16x2(w[k] >> 16);
            }
          }
          tmem_st16(tmem + C::TM_A + 64 * pb + lane_base + 16 * q4, outw);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(code_empty + 8 * cs);   // the codes are in registers or TMEM
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full + 8 * pb);
      }
    }
  } else if (warp < 4 + C::FOLD_WARPS) {
    // ---------------- fold: warps 4 .. 4 + FOLD_WARPS - 1, TMEM lane quarter warp % 4 ----------------
    constexpr int FSPLIT = C::FOLD_WARPS / 4;  // column groups
    constexpr int NCOL = BN / FSPLIT;          // columns each folding thread owns
    const int w = warp - 4;
    const int col0 = (w >> 2) * NCOL;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    // The block scales of a unit, one unit ahead: lane l holds those of K blocks kb0 + l and
    // kb0 + 32 + l, so a unit's first fold does not wait for a cold load behind the code stream.
    auto load_scales = [&](int u, float& s0, float& s1) {
      s0 = s1 = 0.f;
      if (u >= g.total_units) return;
      int mt, nt, b, s;
      decode_unit(g, u, mt, nt, b, s);
      const float* sc = fa.scale + (long long)b * fa.scale_batch + (long long)mt * fa.scale_ld;
      const int kb0 = s * g.kb_per_split, nkb = min(g.k_blocks, kb0 + g.kb_per_split) - kb0;
      if (lane < nkb) s0 = sc[kb0 + lane];
      if (lane + 32 < nkb) s1 = sc[kb0 + 32 + lane];
    };
    float s0, s1;
    load_scales(blockIdx.x, s0, s1);
    float acc[NCOL];
    int j = 0, uo = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x) {
      int mt, nt, b, s;
      decode_unit(g, u, mt, nt, b, s);
      const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
      const float c0 = s0, c1 = s1;
      load_scales(u + gridDim.x, s0, s1);
#pragma unroll
      for (int c = 0; c < NCOL; ++c) acc[c] = 0.f;
      const float* sc = fa.scale + (long long)b * fa.scale_batch + (long long)mt * fa.scale_ld;
      for (int kb = kb0; kb < kb1; ++kb, ++j) {
        const int pp = j % C::NP, i = kb - kb0;
        const float scl = i < 32 ? __shfl_sync(0xffffffffu, c0, i) : i < 64 ? __shfl_sync(0xffffffffu, c1, i - 32) : sc[kb];
        if (!mbar_wait_warp(part_full + 8 * pp, (j / C::NP) & 1, abort_word, g.flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < NCOL / 16; ++c) {
          uint32_t v[16];
          tmem_ld16(tmem + C::TM_P + BN * pp + col0 + lane_base + 16 * c, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) acc[16 * c + k] = fmaf(scl, __uint_as_float(v[k]), acc[16 * c + k]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(part_free + 8 * pp);
      }
      if (!ok) break;
      // hand the tile to the epilogue warps once they have read out the previous one
      if (!mbar_wait_warp(out_free, (uo & 1) ^ 1, abort_word, g.flag)) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < NCOL / 16; ++c) {
        uint32_t outv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) outv[k] = __float_as_uint(acc[16 * c + k]);
        tmem_st16(tmem + C::TM_OUT + col0 + lane_base + 16 * c, outv);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full);
      ++uo;
    }
  } else if (warp >= 14) {
    // ---------------- epilogue: the finished tile, TMEM lane quarter warp % 4 -> global ----------------
    griddep_wait();   // the output belongs to the stream's earlier kernels
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    int uo = 0, chunk = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x, ++uo) {
      int mt, nt, b, s;
      decode_unit(g, u, mt, nt, b, s);
      if (!mbar_wait_warp(out_full, uo & 1, abort_word, g.flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < BN / 16 && ok; ++c) {
        uint32_t v[16];
        tmem_ld16(tmem + C::TM_OUT + lane_base + 16 * c, v);
        tmem_ld_wait();
        ok = gemm_store_t16(g, mt, r, nt * BN + 16 * c, s, b, v, smem + C::STG_OFF, chunk++, stg_bars, abort_word);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_free);   // the fold may write the next tile
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
