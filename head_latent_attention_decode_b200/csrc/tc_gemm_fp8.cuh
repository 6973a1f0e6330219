// Decode GEMM with FP8-E4M3 weights and fp32 128 x 128 block scales on tcgen05
// ("Struct MlaWeights", field wq_a_fp8: one byte per weight, dequantised in
// fp32 before the MAC with bf16 activations).
//   D[b][m][n] = sum_kb scale[b][m/128][kb] * sum_{k in kb} e4m3(A[b][m][k]) * B[b][n][k]
// A = the FP8 weight matrix (M = output features, 128 per tile = one scale row),
// B = the tokens converted to f16 (N = BN; exact for |x| in f16's normal range,
// which holds every activation of this layer). Per 128-wide K block:
//   TMA brings the 128 x 128 code tile and the 2 x [BN x 64] f16 token tiles;
//   warps 0-7 decode the codes to f16 with cvt.rn.f16x2.e4m3x2 (exact: every
//   E4M3 value is an f16 value) into a 128-byte-swizzled tile;
//   tcgen05 (kind::f16, f16 x f16 -> fp32) multiplies that block alone into one
//   of two TMEM partials;
//   warps 0-7 add scale * partial to fp32 registers (two column halves).
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
  static constexpr int A8 = 128 * 128;             // FP8 code tile
  static constexpr int BB = BN * 64 * 2;           // one [BN x 64] bf16 tile
  static constexpr int STAGE = A8 + 2 * BB;
  static constexpr int ABF = 2 * 128 * 64 * 2;     // decoded A: two [128 x 64] f16 tiles
  static constexpr int ST_RAW = (212 * 1024 - 2 * ABF - 1280) / STAGE;
  static constexpr int STAGES = ST_RAW > 6 ? 6 : ST_RAW;
  static constexpr int ABF_OFF = STAGES * STAGE;
  static constexpr int BAR_OFF = ABF_OFF + 2 * ABF;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;
  static constexpr int TMEM_COLS = (2 * BN) < 32 ? 32 : 2 * BN;
};

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

// warps 0-7 decode the codes (warpgroup h: k-half h of every row) and fold the
// scaled partials (warpgroup h: column half h, or all columns by warps 0-3 when
// BN < 32); warp 8 issues TMA, warp 9 the MMAs.
template <int BN>
__global__ void __launch_bounds__(320, 1)
    tc_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       Fp8GemmArgs fa) {
  using C = Fp8Cfg<BN>;
  const GemmArgs& g = fa.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + C::BAR_OFF;
  auto full_bar = [&](int s) { return bar + 8 * s; };
  auto empty_bar = [&](int s) { return bar + 8 * (C::STAGES + s); };
  const uint32_t conv_full = bar + 8 * (2 * C::STAGES);        // [2]
  const uint32_t conv_free = conv_full + 16;                    // [2]
  const uint32_t part_full = conv_free + 16;                    // [2]
  const uint32_t part_free = part_full + 16;                    // [2]
  const uint32_t fin = part_free + 16;
  uint32_t* tmem_slot = (uint32_t*)(smem + C::BAR_OFF + 8 * (2 * C::STAGES) + 80);
  volatile int* abort_word = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(conv_full + 8 * i, 256);
      mbar_init(conv_free + 8 * i, 1);
      mbar_init(part_full + 8 * i, 1);
      mbar_init(part_free + 8 * i, BN >= 32 ? 256 : 128);
    }
    mbar_init(fin, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) { prefetch_tmap(&tmA); prefetch_tmap(&tmB); }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      // the weight codes of the first STAGES k-blocks go out before the wait for
      // the previous kernel (no earlier kernel of the stream writes them)
      {
        int it = 0;
        for (int u = blockIdx.x; u < g.total_units && it < C::STAGES; u += gridDim.x) {
          int mt, nt, b, s;
          decode_unit(g, u, mt, nt, b, s);
          const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
          for (int kb = kb0; kb < kb1 && it < C::STAGES; ++kb, ++it) {
            mbar_arrive_expect_tx(full_bar(it), C::STAGE);
            tma_load_3d(sbase + it * C::STAGE, &tmA, full_bar(it), kb * 128, mt * 128, b);
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
          const int st = it % C::STAGES;
          const uint32_t dst = sbase + st * C::STAGE;
          if (it >= C::STAGES) {
            if (!mbar_wait(empty_bar(st), ((it / C::STAGES) & 1) ^ 1, abort_word, g.flag)) { ok = false; break; }
            mbar_arrive_expect_tx(full_bar(st), C::STAGE);
            tma_load_3d(dst, &tmA, full_bar(st), kb * 128, mt * 128, b);
          }
          const int br = nt * BN;
          if (g.b_rows_dim2) {
            tma_load_3d(dst + C::A8, &tmB, full_bar(st), kb * 128, b, br);
            tma_load_3d(dst + C::A8 + C::BB, &tmB, full_bar(st), kb * 128 + 64, b, br);
          } else {
            tma_load_3d(dst + C::A8, &tmB, full_bar(st), kb * 128, br, b);
            tma_load_3d(dst + C::A8 + C::BB, &tmB, full_bar(st), kb * 128 + 64, br, b);
          }
        }
      }
      const int first = it > C::STAGES ? it - C::STAGES : 0;
      for (int j = first; j < it; ++j) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(full_bar(j % C::STAGES), (j / C::STAGES) & 1))
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer: one 128-wide K block into one TMEM partial ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, BN);
      // descriptors built once; buffers and k-steps add their byte offset >> 4
      const uint64_t da0 = sdesc_sw128(sbase + C::ABF_OFF), db0 = sdesc_sw128(sbase + C::A8);
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x) {
        int mt, nt, b, s;
        decode_unit(g, u, mt, nt, b, s);
        const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int st = it % C::STAGES, cb = it & 1;
          if (!mbar_wait(full_bar(st), (it / C::STAGES) & 1, abort_word, g.flag)) { ok = false; break; }
          if (!mbar_wait(conv_full + 8 * cb, (it >> 1) & 1, abort_word, g.flag)) { ok = false; break; }
          if (!mbar_wait(part_free + 8 * cb, ((it >> 1) & 1) ^ 1, abort_word, g.flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = da0 + (uint64_t)(cb * (C::ABF / 16)), db = db0 + (uint64_t)(st * (C::STAGE / 16));
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(tmem + cb * BN, da + (kk * 16384 + 32 * k) / 16, db + (kk * C::BB + 32 * k) / 16, idesc,
                       (kk > 0 || k > 0) ? 1u : 0u);
          mma_commit(part_full + 8 * cb);
          mma_commit(conv_free + 8 * cb);
          mma_commit(empty_bar(st));
        }
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(g.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else {
    // ---------------- warps 0-7: decode codes, fold scaled partials, epilogue ----------------
    griddep_wait();   // the output belongs to the stream's earlier kernels
    constexpr int FSPLIT = BN >= 32 ? 2 : 1;   // warpgroups that fold
    constexpr int NCOL = BN / FSPLIT;          // columns each folding thread owns
    const int t = threadIdx.x;
    const int r = t & 127;                     // A row of the tile = TMEM lane
    const int half = t >> 7;                   // warpgroup: k-half to decode, column half to fold
    const bool folds = half < FSPLIT;
    const int col0 = half * NCOL;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float acc[NCOL];
    int it = 0;
    bool ok = true;
    // decode k-half `half` of row r of the A tile of iteration `j` (stage j % STAGES) into buffer j & 1
    auto convert = [&](int j) -> bool {
      const int st = j % C::STAGES, cb = j & 1;
      if (!mbar_wait_warp(full_bar(st), (j / C::STAGES) & 1, abort_word, g.flag)) return false;
      if (!mbar_wait_warp(conv_free + 8 * cb, ((j >> 1) & 1) ^ 1, abort_word, g.flag)) return false;
      const uint8_t* arow = smem + st * C::STAGE + r * 128;
      uint8_t* orow = smem + C::ABF_OFF + cb * C::ABF + half * 16384 + r * 128;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {         // 16 codes = elements 16q .. 16q+15 of the row
        const int q = 4 * half + qq;
        const uint4 v = *reinterpret_cast<const uint4*>(arow + ((q ^ (r & 7)) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t outw[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          outw[2 * k] = e4m3x2_to_f16x2(w[k] & 0xFFFF);
          outw[2 * k + 1] = e4m3x2_to_f16x2(w[k] >> 16);
        }
        const int c0 = 2 * qq;
        *reinterpret_cast<uint4*>(orow + ((c0 ^ (r & 7)) << 4)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        *reinterpret_cast<uint4*>(orow + (((c0 + 1) ^ (r & 7)) << 4)) = make_uint4(outw[4], outw[5], outw[6], outw[7]);
      }
      fence_proxy_async_smem();
      mbar_arrive(conv_full + 8 * cb);
      return true;
    };
    // the global iteration index of each work unit's first K block
    int first_it = 0;
    for (int u = blockIdx.x; u < g.total_units && ok; u += gridDim.x) {
      int mt, nt, b, s;
      decode_unit(g, u, mt, nt, b, s);
      const int kb0 = s * g.kb_per_split, kb1 = min(g.k_blocks, kb0 + g.kb_per_split);
      const int nkb = kb1 - kb0;
      first_it = it;
#pragma unroll
      for (int j = 0; j < NCOL; ++j) acc[j] = 0.f;
      const float* sc = fa.scale + (long long)b * fa.scale_batch + (long long)mt * fa.scale_ld;
      if (nkb > 0 && !convert(first_it)) { ok = false; break; }
      for (int i = 0; i < nkb; ++i) {
        const int j = first_it + i;
        if (i + 1 < nkb && !convert(j + 1)) { ok = false; break; }
        if (!folds) continue;
        const int pb = j & 1;
        if (!mbar_wait_warp(part_full + 8 * pb, (j >> 1) & 1, abort_word, g.flag)) { ok = false; break; }
        tc_fence_after();
        const float scl = sc[kb0 + i];
#pragma unroll
        for (int c = 0; c < NCOL / 16; ++c) {
          uint32_t v[16];
          tmem_ld16(tmem + pb * BN + col0 + lane_base + 16 * c, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) acc[16 * c + k] = fmaf(scl, __uint_as_float(v[k]), acc[16 * c + k]);
        }
        tc_fence_before();
        mbar_arrive(part_free + 8 * pb);
      }
      if (!ok) break;
      it = first_it + nkb;
      if (!folds) continue;
      const int m = mt * 128 + r;
#pragma unroll
      for (int c = 0; c < NCOL / 16; ++c) {
        uint32_t outv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) outv[k] = __float_as_uint(acc[16 * c + k]);
        gemm_store(g, m, nt * BN + col0 + 16 * c, s, b, outv);
      }
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
