// Absorbed split-KV decode attention on tcgen05 for few heads (H <= 32), with
// the DeepSeek latent (kv_lora_rank 512, qk_rope 64) and cache blocks of a
// multiple of 64 rows. The MMAs run transposed so that the cache rows, not the
// heads, fill the tensor core's M = 128:
//   S^T = tile . [q_abs | q_pe]^T     M 128 rows x N NH heads, K 576
//   softmax down each head's column (cross-row max through shuffles and a
//   4-warp exchange; per-row partial sums reduced once at the end), lazy
//   rescale of O^T when a head's max grows by more than 2^8
//   O^T += V^T . P^T                  4 x (M 128 latent x N NH heads, K 128 rows),
//                                     V^T read MN-major from the same tile
// One CTA per (sequence, split), no cluster and no score exchange; S^T and O^T
// take 6 NH TMEM columns. A 128-row tile occupies five 32 KB ring entries (four
// latent pairs and the rotary block); P.V frees each latent pair as soon as its
// MMAs finish so the next tile streams in behind it.
#pragma once

#include "tc_attn.cuh"

namespace mla {
namespace tc {

template <int NH>
struct AttnSmallSmem {
  static constexpr int NP = NH <= 16 ? 6 : 5;                  // ring entries of 32 KB (two [128 x 64] k-block slots)
  static constexpr int RING_OFF = 0;
  static constexpr int Q_OFF = NP * 32768;                     // 9 x [NH x 64] bf16
  static constexpr int QKB = NH * 128;
  static constexpr int P_OFF = Q_OFF + 9 * QKB;                // 2 buffers x 2 x [NH x 64] bf16
  static constexpr int RED_OFF = P_OFF + 4 * QKB;              // 2 x 4 x NH fp32
  static constexpr int BAR_OFF = RED_OFF + 2 * 4 * NH * 4 + 1024;   // keep barriers 8-byte aligned
  static constexpr int SIZE = 1024 + BAR_OFF + 256;
  static constexpr int TMEM_COLS = 6 * NH <= 128 ? 128 : 256;
};

template <int NH>
__global__ void __launch_bounds__(192, 1)
    tc_attn_small_kernel(const __grid_constant__ CUtensorMap tm_qabs, const __grid_constant__ CUtensorMap tm_qpe,
                         const __grid_constant__ CUtensorMap tm_cache, TcAttnArgs a) {
  using SM = AttnSmallSmem<NH>;
  constexpr int ATS_NP = SM::NP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t ring_s = sbase + SM::RING_OFF, q_s = sbase + SM::Q_OFF, p_s = sbase + SM::P_OFF;
  float* red = (float*)(smem + SM::RED_OFF);
  const uint32_t bar = sbase + SM::BAR_OFF;
  const uint32_t full_b = bar, empty_b = bar + 8 * ATS_NP;
  const uint32_t s_full_b = empty_b + 8 * ATS_NP, s_free_b = s_full_b + 16, p_full_b = s_free_b + 16;
  const uint32_t pbuf_free_b = p_full_b + 16, q_full = pbuf_free_b + 16, o_done = q_full + 8, fin = o_done + 8;
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 192);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 196);

  const int b = blockIdx.x / a.splits, sp = blockIdx.x % a.splits;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int L = a.ctx[b];
  if (L < 1 || L > a.max_ctx || L > a.mbps * a.bs) {
    if (threadIdx.x == 0 && sp == 0) set_flag(a.flag, MLA_FLAG_BAD_CONTEXT);
    L = 0;
  }
  const int r0 = sp * a.chunk, r1 = min(L, r0 + a.chunk);
  const int T = r1 > r0 ? (r1 - r0 + 127) / 128 : 0;
  const long long unit = (long long)b * a.splits + sp;
  if (T == 0) {
    if (threadIdx.x < a.H) {
      a.part_ml[(unit * a.H + threadIdx.x) * 2] = -INFINITY;
      a.part_ml[(unit * a.H + threadIdx.x) * 2 + 1] = 0.f;
    }
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < ATS_NP; ++i) { mbar_init(full_b + 8 * i, 1); mbar_init(empty_b + 8 * i, 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full_b + 8 * i, 1);
      mbar_init(s_free_b + 8 * i, 128);
      mbar_init(p_full_b + 8 * i, 128);
      mbar_init(pbuf_free_b + 8 * i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), SM::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_s = tmem, tm_o = tmem + 2 * NH;   // S^T buffers [0,NH) [NH,2NH); O^T group g at 2NH + g NH

  if (warp == 4) {
    // ---------------- TMA producer: per tile 4 latent pairs, then the rotary block ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_cache);
      mbar_arrive_expect_tx(q_full, 9 * SM::QKB);
      for (int j = 0; j < 8; ++j) tma_load_3d(q_s + j * SM::QKB, &tm_qabs, q_full, 64 * j, b * a.H, 0);
      tma_load_3d(q_s + 8 * SM::QKB, &tm_qpe, q_full, 0, b * a.H, 0);
      int e = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        long long row[2];
        for (int hf = 0; hf < 2; ++hf) {
          const int j0 = r0 + 128 * t + 64 * hf;
          row[hf] = -64;
          if (j0 < r1) {
            const int blk = a.block_table[(long long)b * a.mbps + j0 / a.bs];
            if (blk >= 0 && blk < a.n_blocks) row[hf] = (long long)blk * a.bs + (j0 % a.bs);
            else set_flag(a.flag, MLA_FLAG_BAD_BLOCK);
          }
        }
        for (int i = 0; i < 5; ++i, ++e) {
          const int slot = e % ATS_NP;
          if (!mbar_wait(empty_b + 8 * slot, ((e / ATS_NP) & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
          const uint32_t dst = ring_s + slot * 32768;
          const uint32_t fb = full_b + 8 * slot;
          if (i < 4) {
            mbar_arrive_expect_tx(fb, 32768);
            for (int kk = 0; kk < 2; ++kk)
              for (int hf = 0; hf < 2; ++hf)
                tma_load_3d(dst + kk * 16384 + hf * 8192, &tm_cache, fb, a.lat_col0 + 128 * i + 64 * kk,
                            (int)row[hf], 0);
          } else {
            mbar_arrive_expect_tx(fb, 16384);
            for (int hf = 0; hf < 2; ++hf)
              tma_load_3d(dst + hf * 8192, &tm_cache, fb, a.rope_col0, (int)row[hf], 0);
          }
        }
      }
      {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(q_full, 0)) if (global_timer_ns() - t0 > WAIT_LIMIT_NS) break;
      }
      for (int u = (e > ATS_NP ? e - ATS_NP : 0); u < e; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(full_b + 8 * (u % ATS_NP), (u / ATS_NP) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, NH);
      constexpr uint32_t idesc_o = idesc_bf16(128, NH, 0, 1);
      bool ok = mbar_wait(q_full, 0, abort_word, a.flag);
      for (int t = 0; ok && t < T; ++t) {
        const int sb = t & 1, e0 = 5 * t;
        // S^T(t) over the five entries of the tile
        if (!mbar_wait(s_free_b + 8 * sb, ((t >> 1) & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
        for (int i = 0; i < 5 && ok; ++i) {
          const int e = e0 + i, slot = e % ATS_NP;
          if (!mbar_wait(full_b + 8 * slot, (e / ATS_NP) & 1, abort_word, a.flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = ring_s + slot * 32768;
          const int nk = (i < 4) ? 2 : 1;
          for (int kk = 0; kk < nk; ++kk) {
            const uint32_t qk = q_s + ((i < 4) ? (2 * i + kk) : 8) * SM::QKB;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(tm_s + NH * sb, sdesc_sw128(base + kk * 16384 + 32 * k), sdesc_sw128(qk + 32 * k), idesc_s,
                       (i > 0 || kk > 0 || k > 0) ? 1u : 0u);
          }
          if (i == 4) mma_commit(empty_b + 8 * slot);   // the rotary block is done
        }
        if (!ok) break;
        mma_commit(s_full_b + 8 * sb);
        // O^T(t) += V^T . P^T(t), freeing each latent pair as its MMAs finish
        if (!mbar_wait(p_full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pb = p_s + sb * 2 * SM::QKB;
        for (int g = 0; g < 4; ++g) {
          const int slot = (e0 + g) % ATS_NP;
          const uint32_t v = ring_s + slot * 32768;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_bf16(tm_o + NH * g, sdesc_sw128_mn(v + 2048 * k, 16384),
                     sdesc_sw128(pb + (k >> 2) * SM::QKB + 32 * (k & 3)), idesc_o, (t > 0 || k > 0) ? 1u : 0u);
          mma_commit(empty_b + 8 * slot);
        }
        mma_commit(o_done);
        mma_commit(pbuf_free_b + 8 * sb);
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else {
    // ---------------- softmax: thread i <-> tile row i <-> TMEM lane i ----------------
    const int i = threadIdx.x;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_ref[NH], l_part[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; }
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1;
      const int valid_rows = min(128, r1 - (r0 + 128 * t));
      const int hf = i >> 6;
      bool blk_ok = true;
      {
        const int j0 = r0 + 128 * t + 64 * hf;
        if (j0 < r1) {
          const int blk = a.block_table[(long long)b * a.mbps + j0 / a.bs];
          blk_ok = blk >= 0 && blk < a.n_blocks;
        }
      }
      const bool valid = (i < valid_rows) && blk_ok;
      if (!mbar_wait_warp(s_full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tc_fence_after();
      float s[NH];
#pragma unroll
      for (int c = 0; c < NH / 16; ++c) tmem_ld16(tm_s + NH * sb + lane_base + 16 * c, (uint32_t*)&s[16 * c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free_b + 8 * sb);
      // per-head max down the tile's rows
      float* rb = red + sb * 4 * NH;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float v = valid ? s[h] : -INFINITY;
        v = warp_max(v);
        if (lane == 0) rb[warp * NH + h] = v;
      }
      named_bar_sync(1, 128);
      float alpha[NH];
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float mt = fmaxf(fmaxf(rb[h], rb[NH + h]), fmaxf(rb[2 * NH + h], rb[3 * NH + h])) * a.scale_log2;
        alpha[h] = 1.f;
        if (mt > m_ref[h] + 8.f) {
          if (m_ref[h] != -INFINITY) { alpha[h] = ex2_approx(m_ref[h] - mt); rescale = true; }
          m_ref[h] = mt;
        }
      }
      // P^T(t) into buffer sb once P.V of tile t-2 has released it
      if (!mbar_wait_warp(pbuf_free_b + 8 * sb, ((t >> 1) & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
      uint8_t* pbuf = smem + SM::P_OFF + sb * 2 * SM::QKB + (i >> 6) * SM::QKB;
      const int col = i & 63;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float p = (valid && m_ref[h] != -INFINITY) ? ex2_approx(fmaf(s[h], a.scale_log2, -m_ref[h])) : 0.f;
        const bf16 pb = __float2bfloat16_rn(p);
        l_part[h] = l_part[h] * alpha[h] + __bfloat162float(pb);
        *reinterpret_cast<bf16*>(pbuf + h * 128 + ((((col >> 3) ^ (h & 7))) << 4) + (col & 7) * 2) = pb;
      }
      if (rescale && t >= 1) {   // identical on every thread: m_ref is shared
        if (!mbar_wait_warp(o_done, (t - 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int c = 0; c < NH / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tm_o + NH * g + lane_base + 16 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha[16 * c + k]);
            tmem_st16(tm_o + NH * g + lane_base + 16 * c, o);
          }
        tmem_st_wait();
      }
      if (valid_rows < 128 || !blk_ok) {
        // rows past the context may hold anything (even NaN); P is 0 there, but
        // 0 * NaN is not, so clear row i of the tile's eight latent slots
        if (!valid) {
          for (int g = 0; g < 4; ++g) {
            uint8_t* rowp = smem + SM::RING_OFF + ((5 * t + g) % ATS_NP) * 32768 + i * 128;
            for (int kk = 0; kk < 2; ++kk)
#pragma unroll
              for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(rowp + kk * 16384 + 16 * c) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full_b + 8 * sb);
    }
    if (ok && mbar_wait_warp(o_done, (T - 1) & 1, abort_word, a.flag)) {
      tc_fence_after();
      // l per head = sum of the 128 rows' partial sums
      named_bar_sync(1, 128);
      float* rl = red;   // reuse: [4][NH]
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float v = warp_sum(l_part[h]);
        if (lane == 0) rl[warp * NH + h] = v;
      }
      named_bar_sync(1, 128);
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int c = 0; c < NH / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tm_o + NH * g + lane_base + 16 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int h = 16 * c + k;
            if (h < a.H) a.part_o[(unit * a.H + h) * 512 + 128 * g + i] = __uint_as_float(o[k]);
          }
        }
      if (i == 0) {
#pragma unroll
        for (int h = 0; h < NH; ++h)
          if (h < a.H) {
            a.part_ml[(unit * a.H + h) * 2] = m_ref[h] * 0.69314718055994531f;
            a.part_ml[(unit * a.H + h) * 2 + 1] = rl[h] + rl[NH + h] + rl[2 * NH + h] + rl[3 * NH + h];
          }
      }
    } else if (i < a.H) {
      a.part_ml[(unit * a.H + i) * 2] = -INFINITY;
      a.part_ml[(unit * a.H + i) * 2 + 1] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, SM::TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace mla
