// Causal expanded prefill attention on tcgen05 for qk_nope 128, qk_rope 64,
// v_dim 128 ("QKV CTE MLA Kernel API Reference", qkv_mla_mx, Final assembly:
// K_h = [k_nope_h | k_pe] with the rotated k_pe shared by every head, V_h from
// the value half of wkv_b's output).
//
// One CTA per (128-query tile, head), head-major. Per 128-key tile j <= the query tile:
//   S = Q_h . K_h^T           tcgen05, M 128 x N 128, K 192 (Q resident in smem)
//   online softmax, one thread per query row holding its whole score row in
//   registers, lazy rescale of O when the row max grows by more than 2^8; keys
//   past the query (diagonal tile) and past the sequence are masked (the other
//   tiles skip the masks); P (bf16) is written into TMEM over S
//   O += P . V_h              tcgen05 with A = P in TMEM, M 128 x N 128, K 128,
//                             V read MN-major from its TMA tile
// K/V tiles stream through a 2-stage TMA ring; S runs one tile ahead of P.V.
// Warps 0-7 run the softmax (two threads per query row, 64 columns each, the
// row maxima exchanged through shared memory), warp 8 issues TMA, warp 9 MMAs.
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

struct TcPrefillAttnArgs {
  int S, H, q_tiles;
  float scale_log2;
  bf16* out;          // [S, H * 128]
  int* flag;
};

struct PaSmem {
  static constexpr int Q_OFF = 0;                         // 3 x [128 x 64] bf16
  static constexpr int STAGE = 5 * 16384;                 // K: 3 x [128 x 64], V: 2 x [128 x 64]
  static constexpr int ST_OFF = 3 * 16384;
  static constexpr int MX_OFF = ST_OFF + 2 * STAGE;       // [2 buffers][2 halves][128] fp32 row maxima
  static constexpr int LX_OFF = MX_OFF + 2 * 2 * 128 * 4;  // [2 halves][128] fp32 row sums
  static constexpr int BAR_OFF = LX_OFF + 2 * 128 * 4;
  static constexpr int SIZE = 1024 + BAR_OFF + 256;
};
// TMEM columns: S/P buffers [0,128) [128,256), O [256,384)
constexpr uint32_t PA_TM_S = 0, PA_TM_O = 256;

__global__ void __launch_bounds__(320, 1)
    tc_prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                           const __grid_constant__ CUtensorMap tm_kpe, TcPrefillAttnArgs a) {
  using SM = PaSmem;
  griddep_wait();   // the inputs all come from the stream's earlier kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + SM::Q_OFF, st_s = sbase + SM::ST_OFF, bar = sbase + SM::BAR_OFF;
  const uint32_t full_b = bar, empty_b = bar + 16, s_full_b = bar + 32, p_full_b = bar + 48;
  const uint32_t sp_empty_b = bar + 64, q_full = bar + 80, o_done = bar + 88, fin = bar + 96;
  const uint32_t mx_b = bar + 104, lx_b = bar + 120;   // [2] half-row maxima posted; half-row sums posted
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 128);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 132);

  // head-major order so that the CTAs in flight share one or two heads' K/V in
  // L2; within a head the heaviest query tiles (causal work grows with the
  // tile index) go first
  const int h = (int)(blockIdx.x / a.q_tiles);
  const int qt = a.q_tiles - 1 - (int)(blockIdx.x % a.q_tiles);
  const int T = qt + 1;                       // key tiles 0..qt
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(full_b + 8 * i, 1);
      mbar_init(empty_b + 8 * i, 1);
      mbar_init(s_full_b + 8 * i, 1);
      mbar_init(p_full_b + 8 * i, 8);   // one arrival per softmax warp
      mbar_init(mx_b + 8 * i, 8);
      mbar_init(sp_empty_b + 8 * i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    mbar_init(lx_b, 8);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_kv);
      mbar_arrive_expect_tx(q_full, 3 * 16384);
      for (int j = 0; j < 3; ++j) tma_load_3d(q_s + j * 16384, &tm_q, q_full, h * 192 + 64 * j, qt * 128, 0);
      int t = 0;
      for (; t < T; ++t) {
        const int st = t & 1;
        if (!mbar_wait(empty_b + 8 * st, ((t >> 1) & 1) ^ 1, abort_word, a.flag)) break;
        const uint32_t dst = st_s + st * SM::STAGE;
        mbar_arrive_expect_tx(full_b + 8 * st, 5 * 16384);
        tma_load_3d(dst, &tm_kv, full_b + 8 * st, h * 256, t * 128, 0);               // k_nope 0..63
        tma_load_3d(dst + 16384, &tm_kv, full_b + 8 * st, h * 256 + 64, t * 128, 0);  // k_nope 64..127
        tma_load_3d(dst + 2 * 16384, &tm_kpe, full_b + 8 * st, 0, t * 128, 0);        // k_pe
        tma_load_3d(dst + 3 * 16384, &tm_kv, full_b + 8 * st, h * 256 + 128, t * 128, 0);  // v 0..63
        tma_load_3d(dst + 4 * 16384, &tm_kv, full_b + 8 * st, h * 256 + 192, t * 128, 0);  // v 64..127
      }
      {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(q_full, 0)) if (global_timer_ns() - t0 > WAIT_LIMIT_NS) break;
      }
      for (int u = (t > 2 ? t - 2 : 0); u < t; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(full_b + 8 * (u & 1), (u >> 1) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128);
      constexpr uint32_t idesc_o = idesc_bf16(128, 128, 1);
      bool ok = mbar_wait(q_full, 0, abort_word, a.flag);
      // descriptors built once; buffers and k-steps add their byte offset >> 4
      const uint64_t d_q = sdesc_sw128(q_s), d_k = sdesc_sw128(st_s);
      const uint64_t d_v = sdesc_sw128_mn(st_s + 3 * 16384, 16384);
      int next_s = 0, next_o = 0;
      uint64_t t_last = global_timer_ns();
      while (ok && next_o < T) {
        bool did = false;
        if (next_s < T && next_s < next_o + 2) {
          const int t = next_s, st = t & 1;
          if (mbar_test(full_b + 8 * st, (t >> 1) & 1) && mbar_test(sp_empty_b + 8 * st, ((t >> 1) & 1) ^ 1)) {
            tc_fence_after();
            const uint64_t dk = d_k + (uint64_t)(st * (SM::STAGE / 16));
#pragma unroll
            for (int j = 0; j < 3; ++j)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + PA_TM_S + 128 * st, d_q + (j * 16384 + 32 * k) / 16, dk + (j * 16384 + 32 * k) / 16,
                         idesc_s, (j > 0 || k > 0) ? 1u : 0u);
            mma_commit(s_full_b + 8 * st);
            ++next_s;
            did = true;
          }
        }
        if (!did && next_o < next_s) {
          const int u = next_o, st = u & 1;
          if (mbar_test(p_full_b + 8 * st, (u >> 1) & 1)) {
            tc_fence_after();
            const uint64_t dv = d_v + (uint64_t)(st * (SM::STAGE / 16));
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_bf16_ts(tmem + PA_TM_O, tmem + PA_TM_S + 128 * st + 8 * k, dv + 2048 * k / 16, idesc_o,
                          (u > 0 || k > 0) ? 1u : 0u);
            mma_commit(o_done);
            mma_commit(sp_empty_b + 8 * st);
            mma_commit(empty_b + 8 * st);
            ++next_o;
            did = true;
          }
        }
        if (did) {
          t_last = global_timer_ns();
        } else if (*abort_word) {
          ok = false;
        } else if (global_timer_ns() - t_last > WAIT_LIMIT_NS) {
          *abort_word = 1;
          set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT);
          ok = false;
        }
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else {
    // ---------------- softmax: two threads per query row (TMEM lane), 64 columns each ----------------
    const int row = threadIdx.x & 127, half = threadIdx.x >> 7;
    const int qi = qt * 128 + row;                // this thread's query position
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float* mx = (float*)(smem + SM::MX_OFF);      // [sb][half][row]
    float* lx = (float*)(smem + SM::LX_OFF);      // [half][row]
    float m_ref = -INFINITY, l = 0.f;             // the same reference in both threads of a row
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1;
      // keys k0 .. k0+127; key k valid iff k <= qi and k < S
      const int k0 = t * 128;
      const int lim = min(qi, a.S - 1) - k0 + 1 - 64 * half;   // valid columns of this half: [0, lim)
      if (!mbar_wait_warp(s_full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = tmem + PA_TM_S + 128 * sb + lane_base;
      // this half of the score row in registers
      uint32_t r[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(sa + 64 * half + 16 * c, r + 16 * c);
      tmem_ld_wait();
      // only the diagonal (or the sequence's last) tile has masked columns
      const bool full = __all_sync(0xffffffffu, lim >= 64);
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full) {
#pragma unroll
        for (int j = 0; j < 64; ++j) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(r[j]));
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (j < lim) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(r[j]));
      }
      // the row max from both halves (a rendezvous of the eight warps on an mbarrier: a bounded wait)
      mx[(sb * 2 + half) * 128 + row] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(mx_b + 8 * sb);
      if (!mbar_wait_warp(mx_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      const float mt = fmaxf(mx[(sb * 2) * 128 + row], mx[(sb * 2 + 1) * 128 + row]) * a.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + 8.f) {
        if (m_ref != -INFINITY) { alpha = ex2_approx(m_ref - mt); rescale = true; }
        m_ref = mt;
      }
      const float nm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      if (__any_sync(0xffffffffu, rescale) && t >= 1) {
        if (!mbar_wait_warp(o_done, (t - 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < 4; ++c) {   // this half's 64 columns of O
          uint32_t o[16];
          const uint32_t oa = tmem + PA_TM_O + lane_base + 64 * half + 16 * c;
          tmem_ld16(oa, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st16(oa, o);
        }
      }
      // P = 2^(s*scale - m) in bf16, written over S: this half's 32 column pairs.
      // Both halves loaded their scores before the rendezvous, so no score is overwritten unread.
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const int col = 32 * c + j;
          float p0 = ex2_approx(fmaf(__uint_as_float(r[col]), a.scale_log2, nm));
          float p1 = ex2_approx(fmaf(__uint_as_float(r[col + 1]), a.scale_log2, nm));
          if (!full) {
            p0 = col < lim ? p0 : 0.f;
            p1 = col + 1 < lim ? p1 : 0.f;
          }
          __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          ps[(j >> 1) & 3] += __low2float(pb) + __high2float(pb);
          pk[j >> 1] = *reinterpret_cast<uint32_t*>(&pb);
        }
        tmem_st16(sa + 32 * half + 16 * c, pk);
      }
      l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full_b + 8 * sb);
    }
    // every MMA, the last P.V included, has completed once `fin` does (waiting
    // on o_done's parity could pass while an earlier P.V is still running)
    if (ok && mbar_wait_warp(fin, 0, abort_word, a.flag)) {
      tc_fence_after();
      // the row sum from both halves
      lx[half * 128 + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(lx_b);
      if (mbar_wait_warp(lx_b, 0, abort_word, a.flag)) {
        const float lsum = lx[row] + lx[128 + row];
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        bf16* o_row = a.out + (long long)qi * a.H * 128 + h * 128 + 64 * half;
        for (int c = 0; c < 4; ++c) {
          uint32_t o[16];
          tmem_ld16(tmem + PA_TM_O + lane_base + 64 * half + 16 * c, o);
          tmem_ld_wait();
          if (qi < a.S) {
            uint4 w0, w1;
            w0.x = pack_bf16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
            w0.y = pack_bf16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
            w0.z = pack_bf16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
            w0.w = pack_bf16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
            w1.x = pack_bf16x2(__uint_as_float(o[8]) * inv, __uint_as_float(o[9]) * inv);
            w1.y = pack_bf16x2(__uint_as_float(o[10]) * inv, __uint_as_float(o[11]) * inv);
            w1.z = pack_bf16x2(__uint_as_float(o[12]) * inv, __uint_as_float(o[13]) * inv);
            w1.w = pack_bf16x2(__uint_as_float(o[14]) * inv, __uint_as_float(o[15]) * inv);
            *reinterpret_cast<uint4*>(o_row + 16 * c) = w0;
            *reinterpret_cast<uint4*>(o_row + 16 * c + 8) = w1;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace mla
