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
// K and V tiles stream through separate 2-stage TMA rings: a K tile is released
// as soon as its S completes, a V tile when its P.V does, so the next K tiles
// load while the softmax runs instead of waiting for P.V. S runs one tile ahead
// of P.V.
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
  const float* sink;  // [H] sink logits (one more softmax column, no value), or NULL
};

struct PaSmem {
  static constexpr int Q_OFF = 0;                         // 3 x [128 x 64] bf16
  static constexpr int KSTAGE = 3 * 16384;                // k_nope 2 x [128 x 64], k_pe [128 x 64]
  static constexpr int VSTAGE = 2 * 16384;                // v 2 x [128 x 64]
  static constexpr int K_OFF = 3 * 16384;
  static constexpr int V_OFF = K_OFF + 2 * KSTAGE;
  static constexpr int MX_OFF = V_OFF + 2 * VSTAGE;       // [3 buffers][2 halves][128] fp32 row maxima
  static constexpr int LX_OFF = MX_OFF + 3 * 2 * 128 * 4;  // [2 halves][128] fp32 row sums
  static constexpr int BAR_OFF = LX_OFF + 2 * 128 * 4;
  static constexpr int SIZE = 1024 + BAR_OFF + 256;
};
// TMEM columns: S/P buffers [0,128) [128,256) [256,384), O [384,512)
constexpr uint32_t PA_TM_S = 0, PA_TM_O = 384;
constexpr int PA_SBUF = 3;   // S/P buffers: S runs up to three tiles ahead of P.V

__global__ void __launch_bounds__(320, 1)
    tc_prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                           const __grid_constant__ CUtensorMap tm_kpe, TcPrefillAttnArgs a) {
  using SM = PaSmem;
  griddep_wait();   // the inputs all come from the stream's earlier kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + SM::Q_OFF, k_s = sbase + SM::K_OFF, v_s = sbase + SM::V_OFF;
  const uint32_t bar = sbase + SM::BAR_OFF;
  const uint32_t kfull_b = bar, kempty_b = bar + 16;                        // [2] K ring
  const uint32_t vfull_b = bar + 32, vempty_b = bar + 48;                    // [2] V ring
  const uint32_t s_full_b = bar + 64, p_full_b = bar + 88, sp_empty_b = bar + 112;   // [3] per S/P buffer
  const uint32_t mx_b = bar + 136;                                           // [3] half-row maxima posted
  // o_done[u & 1] completes with P.V(u): with S up to three tiles ahead, P.V may lag the
  // softmax by two tiles, which one barrier's parity could not tell apart
  const uint32_t q_full = bar + 160, o_done = bar + 168, fin = bar + 184, lx_b = bar + 192;
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 224);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 228);

  // head-major order so that the CTAs in flight share one or two heads' K/V in
  // L2; within a head the heaviest query tiles (causal work grows with the
  // tile index) go first
  const int h = (int)(blockIdx.x / a.q_tiles);
  const int qt = a.q_tiles - 1 - (int)(blockIdx.x % a.q_tiles);
  const int T = qt + 1;                       // key tiles 0..qt
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(kfull_b + 8 * i, 1);
      mbar_init(kempty_b + 8 * i, 1);
      mbar_init(vfull_b + 8 * i, 1);
      mbar_init(vempty_b + 8 * i, 1);
    }
    for (int i = 0; i < PA_SBUF; ++i) {
      mbar_init(s_full_b + 8 * i, 1);
      mbar_init(p_full_b + 8 * i, 8);   // one arrival per softmax warp
      mbar_init(mx_b + 8 * i, 8);
      mbar_init(sp_empty_b + 8 * i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(o_done, 1);
    mbar_init(o_done + 8, 1);
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
      // K(t) needs S(t-2) done, V(t) needs P.V(t-2) done: issue each as soon as its slot frees
      int kt = 0, vt = 0;
      bool ok = true;
      uint64_t t_last = global_timer_ns();
      while (ok && (kt < T || vt < T)) {
        bool did = false;
        if (kt < T && mbar_test(kempty_b + 8 * (kt & 1), ((kt >> 1) & 1) ^ 1)) {
          const uint32_t kb = kfull_b + 8 * (kt & 1), dst = k_s + (kt & 1) * SM::KSTAGE;
          mbar_arrive_expect_tx(kb, 3 * 16384);
          tma_load_3d(dst, &tm_kv, kb, h * 256, kt * 128, 0);               // k_nope 0..63
          tma_load_3d(dst + 16384, &tm_kv, kb, h * 256 + 64, kt * 128, 0);  // k_nope 64..127
          tma_load_3d(dst + 2 * 16384, &tm_kpe, kb, 0, kt * 128, 0);        // k_pe
          ++kt;
          did = true;
        }
        if (vt < kt && mbar_test(vempty_b + 8 * (vt & 1), ((vt >> 1) & 1) ^ 1)) {
          const uint32_t vb = vfull_b + 8 * (vt & 1), dst = v_s + (vt & 1) * SM::VSTAGE;
          mbar_arrive_expect_tx(vb, 2 * 16384);
          tma_load_3d(dst, &tm_kv, vb, h * 256 + 128, vt * 128, 0);           // v 0..63
          tma_load_3d(dst + 16384, &tm_kv, vb, h * 256 + 192, vt * 128, 0);   // v 64..127
          ++vt;
          did = true;
        }
        if (did) {
          t_last = global_timer_ns();
        } else if (*abort_word) {
          ok = false;
        } else if (global_timer_ns() - t_last > WAIT_LIMIT_NS) {
          *abort_word = 1;
          set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT);
          ok = false;
        } else {
          __nanosleep(32);
        }
      }
      // drain the loads still in flight
      {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(q_full, 0)) if (global_timer_ns() - t0 > WAIT_LIMIT_NS) break;
      }
      for (int u = (kt > 2 ? kt - 2 : 0); u < kt; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(kfull_b + 8 * (u & 1), (u >> 1) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
      for (int u = (vt > 2 ? vt - 2 : 0); u < vt; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(vfull_b + 8 * (u & 1), (u >> 1) & 1))
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
      const uint64_t d_q = sdesc_sw128(q_s), d_k = sdesc_sw128(k_s);
      const uint64_t d_v = sdesc_sw128_mn(v_s, 16384);
      int next_s = 0, next_o = 0;
      uint32_t idle = 0;
      uint64_t t_idle = 0;
      while (ok && next_o < T) {
        bool did = false;
        // P.V first: the S buffer it frees is what lets S run ahead
        if (next_o < next_s) {
          const int u = next_o, sb = u % PA_SBUF, vs = u & 1;
          if (mbar_test(p_full_b + 8 * sb, (u / PA_SBUF) & 1) && mbar_test(vfull_b + 8 * vs, (u >> 1) & 1)) {
            tc_fence_after();
            const uint64_t dv = d_v + (uint64_t)(vs * (SM::VSTAGE / 16));
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_bf16_ts(tmem + PA_TM_O, tmem + PA_TM_S + 128 * sb + 8 * k, dv + 2048 * k / 16, idesc_o,
                          (u > 0 || k > 0) ? 1u : 0u);
            mma_commit(o_done + 8 * (u & 1));
            mma_commit(sp_empty_b + 8 * sb);
            mma_commit(vempty_b + 8 * vs);
            ++next_o;
            did = true;
          }
        }
        if (!did && next_s < T && next_s < next_o + PA_SBUF) {
          const int t = next_s, sb = t % PA_SBUF, ks = t & 1;
          if (mbar_test(kfull_b + 8 * ks, (t >> 1) & 1) &&
              mbar_test(sp_empty_b + 8 * sb, ((t / PA_SBUF) & 1) ^ 1)) {
            tc_fence_after();
            const uint64_t dk = d_k + (uint64_t)(ks * (SM::KSTAGE / 16));
#pragma unroll
            for (int j = 0; j < 3; ++j)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + PA_TM_S + 128 * sb, d_q + (j * 16384 + 32 * k) / 16, dk + (j * 16384 + 32 * k) / 16,
                         idesc_s, (j > 0 || k > 0) ? 1u : 0u);
            mma_commit(s_full_b + 8 * sb);
            mma_commit(kempty_b + 8 * ks);
            ++next_s;
            did = true;
          }
        }
        // the clock is read only while idle: first idle pass, then every 64th; an
        // idle pass backs off so that the polling does not take issue slots from
        // the softmax warps sharing this scheduler
        if (did) {
          idle = 0;
        } else if (*abort_word) {
          ok = false;
        } else {
          if ((++idle & 63) == 1) {
            const uint64_t now = global_timer_ns();
            if (idle == 1) {
              t_idle = now;
            } else if (now - t_idle > WAIT_LIMIT_NS) {
              *abort_word = 1;
              set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT);
              ok = false;
            }
          }
          __nanosleep(32);
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
    float* mx = (float*)(smem + SM::MX_OFF);      // [sb][half][row], sb = S/P buffer
    float* lx = (float*)(smem + SM::LX_OFF);      // [half][row]
    float m_ref = -INFINITY, l = 0.f;             // the same reference in both threads of a row
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t % PA_SBUF, ph = (t / PA_SBUF) & 1;
      // keys k0 .. k0+127; key k valid iff k <= qi and k < S
      const int k0 = t * 128;
      const int lim = min(qi, a.S - 1) - k0 + 1 - 64 * half;   // valid columns of this half: [0, lim)
      if (!mbar_wait_warp(s_full_b + 8 * sb, ph, abort_word, a.flag)) { ok = false; break; }
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
      if (!mbar_wait_warp(mx_b + 8 * sb, ph, abort_word, a.flag)) { ok = false; break; }
      const float mt = fmaxf(mx[(sb * 2) * 128 + row], mx[(sb * 2 + 1) * 128 + row]) * a.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + 8.f) {
        if (m_ref != -INFINITY) { alpha = ex2_approx(m_ref - mt); rescale = true; }
        m_ref = mt;
      }
      const float nm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      if (__any_sync(0xffffffffu, rescale) && t >= 1) {
        if (!mbar_wait_warp(o_done + 8 * ((t - 1) & 1), ((t - 1) >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
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
        float lsum = lx[row] + lx[128 + row];
        // a sink logit z joins the denominator as e^z (m_ref is in log2 units of the scaled scores)
        if (a.sink && lsum > 0.f) lsum += ex2_approx(fmaf(a.sink[h], 1.4426950408889634f, -m_ref));
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
