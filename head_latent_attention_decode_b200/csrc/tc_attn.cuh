// Absorbed split-KV decode attention on tcgen05 for kv_lora_rank 512 and
// qk_rope 64 (the DeepSeek MLA latent), bf16 cache with blocks of a multiple
// of 64 rows.
//
// One 2-CTA cluster per (sequence, KV split). All heads of the token form the
// MMA's M = 128 rows (fewer heads are padded). CTA r owns latent columns
// [256 r, 256 r + 256); CTA 0 also owns the 64 rotary columns. Per 64-row
// cache tile:
//   S_r = [q_abs | q_pe]_r . tile_r^T        (tcgen05, M 128 x N 64, K 256/320)
//   S   = S_0 + S_1                          (partials swapped through DSMEM)
//   online softmax per head (one thread per head, nothing to reduce across
//   threads), lazy rescale of the TMEM accumulator when the max grows by > 2^8
//   O_r += P . V_r                           (tcgen05, M 128 x N 256, K 64,
//                                             V = the same smem tile read MN-major)
// so every cache byte is read from HBM once and O (128 x 512 fp32) is split
// over the two CTAs' TMEM. Partials (unnormalised O, running max, sum) go to
// the workspace and attn_combine_kernel merges the splits.
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

struct TcAttnArgs {
  int n, H, splits, chunk;
  int bs, n_blocks, mbps, max_ctx;
  const int* block_table;
  const int* ctx;
  int lat_col0, rope_col0;
  float scale_log2;
  float* part_o;   // [n, splits, H, 512]
  float* part_ml;  // [n, splits, H, 2]
  int* flag;
};

struct AttnSmem {
  static constexpr int Q_OFF = 0;                        // 5 x [128 x 64] bf16
  static constexpr int TILE_OFF = 5 * 16384;             // 2 stages x 5 x [64 x 64] bf16
  static constexpr int P_OFF = TILE_OFF + 2 * 5 * 8192;  // [128 x 64] bf16
  static constexpr int X_OFF = P_OFF + 16384;            // [128 x 64] fp32 (peer's partial S)
  static constexpr int BAR_OFF = X_OFF + 32768;
  static constexpr int SIZE = 1024 + BAR_OFF + 256;
};

__device__ __forceinline__ int attn_tile_rows(const TcAttnArgs& a, int b, int j0, int r1, long long* row) {
  const int blk = a.block_table[(long long)b * a.mbps + j0 / a.bs];
  if (blk < 0 || blk >= a.n_blocks) {
    *row = -64;
    return -1;
  }
  *row = (long long)blk * a.bs + (j0 % a.bs);
  return min(64, r1 - j0);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    tc_attn_decode_kernel(const __grid_constant__ CUtensorMap tm_qabs, const __grid_constant__ CUtensorMap tm_qpe,
                          const __grid_constant__ CUtensorMap tm_cache, TcAttnArgs a) {
  using SM = AttnSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + SM::Q_OFF, tile_s = sbase + SM::TILE_OFF, p_s = sbase + SM::P_OFF;
  const uint32_t x_s = sbase + SM::X_OFF, bar = sbase + SM::BAR_OFF;
  const uint32_t full_b = bar, empty_b = bar + 16, q_full = bar + 32, s_full_b = bar + 40, s_empty_b = bar + 56;
  const uint32_t p_full = bar + 72, o_done = bar + 80, x_full = bar + 88, x_free = bar + 96, fin = bar + 104;
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 128);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 132);

  const uint32_t r = cluster_ctarank(), peer = r ^ 1u;
  const int cid = blockIdx.x >> 1;
  const int b = cid / a.splits, sp = cid % a.splits;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int L = a.ctx[b];
  if (L < 1 || L > a.max_ctx || L > a.mbps * a.bs) {
    if (threadIdx.x == 0 && r == 0 && sp == 0) set_flag(a.flag, MLA_FLAG_BAD_CONTEXT);
    L = 0;
  }
  const int r0 = sp * a.chunk, r1 = min(L, r0 + a.chunk);
  const int T = r1 > r0 ? (r1 - r0 + 63) / 64 : 0;
  const long long unit = (long long)b * a.splits + sp;
  if (T == 0) {   // both CTAs of the cluster take this branch together
    if (r == 0 && threadIdx.x < a.H && threadIdx.x < 128) {
      a.part_ml[(unit * a.H + threadIdx.x) * 2] = -INFINITY;
      a.part_ml[(unit * a.H + threadIdx.x) * 2 + 1] = 0.f;
    }
    return;
  }
  const int nkb = (r == 0) ? 5 : 4;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(full_b + 8 * i, 1);
      mbar_init(empty_b + 8 * i, 1);
      mbar_init(s_full_b + 8 * i, 1);
      mbar_init(s_empty_b + 8 * i, 128);
    }
    mbar_init(q_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(x_full, 128);
    mbar_init(x_free, 128);
    mbar_init(fin, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_S = tmem, tmem_O = tmem + 256;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_cache);
      mbar_arrive_expect_tx(q_full, nkb * 16384);
      for (int j = 0; j < 4; ++j)
        tma_load_3d(q_s + j * 16384, &tm_qabs, q_full, (int)r * 256 + 64 * j, b * a.H, 0);
      if (r == 0) tma_load_3d(q_s + 4 * 16384, &tm_qpe, q_full, 0, b * a.H, 0);
      int t = 0;
      for (; t < T; ++t) {
        const int st = t & 1;
        if (!mbar_wait(empty_b + 8 * st, ((t >> 1) & 1) ^ 1, abort_word, a.flag)) break;
        long long row;
        if (attn_tile_rows(a, b, r0 + 64 * t, r1, &row) < 0 && r == 0) set_flag(a.flag, MLA_FLAG_BAD_BLOCK);
        mbar_arrive_expect_tx(full_b + 8 * st, nkb * 8192);
        const uint32_t dst = tile_s + st * 5 * 8192;
        for (int j = 0; j < 4; ++j)
          tma_load_3d(dst + j * 8192, &tm_cache, full_b + 8 * st, a.lat_col0 + (int)r * 256 + 64 * j, (int)row, 0);
        if (r == 0) tma_load_3d(dst + 4 * 8192, &tm_cache, full_b + 8 * st, a.rope_col0, (int)row, 0);
      }
      // drain the loads still in flight
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(q_full, 0)) if (global_timer_ns() - t0 > WAIT_LIMIT_NS) break;
      for (int u = (t > 2 ? t - 2 : 0); u < t; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(full_b + 8 * (u & 1), (u >> 1) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64);
      constexpr uint32_t idesc_o = idesc_bf16(128, 256, 1);
      bool ok = mbar_wait(q_full, 0, abort_word, a.flag);
      auto issue_o = [&](int u) -> bool {
        if (!mbar_wait(p_full, u & 1, abort_word, a.flag)) return false;
        tc_fence_after();
        const uint32_t v = tile_s + (u & 1) * 5 * 8192;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16(tmem_O, sdesc_sw128(p_s + 32 * k), sdesc_sw128_mn(v + 2048 * k, 8192), idesc_o,
                   (u > 0 || k > 0) ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(empty_b + 8 * (u & 1));
        return true;
      };
      int t = 0;
      for (; ok && t < T; ++t) {
        const int sb = t & 1;
        if (!mbar_wait(s_empty_b + 8 * sb, ((t >> 1) & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
        if (!mbar_wait(full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tl = tile_s + sb * 5 * 8192;
        for (int j = 0; j < nkb; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16(tmem_S + sb * 64, sdesc_sw128(q_s + j * 16384 + 32 * k), sdesc_sw128(tl + j * 8192 + 32 * k),
                     idesc_s, (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(s_full_b + 8 * sb);
        if (t >= 1 && !issue_o(t - 1)) { ok = false; break; }
      }
      if (ok) issue_o(T - 1);
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else {
    // ---------------- softmax: thread h <-> head h <-> TMEM lane h ----------------
    const int h = threadIdx.x;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t peer_x = mapa_shared(x_s + h * 256, peer);
    const uint32_t peer_x_full = mapa_shared(x_full, peer), peer_x_free = mapa_shared(x_free, peer);
    const float4* xloc = (const float4*)(smem + SM::X_OFF + h * 256);
    uint8_t* prow = smem + SM::P_OFF + h * 128;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1;
      long long row_unused;
      int valid = attn_tile_rows(a, b, r0 + 64 * t, r1, &row_unused);
      if (valid < 0) valid = 0;
      if (!mbar_wait_warp(s_full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tc_fence_after();
      float s[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(tmem_S + sb * 64 + lane_base + 16 * c, (uint32_t*)&s[16 * c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_empty_b + 8 * sb);
      // swap partial scores with the peer CTA
      if (t >= 1 && !mbar_wait_cluster_warp(x_free, (t - 1) & 1, abort_word, a.flag)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 16; ++c)   // chunk c of row h lives at slot c ^ (h & 15): no bank conflicts
        st_cluster_v4(peer_x + 16 * (c ^ (h & 15)), s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
      mbar_arrive_remote(peer_x_full);
      if (!mbar_wait_cluster_warp(x_full, t & 1, abort_word, a.flag)) { ok = false; break; }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = xloc[c ^ (h & 15)];
        s[4 * c] += v.x; s[4 * c + 1] += v.y; s[4 * c + 2] += v.z; s[4 * c + 3] += v.w;
      }
      mbar_arrive_remote(peer_x_free);
      // online softmax in log2 units with a lazily moved reference max
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        s[j] = (j < valid) ? s[j] * a.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[j]);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + 8.f) {
        if (m_ref != -INFINITY) { alpha = exp2f(m_ref - mt); rescale = true; }
        m_ref = mt;
      }
      float psum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const float p0 = (m_ref == -INFINITY) ? 0.f : exp2f(s[j] - m_ref);
        const float p1 = (m_ref == -INFINITY) ? 0.f : exp2f(s[j + 1] - m_ref);
        __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
        psum += __low2float(pb) + __high2float(pb);
        pk[j >> 1] = *reinterpret_cast<uint32_t*>(&pb);
      }
      // O(t-1) complete: P may be overwritten and O rescaled
      if (t >= 1 && !mbar_wait_warp(o_done, (t - 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale) && t >= 1) {
        for (int c = 0; c < 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tmem_O + lane_base + 16 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st16(tmem_O + lane_base + 16 * c, o);
        }
        tmem_st_wait();
      }
      l = l * alpha + psum;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) << 4)) = v;
      }
      if (valid < 64) {
        // rows past the context may hold anything (even NaN); P is 0 there, but
        // 0 * NaN is not, so clear them in the four latent slots before P.V
        uint8_t* tl = smem + SM::TILE_OFF + (t & 1) * 5 * 8192;
        const int nbytes = (64 - valid) * 128;
        for (int i = h * 16; i < 4 * nbytes; i += 128 * 16) {
          const int j = i / nbytes, off = i % nbytes;
          *reinterpret_cast<uint4*>(tl + j * 8192 + valid * 128 + off) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && mbar_wait_warp(o_done, (T - 1) & 1, abort_word, a.flag)) {
      tc_fence_after();
      float* po = a.part_o + (unit * a.H + h) * 512 + r * 256;
      for (int c = 0; c < 16; ++c) {
        uint32_t o[16];
        tmem_ld16(tmem_O + lane_base + 16 * c, o);
        tmem_ld_wait();
        if (h < a.H) {
#pragma unroll
          for (int k = 0; k < 16; k += 4)
            *reinterpret_cast<float4*>(po + 16 * c + k) =
                make_float4(__uint_as_float(o[k]), __uint_as_float(o[k + 1]), __uint_as_float(o[k + 2]),
                            __uint_as_float(o[k + 3]));
        }
      }
      if (r == 0 && h < a.H) {
        a.part_ml[(unit * a.H + h) * 2] = m_ref * 0.69314718055994531f;   // natural-log units
        a.part_ml[(unit * a.H + h) * 2 + 1] = l;
      }
    } else if (r == 0 && h < a.H) {
      a.part_ml[(unit * a.H + h) * 2] = -INFINITY;
      a.part_ml[(unit * a.H + h) * 2 + 1] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  cluster_sync_all();   // no CTA leaves while its peer may still touch its shared memory
}

}  // namespace tc
}  // namespace mla
