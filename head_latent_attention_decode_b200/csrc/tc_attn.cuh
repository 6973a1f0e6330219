// Absorbed split-KV decode attention on tcgen05 for kv_lora_rank 512 and
// qk_rope 64 (the DeepSeek MLA latent), bf16 cache with blocks of a multiple
// of 64 rows.
//
// One 2-CTA cluster per (sequence, KV split). All heads of the token form the
// MMA's M = 128 rows (fewer heads are padded with zeros). CTA r owns latent
// columns [256 r, 256 r + 256); CTA 0 also owns the 64 rotary columns. Per
// 64-row cache tile:
//   S_r = [q_abs | q_pe]_r . tile_r^T      (tcgen05, M 128 x N 64, K 256 / 320;
//                                          the latent part of Q lives in TMEM)
//   S   = S_0 + S_1                        (the partials swap through DSMEM in f16,
//                                          into two alternating buffers)
//   online softmax, one thread per head (nothing to reduce across threads),
//   lazy rescale of the TMEM accumulator when the max grows by more than 2^8;
//   P (bf16) is written back into TMEM over S
//   O_r += P . V_r                         (tcgen05 with A = P in TMEM, M 128 x
//                                          N 256, K 64; V = the same shared-memory
//                                          tile read MN-major)
// Every cache byte is read from HBM once, O (128 x 512 fp32) is split over the
// two CTAs' TMEM, and a 3-deep ring of tiles keeps loads in flight while the
// MMA thread issues S of later tiles ahead of P.V of earlier ones. Warps 0-3
// run the softmax, warps 6-9 send each tile's partial scores to the peer as
// soon as S lands, warp 4 issues TMA and warp 5 the MMAs. Partials
// (unnormalised O, reference max, sum) go to the workspace and
// attn_combine_kernel merges the splits.
#pragma once

#include "tc_common.cuh"

namespace mla {
namespace tc {

struct TcAttnArgs {
  int n, H, splits, chunk;
  int bs, n_blocks, mbps, max_ctx;
  const int* block_table;
  const int* ctx;
  const bf16* q_abs;   // [n, H, 512]
  int lat_col0, rope_col0;
  float scale_log2;
  float* part_o;   // [n, splits, H, 512]
  float* part_ml;  // [n, splits, H, 2], and the same again at part_ml + ml_r
  int* flag;
  // CTA r of the pair stores its own (m, l) at part_ml + r * ml_r. The two
  // CTAs add the same two partial scores in a different rounding (own fp32 +
  // peer f16), so each half of the latent is normalised with its own statistics.
  long long ml_r;
};

constexpr int ATT_NST = 3;                      // tile ring depth
constexpr int ATT_THREADS = 320;                // 4 softmax, 1 TMA, 1 MMA, 4 sender warps
struct AttnSmem {
  static constexpr int STAGE = 5 * 8192;        // 4 latent + 1 rope slot of [64 rows x 64 cols] bf16
  static constexpr int TILE_OFF = 0;
  static constexpr int QR_OFF = ATT_NST * STAGE;  // q_pe [128 x 64] bf16 (CTA 0)
  static constexpr int X_OFF = QR_OFF + 16384;    // 2 x [128 x 64] f16, the peer's partial S (double-buffered)
  static constexpr int STG_OFF = X_OFF + 32768;   // [128 x 64] f16, our partial on its way out
  static constexpr int BAR_OFF = STG_OFF + 16384;
  static constexpr int SIZE = 1024 + BAR_OFF + 256;
};
// TMEM columns: Q latent [0,128) (bf16 pairs), S/P buffers [128,192) [192,256), O [256,512)
constexpr uint32_t ATT_TM_Q = 0, ATT_TM_S = 128, ATT_TM_O = 256;

__device__ __forceinline__ int attn_tile_rows(const TcAttnArgs& a, int b, int j0, int r1, long long* row) {
  const int blk = a.block_table[(long long)b * a.mbps + j0 / a.bs];
  if (blk < 0 || blk >= a.n_blocks) {
    *row = -64;
    return -1;
  }
  *row = (long long)blk * a.bs + (j0 % a.bs);
  return min(64, r1 - j0);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(ATT_THREADS, 1)
    tc_attn_decode_kernel(const __grid_constant__ CUtensorMap tm_qpe, const __grid_constant__ CUtensorMap tm_cache,
                          const __grid_constant__ CUtensorMap tm_lat, TcAttnArgs a) {
  using SM = AttnSmem;
  griddep_wait();   // the inputs all come from the stream's earlier kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tile_s = sbase + SM::TILE_OFF, qr_s = sbase + SM::QR_OFF, x_s = sbase + SM::X_OFF;
  const uint32_t bar = sbase + SM::BAR_OFF;
  // barriers (8 B each)
  const uint32_t full_b = bar;                 // [ATT_NST] tile landed
  const uint32_t empty_b = bar + 8 * ATT_NST;  // [ATT_NST] tile consumed by P.V
  const uint32_t s_full_b = bar + 16 * ATT_NST;        // [2]
  const uint32_t p_full_b = s_full_b + 16;             // [2]
  const uint32_t sp_empty_b = p_full_b + 16;           // [2] S/P buffer free (P.V done)
  const uint32_t q_ready = sp_empty_b + 16, qr_full = q_ready + 8, o_done = qr_full + 8;
  const uint32_t x_full_b = o_done + 8, x_free_b = x_full_b + 16, fin = x_free_b + 16;   // x_full[2], x_free[2]
  const uint32_t s_read_b = fin + 8;   // [2] the sender has read S(t) out of TMEM
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 192);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 196);

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
  float* const ml = a.part_ml + r * a.ml_r;   // this CTA's (m, l) copy
  if (T == 0) {   // both CTAs of the cluster take this branch together
    if (threadIdx.x < a.H && threadIdx.x < 128) {
      ml[(unit * a.H + threadIdx.x) * 2] = -INFINITY;
      ml[(unit * a.H + threadIdx.x) * 2 + 1] = 0.f;
    }
    return;
  }
  const int nkb = (r == 0) ? 5 : 4;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ATT_NST; ++i) { mbar_init(full_b + 8 * i, 1); mbar_init(empty_b + 8 * i, 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full_b + 8 * i, 1);
      mbar_init(p_full_b + 8 * i, 128);
      mbar_init(sp_empty_b + 8 * i, 1);
    }
    mbar_init(q_ready, 128);
    mbar_init(qr_full, 1);
    mbar_init(o_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(x_full_b + 8 * i, 1);
      mbar_init(x_free_b + 8 * i, 4);
    }
    for (int i = 0; i < 2; ++i) mbar_init(s_read_b + 8 * i, 128);
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
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_cache);
      prefetch_tmap(&tm_lat);
      if (r == 0) {
        mbar_arrive_expect_tx(qr_full, 16384);
        tma_load_3d(qr_s, &tm_qpe, qr_full, 0, b * a.H, 0);
      }
      int t = 0;
      for (; t < T; ++t) {
        const int st = t % ATT_NST;
        if (!mbar_wait(empty_b + 8 * st, ((t / ATT_NST) & 1) ^ 1, abort_word, a.flag)) break;
        long long row;
        if (attn_tile_rows(a, b, r0 + 64 * t, r1, &row) < 0 && r == 0) set_flag(a.flag, MLA_FLAG_BAD_BLOCK);
        mbar_arrive_expect_tx(full_b + 8 * st, nkb * 8192);
        const uint32_t dst = tile_s + st * SM::STAGE;
        // the 4 latent k-blocks of the 64 rows in one box: [8 row octets][4 k-blocks][8 rows][128 B]
        tma_load_4d(dst, &tm_lat, full_b + 8 * st, 0, 0, a.lat_col0 / 64 + 4 * (int)r, (int)(row / 8));
        if (r == 0) tma_load_3d(dst + 4 * 8192, &tm_cache, full_b + 8 * st, a.rope_col0, (int)row, 0);
      }
      // drain the loads still in flight
      if (r == 0) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(qr_full, 0)) if (global_timer_ns() - t0 > WAIT_LIMIT_NS) break;
      }
      for (int u = (t > ATT_NST ? t - ATT_NST : 0); u < t; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(full_b + 8 * (u % ATT_NST), (u / ATT_NST) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 5) {
    // ---------------- MMA issuer: S runs up to two tiles ahead of P.V ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64);
      constexpr uint32_t idesc_o = idesc_bf16(128, 256, 1);
      bool ok = mbar_wait(q_ready, 0, abort_word, a.flag);
      if (ok && r == 0) ok = mbar_wait(qr_full, 0, abort_word, a.flag);
      tc_fence_after();
      // descriptors built once; stages and k-steps add their byte offset >> 4
      const uint64_t d_t = sdesc_sw128_sbo(tile_s, 4096), d_rope = sdesc_sw128(tile_s + 4 * 8192);
      const uint64_t d_qr = sdesc_sw128(qr_s), d_v = sdesc_sw128_mn_sbo(tile_s, 1024, 4096);
      int next_s = 0, next_o = 0;
      uint64_t t_last = global_timer_ns();
      while (ok && next_o < T) {
        bool did = false;
        if (next_s < T && next_s < next_o + 2) {
          const int t = next_s, st = t % ATT_NST, sb = t & 1;
          if (mbar_test(full_b + 8 * st, (t / ATT_NST) & 1) && mbar_test(sp_empty_b + 8 * sb, ((t >> 1) & 1) ^ 1)) {
            tc_fence_after();
            const uint64_t dt = d_t + (uint64_t)(st * (SM::STAGE / 16));
            const uint32_t d = tmem + ATT_TM_S + 64 * sb;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_bf16_ts(d, tmem + ATT_TM_Q + 32 * j + 8 * k, dt + (j * 1024 + 32 * k) / 16, idesc_s,
                            (j > 0 || k > 0) ? 1u : 0u);
            if (r == 0) {
              const uint64_t dr = d_rope + (uint64_t)(st * (SM::STAGE / 16));
#pragma unroll
              for (int k = 0; k < 4; ++k) mma_bf16(d, d_qr + 2 * k, dr + 2 * k, idesc_s, 1u);
            }
            mma_commit(s_full_b + 8 * sb);
            ++next_s;
            did = true;
          }
        }
        if (!did && next_o < next_s) {
          const int u = next_o, st = u % ATT_NST, sb = u & 1;
          if (mbar_test(p_full_b + 8 * sb, (u >> 1) & 1)) {
            tc_fence_after();
            const uint64_t dv = d_v + (uint64_t)(st * (SM::STAGE / 16));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16_ts(tmem + ATT_TM_O, tmem + ATT_TM_S + 64 * sb + 8 * k, dv + 8192 * k / 16, idesc_o,
                          (u > 0 || k > 0) ? 1u : 0u);
            mma_commit(o_done);
            mma_commit(sp_empty_b + 8 * sb);
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
        } else {
          __nanosleep(32);   // leave the issue slots to the softmax warp on this sub-partition
        }
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else if (warp >= 6) {
    // ---------------- senders: S_r(k) -> staging -> one bulk copy into the peer's X ----------------
    const int h = 32 * (warp & 3) + lane;                 // TMEM lane quarter of this warp
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const bool issuer = (warp == 6 && lane == 0);
    const uint32_t peer_x = mapa_shared(x_s, peer), peer_x_full = mapa_shared(x_full_b, peer);
    const uint32_t stg_s = sbase + SM::STG_OFF;
    uint4* stg_row = (uint4*)(smem + SM::STG_OFF + h * 128);
    for (int k = 0; k < T; ++k) {
      const int kb = k & 1;
      if (!mbar_wait_warp(s_full_b + 8 * kb, (k >> 1) & 1, abort_word, a.flag)) break;
      tc_fence_after();
      float v[64];
      const uint32_t sa = tmem + ATT_TM_S + 64 * kb + lane_base;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(sa + 16 * c, (uint32_t*)&v[16 * c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_read_b + 8 * kb);
      if (issuer) bulk_wait_read_all();                  // the previous copy has left the staging buffer
      named_bar_sync(2, 128);
      // the partial goes out in f16 (half the distributed-shared-memory bytes of fp32; the
      // partial scores stay far inside f16's range and its 11-bit significand costs the
      // scores ~1e-3 relative, well inside the output tolerance)
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // chunk c (8 values) of row h at slot c ^ (h & 7): no bank conflicts
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __half2 hv = __floats2half2_rn(v[8 * c + 2 * j], v[8 * c + 2 * j + 1]);
          w[j] = *reinterpret_cast<uint32_t*>(&hv);
        }
        stg_row[c ^ (h & 7)] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(2, 128);
      if (issuer) {
        // the peer has consumed what we sent for tile k - 2 into the same buffer
        const int xb = k & 1;
        bool ok = mbar_wait_cluster(x_free_b + 8 * xb, ((k >> 1) & 1) ^ 1, abort_word, a.flag);
        if (ok) {
          bulk_copy_to_peer(peer_x + xb * 16384, stg_s, 16384, peer_x_full + 8 * xb);
          bulk_commit_group();
        }
      }
    }
    if (issuer) bulk_wait_read_all();
  } else {
    // ---------------- softmax: thread h <-> head h <-> TMEM lane h ----------------
    const int h = threadIdx.x;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // Q latent half of head h -> TMEM (bf16 pairs), zero for padding heads
    {
      const uint4* src = (const uint4*)(a.q_abs + ((long long)b * a.H + (h < a.H ? h : 0)) * 512 + r * 256);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t q[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 v = (h < a.H) ? src[4 * c + k] : make_uint4(0, 0, 0, 0);
          q[4 * k] = v.x; q[4 * k + 1] = v.y; q[4 * k + 2] = v.z; q[4 * k + 3] = v.w;
        }
        tmem_st16(tmem + ATT_TM_Q + lane_base + 16 * c, q);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    const uint32_t peer_x_free = mapa_shared(x_free_b, peer);
    // block of tile t, loaded one tile ahead (only its validity is needed here)
    auto tile_block = [&](int t) -> int {
      return t < T ? a.block_table[(long long)b * a.mbps + (r0 + 64 * t) / a.bs] : 0;
    };
    int blk_next = tile_block(0);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1, st = t % ATT_NST;
      const int blk = blk_next;
      blk_next = tile_block(t + 1);
      const int valid = (blk >= 0 && blk < a.n_blocks) ? min(64, r1 - (r0 + 64 * t)) : 0;
      const int xb = t & 1;
      if (h == 0) mbar_arrive_expect_tx(x_full_b + 8 * xb, 16384);
      if (!mbar_wait_warp(x_full_b + 8 * xb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      if (!mbar_wait_warp(s_full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tc_fence_after();
      float v[64];
      const uint32_t sp_addr = tmem + ATT_TM_S + 64 * sb + lane_base;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16(sp_addr + 16 * c, (uint32_t*)&v[16 * c]);
      tmem_ld_wait();
      const uint4* xloc = (const uint4*)(smem + SM::X_OFF + xb * 16384 + h * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 x = xloc[c ^ (h & 7)];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
          v[8 * c + 2 * j] += f.x;
          v[8 * c + 2 * j + 1] += f.y;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(peer_x_free + 8 * xb);
      // online softmax in log2 units with a lazily moved reference max
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (valid < 64) {
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = (j < valid) ? v[j] : -INFINITY;   // also drops NaN past the context
      }
#pragma unroll
      for (int j = 0; j < 64; ++j) m4[j & 3] = fmaxf(m4[j & 3], v[j]);
      const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + 8.f) {
        if (m_ref != -INFINITY) { alpha = ex2_approx(m_ref - mt); rescale = true; }
        m_ref = mt;
      }
      const float nm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const float e0 = ex2_approx(fmaf(v[j], a.scale_log2, nm)), e1 = ex2_approx(fmaf(v[j + 1], a.scale_log2, nm));
        __nv_bfloat162 pb = __floats2bfloat162_rn(e0, e1);
        ps[(j >> 1) & 3] += e0 + e1;
        pk[j >> 1] = *reinterpret_cast<uint32_t*>(&pb);
      }
      const float psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
      if (__any_sync(0xffffffffu, rescale) && t >= 1) {
        // P.V of the previous tiles must be complete before O is touched
        if (!mbar_wait_warp(o_done, (t - 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tmem + ATT_TM_O + lane_base + 16 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st16(tmem + ATT_TM_O + lane_base + 16 * c, o);
        }
      }
      l = l * alpha + psum;
      if (valid < 64) {
        // rows past the context may hold anything (even NaN); P is 0 there, but
        // 0 * NaN is not, so clear them in the four latent slots before P.V
        // latent rows are laid out [8 row octets][4 k-blocks][8 rows][128 B]
        uint8_t* tl = smem + SM::TILE_OFF + st * SM::STAGE;
        for (int row = valid + (h >> 1); row < 64; row += 64) {
          uint8_t* rp = tl + (row >> 3) * 4096 + (row & 7) * 128 + (h & 1) * 2048;
#pragma unroll
          for (int c = 0; c < 16; ++c)   // two of the four k-blocks: 256 bytes
            *reinterpret_cast<uint4*>(rp + (c >> 3) * 1024 + 16 * (c & 7)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      // the sender must have read S(t) before P overwrites it
      if (!mbar_wait_warp(s_read_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tmem_st16(sp_addr, pk);            // P over S: 32 columns of bf16 pairs
      tmem_st16(sp_addr + 16, pk + 16);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full_b + 8 * sb);
    }
    // every MMA, the last P.V included, has completed once `fin` does (waiting
    // on o_done's parity could pass while an earlier P.V is still running)
    if (ok && mbar_wait_warp(fin, 0, abort_word, a.flag)) {
      tc_fence_after();
      float* po = a.part_o + (unit * a.H + h) * 512 + r * 256;
      for (int c = 0; c < 16; ++c) {
        uint32_t o[16];
        tmem_ld16(tmem + ATT_TM_O + lane_base + 16 * c, o);
        tmem_ld_wait();
        if (h < a.H) {
#pragma unroll
          for (int k = 0; k < 16; k += 4)
            *reinterpret_cast<float4*>(po + 16 * c + k) =
                make_float4(__uint_as_float(o[k]), __uint_as_float(o[k + 1]), __uint_as_float(o[k + 2]),
                            __uint_as_float(o[k + 3]));
        }
      }
      if (h < a.H) {
        ml[(unit * a.H + h) * 2] = m_ref * 0.69314718055994531f;   // natural-log units
        ml[(unit * a.H + h) * 2 + 1] = l;
      }
    } else if (h < a.H) {
      ml[(unit * a.H + h) * 2] = -INFINITY;
      ml[(unit * a.H + h) * 2 + 1] = 0.f;
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
