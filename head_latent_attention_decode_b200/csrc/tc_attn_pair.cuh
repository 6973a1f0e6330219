// Absorbed split-KV decode attention on tcgen05 for few heads (H <= 32), with
// the DeepSeek latent (kv_lora_rank 512, qk_rope 64) and cache blocks of a
// multiple of 64 rows. The MMAs run transposed so that the cache rows, not the
// heads, fill the tensor core's M = 128, and one 2-CTA cluster per (sequence,
// split) divides every 128-row tile by columns:
//   CTA r holds latent columns [256 r, 256 r + 256) of each tile, and the 64
//   rotary columns of the tiles t with t % 2 == r;
//   S_r^T = tile_r . Q_r^T               M 128 rows x N NH heads, K 256 or 320
//   S^T   = S_r^T + S_peer^T             each softmax thread sends its row (NH
//                                        values, in f16) into the peer's shared
//                                        memory with st.async, ahead of its own
//                                        softmax
//   softmax down each head's column with a lazily moved reference max: the
//   rows vote whether any score exceeds its head's reference by more than 2^8,
//   and only then are the column maxima reduced (warp redux and a 4-warp
//   exchange) and O^T rescaled; per-row partial sums are reduced once at the
//   end. Both CTAs add the same two partials, each its own in fp32 and the
//   peer's in f16, so their P^T agree to the f16 rounding of a partial score
//   O_r^T += V_r^T . P^T                 2 x (M 128 latent x N NH, K 128 rows),
//                                        V^T read MN-major from the same tile
// A CTA keeps 64 KB of a tile until its P.V (half of what one CTA holding the
// whole tile needs), so its ring of 32 KB entries holds two and a half (NH 16)
// or two (NH 32) tiles and the next tiles stream in during the softmax.
#pragma once

#include "tc_attn.cuh"

namespace mla {
namespace tc {

template <int NH>
struct AttnPairSmem {
  // ring entries: [128 rows x 128 latent] bf16, 32 KB, laid out [16 row octets][2 k-blocks][8 rows][128 B]
  static constexpr int NPR = NH <= 16 ? 5 : 4;
  static constexpr int QKB = NH * 128;                   // one [NH x 64] bf16 k-block of Q or P^T
  static constexpr int XB = 128 * NH * 2;                // one [128 x NH] f16 partial S^T
  static constexpr int RING_OFF = 0;
  static constexpr int ROPE_OFF = NPR * 32768;           // [128 x 64] rotary block of the current tile
  static constexpr int Q_OFF = ROPE_OFF + 16384;         // this CTA's 4 latent k-blocks of Q, then q_pe
  static constexpr int P_OFF = Q_OFF + 5 * QKB;          // 2 buffers x 2 k-blocks of P^T
  static constexpr int X_OFF = P_OFF + 4 * QKB;          // 2 buffers: the peer's partial S^T
  static constexpr int RED_OFF = X_OFF + 2 * XB;         // 4 x NH fp32 column maxima, then 4 x NH row sums
  static constexpr int BAR_OFF = RED_OFF + 2 * 4 * NH * 4;
  static constexpr int SIZE = 1024 + BAR_OFF + 512;
  static constexpr int TMEM_COLS = 4 * NH <= 64 ? 64 : 128;   // S^T x 2, O^T x 2
};

template <int NH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(224, 1)
    tc_attn_pair_kernel(const __grid_constant__ CUtensorMap tm_qabs, const __grid_constant__ CUtensorMap tm_qpe,
                        const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_lat,
                        TcAttnArgs a) {
  using SM = AttnPairSmem<NH>;
  griddep_wait();   // the inputs all come from the stream's earlier kernels
  constexpr int NPR = SM::NPR, QKB = SM::QKB;
  constexpr int CPR = NH / 8;                  // 16-byte chunks per row of an f16 partial
  constexpr int XSH = NH == 16 ? 2 : 1;        // chunk swizzle: the rows of one 128-byte line cover all 32 banks
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t ring_s = sbase + SM::RING_OFF, rope_s = sbase + SM::ROPE_OFF, q_s = sbase + SM::Q_OFF,
                 p_s = sbase + SM::P_OFF, x_s = sbase + SM::X_OFF;
  float* red = (float*)(smem + SM::RED_OFF);
  const uint32_t bar = sbase + SM::BAR_OFF;
  const uint32_t full_b = bar, empty_b = bar + 8 * NPR;          // [NPR] ring entry landed / consumed by P.V
  const uint32_t rfull = empty_b + 8 * NPR, rempty = rfull + 8;   // rotary block landed / consumed by S
  const uint32_t q_full = rempty + 8;
  const uint32_t s_full_b = q_full + 8, s_free_b = s_full_b + 16;          // [2] S^T ready / read
  const uint32_t p_full_b = s_free_b + 16, pbuf_free_b = p_full_b + 16;    // [2] P^T written / consumed
  const uint32_t o_done = pbuf_free_b + 16;
  const uint32_t x_full_b = o_done + 8, x_free_b = x_full_b + 16;          // [2] peer partial in / our X free
  const uint32_t fin = x_free_b + 16;
  const uint32_t red_b = fin + 8, l_done = red_b + 16;                     // [2] votes posted; row sums posted
  const uint32_t red2_b = l_done + 8;                                      // column maxima posted
  const uint32_t fin_s = red2_b + 8;                                       // every S^T MMA complete
  volatile int* vote = (volatile int*)(smem + SM::BAR_OFF + 392);          // [2] last tile that voted
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 384);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 388);

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
  const int T = r1 > r0 ? (r1 - r0 + 127) / 128 : 0;
  const long long unit = (long long)b * a.splits + sp;
  // CTA r stores its own (m, l) at part_ml + r * ml_r: the two CTAs add the
  // same two partial scores in a different rounding (own fp32 + peer f16), so
  // their lazily moved reference maxima can differ, and each latent half is
  // normalised with the statistics of the CTA that accumulated it
  float* const ml = a.part_ml + r * a.ml_r;
  if (T == 0) {   // both CTAs of the cluster take this branch together
    if (threadIdx.x < a.H) {
      ml[(unit * a.H + threadIdx.x) * 2] = -INFINITY;
      ml[(unit * a.H + threadIdx.x) * 2 + 1] = 0.f;
    }
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NPR; ++i) { mbar_init(full_b + 8 * i, 1); mbar_init(empty_b + 8 * i, 1); }
    mbar_init(rfull, 1);
    mbar_init(rempty, 1);
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full_b + 8 * i, 1);
      mbar_init(s_free_b + 8 * i, 4);   // one arrival per softmax warp
      mbar_init(p_full_b + 8 * i, 4);
      mbar_init(pbuf_free_b + 8 * i, 1);
      mbar_init(x_full_b + 8 * i, 1);
      mbar_init(x_free_b + 8 * i, 4);
    }
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    mbar_init(red_b, 4);
    mbar_init(red_b + 8, 4);
    mbar_init(l_done, 4);
    mbar_init(red2_b, 4);
    mbar_init(fin_s, 1);
    vote[0] = -1;
    vote[1] = -1;
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(smem_u32(tmem_slot), SM::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before any remote arrive or st.async
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tm_s = tmem, tm_o = tmem + 2 * NH;   // S^T buffers [0,NH) [NH,2NH); O^T group g at 2NH + g NH

  if (warp == 4) {
    // ---------------- TMA producer: per tile the rotary block (when ours), then 2 latent entries ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_cache);
      prefetch_tmap(&tm_lat);
      mbar_arrive_expect_tx(q_full, 5 * QKB);
      for (int j = 0; j < 4; ++j) tma_load_3d(q_s + j * QKB, &tm_qabs, q_full, 256 * (int)r + 64 * j, b * a.H, 0);
      tma_load_3d(q_s + 4 * QKB, &tm_qpe, q_full, 0, b * a.H, 0);
      int e = 0, ro = 0;
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        long long row[2];
        for (int hf = 0; hf < 2; ++hf) {
          const int j0 = r0 + 128 * t + 64 * hf;
          row[hf] = -64;
          if (j0 < r1) {
            const int blk = a.block_table[(long long)b * a.mbps + j0 / a.bs];
            if (blk >= 0 && blk < a.n_blocks) row[hf] = (long long)blk * a.bs + (j0 % a.bs);
            else if (r == 0) set_flag(a.flag, MLA_FLAG_BAD_BLOCK);
          }
        }
        if ((t & 1) == (int)r) {
          if (!mbar_wait(rempty, (ro & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
          mbar_arrive_expect_tx(rfull, 16384);
          for (int hf = 0; hf < 2; ++hf) tma_load_3d(rope_s + hf * 8192, &tm_cache, rfull, a.rope_col0, (int)row[hf], 0);
          ++ro;
        }
        for (int g = 0; g < 2; ++g, ++e) {
          const int slot = e % NPR;
          if (!mbar_wait(empty_b + 8 * slot, ((e / NPR) & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
          const uint32_t dst = ring_s + slot * 32768, fb = full_b + 8 * slot;
          mbar_arrive_expect_tx(fb, 32768);
          // one box per cache block: both 64-column k-blocks of 64 rows
          for (int hf = 0; hf < 2; ++hf)
            tma_load_4d(dst + hf * 16384, &tm_lat, fb, 0, 0, a.lat_col0 / 64 + 4 * (int)r + 2 * g, (int)(row[hf] / 8));
        }
      }
      // let the loads still in flight land before the CTA can exit
      {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(q_full, 0)) if (global_timer_ns() - t0 > WAIT_LIMIT_NS) break;
      }
      if (ro > 0) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(rfull, (ro - 1) & 1))
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
      for (int u = (e > NPR ? e - NPR : 0); u < e; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(full_b + 8 * (u % NPR), (u / NPR) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 5 || warp == 6) {
    // ---------------- MMA issuers: warp 5 S^T, warp 6 P.V (each commits its own) ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, NH);
      constexpr uint32_t idesc_o = idesc_bf16(128, NH, 0, 1);
      bool ok = mbar_wait(q_full, 0, abort_word, a.flag);
      tc_fence_after();
      // descriptors built once; a k-step or another buffer only adds its byte
      // offset >> 4 to the start-address field (every address stays below 256 KB)
      const uint64_t d_ring = sdesc_sw128_sbo(ring_s, 2048);          // S: tile k-block, K-major
      const uint64_t d_v = sdesc_sw128_mn_sbo(ring_s, 1024, 2048);    // P.V: V^T, MN-major
      const uint64_t d_q = sdesc_sw128(q_s), d_rope = sdesc_sw128(rope_s), d_p = sdesc_sw128(p_s);
      if (warp == 5) {
        int es = 0, ros = 0;
        for (int t = 0; t < T && ok; ++t) {
          const int sb = t & 1;
          const bool rope = (t & 1) == (int)r;
          const int s0 = es % NPR, s1 = (es + 1) % NPR;
          ok = mbar_wait(s_free_b + 8 * sb, ((t >> 1) & 1) ^ 1, abort_word, a.flag) &&
               mbar_wait(full_b + 8 * s0, (es / NPR) & 1, abort_word, a.flag) &&
               mbar_wait(full_b + 8 * s1, ((es + 1) / NPR) & 1, abort_word, a.flag) &&
               (!rope || mbar_wait(rfull, ros & 1, abort_word, a.flag));
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tm_s + NH * sb;
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const uint64_t da = d_ring + (uint64_t)((g ? s1 : s0) * (32768 >> 4));
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_bf16(d, da + (kk * 1024 + 32 * k) / 16, d_q + ((2 * g + kk) * QKB + 32 * k) / 16, idesc_s,
                         (g > 0 || kk > 0 || k > 0) ? 1u : 0u);
          }
          if (rope) {
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_bf16(d, d_rope + 2 * k, d_q + (4 * QKB + 32 * k) / 16, idesc_s, 1u);
            mma_commit(rempty);
            ++ros;
          }
          mma_commit(s_full_b + 8 * sb);
          es += 2;
        }
        mma_commit(fin_s);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(fin_s, 0))
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      } else {
        int eo = 0;
        for (int u = 0; u < T && ok; ++u) {
          const int sb = u & 1;
          if (!(ok = mbar_wait(p_full_b + 8 * sb, (u >> 1) & 1, abort_word, a.flag))) break;
          tc_fence_after();
          const uint64_t dp = d_p + (uint64_t)(sb * (2 * QKB / 16));
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int slot = (eo + g) % NPR;
            const uint64_t dv = d_v + (uint64_t)(slot * (32768 >> 4));
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_bf16(tm_o + NH * g, dv + 4096 * k / 16, dp + ((k >> 2) * QKB + 32 * (k & 3)) / 16, idesc_o,
                       (u > 0 || k > 0) ? 1u : 0u);
            mma_commit(empty_b + 8 * slot);
          }
          mma_commit(o_done);
          mma_commit(pbuf_free_b + 8 * sb);
          eo += 2;
        }
        mma_commit(fin);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(fin, 0))
          if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else {
    // ---------------- softmax: thread i <-> tile row i <-> TMEM lane i ----------------
    const int i = threadIdx.x;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t peer_x = mapa_shared(x_s, peer), peer_x_full = mapa_shared(x_full_b, peer);
    const uint32_t peer_x_free = mapa_shared(x_free_b, peer);
    const int xsw = (i >> XSH) & (CPR - 1);
    float m_ref[NH], l_part[NH], cur[NH], nxt[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; }
    // Our partial S_r^T(u) out of TMEM into nxt, and row i of it into the peer's X[u & 1].
    auto fetch_send = [&](int u) -> bool {
      const int sb = u & 1;
      if (!mbar_wait_warp(s_full_b + 8 * sb, (u >> 1) & 1, abort_word, a.flag)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < NH / 16; ++c) tmem_ld16(tm_s + NH * sb + lane_base + 16 * c, (uint32_t*)&nxt[16 * c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free_b + 8 * sb);
      // the peer has read what we sent for tile u - 2 out of this buffer
      if (!mbar_wait_cluster_warp(x_free_b + 8 * sb, ((u >> 1) & 1) ^ 1, abort_word, a.flag)) return false;
      // the partial crosses in f16 (half the bytes; partial scores stay far inside its range)
      const uint32_t dst = peer_x + sb * SM::XB + i * (NH * 2);
#pragma unroll
      for (int c = 0; c < CPR; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __half2 hv = __floats2half2_rn(nxt[8 * c + 2 * j], nxt[8 * c + 2 * j + 1]);
          w[j] = *reinterpret_cast<uint32_t*>(&hv);
        }
        st_async_v4_b32(dst + 16 * (c ^ xsw), w[0], w[1], w[2], w[3], peer_x_full + 8 * sb);
      }
      return true;
    };
    // block id of this thread's row in tile t, loaded one tile ahead
    auto row_block = [&](int t) -> int {
      const int j0 = r0 + 128 * t + 64 * (i >> 6);
      return j0 < r1 ? a.block_table[(long long)b * a.mbps + j0 / a.bs] : 0;
    };
    int blk_next = row_block(0);
    bool ok = fetch_send(0);
#pragma unroll
    for (int h = 0; h < NH; ++h) cur[h] = nxt[h];
    int sent = 1;     // tiles whose partial this warp has sent
    int n_slow = 0;   // tiles that needed the column maxima (phases of red2_b)
    for (int t = 0; t < T && ok; ++t) {
      const int sb = t & 1;
      // send the next tile's partial now if its S^T is already there (warp-uniform test)
      if (t + 1 < T && sent == t + 1) {
        const int ready = __shfl_sync(0xffffffffu, lane == 0 ? (int)mbar_test(s_full_b + 8 * ((t + 1) & 1),
                                                                             ((t + 1) >> 1) & 1)
                                                            : 0, 0);
        if (ready) {
          if (!fetch_send(t + 1)) { ok = false; break; }
          sent = t + 2;
        }
      }
      const int valid_rows = min(128, r1 - (r0 + 128 * t));
      const bool valid = (i < valid_rows) && blk_next >= 0 && blk_next < a.n_blocks;
      if (t + 1 < T) blk_next = row_block(t + 1);
      // S^T = ours + the peer's partial
      if (i == 0) mbar_arrive_expect_tx(x_full_b + 8 * sb, SM::XB);
      if (!mbar_wait_warp(x_full_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      {
        const uint4* xr = (const uint4*)(smem + SM::X_OFF + sb * SM::XB + i * (NH * 2));
#pragma unroll
        for (int c = 0; c < CPR; ++c) {
          const uint4 x = xr[c ^ xsw];
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
            cur[8 * c + 2 * j] += f.x;
            cur[8 * c + 2 * j + 1] += f.y;
          }
        }
      }
      // the warp's reads of X have returned (their sums are in registers), so a
      // relaxed arrive suffices; a release at cluster scope would stall the warp
      // until all its earlier memory traffic is visible cluster-wide
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(peer_x_free + 8 * sb);
      // A head's reference max moves only when the tile's column max exceeds it
      // by more than 2^8, i.e. when some row does. So the rows vote first and
      // the column maxima are reduced only on the (rare) tiles that need them.
      bool need = false;
#pragma unroll
      for (int h = 0; h < NH; ++h) need |= valid && (cur[h] * a.scale_log2 > m_ref[h] + 8.f);
      if (__any_sync(0xffffffffu, need) && lane == 0) vote[sb] = t;
      // rendezvous of the four softmax warps on an mbarrier (a bounded wait, unlike bar.sync)
      __syncwarp();
      if (lane == 0) mbar_arrive(red_b + 8 * sb);
      if (!mbar_wait_warp(red_b + 8 * sb, (t >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      float alpha[NH];
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < NH; ++h) alpha[h] = 1.f;
      if (vote[sb] == t) {   // the same on every thread
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float v = warp_max_f32(valid ? cur[h] : -INFINITY);
          if (lane == 0) red[warp * NH + h] = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(red2_b);
        if (!mbar_wait_warp(red2_b, n_slow & 1, abort_word, a.flag)) { ok = false; break; }
        ++n_slow;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float mt =
              fmaxf(fmaxf(red[h], red[NH + h]), fmaxf(red[2 * NH + h], red[3 * NH + h])) * a.scale_log2;
          if (mt > m_ref[h] + 8.f) {
            if (m_ref[h] != -INFINITY) { alpha[h] = ex2_approx(m_ref[h] - mt); rescale = true; }
            m_ref[h] = mt;
          }
        }
      }
      // P^T(t) into buffer sb once P.V of tile t-2 has released it
      if (!mbar_wait_warp(pbuf_free_b + 8 * sb, ((t >> 1) & 1) ^ 1, abort_word, a.flag)) { ok = false; break; }
      uint8_t* pbuf = smem + SM::P_OFF + sb * 2 * QKB + (i >> 6) * QKB;
      const int col = i & 63;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float p = (valid && m_ref[h] != -INFINITY) ? ex2_approx(fmaf(cur[h], a.scale_log2, -m_ref[h])) : 0.f;
        const bf16 pb = __float2bfloat16_rn(p);
        l_part[h] = l_part[h] * alpha[h] + __bfloat162float(pb);
        *reinterpret_cast<bf16*>(pbuf + h * 128 + ((((col >> 3) ^ (h & 7))) << 4) + (col & 7) * 2) = pb;
      }
      if (rescale && t >= 1) {   // identical on every thread: m_ref is shared
        // P.V(t-2) is complete (its P^T buffer was released), so this waits for P.V(t-1)
        if (!mbar_wait_warp(o_done, (t - 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < 2; ++g)
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
      if (!valid) {
        // rows past the context may hold anything (even NaN); P is 0 there, but
        // 0 * NaN is not, so clear row i of the tile's two latent entries
        for (int g = 0; g < 2; ++g) {
          uint8_t* rowp = smem + SM::RING_OFF + ((2 * t + g) % NPR) * 32768 + (i >> 3) * 2048 + (i & 7) * 128;
          for (int kk = 0; kk < 2; ++kk)
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(rowp + kk * 1024 + 16 * c) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full_b + 8 * sb);
      if (t + 1 < T && sent == t + 1) {
        if (!fetch_send(t + 1)) { ok = false; break; }
        sent = t + 2;
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) cur[h] = nxt[h];
    }
    // every MMA (the last P.V included) has completed once `fin` does
    if (ok && mbar_wait_warp(fin, 0, abort_word, a.flag)) {
      tc_fence_after();
      // l per head = sum of the 128 rows' partial sums
      float* rl = red + 4 * NH;   // [4][NH]
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float v = warp_sum(l_part[h]);
        if (lane == 0) rl[warp * NH + h] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(l_done);
      for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int c = 0; c < NH / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tm_o + NH * g + lane_base + 16 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int h = 16 * c + k;
            if (h < a.H) a.part_o[(unit * a.H + h) * 512 + 256 * r + 128 * g + i] = __uint_as_float(o[k]);
          }
        }
      if (i == 0 && mbar_wait(l_done, 0, abort_word, a.flag)) {
#pragma unroll
        for (int h = 0; h < NH; ++h)
          if (h < a.H) {
            ml[(unit * a.H + h) * 2] = m_ref[h] * 0.69314718055994531f;
            ml[(unit * a.H + h) * 2 + 1] = rl[h] + rl[NH + h] + rl[2 * NH + h] + rl[3 * NH + h];
          }
      }
    } else if (i < a.H) {
      ml[(unit * a.H + i) * 2] = -INFINITY;
      ml[(unit * a.H + i) * 2 + 1] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, SM::TMEM_COLS);
  }
  cluster_sync_all();   // no CTA leaves while its peer may still touch its shared memory
}

}  // namespace tc
}  // namespace mla
