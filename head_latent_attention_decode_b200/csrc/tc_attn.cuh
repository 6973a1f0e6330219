// Absorbed split-KV decode attention on tcgen05 for kv_lora_rank 512 and
// qk_rope 64 (the DeepSeek MLA latent), bf16 cache with blocks of a multiple
// of 64 rows.
//
// Persistent and balanced: the batch's 64-row cache tiles, sequence after
// sequence, form one list, and 2-CTA cluster c takes the c-th equal slice of
// it (so every SM pair streams the same number of tiles whatever the context
// lengths). The part of a sequence inside one slice is a segment; each
// segment leaves one split partial (unnormalised O, reference max, sum), and
// attn_combine_kernel merges a sequence's segments.
//
// Per tile: all heads of the token form the MMA's M = 128 rows (fewer heads
// are padded with zeros). CTA r owns latent columns [256 r, 256 r + 256) of
// every tile and the 64 rotary columns of the tiles with odd-even index r:
//   S_r = [q_abs | q_pe]_r . tile_r^T      (tcgen05, M 128 x N 64, K 256 or 320;
//                                          the latent part of Q lives in TMEM,
//                                          q_pe in shared memory; two S buffers)
//   S   = S_r + S_peer                     (the partials swap through DSMEM in
//                                          f16, into two alternating buffers)
//   online softmax, two threads per head (each half of the tile's 64 columns;
//   the halves' maxima meet in shared memory), with a lazily moved reference
//   max: the accumulator is rescaled only when a head's max grows by more than
//   2^8; P (bf16) is written over the peer partial it was computed from, in
//   the MMA's operand layout
//   O_r += P . V_r                         (tcgen05, A = P from shared memory,
//                                          M 128 x N 256, K 64; V = the same
//                                          shared-memory tile read MN-major)
// Every cache byte is read from HBM once and O (128 x 512 fp32) is split over
// the two CTAs' TMEM. A tile's latent stage is held from its load until its
// P.V, its rotary block (every other tile) only until its S, so the latent
// blocks have a 4-deep ring and the rotary blocks 3 slots of their own. S
// alternates between two TMEM buffers, so S(i + 1) runs, and its partial
// crosses to the peer, while the softmax still works on S(i). Warps 0-7 run
// the softmax (warp w: TMEM lane quarter w % 4, column half w / 4), warp 8
// issues TMA, warp 9 the score MMAs and warp 14 the P.V MMAs (one thread each,
// so a P.V never waits behind the issue of a later S), and warps 10-13 send
// each tile's partial scores to the peer as soon as S lands.
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
  // balanced schedule (head-major kernel): `units` clusters, each a slice of at
  // least `min_per` tiles (which keeps every sequence within `splits` segments);
  // nseg[b] receives the number of segments (split partials) of sequence b
  const bf16* q_pe;   // [n, H, 64]
  int units, min_per;
  int* nseg;
};

constexpr int ATT_NST = 4;                      // latent ring depth
constexpr int ATT_NRP = 3;                      // rotary slots (the tiles of this CTA's parity)
constexpr int ATT_THREADS = 480;                // 8 softmax, 1 TMA, 1 S-MMA, 4 sender, 1 P.V-MMA warps
constexpr int ATT_MAX_SEQ = 256;                // sequences per call (the prefix table in shared memory)
struct AttnSmem {
  static constexpr int STAGE = 4 * 8192;        // the 4 latent k-blocks of [64 rows x 64 cols] bf16
  static constexpr int TILE_OFF = 0;
  static constexpr int ROPE_OFF = ATT_NST * STAGE;          // ATT_NRP x [64 x 64] bf16 rotary blocks
  static constexpr int QPE_OFF = ROPE_OFF + ATT_NRP * 8192;   // [128 x 64] bf16 q_pe (MMA operand layout)
  static constexpr int X_OFF = QPE_OFF + 16384;   // 2 x [128 x 64] f16 peer partial S, then P (bf16) over it
  static constexpr int STG_OFF = X_OFF + 32768;   // [128 x 64] f16, our partial on its way out
  static constexpr int RED_OFF = STG_OFF + 16384; // [2 tiles][2 halves][128] fp32 half-row maxima, then [128] l
  static constexpr int PREF_OFF = RED_OFF + 2 * 2 * 128 * 4 + 128 * 4;   // [ATT_MAX_SEQ + 1] tile prefix sums
  static constexpr int BAR_OFF = PREF_OFF + (ATT_MAX_SEQ + 4) * 4;
  static constexpr int SIZE = 1024 + BAR_OFF + 512;
  static_assert(SIZE <= 227 * 1024, "shared memory per CTA");
};
// TMEM columns: Q latent [0,128) (bf16 pairs), S buffers [128,192) [192,256), O [256,512)
constexpr uint32_t ATT_TM_Q = 0, ATT_TM_S = 128, ATT_TM_O = 256;

// Walks a cluster's slice of the batch's tile list: sequence b, its tile lt.
struct TileWalk {
  const int* pref;   // pref[b] = tiles of sequences 0..b-1 (shared memory)
  int n, b, lt;
  __device__ void start(int g) {
    b = 0;
    while (b < n && pref[b + 1] <= g) ++b;
    lt = g - pref[b];
  }
  __device__ bool seg_last() const { return pref[b] + lt + 1 == pref[b + 1]; }
  __device__ void next() {
    if (seg_last()) {
      ++b;
      while (b < n && pref[b + 1] == pref[b]) ++b;
      lt = 0;
    } else {
      ++lt;
    }
  }
};

// Context length of sequence b as the schedule counts it (0 when invalid).
__device__ __forceinline__ int attn_seq_len(const TcAttnArgs& a, int b) {
  const int L = a.ctx[b];
  return (L < 1 || L > a.max_ctx || L > a.mbps * a.bs) ? 0 : L;
}

// The balanced schedule of a persistent attention kernel: the prefix sum of
// the batch's tiles of `tile_rows` rows, in shared memory (pref[b] = tiles of
// sequences 0..b-1, n + 1 entries, n <= 256), and the slice [g0, g1) of the
// flattened tile list that cluster c takes (slices of `per` tiles, at least
// a.min_per). Block 0 of the grid writes each sequence's segment count to
// a.nseg. Every thread of the CTA calls it; it ends with a __syncthreads.
__device__ __forceinline__ void attn_schedule(const TcAttnArgs& a, int tile_rows, int* pref, int c, uint32_t r,
                                              int warp, int lane, int* per_out, int* g0_out, int* g1_out) {
  if (warp == 0) {
    int cnt[8], sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int b = 8 * lane + k;
      int T = 0;
      if (b < a.n) {
        const int L = attn_seq_len(a, b);
        if (L == 0 && c == 0 && r == 0) set_flag(a.flag, MLA_FLAG_BAD_CONTEXT);
        T = (L + tile_rows - 1) / tile_rows;
      }
      cnt[k] = T;
      sum += T;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int b = 8 * lane + k;
      if (b < a.n) pref[b] = run;
      run += cnt[k];
    }
    if (lane == 31) pref[a.n] = incl;   // the batch's tile count
  }
  __syncthreads();
  const int total = pref[a.n];
  int per = (total + a.units - 1) / a.units;
  if (per < a.min_per) per = a.min_per;
  if (blockIdx.x == 0) {   // segments of each sequence, for the merge
    for (int b = threadIdx.x; b < a.n; b += blockDim.x) {
      const int T = pref[b + 1] - pref[b];
      a.nseg[b] = T > 0 ? (pref[b] + T - 1) / per - pref[b] / per + 1 : 0;
    }
  }
  *per_out = per;
  *g0_out = c * per;
  *g1_out = min(total, c * per + per);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(ATT_THREADS, 1)
    tc_attn_decode_kernel(const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_lat,
                          TcAttnArgs a) {
  using SM = AttnSmem;
  griddep_wait();   // the inputs all come from the stream's earlier kernels
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tile_s = sbase + SM::TILE_OFF, x_s = sbase + SM::X_OFF;
  float* red = (float*)(smem + SM::RED_OFF);      // [tile & 1][half][head]
  float* red_l = red + 2 * 2 * 128;                // [head]: the second half's row sum
  int* pref = (int*)(smem + SM::PREF_OFF);
  const uint32_t bar = sbase + SM::BAR_OFF;
  // barriers (8 B each)
  const uint32_t full_b = bar;                        // [ATT_NST] tile landed
  const uint32_t empty_b = bar + 8 * ATT_NST;         // [ATT_NST] tile consumed by P.V
  const uint32_t s_full = bar + 16 * ATT_NST;         // [2] S_r(i) complete, in buffer i & 1
  const uint32_t s_free = s_full + 16;                // [2] S read by the 8 softmax and 4 sender warps
  const uint32_t p_full_b = s_free + 16;              // [2] P(i) in shared memory (8 softmax warps)
  const uint32_t x_full_b = p_full_b + 16;            // [2 buffers][4 lane quarters] peer partial rows landed
  const uint32_t x_free_b = x_full_b + 64;            // [2] the peer's P.V has released its buffer
  const uint32_t q_ready = x_free_b + 16;             // Q of the next segment in TMEM (8 softmax warps)
  const uint32_t o_done = q_ready + 8;                // each P.V
  const uint32_t o_seg = o_done + 8;                  // the last P.V of a segment
  const uint32_t o_free = o_seg + 8;                  // O of a segment read out (8 softmax warps)
  const uint32_t fin = o_free + 8;
  const uint32_t xch_b = fin + 8;                     // [4 quarters][2] the two halves' maxima posted
  const uint32_t l_done = xch_b + 64;                 // [4] the second half's row sums posted
  const uint32_t rope_empty = l_done + 32;            // [ATT_NRP] rotary block consumed by S
  uint32_t* tmem_slot = (uint32_t*)(smem + SM::BAR_OFF + 448);
  volatile int* abort_word = (volatile int*)(smem + SM::BAR_OFF + 452);

  const uint32_t r = cluster_ctarank(), peer = r ^ 1u;
  const int c = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- the schedule: tile prefix over the batch, then this cluster's slice ----
  int per, g0, g1;
  attn_schedule(a, 64, pref, c, r, warp, lane, &per, &g0, &g1);
  if (g0 >= g1) return;   // both CTAs of the cluster take this branch together
  const int N = g1 - g0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ATT_NST; ++i) { mbar_init(full_b + 8 * i, 1); mbar_init(empty_b + 8 * i, 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(s_full + 8 * i, 1); mbar_init(s_free + 8 * i, 12); }
    for (int i = 0; i < ATT_NRP; ++i) mbar_init(rope_empty + 8 * i, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(p_full_b + 8 * i, 8);
      for (int k = 0; k < 4; ++k) mbar_init(x_full_b + 8 * (4 * i + k), 1);
      mbar_init(x_free_b + 8 * i, 1);
    }
    mbar_init(q_ready, 8);
    mbar_init(o_done, 1);
    mbar_init(o_seg, 1);
    mbar_init(o_free, 8);
    mbar_init(fin, 2);   // both issuing threads' last commits
    for (int i = 0; i < 8; ++i) mbar_init(xch_b + 8 * i, 2);
    for (int i = 0; i < 4; ++i) mbar_init(l_done + 8 * i, 1);
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

  if (warp == 8) {
    // ---------------- TMA producer (lane 0 issues; lane k holds the block id of tile i + k) ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_cache);
      prefetch_tmap(&tm_lat);
    }
    TileWalk w{pref, a.n, 0, 0};
    w.start(g0);
    int i = 0, blkv = 0;
    for (; i < N; ++i, w.next()) {
      if ((i & 31) == 0) {   // the block ids of the next 32 tiles, loaded in parallel
        TileWalk wk = w;
        for (int k = 0; k < lane && i + k + 1 < N; ++k) wk.next();
        blkv = (i + lane < N) ? a.block_table[(long long)wk.b * a.mbps + (64 * wk.lt) / a.bs] : 0;
      }
      const int blk = __shfl_sync(0xffffffffu, blkv, i & 31);
      const int st = i % ATT_NST;
      const bool rope = (i & 1) == (int)r;
      const int ri = (i >> 1) % ATT_NRP;
      if (!mbar_wait_warp(empty_b + 8 * st, ((i / ATT_NST) & 1) ^ 1, abort_word, a.flag)) break;
      if (rope && !mbar_wait_warp(rope_empty + 8 * ri, (((i >> 1) / ATT_NRP) & 1) ^ 1, abort_word, a.flag)) break;
      if (lane == 0) {
        const int j0 = 64 * w.lt;
        long long row = -64;
        if (blk >= 0 && blk < a.n_blocks) row = (long long)blk * a.bs + (j0 % a.bs);
        else if (r == 0) set_flag(a.flag, MLA_FLAG_BAD_BLOCK);
        mbar_arrive_expect_tx(full_b + 8 * st, rope ? 5 * 8192 : 4 * 8192);
        const uint32_t dst = tile_s + st * SM::STAGE;
        // the 4 latent k-blocks of the 64 rows in one box: [8 row octets][4 k-blocks][8 rows][128 B]
        tma_load_4d(dst, &tm_lat, full_b + 8 * st, 0, 0, a.lat_col0 / 64 + 4 * (int)r, (int)(row / 8));
        if (rope) tma_load_3d(sbase + SM::ROPE_OFF + ri * 8192, &tm_cache, full_b + 8 * st, a.rope_col0, (int)row, 0);
      }
    }
    // drain the loads still in flight
    if (lane == 0) {
      for (int u = (i > ATT_NST ? i - ATT_NST : 0); u < i; ++u) {
        const uint64_t t1 = global_timer_ns();
        while (!mbar_try_wait(full_b + 8 * (u % ATT_NST), (u / ATT_NST) & 1))
          if (global_timer_ns() - t1 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
      }
    }
  } else if (warp == 9) {
    // ---------------- S issuer: S(t) into buffer t & 1 once its tile has landed ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64);
      // descriptors built once; stages and k-steps add their byte offset >> 4
      const uint64_t d_t = sdesc_sw128_sbo(tile_s, 4096), d_rope = sdesc_sw128(sbase + SM::ROPE_OFF);
      const uint64_t d_qpe = sdesc_sw128(sbase + SM::QPE_OFF);
      TileWalk ws{pref, a.n, 0, 0};
      ws.start(g0);
      int ks = 0;
      for (int t = 0; t < N; ++t, ws.next()) {
        const int st = t % ATT_NST;
        const bool first = (t == 0 || ws.lt == 0), last = (t == N - 1 || ws.seg_last());
        if (!mbar_wait(full_b + 8 * st, (t / ATT_NST) & 1, abort_word, a.flag) ||
            !mbar_wait(s_free + 8 * (t & 1), ((t >> 1) & 1) ^ 1, abort_word, a.flag) ||
            (first && !mbar_wait(q_ready, ks & 1, abort_word, a.flag)))
          break;
        tc_fence_after();
        const uint64_t dt = d_t + (uint64_t)(st * (SM::STAGE / 16));
        const uint32_t d = tmem + ATT_TM_S + 64 * (t & 1);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ts(d, tmem + ATT_TM_Q + 32 * j + 8 * k, dt + (j * 1024 + 32 * k) / 16, idesc_s,
                        (j > 0 || k > 0) ? 1u : 0u);
        if ((t & 1) == (int)r) {
          const int ri = (t >> 1) % ATT_NRP;
          const uint64_t dr = d_rope + (uint64_t)(ri * (8192 / 16));
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_bf16(d, d_qpe + 2 * k, dr + 2 * k, idesc_s, 1u);
          mma_commit(rope_empty + 8 * ri);
        }
        mma_commit(s_full + 8 * (t & 1));
        if (last) ++ks;
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else if (warp == 14) {
    // ---------------- P.V issuer: O += P(u) . V(u) as soon as P(u) is written ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16(128, 256, 1);
      const uint64_t d_v = sdesc_sw128_mn_sbo(tile_s, 1024, 4096), d_p = sdesc_sw128(x_s);
      TileWalk wo{pref, a.n, 0, 0};
      wo.start(g0);
      int ko = 0;
      for (int u = 0; u < N; ++u, wo.next()) {
        const int st = u % ATT_NST, xb = u & 1;
        const bool first = (u == 0 || wo.lt == 0), last = (u == N - 1 || wo.seg_last());
        if (!mbar_wait(p_full_b + 8 * xb, (u >> 1) & 1, abort_word, a.flag) ||
            (first && ko > 0 && !mbar_wait(o_free, (ko - 1) & 1, abort_word, a.flag)))
          break;
        tc_fence_after();
        const uint64_t dv = d_v + (uint64_t)(st * (SM::STAGE / 16));
        const uint64_t dp = d_p + (uint64_t)(xb * (16384 / 16));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16(tmem + ATT_TM_O, dp + 2 * k, dv + 8192 * k / 16, idesc_o, (!first || k > 0) ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(empty_b + 8 * st);
        mma_commit_cta_mask(x_free_b + 8 * xb, (uint16_t)(1u << peer));   // our buffer xb is the peer's to fill
        if (last) { mma_commit(o_seg); ++ko; }
      }
      mma_commit(fin);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(fin, 0))
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) { set_flag(a.flag, MLA_FLAG_WAIT_TIMEOUT); break; }
    }
  } else if (warp >= 10) {   // warps 10-13
    // ---------------- senders: S_r(i) -> staging -> per warp, one bulk copy of its 32 rows into the
    // peer's X, landing on that quarter's barrier (the peer's softmax warps of the quarter wait for it alone)
    const int qs = warp & 3;                              // TMEM lane quarter of this warp
    const int h = 32 * qs + lane;
    const uint32_t lane_base = (uint32_t)(qs * 32) << 16;
    const uint32_t peer_x = mapa_shared(x_s, peer), peer_x_full = mapa_shared(x_full_b, peer);
    const uint32_t stg_s = sbase + SM::STG_OFF + 4096 * qs;   // this warp's rows, 4 KB
    uint4* stg_row = (uint4*)(smem + SM::STG_OFF + h * 128);
    for (int i = 0; i < N; ++i) {
      if (!mbar_wait_warp(s_full + 8 * (i & 1), (i >> 1) & 1, abort_word, a.flag)) break;
      tc_fence_after();
      float v[64];
      const uint32_t sa = tmem + ATT_TM_S + 64 * (i & 1) + lane_base;
#pragma unroll
      for (int k = 0; k < 4; ++k) tmem_ld16(sa + 16 * k, (uint32_t*)&v[16 * k]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + 8 * (i & 1));
      if (lane == 0) bulk_wait_read_all();               // this warp's previous copy has left its rows
      __syncwarp();
      // the partial goes out in f16 (half the distributed-shared-memory bytes of fp32; the
      // partial scores stay far inside f16's range and its 11-bit significand costs the
      // scores ~1e-3 relative, well inside the output tolerance)
#pragma unroll
      for (int k = 0; k < 8; ++k) {  // chunk k (8 values) of row h at slot k ^ (h & 7): no bank conflicts
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __half2 hv = __floats2half2_rn(v[8 * k + 2 * j], v[8 * k + 2 * j + 1]);
          w[j] = *reinterpret_cast<uint32_t*>(&hv);
        }
        stg_row[k ^ (h & 7)] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // the peer's P.V(i - 2) has released the buffer we send into
        const int xb = i & 1;
        if (mbar_wait_cluster(x_free_b + 8 * xb, ((i >> 1) & 1) ^ 1, abort_word, a.flag)) {
          bulk_copy_to_peer(peer_x + xb * 16384 + 4096 * qs, stg_s, 4096, peer_x_full + 8 * (4 * xb + qs));
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_read_all();
  } else {
    // ---------------- softmax: head h <-> TMEM lane h, columns [32 g, 32 g + 32) of each tile ----------------
    const int q = warp & 3, g = warp >> 2;
    const int h = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    // this half's share of sequence b's query: 128 latent values of CTA r's half
    // -> TMEM columns [64 g, 64 g + 64), 32 rotary values -> [128 + 16 g, 128 + 16 g + 16)
    auto load_q = [&](int b) {
      const bool live = h < a.H;
      const long long qh = (long long)b * a.H + (live ? h : 0);
      const uint4* src = (const uint4*)(a.q_abs + qh * 512 + r * 256 + 128 * g);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        uint32_t qv[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 v = live ? src[4 * k4 + k] : make_uint4(0, 0, 0, 0);
          qv[4 * k] = v.x; qv[4 * k + 1] = v.y; qv[4 * k + 2] = v.z; qv[4 * k + 3] = v.w;
        }
        tmem_st16(tmem + ATT_TM_Q + lane_base + 64 * g + 16 * k4, qv);
      }
      // q_pe row h, chunks 4 g .. 4 g + 3, in the 128-byte-swizzled K-major operand layout
      const uint4* pe = (const uint4*)(a.q_pe + qh * 64 + 32 * g);
      uint4* qrow = (uint4*)(smem + SM::QPE_OFF + h * 128);
#pragma unroll
      for (int k = 0; k < 4; ++k) qrow[(4 * g + k) ^ (h & 7)] = live ? pe[k] : make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    };
    TileWalk w{pref, a.n, 0, 0};
    w.start(g0);
    load_q(w.b);
    // block of tile i + 1, loaded one tile ahead (only its validity is needed here)
    auto tile_block = [&](const TileWalk& t) { return a.block_table[(long long)t.b * a.mbps + (64 * t.lt) / a.bs]; };
    int blk_next = tile_block(w);
    int seq_len = attn_seq_len(a, w.b);
    float m_ref = -INFINITY, l = 0.f;
    int tseg = 0, kseg = 0;   // tile within the segment, segments done
    bool ok = true;
    for (int i = 0; i < N && ok; ++i, w.next()) {
      const int b = w.b, lt = w.lt, st = i % ATT_NST, xb = i & 1;
      const bool last = (i == N - 1 || w.seg_last());
      const int blk = blk_next;
      if (i + 1 < N) {
        TileWalk wn = w;
        wn.next();
        blk_next = tile_block(wn);
      }
      const int valid = (blk >= 0 && blk < a.n_blocks) ? min(64, seq_len - 64 * lt) : 0;
      if (g == 0 && lane == 0) mbar_arrive_expect_tx(x_full_b + 8 * (4 * xb + q), 4096);   // this quarter's rows
      if (!mbar_wait_warp(s_full + 8 * xb, (i >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      tc_fence_after();
      float v[32];
      const uint32_t sp_addr = tmem + ATT_TM_S + 64 * xb + 32 * g + lane_base;
      tmem_ld16(sp_addr, (uint32_t*)&v[0]);
      tmem_ld16(sp_addr + 16, (uint32_t*)&v[16]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + 8 * xb);   // S(i + 2) may overwrite the buffer
      if (!mbar_wait_warp(x_full_b + 8 * (4 * xb + q), (i >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      // row h, chunks 4 g .. 4 g + 3 of the peer's partial; P(i) later goes to exactly these bytes
      uint4* xrow = (uint4*)(smem + SM::X_OFF + xb * 16384 + h * 128);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 x = xrow[(4 * g + k) ^ (h & 7)];
        const uint32_t wx[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wx[j]));
          v[8 * k + 2 * j] += f.x;
          v[8 * k + 2 * j + 1] += f.y;
        }
      }
      if (valid < 64) {
        const int vc = valid - 32 * g;   // valid columns of this half
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (j < vc) ? v[j] : -INFINITY;   // also drops NaN past the context
      }
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], v[j]);
      const float mloc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      // the two halves of head h meet: both then take the same decisions
      red[(xb * 2 + g) * 128 + h] = mloc;
      __syncwarp();
      if (lane == 0) mbar_arrive(xch_b + 8 * (2 * q + xb));
      if (!mbar_wait_warp(xch_b + 8 * (2 * q + xb), (i >> 1) & 1, abort_word, a.flag)) { ok = false; break; }
      const float mt = fmaxf(mloc, red[(xb * 2 + (g ^ 1)) * 128 + h]) * a.scale_log2;
      // online softmax in log2 units with a lazily moved reference max
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_ref + 8.f) {
        if (m_ref != -INFINITY) { alpha = ex2_approx(m_ref - mt); rescale = true; }
        m_ref = mt;
      }
      const float nm = (m_ref == -INFINITY) ? 0.f : -m_ref;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float e0 = ex2_approx(fmaf(v[j], a.scale_log2, nm)), e1 = ex2_approx(fmaf(v[j + 1], a.scale_log2, nm));
        __nv_bfloat162 pb = __floats2bfloat162_rn(e0, e1);
        ps[(j >> 1) & 3] += e0 + e1;
        pk[j >> 1] = *reinterpret_cast<uint32_t*>(&pb);
      }
      const float psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
      if (__any_sync(0xffffffffu, rescale) && tseg >= 1) {
        // P.V(i - 2) is complete (its release let the peer fill this X buffer), so
        // waiting for the phase of P.V(i - 1) cannot pass early; O must not be
        // touched before it completes
        if (!mbar_wait_warp(o_done, (i - 1) & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
        for (int k = 0; k < 8; ++k) {
          uint32_t o[16];
          const uint32_t oa = tmem + ATT_TM_O + lane_base + 128 * g + 16 * k;
          tmem_ld16(oa, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st16(oa, o);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      l = l * alpha + psum;
      if (valid < 64) {
        // rows past the context may hold anything (even NaN); P is 0 there, but
        // 0 * NaN is not, so clear them in the four latent slots before P.V
        // (latent rows are laid out [8 row octets][4 k-blocks][8 rows][128 B])
        const int ti = g * 128 + h, row = valid + (ti >> 2);
        if (row < 64) {
          uint8_t* rp = smem + SM::TILE_OFF + st * SM::STAGE + (row >> 3) * 4096 + (ti & 3) * 1024 + (row & 7) * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(rp + 16 * k) = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        xrow[(4 * g + k) ^ (h & 7)] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full_b + 8 * xb);
      ++tseg;
      if (last) {
        // the segment's S MMAs are all complete (the softmax read each S): the next
        // segment's query may replace this one while the last P.V runs
        if (i + 1 < N) {
          TileWalk wn = w;
          wn.next();
          load_q(wn.b);
          seq_len = attn_seq_len(a, wn.b);
        }
        const int j = c - pref[b] / per;               // this segment's split slot in sequence b
        const long long unit = (long long)b * a.splits + j;
        float* const ml = a.part_ml + r * a.ml_r;      // this CTA's (m, l) copy
        if (!mbar_wait_warp(o_seg, kseg & 1, abort_word, a.flag)) { ok = false; break; }
        tc_fence_after();
        float* po = a.part_o + (unit * a.H + h) * 512 + r * 256 + 128 * g;
        for (int k = 0; k < 8; ++k) {
          uint32_t o[16];
          tmem_ld16(tmem + ATT_TM_O + lane_base + 128 * g + 16 * k, o);
          tmem_ld_wait();
          if (h < a.H) {
#pragma unroll
            for (int jj = 0; jj < 16; jj += 4)
              *reinterpret_cast<float4*>(po + 16 * k + jj) =
                  make_float4(__uint_as_float(o[jj]), __uint_as_float(o[jj + 1]), __uint_as_float(o[jj + 2]),
                              __uint_as_float(o[jj + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);   // the next segment's first P.V may overwrite O
        // the row sum is the two halves' sums
        if (g == 1) {
          red_l[h] = l;
          __syncwarp();
          if (lane == 0) mbar_arrive(l_done + 8 * q);
        } else if (mbar_wait_warp(l_done + 8 * q, kseg & 1, abort_word, a.flag)) {
          if (h < a.H) {
            ml[(unit * a.H + h) * 2] = m_ref * 0.69314718055994531f;   // natural-log units
            ml[(unit * a.H + h) * 2 + 1] = l + red_l[h];
          }
        } else {
          ok = false;
          break;
        }
        m_ref = -INFINITY;
        l = 0.f;
        tseg = 0;
        ++kseg;
      }
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
