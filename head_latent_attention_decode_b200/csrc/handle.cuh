// Host-side state of one MLA layer: configuration, the repacked weight blob's
// layout, and what the tensor-core path prepares at init.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

#include "../../include/mla.h"
#include "tc_state.cuh"

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
static inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// Launches of this library's kernels (mla_kernel_launch_count).
void mla_count_launch(int k);

// Kernel timer (mla_set_kernel_timer): bracket a launch with event records.
void mla_timer_begin(const char* kernel, cudaStream_t s);
void mla_timer_end(const char* kernel, cudaStream_t s);

// Repacked weight blob.
// Every matrix is stored K-major, [N, K] (the transpose of the pages' [in,
// out] form), so that one output feature's weights are contiguous:
//   W1   [Nq1 + R, D]   rows [0, Nq1) = wq_a^T (or q_proj^T), then wkv_a^T
//   Wqb  [H*(d_n+d_r), r_q]                          (r_q > 0)
//   Wuk  [H][r_kv][d_n]   Wuk[h][c][p] = wkv_b[c][h*(d_n+d_v) + p]
//   Wuv  [H][d_v][r_kv]   Wuv[h][d][c] = wkv_b[c][h*(d_n+d_v) + d_n + d]
//   Wkvb [H*(d_n+d_v), r_kv]                          (prefill)
//   Wo   [D, H*d_v]                                   (dense output projection)
//   Woa  [G][r_o][(H/G)*d_v]  Woa[g][j][i] = wo_a[g*(H/G)*d_v + i][j]   (grouped, o_lora_rank > 0)
//   Wob  [D, G*r_o]
// FP8 blobs add fp32 scales per 128x128 block of each K-major matrix,
// [ceil(N/128)][ceil(K/128)].
struct WeightLayout {
  int Nq1, N1, R, Hq, Hkv;
  size_t esz;
  size_t W1, Wqb, Wuk, Wuv, Wkvb, Wo, Woa, Wob, gq, gkv, sink;
  int G, ro, Kg;   // grouped output projection: groups, low rank, inputs per group (0 = dense wo)
  size_t sW1, sWqb, sWuk, sWuv, sWkvb, sWo;
  size_t total;
};

struct mla_handle {
  mla_config cfg;
  WeightLayout L;
  float scale;
  char* base;
  int has_sink;   // attn_sink given at init: one fp32 logit per head at base + L.sink
  int device;
  TcState tc;
  // mla_decode_step_host: page-locked packing buffer for the step's int32
  // inputs, and an event marking the end of the last transfer out of it
  void* host_pack = nullptr;
  size_t host_pack_bytes = 0;
  cudaEvent_t pack_done = nullptr;
  // ... and the step captured as a CUDA graph (on the library's own stream),
  // replayed while the call's buffers and sizes repeat
  cudaStream_t capture_stream = nullptr;
  cudaGraphExec_t step_exec = nullptr;
  unsigned long long step_key[14] = {0};
  int step_launches = 0;
  ~mla_handle() {
    if (pack_done) { cudaEventSynchronize(pack_done); cudaEventDestroy(pack_done); }
    if (host_pack) cudaFreeHost(host_pack);
    if (step_exec) cudaGraphExecDestroy(step_exec);
    if (capture_stream) cudaStreamDestroy(capture_stream);
  }
};

