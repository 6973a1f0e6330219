// mla_decode_qkv_noalloc: the decode front-fold with its scratch in a fixed
// device array owned by this library, for callers that cannot allocate.
//
// Who needs it: a caller whose device memory is fully reserved up front by
// its own pool (an inference server that plans every byte at start-up) has
// nothing to give as a workspace, and a caller on a latency-critical serving
// path cannot call cudaMalloc there, because cudaMalloc synchronises the whole
// device and stalls every stream. This entry point lets them run the
// front-fold without a workspace argument.
//
// Cost: every GPU that loads the library holds MLA_NOALLOC_SCRATCH_BYTES of
// device memory until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mla.h"

// Workspace bytes the decode front-fold needs for n tokens, without the
// prefill-only buffers (mla_abi.cu).
size_t mla_decode_workspace_bytes_internal(const mla_handle* h, int n);

// The scratch itself. In host code this name is only a host-side stand-in for
// the device symbol: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch on the current device (set up once per
// device, with that device current). Looking the symbol up loads the module
// that holds the array, which is when its device memory is taken: with CUDA's
// lazy module loading that is the first lookup, not the library's load.
static int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MLA_OK;
}

// Called by mla_init_weights with the handle's device current, so that the
// array is committed when the first handle on a device is created rather than
// at the first allocation-free call (a caller whose pool has reserved the rest
// of the device by then could not take it later). A failure here only defers
// the lookup to that first call.
void mla_noalloc_prepare_device() {
  void* p = nullptr;
  (void)noalloc_scratch(&p);
  cudaGetLastError();
}

extern "C" int mla_decode_qkv_noalloc(mla_handle* h, const void* hidden, int n, const float* cos,
                                      const float* sin, void* kv_cache, int n_blocks,
                                      const int32_t* slot_mapping, void* q_abs, void* q_pe, void* stream) {
  if (!h || n < 0) return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  const size_t need = mla_decode_workspace_bytes_internal(h, n);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > (size_t)MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;   // batch too large for the array
  void* ws = nullptr;
  const int st = noalloc_scratch(&ws);
  if (st != MLA_OK) return st;
  // the array keeps the previous call's contents: the device flag must start at zero
  if (cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  return mla_decode_qkv(h, hidden, n, cos, sin, kv_cache, n_blocks, slot_mapping, q_abs, q_pe, nullptr, ws,
                        (size_t)MLA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int mla_noalloc_read_device_flag(int* flag_out, void* stream) {
  if (!flag_out) return MLA_ERR_INVALID_ARG;
  void* ws = nullptr;
  const int st = noalloc_scratch(&ws);
  if (st != MLA_OK) return st;
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  *flag_out = v;
  return v ? MLA_ERR_DEVICE_FLAG : MLA_OK;
}
