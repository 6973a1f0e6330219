// Shared device helpers of the MLA library: element loads/stores for the
// storage types (fp32, bf16, FP8-E4M3 codes), warp reductions, the sticky
// device flag and a launch counter.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// FP8-E4M3 (OCP) decode, written from the format definition: sign bit,
// 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is subnormal
// (m/8 * 2^-6); S.1111.111 is NaN; no infinities. Every code is exact in fp32
// (and in bf16).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  const uint32_t s = (code >> 7) & 1u, e = (code >> 3) & 0xFu, m = code & 7u;
  float v;
  if (e == 0) {
    v = (float)m * 0.001953125f;  // m * 2^-9
  } else if (e == 15 && m == 7) {
    v = __int_as_float(0x7fc00000);
  } else {
    v = __int_as_float((int)(((e + 120u) << 23) | (m << 20)));  // (1 + m/8) 2^(e-7)
  }
  return s ? -v : v;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(uint8_t x) { return e4m3_to_f32(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum (blockDim.x a multiple of 32, <= 1024). `red` >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.f;
  t = warp_sum(t);
  return t;
}

__device__ __forceinline__ void set_flag(int* flag, int bits) {
  if (flag) atomicOr(flag, bits);
}

// Programmatic dependent launch. griddep_wait: block until the grids this one
// depends on have completed and their memory is visible (returns at once
// without such a dependency). griddep_launch_dependents: let the next grid of
// the stream launch once every CTA of this one has called it or exited; call it
// only after this CTA holds its tensor memory, so that an early CTA of the next
// grid can never take tensor memory that a CTA of this grid still waits for.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
}  // namespace mla
