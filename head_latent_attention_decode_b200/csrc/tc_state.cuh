// What the tensor-core (tcgen05) path keeps per layer handle: TMA tensor maps
// of the repacked weights (built once at init) and the device's SM count.
#pragma once

#include <cuda.h>

struct TcState {
  int enabled;       // bf16 activations with bf16 weights on an sm_100 device (all tcgen05 GEMMs)
  int attn;          // bf16 activations on an sm_100 device (tcgen05 attention, any weight dtype)
  int fp8;           // FP8 weights with bf16 activations: tcgen05 decode GEMMs on decoded FP8 tiles
  int pf8;           // FP8 weights, prefill on the bf16 tcgen05 path after a per-call dequantisation
  int num_sms;
  // weights as the A operand (decode, swap-AB): 128-row boxes
  CUtensorMap a_W1, a_Wqb, a_Wuk, a_Wuv, a_Wo, a_Woa, a_Wob;
  // FP8 weight codes as the A operand (decode): 128 x 128-byte boxes
  CUtensorMap a8_W1, a8_Wqb, a8_Wuk, a8_Wuv, a8_Wo;
  // weights as the B operand (prefill): 256-row boxes
  CUtensorMap b_W1q, b_W1kv, b_W1, b_Wqb, b_Wkvb, b_Wo, b_Woa, b_Wob;
  int bn_oa;         // N tile of the grouped output projection's per-group GEMM (prefill)
};
