// Per-(token, head) symmetric INT8 quantisation of one cached K or V row
// ("Performance and Memory", "KV cache INT8" table and the sentence under it:
// per-token, per-head symmetric INT8 with one FP16 scale per (token, head)).
//
//   scale = fp16_rne(max|x| / 127)              (x: the row's fp16 values)
//   code  = clamp(rint(x / float(scale)), -127, 127),  scale == 0 -> code 0
//
// Every step is an IEEE fp32 operation (correctly rounded division, rint ties
// to even), so a code is a pure function of the row.  The standalone
// quantisation hook, the prefill cache append and the decode cache append all
// call these two functions, so the hot path's codes are the hook's codes.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace tl {

// fp16 scale of a row whose largest magnitude is `absmax` (an fp16 value
// widened to fp32).
__device__ __forceinline__ __half kv_int8_scale(float absmax) {
  return __float2half_rn(__fdiv_rn(absmax, 127.0f));
}

// INT8 code of one value `x` (an fp16 value widened to fp32) under the row's
// scale `s` (the fp16 scale widened to fp32).
__device__ __forceinline__ int8_t kv_int8_code(float x, float s) {
  if (s == 0.0f) return 0;
  const float r = fminf(fmaxf(rintf(__fdiv_rn(x, s)), -127.0f), 127.0f);
  return (int8_t)(int)r;
}

}  // namespace tl
