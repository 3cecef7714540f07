// Weight packer (group-wise symmetric INT4 / INT3, and the sign-of-frac bits
// of cross-iteration rounding) and per-(token, head) INT8 KV quantisation.
//
// INT4 follows the low-bit body format of "TinyLoop Framework" ("What Makes It
// Different": INT2/INT4 execution); INT3 follows "Current Status", core
// inference table, INT3 GEMM row (8 levels, 3 bits per weight, 10 values per
// 32-bit word).  INT8 KV follows "Performance and Memory", "KV cache INT8"
// (per-token per-head symmetric INT8, one FP16 scale per (token, head)).
//
// Every integer decision is an IEEE fp32 operation (correctly rounded division
// __fdiv_rn, rintf ties-to-even, __float2half_rn), so the codes are a pure
// function of the inputs.
#include "kv_quant.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int quant_code(float w, float s, float qmin, float qmax) {
  if (s == 0.0f) return 0;
  float r = rintf(__fdiv_rn(w, s));
  r = fminf(fmaxf(r, qmin), qmax);
  return (int)r;
}

// One warp per (row, group): scale = fp16(absmax / qmax).
__global__ void pack_scales_kernel(const float* __restrict__ w, int K, int G, long n_groups,
                                   float qmax, __half* __restrict__ scales) {
  long gw = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (gw >= n_groups) return;
  long groups_per_row = K / G;
  long row = gw / groups_per_row, grp = gw % groups_per_row;
  const float* p = w + row * (long)K + grp * G;
  float m = 0.0f;
  for (int i = lane; i < G; i += 32) m = fmaxf(m, fabsf(p[i]));
  m = warp_max(m);
  if (lane == 0) scales[gw] = __float2half_rn(__fdiv_rn(m, qmax));
}

// One thread per INT4 word: eight codes u = code + 8, lowest k in bits 0..3.
__global__ void pack_int4_words_kernel(const float* __restrict__ w, int K, int G, long n_words,
                                       const __half* __restrict__ scales,
                                       uint32_t* __restrict__ packed) {
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_words) return;
  int wpr = K / 8;
  long row = i / wpr;
  int j = (int)(i % wpr);
  int k0 = 8 * j;
  float s = __half2float(scales[row * (K / G) + k0 / G]);
  const float* p = w + row * (long)K + k0;
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int c = quant_code(p[e], s, -8.0f, 7.0f);
    word |= (uint32_t)(c + 8) << (4 * e);
  }
  packed[i] = word;
}

// One thread per INT3 word: ten codes u = code + 4 at bits 3i, padding u = 4.
__global__ void pack_int3_words_kernel(const float* __restrict__ w, int K, int G, int wpr,
                                       long n_words, const __half* __restrict__ scales,
                                       uint32_t* __restrict__ packed) {
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_words) return;
  long row = i / wpr;
  int j = (int)(i % wpr);
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 10; ++e) {
    int k = 10 * j + e;
    int c = 0;
    if (k < K) {
      float s = __half2float(scales[row * (K / G) + k / G]);
      c = quant_code(w[row * (long)K + k], s, -4.0f, 3.0f);
    }
    word |= (uint32_t)(c + 4) << (3 * e);
  }
  packed[i] = word;
}

// One thread per sign word: bit e of word j of a row is 1 when the fp32
// quotient w / s of element 32 j + e lies above its code (the same quotient
// and code as the packer's), 0 otherwise and past K.
__global__ void pack_sign_bits_kernel(const float* __restrict__ w, int K, int G, int spr,
                                      long n_words, float qmin, float qmax,
                                      const __half* __restrict__ scales,
                                      uint32_t* __restrict__ sign) {
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_words) return;
  long row = i / spr;
  int j = (int)(i % spr);
  uint32_t word = 0;
  for (int e = 0; e < 32; ++e) {
    const int k = 32 * j + e;
    if (k >= K) break;
    const float s = __half2float(scales[row * (K / G) + k / G]);
    if (s == 0.0f) continue;
    const float r = __fdiv_rn(w[row * (long)K + k], s);
    const float c = fminf(fmaxf(rintf(r), qmin), qmax);
    if (r > c) word |= 1u << e;
  }
  sign[i] = word;
}

__global__ void unpack_kernel(const uint32_t* __restrict__ packed, int K, int bits, int wpr,
                              long n_words, int8_t* __restrict__ codes) {
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_words) return;
  long row = i / wpr;
  int j = (int)(i % wpr);
  uint32_t word = packed[i];
  int8_t* out = codes + row * (long)K;
  if (bits == 4) {
#pragma unroll
    for (int e = 0; e < 8; ++e) out[8 * j + e] = (int8_t)((int)((word >> (4 * e)) & 15u) - 8);
  } else {
#pragma unroll
    for (int e = 0; e < 10; ++e) {
      int k = 10 * j + e;
      if (k < K) out[k] = (int8_t)((int)((word >> (3 * e)) & 7u) - 4);
    }
  }
}

// One warp per row of hd <= 256 fp16 values.
__global__ void kv_quant_int8_kernel(const __half* __restrict__ x, int rows, int hd,
                                     int8_t* __restrict__ codes, __half* __restrict__ scales) {
  long row = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __half* p = x + row * hd;
  float v[8];
  float m = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int i = lane + 32 * e;
    v[e] = (i < hd) ? __half2float(p[i]) : 0.0f;
    m = fmaxf(m, fabsf(v[e]));
  }
  m = warp_max(m);
  const __half sh = kv_int8_scale(m);
  const float s = __half2float(sh);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    int i = lane + 32 * e;
    if (i < hd) codes[row * hd + i] = kv_int8_code(v[e], s);
  }
  if (lane == 0) scales[row] = sh;
}

inline unsigned blocks_for(long n, int threads) { return (unsigned)((n + threads - 1) / threads); }

}  // namespace

tl_status launch_pack(const float* w, int N, int K, int bits, int group, uint32_t* packed,
                      uint16_t* scales, cudaStream_t s) {
  long n_groups = (long)N * (K / group);
  __half* sc = reinterpret_cast<__half*>(scales);
  pack_scales_kernel<<<blocks_for(n_groups * 32, 256), 256, 0, s>>>(
      w, K, group, n_groups, bits == 4 ? 7.0f : 3.0f, sc);
  TL_LAUNCH_CHECK();
  if (bits == 4) {
    long n_words = (long)N * (K / 8);
    pack_int4_words_kernel<<<blocks_for(n_words, 256), 256, 0, s>>>(w, K, group, n_words, sc,
                                                                     packed);
  } else {
    int wpr = ((K + 9) / 10 + 3) / 4 * 4;
    long n_words = (long)N * wpr;
    pack_int3_words_kernel<<<blocks_for(n_words, 256), 256, 0, s>>>(w, K, group, wpr, n_words,
                                                                     sc, packed);
  }
  TL_LAUNCH_CHECK();
  return ok();
}

tl_status launch_pack_sign_bits(const float* w, int N, int K, int bits, int group,
                               const uint16_t* scales, uint32_t* sign, cudaStream_t s) {
  const int spr = (K + 31) / 32;
  const long n_words = (long)N * spr;
  pack_sign_bits_kernel<<<blocks_for(n_words, 256), 256, 0, s>>>(
      w, K, group, spr, n_words, bits == 4 ? -8.0f : -4.0f, bits == 4 ? 7.0f : 3.0f,
      reinterpret_cast<const __half*>(scales), sign);
  TL_LAUNCH_CHECK();
  return ok();
}

tl_status launch_unpack(const uint32_t* packed, int N, int K, int bits, int8_t* codes,
                        cudaStream_t s) {
  int wpr = bits == 4 ? K / 8 : ((K + 9) / 10 + 3) / 4 * 4;
  long n_words = (long)N * wpr;
  unpack_kernel<<<blocks_for(n_words, 256), 256, 0, s>>>(packed, K, bits, wpr, n_words, codes);
  TL_LAUNCH_CHECK();
  return ok();
}

tl_status launch_kv_quant_int8(const __half* x, int rows, int hd, int8_t* codes, __half* scales,
                               cudaStream_t s) {
  if (rows == 0) return ok();
  kv_quant_int8_kernel<<<blocks_for((long)rows * 32, 256), 256, 0, s>>>(x, rows, hd, codes,
                                                                        scales);
  TL_LAUNCH_CHECK();
  return ok();
}

}  // namespace tl
