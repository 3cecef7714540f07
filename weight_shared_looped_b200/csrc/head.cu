// Greedy head over the tied embedding, the token choice a self-speculative
// step needs to compare its draft tokens with its verify tokens ("Current
// Status", speculative and adaptive decode table, self-speculative row):
//   id[r] = argmax over v of sum_k y[r][k] * E[v][k]   (lowest v wins a tie)
// for up to 8 rows of final-norm outputs y (fp32) and the fp16 embedding E
// [V][d].  The looped forward itself ends at the final RMSNorm; this head is
// used only by the speculative driver.
//
// Pass 1 streams E once (16-byte loads, all CTAs resident): a warp scores one
// vocabulary row at a time for every y row (fp32 products, per-lane sums in
// k order, xor-tree reduction: a fixed order), keeps its best (score, id)
// per y row, and the CTA's warps merge in warp order into one partial per
// CTA.  Pass 2 merges the partials in CTA order.
#include "tl_launch.cuh"

namespace tl {
namespace {

constexpr int HEAD_THREADS = 256;
constexpr int HEAD_WARPS = HEAD_THREADS / 32;

__device__ __forceinline__ bool better(float s, int v, float bs, int bv) {
  return s > bs || (s == bs && v < bv);
}

__global__ void __launch_bounds__(HEAD_THREADS) head_partial_kernel(const float* __restrict__ y, int n,
                                                                    const __half* __restrict__ E,
                                                                    int V, int d,
                                                                    float* __restrict__ part_s,
                                                                    int* __restrict__ part_v) {
  extern __shared__ __align__(16) float ys[];   // [n][d]
  __shared__ float ws[HEAD_WARPS][8];
  __shared__ int wv[HEAD_WARPS][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_enter();
  for (int i = threadIdx.x * 4; i < n * d; i += HEAD_THREADS * 4)
    *reinterpret_cast<float4*>(ys + i) = *reinterpret_cast<const float4*>(y + i);
  __syncthreads();
  float bs[8];
  int bv[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    bs[r] = -INFINITY;
    bv[r] = 0x7fffffff;
  }
  const int nvec = d / 8;                                  // 16-byte vectors per row
  const int gw = blockIdx.x * HEAD_WARPS + warp, nw = gridDim.x * HEAD_WARPS;
  for (int v = gw; v < V; v += nw) {
    const uint4* row = reinterpret_cast<const uint4*>(E + (size_t)v * d);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = lane; j < nvec; j += 32) {
      const uint4 w = __ldg(row + j);
      const __half2* h2 = reinterpret_cast<const __half2*>(&w);
      float e[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(h2[q]);
        e[2 * q] = f.x;
        e[2 * q + 1] = f.y;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < n) {
          const float* yr = ys + (size_t)r * d + 8 * j;
          const float4 y0 = *reinterpret_cast<const float4*>(yr);
          const float4 y1 = *reinterpret_cast<const float4*>(yr + 4);
          float a = acc[r];
          a = fmaf(e[0], y0.x, a);
          a = fmaf(e[1], y0.y, a);
          a = fmaf(e[2], y0.z, a);
          a = fmaf(e[3], y0.w, a);
          a = fmaf(e[4], y1.x, a);
          a = fmaf(e[5], y1.y, a);
          a = fmaf(e[6], y1.z, a);
          a = fmaf(e[7], y1.w, a);
          acc[r] = a;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < n) {
        float s = acc[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (better(s, v, bs[r], bv[r])) {
          bs[r] = s;
          bv[r] = v;
        }
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      ws[warp][r] = bs[r];
      wv[warp][r] = bv[r];
    }
  }
  __syncthreads();
  if (threadIdx.x < n) {
    const int r = threadIdx.x;
    float s = ws[0][r];
    int v = wv[0][r];
    for (int w = 1; w < HEAD_WARPS; ++w)
      if (better(ws[w][r], wv[w][r], s, v)) {
        s = ws[w][r];
        v = wv[w][r];
      }
    part_s[(size_t)blockIdx.x * 8 + r] = s;
    part_v[(size_t)blockIdx.x * 8 + r] = v;
  }
}

__global__ void head_merge_kernel(const float* __restrict__ part_s, const int* __restrict__ part_v,
                                  int parts, int n, int32_t* __restrict__ ids) {
  pdl_enter();
  const int r = threadIdx.x;
  if (r >= n) return;
  float s = part_s[r];
  int v = part_v[r];
  for (int c = 1; c < parts; ++c)
    if (better(part_s[(size_t)c * 8 + r], part_v[(size_t)c * 8 + r], s, v)) {
      s = part_s[(size_t)c * 8 + r];
      v = part_v[(size_t)c * 8 + r];
    }
  ids[r] = v;
}

}  // namespace

int head_parts() { return 148 * 4; }

tl_status launch_greedy_head(const float* y, int n, const __half* E, int V, int d, float* part_s,
                             int* part_v, int32_t* ids, cudaStream_t s) {
  if (n < 1 || n > 8) return set_error(TL_ERR_INVALID_ARG, "greedy head: %d rows", n);
  if (d % 8 != 0) return set_error(TL_ERR_UNSUPPORTED, "greedy head: d %% 8");
  static std::atomic<uint64_t> attr_done{0};
  TL_TRY(once_per_device(attr_done, []() -> tl_status {
    TL_CUDA(cudaFuncSetAttribute(head_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 200 * 1024));
    return ok();
  }));
  const size_t smem = (size_t)n * d * sizeof(float);
  if (smem > 200 * 1024) return set_error(TL_ERR_UNSUPPORTED, "greedy head: %d x %d too large", n, d);
  const int parts = head_parts();
  TL_LAUNCH_PDL(head_partial_kernel, parts, HEAD_THREADS, smem, s, y, n, E, V, d, part_s, part_v);
  TL_LAUNCH_PDL(head_merge_kernel, 1, 32, 0, s, (const float*)part_s, (const int*)part_v, parts, n,
                ids);
  return ok();
}

}  // namespace tl
