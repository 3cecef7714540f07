// Row-wise kernels of the looped block: embedding gather, split-K reduction +
// residual add + RMSNorm (pre-norm; the final RMSNorm replaces the output head:
// "Performance and Memory", "Benchmark Shape Matters", no logits), RoPE on q/k
// with the K/V cache append (fp16, or per-(token, head) INT8 with one fp16
// scale: "Performance and Memory", "KV cache INT8"), and SwiGLU.
//
// Every reduction runs in a fixed order that depends only on the row length,
// so a row's result never depends on how many rows share the launch.
#include "tl_launch.cuh"

namespace tl {
namespace {

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

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ embed
__global__ void embed_kernel(EmbedArgs a) {
  pdl_enter();
  const int row = blockIdx.x;
  const int src = a.src_row ? a.src_row[row] : row;
  float* h = a.h + (size_t)row * a.d;
  if (a.ids) {
    int id = a.ids[src];
    if (id < 0 || id >= a.vocab) {
      set_status(a.status, TL_ERR_INVALID_ARG);
      id = 0;
    }
    const __half* e = a.embed + (size_t)id * a.d;
    for (int i = threadIdx.x; i < a.d; i += blockDim.x) h[i] = __half2float(e[i]);
  } else {
    const __half* e = a.h_in + (size_t)src * a.d;
    for (int i = threadIdx.x; i < a.d; i += blockDim.x) h[i] = __half2float(e[i]);
  }
}

// ------------------------------------------------------------------ residual + RMSNorm
constexpr int NORM_THREADS = 256;

// PER = d / 256 elements per thread.  Partial sums are loaded four splits at a
// time (independent loads in flight) and added in split order.
template <int PER>
__global__ void __launch_bounds__(NORM_THREADS) residual_norm_kernel(NormArgs a) {
  pdl_enter();
  __shared__ float red[NORM_THREADS / 32];
  const int row = blockIdx.x;
  float* h = a.h + (size_t)row * a.d;
  const int out_row = a.out_row ? a.out_row[row] : row;
  float v[PER];
  const bool add = row < a.n_add && a.S > 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) v[e] = h[threadIdx.x + e * NORM_THREADS];
  if (add) {
    const size_t sstride = (size_t)a.part_rows * a.d;
    const float* p0 = a.part + (size_t)row * a.d + threadIdx.x;
    int sp = 0;
    for (; sp + 4 <= a.S; sp += 4) {
      float t[4][PER];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < PER; ++e) t[q][e] = p0[(sp + q) * sstride + e * NORM_THREADS];
#pragma unroll
      for (int e = 0; e < PER; ++e) v[e] = (((v[e] + t[0][e]) + t[1][e]) + t[2][e]) + t[3][e];
    }
    for (; sp < a.S; ++sp)
#pragma unroll
      for (int e = 0; e < PER; ++e) v[e] += p0[sp * sstride + e * NORM_THREADS];
#pragma unroll
    for (int e = 0; e < PER; ++e) h[threadIdx.x + e * NORM_THREADS] = v[e];
  }
  if (a.trace) {
    float* tr = a.trace + (size_t)out_row * a.d;
#pragma unroll
    for (int e = 0; e < PER; ++e) tr[threadIdx.x + e * NORM_THREADS] = v[e];
  }
  const bool want_x = row < a.n_next;
  const bool want_y = row >= a.fin_lo && row < a.fin_hi;
  if (!want_x && !want_y) return;
  float ss = 0.0f;
#pragma unroll
  for (int e = 0; e < PER; ++e) ss = fmaf(v[e], v[e], ss);
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int w = 0; w < NORM_THREADS / 32; ++w) tot += red[w];
  const float r = rsqrtf(tot / (float)a.d + a.eps);
  if (want_x) {
    __half* x = a.x + (size_t)row * a.d;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int i = threadIdx.x + e * NORM_THREADS;
      x[i] = __float2half_rn(v[e] * r * a.gamma_next[i]);
    }
  } else {
    float* y = a.y + (size_t)out_row * a.d;
    bool bad = false;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int i = threadIdx.x + e * NORM_THREADS;
      const float o = v[e] * r * a.gamma_final[i];
      bad |= !isfinite(o);
      y[i] = o;
    }
    if (bad) set_status(a.status, TL_ERR_NUMERIC);
  }
}

// ------------------------------------------------------------------ RoPE + KV append
// One warp per (row, head).  Lane l handles rotate-half pairs (i, i + hd/2)
// for i = l, l + 32 (hd = 128) or i = l (hd = 64).
__global__ void rope_kv_kernel(RopeKvArgs a) {
  pdl_enter();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= a.rows * a.H) return;
  const int row = wid / a.H, head = wid % a.H;
  const int half = a.hd / 2;
  const int npair = half / 32;   // 1 or 2
  int kv_lane = a.lane, pos = row;
  if (a.decode) {
    kv_lane = a.lane_of_row[row];
    pos = a.hdr->pos[kv_lane];
  }
  const size_t row3 = (size_t)row * 3 * a.d;
  const size_t split_stride = (size_t)a.rows * 3 * a.d;
  float q[2][2], k[2][2], v[2][2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    if (p < npair) {
      int i = lane + 32 * p;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        size_t col = (size_t)head * a.hd + i + hh * half;
        float sq = 0.f, sk = 0.f, sv = 0.f;
        for (int s = 0; s < a.S; ++s) {
          const float* ps = a.part + s * split_stride + row3;
          sq += ps[col];
          sk += ps[a.d + col];
          sv += ps[2 * a.d + col];
        }
        q[p][hh] = sq;
        k[p][hh] = sk;
        v[p][hh] = sv;
      }
      float2 cs = a.rope_cs[(size_t)pos * half + i];
      float q0 = q[p][0], q1 = q[p][1], k0 = k[p][0], k1 = k[p][1];
      q[p][0] = q0 * cs.x - q1 * cs.y;
      q[p][1] = q1 * cs.x + q0 * cs.y;
      k[p][0] = k0 * cs.x - k1 * cs.y;
      k[p][1] = k1 * cs.x + k0 * cs.y;
    }
  }
  __half kh[2][2], vh[2][2];
  float kmax = 0.f, vmax = 0.f;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    if (p < npair) {
      int i = lane + 32 * p;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        size_t col = (size_t)row * a.d + (size_t)head * a.hd + i + hh * half;
        a.q[col] = __float2half_rn(q[p][hh]);
        kh[p][hh] = __float2half_rn(k[p][hh]);
        vh[p][hh] = __float2half_rn(v[p][hh]);
        if (a.k) a.k[col] = kh[p][hh];
        if (a.v) a.v[col] = vh[p][hh];
        kmax = fmaxf(kmax, fabsf(__half2float(kh[p][hh])));
        vmax = fmaxf(vmax, fabsf(__half2float(vh[p][hh])));
      }
    }
  }
  if (!a.kv_base) return;
  char* layer = a.kv_base + (size_t)(a.hdr->cum_layers[kv_lane] + a.layer) * a.layer_bytes;
  const size_t eoff = ((size_t)head * a.max_ctx + pos) * a.hd;
  if (!a.kv_int8) {
    __half* K = reinterpret_cast<__half*>(layer) + eoff;
    __half* V = reinterpret_cast<__half*>(layer + a.kv_region_bytes) + eoff;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      if (p < npair) {
        int i = lane + 32 * p;
        K[i] = kh[p][0];
        K[i + half] = kh[p][1];
        V[i] = vh[p][0];
        V[i + half] = vh[p][1];
      }
    }
  } else {
    kmax = warp_max(kmax);
    vmax = warp_max(vmax);
    __half ksh = __float2half_rn(__fdiv_rn(kmax, 127.0f));
    __half vsh = __float2half_rn(__fdiv_rn(vmax, 127.0f));
    float ks = __half2float(ksh), vs = __half2float(vsh);
    int8_t* K = reinterpret_cast<int8_t*>(layer) + eoff;
    int8_t* V = reinterpret_cast<int8_t*>(layer + a.kv_region_bytes) + eoff;
    __half* scales = reinterpret_cast<__half*>(layer + 2 * a.kv_region_bytes);
    const size_t soff = (size_t)head * a.max_ctx + pos;
    const size_t scale_region = (a.layer_bytes - 2 * a.kv_region_bytes) / 2;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      if (p < npair) {
        int i = lane + 32 * p;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float kx = __half2float(kh[p][hh]), vx = __half2float(vh[p][hh]);
          int kc = ks == 0.f ? 0 : (int)fminf(fmaxf(rintf(__fdiv_rn(kx, ks)), -127.f), 127.f);
          int vc = vs == 0.f ? 0 : (int)fminf(fmaxf(rintf(__fdiv_rn(vx, vs)), -127.f), 127.f);
          K[i + hh * half] = (int8_t)kc;
          V[i + hh * half] = (int8_t)vc;
        }
      }
    }
    if (lane == 0) {
      scales[soff] = ksh;
      *reinterpret_cast<__half*>(reinterpret_cast<char*>(scales) + scale_region + soff * 2) = vsh;
    }
  }
}

// ------------------------------------------------------------------ SwiGLU
__global__ void swiglu_kernel(const float* __restrict__ part, int S, int rows, int F,
                              __half* __restrict__ u) {
  pdl_enter();
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  size_t n = (size_t)rows * F;
  if (i >= n) return;
  size_t r = i / F, f = i % F;
  const size_t split_stride = (size_t)rows * 2 * F;
  float g = 0.f, up = 0.f;
  for (int s = 0; s < S; ++s) {
    const float* p = part + s * split_stride + r * 2 * F;
    g += p[f];
    up += p[F + f];
  }
  float silu = g / (1.0f + __expf(-g));
  u[i] = __float2half_rn(silu * up);
}

__global__ void set_pos_kernel(KvHeader* hdr, int lane, int value) {
  pdl_enter();
  if (lane < 0) {
    for (int i = 0; i < kMaxLanes; ++i) hdr->pos[i] = value;
  } else {
    hdr->pos[lane] = value;
  }
}

__global__ void advance_pos_kernel(KvHeader* hdr, int n_lanes) {
  pdl_enter();
  int i = threadIdx.x;
  if (i < n_lanes) hdr->pos[i] += 1;
}

}  // namespace

tl_status launch_embed(const EmbedArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  TL_LAUNCH_PDL(embed_kernel, a.rows, 256, 0, s, a);
  return ok();
}

tl_status launch_residual_norm(const NormArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  switch (a.d / NORM_THREADS) {
    case 1: TL_LAUNCH_PDL(residual_norm_kernel<1>, a.rows, NORM_THREADS, 0, s, a); break;
    case 2: TL_LAUNCH_PDL(residual_norm_kernel<2>, a.rows, NORM_THREADS, 0, s, a); break;
    case 4: TL_LAUNCH_PDL(residual_norm_kernel<4>, a.rows, NORM_THREADS, 0, s, a); break;
    case 8: TL_LAUNCH_PDL(residual_norm_kernel<8>, a.rows, NORM_THREADS, 0, s, a); break;
    case 16: TL_LAUNCH_PDL(residual_norm_kernel<16>, a.rows, NORM_THREADS, 0, s, a); break;
    case 32: TL_LAUNCH_PDL(residual_norm_kernel<32>, a.rows, NORM_THREADS, 0, s, a); break;
    default: return set_error(TL_ERR_UNSUPPORTED, "d_model %d: the norm needs d/256 in {1,2,4,...,32}", a.d);
  }
  TL_LAUNCH_CHECK();
  return ok();
}

tl_status launch_rope_kv(const RopeKvArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  long warps = (long)a.rows * a.H;
  TL_LAUNCH_PDL(rope_kv_kernel, (unsigned)((warps * 32 + 127) / 128), 128, 0, s, a);
  return ok();
}

tl_status launch_swiglu(const float* part, int S, int rows, int F, __half* u, cudaStream_t s) {
  if (rows == 0) return ok();
  size_t n = (size_t)rows * F;
  TL_LAUNCH_PDL(swiglu_kernel, (unsigned)((n + 255) / 256), 256, 0, s, part, S, rows, F, u);
  return ok();
}

tl_status launch_set_pos(KvHeader* hdr, int lane, int value, cudaStream_t s) {
  TL_LAUNCH_PDL(set_pos_kernel, 1, 1, 0, s, hdr, lane, value);
  return ok();
}

tl_status launch_advance_pos(KvHeader* hdr, int n_lanes, cudaStream_t s) {
  TL_LAUNCH_PDL(advance_pos_kernel, 1, kMaxLanes, 0, s, hdr, n_lanes);
  return ok();
}

}  // namespace tl
