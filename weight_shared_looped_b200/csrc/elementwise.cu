// Row-wise kernels of the looped block: embedding gather, split-K reduction +
// residual add + RMSNorm (pre-norm; the final RMSNorm replaces the output head:
// "Performance and Memory", "Benchmark Shape Matters", no logits), RoPE on q/k
// with the K/V cache append (fp16, or per-(token, head) INT8 with one fp16
// scale: "Performance and Memory", "KV cache INT8"), and SwiGLU.
//
// Every reduction runs in a fixed order that depends only on the row length,
// so a row's result never depends on how many rows share the launch.
#include "kv_quant.cuh"
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
  if (a.exit_it && threadIdx.x == 0) a.exit_it[row] = 0;
  const int src = a.src_row ? a.src_row[row] : row;
  float* h = a.h + (size_t)row * a.d;
  const __half* e;
  if (a.ids) {
    int id = a.ids[src];
    if (id < 0 || id >= a.vocab) {
      set_status(a.status, TL_ERR_INVALID_ARG);
      id = 0;
    }
    e = a.embed + (size_t)id * a.d;
  } else {
    e = a.h_in + (size_t)src * a.d;
  }
  // eight halves per thread and step (d is a multiple of 256)
  for (int i = threadIdx.x * 8; i < a.d; i += blockDim.x * 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(e + i);
    const __half2* hp = reinterpret_cast<const __half2*>(&w);
    const float2 f0 = __half22float2(hp[0]), f1 = __half22float2(hp[1]);
    const float2 f2 = __half22float2(hp[2]), f3 = __half22float2(hp[3]);
    *reinterpret_cast<float4*>(h + i) = make_float4(f0.x, f0.y, f1.x, f1.y);
    *reinterpret_cast<float4*>(h + i + 4) = make_float4(f2.x, f2.y, f3.x, f3.y);
  }
}

// ------------------------------------------------------------------ residual + RMSNorm
// One CTA of d/8 threads per row, each thread two float4 vectors (columns
// 4t.. and d/2 + 4t..).  The split-K partial sums are loaded up to eight
// (d <= 2048) or four splits at a time (independent loads in flight) and added
// in split order.  The sum of
// squares is reduced per thread, per warp (xor tree) and over the warps in
// order: a fixed order that depends only on d.  One CTA per row keeps the
// grid small (a prefill of 128 rows is one CTA per SM) so that it shares the
// SMs with the GEMM CTAs launched early next to it.
constexpr int NORM_MAX_WARPS = 32;

__device__ __forceinline__ void add4(float4& a, const float4 b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}

template <int MAXT, int SP>
__global__ void __launch_bounds__(MAXT) residual_norm_kernel(NormArgs a) {
  __shared__ float red[NORM_MAX_WARPS];
  const int row = blockIdx.x;
  const int nthr = blockDim.x, nw = nthr >> 5;
  const int c0 = threadIdx.x * 4, c1 = a.d / 2 + threadIdx.x * 4;
  // the gains are constants of the model and the lane map an input of the
  // call: read them before waiting for the previous kernel, so no load round
  // trip follows the reduction
  const bool want_x = row < a.n_next;
  const bool want_y = row >= a.fin_lo && row < a.fin_hi;
  const float* gam = want_x ? a.gamma_next : want_y ? a.gamma_final : nullptr;
  float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0;
  if (gam) {
    g0 = *reinterpret_cast<const float4*>(gam + c0);
    g1 = *reinterpret_cast<const float4*>(gam + c1);
  }
  const int out_row = a.out_row ? a.out_row[row] : row;
  pdl_enter();
  float* h = a.h + (size_t)row * a.d;
  float4 v0 = *reinterpret_cast<const float4*>(h + c0);
  float4 v1 = *reinterpret_cast<const float4*>(h + c1);
  const bool frozen = a.ex.skip && a.ex.exit_it[row] != 0;   // stopped by the residual-norm check
  if (row < a.n_add && a.S > 0 && !frozen) {
    const size_t sstride = (size_t)a.part_rows * a.d;
    const float* p0 = a.part + (size_t)row * a.d;
    for (int sp = 0; sp < a.S; sp += SP) {
      const int n = min(SP, a.S - sp);
      float4 t0[SP], t1[SP];
#pragma unroll
      for (int q = 0; q < SP; ++q) {
        if (q < n) {
          t0[q] = __ldcg(reinterpret_cast<const float4*>(p0 + (sp + q) * sstride + c0));
          t1[q] = __ldcg(reinterpret_cast<const float4*>(p0 + (sp + q) * sstride + c1));
        }
      }
#pragma unroll
      for (int q = 0; q < SP; ++q) {
        if (q < n) {
          add4(v0, t0[q]);
          add4(v1, t1[q]);
        }
      }
    }
    *reinterpret_cast<float4*>(h + c0) = v0;
    *reinterpret_cast<float4*>(h + c1) = v1;
  }
  if (a.trace) {
    float* tr = a.trace + (size_t)out_row * a.d;
    *reinterpret_cast<float4*>(tr + c0) = v0;
    *reinterpret_cast<float4*>(tr + c1) = v1;
  }
  if (!want_x && !want_y) return;
  float ss = 0.0f;
  ss = fmaf(v0.x, v0.x, ss);
  ss = fmaf(v0.y, v0.y, ss);
  ss = fmaf(v0.z, v0.z, ss);
  ss = fmaf(v0.w, v0.w, ss);
  ss = fmaf(v1.x, v1.x, ss);
  ss = fmaf(v1.y, v1.y, ss);
  ss = fmaf(v1.z, v1.z, ss);
  ss = fmaf(v1.w, v1.w, ss);
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
  for (int w = 0; w < nw; ++w) tot += red[w];
  const float r = rsqrtf(tot / (float)a.d + a.eps);
  // the residual-norm check on the stream entering the next loop iteration
  if (a.ex.check_iter > 0 && threadIdx.x == 0 && row < a.n_next && a.ex.exit_it[row] == 0 &&
      sqrtf(tot) > a.ex.tau)
    a.ex.exit_it[row] = a.ex.check_iter;
  if (a.loops_out && want_y && threadIdx.x == 0) {
    const int e = a.ex.exit_it ? a.ex.exit_it[row] : 0;
    a.loops_out[out_row] = e != 0 ? e : a.L_all > 0 ? a.L_all : a.L_row[row];
  }
  auto out_x = [&](int c, const float4 v, const float4 g) {
    const __half2 lo = __halves2half2(__float2half_rn(v.x * r * g.x), __float2half_rn(v.y * r * g.y));
    const __half2 hi = __halves2half2(__float2half_rn(v.z * r * g.z), __float2half_rn(v.w * r * g.w));
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.x + (size_t)row * a.d + c) = pk;
  };
  auto out_y = [&](int c, const float4 v, const float4 g) -> bool {
    float4 o;
    o.x = v.x * r * g.x;
    o.y = v.y * r * g.y;
    o.z = v.z * r * g.z;
    o.w = v.w * r * g.w;
    *reinterpret_cast<float4*>(a.y + (size_t)out_row * a.d + c) = o;
    return !isfinite(o.x) || !isfinite(o.y) || !isfinite(o.z) || !isfinite(o.w);
  };
  if (want_x) {
    out_x(c0, v0, g0);
    out_x(c1, v1, g1);
  } else {
    const bool bad0 = out_y(c0, v0, g0);
    const bool bad1 = out_y(c1, v1, g1);
    if (bad0 || bad1) set_status(a.status, TL_ERR_NUMERIC);
  }
}

// ------------------------------------------------------------------ RoPE + KV append
// One warp per (row, head).  Lane l handles rotate-half pairs (i, i + hd/2)
// for i = l, l + 32 (hd = 128) or i = l (hd = 64).
__global__ void rope_kv_kernel(RopeKvArgs a) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool active = wid < a.rows * a.H;
  const int row = wid / a.H, head = wid % a.H;
  const int half = a.hd / 2;
  const int npair = half / 32;   // 1 or 2
  int kv_lane = a.lane, pos = a.pos0 + row;
  // prefill: the positions are the row indices, and the RoPE table and the
  // cache's layer offsets are constants: read them before waiting for the QKV
  // projection
  float2 csp[2] = {make_float2(1.f, 0.f), make_float2(1.f, 0.f)};
  int cum = 0;
  if (active && !a.decode) {
#pragma unroll
    for (int p = 0; p < 2; ++p)
      if (p < npair) csp[p] = a.rope_cs[(size_t)pos * half + lane + 32 * p];
    if (a.kv_base) cum = a.hdr->cum_layers[kv_lane];
  }
  pdl_enter();
  if (!active) return;
  if (a.decode) {
    kv_lane = a.lane_of_row[row];
    pos = a.hdr->pos[kv_lane];
#pragma unroll
    for (int p = 0; p < 2; ++p)
      if (p < npair) csp[p] = a.rope_cs[(size_t)pos * half + lane + 32 * p];
    if (a.kv_base) cum = a.hdr->cum_layers[kv_lane];
  }
  // columns of the partial sums: q | k | v, or k | v only
  const int ncol = a.kv_only ? 2 : 3;
  const size_t koff = a.kv_only ? 0 : (size_t)a.d, voff = koff + a.d;
  const size_t row3 = (size_t)row * ncol * a.d;
  const size_t split_stride = (size_t)a.rows * ncol * a.d;
  float q[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, k[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  float v[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  // partial sums: all q/k/v elements of up to four splits in flight, added in
  // split order
  for (int s0 = 0; s0 < a.S; s0 += 4) {
    const int ns = min(4, a.S - s0);
    float t[4][2][2][3];
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          if (s < ns && p < npair) {
            const float* ps = a.part + (size_t)(s0 + s) * split_stride + row3 +
                              (size_t)head * a.hd + lane + 32 * p + hh * half;
            t[s][p][hh][0] = a.kv_only ? 0.f : __ldcg(ps);
            t[s][p][hh][1] = __ldcg(ps + koff);
            t[s][p][hh][2] = __ldcg(ps + voff);
          }
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          if (s < ns && p < npair) {
            q[p][hh] += t[s][p][hh][0];
            k[p][hh] += t[s][p][hh][1];
            v[p][hh] += t[s][p][hh][2];
          }
  }
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    if (p < npair) {
      const float2 cs = csp[p];
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
        if (a.q) a.q[col] = __float2half_rn(q[p][hh]);
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
  char* layer = a.kv_base + (size_t)(cum + a.layer) * a.layer_bytes;
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
    const __half ksh = kv_int8_scale(kmax);
    const __half vsh = kv_int8_scale(vmax);
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
          K[i + hh * half] = kv_int8_code(kx, ks);
          V[i + hh * half] = kv_int8_code(vx, vs);
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

__global__ void add_pos_kernel(KvHeader* hdr, int lane, int n) {
  pdl_enter();
  hdr->pos[lane] += n;
}

__global__ void set_i32_kernel(int32_t* p, int value) {
  pdl_enter();
  *p = value;
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
  // d = 256 * 2^k: d / 8 threads (32 .. 1024)
  if (a.d < 256 || a.d > 8192 || (a.d & (a.d - 1)) != 0)
    return set_error(TL_ERR_UNSUPPORTED, "d_model %d: the norm needs a power of two in [256, 8192]", a.d);
  // up to 2048 columns: 256 threads with eight splits in flight, or sixteen
  // for the prefill projections' 9-16 splits (one round trip instead of two;
  // at decode the larger kernel measured slower); wider rows: four at a time
  if (a.d <= 2048 && a.rows > 8 && a.S > 8 && a.S <= 16)
    TL_LAUNCH_PDL((residual_norm_kernel<256, 16>), a.rows, a.d / 8, 0, s, a);
  else if (a.d <= 2048)
    TL_LAUNCH_PDL((residual_norm_kernel<256, 8>), a.rows, a.d / 8, 0, s, a);
  else
    TL_LAUNCH_PDL((residual_norm_kernel<1024, 4>), a.rows, a.d / 8, 0, s, a);
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

tl_status launch_add_pos(KvHeader* hdr, int lane, int n, cudaStream_t s) {
  TL_LAUNCH_PDL(add_pos_kernel, 1, 1, 0, s, hdr, lane, n);
  return ok();
}

namespace {
__global__ void append_rows_kernel(AppendRowsArgs a) {
  pdl_enter();
  const int r = blockIdx.x;
  const int pos = a.hdr->pos[a.lane[r]] + a.off[r];
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)r * a.d);
  uint4* dst = reinterpret_cast<uint4*>(a.slot[r] + (size_t)pos * a.d);
  for (int i = threadIdx.x; i < a.d / 8; i += blockDim.x) dst[i] = src[i];
}
}  // namespace

tl_status launch_append_rows(const AppendRowsArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  if (a.d % 8 != 0) return set_error(TL_ERR_UNSUPPORTED, "append rows: d %% 8");
  TL_LAUNCH_PDL(append_rows_kernel, a.rows, 256, 0, s, a);
  return ok();
}

tl_status launch_set_i32(int32_t* p, int value, cudaStream_t s) {
  TL_LAUNCH_PDL(set_i32_kernel, 1, 1, 0, s, p, value);
  return ok();
}

tl_status launch_advance_pos(KvHeader* hdr, int n_lanes, cudaStream_t s) {
  TL_LAUNCH_PDL(advance_pos_kernel, 1, kMaxLanes, 0, s, hdr, n_lanes);
  return ok();
}

}  // namespace tl
