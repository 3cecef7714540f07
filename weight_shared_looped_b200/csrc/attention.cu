// Causal attention: softmax(q k^T / sqrt(hd)) v per head.
//
// Prefill: tiled over key blocks with an online (running max / running sum)
// softmax, the role the pages give the tiled prefill kernel ("Performance and
// Memory", "Current Benchmark States": full prefill attention 0.143 ms ->
// 0.087 ms with the safer tiled path).
// Decode: one query per (lane, head) against the lane's cached keys 0..pos,
// FP16 or INT8 (code * fp16 scale) ("Production Roadmap", Stage 2: keep the
// direct cached single-query path for decode; "Performance and Memory", "KV
// cache INT8").  The context is split into fixed 64-key chunks (a function of
// the position only) whose partial results are merged in chunk order, so a
// lane's output does not depend on the other lanes.
#include "tl_internal.cuh"

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

// ------------------------------------------------------------------ prefill
constexpr int PQ = 16;     // queries per CTA (4 warps x 4)
constexpr int PK = 64;     // keys per tile

template <int HD>
__global__ void __launch_bounds__(128) attn_prefill_kernel(const __half* __restrict__ q,
                                                           const __half* __restrict__ k,
                                                           const __half* __restrict__ v,
                                                           __half* __restrict__ out, int T,
                                                           int H, float scale) {
  __shared__ __align__(16) __half Ks[PK][HD + 2];
  __shared__ __align__(16) __half Vs[PK][HD + 8];
  __shared__ float Qs[PQ][HD];
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * PQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = H * HD;
  constexpr int DPL = HD / 32;   // output dims per lane

  for (int i = threadIdx.x; i < PQ * HD; i += 128) {
    int r = i / HD, e = i % HD;
    int t = q0 + r;
    Qs[r][e] = t < T ? __half2float(q[(size_t)t * d + head * HD + e]) * scale : 0.f;
  }
  float m[4], l[4], acc[4][DPL];
#pragma unroll
  for (int qi = 0; qi < 4; ++qi) {
    m[qi] = -INFINITY;
    l[qi] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[qi][e] = 0.f;
  }
  const int q_last = min(q0 + PQ, T) - 1;   // highest query position in this CTA
  for (int k0 = 0; k0 <= q_last; k0 += PK) {
    __syncthreads();
    for (int i = threadIdx.x; i < PK * (HD / 2); i += 128) {
      int r = i / (HD / 2), e2 = (i % (HD / 2)) * 2;
      int t = k0 + r;
      __half2 kk = __float2half2_rn(0.f), vv = __float2half2_rn(0.f);
      if (t < T) {
        kk = *reinterpret_cast<const __half2*>(k + (size_t)t * d + head * HD + e2);
        vv = *reinterpret_cast<const __half2*>(v + (size_t)t * d + head * HD + e2);
      }
      *reinterpret_cast<__half2*>(&Ks[r][e2]) = kk;
      *reinterpret_cast<__half2*>(&Vs[r][e2]) = vv;
    }
    __syncthreads();
#pragma unroll
    for (int qi = 0; qi < 4; ++qi) {
      const int qr = warp * 4 + qi;
      const int qpos = q0 + qr;
      if (qpos >= T) continue;   // warp-uniform
      float s[2];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int j = lane + 32 * jj;
        float dot = 0.f;
#pragma unroll 8
        for (int e = 0; e < HD; e += 2) {
          float2 kf = __half22float2(*reinterpret_cast<const __half2*>(&Ks[j][e]));
          dot = fmaf(Qs[qr][e], kf.x, dot);
          dot = fmaf(Qs[qr][e + 1], kf.y, dot);
        }
        s[jj] = (k0 + j <= qpos) ? dot : -INFINITY;
      }
      float mt = warp_max(fmaxf(s[0], s[1]));
      float m_new = fmaxf(m[qi], mt);
      float corr = __expf(m[qi] - m_new);
      float p0 = __expf(s[0] - m_new), p1 = __expf(s[1] - m_new);
      l[qi] = l[qi] * corr + warp_sum(p0 + p1);
      m[qi] = m_new;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[qi][e] *= corr;
      const int jmax = min(PK, qpos - k0 + 1);
      for (int j = 0; j < jmax; ++j) {
        float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
        for (int e = 0; e < DPL; e += 2) {
          float2 vf = __half22float2(*reinterpret_cast<const __half2*>(&Vs[j][lane * DPL + e]));
          acc[qi][e] = fmaf(pj, vf.x, acc[qi][e]);
          acc[qi][e + 1] = fmaf(pj, vf.y, acc[qi][e + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int qi = 0; qi < 4; ++qi) {
    const int qpos = q0 + warp * 4 + qi;
    if (qpos >= T) continue;
    const float inv = 1.0f / l[qi];
#pragma unroll
    for (int e = 0; e < DPL; e += 2) {
      __half2 o = __floats2half2_rn(acc[qi][e] * inv, acc[qi][e + 1] * inv);
      *reinterpret_cast<__half2*>(out + (size_t)qpos * d + head * HD + lane * DPL + e) = o;
    }
  }
}

// ------------------------------------------------------------------ decode
// grid (max_chunks, H, rows); 4 warps, 16 keys each.
template <int HD>
__global__ void __launch_bounds__(128) attn_decode_partial_kernel(DecodeAttnArgs a) {
  constexpr int DPL = HD / 32;
  __shared__ float sc[kDecodeChunk];
  __shared__ float wacc[4][HD];
  __shared__ float wl[4];
  const int chunk = blockIdx.x, head = blockIdx.y, row = blockIdx.z;
  const int lane_id = a.lane_of_row[row];
  const int n_keys = a.hdr->pos[lane_id] + 1;   // the current token is already appended
  const int n_chunks = (n_keys + kDecodeChunk - 1) / kDecodeChunk;
  if (chunk >= n_chunks) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = rsqrtf((float)HD);

  float qv[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e)
    qv[e] = __half2float(a.q[(size_t)row * a.d + head * HD + lane * DPL + e]) * scale;

  const char* layer =
      a.kv_base + (size_t)(a.hdr->cum_layers[lane_id] + a.layer) * a.layer_bytes;
  const size_t head_off = (size_t)head * a.max_ctx;
  const size_t scale_region = (a.layer_bytes - 2 * a.kv_region_bytes) / 2;
  const __half* ksc = reinterpret_cast<const __half*>(layer + 2 * a.kv_region_bytes);
  const __half* vsc = reinterpret_cast<const __half*>(layer + 2 * a.kv_region_bytes + scale_region);

  auto load_row = [&](int which, int pos, float* out) {
    const size_t eoff = (head_off + pos) * HD + lane * DPL;
    if (!a.kv_int8) {
      const __half* p = reinterpret_cast<const __half*>(layer + which * a.kv_region_bytes) + eoff;
#pragma unroll
      for (int e = 0; e < DPL; e += 2) {
        float2 f = __half22float2(*reinterpret_cast<const __half2*>(p + e));
        out[e] = f.x;
        out[e + 1] = f.y;
      }
    } else {
      const int8_t* p = reinterpret_cast<const int8_t*>(layer + which * a.kv_region_bytes) + eoff;
      const float s = __half2float((which == 0 ? ksc : vsc)[head_off + pos]);
#pragma unroll
      for (int e = 0; e < DPL; ++e) out[e] = (float)p[e] * s;
    }
  };

  const int base = chunk * kDecodeChunk;
  for (int i = 0; i < kDecodeChunk / 4; ++i) {
    const int j = warp * (kDecodeChunk / 4) + i;
    const int pos = base + j;
    float s = -INFINITY;
    if (pos < n_keys) {
      float kr[DPL];
      load_row(0, pos, kr);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) dot = fmaf(qv[e], kr[e], dot);
      s = warp_sum(dot);
    }
    if (lane == 0) sc[j] = s;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int j = 0; j < kDecodeChunk; ++j) m = fmaxf(m, sc[j]);
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float lsum = 0.f;
  for (int i = 0; i < kDecodeChunk / 4; ++i) {
    const int j = warp * (kDecodeChunk / 4) + i;
    const int pos = base + j;
    if (pos >= n_keys) break;
    const float p = __expf(sc[j] - m);
    lsum += p;
    float vr[DPL];
    load_row(1, pos, vr);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(p, vr[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) wacc[warp][lane * DPL + e] = acc[e];
  if (lane == 0) wl[warp] = lsum;
  __syncthreads();
  float* dst = a.scratch + (((size_t)row * a.H + head) * a.max_chunks + chunk) * (HD + 2);
  for (int e = threadIdx.x; e < HD; e += 128)
    dst[e] = wacc[0][e] + wacc[1][e] + wacc[2][e] + wacc[3][e];
  if (threadIdx.x == 0) {
    dst[HD] = m;
    dst[HD + 1] = wl[0] + wl[1] + wl[2] + wl[3];
  }
}

// grid (H, rows); merge the chunks of one (row, head) in chunk order.
template <int HD>
__global__ void __launch_bounds__(HD) attn_decode_merge_kernel(DecodeAttnArgs a) {
  const int head = blockIdx.x, row = blockIdx.y;
  const int lane_id = a.lane_of_row[row];
  const int n_keys = a.hdr->pos[lane_id] + 1;
  const int n_chunks = (n_keys + kDecodeChunk - 1) / kDecodeChunk;
  const float* src = a.scratch + ((size_t)row * a.H + head) * a.max_chunks * (HD + 2);
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, src[c * (HD + 2) + HD]);
  float L = 0.f, o = 0.f;
  const int e = threadIdx.x;
  for (int c = 0; c < n_chunks; ++c) {
    const float* p = src + c * (HD + 2);
    const float w = __expf(p[HD] - M);
    L = fmaf(p[HD + 1], w, L);
    o = fmaf(p[e], w, o);
  }
  a.out[(size_t)row * a.d + head * HD + e] = __float2half_rn(o / L);
}

}  // namespace

tl_status launch_attn_prefill(const __half* q, const __half* k, const __half* v, __half* out,
                              int T, int H, int hd, cudaStream_t s) {
  if (T == 0) return ok();
  dim3 grid((T + PQ - 1) / PQ, H);
  const float scale = 1.0f / sqrtf((float)hd);
  if (hd == 128)
    attn_prefill_kernel<128><<<grid, 128, 0, s>>>(q, k, v, out, T, H, scale);
  else if (hd == 64)
    attn_prefill_kernel<64><<<grid, 128, 0, s>>>(q, k, v, out, T, H, scale);
  else
    return set_error(TL_ERR_UNSUPPORTED, "head_dim %d not supported", hd);
  TL_LAUNCH_CHECK();
  return ok();
}

tl_status launch_attn_decode(const DecodeAttnArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  dim3 g1(a.max_chunks, a.H, a.rows), g2(a.H, a.rows);
  if (a.hd == 128) {
    attn_decode_partial_kernel<128><<<g1, 128, 0, s>>>(a);
    TL_LAUNCH_CHECK();
    attn_decode_merge_kernel<128><<<g2, 128, 0, s>>>(a);
  } else if (a.hd == 64) {
    attn_decode_partial_kernel<64><<<g1, 128, 0, s>>>(a);
    TL_LAUNCH_CHECK();
    attn_decode_merge_kernel<64><<<g2, 64, 0, s>>>(a);
  } else {
    return set_error(TL_ERR_UNSUPPORTED, "head_dim %d not supported", a.hd);
  }
  TL_LAUNCH_CHECK();
  return ok();
}

}  // namespace tl
