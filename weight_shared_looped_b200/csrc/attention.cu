// Causal attention: softmax(q k^T / sqrt(hd)) v per head.
//
// Prefill: tiled over key blocks with an online (running max / running sum)
// softmax, the role the pages give the tiled prefill kernel ("Performance and
// Memory", "Current Benchmark States": full prefill attention 0.143 ms ->
// 0.087 ms with the safer tiled path).
// Decode: one query per (lane, head) against the lane's cached keys 0..pos,
// FP16 or INT8 (code * fp16 scale) ("Production Roadmap", Stage 2: keep the
// direct cached single-query path for decode; "Performance and Memory", "KV
// cache INT8").  The context is split over the CTAs of a thread-block cluster
// by a rule that depends only on the lane's position and the cache size, and
// the partial results are merged in a fixed order, so a lane's output does not
// depend on the other lanes.
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

// ------------------------------------------------------------------ prefill
// Tensor cores (mma.sync m16n8k16, fp16 in, fp32 accumulate): each warp
// owns 16 queries; S = Q K^T and O += P V run on the tensor cores with the
// score fragment reused in registers as the A operand of P V; V fragments come
// from shared memory through ldmatrix.trans.  Online softmax in base 2 with
// the 1/sqrt(hd) scale folded into log2(e).
constexpr int ATT_WARPS = 4;   // warps per CTA, 16 queries each
constexpr int FQ = 16 * ATT_WARPS;   // queries per CTA
constexpr int FK = 64;   // keys per tile

__device__ __forceinline__ void mma_f16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 16-byte cp.async, zero-filled when `valid` is false (rows past T).
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

// Two key tiles are copied per round trip (with the Q tile in the first): a
// seq-128 CTA loads everything it needs at once; longer sequences refill the
// two slots after each pair of tiles.
constexpr int ATT_RES = 2;   // key tiles resident in shared memory at once

template <int HD>
constexpr size_t attn_prefill_smem() {
  return (size_t)(FQ + 2 * ATT_RES * FK) * (HD + 8) * sizeof(__half);
}

template <int HD>
__global__ void __launch_bounds__(32 * ATT_WARPS) attn_prefill_tc_kernel(const __half* __restrict__ q,
                                                              const __half* __restrict__ k,
                                                              const __half* __restrict__ v,
                                                              __half* __restrict__ out, int T,
                                                              int H, float scale_log2) {
  pdl_enter();
  constexpr int LD = HD + 8;                 // halves per smem row (16-byte aligned, no conflicts)
  extern __shared__ __align__(16) __half att_smem[];
  __half (*Qs)[LD] = reinterpret_cast<__half (*)[LD]>(att_smem);                        // [FQ][LD]
  __half (*Kr)[FK][LD] = reinterpret_cast<__half (*)[FK][LD]>(att_smem + FQ * LD);        // [ATT_RES]
  __half (*Vr)[FK][LD] = reinterpret_cast<__half (*)[FK][LD]>(att_smem + (FQ + ATT_RES * FK) * LD);
  const int head = blockIdx.y;
  const int q0 = blockIdx.x * FQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int d = H * HD;
  const int qw = q0 + warp * 16;             // first query of this warp
  constexpr int KS = HD / 16;                // k steps over head_dim
  constexpr int NT = HD / 8;                 // output n tiles over head_dim
  constexpr int CPR = HD / 8;                // 16-byte pieces per row
  constexpr int NTH = 32 * ATT_WARPS;
  const int q_hi = min(q0 + FQ, T) - 1;
  const int ntiles = q_hi / FK + 1;
  // copy key tiles [t0, t0 + ATT_RES) into the resident slots (one round trip)
  auto issue = [&](int t0) {
    for (int tt = 0; tt < ATT_RES; ++tt) {
      const int kt = t0 + tt;
      if (kt >= ntiles) break;
      const int k0 = kt * FK;
      for (int i = threadIdx.x; i < FK * CPR; i += NTH) {
        const int r = i / CPR, c = (i % CPR) * 8;
        const bool ok = k0 + r < T;
        const size_t off = (size_t)(ok ? k0 + r : 0) * d + head * HD + c;
        cp_async16_zfill(&Kr[tt][r][c], k + off, ok);
        cp_async16_zfill(&Vr[tt][r][c], v + off, ok);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  for (int i = threadIdx.x; i < FQ * CPR; i += NTH) {
    const int r = i / CPR, c = (i % CPR) * 8;
    const bool ok = q0 + r < T;
    cp_async16_zfill(&Qs[r][c], q + (size_t)(ok ? q0 + r : 0) * d + head * HD + c, ok);
  }
  issue(0);

  uint32_t qa[KS][4];
  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  for (int kt = 0; kt < ntiles; ++kt) {
    const int k0 = kt * FK;
    if (kt % ATT_RES == 0) {
      if (kt > 0) {
        __syncthreads();                     // every warp is done with the resident tiles
        issue(kt);
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();
    }
    if (kt == 0) {
      // Q fragments (A operand, 16 x HD), rows qw+g and qw+g+8
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c = ks * 16 + 2 * t;
        qa[ks][0] = *reinterpret_cast<const uint32_t*>(&Qs[warp * 16 + g][c]);
        qa[ks][1] = *reinterpret_cast<const uint32_t*>(&Qs[warp * 16 + g + 8][c]);
        qa[ks][2] = *reinterpret_cast<const uint32_t*>(&Qs[warp * 16 + g][c + 8]);
        qa[ks][3] = *reinterpret_cast<const uint32_t*>(&Qs[warp * 16 + g + 8][c + 8]);
      }
    }
    const __half (*Ks)[LD] = Kr[kt % ATT_RES];
    const __half (*Vs)[LD] = Vr[kt % ATT_RES];
    if (k0 > qw + 15) continue;              // this warp's queries all precede the tile
    // S = Q K^T : 16 x 64
    float sc[FK / 8][4];
#pragma unroll
    for (int nt = 0; nt < FK / 8; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&Ks[nt * 8 + g][ks * 16 + 2 * t]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&Ks[nt * 8 + g][ks * 16 + 2 * t + 8]);
        mma_f16(sc[nt], qa[ks], b0, b1);
      }
    }
    // causal mask (key index > query index) and running max
    const int r0 = qw + g, r1 = qw + g + 8;
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int nt = 0; nt < FK / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = k0 + nt * 8 + 2 * t + e;
        float s0 = sc[nt][e] * scale_log2, s1 = sc[nt][2 + e] * scale_log2;
        if (key > r0 || key >= T) s0 = -INFINITY;
        if (key > r1 || key >= T) s1 = -INFINITY;
        sc[nt][e] = s0;
        sc[nt][2 + e] = s1;
        mx0 = fmaxf(mx0, s0);
        mx1 = fmaxf(mx1, s1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    // rows past T have no valid key at all: keep their state finite
    const float base0 = mx0 == -INFINITY ? 0.f : mx0;
    const float base1 = mx1 == -INFINITY ? 0.f : mx1;
    const float corr0 = exp2f(m0 - base0), corr1 = exp2f(m1 - base1);
    m0 = mx0;
    m1 = mx1;
    float ps0 = 0.f, ps1 = 0.f;
    uint32_t pa[FK / 16][4];
#pragma unroll
    for (int nt = 0; nt < FK / 8; ++nt) {
      const float p00 = exp2f(sc[nt][0] - base0), p01 = exp2f(sc[nt][1] - base0);
      const float p10 = exp2f(sc[nt][2] - base1), p11 = exp2f(sc[nt][3] - base1);
      ps0 += p00 + p01;
      ps1 += p10 + p11;
      const int kk = nt >> 1;
      if ((nt & 1) == 0) {
        pa[kk][0] = pack_half2(p00, p01);
        pa[kk][1] = pack_half2(p10, p11);
      } else {
        pa[kk][2] = pack_half2(p00, p01);
        pa[kk][3] = pack_half2(p10, p11);
      }
    }
    l0 = l0 * corr0 + ps0;
    l1 = l1 * corr1 + ps1;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      o[i][0] *= corr0;
      o[i][1] *= corr0;
      o[i][2] *= corr1;
      o[i][3] *= corr1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < FK / 16; ++kk) {
#pragma unroll
      for (int nt2 = 0; nt2 < NT / 2; ++nt2) {
        // four 8x8 tiles: keys kk*16 + {0..7, 8..15} x dims nt2*16 + {0..7, 8..15}
        const int mi = lane >> 3, ri = lane & 7;
        const __half* src = &Vs[kk * 16 + (mi & 1) * 8 + ri][nt2 * 16 + (mi >> 1) * 8];
        uint32_t b0, b1, b2, b3;
        asm volatile(
            "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
            : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
            : "r"((uint32_t)__cvta_generic_to_shared(src)));
        mma_f16(o[2 * nt2], pa[kk], b0, b1);
        mma_f16(o[2 * nt2 + 1], pa[kk], b2, b3);
      }
    }
  }
  // row sums across the quad, normalise, store
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int r0 = qw + g, r1 = qw + g + 8;
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int c = head * HD + nt * 8 + 2 * t;
    if (r0 < T)
      *reinterpret_cast<uint32_t*>(out + (size_t)r0 * d + c) = pack_half2(o[nt][0] * i0, o[nt][1] * i0);
    if (r1 < T)
      *reinterpret_cast<uint32_t*>(out + (size_t)r1 * d + c) = pack_half2(o[nt][2] * i1, o[nt][3] * i1);
  }
}

// ------------------------------------------------------------------ decode (cluster)
// Decode attention for one (row, head) on a thread-block cluster of CL CTAs
// (CL = ceil(max_ctx / 64) capped at 8, fixed per cache).  CTA r takes the
// contiguous keys [r * per, (r + 1) * per) of the lane's n_keys = pos + 1
// (per = ceil(n_keys / CL), which depends only on the lane's own position);
// its cached K/V rows are copied into shared memory before the wait for the
// QKV projection.  The CTA holding position pos forms k and v from the QKV
// partial sums, applies RoPE to k and appends both to the cache.  Each CTA
// keeps its max score, exponential sum and unnormalised P V; rank 0 merges
// the CTAs in rank order through distributed shared memory.
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
__device__ __forceinline__ float cl_ld(const float* local, uint32_t rank) {
  uint32_t addr = (uint32_t)__cvta_generic_to_shared(local), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Four int8 codes of a word to float, exactly: each biased byte goes into the
// low mantissa bits of 2^23 (prmt with the constant's upper bytes), then the
// bias 2^23 + 128 is subtracted.
__device__ __forceinline__ void int8x4_to_float(uint32_t w, float* f) {
  const uint32_t u = w ^ 0x80808080u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t b;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(b) : "r"(u), "r"(0x4B000000u), "r"(0x7650u | (uint32_t)i));
    f[i] = __uint_as_float(b) - 8388736.0f;
  }
}

constexpr int DS_KEYS = 64;     // keys per stage of the streaming decode kernel
constexpr int DS_STAGES = 3;    // stages in flight (cp.async ring)

template <int HD>
__global__ void __launch_bounds__(128) attn_decode_cluster_kernel(DecodeAttnArgs a, int CL,
                                                                  int max_per) {
  constexpr int HALF = HD / 2;
  constexpr int KSPLIT = 128 / HD;              // key slices in the P V step (1 or 2)
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ float qs[HD], kn[HD], vn[HD];
  __shared__ float acc_s[KSPLIT][HD];
  __shared__ float pw[DS_KEYS];                  // weights of the current stage's keys
  __shared__ float stat_s[2];                    // this CTA's max score and exponential sum
  __shared__ float red[4];
  const int crank = blockIdx.x, head = blockIdx.y, row = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int esz = a.kv_int8 ? 1 : 2;
  const int rowb = HD * esz;
  const int stage_bytes = DS_KEYS * rowb;
  unsigned char* kst = dsm;                                        // [DS_STAGES][DS_KEYS][rowb]
  unsigned char* vst = dsm + (size_t)DS_STAGES * stage_bytes;      // [DS_STAGES][DS_KEYS][rowb]
  float* ksc = reinterpret_cast<float*>(dsm + 2 * (size_t)DS_STAGES * stage_bytes);   // [max_per]
  float* vsc = ksc + max_per;
  // positions, the lane map, the RoPE table and the cached rows before pos
  // were written by earlier steps
  const int lane_id = a.lane_of_row[row];
  const int pos = a.hdr->pos[lane_id];
  const int n_keys = pos + 1;
  const int per = (n_keys + CL - 1) / CL;
  const int k0 = min(crank * per, n_keys), k1 = min(k0 + per, n_keys);
  const int nk = k1 - k0;
  const bool owner = nk > 0 && k1 == n_keys;     // holds position pos
  const int n_old = owner ? nk - 1 : nk;
  const int nsub = (nk + DS_KEYS - 1) / DS_KEYS;
  char* layer = const_cast<char*>(a.kv_base) +
                (size_t)(a.hdr->cum_layers[lane_id] + a.layer) * a.layer_bytes;
  const size_t head_off = (size_t)head * a.max_ctx;
  const size_t scale_region = (a.layer_bytes - 2 * a.kv_region_bytes) / 2;
  // copy the cached rows of stage `sub` into ring slot sub % DS_STAGES (one
  // commit group per stage, empty past the end)
  auto issue = [&](int sub) {
    if (sub < nsub) {
      const int lo = sub * DS_KEYS, cnt = min(DS_KEYS, n_old - lo);
      const int pieces = rowb / 16;
      for (int which = 0; which < 2; ++which) {
        const char* src = layer + which * a.kv_region_bytes + (head_off + k0 + lo) * rowb;
        unsigned char* dst = (which ? vst : kst) + (size_t)(sub % DS_STAGES) * stage_bytes;
        for (int i = tid; i < cnt * pieces; i += 128) {
          const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst + i * 16);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src + i * 16)
                       : "memory");
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int st = 0; st < DS_STAGES - 1; ++st) issue(st);
  if (a.kv_int8) {
    const __half* kq = reinterpret_cast<const __half*>(layer + 2 * a.kv_region_bytes);
    const __half* vq = reinterpret_cast<const __half*>(layer + 2 * a.kv_region_bytes + scale_region);
    for (int j = tid; j < n_old; j += 128) {
      ksc[j] = __half2float(kq[head_off + k0 + j]);
      vsc[j] = __half2float(vq[head_off + k0 + j]);
    }
  }
  float2 cs = make_float2(1.f, 0.f);
  if (tid < HD) cs = a.rope_cs[(size_t)pos * HALF + (tid % HALF)];
  pdl_enter();

  // q (and k, v in the owner) from the QKV partial sums, all splits in flight
  const size_t split_stride = (size_t)a.rows * 3 * a.d;
  const float* prow = a.qkv_part + (size_t)row * 3 * a.d + (size_t)head * HD;
  if (tid < HD) {
    float pq[8], pk[8], pv[8];
    float sq = 0.f, sk = 0.f, sv = 0.f;
    for (int s0 = 0; s0 < a.qkv_S; s0 += 8) {
      const int cnt = min(8, a.qkv_S - s0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < cnt) {
          const float* q = prow + (size_t)(s0 + j) * split_stride;
          pq[j] = q[tid];
          pk[j] = owner ? q[a.d + tid] : 0.f;
          pv[j] = owner ? q[2 * a.d + tid] : 0.f;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < cnt) {
          sq += pq[j];
          sk += pk[j];
          sv += pv[j];
        }
      }
    }
    qs[tid] = sq;
    kn[tid] = sk;
    vn[tid] = sv;
  }
  __syncthreads();
  float qr = 0.f, kr = 0.f;
  if (tid < HD) {
    if (tid < HALF) {
      qr = qs[tid] * cs.x - qs[tid + HALF] * cs.y;
      kr = kn[tid] * cs.x - kn[tid + HALF] * cs.y;
    } else {
      qr = qs[tid] * cs.x + qs[tid - HALF] * cs.y;
      kr = kn[tid] * cs.x + kn[tid - HALF] * cs.y;
    }
  }
  __syncthreads();
  // the query is rounded to fp16 as in the prefill path
  if (tid < HD) qs[tid] = __half2float(__float2half_rn(qr)) * rsqrtf((float)HD);
  // owner: the new entry (position pos = key nk - 1 of this CTA) is appended
  // to the cache now and copied into its stage slot when that stage is read
  uint32_t k_new = 0, v_new = 0;     // fp16 bits or int8 code of element tid
  if (owner) {
    const __half kh = __float2half_rn(kr);
    const __half vh = __float2half_rn(tid < HD ? vn[tid] : 0.f);
    if (!a.kv_int8) {
      if (tid < HD) {
        reinterpret_cast<__half*>(layer)[(head_off + pos) * HD + tid] = kh;
        reinterpret_cast<__half*>(layer + a.kv_region_bytes)[(head_off + pos) * HD + tid] = vh;
        k_new = __half_as_ushort(kh);
        v_new = __half_as_ushort(vh);
      }
    } else {
      float km = tid < HD ? fabsf(__half2float(kh)) : 0.f;
      float vm = tid < HD ? fabsf(__half2float(vh)) : 0.f;
      km = warp_max(km);
      vm = warp_max(vm);
      __shared__ float kmax_s[4], vmax_s[4];
      if (lane == 0) {
        kmax_s[warp] = km;
        vmax_s[warp] = vm;
      }
      __syncthreads();
      km = fmaxf(fmaxf(kmax_s[0], kmax_s[1]), fmaxf(kmax_s[2], kmax_s[3]));
      vm = fmaxf(fmaxf(vmax_s[0], vmax_s[1]), fmaxf(vmax_s[2], vmax_s[3]));
      const __half ksh = __float2half_rn(__fdiv_rn(km, 127.0f));
      const __half vsh = __float2half_rn(__fdiv_rn(vm, 127.0f));
      const float ksf = __half2float(ksh), vsf = __half2float(vsh);
      if (tid < HD) {
        const float kx = __half2float(kh), vx = __half2float(vh);
        const int kc = ksf == 0.f ? 0 : (int)fminf(fmaxf(rintf(__fdiv_rn(kx, ksf)), -127.f), 127.f);
        const int vc = vsf == 0.f ? 0 : (int)fminf(fmaxf(rintf(__fdiv_rn(vx, vsf)), -127.f), 127.f);
        reinterpret_cast<int8_t*>(layer)[(head_off + pos) * HD + tid] = (int8_t)kc;
        reinterpret_cast<int8_t*>(layer + a.kv_region_bytes)[(head_off + pos) * HD + tid] = (int8_t)vc;
        k_new = (uint32_t)(uint8_t)(int8_t)kc;
        v_new = (uint32_t)(uint8_t)(int8_t)vc;
      }
      if (tid == 0) {
        reinterpret_cast<__half*>(layer + 2 * a.kv_region_bytes)[head_off + pos] = ksh;
        reinterpret_cast<__half*>(layer + 2 * a.kv_region_bytes + scale_region)[head_off + pos] = vsh;
        ksc[nk - 1] = ksf;
        vsc[nk - 1] = vsf;
      }
    }
  }

  // streaming online softmax over the stages
  constexpr int QD = HD / 4;                     // head_dim quarter of a score thread
  constexpr int G4 = HD / 4, KS4 = 128 / G4;     // P V: 4-dim groups x key slices
  __syncthreads();                               // qs final
  const int qq = tid & 3;                        // this thread's quarter of head_dim
  float qreg[QD];
#pragma unroll
  for (int d = 0; d < QD; ++d) qreg[d] = qs[qq * QD + d];
  float m = -INFINITY, l = 0.f;
  float acc4[4] = {0.f, 0.f, 0.f, 0.f};          // dims 4g..4g+3 over key slice ks
  const int g4 = tid % G4, ks4 = tid / G4;
  for (int sub = 0; sub < nsub; ++sub) {
    issue(sub + DS_STAGES - 1);                  // its slot was freed at the end of the last stage
    asm volatile("cp.async.wait_group %0;" ::"n"(DS_STAGES - 1) : "memory");
    const int slot = sub % DS_STAGES;
    unsigned char* ks_ = kst + (size_t)slot * stage_bytes;
    unsigned char* vs_ = vst + (size_t)slot * stage_bytes;
    const int base = sub * DS_KEYS;
    const int cnt = min(DS_KEYS, nk - base);
    if (owner && nk - 1 - base >= 0 && nk - 1 - base < DS_KEYS && tid < HD) {
      const int r = nk - 1 - base;
      if (!a.kv_int8) {
        reinterpret_cast<unsigned short*>(ks_)[r * HD + tid] = (unsigned short)k_new;
        reinterpret_cast<unsigned short*>(vs_)[r * HD + tid] = (unsigned short)v_new;
      } else {
        ks_[r * HD + tid] = (unsigned char)k_new;
        vs_[r * HD + tid] = (unsigned char)v_new;
      }
    }
    __syncthreads();   // the stage's rows (and the appended entry) are visible
    // scores: four threads per key (one head_dim quarter each), q in registers
    float sc[DS_KEYS / 32];
#pragma unroll
    for (int ps = 0; ps < DS_KEYS / 32; ++ps) {
      const int j = ps * 32 + (tid >> 2);
      float d0 = 0.f, d1 = 0.f;
      if (j < cnt) {
        if (!a.kv_int8) {
          const uint4* src = reinterpret_cast<const uint4*>(ks_ + (size_t)j * rowb + qq * QD * 2);
#pragma unroll
          for (int c = 0; c < QD / 8; ++c) {
            const uint4 w = src[c];
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
            const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&w.z));
            const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&w.w));
            d0 = fmaf(qreg[c * 8 + 0], f0.x, fmaf(qreg[c * 8 + 1], f0.y, d0));
            d1 = fmaf(qreg[c * 8 + 2], f1.x, fmaf(qreg[c * 8 + 3], f1.y, d1));
            d0 = fmaf(qreg[c * 8 + 4], f2.x, fmaf(qreg[c * 8 + 5], f2.y, d0));
            d1 = fmaf(qreg[c * 8 + 6], f3.x, fmaf(qreg[c * 8 + 7], f3.y, d1));
          }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(ks_ + (size_t)j * rowb + qq * QD);
#pragma unroll
          for (int c = 0; c < QD / 16; ++c) {
            const uint4 w = src[c];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float f[4];
              int8x4_to_float(ww[e], f);
              d0 = fmaf(qreg[c * 16 + 4 * e + 0], f[0], d0);
              d1 = fmaf(qreg[c * 16 + 4 * e + 1], f[1], d1);
              d0 = fmaf(qreg[c * 16 + 4 * e + 2], f[2], d0);
              d1 = fmaf(qreg[c * 16 + 4 * e + 3], f[3], d1);
            }
          }
        }
      }
      float sj = d0 + d1;
      sj += __shfl_xor_sync(0xffffffffu, sj, 1);
      sj += __shfl_xor_sync(0xffffffffu, sj, 2);
      sc[ps] = j < cnt ? (a.kv_int8 ? sj * ksc[base + j] : sj) : -INFINITY;
    }
    // stage max, new running max, weights
    float smax = sc[0];
#pragma unroll
    for (int ps = 1; ps < DS_KEYS / 32; ++ps) smax = fmaxf(smax, sc[ps]);
    smax = warp_max(smax);
    if (lane == 0) red[warp] = smax;
    __syncthreads();
    smax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float m_new = fmaxf(m, smax);
    const float alpha = m == -INFINITY ? 0.f : __expf(m - m_new);
    float psum = 0.f;
#pragma unroll
    for (int ps = 0; ps < DS_KEYS / 32; ++ps) {
      const int j = ps * 32 + (tid >> 2);
      const float pj = j < cnt ? __expf(sc[ps] - m_new) : 0.f;
      if (qq == 0) {
        pw[j] = a.kv_int8 ? pj * (j < cnt ? vsc[base + j] : 0.f) : pj;   // INT8: V scale folded in
        psum += pj;
      }
    }
    psum = warp_sum(psum);
    __syncthreads();   // pw visible; red free again
    if (lane == 0) red[warp] = psum;
    // P V: thread (g4, ks4) takes dims 4*g4 .. 4*g4+3 over keys ks4, ks4 + KS4, ...
    {
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      if (!a.kv_int8) {
        for (int j = ks4; j < cnt; j += KS4) {
          const float w = pw[j];
          const uint2 v = *reinterpret_cast<const uint2*>(vs_ + (size_t)j * rowb + g4 * 8);
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
          s4[0] = fmaf(w, f0.x, s4[0]);
          s4[1] = fmaf(w, f0.y, s4[1]);
          s4[2] = fmaf(w, f1.x, s4[2]);
          s4[3] = fmaf(w, f1.y, s4[3]);
        }
      } else {
        for (int j = ks4; j < cnt; j += KS4) {
          const float w = pw[j];
          float f[4];
          int8x4_to_float(*reinterpret_cast<const uint32_t*>(vs_ + (size_t)j * rowb + g4 * 4), f);
          s4[0] = fmaf(w, f[0], s4[0]);
          s4[1] = fmaf(w, f[1], s4[1]);
          s4[2] = fmaf(w, f[2], s4[2]);
          s4[3] = fmaf(w, f[3], s4[3]);
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) acc4[c] = fmaf(acc4[c], alpha, s4[c]);
    }
    __syncthreads();   // red (sums) visible; the stage slot and pw may be reused
    l = fmaf(l, alpha, (red[0] + red[1]) + (red[2] + red[3]));
    m = m_new;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  // combine the key slices in slice order: dims of slice 0 first, then add
  __shared__ float sl_s[KS4][HD];
#pragma unroll
  for (int c = 0; c < 4; ++c) sl_s[ks4][4 * g4 + c] = acc4[c];
  __syncthreads();
  float acc = 0.f;
  if (tid < HD) {
#pragma unroll
    for (int q = 0; q < KS4; ++q) acc += sl_s[q][tid];
  }
  if (tid < HD) acc_s[0][tid] = acc;
  if (tid == 0) {
    stat_s[0] = nk > 0 ? m : -INFINITY;
    stat_s[1] = nk > 0 ? l : 0.f;
  }
  cl_sync();   // every CTA's statistics and P V are in its shared memory
  if (crank == 0) {
    float M = -INFINITY;
    for (int r = 0; r < CL; ++r) M = fmaxf(M, cl_ld(&stat_s[0], (uint32_t)r));
    for (int e = tid; e < HD; e += 128) {
      float L = 0.f, o = 0.f;
      for (int r = 0; r < CL; ++r) {
        const float mr = cl_ld(&stat_s[0], (uint32_t)r);
        const float w = mr == -INFINITY ? 0.f : __expf(mr - M);
        L = fmaf(cl_ld(&stat_s[1], (uint32_t)r), w, L);
        o = fmaf(cl_ld(&acc_s[0][e], (uint32_t)r), w, o);
      }
      a.out[(size_t)row * a.d + head * HD + e] = __float2half_rn(o / L);
    }
  }
  cl_sync();   // no CTA leaves while rank 0 still reads its shared memory
}

}  // namespace

tl_status launch_attn_prefill(const __half* q, const __half* k, const __half* v, __half* out,
                              int T, int H, int hd, cudaStream_t s) {
  if (T == 0) return ok();
  dim3 grid((T + FQ - 1) / FQ, H);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
  static bool attr_done = false;
  if (!attr_done) {
    TL_CUDA(cudaFuncSetAttribute(attn_prefill_tc_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)attn_prefill_smem<128>()));
    TL_CUDA(cudaFuncSetAttribute(attn_prefill_tc_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)attn_prefill_smem<64>()));
    attr_done = true;
  }
  if (hd == 128)
    TL_LAUNCH_PDL(attn_prefill_tc_kernel<128>, grid, 32 * ATT_WARPS, attn_prefill_smem<128>(), s,
                  q, k, v, out, T, H, scale_log2);
  else if (hd == 64)
    TL_LAUNCH_PDL(attn_prefill_tc_kernel<64>, grid, 32 * ATT_WARPS, attn_prefill_smem<64>(), s,
                  q, k, v, out, T, H, scale_log2);
  else
    return set_error(TL_ERR_UNSUPPORTED, "head_dim %d not supported", hd);
  return ok();
}

// Cluster size and staged rows per CTA of the cluster decode kernel for a
// cache of max_ctx positions; 0 when the staged rows would not fit.
static int decode_cluster_size(int max_ctx) {
  const int c = (max_ctx + 63) / 64;
  return c < 1 ? 1 : c > 8 ? 8 : c;
}
static size_t decode_cluster_smem(int max_ctx, int hd, bool int8, int* max_per) {
  const int cl = decode_cluster_size(max_ctx);
  *max_per = (max_ctx + cl - 1) / cl;
  const size_t rowb = (size_t)hd * (int8 ? 1 : 2);
  return 2 * (size_t)DS_STAGES * DS_KEYS * rowb + 2 * (size_t)*max_per * sizeof(float);
}

tl_status launch_attn_decode_fused(const DecodeAttnArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  if (a.hd != 128 && a.hd != 64)
    return set_error(TL_ERR_UNSUPPORTED, "head_dim %d not supported", a.hd);
  int max_per = 0;
  const size_t smem = decode_cluster_smem(a.max_ctx, a.hd, a.kv_int8 != 0, &max_per);
  if (smem > 200 * 1024)
    return set_error(TL_ERR_UNSUPPORTED, "decode attention: %zu bytes of shared memory", smem);
  static bool attr_done = false;
  if (!attr_done) {
    TL_CUDA(cudaFuncSetAttribute(attn_decode_cluster_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
    TL_CUDA(cudaFuncSetAttribute(attn_decode_cluster_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024));
    attr_done = true;
  }
  const int cl = decode_cluster_size(a.max_ctx);
  dim3 grid(cl, a.H, a.rows);
  cudaError_t e = a.hd == 128
      ? launch_pdl_cluster(attn_decode_cluster_kernel<128>, grid, dim3(128), smem, s, (unsigned)cl, a, cl, max_per)
      : launch_pdl_cluster(attn_decode_cluster_kernel<64>, grid, dim3(128), smem, s, (unsigned)cl, a, cl, max_per);
  if (e != cudaSuccess)
    return set_error(TL_ERR_CUDA, "launch of attn_decode_cluster_kernel failed: %s", cudaGetErrorString(e));
  return ok();
}
}  // namespace tl
