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
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "kv_quant.cuh"
#include "tl_launch.cuh"

namespace tl {
namespace {

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
// Decode attention for one (row, head) on a thread-block cluster.  The lane's
// n_keys = pos + 1 keys are split into CL = min(8, ceil(max_ctx / 64)) chunks
// (fixed per cache) of per = ceil(n_keys / CL) contiguous keys, which depends
// only on the lane's own position; a CTA of the cluster streams F consecutive
// chunks (F chosen at launch, the arithmetic being the same for every F), its
// first cached K/V rows copied into shared memory before the wait for the QKV
// projection.  The CTA holding position pos forms k and v from the QKV
// partial sums, applies RoPE to k and appends both to the cache.  Each chunk
// ends with its max score, exponential sum and unnormalised P V, and rank 0
// merges the chunks in order: either every CTA pushes its chunks into rank 0's
// shared memory (distributed shared-memory stores, one mbarrier arrival per
// CTA) and leaves, or, where the push target's shared memory would cost a wave
// of clusters, rank 0 pulls them between two cluster barriers.  Both merges
// do the same arithmetic.
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
__device__ __forceinline__ uint32_t cl_addr(const void* local, uint32_t rank) {
  uint32_t addr = (uint32_t)__cvta_generic_to_shared(local), remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
  return remote;
}
__device__ __forceinline__ float cl_ld(const float* local, uint32_t rank) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cl_addr(local, rank)) : "memory");
  return v;
}
// a store into the shared memory of CTA `rank` of the cluster
__device__ __forceinline__ void cl_st(float* local, uint32_t rank, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cl_addr(local, rank)), "f"(v) : "memory");
}
// one arrival, with release semantics at cluster scope, on an mbarrier of CTA `rank`
__device__ __forceinline__ void cl_arrive(uint64_t* bar, uint32_t rank) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr(bar, rank))
               : "memory");
}
// bounded wait (2 s of global time) for phase 0 of a local mbarrier whose
// arrivals come from the whole cluster
__device__ __forceinline__ bool cl_wait0(uint64_t* bar) {
  const uint32_t addr = (uint32_t)__cvta_generic_to_shared(bar);
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr)
        : "memory");
    if (done) return true;
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    if (i == 0) t0 = t;
    else if (t - t0 > 2000000000ull) return false;
  }
}

constexpr int DS_KEYS = 64;     // keys per stage of the decode kernel

// ------------------------------------------------------------------ decode (tensor cores)
// Within a CTA both products run on the tensor cores (mma.sync m16n8k16,
// fp16 in, fp32 accumulate) in transposed form, so that the single query fills
// the N = 8 side and keys or head_dim elements fill all 16 rows:
//   S^T = K q^T : A = 16 keys x 16 head_dim elements, B = q (column 0)
//   O^T = V^T P^T : A = 16 head_dim elements x 16 keys, B = p (column 0)
// In each 64-key stage warp w owns keys 16w..16w+15.  FP16 K and V tiles
// come through ldmatrix (V transposed).  INT8 codes become exact fp16 values
// in registers (code + 128 in the low mantissa bits of 1024, minus 1152); a
// lane then reads whole 16-byte chunks of its rows, and the k (or m) index of
// each element follows from where it sits in the chunk, the same order being
// used for q and for the output columns.  The scores of a warp sit in lanes
// 4g (keys g and g + 8); the weights reach the P V B operand through two
// shuffles.  Each warp keeps its own running max and sum (base 2); the four
// warps merge at the end of every chunk, then rank 0 of the cluster merges the
// chunks in order.
constexpr int DT_STAGES_I8 = 3;    // stage ring of the tensor-core decode kernel, INT8 cache
constexpr int DT_STAGES_F16 = 2;   // and FP16 cache (twice the bytes per stage)

template <int HD, bool I8>
struct DecTc {
  static constexpr int KB = HD * (I8 ? 1 : 2);          // bytes of a cached row
  static constexpr int NCH = KB / 64;                   // 16-byte chunks per lane and key
  static constexpr bool VPAD = I8 && HD == 64;          // 64-byte INT8 V rows: padded, not swizzled
  static constexpr int ROWK = KB;                       // K stage row
  static constexpr int ROWV = VPAD ? KB + 16 : KB;      // V stage row
  static constexpr int NST = I8 ? DT_STAGES_I8 : DT_STAGES_F16;
  static constexpr int EPC = I8 ? 4 : 2;                // k steps per chunk
  static constexpr int KSTEP = NCH * EPC;               // = HD / 16
  static constexpr size_t STAGE_BYTES = (size_t)DS_KEYS * (ROWK + ROWV);
  // INT8: chunk of a K row read by quad lane t as its h-th chunk
  __host__ __device__ static constexpr int chunk(int t, int h) {
    return NCH == 1 ? t : 2 * t + (h & 1) + 8 * (h >> 1);
  }
  // Stage rows are stored with their 16-byte chunks permuted (XOR with bits
  // of the row index) so that each quarter-warp's INT8 reads and each
  // ldmatrix's eight rows fall on distinct banks without padding.
  __host__ __device__ static constexpr int kphys(int r, int c) {
    return !I8 ? c ^ (r & 7) : NCH == 1 ? c : c ^ (r & 1);
  }
  __host__ __device__ static constexpr int vphys(int r, int c) {
    return VPAD ? c : I8 ? c ^ (r & 6) : c ^ (r & 7);
  }
};

__device__ __forceinline__ void lds128(uint32_t* w, uint32_t addr) {
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void lds64(uint32_t* w, uint32_t addr) {
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// four int8 codes (bytes 0..3 of w) -> fp16 pairs (0,1) and (2,3), exactly
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  uint32_t x0, x1;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(x0) : "r"(u), "r"(0x64646464u), "r"(0x4140u));
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(x1) : "r"(u), "r"(0x64646464u), "r"(0x4342u));
  const __half2 bias = __float2half2_rn(1152.0f);
  lo = h2_bits(__hsub2(*reinterpret_cast<__half2*>(&x0), bias));
  hi = h2_bits(__hsub2(*reinterpret_cast<__half2*>(&x1), bias));
}

// byte e of wa and byte e of wb (int8 codes) -> an fp16 pair, exactly
template <int E>
__device__ __forceinline__ uint32_t i8pair_to_h2(uint32_t wa, uint32_t wb) {
  uint32_t x, y;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(x) : "r"(wa), "r"(wb), "r"((uint32_t)(E | ((E + 4) << 8))));
  // low byte of each half: code ^ 0x80; high byte: 0x64
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(y) : "r"(x), "r"(0x00FF00FFu), "r"(0x64806480u));
  const __half2 bias = __float2half2_rn(1152.0f);
  return h2_bits(__hsub2(*reinterpret_cast<__half2*>(&y), bias));
}

template <int HD, bool I8>
__global__ void __launch_bounds__(128, I8 ? 4 : 3) attn_decode_tc_kernel(DecodeAttnArgs a, int CL,
                                                                       int F, int sc_len, int push) {
  using T = DecTc<HD, I8>;
  constexpr int HALF = HD / 2;
  constexpr int MT = HD / 16;                    // P V m tiles of 16 head_dim elements
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ float qs[HD], kn[HD], vn[HD];
  __shared__ __align__(16) __half qh[HD];
  __shared__ float wm[4], wl[4];
  __shared__ float kmax_s[4], vmax_s[4];
  __shared__ __align__(8) uint64_t mrg_bar;  // push merge, rank 0: one arrival per CTA of the cluster
  __shared__ int mrg_ok;
  const int crank = blockIdx.x, head = blockIdx.y, row = blockIdx.z;   // crank: rank in the cluster
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  unsigned char* kst = dsm;                                          // [NST][DS_KEYS][ROWK]
  unsigned char* vst = dsm + (size_t)T::NST * DS_KEYS * T::ROWK;     // [NST][DS_KEYS][ROWV]
  __half* ksc = reinterpret_cast<__half*>(dsm + (size_t)T::NST * T::STAGE_BYTES);   // [sc_len]
  __half* vsc = ksc + sc_len;
  float* part = reinterpret_cast<float*>(vsc + sc_len);   // [F][HD + 2]: chunk P V, max, sum
  // push merge: rank 0's [CL][HD + 2] of every chunk's (P V, max, sum)
  float* allp = part + (size_t)F * (HD + 2);
  // This CTA takes chunks crank*F .. crank*F + F - 1 of the CL equal chunks of
  // the lane's context, i.e. the contiguous keys [kA, kB).  Each chunk is
  // streamed in 64-key stages from its own start and folded into its own
  // (P V, max, sum), exactly as if one CTA took each chunk.
  // Launch modes: 0 = append the row's new entry and attend (one decode
  // token per lane); 1 = append only; 2 = attend only, every key (the new one
  // included) read from the cache.  Modes 1 then 2 serve several consecutive
  // tokens of one lane (row_off = 0, 1, ...): every token's entry is in the
  // cache before any token attends, and each row's arithmetic is that of a
  // mode-0 decode step at its position.
  const int lane_id = a.row_lane[row];
  const int pos = a.hdr->pos[lane_id] + a.row_off[row];
  const int n_keys = pos + 1;
  const int per = (n_keys + CL - 1) / CL;
  const int kA = min(crank * F * per, n_keys), kB = min(kA + F * per, n_keys);
  const int nkc = kB - kA;
  const bool owner = a.mode != 2 && nkc > 0 && kB == n_keys;
  if (a.mode == 1 && !owner) return;   // nothing to append here, nothing copied yet
  if (a.mode != 1 && push) {
    // the push merge: rank 0's barrier counts one arrival per CTA; its
    // initialisation is published by the cluster barrier arrival here and
    // awaited before the first remote access at the end
    if (crank == 0 && tid == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(
                       (uint32_t)__cvta_generic_to_shared(&mrg_bar)),
                   "r"(gridDim.x));
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  }
  const int n_old = owner ? nkc - 1 : nkc;       // keys of [kA, kB) already cached
  const int NSF = (per + DS_KEYS - 1) / DS_KEYS; // stages of a full chunk
  const int nstage = nkc / per * NSF + (nkc % per + DS_KEYS - 1) / DS_KEYS;
  char* layer = const_cast<char*>(a.kv_base) + (size_t)(a.row_cum[row] + a.layer) * a.layer_bytes;
  const size_t head_off = (size_t)head * a.max_ctx;
  const size_t scale_region = (a.layer_bytes - 2 * a.kv_region_bytes) / 2;
  // stage `sub` into ring slot sub % NST: cached rows are copied, rows past
  // this CTA's keys zero-filled; the owner's new row is left to the append
  // below (no copy races with it).  Thread tid always copies chunk
  // tid % PIECES of rows tid / PIECES + RPP * p, so its shared-memory offsets
  // (chunk permutation included) are fixed.
  constexpr int PIECES = T::KB / 16, RPP = 128 / PIECES, PASSES = DS_KEYS / RPP;
  const int cr0 = tid / PIECES, cpc = tid % PIECES;
  const uint32_t kdst0 = (uint32_t)__cvta_generic_to_shared(kst) + cr0 * T::ROWK + 16 * T::kphys(cr0, cpc);
  const uint32_t vdst0 = (uint32_t)__cvta_generic_to_shared(vst) + cr0 * T::ROWV + 16 * T::vphys(cr0, cpc);
  const char* ksrc0 = layer + (head_off + kA + cr0) * (size_t)T::KB + 16 * cpc;
  // stage s of the CTA: chunk s / NSF, its keys [lo, lo + cnt) relative to kA
  auto stage_keys = [&](int s, int& lo, int& cnt, int& nkj, int& j) {
    int sub = s;                                 // j = s / NSF, sub = s % NSF (F <= 8 steps)
    j = 0;
    while (sub >= NSF) {
      sub -= NSF;
      ++j;
    }
    nkj = min(per, nkc - j * per);
    lo = j * per + sub * DS_KEYS;
    cnt = min(DS_KEYS, nkj - sub * DS_KEYS);
  };
  auto issue = [&](int s) {
    if (s < nstage) {
      int lo, cnt, nkj, j;
      stage_keys(s, lo, cnt, nkj, j);
      const int slot = s % T::NST;
      const uint32_t kd = kdst0 + slot * (DS_KEYS * T::ROWK);
      const uint32_t vd = vdst0 + slot * (DS_KEYS * T::ROWV);
      const char* ks = ksrc0 + (size_t)lo * T::KB;
      const char* vs = ks + a.kv_region_bytes;
      // the new key (if in this stage) is row cr0 + rnew; row cr0 + RPP*p is
      // cached iff RPP*p < rem
      const int rnew = owner && n_old - lo < cnt ? n_old - lo - cr0 : -DS_KEYS;
      const int rem = min(cnt, n_old - lo) - cr0;
#pragma unroll
      for (int p = 0; p < PASSES; ++p) {
        if (RPP * p == rnew) continue;               // the new key's row
        const bool ok = RPP * p < rem;
        const uint32_t n = ok ? 16 : 0;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(kd + p * RPP * T::ROWK),
                     "l"(ok ? ks + p * RPP * T::KB : layer), "r"(n) : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(vd + p * RPP * T::ROWV),
                     "l"(ok ? vs + p * RPP * T::KB : layer), "r"(n) : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // the first stages are copied before the wait for the previous kernel: they
  // hold entries of earlier steps only -- except in mode 2, where the
  // previous kernel appended some of them, with late_prefetch, where the
  // previous kernels rebuilt them, and in mode 1, which copies nothing
  if (a.mode == 0 && !a.late_prefetch) {
#pragma unroll
    for (int st = 0; st < T::NST - 1; ++st) issue(st);
  }
  pdl_enter();
  if (a.mode == 2 || (a.mode == 0 && a.late_prefetch)) {
#pragma unroll
    for (int st = 0; st < T::NST - 1; ++st) issue(st);
  }

  // the cached keys' scales, the RoPE pair and the QKV partial sums are all
  // requested before any of them is used (one round trip)
  constexpr int SCU = 4;                         // scale loads in flight per thread
  const __half* kq = reinterpret_cast<const __half*>(layer + 2 * a.kv_region_bytes) + head_off + kA;
  const __half* vq = reinterpret_cast<const __half*>(layer + 2 * a.kv_region_bytes + scale_region) +
                     head_off + kA;
  __half ksr[SCU], vsr[SCU];
  if (I8) {
#pragma unroll
    for (int u = 0; u < SCU; ++u) {
      const int j = tid + 128 * u;
      if (j < n_old) {
        ksr[u] = kq[j];
        vsr[u] = vq[j];
      }
    }
  }
  float2 cs = make_float2(1.f, 0.f);
  if (tid < HD) cs = a.rope_cs[(size_t)pos * HALF + (tid % HALF)];
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
  if (I8) {
#pragma unroll
    for (int u = 0; u < SCU; ++u) {
      const int j = tid + 128 * u;
      if (j < n_old) {
        ksc[j] = ksr[u];
        vsc[j] = vsr[u];
      }
    }
    for (int j = tid + 128 * SCU; j < n_old; j += 128) {   // longer contexts
      ksc[j] = kq[j];
      vsc[j] = vq[j];
    }
  }
  for (int i = tid; i < F * (HD + 2); i += 128)   // chunks without keys stay empty
    part[i] = i % (HD + 2) == HD ? -INFINITY : 0.f;
  __syncthreads();
  float kr = 0.f;
  if (tid < HD) {
    float qr;
    if (tid < HALF) {
      qr = qs[tid] * cs.x - qs[tid + HALF] * cs.y;
      kr = kn[tid] * cs.x - kn[tid + HALF] * cs.y;
    } else {
      qr = qs[tid] * cs.x + qs[tid - HALF] * cs.y;
      kr = kn[tid] * cs.x + kn[tid - HALF] * cs.y;
    }
    qh[tid] = __float2half_rn(qr);               // the query in fp16, as in the prefill path
  }
  // owner: the new entry (position pos = key n_old of this CTA) is appended
  // to the cache now and written into its stage row when that stage is read
  uint32_t k_new = 0, v_new = 0;     // fp16 bits or int8 code of element tid
  if (owner) {
    const __half kh = __float2half_rn(kr);
    const __half vh = __float2half_rn(tid < HD ? vn[tid] : 0.f);
    if (!I8) {
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
      if (lane == 0) {
        kmax_s[warp] = km;
        vmax_s[warp] = vm;
      }
      __syncthreads();
      km = fmaxf(fmaxf(kmax_s[0], kmax_s[1]), fmaxf(kmax_s[2], kmax_s[3]));
      vm = fmaxf(fmaxf(vmax_s[0], vmax_s[1]), fmaxf(vmax_s[2], vmax_s[3]));
      const __half ksh = kv_int8_scale(km);
      const __half vsh = kv_int8_scale(vm);
      const float ksf = __half2float(ksh), vsf = __half2float(vsh);
      if (tid < HD) {
        const float kx = __half2float(kh), vx = __half2float(vh);
        const int kc = kv_int8_code(kx, ksf);
        const int vc = kv_int8_code(vx, vsf);
        reinterpret_cast<int8_t*>(layer)[(head_off + pos) * HD + tid] = (int8_t)kc;
        reinterpret_cast<int8_t*>(layer + a.kv_region_bytes)[(head_off + pos) * HD + tid] = (int8_t)vc;
        k_new = (uint32_t)(uint8_t)(int8_t)kc;
        v_new = (uint32_t)(uint8_t)(int8_t)vc;
      }
      if (tid == 0) {
        reinterpret_cast<__half*>(layer + 2 * a.kv_region_bytes)[head_off + pos] = ksh;
        reinterpret_cast<__half*>(layer + 2 * a.kv_region_bytes + scale_region)[head_off + pos] = vsh;
        ksc[n_old] = ksh;
        vsc[n_old] = vsh;
      }
    }
  }
  if (a.mode == 1) return;   // append only: the entry is in the cache
  __syncthreads();   // qh final

  // q as the B operand of S^T (column 0: lanes g == 0).  k step ks covers
  // head_dim elements lo, lo+1 (k indices 2t, 2t+1) and hi, hi+1 (2t+8, 2t+9):
  // FP16: lo = 16ks + 2t, hi = lo + 8 (the ldmatrix order); INT8 (ks = 4h + e):
  // lo = 16 chunk(t, h) + 4e, hi = lo + 2 (four consecutive codes of a word).
  uint32_t qb[T::KSTEP][2];
#pragma unroll
  for (int ks = 0; ks < T::KSTEP; ++ks) {
    const int lo = I8 ? 16 * T::chunk(t, ks / 4) + 4 * (ks % 4) : 16 * ks + 2 * t;
    const int hi = I8 ? lo + 2 : lo + 8;
    qb[ks][0] = g == 0 ? *reinterpret_cast<const uint32_t*>(&qh[lo]) : 0u;
    qb[ks][1] = g == 0 ? *reinterpret_cast<const uint32_t*>(&qh[hi]) : 0u;
  }
  const float csc = rsqrtf((float)HD) * 1.4426950408889634f;   // 1/sqrt(hd) in base 2
  float m = -INFINITY, l = 0.f;
  float o[MT][4];                                // O^T tiles; column 0 (lanes t == 0) is the output
#pragma unroll
  for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int kw = 16 * warp;                      // this warp's first key in a stage
  // slot-0 shared-memory addresses of this lane's reads
  uint32_t k_addr, v_addr;
  int kmask = 0, vmask = 0;
  if constexpr (I8) {
    k_addr = (uint32_t)__cvta_generic_to_shared(kst) + (kw + g) * T::ROWK;   // + chunk, + 8 rows
    v_addr = (uint32_t)__cvta_generic_to_shared(vst) + (kw + 2 * t) * T::ROWV +
             (T::VPAD ? (HD / 8) * g : 16 * T::vphys(2 * t, g));
  } else {
    // ldmatrix rows: K lane l -> key kw + (l & 7) + 8 ((l >> 3) & 1), chunk 2ks + (l >> 4);
    // V lane l -> key kw + (l & 7) + 8 (l >> 4), chunk 2mt + ((l >> 3) & 1)
    k_addr = (uint32_t)__cvta_generic_to_shared(kst) + (kw + (lane & 7) + 8 * ((lane >> 3) & 1)) * T::ROWK;
    v_addr = (uint32_t)__cvta_generic_to_shared(vst) + (kw + (lane & 7) + 8 * (lane >> 4)) * T::ROWV;
    kmask = (lane >> 4) ^ (lane & 7);            // chunk 2ks + (l >> 4) is stored at 2ks ^ kmask
    vmask = ((lane >> 3) & 1) ^ (lane & 7);
  }
  for (int st = 0; st < nstage; ++st) {
    asm volatile("cp.async.wait_group %0;" ::"n"(T::NST - 2) : "memory");
    const int slot = st % T::NST;
    int base, cnt, nkj, jc;
    stage_keys(st, base, cnt, nkj, jc);
    if (owner && n_old >= base && n_old - base < cnt && tid < HD) {
      const int r = n_old - base;
      const int byte = tid * (I8 ? 1 : 2), c = byte >> 4, off = byte & 15;
      unsigned char* kd = kst + (size_t)slot * DS_KEYS * T::ROWK + (size_t)r * T::ROWK + 16 * T::kphys(r, c) + off;
      unsigned char* vd = vst + (size_t)slot * DS_KEYS * T::ROWV + (size_t)r * T::ROWV + 16 * T::vphys(r, c) + off;
      if (!I8) {
        *reinterpret_cast<unsigned short*>(kd) = (unsigned short)k_new;
        *reinterpret_cast<unsigned short*>(vd) = (unsigned short)v_new;
      } else {
        *kd = (unsigned char)k_new;
        *vd = (unsigned char)v_new;
      }
    }
    __syncthreads();   // stage st visible; every warp is done with stage st - 1
    issue(st + T::NST - 1);                      // into the slot of stage st - 1
    if (kw < cnt) {                              // some key of this warp in the stage
      // S^T = K q^T: lane 4g ends with the scores of keys kw + g (s[0]) and kw + g + 8 (s[2])
      float s[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kb_ = k_addr + slot * (DS_KEYS * T::ROWK);
      if constexpr (I8) {
#pragma unroll
        for (int h = 0; h < T::NCH; ++h) {
          const int ph = 16 * T::kphys(g, T::chunk(t, h));   // rows kw+g, kw+g+8: same parity
          uint32_t w0[4], w1[4];
          lds128(w0, kb_ + ph);
          lds128(w1, kb_ + 8 * T::ROWK + ph);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t af[4];
            i8x4_to_h2x2(w0[e], af[0], af[2]);
            i8x4_to_h2x2(w1[e], af[1], af[3]);
            mma_f16(s, af, qb[4 * h + e][0], qb[4 * h + e][1]);
          }
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < T::KSTEP; ++ks) {
          uint32_t af[4];
          ldsm_x4(af, kb_ + 16 * ((2 * ks) ^ kmask));
          mma_f16(s, af, qb[ks][0], qb[ks][1]);
        }
      }
      // online softmax over the warp's 16 keys (lanes t == 0)
      float ks0 = 1.f, ks1 = 1.f, vs0 = 1.f, vs1 = 1.f;
      if constexpr (I8) {   // the scale arrays are padded to whole stages: no bound check
        ks0 = __half2float(ksc[base + kw + g]);
        ks1 = __half2float(ksc[base + kw + g + 8]);
        vs0 = __half2float(vsc[base + kw + g]);
        vs1 = __half2float(vsc[base + kw + g + 8]);
      }
      const bool v0 = t == 0 && kw + g < cnt, v1 = t == 0 && kw + g + 8 < cnt;
      const float x0 = v0 ? s[0] * csc * ks0 : -INFINITY;
      const float x1 = v1 ? s[2] * csc * ks1 : -INFINITY;
      float mx = fmaxf(x0, x1);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m, mx);
      const float alpha = m == -INFINITY ? 0.f : exp2f(m - m_new);
      const float p0 = v0 ? exp2f(x0 - m_new) : 0.f;
      const float p1 = v1 ? exp2f(x1 - m_new) : 0.f;
      l = fmaf(l, alpha, p0 + p1);
      if (__any_sync(0xffffffffu, m_new != m)) {
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          o[i][0] *= alpha;
          o[i][2] *= alpha;
        }
      }
      m = m_new;
      // P^T as the B operand (column 0: lanes g == 0 hold keys 2t, 2t+1 | 2t+8, 2t+9)
      // (the scales past the stage's keys are stale: select, do not multiply)
      const uint32_t hp = pack_half2(I8 ? (v0 ? p0 * vs0 : 0.f) : p0, I8 ? (v1 ? p1 * vs1 : 0.f) : p1);   // keys g | g + 8
      const uint32_t pu = __shfl_sync(0xffffffffu, hp, 8 * t);       // keys 2t | 2t + 8
      const uint32_t pv = __shfl_sync(0xffffffffu, hp, 8 * t + 4);   // keys 2t + 1 | 2t + 9
      uint32_t pb0, pb1;
      asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(pb0) : "r"(pu), "r"(pv));
      asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(pb1) : "r"(pu), "r"(pv));
      if (g != 0) pb0 = pb1 = 0u;
      // O^T += V^T P^T
      const uint32_t vb = v_addr + slot * (DS_KEYS * T::ROWV);
      if constexpr (!I8) {
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          uint32_t af[4];
          ldsm_x4_trans(af, vb + 16 * ((2 * i) ^ vmask));
          mma_f16(o[i], af, pb0, pb1);
        }
      } else {
        constexpr int NW = HD / 32;                // words of a V row per lane
        uint32_t ra[4], rb[4], rc[4], rd[4];
        if constexpr (NW == 4) {
          lds128(ra, vb);
          lds128(rb, vb + T::ROWV);
          lds128(rc, vb + 8 * T::ROWV);
          lds128(rd, vb + 9 * T::ROWV);
        } else {
          lds64(ra, vb);
          lds64(rb, vb + T::ROWV);
          lds64(rc, vb + 8 * T::ROWV);
          lds64(rd, vb + 9 * T::ROWV);
        }
        // tile i, row g + 8h <-> byte 2i + h of the lane's chunk
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          const int w = i >> 1;
          uint32_t af[4];
          if (i & 1) {
            af[0] = i8pair_to_h2<2>(ra[w], rb[w]);
            af[1] = i8pair_to_h2<3>(ra[w], rb[w]);
            af[2] = i8pair_to_h2<2>(rc[w], rd[w]);
            af[3] = i8pair_to_h2<3>(rc[w], rd[w]);
          } else {
            af[0] = i8pair_to_h2<0>(ra[w], rb[w]);
            af[1] = i8pair_to_h2<1>(ra[w], rb[w]);
            af[2] = i8pair_to_h2<0>(rc[w], rd[w]);
            af[3] = i8pair_to_h2<1>(rc[w], rd[w]);
          }
          mma_f16(o[i], af, pb0, pb1);
        }
      }
    }
    if (base + cnt - jc * per == nkj) {
      // last stage of chunk jc: the four warps' states are merged, in
      // warp order, into the chunk's (P V, max, sum); the stage's K slot is
      // free until the next iteration's barrier and holds the warp states
      __syncthreads();
      float (*wo)[HD] = reinterpret_cast<float (*)[HD]>(kst + (size_t)slot * DS_KEYS * T::ROWK);
      float lw = l;
      lw += __shfl_xor_sync(0xffffffffu, lw, 4);
      lw += __shfl_xor_sync(0xffffffffu, lw, 8);
      lw += __shfl_xor_sync(0xffffffffu, lw, 16);
      if (t == 0) {
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          const int d0 = I8 ? (HD / 8) * g + 2 * i : 16 * i + g;   // output row g of tile i
          const int d1 = I8 ? d0 + 1 : d0 + 8;                     // and row g + 8
          wo[warp][d0] = o[i][0];
          wo[warp][d1] = o[i][2];
        }
        if (g == 0) {
          wm[warp] = m;
          wl[warp] = lw;
        }
      }
      __syncthreads();
      if (tid < HD) {
        const float M = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
        float acc = 0.f, L = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float wt = wm[w] == -INFINITY ? 0.f : exp2f(wm[w] - M);
          acc = fmaf(wo[w][tid], wt, acc);
          L = fmaf(wl[w], wt, L);
        }
        float* pj = part + jc * (HD + 2);
        pj[tid] = acc;
        if (tid == 0) {
          pj[HD] = M;
          pj[HD + 1] = L;
        }
      }
      m = -INFINITY;
      l = 0.f;
#pragma unroll
      for (int i = 0; i < MT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  if (push) {
    __syncthreads();   // this CTA's chunk results are complete
    // push them into rank 0 (chunk c = crank * F + j goes to its slot c), then
    // one arrival; every CTA but rank 0 is done after that
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");   // rank 0's barrier is set up
    for (int j = 0; j < F; ++j) {
      const int c = crank * F + j;
      if (c < CL)
        for (int i = tid; i < HD + 2; i += 128)
          cl_st(allp + (size_t)c * (HD + 2) + i, 0u, part[j * (HD + 2) + i]);
    }
    __syncthreads();
    if (tid == 0) cl_arrive(&mrg_bar, 0u);
    if (crank != 0) return;
    if (tid == 0) mrg_ok = cl_wait0(&mrg_bar) ? 1 : 0;
    __syncthreads();
    if (!mrg_ok) {
      if (tid == 0 && a.status) atomicCAS(a.status, 0, (int)TL_ERR_TIMEOUT);
      return;
    }
    if (tid < HD) {
      // the chunks merged in order from rank 0's own shared memory
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c < CL) M = fmaxf(M, allp[c * (HD + 2) + HD]);
      float L = 0.f, acc = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c < CL) {
          const float mc = allp[c * (HD + 2) + HD];
          const float w = mc == -INFINITY ? 0.f : exp2f(mc - M);
          L = fmaf(allp[c * (HD + 2) + HD + 1], w, L);
          acc = fmaf(allp[c * (HD + 2) + tid], w, acc);
        }
      }
      a.out[(size_t)row * a.d + head * HD + tid] = __float2half_rn(acc / L);
    }
    return;
  }
  cl_sync();   // every CTA's chunk results are in its shared memory
  if (crank == 0 && tid < HD) {
    // pull merge: chunk c sits in CTA c / F, slot c % F; all remote reads are
    // issued before any is used, then the chunks are merged in order (the same
    // arithmetic as the push merge)
    float mr[8], lr[8], ar[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < CL) {
        const float* pc = part + (c % F) * (HD + 2);
        mr[c] = cl_ld(pc + HD, (uint32_t)(c / F));
        lr[c] = cl_ld(pc + HD + 1, (uint32_t)(c / F));
        ar[c] = cl_ld(pc + tid, (uint32_t)(c / F));
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < CL) M = fmaxf(M, mr[c]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < CL) {
        const float w = mr[c] == -INFINITY ? 0.f : exp2f(mr[c] - M);
        L = fmaf(lr[c], w, L);
        acc = fmaf(ar[c], w, acc);
      }
    }
    a.out[(size_t)row * a.d + head * HD + tid] = __float2half_rn(acc / L);
  }
  cl_sync();   // no CTA leaves while rank 0 still reads its shared memory
}

}  // namespace

tl_status launch_attn_prefill(const __half* q, const __half* k, const __half* v, __half* out,
                              int T, int H, int hd, cudaStream_t s) {
  if (T == 0) return ok();
  dim3 grid((T + FQ - 1) / FQ, H);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
  static std::atomic<uint64_t> attr_done{0};
  TL_TRY(once_per_device(attr_done, []() -> tl_status {
    TL_CUDA(cudaFuncSetAttribute(attn_prefill_tc_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)attn_prefill_smem<128>()));
    TL_CUDA(cudaFuncSetAttribute(attn_prefill_tc_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)attn_prefill_smem<64>()));
    return ok();
  }));
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

// Chunks of the decode split for a cache of max_ctx positions: ceil(max_ctx /
// 64) capped at 8.  It depends on the cache alone, so a lane's arithmetic does
// not depend on the batch; how many chunks one CTA takes (below) does not
// change that arithmetic.
static int decode_cluster_size(int max_ctx) {
  const int c = (max_ctx + 63) / 64;
  return c < 1 ? 1 : c > 8 ? 8 : c;
}
template <int HD, bool I8>
static size_t decode_tc_smem(int sc_len, int F, int push_cl) {
  return (size_t)DecTc<HD, I8>::NST * DecTc<HD, I8>::STAGE_BYTES +
         2 * (size_t)sc_len * sizeof(__half) + (size_t)(F + push_cl) * (HD + 2) * sizeof(float);
}
constexpr size_t kDecodeSmemCap = 200 * 1024;

// Clusters of `pc` CTAs of the decode kernel that fit on the GPU at once.
template <int HD, bool I8>
static int decode_active_clusters(int pc, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, size_t>, int> cache;   // (device, pc, smem)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = -1;
  }
  const auto key = std::make_tuple(dev, pc, smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pc, 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pc;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)attn_decode_tc_kernel<HD, I8>, &cfg) !=
          cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    n = 1;
  }
  cache[key] = n;
  return n;
}

template <int HD, bool I8>
static tl_status launch_decode_tc(const DecodeAttnArgs& a, cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  TL_TRY(once_per_device(attr_done, []() -> tl_status {
    TL_CUDA(cudaFuncSetAttribute(attn_decode_tc_kernel<HD, I8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecodeSmemCap));
    return ok();
  }));
  const int cl = decode_cluster_size(a.max_ctx);
  const int max_per = (a.max_ctx + cl - 1) / cl;   // keys of a chunk at most
  // chunks per CTA: the fewest that run every (row, head) cluster in the
  // fewest waves
  // fewest waves; on a tie the push merge (its rank 0 holds every chunk's
  // record: more shared memory per CTA, one cluster barrier instead of two)
  int best_f = 0, best_waves = 0, best_push = 0;
  size_t best_smem = 0;
  int best_sc = 0;
  for (int f = a.chunks > 0 ? std::min(a.chunks, cl) : 1; f <= cl; f *= 2) {
    const int sc_len = I8 ? (f * max_per + DS_KEYS + 7) / 8 * 8 : 0;   // a stage past the last key
    for (int push = 1; push >= 0; --push) {
      const size_t smem = decode_tc_smem<HD, I8>(sc_len, f, push ? cl : 0);
      if (smem > kDecodeSmemCap) continue;
      const int pc = (cl + f - 1) / f;
      const int active = decode_active_clusters<HD, I8>(pc, smem);
      const int waves = (a.rows * a.H + active - 1) / active;
      if (best_f == 0 || waves < best_waves) {
        best_f = f;
        best_waves = waves;
        best_smem = smem;
        best_sc = sc_len;
        best_push = push;
      }
    }
    if (a.chunks > 0) break;   // fixed by the caller
  }
  if (best_f == 0)
    return set_error(TL_ERR_UNSUPPORTED, "decode attention: a cache of %d positions needs too much shared memory",
                     a.max_ctx);
  const int pc = (cl + best_f - 1) / best_f;
  dim3 grid(pc, a.H, a.rows);
  const cudaError_t e = launch_pdl_cluster(attn_decode_tc_kernel<HD, I8>, grid, dim3(128), best_smem, s,
                                           (unsigned)pc, a, cl, best_f, best_sc, best_push);
  if (e != cudaSuccess)
    return set_error(TL_ERR_CUDA, "launch of attn_decode_tc_kernel failed: %s", cudaGetErrorString(e));
  return ok();
}

tl_status launch_attn_decode_fused(const DecodeAttnArgs& a, cudaStream_t s) {
  if (a.rows == 0) return ok();
  if (a.rows > kMaxLanes) return set_error(TL_ERR_INVALID_ARG, "decode attention: %d rows", a.rows);
  const bool i8 = a.kv_int8 != 0;
  if (a.hd == 128) return i8 ? launch_decode_tc<128, true>(a, s) : launch_decode_tc<128, false>(a, s);
  if (a.hd == 64) return i8 ? launch_decode_tc<64, true>(a, s) : launch_decode_tc<64, false>(a, s);
  return set_error(TL_ERR_UNSUPPORTED, "head_dim %d not supported", a.hd);
}
}  // namespace tl
