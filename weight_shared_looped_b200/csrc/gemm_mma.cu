// Quantised-weight GEMM for small token counts (decode lanes, short prompts):
//   part[z][t][n] = sum over k in split z of x[t][k] * W[n][k],
//   W[n][k] = code[n][k] * scale[n][k / G]   (group-wise symmetric INT4).
//
// Weights are the A operand of mma.sync m16n8k16 (16 output features x 16 k),
// tokens the B operand (8 per n-tile).  Each thread dequantises its A-fragment
// elements straight from the packed words into exact fp16 integers (no shared
// memory round trip):
//   byte t of a word holds the codes of k = 2t and 2t+1 (low, high nibble);
//   prmt copies that byte to bytes 0 and 2, a lop3 keeps the low nibble in the
//   low half and the high nibble at bits 20..23 and ORs in the fp16 exponent of
//   1024, and one HFMA2 with (1, 1/16) and (-1032, -72) leaves the two codes
//   as exact fp16 values.
// The fp32 tensor-core sums of each 64-wide k chunk (one chunk never crosses a
// group since G is 64 or 128) are multiplied by the group scale in fp32 and
// added to the running total, so the only rounding besides fp32 accumulation
// is the fp16 rounding of the activations.
//
// Each output column (token) is computed independently of the others and the
// split count depends only on (N, K, T-class), so a token's result does not
// depend on which other tokens share the launch.
#include "tl_launch.cuh"

namespace tl {
namespace {

constexpr int KC = 64;         // k per chunk
constexpr int ROWS_CTA = 64;   // 4 warps x 16 rows
constexpr int THREADS = 128;

__device__ __forceinline__ uint32_t dequant_pair(uint32_t w, uint32_t sel) {
  uint32_t x, h;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(x) : "r"(w), "r"(0u), "r"(sel));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(x), "r"(0x00F0000Fu), "r"(0x64006400u));
  const __half2 mul = __halves2half2(__float2half_rn(1.0f), __float2half_rn(0.0625f));
  const __half2 add = __halves2half2(__float2half_rn(-1032.0f), __float2half_rn(-72.0f));
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&h), mul, add);
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int NT>
__global__ void __launch_bounds__(THREADS) gemm_w4_mma_kernel(GemmArgs a) {
  pdl_enter();
  __shared__ __align__(16) __half xs[NT][KC + 8];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rowA = blockIdx.x * ROWS_CTA + warp * 16 + g;   // and rowA + 8
  const int tok0 = blockIdx.y * NT;
  const int n_chunks = a.K / KC;
  const int per_split = n_chunks / a.splits;
  const int c_begin = blockIdx.z * per_split;
  const int c_end = c_begin + per_split;
  const int wpr = a.K / 8;
  const int gsh = __ffs(a.G) - 1;             // the group size is 64 or 128
  const int gpr = a.K >> gsh;

  const uint32_t* wr[2];
  const __half* sr[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int row = rowA + 8 * r;
    if (row < a.n_split) {
      wr[r] = a.w0 + (size_t)row * wpr;
      sr[r] = a.s0 + (size_t)row * gpr;
    } else {
      wr[r] = a.w1 + (size_t)(row - a.n_split) * wpr;
      sr[r] = a.s1 + (size_t)(row - a.n_split) * gpr;
    }
  }
  const uint32_t sel = (uint32_t)t | 0x40u | ((uint32_t)t << 8) | 0x4000u;

  float acc[NT / 8][4];
#pragma unroll
  for (int i = 0; i < NT / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  uint4 nxt[2][2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const uint4* p = reinterpret_cast<const uint4*>(wr[r] + c_begin * 8);
    nxt[r][0] = __ldg(p);
    nxt[r][1] = __ldg(p + 1);
  }

  for (int c = c_begin; c < c_end; ++c) {
    __syncthreads();
    for (int i = threadIdx.x; i < NT * (KC / 8); i += THREADS) {
      int tr = i / (KC / 8), col = (i % (KC / 8)) * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (tok0 + tr < a.T)
        v = *reinterpret_cast<const uint4*>(a.x + (size_t)(tok0 + tr) * a.K + c * KC + col);
      *reinterpret_cast<uint4*>(&xs[tr][col]) = v;
    }
    uint4 cur[2][2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      cur[r][0] = nxt[r][0];
      cur[r][1] = nxt[r][1];
    }
    if (c + 1 < c_end) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint4* p = reinterpret_cast<const uint4*>(wr[r] + (c + 1) * 8);
        nxt[r][0] = __ldg(p);
        nxt[r][1] = __ldg(p + 1);
      }
    }
    const float s0 = __half2float(sr[0][(c * KC) >> gsh]);
    const float s1 = __half2float(sr[1][(c * KC) >> gsh]);
    __syncthreads();

    float cacc[NT / 8][4];
#pragma unroll
    for (int i = 0; i < NT / 8; ++i) cacc[i][0] = cacc[i][1] = cacc[i][2] = cacc[i][3] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&cur[0][j >> 1]);
      const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&cur[1][j >> 1]);
      const int wi = (j & 1) * 2;   // words 2j, 2j+1 of the chunk
      uint32_t A[4];
      A[0] = dequant_pair(w0[wi], sel);       // row g,   k = 16j + 2t, +1
      A[1] = dequant_pair(w1[wi], sel);       // row g+8
      A[2] = dequant_pair(w0[wi + 1], sel);   // row g,   k = 16j + 8 + 2t, +1
      A[3] = dequant_pair(w1[wi + 1], sel);   // row g+8
#pragma unroll
      for (int nt = 0; nt < NT / 8; ++nt) {
        uint32_t b0 = *reinterpret_cast<const uint32_t*>(&xs[nt * 8 + g][16 * j + 2 * t]);
        uint32_t b1 = *reinterpret_cast<const uint32_t*>(&xs[nt * 8 + g][16 * j + 2 * t + 8]);
        mma16816(cacc[nt], A, b0, b1);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT / 8; ++nt) {
      acc[nt][0] = fmaf(cacc[nt][0], s0, acc[nt][0]);
      acc[nt][1] = fmaf(cacc[nt][1], s0, acc[nt][1]);
      acc[nt][2] = fmaf(cacc[nt][2], s1, acc[nt][2]);
      acc[nt][3] = fmaf(cacc[nt][3], s1, acc[nt][3]);
    }
  }

  float* out = a.part + (size_t)blockIdx.z * a.T * a.N;
#pragma unroll
  for (int nt = 0; nt < NT / 8; ++nt) {
    int tk = tok0 + nt * 8 + 2 * t;
    if (tk < a.T) {
      out[(size_t)tk * a.N + rowA] = acc[nt][0];
      out[(size_t)tk * a.N + rowA + 8] = acc[nt][2];
    }
    if (tk + 1 < a.T) {
      out[(size_t)(tk + 1) * a.N + rowA] = acc[nt][1];
      out[(size_t)(tk + 1) * a.N + rowA + 8] = acc[nt][3];
    }
  }
}

// ---------------------------------------------------------------- decode GEMV
// T <= 8 tokens.  The k order inside the MMA is a free choice as long as A and
// B use the same one, so each lane owns two whole packed words (16 k) of its
// two rows per 64-wide chunk: lane (g, t) loads words 2t and 2t+1 of rows g
// and g+8 (8 distinct bytes each, no duplicate loads).  A word's nibble pairs
// (i, i+4) come out of one lop3 each: w & 0x000F000F | 0x6400_6400 is the fp16
// pair (1024 + u_0, 1024 + u_4), less 1032 the exact codes; w & 0x00F000F0 |
// 0x6400_6400 is (1024 + 16 u_1, 1024 + 16 u_5), and one HFMA2 (x / 16 - 72)
// gives those codes exactly; w >> 8 yields pairs (2, 6) and (3, 7) the same
// way (one shift per word).  The activations are staged once per CTA with
// every 8-k group stored in the order 0 4 1 5 2 6 3 7, so the matching B pairs
// are adjacent and one 8-byte shared load feeds a k step.
constexpr int GV_ROWS = 128;      // 8 warps x 16 rows
constexpr int GV_THREADS = 256;
constexpr int GV_BATCH = 8;       // 64-k chunks loaded ahead per batch

__device__ __forceinline__ uint32_t nib_pair(uint32_t w) {   // nibbles 0 and 4
  uint32_t h;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&h),
                      __halves2half2(__float2half_rn(1032.0f), __float2half_rn(1032.0f)));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t nib_pair_hi(uint32_t w) {   // nibbles 1 and 5
  uint32_t h;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(w), "r"(0x00F000F0u), "r"(0x64006400u));
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&h),
                      __halves2half2(__float2half_rn(0.0625f), __float2half_rn(0.0625f)),
                      __halves2half2(__float2half_rn(-72.0f), __float2half_rn(-72.0f)));
  return *reinterpret_cast<uint32_t*>(&r);
}

__global__ void __launch_bounds__(GV_THREADS) gemv_w4_kernel(GemmArgs a) {
  extern __shared__ __align__(16) __half gv_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m0 = blockIdx.x * GV_ROWS;
  const int n_chunks = a.K / KC;
  const int per = n_chunks / a.splits;
  const int c0 = blockIdx.z * per;
  const int krange = per * KC;
  const int xstride = krange + 4;             // halves; row stride = 2 (mod 32) words
  __half* xs = gv_smem;                       // [8][xstride], k-permuted
  const int gsh = __ffs(a.G) - 1;            // the group size is 64 or 128
  const int gpr = a.K >> gsh;
  const int g_lo = (c0 * KC) >> gsh;
  const int n_groups = ((krange + a.G - 1) >> gsh) + 1;
  __half* ss = xs + 8 * xstride;              // [128][n_groups] scales of this CTA

  // Weights and scales are constants of the model: stage the scales and issue
  // the first batch of weight loads before waiting for the previous kernel, so
  // their latency overlaps its tail.  (Loops are laid out so that no index
  // needs an integer division.)
  constexpr int SROWS = GV_ROWS / (GV_THREADS / 32);   // rows per warp
  for (int g0 = 0; g0 < n_groups; g0 += 32) {
    const int gg = g0 + lane;
    __half sv[SROWS];
#pragma unroll
    for (int k = 0; k < SROWS; ++k) {       // all loads in flight before any store
      const int row = m0 + warp + k * (GV_THREADS / 32);
      const __half* sp = row < a.n_split ? a.s0 + (size_t)row * gpr
                                         : a.s1 + (size_t)(row - a.n_split) * gpr;
      sv[k] = gg < n_groups && g_lo + gg < gpr ? sp[g_lo + gg] : __float2half_rn(0.f);
    }
#pragma unroll
    for (int k = 0; k < SROWS; ++k)
      if (gg < n_groups) ss[(warp + k * (GV_THREADS / 32)) * n_groups + gg] = sv[k];
  }
  const int rowA = m0 + warp * 16 + g;
  const uint2* wr[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = rowA + 8 * r;
    const uint32_t* base = row < a.n_split ? a.w0 + (size_t)row * (a.K / 8)
                                           : a.w1 + (size_t)(row - a.n_split) * (a.K / 8);
    wr[r] = reinterpret_cast<const uint2*>(base + c0 * 8) + t;   // words 2t, 2t+1 of chunk 0
  }
  uint2 cur[GV_BATCH][2], nxt[GV_BATCH][2];
#pragma unroll
  for (int b = 0; b < GV_BATCH; ++b) {
    const bool in = b < per;
    nxt[b][0] = in ? __ldg(wr[0] + b * 4) : make_uint2(0u, 0u);
    nxt[b][1] = in ? __ldg(wr[1] + b * 4) : make_uint2(0u, 0u);
  }
  pdl_enter();   // the activations below come from the previous kernel

  // stage x (rows >= T are zero), permuting each 8-k group to 0 4 1 5 2 6 3 7;
  // item i is token row i / Q, 8-k group i % Q
  const int Q = krange / 8, n_items = 8 * Q;
  const int qsh = (Q & (Q - 1)) == 0 ? __ffs(Q) - 1 : -1;
  auto item = [&](int i, int& r, int& q) {
    if (qsh >= 0) {
      r = i >> qsh;
      q = i & (Q - 1);
    } else {
      r = i / Q;
      q = i - r * Q;
    }
  };
  auto put = [&](int r, int q, uint4 v) {
    const __half* e = reinterpret_cast<const __half*>(&v);
    __half2 p0 = __halves2half2(e[0], e[4]), p1 = __halves2half2(e[1], e[5]);
    __half2 p2 = __halves2half2(e[2], e[6]), p3 = __halves2half2(e[3], e[7]);
    uint2* d = reinterpret_cast<uint2*>(xs + r * xstride + q * 8);   // 8-byte aligned
    d[0] = make_uint2(*reinterpret_cast<uint32_t*>(&p0), *reinterpret_cast<uint32_t*>(&p1));
    d[1] = make_uint2(*reinterpret_cast<uint32_t*>(&p2), *reinterpret_cast<uint32_t*>(&p3));
  };
  if (a.x_part) {
    for (int i = threadIdx.x; i < n_items; i += GV_THREADS) {
      int r, q;
      item(i, r, q);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < a.T) {
        // SwiGLU of the gate|up partial sums, rounded to fp16 like the unfused path
        __half hv[8];
        const size_t stride = (size_t)a.T * 2 * a.x_F;
        for (int e = 0; e < 8; ++e) {
          const size_t kk = (size_t)c0 * KC + q * 8 + e;
          float gs = 0.f, us = 0.f;
          for (int sp = 0; sp < a.x_S; ++sp) {
            const float* p = a.x_part + sp * stride + (size_t)r * 2 * a.x_F;
            gs += p[kk];
            us += p[a.x_F + kk];
          }
          hv[e] = __float2half_rn(gs / (1.0f + __expf(-gs)) * us);
        }
        v = *reinterpret_cast<const uint4*>(hv);
      }
      put(r, q, v);
    }
  } else {
    // four items per thread at a time, all loads in flight before any store
    for (int i0 = threadIdx.x; i0 < n_items; i0 += 4 * GV_THREADS) {
      uint4 v[4];
      int rr[4], qq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * GV_THREADS;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        rr[u] = 0;
        qq[u] = 0;
        if (i < n_items) {
          item(i, rr[u], qq[u]);
          if (rr[u] < a.T)
            v[u] = *reinterpret_cast<const uint4*>(a.x + (size_t)rr[u] * a.K + c0 * KC + qq[u] * 8);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + u * GV_THREADS < n_items) put(rr[u], qq[u], v[u]);
    }
  }
  const __half* srow0 = ss + (warp * 16 + g) * n_groups;
  const __half* srow1 = srow0 + 8 * n_groups;
  __syncthreads();

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int cb = 0; cb < per; cb += GV_BATCH) {
#pragma unroll
    for (int b = 0; b < GV_BATCH; ++b) {
      cur[b][0] = nxt[b][0];
      cur[b][1] = nxt[b][1];
    }
#pragma unroll
    for (int b = 0; b < GV_BATCH; ++b) {
      const int c = cb + GV_BATCH + b;
      const bool in = c < per;
      nxt[b][0] = in ? __ldg(wr[0] + c * 4) : make_uint2(0u, 0u);
      nxt[b][1] = in ? __ldg(wr[1] + c * 4) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int b = 0; b < GV_BATCH; ++b) {
      const int c = cb + b;
      if (c >= per) break;
      float cacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t w0 = (j < 2) ? cur[b][0].x : cur[b][0].y;   // row g
        const uint32_t w1 = (j < 2) ? cur[b][1].x : cur[b][1].y;   // row g + 8
        const int sh = (j & 1) * 8;                                  // nibble pairs 0,1 or 2,3
        uint32_t A[4];
        A[0] = nib_pair(w0 >> sh);
        A[1] = nib_pair(w1 >> sh);
        A[2] = nib_pair_hi(w0 >> sh);
        A[3] = nib_pair_hi(w1 >> sh);
        const uint2 bx =
            *reinterpret_cast<const uint2*>(xs + g * xstride + c * KC + 16 * t + 4 * j);
        mma16816(cacc, A, bx.x, bx.y);
      }
      const int sidx = (((c0 + c) * KC) >> gsh) - g_lo;
      const float s0 = __half2float(srow0[sidx]);
      const float s1 = __half2float(srow1[sidx]);
      acc[0] = fmaf(cacc[0], s0, acc[0]);
      acc[1] = fmaf(cacc[1], s0, acc[1]);
      acc[2] = fmaf(cacc[2], s1, acc[2]);
      acc[3] = fmaf(cacc[3], s1, acc[3]);
    }
  }
  float* out = a.part + (size_t)blockIdx.z * a.T * a.N;
  const int tk = 2 * t;
  if (tk < a.T) {
    out[(size_t)tk * a.N + rowA] = acc[0];
    out[(size_t)tk * a.N + rowA + 8] = acc[2];
  }
  if (tk + 1 < a.T) {
    out[(size_t)(tk + 1) * a.N + rowA] = acc[1];
    out[(size_t)(tk + 1) * a.N + rowA + 8] = acc[3];
  }
}

__global__ void split_sum_kernel(const float* __restrict__ part, int S, long n,
                                 float* __restrict__ y) {
  pdl_enter();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = part[i];
  for (int s = 1; s < S; ++s) acc += part[(long)s * n + i];
  y[i] = acc;
}

int token_tile(int T) { return T <= 8 ? 8 : T <= 16 ? 16 : T <= 32 ? 32 : 64; }

}  // namespace

// Split-K factor: a power of two that keeps every split a whole number of
// 64-wide chunks and gives at least two CTAs per SM.  Decode-sized calls
// (T <= 8) always use the T <= 8 branch, so a lane's reduction order does not
// depend on how many lanes are active.
int gemm_mma_splits(int N, int K, int T) {
  int n_chunks = K / KC;
  int tiles = (N / ROWS_CTA) * ((T + token_tile(T) - 1) / token_tile(T));
  int s = 1;
  while (tiles * s < 2 * 148 && s * 2 <= 16 && n_chunks % (s * 2) == 0 && n_chunks / (s * 2) >= 2)
    s *= 2;
  return s;
}

tl_status launch_split_sum(const float* part, int S, long n, float* y, cudaStream_t s) {
  if (n == 0) return ok();
  TL_LAUNCH_PDL(split_sum_kernel, (unsigned)((n + 255) / 256), 256, 0, s, part, S, n, y);
  return ok();
}

bool gemv_eligible(int N, int K, int T) { return T <= 8 && N % GV_ROWS == 0 && K % KC == 0; }

// Decode split count: each split covers at most 2048 k (the staged activations
// then fit in 33 KB of shared memory) and at least 4 chunks; splits double
// while the grid still fits one wave of two CTAs per SM.  Depends on (N, K)
// only.
int gemv_splits(int N, int K) {
  const int n_chunks = K / KC;
  int s = 1;
  while (n_chunks / s > 32 && n_chunks % (2 * s) == 0) s *= 2;
  while ((N / GV_ROWS) * 2 * s <= 2 * 148 && n_chunks % (2 * s) == 0 && n_chunks / (2 * s) >= 4)
    s *= 2;
  return s;
}

int gemm_splits(int N, int K, int T) {
  if (gemv_eligible(N, K, T)) return gemv_splits(N, K);
  return gemm_tc_eligible(N, K, T) ? gemm_tc_splits(N, K, T) : gemm_mma_splits(N, K, T);
}

tl_status launch_gemv(const GemmArgs& a, cudaStream_t s) {
  if (a.T == 0) return ok();
  const int per = (a.K / KC) / a.splits;
  const int krange = per * KC;
  const int n_groups = (krange + a.G - 1) / a.G + 1;
  const size_t smem = (size_t)8 * (krange + 4) * 2 + (size_t)GV_ROWS * n_groups * 2;
  if (smem > 48 * 1024) return set_error(TL_ERR_UNSUPPORTED, "decode GEMV split too wide");
  dim3 grid(a.N / GV_ROWS, 1, a.splits);
  TL_LAUNCH_PDL(gemv_w4_kernel, grid, GV_THREADS, smem, s, a);
  return ok();
}

tl_status launch_gemm(const GemmArgs& a, cudaStream_t s) {
  if (a.swiglu_u) {
    if (!gemm_tc_eligible(a.N, a.K, a.T) || a.splits != 1 || a.N != 2 * a.n_split ||
        a.n_split % 64 != 0 || a.x_part)
      return set_error(TL_ERR_UNSUPPORTED,
                       "the fused SwiGLU epilogue needs the one-split tensor-core GEMM");
    return launch_gemm_tc(a, s);
  }
  if (gemv_eligible(a.N, a.K, a.T)) return launch_gemv(a, s);
  if (a.x_part)
    return set_error(TL_ERR_UNSUPPORTED, "fused SwiGLU staging needs the decode GEMV");
  if (gemm_tc_eligible(a.N, a.K, a.T)) return launch_gemm_tc(a, s);
  return launch_gemm_mma(a, s);
}

tl_status launch_gemm_mma(const GemmArgs& a, cudaStream_t s) {
  if (a.T == 0) return ok();
  const int nt = token_tile(a.T);
  dim3 grid(a.N / ROWS_CTA, (a.T + nt - 1) / nt, a.splits);
  switch (nt) {
    case 8: TL_LAUNCH_PDL(gemm_w4_mma_kernel<8>, grid, THREADS, 0, s, a); break;
    case 16: TL_LAUNCH_PDL(gemm_w4_mma_kernel<16>, grid, THREADS, 0, s, a); break;
    case 32: TL_LAUNCH_PDL(gemm_w4_mma_kernel<32>, grid, THREADS, 0, s, a); break;
    default: TL_LAUNCH_PDL(gemm_w4_mma_kernel<64>, grid, THREADS, 0, s, a); break;
  }
  return ok();
}

}  // namespace tl
