// Quantised-weight GEMM for small INT4 token counts (short prompts):
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
// 64-wide chunks and gives at least two CTAs per SM.
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

int gemm_splits(int N, int K, int T, int bits, bool sign) {
  return gemm_tc_eligible(N, K, T, bits, sign) ? gemm_tc_splits(N, K, T) : gemm_mma_splits(N, K, T);
}

tl_status launch_gemm(const GemmArgs& a, cudaStream_t s) {
  if (a.swiglu_u) {
    if (!gemm_tc_eligible(a.N, a.K, a.T, a.bits, a.g0 != nullptr) || a.splits != 1 ||
        a.N != 2 * a.n_split ||
        a.n_split % 64 != 0)
      return set_error(TL_ERR_UNSUPPORTED,
                       "the fused SwiGLU epilogue needs the one-split tensor-core GEMM");
    return launch_gemm_tc(a, s);
  }
  if (gemm_tc_eligible(a.N, a.K, a.T, a.bits, a.g0 != nullptr)) return launch_gemm_tc(a, s);
  if (a.bits == 3 || a.g0 != nullptr)
    return set_error(TL_ERR_UNSUPPORTED, "INT3 or sign-bit GEMM: N %% 128 and K %% 64 required");
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
