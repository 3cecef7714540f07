// Decode-sized quantised-weight projections (T <= 8 tokens), one launch per
// projection, with the neighbouring row-wise work folded in:
//   y[t][n] = sum over k of x[t][k] * W[n][k],   W[n][k] = code[n][k] * scale[n][k / G]
// for canonical INT4 (8 codes per word) or INT3 (10 codes per word) weights.
//
// A CTA owns MT tiles of 16 weight rows over the whole of K; its sixteen warps
// split K (MT = 1: sixteen k ranges; MT = 2: eight per tile), so no split-K
// partial sums leave the CTA: the warps' results are added in shared memory in
// warp order, a fixed order that depends only on (N, K, MT).  Every token
// column is computed independently of the others, so a token's result does
// not depend on which other tokens share the launch.
//
// Weights are the A operand of mma.sync m16n8k16 (16 rows x 16 k), tokens the
// B operand (8 columns).  Lane (g, t) of a warp reads one 16-byte vector of
// packed words of row g and one of row g + 8 per chunk:
//   INT4: chunk = 128 k; the lane's vector holds k = 32t .. 32t + 31 of the
//         chunk; each word yields its code pairs (0,4) (1,5) (2,6) (3,7) with
//         one lop3 (and one shift per word) and one HFMA2, as exact fp16
//         integers; with G = 128 a chunk is one scale group, whose fp32 sum is
//         scaled once per chunk; with G = 64 lanes t = 0, 1 hold the chunk's
//         first group and t = 2, 3 its second, so each k step runs twice, once
//         per group with the other lanes' A registers zero, into two fp32 sums;
//   INT3: chunk = 16 words = 160 codes (the canonical rows are padded to
//         whole 16-byte vectors); the lane's vector holds codes 40t .. 40t + 39
//         of the chunk; code pairs (i, i + 6) of a word come out of one shift
//         and one lop3, codes 4 and 5 pair across two words through one prmt;
//         a lane's 40 codes may straddle a scale group, so the pair is scaled
//         in fp16 before the MMA (fp16(code * scale), as the tensor-core
//         prefill GEMM does).
// The k order inside an MMA is free as long as A and B agree, so the
// activations are staged in shared memory in the order the lanes' codes come
// out, and ldmatrix feeds them to the B operand.
//
// Folded work (template EPI / NORM):
//   NORM   the CTA forms its activations itself: x = fp16(rmsnorm(h) * gamma)
//          from the fp32 residual stream (the pre-norm before the QKV and the
//          gate/up projections), so no separate norm kernel runs at decode;
//   EPI_OUT   y -> out (fp32 [T][N]);
//   EPI_RESID y is added into the fp32 residual stream h (the O and down
//             projections; each element has exactly one writer), and the
//             down projection writes the per-layer trace;
//   EPI_SWIGLU tile 0 holds 16 gate rows and tile 1 the same 16 up rows:
//             u = fp16(silu(gate) * up).
// Weights, scales and gains are constants of the model: they are requested
// before the wait for the previous kernel, so their latency overlaps its tail.
#include <algorithm>
#include <cstring>

#include "tl_launch.cuh"

namespace tl {
namespace {

constexpr int DG_THREADS = 512;   // sixteen warps: more MMA chains in flight per SM
constexpr int DG_WARPS = 16;

enum { EPI_OUT = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };

template <int BITS>
struct DgFmt {
  static constexpr int CW = BITS == 4 ? 128 : 160;   // codes per chunk (one row)
};

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t lop3_ea(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));   // (a & b) | c
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t hfma2_bits(uint32_t x, __half2 m, __half2 a) {
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&x), m, a);
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2_bits(uint32_t x, uint32_t s) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&x), *reinterpret_cast<__half2*>(&s));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 h2c(float lo, float hi) {
  return __halves2half2(__float2half_rn(lo), __float2half_rn(hi));
}

// ---- INT4: the four exact fp16 code pairs of one word (nibbles (0,4) (1,5) (2,6) (3,7))
__device__ __forceinline__ void int4_pairs(uint32_t w, uint32_t* p) {
  const __half2 one = h2c(1.f, 1.f), sixteenth = h2c(0.0625f, 0.0625f);
  const __half2 lo_b = h2c(-1032.f, -1032.f), hi_b = h2c(-72.f, -72.f);
  const uint32_t w8 = w >> 8;
  p[0] = hfma2_bits(lop3_ea(w, 0x000F000Fu, 0x64006400u), one, lo_b);          // 1024 + u - 1032
  p[1] = hfma2_bits(lop3_ea(w, 0x00F000F0u, 0x64006400u), sixteenth, hi_b);    // (1024 + 16u)/16 - 72
  p[2] = hfma2_bits(lop3_ea(w8, 0x000F000Fu, 0x64006400u), one, lo_b);
  p[3] = hfma2_bits(lop3_ea(w8, 0x00F000F0u, 0x64006400u), sixteenth, hi_b);
}

// ---- INT3: codes (i, i + 6) of one word: bits 3i and 3i + 18 after a shift
// by 3i land at bits 0-2 (1024 + u) and 18-20 (1024 + 4u of the upper half)
template <int I>
__device__ __forceinline__ uint32_t int3_pair_i6(uint32_t w) {
  const uint32_t x = lop3_ea(w >> (3 * I), 0x001C0007u, 0x64006400u);
  return hfma2_bits(x, h2c(1.f, 0.25f), h2c(-1028.f, -260.f));
}
// code 4 of words a and b (bits 12-14: bits 4-6 of byte 1)
__device__ __forceinline__ uint32_t int3_pair_c4(uint32_t a, uint32_t b) {
  const uint32_t x = lop3_ea(prmt(a, b, 0x0501u), 0x00700070u, 0x64006400u);
  return hfma2_bits(x, h2c(0.0625f, 0.0625f), h2c(-68.f, -68.f));
}
// code 5 of words a and b (bits 15-17: bit 7 of byte 1 and bits 0-1 of byte 2)
__device__ __forceinline__ uint32_t int3_pair_c5(uint32_t a, uint32_t b) {
  const uint32_t x = lop3_ea(prmt(a, b, 0x6521u), 0x03800380u, 0x64006400u);
  return hfma2_bits(x, h2c(0.0078125f, 0.0078125f), h2c(-12.f, -12.f));
}

// ---- cross-iteration rounding: the odd-iteration code is code + 1 where the
// sign-of-frac bit is set and code - 1 where it is clear.  pm1 turns bits 15
// and 31 of x into the fp16 pair (+-1, +-1); adding it to an exact code pair
// is exact.
__device__ __forceinline__ uint32_t pm1(uint32_t x) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(x), "r"(0x80008000u), "r"(0xBC00BC00u));
  return d;   // (x & 0x80008000) ^ 0xBC00BC00: bit set -> +1, clear -> -1
}
__device__ __forceinline__ uint32_t hadd2_bits(uint32_t a, uint32_t b) {
  __half2 r = __hadd2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
// INT4: the pairs (i, i + 4), i = 0..3, of word q of a lane's vector have their
// bits at i and i + 4 of byte q of the vector's sign word; spreading two bytes
// as low nibbles at bits 0-3 / 8-11 and high nibbles at 16-19 / 24-27 puts
// the pair's bits 16 apart, one shift away from bits 15 and 31.
__device__ __forceinline__ void int4_sign_fix(uint32_t sw, int q, uint32_t* p) {
  const uint32_t h = q < 2 ? sw : sw >> 16;
  const uint32_t P = (h & 0x0F0Fu) | ((h & 0xF0F0u) << 12);
  const int base = (q & 1) ? 7 : 15;
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = hadd2_bits(p[i], pm1(P << (base - i)));
}
// INT3: S holds the sign bits of a lane's 40 codes (bit L for code L =
// 10 q + i).  Pair (i, i + 6) of word q: bits 10q + i and 10q + i + 6.
template <int I>
__device__ __forceinline__ uint32_t int3_sign_i6(uint64_t S, int q) {
  const uint32_t w = (uint32_t)(S >> (10 * q)) & 0x3FFu;
  return pm1((w | (w << 10)) << (15 - I));
}
// Pairs c4 (codes 4 and 14 of word pair (0, 1), or 24 and 34 of (2, 3)) and
// c5 (5 and 15, or 25 and 35): bits o, o + 1, o + 10, o + 11 with o = 4 or 24.
__device__ __forceinline__ uint32_t int3_sign_c4(uint64_t S, int o) {
  const uint32_t u = (uint32_t)(S >> o) & 0xC03u;
  return pm1((u | (u << 6)) << 15);
}
__device__ __forceinline__ uint32_t int3_sign_c5(uint64_t S, int o) {
  const uint32_t u = (uint32_t)(S >> o) & 0xC03u;
  return pm1((u | (u << 6)) << 14);
}

// Position, in a staged activation row, of element k of the original row.
// INT4: k = 128c + 32t + 8q + e -> k step 2q + ((e >> 1) & 1), slot 2t + 8 (e odd) + (e >= 4).
// INT3: k = 160c + 40t + L (L = 10q + i) -> see int3_slot.
__device__ __forceinline__ int int3_slot(int L, int t, int& j) {
  const int q = L / 10, i = L - 10 * q;
  switch (i) {
    case 0: j = 2 * q; return 2 * t;
    case 6: j = 2 * q; return 2 * t + 1;
    case 1: j = 2 * q; return 2 * t + 8;
    case 7: j = 2 * q; return 2 * t + 9;
    case 2: j = 2 * q + 1; return 2 * t;
    case 8: j = 2 * q + 1; return 2 * t + 1;
    case 3: j = 2 * q + 1; return 2 * t + 8;
    case 9: j = 2 * q + 1; return 2 * t + 9;
    case 4: j = 8 + (q >> 1); return 2 * t + (q & 1);
    default: j = 8 + (q >> 1); return 2 * t + 8 + (q & 1);   // i == 5
  }
}

// INT3 staging by packed word: the ten codes L = 10q + i (i = 0..9) of the
// word of lane t, word q of chunk c go to these positions of the staged row
// (the slot table of int3_slot, unrolled with i known at compile time).
__device__ __forceinline__ void int3_word_slots(int c, int t, int q, int* pos) {
  const int base = c * 160 + 2 * t;
  const int j0 = 16 * (2 * q), j1 = 16 * (2 * q + 1), j8 = 16 * (8 + (q >> 1));
  pos[0] = base + j0;                 // i = 0
  pos[1] = base + j0 + 8;             // i = 1
  pos[2] = base + j1;                 // i = 2
  pos[3] = base + j1 + 8;             // i = 3
  pos[4] = base + j8 + (q & 1);       // i = 4
  pos[5] = base + j8 + 8 + (q & 1);   // i = 5
  pos[6] = base + j0 + 1;             // i = 6
  pos[7] = base + j0 + 9;             // i = 7
  pos[8] = base + j1 + 1;             // i = 8
  pos[9] = base + j1 + 9;             // i = 9
}

template <int BITS>
__device__ __forceinline__ int xpos(int k) {
  if (BITS == 4) {
    const int c = k >> 7, r = k & 127, t = r >> 5, q = (r >> 3) & 3, e = k & 7;
    const int j = 2 * q + ((e >> 1) & 1);
    const int s = 2 * t + ((e & 1) ? 8 : 0) + (e >= 4 ? 1 : 0);
    return c * 128 + 16 * j + s;
  } else {
    const int c = k / 160, r = k - 160 * c, t = r / 40, L = r - 40 * t;
    int j;
    const int s = int3_slot(L, t, j);
    return c * 160 + 16 * j + s;
  }
}

struct DgArgs {
  const uint32_t* w0;   // canonical packed rows; unit u is rows u*16 .. u*16+15
  const __half* s0;     //   (EPI_SWIGLU: w0 = gate, w1 = up, both rows u*16 ..)
  const uint32_t* w1;
  const __half* s1;
  const uint32_t* g0;   // sign-of-frac bits of w0's / w1's rows [N][spr] (odd iterations)
  const uint32_t* g1;
  int spr;              // sign words per row (K / 32)
  int N, K, G, wpr;     // output rows (per matrix), K, group, packed words per row
  int T;                // active token rows (1..8)
  int n_units;          // N / 16
  int stages;           // weight stages in shared memory
  int row_bytes;        // bytes of one packed row (wpr * 4)
  const __half* x;      // fp16 [T][K] activations (when !NORM)
  const float* h;       // fp32 [T][K] residual stream (NORM)
  const float* gamma;   // fp32 [K] (NORM)
  __half* x_out;        // NORM, optional: the fp16 activations x [T][K], natural order (CTA 0)
  float eps;
  float* out;           // EPI_OUT: fp32 [T][N]
  float* hres;          // EPI_RESID: fp32 [rows][N], += y
  __half* u;            // EPI_SWIGLU: fp16 [T][N]
  float* trace;         // EPI_RESID, optional: fp32 [trace_rows][N] rows indexed by out_row
  const int32_t* out_row;
  int trace_rows;       // rows T .. trace_rows-1 are copied from hres unchanged
  int* status;          // a bounded wait that runs out records TL_ERR_TIMEOUT here
  ExitArgs ex;          // the per-iteration residual-norm check
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t dg_globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for an mbarrier phase: false once 2 s of global time have passed.
__device__ __forceinline__ bool dg_wait(uint32_t bar, uint32_t parity) {
  uint64_t start = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if (i == 0) start = dg_globaltimer();
    else if ((i & 63) == 0 && dg_globaltimer() - start > 2000000000ull) return false;
  }
}

// Stage layout of one 16-row tile: two groups of eight consecutive packed
// rows (rows 0-7 and 8-15 of the tile), each group one bulk copy, the second
// group 64 bytes further than the end of the first, so that the two rows any
// quarter-warp reads (MMA rows 2p and 2p + 1 below) sit half a bank period
// apart.  MMA row r of the tile (lane g = r & 7 holds rows g and g + 8) is
// packed row dg_row(r): rows 2p, 2p + 1 of an MMA tile come from different
// groups.  The epilogue writes row r's result to output row dg_row(r).
__device__ __forceinline__ int dg_row(int r) { return ((r & 1) << 3) | ((r & 8) >> 1) | ((r & 7) >> 1); }
__device__ __forceinline__ size_t dg_grp_bytes(int row_bytes) { return (size_t)8 * row_bytes + 64; }
__device__ __forceinline__ size_t dg_row_off(int r, int row_bytes) {
  const int pr = dg_row(r);
  return (size_t)(pr >> 3) * dg_grp_bytes(row_bytes) + (size_t)(pr & 7) * row_bytes;
}

// The weights, scales (and sign rows) of one unit into its stage: lanes
// 0 .. 2 MT - 1 of the calling warp copy the row groups, then one lane per
// tile its scales (and its sign rows, one copy each).
template <int MT, bool SGN>
__device__ __forceinline__ void dg_issue_unit(const DgArgs& a, int unit, unsigned char* stage,
                                              uint32_t bar, int lane) {
  const uint32_t grp_copy = 8u * (uint32_t)a.row_bytes;
  const size_t grp = dg_grp_bytes(a.row_bytes), tile = 2 * grp;
  const int gpr = a.K / a.G;
  const uint32_t sc_bytes = 16u * gpr * 2;
  const uint32_t sg_bytes = SGN ? 16u * a.spr * 4 : 0u;   // a tile's sign rows, one copy
  if (lane == 0) {
    const uint32_t total = MT * (2 * grp_copy + sc_bytes + sg_bytes);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(total)
                 : "memory");
  }
  __syncwarp();
  const int r0 = unit * 16;
  if (lane < 2 * MT) {
    const int m = lane >> 1, q = lane & 1;   // tile m, rows 8q .. 8q + 7
    const uint32_t* src = (m == 0 ? a.w0 : a.w1) + (size_t)(r0 + 8 * q) * a.wpr;
    const uint32_t dst = smem_u32(stage + (size_t)m * tile + (size_t)q * grp);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(grp_copy), "r"(bar)
        : "memory");
  }
  if (lane < MT) {
    const __half* src = (lane == 0 ? a.s0 : a.s1) + (size_t)r0 * gpr;
    const uint32_t dst = smem_u32(stage + (size_t)MT * tile + (size_t)lane * sc_bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(sc_bytes), "r"(bar)
        : "memory");
    if (SGN) {
      const uint32_t* gsrc = (lane == 0 ? a.g0 : a.g1) + (size_t)r0 * a.spr;
      const uint32_t gdst = smem_u32(stage + (size_t)MT * tile + (size_t)MT * sc_bytes +
                                     (size_t)lane * sg_bytes);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(gdst),
          "l"(gsrc), "r"(sg_bytes), "r"(bar)
          : "memory");
    }
  }
}

// One CTA per SM (at most): CTA c takes units c, c + gridDim.x, ...; a unit is
// 16 weight rows (EPI_SWIGLU: 16 gate rows and the same 16 up rows).  The
// units' packed words and scales stream through a ring of `stages` shared-
// memory stages filled by bulk copies; the first stages are requested before
// the wait for the previous kernel (weights are constants of the model), and
// the CTA leaves room on its SM for the next kernel's CTA to do the same.
// UM > 0: every unit of the CTA (at most UM) is resident at once, copied in
// before the dependency wait; the warps compute them back to back into
// per-unit sums and one reduction and one epilogue close the launch.  UM == 0:
// the units stream through a ring of a.stages stages, one reduction per unit.
template <int BITS, int MT, bool NORM, int EPI, int UM, bool SGN, bool WIDE>
__global__ void __launch_bounds__(DG_THREADS, 1) gemv_dec_kernel(DgArgs a) {
  using Fm = DgFmt<BITS>;
  constexpr int CW = Fm::CW;
  constexpr int W = DG_WARPS / MT;                 // warps (k ranges) per tile
  extern __shared__ __align__(128) unsigned char dg_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m = warp / W, ks = warp - m * W;
  const int nvec = a.wpr >> 2;                     // 16-byte vectors per packed row
  const int nch = (nvec + 3) >> 2;                 // chunks per row
  const int c_lo = ks * nch / W, c_hi = (ks + 1) * nch / W;
  const int xw = nch * CW + 8;                     // staged activation row, halves
  const int gsh = __ffs(a.G) - 1;
  const int gpr = a.K >> gsh;
  const bool g64 = BITS == 4 && a.G == 64;
  const size_t tile_bytes = 2 * dg_grp_bytes(a.row_bytes);
  const size_t stage_bytes = (size_t)MT * tile_bytes + (size_t)MT * 16 * gpr * 2 +
                             (SGN ? (size_t)MT * 16 * a.spr * 4 : 0);
  unsigned char* stages = dg_smem;
  __half* xs = reinterpret_cast<__half*>(dg_smem + (size_t)a.stages * stage_bytes);   // [T][xw]
  float* red = reinterpret_cast<float*>(xs + (size_t)a.T * xw);      // [max(2, UM)][MT][W][16][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + (UM > 2 ? UM : 2) * DG_WARPS * 16 * 8);
  __shared__ __align__(16) uint32_t zero16[4];
  __shared__ float nred[8][DG_WARPS];
  __shared__ int abort_flag;
  const int n_my = (a.n_units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < a.stages; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bars + i)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    zero16[0] = zero16[1] = zero16[2] = zero16[3] = 0u;
    abort_flag = 0;
  }
  __syncthreads();
  // the first units' weights: requested before the dependency wait
  int issued = min(a.stages, n_my);   // units whose copies were issued (the same in every thread)
  int stop = n_my;                    // the unit a timed-out wait stopped at
  if (warp == 0)
    for (int j = 0; j < a.stages && j < n_my; ++j)
      dg_issue_unit<MT, SGN>(a, blockIdx.x + j * gridDim.x, stages + (size_t)j * stage_bytes,
                        smem_u32(bars + j), lane);
  // the gains are constants of the model: requested before the dependency
  // wait (rows of d <= 2048 take two float4 per thread)
  constexpr int NV = 2;
  float4 gpre[NV];
  const bool small_k = a.K <= 4 * DG_THREADS * NV;
  if (NORM && BITS == 4 && small_k) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int k = 4 * tid + 4 * DG_THREADS * i;
      gpre[i] = k < a.K ? __ldg(reinterpret_cast<const float4*>(a.gamma + k))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  pdl_enter();   // activations and the residual stream come from the previous kernels

  // ---- stage the activations (permuted) into xs; padding codes see zeros
  const int kpad = nch * CW;
  if (NORM && BITS == 4 && small_k && a.T <= 2) {
    // one pass: the (at most two) rows stay in registers between the sum of
    // squares and the scaling; same arithmetic and order as the general path
    float4 hv[2][NV];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int k = 4 * tid + 4 * DG_THREADS * i;
        hv[b][i] = b < a.T && k < a.K ? *reinterpret_cast<const float4*>(a.h + (size_t)b * a.K + k)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (b < a.T) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          ss = fmaf(hv[b][i].x, hv[b][i].x, ss);
          ss = fmaf(hv[b][i].y, hv[b][i].y, ss);
          ss = fmaf(hv[b][i].z, hv[b][i].z, ss);
          ss = fmaf(hv[b][i].w, hv[b][i].w, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) nred[b][warp] = ss;
      }
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (b < a.T) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < DG_WARPS; ++w) tot += nred[b][w];
        if (a.ex.check_iter > 0 && blockIdx.x == 0 && tid == 0 && a.ex.exit_it[b] == 0 &&
            sqrtf(tot) > a.ex.tau)
          a.ex.exit_it[b] = a.ex.check_iter;
        const float r = rsqrtf(tot / (float)a.K + a.eps);
        __half* xr = xs + (size_t)b * xw;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const int k = 4 * tid + 4 * DG_THREADS * i;
          if (k < a.K) {
            const float4 v = hv[b][i], gm = gpre[i];
            const __half x0 = __float2half_rn(v.x * r * gm.x), x1 = __float2half_rn(v.y * r * gm.y);
            const __half x2 = __float2half_rn(v.z * r * gm.z), x3 = __float2half_rn(v.w * r * gm.w);
            xr[xpos<BITS>(k)] = x0;
            xr[xpos<BITS>(k + 1)] = x1;
            xr[xpos<BITS>(k + 2)] = x2;
            xr[xpos<BITS>(k + 3)] = x3;
            if (a.x_out && blockIdx.x == 0) {
              __half2* xo = reinterpret_cast<__half2*>(a.x_out + (size_t)b * a.K + k);
              xo[0] = __halves2half2(x0, x1);
              xo[1] = __halves2half2(x2, x3);
            }
          }
        }
        for (int k = a.K + tid; k < kpad; k += DG_THREADS) xr[xpos<BITS>(k)] = __float2half_rn(0.f);
      }
    }
  } else if (WIDE && NORM && BITS == 4 && a.K <= 4 * DG_THREADS) {
    // three to eight rows of d <= 2048: one float4 of every row per thread,
    // all rows' loads in flight together and kept in registers between the
    // sum of squares and the scaling (same arithmetic and order per row as
    // the general path)
    float4 hv[8];
    const int k = 4 * tid;
#pragma unroll
    for (int b = 0; b < 8; ++b)
      hv[b] = b < a.T && k < a.K ? *reinterpret_cast<const float4*>(a.h + (size_t)b * a.K + k)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    float ss[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      ss[b] = fmaf(hv[b].x, hv[b].x, 0.f);
      ss[b] = fmaf(hv[b].y, hv[b].y, ss[b]);
      ss[b] = fmaf(hv[b].z, hv[b].z, ss[b]);
      ss[b] = fmaf(hv[b].w, hv[b].w, ss[b]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int b = 0; b < 8; ++b) ss[b] += __shfl_xor_sync(0xffffffffu, ss[b], o);
    if (lane == 0)
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (b < a.T) nred[b][warp] = ss[b];
    __syncthreads();
    const float4 gm = gpre[0];
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (b < a.T) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < DG_WARPS; ++w) tot += nred[b][w];
        if (a.ex.check_iter > 0 && blockIdx.x == 0 && tid == 0 && a.ex.exit_it[b] == 0 &&
            sqrtf(tot) > a.ex.tau)
          a.ex.exit_it[b] = a.ex.check_iter;
        const float r = rsqrtf(tot / (float)a.K + a.eps);
        if (k < a.K) {
          const float4 v = hv[b];
          __half* xr = xs + (size_t)b * xw;
          const __half x0 = __float2half_rn(v.x * r * gm.x), x1 = __float2half_rn(v.y * r * gm.y);
          const __half x2 = __float2half_rn(v.z * r * gm.z), x3 = __float2half_rn(v.w * r * gm.w);
          xr[xpos<BITS>(k)] = x0;
          xr[xpos<BITS>(k + 1)] = x1;
          xr[xpos<BITS>(k + 2)] = x2;
          xr[xpos<BITS>(k + 3)] = x3;
          if (a.x_out && blockIdx.x == 0) {
            __half2* xo = reinterpret_cast<__half2*>(a.x_out + (size_t)b * a.K + k);
            xo[0] = __halves2half2(x0, x1);
            xo[1] = __halves2half2(x2, x3);
          }
        }
      }
    }
  } else if (NORM) {
    // x = fp16(h * rsqrt(mean(h^2) + eps) * gamma) per token row, the sum of
    // squares in a fixed order (per thread, xor tree, warps in order)
    for (int b = 0; b < a.T; ++b) {
      const float* hr = a.h + (size_t)b * a.K;
      float ss = 0.f;
      for (int k = 4 * tid; k < a.K; k += 4 * DG_THREADS) {
        const float4 v = *reinterpret_cast<const float4*>(hr + k);
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) nred[b][warp] = ss;
    }
    __syncthreads();
    for (int b = 0; b < a.T; ++b) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < DG_WARPS; ++w) tot += nred[b][w];
      // the residual-norm check on the stream entering this loop iteration
      // (every CTA computes the same sum; CTA 0 records the decision)
      if (a.ex.check_iter > 0 && blockIdx.x == 0 && tid == 0 && a.ex.exit_it[b] == 0 &&
          sqrtf(tot) > a.ex.tau)
        a.ex.exit_it[b] = a.ex.check_iter;
      const float r = rsqrtf(tot / (float)a.K + a.eps);
      const float* hr = a.h + (size_t)b * a.K;
      __half* xr = xs + (size_t)b * xw;
      if (BITS == 4) {
        for (int k = 4 * tid; k < a.K; k += 4 * DG_THREADS) {
          const float4 v = *reinterpret_cast<const float4*>(hr + k);
          const float4 gm = __ldg(reinterpret_cast<const float4*>(a.gamma + k));
          const __half x0 = __float2half_rn(v.x * r * gm.x), x1 = __float2half_rn(v.y * r * gm.y);
          const __half x2 = __float2half_rn(v.z * r * gm.z), x3 = __float2half_rn(v.w * r * gm.w);
          xr[xpos<BITS>(k)] = x0;
          xr[xpos<BITS>(k + 1)] = x1;
          xr[xpos<BITS>(k + 2)] = x2;
          xr[xpos<BITS>(k + 3)] = x3;
          if (a.x_out && blockIdx.x == 0) {
            __half2* xo = reinterpret_cast<__half2*>(a.x_out + (size_t)b * a.K + k);
            xo[0] = __halves2half2(x0, x1);
            xo[1] = __halves2half2(x2, x3);
          }
        }
      } else {
        for (int wd = tid; wd < nch * 16; wd += DG_THREADS) {
          const int c = wd >> 4, t = (wd >> 2) & 3, q = wd & 3;
          const int k0 = c * 160 + 40 * t + 10 * q;
          int pos[10];
          int3_word_slots(c, t, q, pos);
#pragma unroll
          for (int i = 0; i < 10; ++i) {
            const __half xv = k0 + i < a.K ? __float2half_rn(hr[k0 + i] * r * __ldg(a.gamma + k0 + i))
                                           : __float2half_rn(0.f);
            xr[pos[i]] = xv;
            if (a.x_out && blockIdx.x == 0 && k0 + i < a.K) a.x_out[(size_t)b * a.K + k0 + i] = xv;
          }
        }
      }
    }
  } else if (WIDE && BITS == 4 && a.T > 2) {
    // three to eight rows: the vectors of eight consecutive k of all rows
    // ([T][K] contiguous), eight per thread in flight; each becomes four
    // half2 stores
    const int kv = a.K >> 3, total = a.T * kv;
    for (int e0 = tid; e0 < total; e0 += 8 * DG_THREADS) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * DG_THREADS;
        if (e < total) v[i] = *reinterpret_cast<const uint4*>(a.x + (size_t)e * 8);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * DG_THREADS;
        if (e < total) {
          const int b = e / kv, k = (e - b * kv) * 8;
          const __half* h8 = reinterpret_cast<const __half*>(&v[i]);
          __half* xr = xs + (size_t)b * xw + xpos<4>(k);   // element 0: k step 2q, slot 2t
          *reinterpret_cast<__half2*>(xr) = __halves2half2(h8[0], h8[4]);
          *reinterpret_cast<__half2*>(xr + 8) = __halves2half2(h8[1], h8[5]);
          *reinterpret_cast<__half2*>(xr + 16) = __halves2half2(h8[2], h8[6]);
          *reinterpret_cast<__half2*>(xr + 24) = __halves2half2(h8[3], h8[7]);
        }
      }
    }
  } else {
    for (int b = 0; b < a.T; ++b) {
      const __half* src = a.x + (size_t)b * a.K;
      __half* xr = xs + (size_t)b * xw;
      if (BITS == 4) {
        // eight consecutive k -> four half2 stores
        for (int k = 8 * tid; k < a.K; k += 8 * DG_THREADS) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + k);
          const __half* e = reinterpret_cast<const __half*>(&v);
          const int base = xpos<4>(k);   // position of element 0 (k-step 2q, slot 2t)
          *reinterpret_cast<__half2*>(xr + base) = __halves2half2(e[0], e[4]);
          *reinterpret_cast<__half2*>(xr + base + 8) = __halves2half2(e[1], e[5]);
          *reinterpret_cast<__half2*>(xr + base + 16) = __halves2half2(e[2], e[6]);
          *reinterpret_cast<__half2*>(xr + base + 24) = __halves2half2(e[3], e[7]);
        }
      } else {
        // one packed word (ten codes, ten consecutive k) per thread and step
        for (int wd = tid; wd < nch * 16; wd += DG_THREADS) {
          const int c = wd >> 4, t = (wd >> 2) & 3, q = wd & 3;
          const int k0 = c * 160 + 40 * t + 10 * q;
          int pos[10];
          int3_word_slots(c, t, q, pos);
#pragma unroll
          for (int i = 0; i < 10; ++i)
            xr[pos[i]] = k0 + i < a.K ? src[k0 + i] : __float2half_rn(0.f);
        }
      }
    }
  }
  __syncthreads();

  // ldmatrix rows: lane l supplies token row l & 7 (a zero block for rows >= T)
  const int lr = lane & 7, lq = lane >> 3;
  const uint32_t zaddr = smem_u32(zero16);
  const bool lrow_ok = lr < a.T;
  const uint32_t lbase = lrow_ok ? smem_u32(xs + (size_t)lr * xw + 8 * lq) : zaddr;
  const uint32_t lmul = lrow_ok ? 2u : 0u;   // bytes per staged element (0: stay on the zero block)

  // this warp's chunks of its tile of the unit in `stage`, added into acc
  auto unit_mma = [&](const unsigned char* stage, float* acc) {
    // ---- the MMAs: this warp's chunks of its tile, words and scales from the stage
    // MMA rows g and g + 8 of tile m: packed rows dg_row(g), dg_row(g + 8)
    const int pr0 = dg_row(g), pr1 = dg_row(g + 8);
    const unsigned char* tile_base = stage + (size_t)m * tile_bytes;
    const unsigned char* wt0 = tile_base + dg_row_off(g, a.row_bytes);
    const unsigned char* wt1 = tile_base + dg_row_off(g + 8, a.row_bytes);
    const __half* sct = reinterpret_cast<const __half*>(stage + (size_t)MT * tile_bytes +
                                                        (size_t)m * 16 * gpr * 2);
    const __half* st0 = sct + (size_t)pr0 * gpr;
    const __half* st1 = sct + (size_t)pr1 * gpr;
    // the tile's sign rows (odd iterations), same rows
    const uint32_t* sgt = reinterpret_cast<const uint32_t*>(
        stage + (size_t)MT * tile_bytes + (size_t)MT * 16 * gpr * 2 + (size_t)m * 16 * a.spr * 4);
    const uint32_t* sg0 = sgt + (size_t)pr0 * a.spr;
    const uint32_t* sg1 = sgt + (size_t)pr1 * a.spr;
    for (int c = c_lo; c < c_hi; ++c) {
      const int vi = 4 * c + t;
      uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
      if (vi < nvec) {
        v0 = *reinterpret_cast<const uint4*>(wt0 + (size_t)vi * 16);
        v1 = *reinterpret_cast<const uint4*>(wt1 + (size_t)vi * 16);
      }
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&v0);   // row g
      const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&v1);   // row g + 8
      const uint32_t xb = lbase + lmul * (uint32_t)(c * CW);
      if (BITS == 4) {
        // the vector's 32 codes have one sign word (rows g and g + 8)
        const uint32_t sw0 = SGN && vi < nvec ? sg0[vi] : 0u;
        const uint32_t sw1 = SGN && vi < nvec ? sg1[vi] : 0u;
        const int ga = g64 ? 2 * c : c;
        float ca[4] = {0.f, 0.f, 0.f, 0.f}, cb2[4] = {0.f, 0.f, 0.f, 0.f};
        const bool first = t < 2;   // G = 64: this lane's codes are in the chunk's first group
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t p0[4], p1[4];
          int4_pairs(w0[q], p0);
          int4_pairs(w1[q], p1);
          if (SGN) {
            int4_sign_fix(sw0, q, p0);
            int4_sign_fix(sw1, q, p1);
          }
          uint32_t b[4];
          ldsm_x4(b, xb + lmul * (uint32_t)(32 * q));   // k steps 2q and 2q + 1
          const uint32_t A0[4] = {p0[0], p1[0], p0[1], p1[1]};
          const uint32_t A1[4] = {p0[2], p1[2], p0[3], p1[3]};
          if (!g64) {
            mma16816(ca, A0, b[0], b[1]);
            mma16816(ca, A1, b[2], b[3]);
          } else {
            const uint32_t z[4] = {0u, 0u, 0u, 0u};
            mma16816(ca, first ? A0 : z, b[0], b[1]);
            mma16816(ca, first ? A1 : z, b[2], b[3]);
            mma16816(cb2, first ? z : A0, b[0], b[1]);
            mma16816(cb2, first ? z : A1, b[2], b[3]);
          }
        }
        const float f0 = __half2float(st0[ga]), f1 = __half2float(st1[ga]);
        acc[0] = fmaf(ca[0], f0, acc[0]);
        acc[1] = fmaf(ca[1], f0, acc[1]);
        acc[2] = fmaf(ca[2], f1, acc[2]);
        acc[3] = fmaf(ca[3], f1, acc[3]);
        if (g64) {
          const float e0 = __half2float(st0[ga + 1]), e1 = __half2float(st1[ga + 1]);
          acc[0] = fmaf(cb2[0], e0, acc[0]);
          acc[1] = fmaf(cb2[1], e0, acc[1]);
          acc[2] = fmaf(cb2[2], e1, acc[2]);
          acc[3] = fmaf(cb2[3], e1, acc[3]);
        }
      } else {
        // INT3: the lane's codes 40t + L with L < bnd are in the lower scale
        // group; bnd is a multiple of 8 (chunk, lane and group starts all
        // are), so each octet of codes L = 8o .. 8o + 7 has one scale
        const int k0 = c * CW + 40 * t;
        const int ga = min(k0 >> gsh, gpr - 1), gb = min(ga + 1, gpr - 1);
        const int bnd = (((k0 >> gsh) + 1) << gsh) - k0;
        const __half sa0 = st0[ga], sb0 = st0[gb], sa1 = st1[ga], sb1 = st1[gb];
        __half so0[5], so1[5];
#pragma unroll
        for (int oc = 0; oc < 5; ++oc) {
          so0[oc] = 8 * oc < bnd ? sa0 : sb0;
          so1[oc] = 8 * oc < bnd ? sa1 : sb1;
        }
        // the sign bits of the lane's 40 codes (bit L for code L), rows g and g + 8
        uint64_t S0 = 0, S1 = 0;
        if (SGN) {
          const int wi = (5 * vi) >> 2, o = 8 * (vi & 3);
          const uint32_t a0 = wi < a.spr ? sg0[wi] : 0u, b0 = wi + 1 < a.spr ? sg0[wi + 1] : 0u;
          const uint32_t a1 = wi < a.spr ? sg1[wi] : 0u, b1 = wi + 1 < a.spr ? sg1[wi + 1] : 0u;
          S0 = ((((uint64_t)b0) << 32) | a0) >> o;
          S1 = ((((uint64_t)b1) << 32) | a1) >> o;
        }
#define TL_FX(p, corr) (SGN ? hadd2_bits((p), (corr)) : (p))
#define TL_SC(p, La, Lb, so) hmul2_bits((p), h2bits(__halves2half2(so[(La) >> 3], so[(Lb) >> 3])))
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t b[4];
          ldsm_x4(b, xb + lmul * (uint32_t)(32 * q));   // k steps 2q, 2q + 1
          const int L = 10 * q;
          const uint32_t A0[4] = {
              TL_SC(TL_FX(int3_pair_i6<0>(w0[q]), int3_sign_i6<0>(S0, q)), L, L + 6, so0),
              TL_SC(TL_FX(int3_pair_i6<0>(w1[q]), int3_sign_i6<0>(S1, q)), L, L + 6, so1),
              TL_SC(TL_FX(int3_pair_i6<1>(w0[q]), int3_sign_i6<1>(S0, q)), L + 1, L + 7, so0),
              TL_SC(TL_FX(int3_pair_i6<1>(w1[q]), int3_sign_i6<1>(S1, q)), L + 1, L + 7, so1)};
          const uint32_t A1[4] = {
              TL_SC(TL_FX(int3_pair_i6<2>(w0[q]), int3_sign_i6<2>(S0, q)), L + 2, L + 8, so0),
              TL_SC(TL_FX(int3_pair_i6<2>(w1[q]), int3_sign_i6<2>(S1, q)), L + 2, L + 8, so1),
              TL_SC(TL_FX(int3_pair_i6<3>(w0[q]), int3_sign_i6<3>(S0, q)), L + 3, L + 9, so0),
              TL_SC(TL_FX(int3_pair_i6<3>(w1[q]), int3_sign_i6<3>(S1, q)), L + 3, L + 9, so1)};
          mma16816(acc, A0, b[0], b[1]);
          mma16816(acc, A1, b[2], b[3]);
        }
        {
          uint32_t b[4];
          ldsm_x4(b, xb + lmul * 128u);                  // k steps 8 and 9
          const uint32_t A0[4] = {
              TL_SC(TL_FX(int3_pair_c4(w0[0], w0[1]), int3_sign_c4(S0, 4)), 4, 14, so0),
              TL_SC(TL_FX(int3_pair_c4(w1[0], w1[1]), int3_sign_c4(S1, 4)), 4, 14, so1),
              TL_SC(TL_FX(int3_pair_c5(w0[0], w0[1]), int3_sign_c5(S0, 4)), 5, 15, so0),
              TL_SC(TL_FX(int3_pair_c5(w1[0], w1[1]), int3_sign_c5(S1, 4)), 5, 15, so1)};
          const uint32_t A1[4] = {
              TL_SC(TL_FX(int3_pair_c4(w0[2], w0[3]), int3_sign_c4(S0, 24)), 24, 34, so0),
              TL_SC(TL_FX(int3_pair_c4(w1[2], w1[3]), int3_sign_c4(S1, 24)), 24, 34, so1),
              TL_SC(TL_FX(int3_pair_c5(w0[2], w0[3]), int3_sign_c5(S0, 24)), 25, 35, so0),
              TL_SC(TL_FX(int3_pair_c5(w1[2], w1[3]), int3_sign_c5(S1, 24)), 25, 35, so1)};
          mma16816(acc, A0, b[0], b[1]);
          mma16816(acc, A1, b[2], b[3]);
        }
#undef TL_SC
#undef TL_FX
      }
    }

  };
  // the unit's outputs from the warps' sums in redj (threads tid < 128)
  auto unit_epilogue = [&](int unit, const float* redj) {
    if (EPI == EPI_SWIGLU) {
      if (tid < 16 * 8) {
        const int r = tid >> 3, b = tid & 7;
        if (b < a.T) {
          float gs = 0.f, us = 0.f;
#pragma unroll
          for (int w = 0; w < W; ++w) {
            gs += redj[((0 * W + w) * 16 + r) * 8 + b];
            us += redj[((1 * W + w) * 16 + r) * 8 + b];
          }
          const float silu = gs / (1.0f + __expf(-gs));
          a.u[(size_t)b * a.N + unit * 16 + dg_row(r)] = __float2half_rn(silu * us);
        }
      }
    } else {
      if (tid < 16 * 8) {
        const int r = tid >> 3, b = tid & 7;
        const int n = unit * 16 + dg_row(r);
        float y = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) y += redj[(w * 16 + r) * 8 + b];
        if (EPI == EPI_OUT) {
          if (b < a.T) a.out[(size_t)b * a.N + n] = y;
        } else {
          if (b < a.T) {
            float* hp = a.hres + (size_t)b * a.N + n;
            const bool frozen = a.ex.skip && a.ex.exit_it[b] != 0;   // stopped by the check
            const float hn = frozen ? *hp : *hp + y;
            *hp = hn;
            if (a.trace) a.trace[(size_t)a.out_row[b] * a.N + n] = hn;
          } else if (a.trace && b < a.trace_rows) {
            // lanes that ran fewer iterations keep their last value in the trace
            a.trace[(size_t)a.out_row[b] * a.N + n] = a.hres[(size_t)b * a.N + n];
          }
        }
      }
    }
  };
  if (UM > 0) {
    // every unit resident: back to back, then one reduction
    float acc[UM > 0 ? UM : 1][4];
#pragma unroll
    for (int u = 0; u < (UM > 0 ? UM : 1); ++u) {
      acc[u][0] = acc[u][1] = acc[u][2] = acc[u][3] = 0.f;
      if (u < n_my) {
        if (!dg_wait(smem_u32(bars + u), 0u)) abort_flag = 1;
        unit_mma(stages + (size_t)u * stage_bytes, acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < (UM > 0 ? UM : 1); ++u) {
      if (u < n_my) {
        float* rw = red + ((size_t)u * DG_WARPS + m * W + ks) * 16 * 8;
        rw[g * 8 + 2 * t] = acc[u][0];
        rw[g * 8 + 2 * t + 1] = acc[u][1];
        rw[(g + 8) * 8 + 2 * t] = acc[u][2];
        rw[(g + 8) * 8 + 2 * t + 1] = acc[u][3];
      }
    }
    __syncthreads();
    if (abort_flag) {
      stop = 0;
    } else {
      for (int u = 0; u < n_my; ++u)
        unit_epilogue(blockIdx.x + u * gridDim.x, red + (size_t)u * DG_WARPS * 16 * 8);
    }
  } else {
  for (int j = 0; j < n_my; ++j) {
    const int unit = blockIdx.x + j * gridDim.x;
    const int st = j % a.stages;
    unsigned char* stage = stages + (size_t)st * stage_bytes;
    if (!dg_wait(smem_u32(bars + st), (uint32_t)(j / a.stages) & 1u)) abort_flag = 1;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    unit_mma(stage, acc);
    // ---- the warps' sums, added in warp order (red alternates between two halves)
    float* redj = red + (size_t)(j & 1) * DG_WARPS * 16 * 8;
    float* rw = redj + ((size_t)(m * W + ks) * 16) * 8;      // [16 rows][8 tokens]
    rw[g * 8 + 2 * t] = acc[0];
    rw[g * 8 + 2 * t + 1] = acc[1];
    rw[(g + 8) * 8 + 2 * t] = acc[2];
    rw[(g + 8) * 8 + 2 * t + 1] = acc[3];
    __syncthreads();   // every warp is done with this stage and wrote its sums
    if (abort_flag) {
      stop = j;
      break;
    }
    // refill the stage with the unit `stages` ahead
    if (j + a.stages < n_my) {
      if (warp == 0)
        dg_issue_unit<MT, SGN>(a, unit + a.stages * gridDim.x, stage, smem_u32(bars + st), lane);
      ++issued;
    }
    unit_epilogue(unit, redj);
  }
  }
  if (tid == 0 && abort_flag && a.status) atomicCAS(a.status, 0, (int)TL_ERR_TIMEOUT);
  if (abort_flag && tid == 0) {
    // wait (bounded) for the copies still in flight before the CTA leaves:
    // units stop .. issued - 1
    for (int jj = stop; jj < issued; ++jj)
      dg_wait(smem_u32(bars + jj % a.stages), (uint32_t)(jj / a.stages) & 1u);
  }
}

int dg_sm_count() {
  static std::atomic<int> cached{0};
  int n = cached.load();
  if (n > 0) return n;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 148;
  }
  cached.store(n);
  return n;
}

// Shared memory a CTA may take and still leave room on its SM for the next
// kernel's CTA; a unit that does not fit with its activations takes more.
constexpr size_t kDgSmemShare = 110 * 1024;
// the most dynamic shared memory one CTA may take on sm_100 (232448 bytes in
// all) less room for the kernel's static shared memory
constexpr size_t kDgSmemMax = 232448 - 1024;

template <int BITS, int MT, bool NORM, int EPI, int UM, bool SGN, bool WIDE>
tl_status launch_dg_um(const DgArgs& a, int grid, size_t smem, cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  TL_TRY(once_per_device(attr_done, []() -> tl_status {
    TL_CUDA(cudaFuncSetAttribute(gemv_dec_kernel<BITS, MT, NORM, EPI, UM, SGN, WIDE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDgSmemMax));
    return ok();
  }));
  TL_LAUNCH_PDL((gemv_dec_kernel<BITS, MT, NORM, EPI, UM, SGN, WIDE>), grid, DG_THREADS, smem, s, a);
  return ok();
}

template <int BITS, int MT, bool NORM, int EPI, bool SGN, bool WIDE>
tl_status launch_dg(DgArgs a, cudaStream_t s) {
  const int nvec = a.wpr / 4, nch = (nvec + 3) / 4;
  const size_t xw = (size_t)nch * DgFmt<BITS>::CW + 8;
  const size_t row_bytes = (size_t)a.wpr * 4;
  a.row_bytes = (int)row_bytes;
  const size_t stage = (size_t)MT * 2 * (8 * row_bytes + 64) + (size_t)MT * 16 * (a.K / a.G) * 2 +
                       (SGN ? (size_t)MT * 16 * a.spr * 4 : 0);
  const int grid = std::min(a.n_units, dg_sm_count());
  const int per_cta = (a.n_units + grid - 1) / grid;
  const size_t red_unit = (size_t)DG_WARPS * 16 * 8 * 4;
  const size_t fixed0 = (size_t)a.T * xw * 2 + 8 * 8 + 128;
  // every unit resident when they fit (one reduction per launch)
  const int um = per_cta <= 1 ? 1 : per_cta <= 2 ? 2 : per_cta <= 4 ? 4 : per_cta <= 8 ? 8 : 0;
  if (um > 0) {
    const size_t smem = fixed0 + (size_t)std::max(um, 2) * red_unit + (size_t)per_cta * stage;
    if (smem <= kDgSmemMax) {
      a.stages = per_cta;
      switch (um) {
        case 1: return launch_dg_um<BITS, MT, NORM, EPI, 1, SGN, WIDE>(a, grid, smem, s);
        case 2: return launch_dg_um<BITS, MT, NORM, EPI, 2, SGN, WIDE>(a, grid, smem, s);
        case 4: return launch_dg_um<BITS, MT, NORM, EPI, 4, SGN, WIDE>(a, grid, smem, s);
        default: return launch_dg_um<BITS, MT, NORM, EPI, 8, SGN, WIDE>(a, grid, smem, s);
      }
    }
  }
  // a ring of stages, within the share of the SM that leaves room for the next kernel
  const size_t fixed = fixed0 + 2 * red_unit;
  int stages = 1;
  while (stages < per_cta && stages < 8 && fixed + (stages + 1) * stage <= kDgSmemShare) ++stages;
  const size_t smem = fixed + stages * stage;
  if (smem > kDgSmemMax)
    return set_error(TL_ERR_UNSUPPORTED, "decode GEMV: K = %d x %d tokens needs too much shared memory",
                     a.K, a.T);
  a.stages = stages;
  return launch_dg_um<BITS, MT, NORM, EPI, 0, SGN, WIDE>(a, grid, smem, s);
}

}  // namespace

bool dec_gemv_eligible(int N, int K, int T, int bits) {
  return T >= 1 && T <= 8 && N % 16 == 0 && (bits == 3 || K % 128 == 0);
}

tl_status launch_dec_gemv(const DecGemvArgs& d, cudaStream_t s) {
  if (d.T == 0) return ok();
  if (d.T < 0 || d.T > 8) return set_error(TL_ERR_INVALID_ARG, "decode GEMV: %d tokens", d.T);
  if (!dec_gemv_eligible(d.N, d.K, d.T, d.bits))
    return set_error(TL_ERR_UNSUPPORTED, "decode GEMV: shape N %d K %d", d.N, d.K);
  DgArgs a;
  memset(&a, 0, sizeof(a));
  a.w0 = d.w0;
  a.s0 = d.s0;
  a.w1 = d.w1 ? d.w1 : d.w0;
  a.s1 = d.s1 ? d.s1 : d.s0;
  a.g0 = d.g0;
  a.g1 = d.g1 ? d.g1 : d.g0;
  a.spr = d.K / 32;
  a.N = d.N;
  a.K = d.K;
  a.G = d.G;
  a.wpr = d.bits == 4 ? d.K / 8 : ((d.K + 9) / 10 + 3) / 4 * 4;
  a.T = d.T;
  a.n_units = d.N / 16;
  a.x = d.x;
  a.h = d.h;
  a.gamma = d.gamma;
  a.x_out = d.x_out;
  a.eps = d.eps;
  a.out = d.out;
  a.hres = d.hres;
  a.u = d.u;
  a.trace = d.trace;
  a.out_row = d.out_row;
  a.trace_rows = d.trace_rows;
  a.status = d.status;
  a.ex = d.ex;
  const bool norm = d.h != nullptr;
  const bool sg = d.g0 != nullptr;
  if (sg && (d.K % 32 != 0 || (d.epi == DEC_EPI_SWIGLU && d.g1 == nullptr)))
    return set_error(TL_ERR_UNSUPPORTED, "decode GEMV: sign bits need K %% 32 == 0 (and both matrices')");
  // INT4 launches of three to eight rows take kernels with the staging that
  // keeps every row's loads in flight; one or two rows keep the compact one
  const bool wide = d.T > 2;
#define TL_DG4(MT_, NORM_, EPI_)                                                              \
  (sg ? (wide ? launch_dg<4, MT_, NORM_, EPI_, true, true>(a, s)                            \
              : launch_dg<4, MT_, NORM_, EPI_, true, false>(a, s))                          \
      : (wide ? launch_dg<4, MT_, NORM_, EPI_, false, true>(a, s)                           \
              : launch_dg<4, MT_, NORM_, EPI_, false, false>(a, s)))
#define TL_DG3(MT_, NORM_, EPI_) \
  (sg ? launch_dg<3, MT_, NORM_, EPI_, true, false>(a, s) : launch_dg<3, MT_, NORM_, EPI_, false, false>(a, s))
  switch (d.epi) {
    case DEC_EPI_SWIGLU:
      if (!norm) return set_error(TL_ERR_UNSUPPORTED, "decode GEMV: SwiGLU needs the norm prologue");
      return d.bits == 4 ? TL_DG4(2, true, EPI_SWIGLU) : TL_DG3(2, true, EPI_SWIGLU);
    case DEC_EPI_RESID:
      if (norm) return set_error(TL_ERR_UNSUPPORTED, "decode GEMV: residual epilogue takes x");
      return d.bits == 4 ? TL_DG4(1, false, EPI_RESID) : TL_DG3(1, false, EPI_RESID);
    default:
      if (norm) return d.bits == 4 ? TL_DG4(1, true, EPI_OUT) : TL_DG3(1, true, EPI_OUT);
      if (sg) return set_error(TL_ERR_UNSUPPORTED, "decode GEMV: sign bits need the norm prologue here");
      return d.bits == 4 ? (wide ? launch_dg<4, 1, false, EPI_OUT, false, true>(a, s)
                                 : launch_dg<4, 1, false, EPI_OUT, false, false>(a, s))
                         : launch_dg<3, 1, false, EPI_OUT, false, false>(a, s);
  }
#undef TL_DG4
#undef TL_DG3
}

}  // namespace tl
