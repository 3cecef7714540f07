// Quantised-weight GEMM on the 5th-generation tensor cores (tcgen05), for
// prefill-sized token counts:
//   part[z][t][n] = sum over k in split z of x[t][k] * W[n][k],
//   W[n][k] = code[n][k] * scale[n][k / G]  (group-wise symmetric INT4, or INT3
//   read straight from its canonical 10-codes-per-word rows).
//
// One CTA per SM computes 128 weight rows x BN tokens over a range of 64-wide
// k blocks.  Warp roles:
//   * sixteen dequantisation warps (four groups of four, one warp per TMEM
//     lane quadrant; group g takes k blocks i with i % 4 == g; one thread per
//     weight row) read their row's packed words and scale straight from global
//     memory, two of their k blocks ahead in registers (the first before the
//     wait for the previous kernel: weights are constants of the model), turn
//     the 64 codes into fp16 code*scale pairs and store them with tcgen05.st,
//     so the weight tile is the MMA's A operand and never passes through
//     shared memory, which the activation tiles and the MMA keep busy;
//   * one TMA warp streams the activation tiles x[BN tokens][64 k] (fp16,
//     128-byte swizzled, rows past T read as zero) through a ring that the
//     MMAs free one k block at a time;
//   * a watcher warp waits for each batch's activation tiles (and for the
//     A slot's previous batch to be complete) and arrives on the batch's
//     barrier, so neither the MMA warp nor the dequantisation warps wait on
//     them;
//   * the MMA warp issues tcgen05.mma kind::f16 (M 128, N BN, K 16; A from
//     TMEM, B from shared memory, fp32 accumulation in TMEM) per batch of four
//     k blocks.
// The producer, watcher and MMA warps keep all lanes converged and issue from
// one elect.sync-chosen lane: a lone active lane is starved of issue slots by
// the dequantisation warps sharing its SM sub-partition.  The dequantisation
// warps then read the accumulator back with tcgen05.ld, store fp32 partial
// sums (or, for [gate; up] with one split, fp16 silu(gate) * up) and signal an
// "epilogue done" barrier that the MMA warp waits on before it frees TMEM.
// Every wait on an mbarrier is bounded: when a wait runs out the CTA records
// TL_ERR_TIMEOUT, stops issuing work, waits (bounded) for its copies in
// flight, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tl_launch.cuh"

namespace tl {
namespace {

constexpr int BM = 128;            // weight rows per CTA (MMA M)
constexpr int BK = 64;             // k per stage
constexpr int DQ_GROUPS = 4;       // dequantisation groups, each 4 warps (one per TMEM quadrant)
constexpr int DQ_WARPS = 4 * DQ_GROUPS;
constexpr int XTMA_WARP = DQ_WARPS, MMA_WARP = DQ_WARPS + 1, XWAIT_WARP = DQ_WARPS + 2;
constexpr int THREADS = 32 * (DQ_WARPS + 3);
constexpr int TMEM_COLS = 512;     // the whole of TMEM: one CTA per SM
constexpr int A_COLS = BK / 2;     // TMEM columns per A stage (two fp16 per column)
constexpr int BATCH = DQ_GROUPS;   // k blocks per batch: one per dequantisation group
constexpr size_t kMinSmem = 120 * 1024;   // also keeps it to one CTA per SM
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // a bounded wait gives up after 2 s
template <int BN> struct TcCfg {
  static constexpr int X_STAGES = BN >= 128 ? 12 : 16;        // activation ring (k blocks)
  static constexpr int A_BATCHES = (TMEM_COLS - BN) / (A_COLS * BATCH);   // TMEM A ring (batches)
};

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait for the phase with the given parity to complete: false after
// limit_ns of global time.
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(addr), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for the phase with the given parity to complete: false after
// limit_ns of global time.  The clock is read only once the first try fails.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try(addr, parity)) return true;
  const uint64_t start = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(addr, parity)) return true;
    if ((i & 63) == 0 && globaltimer_ns() - start > limit_ns) return false;
  }
}

// The producer and MMA warps run their loops with all 32 lanes converged and
// issue each TMA copy, MMA and commit from one lane chosen by elect.sync: a
// lone active lane issues far more slowly while the dequantisation warps on
// the same SM sub-partition keep its issue slots busy.
__device__ __forceinline__ void tma_issue_elect(uint64_t* bar, uint32_t bytes, void* dst,
                                                const CUtensorMap* map, int x, int y) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n"
      " @e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3, "
      "{%4, %5}], [%0];\n}\n" ::"r"(smem_u32(bar)),
      "r"(bytes), "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  // K-major, 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset
  d |= (uint64_t)1 << 46;                 // descriptor version for sm_100
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

// The four K=16 MMAs of one 64-wide k block (A columns +8, B descriptor +2
// (32 bytes) per step), then a commit that frees the block's activation slot;
// called by the whole warp, issued by the lane elect.sync picks (the same lane
// every time, so its commits track its own MMAs).
__device__ __forceinline__ void mma_kblock(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, bool accumulate, uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred p, e;\n .reg .b64 b1, b2, b3;\n .reg .b32 a1, a2, a3;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
      " add.u32 a1, %1, 8;\n add.u32 a2, %1, 16;\n add.u32 a3, %1, 24;\n"
      " elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, 1;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, 1;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Bounded wait (when needed) by lane 0 with the outcome (and the CTA's abort flag) broadcast
// to the warp, so the warp stays converged.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const int* abort_flag,
                                          bool needed) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0)
    ok = (!needed || mbar_wait(bar, parity)) && !*(volatile const int*)abort_flag;
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

struct TcArgs {
  int N, K, G, T, n_split;   // n_split % 128 == 0
  int wpr;                   // packed words per row (K / 8 for INT4, the padded INT3 row)
  int splits;                // split z covers k blocks [z*nkb/S, (z+1)*nkb/S)
  const uint32_t* w0;        // canonical INT4 words of rows [0, n_split)
  const uint32_t* w1;        // rows [n_split, N)
  const __half* s0;
  const __half* s1;
  const uint32_t* g0;        // sign-of-frac bits [rows][K / 32] of w0's / w1's rows (SGN)
  const uint32_t* g1;
  float* part;
  int* status;
  __half* swiglu_u;          // fused SwiGLU epilogue: fp16 [T][n_split] (N = 2 * n_split)
};

// The elected lane arrives once on a barrier for the whole warp.
__device__ __forceinline__ void mbar_arrive_elect(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e mbarrier.arrive.shared::cta.b64 _, [%0];\n}\n" ::"r"(smem_u32(bar))
      : "memory");
}

// Cross-iteration rounding: the odd-iteration code is code + 1 where the
// sign-of-frac bit is set and code - 1 where it is clear.  A k block's 64
// sign bits are two words; pair c (codes 2c, 2c + 1) has its bits at 2c and
// 2c + 1.  sign_spread puts the bits of eight pairs of a half word 16 apart
// (even bits stay, odd bits move up 15), so that one shift brings pair c's
// bits to 15 and 31, and pm1 turns those into the fp16 pair (+-1, +-1).
__device__ __forceinline__ uint32_t sign_spread(uint32_t h16) {
  return (h16 & 0x5555u) | ((h16 & 0xAAAAu) << 15);
}
__device__ __forceinline__ uint32_t pm1(uint32_t x) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(x), "r"(0x80008000u), "r"(0xBC00BC00u));
  return d;   // (x & 0x80008000) ^ 0xBC00BC00: bit set -> +1, clear -> -1
}
__device__ __forceinline__ __half2 sign_corr(const uint32_t* gs, int c) {
  const uint32_t d = pm1(gs[c >> 3] << (15 - 2 * (c & 7)));
  return *reinterpret_cast<const __half2*>(&d);
}

// INT3 k block: the 64 codes k0 .. k0 + 63 of one row, k0 = 64m, start at code
// O = k0 mod 10 (0, 4, 8, 2 or 6) of word v[0] of the row's words v[0..7].  O
// is even, so codes 2c and 2c + 1 always share a word: a shift and a mask
// leave the pair at bits 0-5, one multiply by 1 + 2^13 copies it to bits
// 13-18, and a lop3 keeps code 2c at bits 0-2 and code 2c + 1 at bits 16-18
// under the fp16 exponent of 1024; 1024 + u less 1028 is the exact code, then
// the fp16 product with the scale (as for INT4).
template <int O, bool SGN>
__device__ __forceinline__ void int3_kblock(const uint32_t* v, __half2 s2, const uint32_t* gs,
                                            uint32_t* out) {
  const __half2 bias = __halves2half2(__float2half_rn(1028.0f), __float2half_rn(1028.0f));
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const int p = O + 2 * c, q = p / 10, i = p % 10;   // compile-time: i even, i <= 8
    const uint32_t y = ((v[q] >> (3 * i)) & 0x3Fu) * 8193u;
    uint32_t h;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(y), "r"(0x00070007u), "r"(0x64006400u));
    __half2 cv = __hsub2(*reinterpret_cast<__half2*>(&h), bias);
    if (SGN) cv = __hadd2(cv, sign_corr(gs, c));   // odd iteration: the other neighbour
    __half2 wv = __hmul2(cv, s2);
    out[c] = *reinterpret_cast<uint32_t*>(&wv);
  }
}

// 96 registers x 608 threads (58 K of the 64 K register file) still leave
// room for a small CTA of the next or previous kernel on the same SM; at 80
// the compiler schedules the weight loads less freely (gate|up 4% slower),
// and more registers or a third register set of weights gain nothing.
template <int BN, int BITS, bool SGN>
__global__ void __maxnreg__(96)
    gemm_w4_tc_kernel(const __grid_constant__ CUtensorMap map_x, TcArgs a) {
  constexpr int XS = TcCfg<BN>::X_STAGES;
  constexpr int AB = TcCfg<BN>::A_BATCHES;
  constexpr uint32_t X_BYTES = BN * 128;          // BN rows x 64 fp16
  static_assert(BN + AB * BATCH * A_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(AB >= 2 && XS >= 2 * BATCH, "ring depths");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sX = smem;                                        // XS x X_BYTES
  const int nkb_total = a.K / BK;
  const int kb_begin = (int)(((long)blockIdx.z * nkb_total) / a.splits);
  const int nkb = (int)(((long)(blockIdx.z + 1) * nkb_total) / a.splits) - kb_begin;
  const int nbatch = (nkb + BATCH - 1) / BATCH;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + XS * X_BYTES);
  uint64_t* xfull = bars;               // activations of a k block landed
  uint64_t* xempty = xfull + XS;        // MMAs of a k block complete: frees its X slot
  uint64_t* afull = xempty + XS;        // A tiles and activations of a batch ready
  uint64_t* done = afull + AB;          // MMAs of a batch complete: frees its A slots
  uint64_t* accb = done + AB;           // accumulator complete
  uint64_t* epib = accb + 1;            // epilogue finished reading TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epib + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM;
  const int t0 = blockIdx.y * BN;
  // fused SwiGLU: tile rows [0, 64) are gate rows wrow0.., rows [64, 128) the
  // same rows of up
  const bool sw = a.swiglu_u != nullptr;
  const bool second = !sw && m0 >= a.n_split;
  const int wrow0 = sw ? blockIdx.x * (BM / 2) : second ? m0 - a.n_split : m0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int s = 0; s < AB; ++s) {
      mbar_init(&afull[s], DQ_WARPS + 1);   // + the activation watcher
      mbar_init(&done[s], 1);
    }
    mbar_init(accb, 1);
    mbar_init(epib, DQ_WARPS);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&map_x) : "memory");
  }
  __syncwarp();
  if (warp == MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t acc_col = 0;
  const uint32_t a_col0 = BN;

  if (warp == XTMA_WARP) {
    // ---------------------------------------------------------------- activation TMA
    pdl_enter();   // the activations come from the previous kernel
    int issued = 0;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % XS;
      if (!warp_wait(&xempty[s], ((i / XS) - 1) & 1, abort_flag, i >= XS)) {
        if (lane == 0) atomicExch(abort_flag, 1);
        break;
      }
      tma_issue_elect(&xfull[s], X_BYTES, sX + s * X_BYTES, &map_x, (kb_begin + i) * BK, t0);
      issued = i + 1;
    }
    if (lane == 0 && *(volatile int*)abort_flag)
      for (int i = issued > XS ? issued - XS : 0; i < issued; ++i)   // the ones still in flight
        mbar_wait(&xfull[i % XS], (i / XS) & 1);
    __syncwarp();
  } else if (warp == XWAIT_WARP) {
    // ---------------------------------------------------------------- activation watcher
    // waits until a batch's activation tiles have landed and arrives on its
    // afull barrier, so neither the MMA warp nor the dequantisation warps
    // wait on them
    pdl_enter();
    for (int b = 0; b < nbatch; ++b) {
      const int cnt = min(BATCH, nkb - b * BATCH);
      bool okw = true;
      for (int j = 0; j < cnt && okw; ++j) {
        const int i = b * BATCH + j;
        okw = warp_wait(&xfull[i % XS], (i / XS) & 1, abort_flag, true);
      }
      // when the activation ring holds more k blocks than the A ring
      // (XS > AB * BATCH), batch b's tiles can land before the A slot's phase
      // for batch b - AB has completed; arriving then would count towards that
      // phase, so first wait for it
      if (okw && b >= AB) okw = warp_wait(&afull[b % AB], ((b - AB) / AB) & 1, abort_flag, true);
      if (!okw) {
        if (lane == 0) atomicExch(abort_flag, 1);
        break;
      }
      mbar_arrive_elect(&afull[b % AB]);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ---------------------------------------------------------------- MMA
    // per batch: one wait (A tiles written and activations landed), one
    // fence, up to 16 MMAs, one commit per k block (frees its activation
    // slot) and one per batch (frees its A slots)
    pdl_enter();
    const uint32_t idesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    // loop-invariant operands: the X ring's first descriptor (each slot adds
    // X_BYTES >> 4 to the start-address field, which stays below 2^14) and
    // the accumulator / A ring addresses in TMEM
    const uint64_t xdesc0 = smem_desc_sw128(smem_u32(sX));
    const uint32_t d_tm = tmem_base + acc_col;
    int xs = 0;   // X slot of k block i
    for (int b = 0; b < nbatch; ++b) {
      if (!warp_wait(&afull[b % AB], (b / AB) & 1, abort_flag, true)) {
        if (lane == 0) atomicExch(abort_flag, 1);
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int cnt = min(BATCH, nkb - b * BATCH);
      const uint32_t a_b = tmem_base + a_col0 + (b % AB) * BATCH * A_COLS;
      for (int j = 0; j < cnt; ++j) {
        mma_kblock(d_tm, a_b + j * A_COLS, xdesc0 + (uint64_t)(xs * (X_BYTES >> 4)), idesc,
                   (b | j) != 0, &xempty[xs]);
        xs = xs + 1 == XS ? 0 : xs + 1;
      }
      mma_commit_elect(&done[b % AB]);
    }
    mma_commit_elect(accb);   // arrives once all issued MMAs are complete
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- dequant + epilogue
    const int quad = warp & 3;
    const int grp = warp >> 2;                  // this group takes k block grp of every batch
    const int r = quad * 32 + lane;             // weight row within the tile = TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    // this thread's weight row (canonical INT4 words) and scale row
    const int gsh = __ffs(a.G) - 1;             // the group size is 64 or 128
    const size_t wpr = (size_t)a.wpr, gpr = (size_t)a.K >> gsh;
    const uint32_t* wrow;
    const __half* srow;
    const uint32_t* grow = nullptr;   // the row's sign bits (SGN)
    const size_t spr = (size_t)a.K >> 5;
    if (sw) {
      const bool up = r >= BM / 2;
      const size_t row = (size_t)wrow0 + (up ? r - BM / 2 : r);
      wrow = (up ? a.w1 : a.w0) + row * wpr;
      srow = (up ? a.s1 : a.s0) + row * gpr;
      if (SGN) grow = (up ? a.g1 : a.g0) + row * spr;
    } else {
      wrow = (second ? a.w1 : a.w0) + (size_t)(wrow0 + r) * wpr;
      srow = (second ? a.s1 : a.s0) + (size_t)(wrow0 + r) * gpr;
      if (SGN) grow = (second ? a.g1 : a.g0) + (size_t)(wrow0 + r) * spr;
    }
    // The packed words of this row's k block (INT4: 32 bytes; INT3: the three
    // aligned 16-byte vectors holding its 7 or 8 words) and its scale come
    // straight from global memory through the read-only path, two of this
    // group's k blocks ahead in registers (sets 0 and 1 alternate).  Weights
    // are constants of the model: the first loads go out before the wait for
    // the previous kernel.
    struct WSet {
      uint4 a, b, c;
      uint2 sg;   // the k block's 64 sign bits (SGN)
      __half sc;
    };
    WSet set0, set1;
    set0.a = set0.b = set0.c = make_uint4(0u, 0u, 0u, 0u);
    set0.sg = make_uint2(0u, 0u);
    set0.sc = __float2half_rn(0.f);
    set1 = set0;
    auto fetch = [&](int i, WSet& w) {
      if (i < nkb) {
        const int k0 = (kb_begin + i) * BK;
        if (BITS == 4) {
          const uint4* p = reinterpret_cast<const uint4*>(wrow + (size_t)k0 / 8);
          w.a = __ldg(p);
          w.b = __ldg(p + 1);
        } else {
          const int base = (k0 / 10) & ~3;
          const uint4* p = reinterpret_cast<const uint4*>(wrow + base);
          w.a = __ldg(p);
          w.b = __ldg(p + 1);
          w.c = base + 8 < (int)wpr ? __ldg(p + 2) : make_uint4(0u, 0u, 0u, 0u);
        }
        w.sc = __ldg(srow + (k0 >> gsh));
        if (SGN) w.sg = __ldg(reinterpret_cast<const uint2*>(grow + (k0 >> 5)));
      }
    };
    fetch(grp, set0);
    fetch(grp + BATCH, set1);
    const __half2 mul = __halves2half2(__float2half_rn(1.0f), __float2half_rn(0.0625f));
    const __half2 add = __halves2half2(__float2half_rn(-1032.0f), __float2half_rn(-72.0f));
    // one k block of batch b: wait for the A slot, dequantise, store to TMEM,
    // refill the register set with this group's k block two batches on
    auto kblock = [&](int b, WSet& ws) -> bool {
      const int i = b * BATCH + grp;
      // the TMEM slot of this batch is free once batch b - AB is done
      // (a failure elsewhere surfaces here as a timed-out wait)
      if (b >= AB && !mbar_wait(&done[(b - AB) % AB], ((b - AB) / AB) & 1)) return false;
      if (i < nkb) {
        const __half2 s2 = __halves2half2(ws.sc, ws.sc);
        uint32_t gs[4] = {0u, 0u, 0u, 0u};
        if (SGN) {
          gs[0] = sign_spread(ws.sg.x & 0xFFFFu);
          gs[1] = sign_spread(ws.sg.x >> 16);
          gs[2] = sign_spread(ws.sg.y & 0xFFFFu);
          gs[3] = sign_spread(ws.sg.y >> 16);
        }
        uint32_t v[32];
        if (BITS == 4) {
          const uint32_t words[8] = {ws.a.x, ws.a.y, ws.a.z, ws.a.w, ws.b.x, ws.b.y, ws.b.z, ws.b.w};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            // byte c/2... of word c/4: codes of k = 2c (low nibble), 2c + 1 (high)
            const uint32_t bb = c & 3;
            uint32_t x, h;
            asm("prmt.b32 %0, %1, %2, %3;" : "=r"(x) : "r"(words[c >> 2]), "r"(0u),
                "r"(bb | 0x40u | (bb << 8) | 0x4000u));
            asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(x), "r"(0x00F0000Fu), "r"(0x64006400u));
            __half2 cv = __hfma2(*reinterpret_cast<__half2*>(&h), mul, add);   // exact codes
            if (SGN) cv = __hadd2(cv, sign_corr(gs, c));   // odd iteration: the other neighbour
            __half2 wv = __hmul2(cv, s2);                                      // fp16(code * s)
            v[c] = *reinterpret_cast<uint32_t*>(&wv);
          }
        } else {
          // the 8 words from the first code's word on (d = its offset in the
          // aligned vectors), then the k block's alignment case
          const int k0 = (kb_begin + i) * BK;
          const int d = (k0 / 10) & 3;
          const uint32_t u[12] = {ws.a.x, ws.a.y, ws.a.z, ws.a.w, ws.b.x, ws.b.y,
                                  ws.b.z, ws.b.w, ws.c.x, ws.c.y, ws.c.z, ws.c.w};
          uint32_t w8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            w8[j] = d == 0 ? u[j] : d == 1 ? u[j + 1] : d == 2 ? u[j + 2] : u[j + 3];
          switch (k0 % 10) {
            case 0: int3_kblock<0, SGN>(w8, s2, gs, v); break;
            case 2: int3_kblock<2, SGN>(w8, s2, gs, v); break;
            case 4: int3_kblock<4, SGN>(w8, s2, gs, v); break;
            case 6: int3_kblock<6, SGN>(w8, s2, gs, v); break;
            default: int3_kblock<8, SGN>(w8, s2, gs, v); break;
          }
        }
        fetch(i + 2 * BATCH, ws);
        if (b >= AB) asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t taddr = tmem_base + lane_addr + a_col0 + ((b % AB) * BATCH + grp) * A_COLS;
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
            "%27, %28, %29, %30, %31, %32};" ::"r"(taddr),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
            "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
            "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
            "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
            "r"(v[29]), "r"(v[30]), "r"(v[31])
            : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[b % AB]);
      return true;
    };
    // the dequantisation reads only weights and writes only TMEM: it may run
    // ahead of the previous kernel; the epilogue's stores wait for it
    for (int b = 0; b < nbatch; b += 2) {
      if (!kblock(b, set0) || (b + 1 < nbatch && !kblock(b + 1, set1))) {
        atomicExch(abort_flag, 1);
        break;
      }
    }
    pdl_enter();
    // epilogue: accumulator rows = weight rows, columns = tokens
    bool ok = mbar_wait(accb, 0) && !*(volatile int*)abort_flag;
    if (!ok) atomicExch(abort_flag, 1);
    {
      // agree on ok across all dequantisation warps (the SwiGLU epilogue
      // below synchronises groups of four warps)
      uint32_t all;
      asm volatile(
          "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, 1, %2, p;\n"
          " selp.u32 %0, 1, 0, q;\n}\n"
          : "=r"(all)
          : "r"(ok ? 1u : 0u), "n"(32 * DQ_WARPS)
          : "memory");
      ok = all != 0;
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok && sw) {
      // tile rows [0, 64) hold gate, [64, 128) up for the same 64 features;
      // quadrants 2 and 3 pass up through shared memory (the activation ring
      // is idle once the accumulator is complete) to quadrants 0 and 1
      float* xch = reinterpret_cast<float*>(sX) + grp * 32 * (BM / 2);   // [32 tokens][64]
      const int j = r & (BM / 2 - 1);
      const int F = a.n_split;
#pragma unroll 1
      for (int cc = grp; cc < BN / 32; cc += DQ_GROUPS) {
        if (t0 + cc * 32 >= a.T) break;   // uniform across the group
        uint32_t u[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
            "%27, %28, %29, %30, %31}, [%32];"
            : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
              "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
              "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
              "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
              "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
              "=r"(u[31])
            : "r"(tmem_base + lane_addr + acc_col + cc * 32));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (quad >= 2) {
#pragma unroll
          for (int e = 0; e < 32; ++e) xch[e * (BM / 2) + j] = __uint_as_float(u[e]);
        }
        asm volatile("bar.sync %0, %1;" ::"r"(2 + grp), "n"(128) : "memory");
        if (quad < 2) {
          const int tn = min(32, a.T - (t0 + cc * 32));
          __half* o = a.swiglu_u + (size_t)(t0 + cc * 32) * F + wrow0 + j;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (e < tn) {
              // the same arithmetic as the separate SwiGLU kernel on one split
              const float gs = 0.f + __uint_as_float(u[e]);
              const float us = 0.f + xch[e * (BM / 2) + j];
              const float silu = gs / (1.0f + __expf(-gs));
              o[(size_t)e * F] = __float2half_rn(silu * us);
            }
          }
        }
        asm volatile("bar.sync %0, %1;" ::"r"(2 + grp), "n"(128) : "memory");
      }
    } else if (ok) {
      float* out = a.part + (size_t)blockIdx.z * a.T * a.N + (size_t)(m0 + r);
      // this group's 32-token chunks: cc = grp, grp + DQ_GROUPS, ...
#pragma unroll 1
      for (int cc = grp; cc < BN / 32; cc += DQ_GROUPS) {
        if (t0 + cc * 32 >= a.T) break;   // warp-uniform
        uint32_t u[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
            "%27, %28, %29, %30, %31}, [%32];"
            : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
              "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
              "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
              "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
              "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
              "=r"(u[31])
            : "r"(tmem_base + lane_addr + acc_col + cc * 32));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int tn = min(32, a.T - (t0 + cc * 32));
        float* o = out + (size_t)(t0 + cc * 32) * a.N;
        if (tn == 32) {
#pragma unroll
          for (int e = 0; e < 32; ++e) __stcg(o + (size_t)e * a.N, __uint_as_float(u[e]));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e < tn) __stcg(o + (size_t)e * a.N, __uint_as_float(u[e]));
        }
      }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(epib);
  }
  __syncthreads();
  if (warp == MMA_WARP) {
    // free TMEM only once every epilogue warp has finished reading it
    bool ok2 = true;
    if (lane == 0) ok2 = mbar_wait(epib, 0);
    ok2 = __shfl_sync(0xffffffffu, ok2 ? 1 : 0, 0) != 0;
    if (!ok2 && lane == 0) atomicExch(abort_flag, 1);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
  }
  if (warp == MMA_WARP && lane == 0 && *(volatile int*)abort_flag && a.status)
    atomicCAS(a.status, 0, kDevTimeout);
}

// A wait that can never complete: one barrier with an arrival count of 1 that
// nobody arrives on.  The bounded wait gives up after limit_ns and records
// TL_ERR_TIMEOUT, exercising the same path the GEMM pipeline uses.
__global__ void bounded_wait_check_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_ns)) atomicCAS(status, 0, kDevTimeout);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

tl_status get_encoder() {
  if (g_encode) return ok();
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return set_error(TL_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
  return ok();
}

tl_status encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swz) {
  TL_TRY(get_encoder());
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(TL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ok();
}

int tc_tile_n(int T) { return T <= 64 ? 64 : 128; }

template <int BN>
size_t tc_smem_bytes() {
  constexpr int XS = TcCfg<BN>::X_STAGES;
  constexpr int AB = TcCfg<BN>::A_BATCHES;
  size_t b = 1024 + (size_t)XS * BN * 128 + (2 * XS + 2 * AB + 2) * 8 + 16;
  return b < kMinSmem ? kMinSmem : b;
}

template <int BN, int BITS, bool SGN>
tl_status launch_tc_bn(const GemmArgs& g, cudaStream_t s) {
  CUtensorMap mx;
  TL_TRY(encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.x, g.K, g.T, (uint64_t)g.K * 2, BK, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B));
  TcArgs a;
  a.N = g.N;
  a.K = g.K;
  a.G = g.G;
  a.T = g.T;
  a.wpr = BITS == 4 ? g.K / 8 : ((g.K + 9) / 10 + 3) / 4 * 4;
  a.n_split = g.n_split;
  a.splits = g.splits;
  a.w0 = g.w0;
  a.w1 = g.w1;
  a.s0 = g.s0;
  a.s1 = g.s1;
  a.g0 = g.g0;
  a.g1 = g.g1 ? g.g1 : g.g0;
  a.part = g.part;
  a.status = g.status;
  a.swiglu_u = g.swiglu_u;
  const size_t smem = tc_smem_bytes<BN>();
  if (smem > 232448)
    return set_error(TL_ERR_UNSUPPORTED, "tensor-core GEMM needs %zu bytes of shared memory", smem);
  dim3 grid(g.N / BM, (g.T + BN - 1) / BN, g.splits);
  TL_LAUNCH_PDL((gemm_w4_tc_kernel<BN, BITS, SGN>), grid, THREADS, smem, s, mx, a);
  return ok();
}

}  // namespace

tl_status launch_bounded_wait_check(int* status, uint64_t limit_ns, cudaStream_t s) {
  bounded_wait_check_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  TL_LAUNCH_CHECK();
  return ok();
}

// Set-up once per device (driver entry point, shared-memory limit); called
// outside any stream capture.
tl_status gemm_tc_init() {
  static std::atomic<uint64_t> done{0};
  return once_per_device(done, []() -> tl_status {
    TL_TRY(get_encoder());
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<64, 4, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<128, 4, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<64, 3, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<128, 3, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<64, 4, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<128, 4, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<64, 3, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    TL_CUDA(cudaFuncSetAttribute(gemm_w4_tc_kernel<128, 3, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 232448));
    return ok();
  });
}

// Split-K factor for the tensor-core kernel: one CTA per SM, so as many splits
// as fit the 148 SMs in one wave, each at least 3 k blocks long.
int gemm_tc_splits(int N, int K, int T) {
  const int nkb = K / BK;
  const int tiles = (N / BM) * ((T + tc_tile_n(T) - 1) / tc_tile_n(T));
  int s = tiles >= 148 ? 1 : 148 / tiles;
  if (s > nkb / 3) s = nkb / 3;
  return s < 1 ? 1 : s;
}

// INT4 below 64 tokens runs the mma.sync kernel; INT3 runs here at every
// token count (rows past T are read as zero).
bool gemm_tc_eligible(int N, int K, int T, int bits, bool sign) {
  return (T >= 64 || bits == 3 || sign) && T >= 1 && N % BM == 0 && K % BK == 0;
}

tl_status launch_gemm_tc(const GemmArgs& g, cudaStream_t s) {
  if (g.T == 0) return ok();
  if (g.n_split % BM != 0)
    return set_error(TL_ERR_UNSUPPORTED, "tensor-core GEMM needs row split %% 128 == 0");
  if (g.g0 != nullptr && g.K % 64 != 0)
    return set_error(TL_ERR_UNSUPPORTED, "tensor-core GEMM: sign bits need K %% 64 == 0");
  const bool wide = tc_tile_n(g.T) == 128;
  if (g.g0 != nullptr) {
    if (g.bits == 3) return wide ? launch_tc_bn<128, 3, true>(g, s) : launch_tc_bn<64, 3, true>(g, s);
    return wide ? launch_tc_bn<128, 4, true>(g, s) : launch_tc_bn<64, 4, true>(g, s);
  }
  if (g.bits == 3) return wide ? launch_tc_bn<128, 3, false>(g, s) : launch_tc_bn<64, 3, false>(g, s);
  return wide ? launch_tc_bn<128, 4, false>(g, s) : launch_tc_bn<64, 4, false>(g, s);
}

}  // namespace tl
