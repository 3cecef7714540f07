// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/tl.h"

namespace tl {

// ---------------------------------------------------------------- errors
tl_status set_error(tl_status st, const char* fmt, ...);
tl_status ok();

#define TL_CHECK_ARG(cond, ...)                                   \
  do {                                                            \
    if (!(cond)) return ::tl::set_error(TL_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

// A failed runtime call is reported and its error taken out of the runtime's
// last-error slot, so that a later, unrelated launch check does not report it
// again (a sticky error stays with the context whatever is done here).
#define TL_CUDA(call)                                                         \
  do {                                                                        \
    cudaError_t e_ = (call);                                                  \
    if (e_ != cudaSuccess) {                                                  \
      cudaGetLastError();                                                     \
      return ::tl::set_error(TL_ERR_CUDA, "%s failed: %s (%s:%d)", #call,    \
                             cudaGetErrorString(e_), __FILE__, __LINE__);    \
    }                                                                         \
  } while (0)

#define TL_LAUNCH_CHECK() TL_CUDA(cudaGetLastError())

#define TL_TRY(expr)                         \
  do {                                       \
    tl_status s_ = (expr);                   \
    if (s_ != TL_OK) return s_;              \
  } while (0)

// ---------------------------------------------------------------- limits
constexpr int kMaxLanes = 8;
constexpr int kMaxL = 64;
constexpr int kMaxLayers = 16 + kMaxL;   // pre-blocks + loop iterations
constexpr int kKvHeaderBytes = 4096;

// Device status codes written by kernels (same numbers as tl_status).
constexpr int kDevTimeout = TL_ERR_TIMEOUT;
constexpr int kDevNumeric = TL_ERR_NUMERIC;

// KV header at the start of the caller's KV buffer.
struct KvHeader {
  int32_t pos[kMaxLanes];         // cached tokens per lane
  int32_t cum_layers[kMaxLanes];  // layers of all lanes before this one
};

// Per-iteration residual-norm check (see tl_model_set_exit_threshold): a row
// whose residual stream leaves loop iteration i - 1 with an L2 norm above tau
// gets exit_it[row] = i and runs no further residual updates.
struct ExitArgs {
  float tau;                 // < 0: no check
  int32_t* exit_it;          // [rows]: 0 while the row runs, else the iterations it ran
  int check_iter;            // > 0: record check_iter for rows above tau (the norm's input row)
  int skip;                  // 1: rows with exit_it != 0 keep their residual stream
};

// ---------------------------------------------------------------- kernels (host launchers)

// packing (pack.cu)
tl_status launch_pack(const float* w, int N, int K, int bits, int group, uint32_t* packed,
                      uint16_t* scales, cudaStream_t s);
tl_status launch_unpack(const uint32_t* packed, int N, int K, int bits, int8_t* codes,
                        cudaStream_t s);
tl_status launch_pack_sign_bits(const float* w, int N, int K, int bits, int group,
                               const uint16_t* scales, uint32_t* sign, cudaStream_t s);
tl_status launch_kv_quant_int8(const __half* x, int rows, int hd, int8_t* codes, __half* scales,
                               cudaStream_t s);

// quantised-weight GEMM (gemm_mma.cu): part[z][t][n] = sum_{k in split z} x[t][k] * W[n][k]
struct GemmArgs {
  int bits;             // 4, or 3 (canonical INT3 rows, tensor-core kernel only)
  const uint32_t* w0;   // canonical packed words, rows [0, n_split)
  const __half* s0;
  const uint32_t* w1;   // rows [n_split, N) (may equal w0 when n_split == N)
  const __half* s1;
  // sign-of-frac bits of the rows of w0 / w1 (tl_pack_sign_bits layout): when
  // set, the odd-iteration codes (code + 1 where the bit is set, code - 1
  // where clear) are used; tensor-core kernel only
  const uint32_t* g0;
  const uint32_t* g1;
  int n_split;
  int N, K, G;
  const __half* x;      // fp16 [T][K]
  int T;
  float* part;          // fp32 [S][T][N]
  int splits;           // S (from gemm_splits)
  int* status;          // device status word for bounded-wait timeouts (may be null)
  // tensor-core kernel with one split only, for [gate; up] weights (n_split =
  // F, N = 2F): when swiglu_u is set, each CTA takes 64 gate rows and the same
  // 64 up rows and writes swiglu_u[t][f] = fp16(silu(gate) * up) (fp16 [T][F])
  // instead of partial sums
  __half* swiglu_u;
};
// Shape checks shared by the linear-layer entry points (tl_linear and
// tl_linear_noalloc): N, K multiples of 64, group 64 or 128 dividing K,
// 1 <= T <= 8192.
tl_status check_linear(int N, int K, int group, int T);
// Split count of the kernel launch_gemm picks for (N, K, T): the tensor-core
// kernel for T >= 64, the mma.sync register-dequant kernel below that (the
// decode projections use launch_dec_gemv instead).
int gemm_splits(int N, int K, int T, int bits = 4, bool sign = false);
tl_status launch_gemm(const GemmArgs& a, cudaStream_t s);
// the two kernels
int gemm_mma_splits(int N, int K, int T);
tl_status launch_gemm_mma(const GemmArgs& a, cudaStream_t s);
bool gemm_tc_eligible(int N, int K, int T, int bits = 4, bool sign = false);
int gemm_tc_splits(int N, int K, int T);
tl_status launch_gemm_tc(const GemmArgs& a, cudaStream_t s);
tl_status gemm_tc_init();
tl_status launch_bounded_wait_check(int* status, uint64_t limit_ns, cudaStream_t s);
// y[t][n] = sum_{s < S} part[s][t][n], in order s = 0, 1, ...
tl_status launch_split_sum(const float* part, int S, long n, float* y, cudaStream_t s);

// decode-sized projections (gemv_dec.cu): T <= 8 tokens, no split-K, the
// pre-norm, residual add and SwiGLU folded in (see the file's header)
enum DecEpi { DEC_EPI_OUT = 0, DEC_EPI_RESID = 1, DEC_EPI_SWIGLU = 2 };
struct DecGemvArgs {
  const uint32_t* w0;   // canonical packed words (bits 3 or 4) [N][wpr]
  const __half* s0;     // fp16 scales [N][K/G]
  const uint32_t* w1;   // DEC_EPI_SWIGLU: the up matrix (w0 = gate)
  const __half* s1;
  const uint32_t* g0;   // null, or the sign-of-frac bits of w0's rows [N][K/32]: the
  const uint32_t* g1;   //   odd-iteration codes (g1: of w1's rows); K % 128 == 0
  int N, K, G, bits, T;
  const __half* x;      // fp16 [T][K] activations, or null with h set
  const float* h;       // fp32 [T][K] residual stream: x = fp16(rmsnorm(h) * gamma)
  const float* gamma;
  __half* x_out;        // with h: null, or written with those fp16 x rows [T][K]
  float eps;
  int epi;              // DecEpi
  float* out;           // DEC_EPI_OUT: fp32 [T][N]
  float* hres;          // DEC_EPI_RESID: fp32 residual [rows][N], += y
  __half* u;            // DEC_EPI_SWIGLU: fp16 [T][N]
  float* trace;         // DEC_EPI_RESID: null or fp32 [trace_rows][N] (rows by out_row)
  const int32_t* out_row;
  int trace_rows;
  int* status;          // null, or the model status word (a bounded wait that runs out)
  ExitArgs ex;          // norm prologue: record rows above tau; residual epilogue: skip them
};
bool dec_gemv_eligible(int N, int K, int T, int bits);
tl_status launch_dec_gemv(const DecGemvArgs& a, cudaStream_t s);
// The linear-layer hook's kernels: the decode projection kernel for T <= 8
// (no split-K), launch_gemm otherwise (split-K sums in `scratch`, then added
// in split order into y).  linear_splits gives the split count.
int linear_splits(int N, int K, int T);
tl_status launch_linear(const uint32_t* packed, const uint16_t* scales, int N, int K, int group,
                        const uint16_t* x, int T, float* y, float* scratch, cudaStream_t s);

// elementwise (elementwise.cu)
struct EmbedArgs {
  const int32_t* ids;        // [rows] or null
  const __half* h_in;        // [rows][d] or null
  const __half* embed;       // [vocab][d]
  int vocab, d, rows;
  const int32_t* src_row;    // row t reads input row src_row[t] (null = identity)
  float* h;                  // [rows][d]
  int* status;
  int32_t* exit_it;          // null, or [rows]: cleared (every row starts its loop)
};
tl_status launch_embed(const EmbedArgs& a, cudaStream_t s);


struct NormArgs {
  float* h;                  // [rows][d] residual
  int d, rows;               // rows: all rows (trace writes cover all)
  const float* part;         // [S][part_rows][d] partials to add (S may be 0)
  int part_rows;
  int S, n_add;              // rows < n_add get h += sum_s part[s]
  const float* gamma_next;   // rows < n_next: x = fp16(rmsnorm(h) * gamma_next)
  __half* x;
  int n_next;
  const float* gamma_final;  // rows in [fin_lo, fin_hi): y[out_row] = rmsnorm(h) * gamma_final
  float* y;
  int fin_lo, fin_hi;
  float* trace;              // null or [rows][d] (indexed by out_row)
  const int32_t* out_row;    // null = identity
  float eps;
  int* status;
  ExitArgs ex;               // the residual-norm check (tau < 0: off)
  int32_t* loops_out;        // null, or [out rows]: loops run by each row in [fin_lo, fin_hi)
  int L_row[kMaxLanes];      // the row's loop count (rows < kMaxLanes) when L_all == 0
  int L_all;                 // > 0: every row's loop count
};
tl_status launch_residual_norm(const NormArgs& a, cudaStream_t s);

struct RopeKvArgs {
  const float* part;         // [S][rows][3d] QKV partials
  int S, rows, d, H, hd;
  const float2* rope_cs;     // [max_ctx][hd/2] (cos, sin)
  __half* q;                 // [rows][d]
  __half* k;                 // [rows][d] or null
  __half* v;                 // [rows][d] or null
  // cache (null kv_base = uncached)
  char* kv_base;             // start of lane data (after the header)
  const KvHeader* hdr;
  size_t layer_bytes, kv_region_bytes;   // region = K or V array bytes (256-aligned)
  int layer, max_ctx, kv_int8;
  const int32_t* lane_of_row;  // decode: lane of each row; null = prefill of `lane`
  int lane;
  int decode;                  // 1: position = hdr->pos[lane]; 0: position = row index
  int kv_only;                 // 1: part holds [S][rows][2d] K|V sums only; no q is written
  int pos0;                    // decode == 0: position = pos0 + row index
};
tl_status launch_rope_kv(const RopeKvArgs& a, cudaStream_t s);

tl_status launch_swiglu(const float* part, int S, int rows, int F, __half* u, cudaStream_t s);
tl_status launch_set_pos(KvHeader* hdr, int lane, int value, cudaStream_t s);
tl_status launch_advance_pos(KvHeader* hdr, int n_lanes, cudaStream_t s);
tl_status launch_add_pos(KvHeader* hdr, int lane, int n, cudaStream_t s);   // pos[lane] += n
tl_status launch_set_i32(int32_t* p, int value, cudaStream_t s);
// Store-h: row r of x [rows][d] (fp16) goes to row hdr->pos[lane[r]] + off[r]
// of the slot slot[r] ([max_ctx][d]); the position is read on the device, so a
// graph can replay the append at every step.
struct AppendRowsArgs {
  const __half* x;
  int rows, d;
  const KvHeader* hdr;
  __half* slot[kMaxLanes];
  int lane[kMaxLanes];
  int off[kMaxLanes];
};
tl_status launch_append_rows(const AppendRowsArgs& a, cudaStream_t s);

// greedy head over the tied embedding (head.cu): ids[r] = argmax_v y[r] . E[v]
// (lowest v on a tie), n <= 8 rows; part_s / part_v: head_parts() * 8 each
int head_parts();
tl_status launch_greedy_head(const float* y, int n, const __half* E, int V, int d, float* part_s,
                             int* part_v, int32_t* ids, cudaStream_t s);

// attention (attention.cu)
tl_status launch_attn_prefill(const __half* q, const __half* k, const __half* v, __half* out,
                              int T, int H, int hd, cudaStream_t s);
struct DecodeAttnArgs {
  __half* out;               // [rows][d]
  int rows, H, hd, d;
  // q/k/v come from the QKV split-K partials; RoPE, KV append and merge
  const float* qkv_part;     // [S][rows][3d]
  int qkv_S;
  const float2* rope_cs;     // [max_ctx][hd/2]
  const char* kv_base;
  const KvHeader* hdr;
  size_t layer_bytes, kv_region_bytes;
  int layer, max_ctx, kv_int8;
  int row_lane[kMaxLanes];   // lane of each row
  int row_cum[kMaxLanes];    // cache layers of the lanes before that lane
  int row_off[kMaxLanes];    // position of the row's token = the lane's position + row_off
  int mode;                  // 0 append + attend, 1 append only, 2 attend only
  int late_prefetch;         // 1: the cached entries were written by the previous kernel
                             //    (rebuilt K/V): no copy before the dependency wait
  int chunks;                // context chunks per CTA; 0 = fewest waves
  int* status;               // null, or the status word a timed-out merge wait sets
};
tl_status launch_attn_decode_fused(const DecodeAttnArgs& a, cudaStream_t s);

// read-bandwidth probe (probe.cu)
tl_status launch_read_probe(const void* buf, size_t bytes, int passes, uint32_t* sink,
                            cudaStream_t s);

}  // namespace tl
