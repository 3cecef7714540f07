/*
 * tl.h - C ABI of the B200 looped-block library (libtinyloop_b200.so).
 *
 * The library runs the hot path of a weight-shared looped transformer: embed,
 * a few pre-blocks applied once, one shared block applied L times with the same
 * weights, final RMSNorm, no logits ("TinyLoop Framework", the four-step list of
 * the architectural family; "Performance and Memory", "Benchmark Shape
 * Matters").  Prefill and KV-cached decode are both covered ("Production
 * Roadmap", Stage 1: default-on KV-cache decode).
 *
 * Conventions (every function):
 *   - Returns tl_status.  Nothing aborts or exits.  On failure a description is
 *     available from tl_last_error() (thread-local, valid until the next call
 *     on the same thread).
 *   - Argument checks (null pointers, shapes, L range, context overflow, bit
 *     width) happen on the host before any launch; a rejected call launches
 *     nothing and changes no state.
 *   - "device pointer" arguments are caller-owned CUDA device memory (for
 *     example allocated by PyTorch).  The library never frees caller memory.
 *     Where a pointer may be host or device memory it says so.
 *   - Handles (tl_block, tl_model, tl_kv) are library-owned and released by the
 *     matching *_destroy.  A tl_model owns its workspace, RoPE table and CUDA
 *     graphs; a tl_kv owns nothing on the device (its storage is the caller's).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and is asynchronous.  Device-side errors (a bounded wait that ran
 *     out, a non-finite output) are recorded in the model's status word and
 *     returned by tl_sync_status().
 *   - All matrices are row-major.  fp16/bf16 values travel as uint16_t bits.
 */
#ifndef TINYLOOP_B200_TL_H
#define TINYLOOP_B200_TL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tl_stream; /* same type as cudaStream_t */

typedef enum tl_status {
  TL_OK = 0,
  TL_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, L out of range, overflow */
  TL_ERR_CUDA = 2,         /* a CUDA runtime/driver call failed */
  TL_ERR_OOM = 3,          /* a library-owned allocation failed */
  TL_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out */
  TL_ERR_UNSUPPORTED = 5,  /* valid request outside what this build implements */
  TL_ERR_NUMERIC = 6       /* a non-finite value reached an output */
} tl_status;

typedef enum tl_kv_dtype {
  TL_KV_FP16 = 0,  /* K and V as fp16 */
  TL_KV_INT8 = 1,  /* int8 codes + one fp16 scale per (token, head) */
  TL_KV_H = 2      /* store-h: the fp16 input rows x of each block application;
                    * K and V are rebuilt from them at every decode step (see
                    * tl_kv_create) */
} tl_kv_dtype;

/* Description of the last failure on this thread ("" if none). */
const char* tl_last_error(void);

/* ABI version of this header (major * 100 + minor). */
int tl_abi_version(void);

/* ------------------------------------------------------------------------
 * Weight packing.  Group-wise symmetric quantisation along K with one fp16
 * scale per group: INT4 ("TinyLoop Framework", "What Makes It Different":
 * INT2/INT4 low-bit execution) and INT3 ("Current Status", core inference
 * table, INT3 GEMM row: 8 levels, 3 bits per weight, 10 values per 32-bit word,
 * converter --bits 3).
 *
 * Quantisation (both widths, all in IEEE fp32):
 *   scale = fp16_rne(max|w| over the group / qmax)      qmax = 7 (INT4), 3 (INT3)
 *   code  = clamp(rint(w / float(scale)), -qmax-1, qmax)  (rint ties to even;
 *           scale == 0 gives code 0)
 * Canonical packed layout (row n of an [N, K] matrix, row-major):
 *   INT4: K/8 uint32 words per row; u = code + 8; word j holds k = 8j..8j+7,
 *         element 8j+i in bits 4i..4i+3.
 *   INT3: W3 = ceil(K/10) rounded up to a multiple of 4 words per row;
 *         u = code + 4; word j holds k = 10j..10j+9, element 10j+i in bits
 *         3i..3i+2; bits 30-31 zero; unused slots hold u = 4 (code 0).
 *   Scales: fp16 [N, K/group], row-major.
 * ------------------------------------------------------------------------ */

/* Words per packed row for K columns at `bits` (3 or 4). */
tl_status tl_packed_words_per_row(int K, int bits, int* words);

/* Bytes of the packed codes and of the fp16 scales of an [N, K] matrix.
 * Requirements: N >= 1, K >= 1, bits in {3, 4}, group in {64, 128},
 * K % group == 0, and K % 8 == 0 for INT4. */
tl_status tl_packed_bytes(int N, int K, int bits, int group,
                          size_t* code_bytes, size_t* scale_bytes);

/* Quantise and pack an fp32 [N, K] matrix on the device.
 *   w       device pointer, fp32 [N, K]; must be finite.
 *   packed  device pointer, uint32 [N, words_per_row]  (written)
 *   scales  device pointer, fp16   [N, K/group]        (written)
 * Bit-exact with the definition above.  Runs once per matrix, at load time. */
tl_status tl_pack_weights(const float* w, int N, int K, int bits, int group,
                          uint32_t* packed, uint16_t* scales, tl_stream stream);

/* The 1-bit sign-of-frac channel of cross-iteration rounding ("Performance
 * and Memory", "Cross-iteration stochastic rounding": INT4 plus a 1-bit
 * sign-of-frac channel, +25 % storage; "Current Status", architecture-unique
 * features table, deterministic error cancellation row: even loop iterations
 * use the standard rounding, odd iterations apply the sign correction).
 * For element (n, k) with group scale s = the fp16 scale tl_pack_weights
 * wrote and code c:  bit = 1 when s != 0 and the fp32 quotient w / s is
 * greater than c (the rounding went down), else 0.  An odd loop iteration
 * then uses code c + 1 where the bit is set and c - 1 where it is clear: the
 * other neighbour of w / s.
 * Layout: uint32 [N, ceil(K / 32)], row-major; element k of a row is bit
 * k % 32 of word k / 32; bits past K are zero. */
tl_status tl_sign_bits_bytes(int N, int K, size_t* bytes);

/* Write the sign-of-frac bits of an fp32 [N, K] matrix (device pointers).
 *   w       fp32 [N, K], the matrix given to tl_pack_weights
 *   scales  fp16 [N, K/group], the scales tl_pack_weights wrote for it
 *   sign    uint32 [N, ceil(K/32)] (written)
 * Bit-exact with the definition above; same requirements as
 * tl_pack_weights. */
tl_status tl_pack_sign_bits(const float* w, int N, int K, int bits, int group,
                            const uint16_t* scales, uint32_t* sign, tl_stream stream);

/* Test hook: unpack canonical packed words back to int8 codes [N, K]
 * (device pointers). */
tl_status tl_unpack_codes(const uint32_t* packed, int N, int K, int bits,
                          int8_t* codes, tl_stream stream);

/* Per-(token, head) symmetric INT8 KV quantisation ("Performance and Memory",
 * "KV cache INT8" table and the sentence under it: per-token per-head
 * symmetric INT8 with one FP16 scale per (token, head)).  For each row of hd
 * fp16 values x:  scale = fp16_rne(max|x| / 127),  code = clamp(rint(x /
 * float(scale)), -127, 127), scale == 0 gives codes 0; dequantised value is
 * code * scale.
 *   x       device pointer, fp16 [rows, hd]
 *   codes   device pointer, int8 [rows, hd]   (written)
 *   scales  device pointer, fp16 [rows]       (written)
 * Requirements: rows >= 0, 1 <= hd <= 256. */
tl_status tl_kv_quant_int8(const uint16_t* x, int rows, int hd, int8_t* codes,
                           uint16_t* scales, tl_stream stream);

/* Causal self-attention of a prefill (test hook): the block's attention step
 * on its own, with the kernel the block's prefill uses (a tiled kernel with an
 * online softmax: "Production Roadmap", Stage 2, Attention workstream, the
 * tiled prefill kernel; "TinyLoop Framework", table of validated H100
 * numbers, "Full prefill attention" row).  Per head h and query t,
 *   out[t, h] = sum over j <= t of softmax_j(q[t, h] . k[j, h] / sqrt(hd)) v[j, h]
 * with q and k taken as given (the block rotates them before this step).
 * Scores, running maxima, exponentials and sums in fp32; the softmax weights
 * enter the P.V product as fp16; out is rounded to fp16.
 *   q, k, v   device fp16 [T, H * hd], head h in columns [h*hd, (h+1)*hd)
 *   out       device fp16 [T, H * hd]   (written; must not overlap q, k, v)
 * Requirements: 0 <= T <= 8192, 1 <= H <= 256, hd 64 or 128 (other values:
 * TL_ERR_UNSUPPORTED), every pointer 16-byte aligned.  T = 0 does nothing. */
tl_status tl_attention_prefill(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               int T, int H, int hd, uint16_t* out, tl_stream stream);

/* ------------------------------------------------------------------------
 * Blocks.  One pre-norm transformer block: RMSNorm -> fused QKV -> RoPE on q
 * and k -> causal attention -> O projection + residual -> RMSNorm -> SwiGLU
 * (silu(gate) * up) -> down projection + residual.  RoPE is applied on every
 * forward path ("Current Status", model architecture table, RoPE row); the
 * pairing is rotate-half (i, i + head_dim/2), angle = pos * theta^(-2i/hd).
 * The residual stream is fp32 ("Current Status", core inference table: the
 * FP16 residual stream is opt-in, so FP32 is the default).
 * ------------------------------------------------------------------------ */
typedef struct tl_block_desc {
  int d_model;     /* d; 256 * 2^k, at most 8192 */
  int n_heads;     /* H; n_heads * head_dim == d_model (multi-head, no GQA) */
  int head_dim;    /* 64 or 128 */
  int ffn;         /* F; multiple of 128 */
  int bits;        /* 4 or 3 */
  int group;       /* 64 or 128 */
  float eps;       /* RMSNorm epsilon, e.g. 1e-5 */
  float rope_theta;/* e.g. 10000 */
  /* Canonical packed weights (see tl_pack_weights), device pointers.  Rows
   * are output features.  w_qkv is [3d, d] with rows [Q; K; V], head-major. */
  const uint32_t* w_qkv;  const uint16_t* s_qkv;   /* [3d, d] */
  const uint32_t* w_o;    const uint16_t* s_o;     /* [d, d]  */
  const uint32_t* w_gate; const uint16_t* s_gate;  /* [F, d]  */
  const uint32_t* w_up;   const uint16_t* s_up;    /* [F, d]  */
  const uint32_t* w_down; const uint16_t* s_down;  /* [d, F]  */
  const float* gamma_attn;                          /* [d] RMSNorm gain before QKV */
  const float* gamma_ffn;                           /* [d] RMSNorm gain before SwiGLU */
  /* Optional sign-of-frac bits of the five matrices (tl_pack_sign_bits
   * layout), all five or none (NULL): the odd-iteration weights of
   * cross-iteration rounding, used when the block is a model's loop block
   * and tl_model_set_cross_iter turned it on. */
  const uint32_t* sign_qkv;
  const uint32_t* sign_o;
  const uint32_t* sign_gate;
  const uint32_t* sign_up;
  const uint32_t* sign_down;
} tl_block_desc;

typedef struct tl_block tl_block;

/* Validate a block description and wrap it.  The block references the caller's
 * device memory (no copy); that memory must outlive the block and every model
 * built from it.  Every kernel reads the canonical packed words directly, INT3
 * included ("Current Status", core inference table, INT3 GEMM row: 10 values
 * per 32-bit word), so an INT3 block costs its 3.2 bits per weight and
 * nothing more. */
tl_status tl_block_create(const tl_block_desc* desc, tl_block** out);
tl_status tl_block_destroy(tl_block* block);

/* Library-owned device bytes of a block (0: a block allocates nothing). */
tl_status tl_block_device_bytes(const tl_block* block, size_t* bytes);

/* ------------------------------------------------------------------------
 * Models.  Weight memory is tied to unique blocks, not to effective depth
 * ("TinyLoop Framework", "What Makes It Different"): a model references its
 * n_pre + 1 blocks once and L is an argument of every forward call ("Loop count
 * is a runtime knob").
 * ------------------------------------------------------------------------ */
typedef struct tl_model_desc {
  const tl_block* const* pre; /* n_pre blocks applied once each, in order */
  int n_pre;                  /* >= 0 */
  const tl_block* loop;       /* the shared block applied L times */
  const uint16_t* embed;      /* device fp16 [vocab, d] or NULL (hidden-state input only) */
  int vocab;
  const float* gamma_final;   /* device fp32 [d], final RMSNorm gain */
  int max_tokens;             /* largest seq passed to tl_prefill, >= 1 */
  int max_lanes;              /* largest n_lanes passed to tl_decode_step, 1..8 */
  int max_ctx;                /* largest position + 1 any call may reach */
  int max_L;                  /* largest loop count any call may use, 1..64 */
} tl_model_desc;

typedef struct tl_model tl_model;

/* Build a model: allocates the library-owned workspace (sized by max_tokens,
 * max_lanes), the RoPE table (max_ctx) and the status word on the current
 * device.  All blocks must share d_model, n_heads, head_dim and ffn. */
tl_status tl_model_create(const tl_model_desc* desc, tl_model** out);
tl_status tl_model_destroy(tl_model* model);

/* Library-owned device bytes of a model (workspace + tables).  Independent of
 * any L. */
tl_status tl_model_device_bytes(const tl_model* model, size_t* bytes);

/* Enable (default) or disable CUDA-graph replay of the forward calls. */
tl_status tl_model_set_graphs(tl_model* model, int enable);

/* Decode attention splits each lane's context into min(8, ceil(max_ctx / 64))
 * equal chunks (max_ctx of the cache) and merges them in a fixed order; one
 * CTA streams `chunks_per_cta` consecutive chunks.  0 (the default) picks, per
 * call, the fewest chunks per CTA that run all (row, head) pairs in the fewest
 * waves on this GPU.  The result is bit-identical for every value: this is a
 * tuning and testing knob.  Frees the model's captured graphs.
 * Errors: TL_ERR_INVALID_ARG for a NULL model or a value outside [0, 8]. */
tl_status tl_model_set_decode_chunks(tl_model* model, int chunks_per_cta);

/* Per-iteration safety check ("Current Status", architecture-unique features
 * table, per-iteration safety check row: the residual stream's L2 norm is
 * computed every iteration, above a threshold the loop stops; L checkpoints
 * per token).  With tau >= 0, a token (prefill, extend) or lane (decode)
 * whose residual stream leaves loop iteration i - 1 with an L2 norm above tau
 * runs no further residual updates: its stream stays frozen, its output is
 * the final RMSNorm of the frozen stream, and the later iterations' KV slots
 * still receive the K/V its frozen stream produces.  The check costs no extra
 * pass: it reads the sum of squares the iteration's RMSNorm computes anyway.
 * Per-lane loop counts thereby become data-dependent; a lane's result stays
 * independent of the other lanes.  tau < 0 (the default) turns it off.
 * Frees the model's captured graphs.  Errors: TL_ERR_INVALID_ARG for a NULL
 * model, NaN or +infinity. */
tl_status tl_model_set_exit_threshold(tl_model* model, float tau);

/* Cross-iteration rounding ("Performance and Memory", "Cross-iteration
 * stochastic rounding"; "Current Status", architecture-unique features
 * table, deterministic error cancellation row): with on != 0, loop
 * iterations 1, 3, 5, ... (counting from 0) of every forward call run the
 * loop block with each code moved to its other rounding neighbour (code + 1
 * where the block's sign bit is set, code - 1 where it is clear), same
 * scales; iterations 0, 2, ... and the pre-blocks are unchanged.  Every kernel
 * reads the bits next to the packed words; nothing is dequantised ahead.
 * Frees the model's captured graphs.  Errors: TL_ERR_INVALID_ARG for a NULL
 * model or when the loop block has no sign bits. */
tl_status tl_model_set_cross_iter(tl_model* model, int on);

/* Per-iteration weight variants ("Current Status", architecture-unique
 * features table, dual-bit and triple-bit weight swap rows: a low-bit copy of
 * the loop block for the early iterations, a higher-bit one for the later
 * iterations, optionally a third for iteration 0).  Loop iteration i < n runs
 * blocks[i] instead of the loop block (NULL entries keep the loop block);
 * iterations >= n and the pre-blocks are unchanged.  Each block must have the
 * loop block's d_model, n_heads, head_dim, ffn, eps and rope_theta; its bits
 * (3 or 4) and group may differ.  The blocks are referenced, not copied, and
 * must outlive the model (or the next call).  n = 0 clears the variants.
 * With cross-iteration rounding on, an odd iteration uses the sign bits of the
 * block it runs, if that block has them.  Frees the model's captured graphs.
 * Errors: TL_ERR_INVALID_ARG for a NULL model, n < 0 or n > max_L, a NULL
 * `blocks` with n > 0, or a block of another shape. */
tl_status tl_model_set_iteration_blocks(tl_model* model, tl_block* const* blocks, int n);

/* Loop iterations each output row of the last forward call ran (after the
 * stream's work): the loop count L unless the residual-norm check stopped it
 * earlier.  Rows are tokens for tl_prefill / tl_extend and lanes for
 * tl_decode_step.  Synchronises `stream`.
 *   loops  host or device int32 [n] (written) */
tl_status tl_loops_used(tl_model* model, int* loops, int n, tl_stream stream);

/* ------------------------------------------------------------------------
 * KV cache.  Every layer application keeps its own K/V slot: n_pre slots for
 * the pre-blocks and one per loop iteration ("Performance and Memory", "KV
 * cache INT8" table: 10 layers for 2 pre-blocks + L=8).  Lane b has
 * n_pre + L_per_lane[b] slots.
 *
 * Storage is caller-owned: tl_kv_bytes gives the size, the caller allocates
 * one device buffer (256-byte aligned) and tl_kv_create lays the cache out in
 * it.  Layout inside the buffer: a 4 KiB header (per-lane positions), then for
 * each lane b, for each layer l < n_pre + L_b: K [H][max_ctx][hd], V
 * [H][max_ctx][hd] (fp16, or int8 codes), then for INT8 the scales K
 * [H][max_ctx], V [H][max_ctx] (fp16); every region starts on 256 bytes.
 * K is stored after RoPE.
 *
 * TL_KV_H (store-h: "Current Status", KV cache mode table, Store-h (FP16) and
 * tensor-core reconstruction rows; "Claims & Data Sources", h-mode KV
 * reconstruction from shared W_k / W_v): a slot holds, per position, the fp16
 * row x = RMSNorm(h) * gamma_attn that the layer's QKV projection read
 * ([max_ctx][d], d values instead of the 2d of K and V).  At every decode step
 * each layer rebuilds the K and V of a lane's cached positions from those
 * rows with the layer's own W_k, W_v (the quantised-weight GEMM on the tensor
 * cores, RoPE after it) into a workspace that follows the slots in the same
 * buffer (a header, one fp16 K/V layer per lane and the GEMM's partial sums),
 * then attends over them.  Prefill and decode steps support it; tl_extend and
 * tl_spec_step return TL_ERR_UNSUPPORTED.  A decode step rebuilds every
 * position below the lane's position rounded up to a multiple of 128 (at most
 * max_ctx), so its captured graph serves 128 consecutive steps.
 * ------------------------------------------------------------------------ */
typedef struct tl_kv tl_kv;

/* Bytes of one (lane, layer) slot: 2 * align256(H * max_ctx * hd * elem)
 * plus, for INT8, 2 * align256(H * max_ctx * 2) of fp16 scales; for TL_KV_H
 * align256(max_ctx * H * hd * 2).  Host-only. */
tl_status tl_kv_layer_bytes(int n_heads, int head_dim, int max_ctx, tl_kv_dtype dtype,
                            size_t* bytes);

/* Bytes of the cache buffer for n_lanes lanes of max_ctx positions each, lane
 * b running L_per_lane[b] loop iterations: the 4 KiB header, every lane's
 * n_pre + L_b slots (tl_kv_layer_bytes each) and, for TL_KV_H, the rebuild
 * workspace.  Host-only.  Errors: TL_ERR_INVALID_ARG for a NULL model,
 * L_per_lane or bytes, n_lanes outside [1, 8], max_ctx outside [1, the
 * model's max_ctx], an L outside [1, max_L] or an unknown dtype. */
tl_status tl_kv_bytes(const tl_model* model, int n_lanes, int max_ctx,
                      const int* L_per_lane /* host [n_lanes] */,
                      tl_kv_dtype dtype, size_t* bytes);
/* Lays a cache out in `buffer` (device, caller-owned, 256-byte aligned, at
 * least tl_kv_bytes bytes) and sets every lane's position to 0.  The handle
 * references the buffer and the model, which must outlive it; tl_kv_destroy
 * releases the handle (and the model's graphs captured for it), never the
 * buffer.  Errors: those of tl_kv_bytes; TL_ERR_INVALID_ARG for a NULL `out`,
 * a NULL, misaligned or short buffer; TL_ERR_CUDA if the header upload fails. */
tl_status tl_kv_create(const tl_model* model, int n_lanes, int max_ctx,
                       const int* L_per_lane /* host [n_lanes] */,
                       tl_kv_dtype dtype, void* buffer, size_t buffer_bytes,
                       tl_kv** out);
tl_status tl_kv_destroy(tl_kv* kv);
/* Set the position of one lane (lane >= 0) or of every lane (lane == -1) to
 * 0.  Enqueued on `stream`. */
tl_status tl_kv_reset(tl_kv* kv, int lane, tl_stream stream);
/* Host-side position (number of cached tokens) of a lane. */
tl_status tl_kv_position(const tl_kv* kv, int lane, int* pos);
/* Declare that positions 0..pos-1 of a lane already hold valid entries (for a
 * cache filled by the caller through tl_kv_layer_ptrs). */
tl_status tl_kv_set_position(tl_kv* kv, int lane, int pos, tl_stream stream);
/* Device pointers of one (lane, layer) slot: K, V ([H][max_ctx][hd]) and, for
 * INT8, the scales ([H][max_ctx]; NULL for FP16).  TL_KV_H: *k receives the
 * fp16 rows x [max_ctx][d]; *v and the scales are NULL. */
tl_status tl_kv_layer_ptrs(const tl_kv* kv, int lane, int layer, void** k,
                           void** v, uint16_t** k_scale, uint16_t** v_scale);

/* ------------------------------------------------------------------------
 * Forward calls.  Input and output pointers may be host or device memory
 * (copies to and from the model's workspace are enqueued on `stream`; host
 * memory should be pinned for asynchronous copies).
 * ------------------------------------------------------------------------ */

/* Causal prefill of `seq` tokens at positions 0..seq-1 of one lane.
 *   ids      int32 [seq] token ids (needs an embedding), or NULL
 *   h_in     fp16 [seq, d] input hidden states, or NULL (exactly one of the two)
 *   L        loop count, 1..max_L (and <= the lane's L when kv is given)
 *   kv       cache to fill (positions 0..seq-1 of `lane`, position set to seq),
 *            or NULL for an uncached forward
 *   y_out    fp32 [seq, d]: final RMSNorm of the residual stream (no logits)
 *   h_trace  NULL, or fp32 [n_pre + L, seq, d]: the residual stream after each
 *            block application (a test hook)
 * The sequence is processed as one CUDA graph per (seq, L, lane, kv). */
tl_status tl_prefill(tl_model* model, const int32_t* ids, const uint16_t* h_in,
                     int seq, int L, tl_kv* kv, int lane, float* y_out,
                     float* h_trace, tl_stream stream);

/* One cached decode step for lanes 0..n_lanes-1 of `kv`: each lane appends
 * one token at its current position and runs with its own loop count
 * ("Current Status", architecture-unique table, L-aware batching row:
 * per-lane loops, each lane bit-exact with its own run).
 *   ids         int32 [n_lanes], or NULL
 *   h_in        fp16 [n_lanes, d], or NULL (exactly one of the two)
 *   L_per_lane  host int [n_lanes]; 1 <= L_b <= the L the lane's cache holds
 *   y_out       fp32 [n_lanes, d]
 *   h_trace     NULL, or fp32 [n_pre + max_b L_b, n_lanes, d]; rows of lanes
 *               that ran fewer iterations keep their last value
 * A lane's result does not depend on the other lanes or on n_lanes. */
tl_status tl_decode_step(tl_model* model, tl_kv* kv, const int32_t* ids,
                         const uint16_t* h_in, const int* L_per_lane,
                         int n_lanes, float* y_out, float* h_trace,
                         tl_stream stream);

/* Cached forward of `n` consecutive tokens of one lane at its current
 * position p (positions p .. p+n-1), at loop count L: the verify pass of
 * self-speculative decode ("Current Status", speculative and adaptive decode
 * table, self-speculative row: L=2 draft, L=8 verify with the same weights;
 * "TinyLoop Framework", "What Makes It Different": draft and verify reuse the
 * same weights).  Every layer appends the n tokens' K/V to the lane's cache
 * before any of them attends, and token i attends over positions 0 .. p+i.
 * Each token is computed exactly as a one-token decode step at its position
 * would be: the result is bit-identical to n successive decode steps.
 *   ids / h_in  int32 [n] or fp16 [n, d] (exactly one; host or device)
 *   y_out       fp32 [n, d]  (host or device)
 *   h_trace     NULL or fp32 [n_pre + L, n, d]
 * Requirements: 1 <= n <= 8 (and <= the model's max_tokens), 1 <= L <= the
 * lane's loop slots, p + n <= the cache context.  The lane's position
 * becomes p + n. */
tl_status tl_extend(tl_model* model, tl_kv* kv, int lane, const int32_t* ids,
                    const uint16_t* h_in, int n, int L, float* y_out, float* h_trace,
                    tl_stream stream);

/* Greedy next tokens through the tied embedding (the model's embedding used as
 * its output head; the looped forward itself has no logits):
 *   ids[r] = argmax over v of y[r] . E[v]   (fp32 sums; the lowest v wins a tie)
 *   y    device fp32 [n, d] final-norm outputs;  ids  device int32 [n]
 * Requirements: an embedding in the model, 1 <= n <= 8. */
tl_status tl_greedy_head(tl_model* model, const float* y, int n, int32_t* ids,
                         tl_stream stream);

/* One greedy self-speculative step of one lane with one weight set and one
 * cache ("Current Status", self-speculative row; "TinyLoop Framework", "What
 * Makes It Different").  From the input token `token` at the lane's position
 * p: K draft tokens d_1..d_K by K one-token steps at L_draft, each the greedy
 * head of the previous output; then the lane goes back to p and one extend of
 * [token, d_1 .. d_K] at L_verify gives the verify tokens v_1 .. v_{K+1}; the
 * longest prefix with d_i == v_i (m tokens) is accepted.  Writes
 * d_1 .. d_m, v_{m+1} to tokens_out (host int32 [K + 1]) and m + 1 to *n_out
 * (host); the lane's position becomes p + m + 1 (entries past it are
 * overwritten later).  The emitted tokens are those m + 1 greedy decode steps
 * at L_verify would emit.  Synchronises `stream` once (the acceptance is
 * decided on the host).
 * Requirements: 1 <= K <= 7, L_draft and L_verify within the lane's slots,
 * p + K + 1 <= the cache context, 0 <= token < vocab, an embedding. */
tl_status tl_spec_step(tl_model* model, tl_kv* kv, int lane, int32_t token, int K,
                       int L_draft, int L_verify, int32_t* tokens_out, int* n_out,
                       tl_stream stream);

/* ------------------------------------------------------------------------
 * Quantised-weight linear layer (test and measurement hook).  The GEMM every
 * block projection uses:  y[t, n] = sum_k x[t, k] * code[n, k] * scale[n, k/G]
 * for one canonical INT4 matrix (see tl_pack_weights), fp32 accumulation;
 * split-K partial sums, when the kernel uses them, are added in a fixed order.
 *   packed, scales  device, INT4 canonical [N, K/8] words and fp16 [N, K/G]
 *   x               device fp16 [T, K]
 *   y               device fp32 [T, N]   (written)
 *   workspace       device scratch of tl_linear_workspace_bytes(N, K, T) bytes
 *                   (may be NULL when that size is 0)
 * Requirements: N % 64 == 0, K % 64 == 0, group in {64, 128}, K % group == 0,
 * 1 <= T <= 8192; anything else returns TL_ERR_INVALID_ARG (TL_ERR_UNSUPPORTED
 * for another group size) before any launch.  T <= 8 with K % 128 == 0 runs
 * the decode projection kernel and needs no workspace (size 0). */
tl_status tl_linear_workspace_bytes(int N, int K, int T, size_t* bytes);
tl_status tl_linear(const uint32_t* packed, const uint16_t* scales, int N, int K,
                    int group, const uint16_t* x, int T, float* y,
                    void* workspace, tl_stream stream);

/* tl_linear without a caller workspace, for callers that cannot allocate
 * device memory while they run (memory reserved up front by another
 * allocator, work issued inside someone else's open stream capture, fixed
 * real-time budgets).  The TinyLoop pages have no counterpart of this call.
 * Same arguments and result as tl_linear minus the workspace: the split-K
 * partial sums go to a 4 MiB buffer compiled into the library (held on every
 * GPU that loads it until exit).  Calls needing more than 4 MiB of partial
 * sums (S * T * N * 4 bytes) return TL_ERR_INVALID_ARG before any launch.
 * Allocates nothing.  All calls share the buffer, so calls that overlap on the
 * GPU race; each call overwrites what it reads, so nothing needs clearing.
 * The first call on a device looks up the buffer's device address; make it
 * before any stream capture.  The address is kept for the life of the process:
 * a cudaDeviceReset (or anything else that replaces the device's primary
 * context) after that first call is not supported.  Shape requirements and
 * errors are those of tl_linear. */
tl_status tl_linear_noalloc(const uint32_t* packed, const uint16_t* scales, int N,
                            int K, int group, const uint16_t* x, int T, float* y,
                            tl_stream stream);

/* Test hook for the bounded device waits: runs one kernel whose mbarrier wait
 * can never complete (nothing arrives on it).  The wait gives up after
 * limit_us microseconds (1 .. 2e6) and records TL_ERR_TIMEOUT in the model's
 * status word; read it with tl_sync_status.  The kernel returns normally: no
 * trap, no fault, the context stays usable. */
tl_status tl_check_bounded_wait(tl_model* model, unsigned limit_us, tl_stream stream);

/* Measurement hook: read-bandwidth probe.  Reads `bytes` of device memory at
 * `buf` `passes` times with 128-bit loads spread evenly over every SM, folding
 * the words into a value that decides one store to `sink` (so no load is
 * dropped).  A buffer well under the L2 size stays resident after the first
 * pass, so timing this call with CUDA events measures L2 read bandwidth: the
 * denominator of the L2 term of the decode roofline, t = HBM bytes / HBM
 * bandwidth + L2 bytes / L2 bandwidth, which charges the loop block's re-reads
 * within a step (iterations 2..L reuse the same weights: "TinyLoop Framework",
 * "What Makes It Different") at L2 speed.  A buffer several times the L2 size
 * measures HBM read bandwidth instead.
 *   buf    device pointer, 16-byte aligned; bytes a positive multiple of 16
 *   sink   device pointer, uint32 [2] (written: sink[1] = passes)
 *   passes 1 .. 4096
 * No result is computed; errors are TL_ERR_INVALID_ARG before any launch. */
tl_status tl_read_probe(const void* buf, size_t bytes, int passes, uint32_t* sink,
                        tl_stream stream);

/* Synchronise `stream`, then return and clear the model's device status word
 * (TL_OK, TL_ERR_TIMEOUT or TL_ERR_NUMERIC). */
tl_status tl_sync_status(tl_model* model, tl_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* TINYLOOP_B200_TL_H */
