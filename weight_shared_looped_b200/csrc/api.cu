// C ABI of the looped-block library: argument checks, library-owned objects,
// the loop driver and CUDA-graph replay.
//
// Forward order ("TinyLoop Framework", the four steps of the architectural
// family): embed, the pre-blocks once each, the shared loop block L times with
// the same weights (each application with its own KV slot, "Performance and
// Memory", "KV cache INT8": 10 layers = 2 pre-blocks + L=8), final RMSNorm and
// no output head.  L is an argument of every call ("Loop count is a runtime
// knob"); the weights a model references do not depend on it.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <string>
#include <tuple>
#include <vector>
#include <algorithm>
#include <atomic>

#include "tl_internal.cuh"

#define TL_API extern "C" __attribute__((visibility("default")))

namespace tl {

static thread_local std::string g_last_error;

tl_status set_error(tl_status st, const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

tl_status ok() { return TL_OK; }

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static int words_per_row(int K, int bits) {
  return bits == 4 ? K / 8 : ((K + 9) / 10 + 3) / 4 * 4;
}

static tl_status check_matrix(int N, int K, int bits, int group) {
  TL_CHECK_ARG(N >= 1 && K >= 1, "matrix shape [%d, %d] must be positive", N, K);
  if (bits != 3 && bits != 4)
    return set_error(TL_ERR_UNSUPPORTED, "bits = %d: only 3 and 4 are supported", bits);
  if (group != 64 && group != 128)
    return set_error(TL_ERR_UNSUPPORTED, "group = %d: only 64 and 128 are supported", group);
  TL_CHECK_ARG(K % group == 0, "K = %d is not a multiple of group %d", K, group);
  TL_CHECK_ARG(bits != 4 || K % 8 == 0, "INT4 needs K %% 8 == 0 (K = %d)", K);
  return ok();
}

}  // namespace tl

using namespace tl;

// ============================================================================
// Objects
// ============================================================================
struct tl_block {
  tl_block_desc d;   // every kernel reads the caller's canonical words (INT4 or INT3)
};

struct tl_kv {
  uint64_t id;            // unique per created cache; graphs are keyed on it
  const tl_model* model;
  int n_lanes, max_ctx, dtype;
  int L[kMaxLanes];
  int pos[kMaxLanes];
  char* buffer;
  size_t layer_bytes, region_bytes;
  // store-h workspace (TL_KV_H), after the slots in the same buffer: a header
  // whose cum_layers are 0, 1, 2, ..., one fp16 K/V layer per lane (the
  // rebuilt entries) and the rebuild GEMM's partial sums
  KvHeader* h_hdr = nullptr;
  char* h_kv = nullptr;
  float* h_part = nullptr;
  size_t h_layer_bytes = 0, h_region_bytes = 0;
};

struct RowMap {
  int lane[kMaxLanes];   // lane of each decode row
  int cum[kMaxLanes];    // cache layers of the lanes before it
  int off[kMaxLanes];    // the row's position = its lane's position + off
};

struct GraphEntry {
  cudaGraphExec_t exec = nullptr;
  int32_t* lane_of_row = nullptr;   // device, decode graphs
  uint64_t kv_id = 0;               // cache the graph writes (0 = none)
};

struct tl_model {
  tl_model_desc desc;
  std::vector<const tl_block*> pre;
  const tl_block* loop;
  int d, H, hd, F, Tmax;
  float eps;
  bool graphs = true;
  int decode_chunks = 0;   // context chunks per decode-attention CTA; 0 = automatic
  float exit_tau = -1.f;   // per-iteration residual-norm check threshold; < 0 = off
  bool cross_iter = false; // odd loop iterations take the loop block's other rounding neighbours
  std::vector<const tl_block*> iter_blocks;   // loop iteration i < size(): this block (if set)
  cudaStream_t cap_stream = nullptr;
  // workspace
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int32_t* ids;
  __half* hin;
  float* h;
  __half* x;
  __half* attn;
  __half *q, *k, *v;
  __half* u;
  float* part;
  float* y;
  int32_t* lane_map;
  int32_t* ident_map;    // rows 0..7 -> 0..7 (extend, speculative steps)
  int32_t* spec_ids;     // speculative step: the input token and the drafts [16]
  int32_t* spec_ver;     // speculative step: the verify tokens [16]
  int32_t* exit_it;      // per row: 0 while it runs, else the loop iterations it ran
  int32_t* loops;        // per output row: loop iterations run by the last forward
  float* head_ps;        // greedy head partials [head_parts()][8]
  int* head_pv;
  int* status;
  float2* rope;
  std::map<std::string, GraphEntry> graphs_cache;
};

// ============================================================================
// Misc
// ============================================================================
TL_API const char* tl_last_error(void) { return g_last_error.c_str(); }
TL_API int tl_abi_version(void) { return 101; }

// ============================================================================
// Packing
// ============================================================================
TL_API tl_status tl_packed_words_per_row(int K, int bits, int* words) {
  TL_CHECK_ARG(words != nullptr, "words is NULL");
  TL_CHECK_ARG(K >= 1, "K = %d must be positive", K);
  if (bits != 3 && bits != 4)
    return set_error(TL_ERR_UNSUPPORTED, "bits = %d: only 3 and 4 are supported", bits);
  TL_CHECK_ARG(bits != 4 || K % 8 == 0, "INT4 needs K %% 8 == 0 (K = %d)", K);
  *words = words_per_row(K, bits);
  return ok();
}

TL_API tl_status tl_packed_bytes(int N, int K, int bits, int group, size_t* code_bytes,
                                 size_t* scale_bytes) {
  TL_TRY(check_matrix(N, K, bits, group));
  TL_CHECK_ARG(code_bytes && scale_bytes, "output pointer is NULL");
  *code_bytes = (size_t)N * words_per_row(K, bits) * 4;
  *scale_bytes = (size_t)N * (K / group) * 2;
  return ok();
}

TL_API tl_status tl_pack_weights(const float* w, int N, int K, int bits, int group,
                                 uint32_t* packed, uint16_t* scales, tl_stream stream) {
  TL_TRY(check_matrix(N, K, bits, group));
  TL_CHECK_ARG(w && packed && scales, "NULL device pointer");
  return launch_pack(w, N, K, bits, group, packed, scales, (cudaStream_t)stream);
}

TL_API tl_status tl_sign_bits_bytes(int N, int K, size_t* bytes) {
  TL_CHECK_ARG(bytes != nullptr, "bytes is NULL");
  TL_CHECK_ARG(N >= 1 && K >= 1, "matrix shape [%d, %d] must be positive", N, K);
  *bytes = (size_t)N * ((K + 31) / 32) * 4;
  return ok();
}

TL_API tl_status tl_pack_sign_bits(const float* w, int N, int K, int bits, int group,
                                   const uint16_t* scales, uint32_t* sign, tl_stream stream) {
  TL_TRY(check_matrix(N, K, bits, group));
  TL_CHECK_ARG(w && scales && sign, "NULL device pointer");
  return launch_pack_sign_bits(w, N, K, bits, group, scales, sign, (cudaStream_t)stream);
}

TL_API tl_status tl_unpack_codes(const uint32_t* packed, int N, int K, int bits, int8_t* codes,
                                 tl_stream stream) {
  TL_CHECK_ARG(packed && codes, "NULL device pointer");
  TL_CHECK_ARG(N >= 1 && K >= 1, "matrix shape [%d, %d] must be positive", N, K);
  if (bits != 3 && bits != 4)
    return set_error(TL_ERR_UNSUPPORTED, "bits = %d: only 3 and 4 are supported", bits);
  TL_CHECK_ARG(bits != 4 || K % 8 == 0, "INT4 needs K %% 8 == 0 (K = %d)", K);
  return launch_unpack(packed, N, K, bits, codes, (cudaStream_t)stream);
}

TL_API tl_status tl_kv_quant_int8(const uint16_t* x, int rows, int hd, int8_t* codes,
                                  uint16_t* scales, tl_stream stream) {
  TL_CHECK_ARG(rows >= 0, "rows = %d must be >= 0", rows);
  TL_CHECK_ARG(hd >= 1 && hd <= 256, "hd = %d must be in [1, 256]", hd);
  if (rows == 0) return ok();
  TL_CHECK_ARG(x && codes && scales, "NULL device pointer");
  return launch_kv_quant_int8(reinterpret_cast<const __half*>(x), rows, hd, codes,
                              reinterpret_cast<__half*>(scales), (cudaStream_t)stream);
}

TL_API tl_status tl_attention_prefill(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                      int T, int H, int hd, uint16_t* out, tl_stream stream) {
  TL_CHECK_ARG(T >= 0 && T <= 8192, "T = %d out of [0, 8192]", T);
  TL_CHECK_ARG(H >= 1 && H <= 256, "H = %d out of [1, 256]", H);
  if (hd != 64 && hd != 128)
    return set_error(TL_ERR_UNSUPPORTED, "head_dim = %d: only 64 and 128 are supported", hd);
  if (T == 0) return ok();
  TL_CHECK_ARG(q && k && v && out, "NULL device pointer");
  const uintptr_t any = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out;
  TL_CHECK_ARG((any & 15) == 0, "q, k, v and out must be 16-byte aligned");
  return launch_attn_prefill(reinterpret_cast<const __half*>(q), reinterpret_cast<const __half*>(k),
                             reinterpret_cast<const __half*>(v), reinterpret_cast<__half*>(out), T,
                             H, hd, (cudaStream_t)stream);
}

// ============================================================================
// Blocks
// ============================================================================
TL_API tl_status tl_block_create(const tl_block_desc* desc, tl_block** out) {
  TL_CHECK_ARG(desc && out, "NULL argument");
  *out = nullptr;
  const tl_block_desc& d = *desc;
  TL_CHECK_ARG(d.d_model >= 256 && d.d_model <= 8192 && d.d_model % 256 == 0 &&
                   ((d.d_model / 256) & (d.d_model / 256 - 1)) == 0,
               "d_model = %d must be 256 * 2^k, at most 8192", d.d_model);
  if (d.head_dim != 64 && d.head_dim != 128)
    return set_error(TL_ERR_UNSUPPORTED, "head_dim = %d: only 64 and 128", d.head_dim);
  TL_CHECK_ARG(d.n_heads * d.head_dim == d.d_model,
               "n_heads * head_dim = %d must equal d_model = %d", d.n_heads * d.head_dim,
               d.d_model);
  TL_CHECK_ARG(d.ffn >= 128 && d.ffn % 128 == 0, "ffn = %d must be a multiple of 128", d.ffn);
  TL_TRY(check_matrix(3 * d.d_model, d.d_model, d.bits, d.group));
  TL_TRY(check_matrix(d.ffn, d.d_model, d.bits, d.group));
  TL_TRY(check_matrix(d.d_model, d.ffn, d.bits, d.group));
  TL_CHECK_ARG(d.eps > 0.f && std::isfinite(d.eps), "eps must be positive");
  TL_CHECK_ARG(d.rope_theta > 1.f && std::isfinite(d.rope_theta), "rope_theta must be > 1");
  TL_CHECK_ARG(d.w_qkv && d.s_qkv && d.w_o && d.s_o && d.w_gate && d.s_gate && d.w_up &&
                   d.s_up && d.w_down && d.s_down && d.gamma_attn && d.gamma_ffn,
               "NULL weight pointer in block description");
  const int n_sign = (d.sign_qkv != nullptr) + (d.sign_o != nullptr) + (d.sign_gate != nullptr) +
                     (d.sign_up != nullptr) + (d.sign_down != nullptr);
  TL_CHECK_ARG(n_sign == 0 || n_sign == 5,
               "sign bits: give all five matrices' bits or none (%d given)", n_sign);
  std::unique_ptr<tl_block> b(new tl_block());
  b->d = d;
  *out = b.release();
  return ok();
}

TL_API tl_status tl_block_destroy(tl_block* block) {
  delete block;
  return ok();
}

TL_API tl_status tl_block_device_bytes(const tl_block* block, size_t* bytes) {
  TL_CHECK_ARG(block && bytes, "NULL argument");
  *bytes = 0;   // a block references the caller's packed words; it allocates nothing
  return ok();
}

// ============================================================================
// Models
// ============================================================================
namespace {

struct GemmShape {
  int N, K;
};

size_t part_floats(const tl_model* m, int T) {
  const GemmShape gs[4] = {{3 * m->d, m->d}, {m->d, m->d}, {2 * m->F, m->d}, {m->d, m->F}};
  size_t best = 0;
  for (auto& g : gs)
    for (int bits = 3; bits <= 4; ++bits)
      best = std::max(best, (size_t)gemm_splits(g.N, g.K, T, bits) * T * g.N);
  return best;
}

void free_graph(GraphEntry& g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  if (g.lane_of_row) cudaFree(g.lane_of_row);
}

void free_graphs(tl_model* m) {
  for (auto& kv : m->graphs_cache) free_graph(kv.second);
  m->graphs_cache.clear();
}

// Graphs bake in a cache's buffer and geometry: drop them with the cache.
void free_kv_graphs(tl_model* m, uint64_t kv_id) {
  for (auto it = m->graphs_cache.begin(); it != m->graphs_cache.end();) {
    if (it->second.kv_id == kv_id) {
      free_graph(it->second);
      it = m->graphs_cache.erase(it);
    } else {
      ++it;
    }
  }
}

uint64_t next_kv_id() {
  static std::atomic<uint64_t> counter{1};
  return counter.fetch_add(1);
}

}  // namespace

TL_API tl_status tl_model_create(const tl_model_desc* desc, tl_model** out) {
  TL_CHECK_ARG(desc && out, "NULL argument");
  *out = nullptr;
  const tl_model_desc& md = *desc;
  TL_CHECK_ARG(md.loop != nullptr, "loop block is NULL");
  TL_CHECK_ARG(md.n_pre >= 0 && md.n_pre <= 16, "n_pre = %d must be in [0, 16]", md.n_pre);
  TL_CHECK_ARG(md.n_pre == 0 || md.pre != nullptr, "pre is NULL");
  TL_CHECK_ARG(md.gamma_final != nullptr, "gamma_final is NULL");
  TL_CHECK_ARG(md.max_tokens >= 1 && md.max_tokens <= 8192, "max_tokens = %d out of [1, 8192]",
               md.max_tokens);
  TL_CHECK_ARG(md.max_lanes >= 1 && md.max_lanes <= kMaxLanes, "max_lanes = %d out of [1, %d]",
               md.max_lanes, kMaxLanes);
  TL_CHECK_ARG(md.max_ctx >= md.max_tokens && md.max_ctx <= 65536,
               "max_ctx = %d must be in [max_tokens, 65536]", md.max_ctx);
  TL_CHECK_ARG(md.max_L >= 1 && md.max_L <= kMaxL, "max_L = %d out of [1, %d]", md.max_L, kMaxL);
  TL_CHECK_ARG(md.embed == nullptr || md.vocab >= 1, "vocab must be >= 1 with an embedding");
  const tl_block_desc& ld = md.loop->d;
  for (int i = 0; i < md.n_pre; ++i) {
    TL_CHECK_ARG(md.pre[i] != nullptr, "pre[%d] is NULL", i);
    const tl_block_desc& pd = md.pre[i]->d;
    TL_CHECK_ARG(pd.d_model == ld.d_model && pd.n_heads == ld.n_heads &&
                     pd.head_dim == ld.head_dim && pd.ffn == ld.ffn && pd.eps == ld.eps &&
                     pd.rope_theta == ld.rope_theta,
                 "pre[%d] shape differs from the loop block", i);
  }
  TL_TRY(gemm_tc_init());
  std::unique_ptr<tl_model> m(new tl_model());
  m->desc = md;
  for (int i = 0; i < md.n_pre; ++i) m->pre.push_back(md.pre[i]);
  m->loop = md.loop;
  m->d = ld.d_model;
  m->H = ld.n_heads;
  m->hd = ld.head_dim;
  m->F = ld.ffn;
  m->eps = ld.eps;
  m->Tmax = std::max(md.max_tokens, md.max_lanes);
  const int T = m->Tmax, d = m->d, F = m->F;
  size_t maxpart = 0;
  for (int t = 1; t <= T; ++t) maxpart = std::max(maxpart, part_floats(m.get(), t));
  // workspace layout
  struct Slot {
    void** ptr;
    size_t bytes;
  };
  void* p_ids; void* p_hin; void* p_h; void* p_x; void* p_attn; void* p_q; void* p_k; void* p_v;
  void* p_u; void* p_part; void* p_y; void* p_lid; void* p_status; void* p_rope;
  void* p_ident; void* p_sids; void* p_sver; void* p_hps; void* p_hpv; void* p_exit; void* p_loops;
  Slot slots[] = {
      {&p_ids, (size_t)T * 4},
      {&p_hin, (size_t)T * d * 2},
      {&p_h, (size_t)T * d * 4},
      {&p_x, (size_t)T * d * 2},
      {&p_attn, (size_t)T * d * 2},
      {&p_q, (size_t)T * d * 2},
      {&p_k, (size_t)T * d * 2},
      {&p_v, (size_t)T * d * 2},
      {&p_u, (size_t)T * F * 2},
      {&p_part, maxpart * 4},
      {&p_y, (size_t)T * d * 4},
      {&p_lid, (size_t)kMaxLanes * 4},
      {&p_ident, (size_t)kMaxLanes * 4},
      {&p_exit, (size_t)std::max(T, kMaxLanes) * 4},
      {&p_loops, (size_t)std::max(T, kMaxLanes) * 4},
      {&p_sids, 16 * 4},
      {&p_sver, 16 * 4},
      {&p_hps, (size_t)head_parts() * 8 * 4},
      {&p_hpv, (size_t)head_parts() * 8 * 4},
      {&p_status, 256},
      {&p_rope, (size_t)md.max_ctx * (m->hd / 2) * sizeof(float2)},
  };
  size_t total = 0;
  for (auto& s : slots) total += align256(s.bytes);
  if (cudaMalloc(&m->ws, total) != cudaSuccess)
    return set_error(TL_ERR_OOM, "cannot allocate %zu bytes of model workspace", total);
  m->ws_bytes = total;
  char* base = (char*)m->ws;
  for (auto& s : slots) {
    *s.ptr = base;
    base += align256(s.bytes);
  }
  m->ids = (int32_t*)p_ids;
  m->hin = (__half*)p_hin;
  m->h = (float*)p_h;
  m->x = (__half*)p_x;
  m->attn = (__half*)p_attn;
  m->q = (__half*)p_q;
  m->k = (__half*)p_k;
  m->v = (__half*)p_v;
  m->u = (__half*)p_u;
  m->part = (float*)p_part;
  m->y = (float*)p_y;
  m->lane_map = (int32_t*)p_lid;
  m->ident_map = (int32_t*)p_ident;
  m->exit_it = (int32_t*)p_exit;
  m->loops = (int32_t*)p_loops;
  m->spec_ids = (int32_t*)p_sids;
  m->spec_ver = (int32_t*)p_sver;
  m->head_ps = (float*)p_hps;
  m->head_pv = (int*)p_hpv;
  m->status = (int*)p_status;
  m->rope = (float2*)p_rope;
  // RoPE table: angle = pos * theta^(-2i/hd), computed in double, rounded to fp32
  {
    const int half = m->hd / 2;
    std::vector<float2> tab((size_t)md.max_ctx * half);
    for (int p = 0; p < md.max_ctx; ++p)
      for (int i = 0; i < half; ++i) {
        double inv = std::pow((double)ld.rope_theta, -2.0 * i / m->hd);
        double a = (double)p * inv;
        tab[(size_t)p * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    int32_t ident[kMaxLanes];
    for (int i = 0; i < kMaxLanes; ++i) ident[i] = i;
    cudaError_t e1 = cudaMemcpy(m->rope, tab.data(), tab.size() * sizeof(float2),
                                cudaMemcpyHostToDevice);
    cudaError_t e2 = cudaMemcpy(m->lane_map, ident, sizeof(ident), cudaMemcpyHostToDevice);
    if (e2 == cudaSuccess)
      e2 = cudaMemcpy(m->ident_map, ident, sizeof(ident), cudaMemcpyHostToDevice);
    cudaError_t e3 = cudaMemset(m->status, 0, 256);
    if (e3 == cudaSuccess) e3 = cudaMemset(m->exit_it, 0, (size_t)std::max(T, kMaxLanes) * 4);
    if (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess) {
      cudaFree(m->ws);
      return set_error(TL_ERR_CUDA, "model initialisation copy failed");
    }
  }
  if (cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
    cudaFree(m->ws);
    return set_error(TL_ERR_CUDA, "cannot create the capture stream");
  }
  *out = m.release();
  return ok();
}

TL_API tl_status tl_model_destroy(tl_model* model) {
  if (!model) return ok();
  free_graphs(model);
  if (model->cap_stream) cudaStreamDestroy(model->cap_stream);
  if (model->ws) cudaFree(model->ws);
  delete model;
  return ok();
}

TL_API tl_status tl_model_device_bytes(const tl_model* model, size_t* bytes) {
  TL_CHECK_ARG(model && bytes, "NULL argument");
  *bytes = model->ws_bytes;
  return ok();
}

TL_API tl_status tl_model_set_graphs(tl_model* model, int enable) {
  TL_CHECK_ARG(model, "NULL model");
  model->graphs = enable != 0;
  if (!model->graphs) free_graphs(model);
  return ok();
}

TL_API tl_status tl_model_set_exit_threshold(tl_model* model, float tau) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CHECK_ARG(!std::isnan(tau) && tau != INFINITY, "tau must be a finite threshold or negative");
  model->exit_tau = tau < 0.f ? -1.f : tau;
  free_graphs(model);   // captured graphs hold the old threshold
  return ok();
}

TL_API tl_status tl_model_set_cross_iter(tl_model* model, int on) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CHECK_ARG(!on || model->loop->d.sign_qkv != nullptr,
               "cross-iteration rounding needs a loop block with sign bits");
  model->cross_iter = on != 0;
  free_graphs(model);   // captured graphs hold the old weights of odd iterations
  return ok();
}

TL_API tl_status tl_model_set_iteration_blocks(tl_model* model, tl_block* const* blocks, int n) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CHECK_ARG(n >= 0 && n <= model->desc.max_L, "n = %d out of [0, max_L = %d]", n,
               model->desc.max_L);
  TL_CHECK_ARG(n == 0 || blocks, "blocks is NULL");
  const tl_block_desc& L = model->loop->d;
  for (int i = 0; i < n; ++i) {
    if (!blocks[i]) continue;
    const tl_block_desc& b = blocks[i]->d;
    TL_CHECK_ARG(b.d_model == L.d_model && b.n_heads == L.n_heads && b.head_dim == L.head_dim &&
                     b.ffn == L.ffn && b.eps == L.eps && b.rope_theta == L.rope_theta,
                 "iteration %d: the block's shape differs from the loop block's", i);
  }
  model->iter_blocks.assign(n, nullptr);
  for (int i = 0; i < n; ++i) model->iter_blocks[i] = blocks[i];
  free_graphs(model);   // captured graphs hold the old weights
  return ok();
}

TL_API tl_status tl_loops_used(tl_model* model, int* loops, int n, tl_stream stream) {
  TL_CHECK_ARG(model && loops, "NULL argument");
  TL_CHECK_ARG(n >= 1 && n <= std::max(model->Tmax, kMaxLanes), "n = %d out of range", n);
  TL_CUDA(cudaMemcpyAsync(loops, model->loops, (size_t)n * 4, cudaMemcpyDefault,
                          (cudaStream_t)stream));
  TL_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  return ok();
}

TL_API tl_status tl_model_set_decode_chunks(tl_model* model, int chunks_per_cta) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CHECK_ARG(chunks_per_cta >= 0 && chunks_per_cta <= 8, "chunks_per_cta = %d out of [0, 8]",
               chunks_per_cta);
  model->decode_chunks = chunks_per_cta;
  free_graphs(model);   // captured decode graphs hold the old launch shape
  return ok();
}

// ============================================================================
// KV cache
// ============================================================================
namespace {

void kv_geometry_hd(int H, int hd, int max_ctx, int dtype, size_t* layer, size_t* region) {
  if (dtype == TL_KV_H) {   // the fp16 input rows x [max_ctx][H * hd]
    *region = align256((size_t)max_ctx * H * hd * 2);
    *layer = *region;
    return;
  }
  size_t esz = dtype == TL_KV_INT8 ? 1 : 2;
  size_t r = align256((size_t)H * max_ctx * hd * esz);
  size_t l = 2 * r;
  if (dtype == TL_KV_INT8) l += 2 * align256((size_t)H * max_ctx * 2);
  *layer = l;
  *region = r;
}

void kv_geometry(const tl_model* m, int max_ctx, int dtype, size_t* layer, size_t* region) {
  kv_geometry_hd(m->H, m->hd, max_ctx, dtype, layer, region);
}

// Store-h workspace bytes (after the slots): header, one fp16 K/V layer per
// lane, and the rebuild GEMM's partial sums for up to kRebuildRows rows (the
// largest split count x rows over every row count and weight format).
constexpr int kRebuildRows = 512;   // positions per rebuild GEMM

size_t h_workspace_bytes(const tl_model* m, int n_lanes, int max_ctx, size_t* layer16,
                         size_t* region16, size_t* part_off) {
  kv_geometry(m, max_ctx, TL_KV_FP16, layer16, region16);
  size_t part = 0;
  for (int T = 1; T <= std::min(max_ctx, kRebuildRows); ++T)
    for (int bits = 3; bits <= 4; ++bits)
      for (int sg = 0; sg <= 1; ++sg)
        part = std::max(part, (size_t)gemm_splits(2 * m->d, m->d, T, bits, sg != 0) * T);
  *part_off = kKvHeaderBytes + (size_t)n_lanes * *layer16;
  return *part_off + align256(part * 2 * m->d * sizeof(float));
}

tl_status check_kv_args(const tl_model* m, int n_lanes, int max_ctx, const int* L, int dtype) {
  TL_CHECK_ARG(m, "NULL model");
  TL_CHECK_ARG(n_lanes >= 1 && n_lanes <= kMaxLanes, "n_lanes = %d out of [1, %d]", n_lanes,
               kMaxLanes);
  TL_CHECK_ARG(max_ctx >= 1 && max_ctx <= m->desc.max_ctx,
               "max_ctx = %d out of [1, model max_ctx %d]", max_ctx, m->desc.max_ctx);
  TL_CHECK_ARG(L != nullptr, "L_per_lane is NULL");
  for (int b = 0; b < n_lanes; ++b)
    TL_CHECK_ARG(L[b] >= 1 && L[b] <= m->desc.max_L, "L_per_lane[%d] = %d out of [1, %d]", b,
                 L[b], m->desc.max_L);
  TL_CHECK_ARG(dtype == TL_KV_FP16 || dtype == TL_KV_INT8 || dtype == TL_KV_H,
               "unknown KV dtype %d", dtype);
  return ok();
}

}  // namespace

TL_API tl_status tl_kv_layer_bytes(int n_heads, int head_dim, int max_ctx, tl_kv_dtype dtype,
                                   size_t* bytes) {
  TL_CHECK_ARG(bytes, "bytes is NULL");
  TL_CHECK_ARG(n_heads >= 1 && head_dim >= 1 && max_ctx >= 1, "sizes must be positive");
  TL_CHECK_ARG(dtype == TL_KV_FP16 || dtype == TL_KV_INT8 || dtype == TL_KV_H,
               "unknown KV dtype %d", dtype);
  size_t region;
  kv_geometry_hd(n_heads, head_dim, max_ctx, dtype, bytes, &region);
  return ok();
}

TL_API tl_status tl_kv_bytes(const tl_model* model, int n_lanes, int max_ctx,
                             const int* L_per_lane, tl_kv_dtype dtype, size_t* bytes) {
  TL_TRY(check_kv_args(model, n_lanes, max_ctx, L_per_lane, dtype));
  TL_CHECK_ARG(bytes, "bytes is NULL");
  size_t layer, region;
  kv_geometry(model, max_ctx, dtype, &layer, &region);
  size_t layers = 0;
  for (int b = 0; b < n_lanes; ++b) layers += (size_t)model->desc.n_pre + L_per_lane[b];
  *bytes = kKvHeaderBytes + layers * layer;
  if (dtype == TL_KV_H) {
    size_t l16, r16, poff;
    *bytes += h_workspace_bytes(model, n_lanes, max_ctx, &l16, &r16, &poff);
  }
  return ok();
}

TL_API tl_status tl_kv_create(const tl_model* model, int n_lanes, int max_ctx,
                              const int* L_per_lane, tl_kv_dtype dtype, void* buffer,
                              size_t buffer_bytes, tl_kv** out) {
  TL_CHECK_ARG(out, "out is NULL");
  *out = nullptr;
  size_t need = 0;
  TL_TRY(tl_kv_bytes(model, n_lanes, max_ctx, L_per_lane, dtype, &need));
  TL_CHECK_ARG(buffer != nullptr, "buffer is NULL");
  TL_CHECK_ARG(((uintptr_t)buffer & 255) == 0, "buffer must be 256-byte aligned");
  TL_CHECK_ARG(buffer_bytes >= need, "buffer has %zu bytes, %zu needed", buffer_bytes, need);
  std::unique_ptr<tl_kv> kv(new tl_kv());
  kv->id = next_kv_id();
  kv->model = model;
  kv->n_lanes = n_lanes;
  kv->max_ctx = max_ctx;
  kv->dtype = dtype;
  kv->buffer = (char*)buffer;
  kv_geometry(model, max_ctx, dtype, &kv->layer_bytes, &kv->region_bytes);
  KvHeader hdr;
  memset(&hdr, 0, sizeof(hdr));
  int cum = 0;
  for (int b = 0; b < kMaxLanes; ++b) {
    kv->L[b] = b < n_lanes ? L_per_lane[b] : 0;
    kv->pos[b] = 0;
    hdr.cum_layers[b] = cum;
    if (b < n_lanes) cum += model->desc.n_pre + L_per_lane[b];
  }
  TL_CUDA(cudaMemcpy(buffer, &hdr, sizeof(hdr), cudaMemcpyHostToDevice));
  if (dtype == TL_KV_H) {
    size_t layers = 0, poff = 0;
    for (int b = 0; b < n_lanes; ++b) layers += (size_t)model->desc.n_pre + L_per_lane[b];
    char* ws = (char*)buffer + kKvHeaderBytes + layers * kv->layer_bytes;
    h_workspace_bytes(model, n_lanes, max_ctx, &kv->h_layer_bytes, &kv->h_region_bytes, &poff);
    kv->h_hdr = (KvHeader*)ws;
    kv->h_kv = ws + kKvHeaderBytes;
    kv->h_part = (float*)(ws + poff);
    KvHeader hh;
    memset(&hh, 0, sizeof(hh));
    for (int b = 0; b < kMaxLanes; ++b) hh.cum_layers[b] = b;   // lane b: rebuilt layer b
    TL_CUDA(cudaMemcpy(kv->h_hdr, &hh, sizeof(hh), cudaMemcpyHostToDevice));
  }
  *out = kv.release();
  return ok();
}

TL_API tl_status tl_kv_destroy(tl_kv* kv) {
  if (!kv) return ok();
  free_kv_graphs(const_cast<tl_model*>(kv->model), kv->id);
  delete kv;
  return ok();
}

TL_API tl_status tl_kv_reset(tl_kv* kv, int lane, tl_stream stream) {
  TL_CHECK_ARG(kv, "NULL kv");
  TL_CHECK_ARG(lane >= -1 && lane < kv->n_lanes, "lane = %d out of [-1, %d)", lane, kv->n_lanes);
  TL_TRY(launch_set_pos((KvHeader*)kv->buffer, lane, 0, (cudaStream_t)stream));
  for (int b = 0; b < kv->n_lanes; ++b)
    if (lane < 0 || b == lane) kv->pos[b] = 0;
  return ok();
}

TL_API tl_status tl_kv_position(const tl_kv* kv, int lane, int* pos) {
  TL_CHECK_ARG(kv && pos, "NULL argument");
  TL_CHECK_ARG(lane >= 0 && lane < kv->n_lanes, "lane = %d out of [0, %d)", lane, kv->n_lanes);
  *pos = kv->pos[lane];
  return ok();
}

TL_API tl_status tl_kv_set_position(tl_kv* kv, int lane, int pos, tl_stream stream) {
  TL_CHECK_ARG(kv, "NULL kv");
  TL_CHECK_ARG(lane >= 0 && lane < kv->n_lanes, "lane = %d out of [0, %d)", lane, kv->n_lanes);
  TL_CHECK_ARG(pos >= 0 && pos <= kv->max_ctx, "pos = %d out of [0, %d]", pos, kv->max_ctx);
  TL_TRY(launch_set_pos((KvHeader*)kv->buffer, lane, pos, (cudaStream_t)stream));
  kv->pos[lane] = pos;
  return ok();
}

TL_API tl_status tl_kv_layer_ptrs(const tl_kv* kv, int lane, int layer, void** k, void** v,
                                  uint16_t** k_scale, uint16_t** v_scale) {
  TL_CHECK_ARG(kv && k && v && k_scale && v_scale, "NULL argument");
  TL_CHECK_ARG(lane >= 0 && lane < kv->n_lanes, "lane = %d out of [0, %d)", lane, kv->n_lanes);
  const int layers = kv->model->desc.n_pre + kv->L[lane];
  TL_CHECK_ARG(layer >= 0 && layer < layers, "layer = %d out of [0, %d)", layer, layers);
  int cum = 0;
  for (int b = 0; b < lane; ++b) cum += kv->model->desc.n_pre + kv->L[b];
  char* base = kv->buffer + kKvHeaderBytes + (size_t)(cum + layer) * kv->layer_bytes;
  *k = base;
  *v = kv->dtype == TL_KV_H ? nullptr : base + kv->region_bytes;
  if (kv->dtype == TL_KV_INT8) {
    size_t sreg = (kv->layer_bytes - 2 * kv->region_bytes) / 2;
    *k_scale = (uint16_t*)(base + 2 * kv->region_bytes);
    *v_scale = (uint16_t*)(base + 2 * kv->region_bytes + sreg);
  } else {
    *k_scale = nullptr;
    *v_scale = nullptr;
  }
  return ok();
}

// ============================================================================
// Loop driver
// ============================================================================
namespace {

// The block layer `layer` runs: a pre-block, a per-iteration variant, or the
// loop block.
const tl_block* block_at(const tl_model* m, int layer) {
  if (layer < (int)m->pre.size()) return m->pre[layer];
  const size_t it = (size_t)(layer - (int)m->pre.size());
  return it < m->iter_blocks.size() && m->iter_blocks[it] ? m->iter_blocks[it] : m->loop;
}

// Whether layer `layer` is an odd loop iteration run with the other rounding
// neighbours (cross-iteration rounding on).
bool odd_iteration(const tl_model* m, int layer) {
  const int it = layer - (int)m->pre.size();
  return m->cross_iter && it >= 0 && (it & 1) == 1;
}

GemmArgs gemm_args(const tl_model* m, const tl_block* b, int which, const __half* x, int T,
                   bool odd) {
  const tl_block_desc& d = b->d;
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.bits = d.bits;
  a.G = d.group;
  a.x = x;
  a.T = T;
  a.part = m->part;
  switch (which) {
    case 0:  // QKV
      a.w0 = a.w1 = d.w_qkv;
      a.s0 = a.s1 = (const __half*)d.s_qkv;
      a.g0 = a.g1 = d.sign_qkv;
      a.N = a.n_split = 3 * m->d;
      a.K = m->d;
      break;
    case 1:  // O
      a.w0 = a.w1 = d.w_o;
      a.s0 = a.s1 = (const __half*)d.s_o;
      a.g0 = a.g1 = d.sign_o;
      a.N = a.n_split = m->d;
      a.K = m->d;
      break;
    case 2:  // gate | up
      a.w0 = d.w_gate;
      a.s0 = (const __half*)d.s_gate;
      a.w1 = d.w_up;
      a.s1 = (const __half*)d.s_up;
      a.g0 = d.sign_gate;
      a.g1 = d.sign_up;
      a.n_split = m->F;
      a.N = 2 * m->F;
      a.K = m->d;
      break;
    default:  // down
      a.w0 = a.w1 = d.w_down;
      a.s0 = a.s1 = (const __half*)d.s_down;
      a.g0 = a.g1 = d.sign_down;
      a.N = a.n_split = m->d;
      a.K = m->F;
      break;
  }
  if (!odd) a.g0 = a.g1 = nullptr;
  a.splits = gemm_splits(a.N, a.K, T, a.bits, a.g0 != nullptr);
  a.status = m->status;
  return a;
}

// The residual-norm check for a kernel of layer `layer`: `check_iter` > 0
// records rows above the threshold as having run check_iter iterations; loop
// layers skip the residual updates of rows already stopped.
ExitArgs exit_args(const tl_model* m, int layer, int check_iter) {
  ExitArgs e;
  memset(&e, 0, sizeof(e));
  e.tau = m->exit_tau;
  if (m->exit_tau < 0.f) return e;
  e.exit_it = m->exit_it;
  e.check_iter = check_iter;
  e.skip = layer >= (int)m->pre.size() ? 1 : 0;
  return e;
}

NormArgs norm_args(const tl_model* m, int rows) {
  NormArgs n;
  memset(&n, 0, sizeof(n));
  n.h = m->h;
  n.d = m->d;
  n.rows = rows;
  n.x = m->x;
  n.y = m->y;
  n.eps = m->eps;
  n.status = m->status;
  return n;
}

// One prefill block application (everything after the input RMSNorm, up to
// and including the down projection; the residual add of the down projection
// is done by the next norm).
tl_status enqueue_block_body(tl_model* m, const tl_block* b, int layer, int rows, tl_kv* kv,
                             int lane, cudaStream_t s) {
  const bool odd = odd_iteration(m, layer);
  const bool store_h = kv && kv->dtype == TL_KV_H;
  if (store_h) {
    // store-h: the QKV projection's input rows x go to the slot, positions 0..rows-1
    int cum = 0;
    for (int b = 0; b < lane; ++b) cum += (int)m->pre.size() + kv->L[b];
    char* slot = kv->buffer + kKvHeaderBytes + (size_t)(cum + layer) * kv->layer_bytes;
    TL_CUDA(cudaMemcpyAsync(slot, m->x, (size_t)rows * m->d * 2, cudaMemcpyDeviceToDevice, s));
  }
  // QKV
  GemmArgs g = gemm_args(m, b, 0, m->x, rows, odd);
  TL_TRY(launch_gemm(g, s));
  RopeKvArgs r;
  memset(&r, 0, sizeof(r));
  r.part = m->part;
  r.S = g.splits;
  r.rows = rows;
  r.d = m->d;
  r.H = m->H;
  r.hd = m->hd;
  r.rope_cs = m->rope;
  r.q = m->q;
  r.k = m->k;
  r.v = m->v;
  if (kv && !store_h) {
    r.kv_base = kv->buffer + kKvHeaderBytes;
    r.hdr = (const KvHeader*)kv->buffer;
    r.layer_bytes = kv->layer_bytes;
    r.kv_region_bytes = kv->region_bytes;
    r.layer = layer;
    r.max_ctx = kv->max_ctx;
    r.kv_int8 = kv->dtype == TL_KV_INT8;
  }
  r.lane = lane;
  TL_TRY(launch_rope_kv(r, s));
  TL_TRY(launch_attn_prefill(m->q, m->k, m->v, m->attn, rows, m->H, m->hd, s));
  // O projection, then the residual add of its split-K partial sums and the
  // RMSNorm before the MLP in one norm kernel
  g = gemm_args(m, b, 1, m->attn, rows, odd);
  TL_TRY(launch_gemm(g, s));
  NormArgs n = norm_args(m, rows);
  n.part = m->part;
  n.part_rows = rows;
  n.S = g.splits;
  n.n_add = rows;
  n.gamma_next = b->d.gamma_ffn;
  n.n_next = rows;
  n.ex = exit_args(m, layer, 0);
  TL_TRY(launch_residual_norm(n, s));
  // SwiGLU MLP
  g = gemm_args(m, b, 2, m->x, rows, odd);
  if (gemm_tc_eligible(g.N, g.K, rows, g.bits, g.g0 != nullptr) && g.splits == 1 && m->F % 64 == 0) {
    g.swiglu_u = m->u;   // the GEMM's epilogue forms silu(gate) * up
    TL_TRY(launch_gemm(g, s));
  } else {
    TL_TRY(launch_gemm(g, s));
    TL_TRY(launch_swiglu(m->part, g.splits, rows, m->F, m->u, s));
  }
  g = gemm_args(m, b, 3, m->u, rows, odd);
  TL_TRY(launch_gemm(g, s));
  return ok();
}

// Store-h: positions rebuilt for a lane whose next token sits at
// pos + off: pos + off rounded up to a multiple of 128, capped by the cache.
int rebuild_rows(const tl_kv* kv, int lane, int off) {
  const int p = kv->pos[lane] + off;
  return p == 0 ? 0 : std::min(kv->max_ctx, (p + 127) / 128 * 128);
}

// Store-h: rebuild the K/V of every row's lane at positions 0 .. pos - 1 from
// the slot's fp16 input rows: the quantised-weight GEMM of those rows with the
// W_k, W_v rows of the layer's QKV matrix (odd-iteration codes when `odd`),
// then RoPE into the lane's layer of the workspace (fp16, the standard
// layout the decode attention reads).
tl_status rebuild_kv(tl_model* m, const tl_block_desc& bd, int layer, int rows, tl_kv* kv,
                     const RowMap* rm, bool odd, cudaStream_t s) {
  const int d = m->d;
  const size_t wpr = (size_t)words_per_row(d, bd.bits), gpr = (size_t)(d / bd.group);
  for (int i = 0; i < rows; ++i) {
    const int lane = rm->lane[i];
    // every position below the lane's bucket (the step's position rounded up
    // to a multiple of 128, at most the cache size) is rebuilt: the launch
    // shapes then change only every 128 steps, so a captured graph serves
    // them; rows past the position are rebuilt from whatever the slot holds
    // there and never read
    const int pos = rebuild_rows(kv, lane, rm->off[i]);
    const __half* slot = (const __half*)(kv->buffer + kKvHeaderBytes +
                                         (size_t)(rm->cum[i] + layer) * kv->layer_bytes);
    // positions [p0, p0 + n): one GEMM and one RoPE pass each
    for (int p0 = 0; p0 < pos; p0 += kRebuildRows) {
      const int n = std::min(kRebuildRows, pos - p0);
      GemmArgs g;
      memset(&g, 0, sizeof(g));
      g.bits = bd.bits;
      g.G = bd.group;
      g.x = slot + (size_t)p0 * d;
      g.T = n;
      g.part = kv->h_part;
      g.w0 = g.w1 = bd.w_qkv + (size_t)d * wpr;   // rows d .. 3d: W_k, W_v
      g.s0 = g.s1 = (const __half*)bd.s_qkv + (size_t)d * gpr;
      if (odd && bd.sign_qkv) g.g0 = g.g1 = bd.sign_qkv + (size_t)d * (d / 32);
      g.N = g.n_split = 2 * d;
      g.K = d;
      g.splits = gemm_splits(g.N, g.K, n, g.bits, g.g0 != nullptr);
      g.status = m->status;
      TL_TRY(launch_gemm(g, s));
      RopeKvArgs r;
      memset(&r, 0, sizeof(r));
      r.part = kv->h_part;
      r.S = g.splits;
      r.rows = n;
      r.pos0 = p0;
      r.d = d;
      r.H = m->H;
      r.hd = m->hd;
      r.rope_cs = m->rope;
      r.kv_base = kv->h_kv;
      r.hdr = kv->h_hdr;
      r.layer_bytes = kv->h_layer_bytes;
      r.kv_region_bytes = kv->h_region_bytes;
      r.layer = 0;
      r.max_ctx = kv->max_ctx;
      r.lane = lane;
      r.kv_only = 1;
      TL_TRY(launch_rope_kv(r, s));
    }
  }
  return ok();
}

// One decode block application for `rows` active rows: four decode
// projections (the QKV and gate/up ones form their own pre-norm from the
// residual stream; the O and down ones add into it) around the fused decode
// attention.  `trace` (null or [trace_rows][d], rows by lane) receives the
// residual stream after the block for every row, active or not.
tl_status enqueue_decode_layer(tl_model* m, const tl_block* b, int layer, int rows, tl_kv* kv,
                               const RowMap* rm, const int32_t* lane_of_row, float* trace,
                               int trace_rows, bool split_attn, cudaStream_t s) {
  const tl_block_desc& bd = b->d;
  const int d = m->d, F = m->F;
  const bool odd = odd_iteration(m, layer);
  const bool store_h = kv->dtype == TL_KV_H;
  DecGemvArgs p;
  memset(&p, 0, sizeof(p));
  p.G = bd.group;
  p.bits = bd.bits;
  p.T = rows;
  p.eps = m->eps;
  p.status = m->status;
  // QKV: q, k, v sums -> part [1][rows][3d]
  p.w0 = bd.w_qkv;
  p.s0 = (const __half*)bd.s_qkv;
  p.g0 = odd ? bd.sign_qkv : nullptr;
  p.N = 3 * d;
  p.K = d;
  p.h = m->h;
  p.gamma = bd.gamma_attn;
  p.epi = DEC_EPI_OUT;
  p.out = m->part;
  p.x_out = store_h ? m->x : nullptr;   // store-h: the rows to append to the slots
  {
    const int it = layer - (int)m->pre.size();   // the loop iteration this layer runs
    p.ex = exit_args(m, layer, it >= 1 ? it : 0);
    p.ex.skip = 0;
  }
  TL_TRY(launch_dec_gemv(p, s));
  p.ex = exit_args(m, layer, 0);
  p.x_out = nullptr;
  if (store_h) TL_TRY(rebuild_kv(m, bd, layer, rows, kv, rm, odd, s));
  // RoPE, KV append, split attention and merge in one launch
  DecodeAttnArgs da;
  memset(&da, 0, sizeof(da));
  da.out = m->attn;
  da.rows = rows;
  da.H = m->H;
  da.hd = m->hd;
  da.d = d;
  da.kv_base = kv->buffer + kKvHeaderBytes;
  da.hdr = (const KvHeader*)kv->buffer;
  da.layer_bytes = kv->layer_bytes;
  da.kv_region_bytes = kv->region_bytes;
  da.layer = layer;
  da.max_ctx = kv->max_ctx;
  da.kv_int8 = kv->dtype == TL_KV_INT8;
  for (int i = 0; i < kMaxLanes; ++i) {
    da.row_lane[i] = rm->lane[i];
    da.row_cum[i] = rm->cum[i];
    da.row_off[i] = rm->off[i];
  }
  da.qkv_part = m->part;
  da.qkv_S = 1;
  da.rope_cs = m->rope;
  da.chunks = m->decode_chunks;
  da.status = m->status;
  if (store_h) {
    // attend over the rebuilt entries: lane b's are layer b of the workspace
    da.kv_base = kv->h_kv;
    da.layer_bytes = kv->h_layer_bytes;
    da.kv_region_bytes = kv->h_region_bytes;
    da.layer = 0;
    da.kv_int8 = 0;
    for (int i = 0; i < kMaxLanes; ++i) da.row_cum[i] = rm->lane[i];
    da.late_prefetch = 1;
  }
  if (!split_attn) {
    da.mode = 0;
    TL_TRY(launch_attn_decode_fused(da, s));
  } else {
    // several tokens of one lane: every entry is appended before any row attends
    da.mode = 1;
    TL_TRY(launch_attn_decode_fused(da, s));
    da.mode = 2;
    TL_TRY(launch_attn_decode_fused(da, s));
  }
  if (store_h) {
    // this step's input rows join the slots at the rows' positions (read on
    // the device)
    AppendRowsArgs ar;
    memset(&ar, 0, sizeof(ar));
    ar.x = m->x;
    ar.rows = rows;
    ar.d = d;
    ar.hdr = (const KvHeader*)kv->buffer;
    for (int i = 0; i < rows; ++i) {
      ar.slot[i] = (__half*)(kv->buffer + kKvHeaderBytes + (size_t)(rm->cum[i] + layer) * kv->layer_bytes);
      ar.lane[i] = rm->lane[i];
      ar.off[i] = rm->off[i];
    }
    TL_TRY(launch_append_rows(ar, s));
  }
  // O projection, added into the residual stream
  p.w0 = bd.w_o;
  p.s0 = (const __half*)bd.s_o;
  p.g0 = odd ? bd.sign_o : nullptr;
  p.N = d;
  p.K = d;
  p.h = nullptr;
  p.gamma = nullptr;
  p.x = m->attn;
  p.epi = DEC_EPI_RESID;
  p.out = nullptr;
  p.hres = m->h;
  TL_TRY(launch_dec_gemv(p, s));
  // gate | up with the pre-norm, SwiGLU in the epilogue
  p.w0 = bd.w_gate;
  p.s0 = (const __half*)bd.s_gate;
  p.w1 = bd.w_up;
  p.s1 = (const __half*)bd.s_up;
  p.g0 = odd ? bd.sign_gate : nullptr;
  p.g1 = odd ? bd.sign_up : nullptr;
  p.N = F;
  p.K = d;
  p.x = nullptr;
  p.h = m->h;
  p.gamma = bd.gamma_ffn;
  p.epi = DEC_EPI_SWIGLU;
  p.hres = nullptr;
  p.u = m->u;
  TL_TRY(launch_dec_gemv(p, s));
  // down projection, added into the residual stream (and the trace)
  p.w0 = bd.w_down;
  p.s0 = (const __half*)bd.s_down;
  p.g0 = odd ? bd.sign_down : nullptr;
  p.w1 = nullptr;
  p.s1 = nullptr;
  p.g1 = nullptr;
  p.N = d;
  p.K = F;
  p.h = nullptr;
  p.gamma = nullptr;
  p.x = m->u;
  p.epi = DEC_EPI_RESID;
  p.u = nullptr;
  p.hres = m->h;
  p.trace = trace;
  p.out_row = lane_of_row;
  p.trace_rows = trace_rows;
  TL_TRY(launch_dec_gemv(p, s));
  return ok();
}

tl_status enqueue_prefill(tl_model* m, bool use_ids, int seq, int L, tl_kv* kv, int lane,
                          float* trace, cudaStream_t s) {
  const int n_layers = (int)m->pre.size() + L;
  EmbedArgs e;
  memset(&e, 0, sizeof(e));
  e.ids = use_ids ? m->ids : nullptr;
  e.h_in = m->hin;
  e.embed = (const __half*)m->desc.embed;
  e.vocab = m->desc.vocab;
  e.d = m->d;
  e.rows = seq;
  e.h = m->h;
  e.status = m->status;
  e.exit_it = m->exit_it;
  TL_TRY(launch_embed(e, s));
  NormArgs n = norm_args(m, seq);
  n.gamma_next = block_at(m, 0)->d.gamma_attn;
  n.n_next = seq;
  TL_TRY(launch_residual_norm(n, s));
  for (int layer = 0; layer < n_layers; ++layer) {
    const tl_block* b = block_at(m, layer);
    TL_TRY(enqueue_block_body(m, b, layer, seq, kv, lane, s));
    NormArgs en = norm_args(m, seq);
    en.part = m->part;
    en.part_rows = seq;
    en.S = gemm_splits(m->d, m->F, seq, b->d.bits, odd_iteration(m, layer));
    en.n_add = seq;
    {
      // the stream leaving this layer enters loop iteration it + 1
      const int it = layer - (int)m->pre.size();
      en.ex = exit_args(m, layer, it >= 0 && layer + 1 < n_layers ? it + 1 : 0);
    }
    if (layer + 1 < n_layers) {
      en.gamma_next = block_at(m, layer + 1)->d.gamma_attn;
      en.n_next = seq;
    } else {
      en.gamma_final = m->desc.gamma_final;
      en.fin_lo = 0;
      en.fin_hi = seq;
      en.loops_out = m->loops;
      en.L_all = L;
    }
    if (trace) en.trace = trace + (size_t)layer * seq * m->d;
    TL_TRY(launch_residual_norm(en, s));
  }
  if (kv) TL_TRY(launch_set_pos((KvHeader*)kv->buffer, lane, seq, s));
  return ok();
}

// rows are lanes sorted by L descending; active rows at loop iteration i are
// those with L > i (a prefix).
tl_status enqueue_decode(tl_model* m, tl_kv* kv, bool use_ids, int B, const int* L_sorted,
                         const int32_t* lane_of_row, const RowMap* rm, float* trace,
                         cudaStream_t s) {
  const int n_pre = (int)m->pre.size();
  const int Lmax = L_sorted[0];
  const int n_layers = n_pre + Lmax;
  auto active = [&](int layer) {
    if (layer < n_pre) return B;
    int it = layer - n_pre, c = 0;
    for (int i = 0; i < B; ++i) c += L_sorted[i] > it;
    return c;
  };
  EmbedArgs e;
  memset(&e, 0, sizeof(e));
  e.ids = use_ids ? m->ids : nullptr;
  e.h_in = m->hin;
  e.embed = (const __half*)m->desc.embed;
  e.vocab = m->desc.vocab;
  e.d = m->d;
  e.rows = B;
  e.src_row = lane_of_row;
  e.h = m->h;
  e.status = m->status;
  e.exit_it = m->exit_it;
  TL_TRY(launch_embed(e, s));
  for (int layer = 0; layer < n_layers; ++layer) {
    const int act = active(layer);
    TL_TRY(enqueue_decode_layer(m, block_at(m, layer), layer, act, kv, rm, lane_of_row,
                                trace ? trace + (size_t)layer * B * m->d : nullptr, B, false, s));
  }
  // final RMSNorm of every row (a row's residual stream stops changing after
  // its last iteration)
  NormArgs fin = norm_args(m, B);
  fin.gamma_final = m->desc.gamma_final;
  fin.fin_lo = 0;
  fin.fin_hi = B;
  fin.out_row = lane_of_row;
  fin.loops_out = m->loops;
  fin.ex.exit_it = m->exit_tau >= 0.f ? m->exit_it : nullptr;
  for (int i = 0; i < kMaxLanes; ++i) fin.L_row[i] = i < B ? L_sorted[i] : 0;
  TL_TRY(launch_residual_norm(fin, s));
  TL_TRY(launch_advance_pos((KvHeader*)kv->buffer, B, s));
  return ok();
}

// n consecutive tokens of one lane at its current position: a decode step
// whose rows are those tokens (row r at position pos + r), the attention split
// into an append pass and an attend pass.  Each row's arithmetic is that of a
// one-token decode step at its position.
tl_status enqueue_extend(tl_model* m, tl_kv* kv, int lane, bool use_ids, int n, int L,
                         float* trace, cudaStream_t s) {
  RowMap rm;
  int cum = 0;
  for (int b = 0; b < lane; ++b) cum += (int)m->pre.size() + kv->L[b];
  for (int i = 0; i < kMaxLanes; ++i) {
    rm.lane[i] = lane;
    rm.cum[i] = cum;
    rm.off[i] = i;
  }
  EmbedArgs e;
  memset(&e, 0, sizeof(e));
  e.ids = use_ids ? m->ids : nullptr;
  e.h_in = m->hin;
  e.embed = (const __half*)m->desc.embed;
  e.vocab = m->desc.vocab;
  e.d = m->d;
  e.rows = n;
  e.h = m->h;
  e.status = m->status;
  e.exit_it = m->exit_it;
  TL_TRY(launch_embed(e, s));
  const int n_layers = (int)m->pre.size() + L;
  for (int layer = 0; layer < n_layers; ++layer)
    TL_TRY(enqueue_decode_layer(m, block_at(m, layer), layer, n, kv, &rm, m->ident_map,
                                trace ? trace + (size_t)layer * n * m->d : nullptr, n, true, s));
  NormArgs fin = norm_args(m, n);
  fin.gamma_final = m->desc.gamma_final;
  fin.fin_lo = 0;
  fin.fin_hi = n;
  fin.loops_out = m->loops;
  fin.ex.exit_it = m->exit_tau >= 0.f ? m->exit_it : nullptr;
  fin.L_all = L;
  TL_TRY(launch_residual_norm(fin, s));
  TL_TRY(launch_add_pos((KvHeader*)kv->buffer, lane, n, s));
  return ok();
}

template <typename F>
tl_status run_graph(tl_model* m, const std::string& key, uint64_t kv_id, cudaStream_t stream,
                    F&& enqueue, const int32_t* lane_map = nullptr) {
  if (!m->graphs) return enqueue(stream, nullptr);
  auto it = m->graphs_cache.find(key);
  if (it == m->graphs_cache.end()) {
    if (m->graphs_cache.size() >= 64) free_graphs(m);
    GraphEntry ge;
    ge.kv_id = kv_id;
    if (lane_map) {
      if (cudaMalloc(&ge.lane_of_row, kMaxLanes * 4) != cudaSuccess)
        return set_error(TL_ERR_OOM, "cannot allocate a graph lane map");
      if (cudaMemcpy(ge.lane_of_row, lane_map, kMaxLanes * 4, cudaMemcpyHostToDevice) !=
          cudaSuccess) {
        cudaFree(ge.lane_of_row);
        return set_error(TL_ERR_CUDA, "cannot upload a graph lane map");
      }
    }
    TL_CUDA(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
    tl_status st = enqueue(m->cap_stream, ge.lane_of_row);
    cudaGraph_t graph = nullptr;
    cudaError_t ce = cudaStreamEndCapture(m->cap_stream, &graph);
    if (st != TL_OK || ce != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      if (ge.lane_of_row) cudaFree(ge.lane_of_row);
      if (st != TL_OK) return st;
      return set_error(TL_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(ce));
    }
    ce = cudaGraphInstantiate(&ge.exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ce != cudaSuccess) {
      if (ge.lane_of_row) cudaFree(ge.lane_of_row);
      return set_error(TL_ERR_CUDA, "graph instantiation failed: %s", cudaGetErrorString(ce));
    }
    it = m->graphs_cache.emplace(key, ge).first;
  }
  TL_CUDA(cudaGraphLaunch(it->second.exec, stream));
  return ok();
}

}  // namespace

TL_API tl_status tl_prefill(tl_model* model, const int32_t* ids, const uint16_t* h_in, int seq,
                            int L, tl_kv* kv, int lane, float* y_out, float* h_trace,
                            tl_stream stream) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CHECK_ARG((ids == nullptr) != (h_in == nullptr), "give exactly one of ids and h_in");
  TL_CHECK_ARG(ids == nullptr || model->desc.embed != nullptr, "ids given but no embedding");
  TL_CHECK_ARG(seq >= 1 && seq <= model->desc.max_tokens, "seq = %d out of [1, %d]", seq,
               model->desc.max_tokens);
  TL_CHECK_ARG(L >= 1 && L <= model->desc.max_L, "L = %d out of [1, %d]", L, model->desc.max_L);
  TL_CHECK_ARG(y_out != nullptr, "y_out is NULL");
  if (kv) {
    TL_CHECK_ARG(kv->model == model, "kv was created for another model");
    TL_CHECK_ARG(lane >= 0 && lane < kv->n_lanes, "lane = %d out of [0, %d)", lane, kv->n_lanes);
    TL_CHECK_ARG(L <= kv->L[lane], "L = %d exceeds the %d loop slots of lane %d", L, kv->L[lane],
                 lane);
    TL_CHECK_ARG(seq <= kv->max_ctx, "seq = %d exceeds the cache context %d", seq, kv->max_ctx);
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int d = model->d;
  if (ids) TL_CUDA(cudaMemcpyAsync(model->ids, ids, (size_t)seq * 4, cudaMemcpyDefault, s));
  else TL_CUDA(cudaMemcpyAsync(model->hin, h_in, (size_t)seq * d * 2, cudaMemcpyDefault, s));
  char key[256];
  const uint64_t kv_id = kv ? kv->id : 0;
  snprintf(key, sizeof(key), "P|%d|%d|%llu|%d|%d|%p", seq, L, (unsigned long long)kv_id, lane,
           ids ? 1 : 0, (void*)h_trace);
  const bool use_ids = ids != nullptr;
  TL_TRY(run_graph(model, key, kv_id, s, [&](cudaStream_t cs, int32_t*) {
    return enqueue_prefill(model, use_ids, seq, L, kv, lane, h_trace, cs);
  }));
  TL_CUDA(cudaMemcpyAsync(y_out, model->y, (size_t)seq * d * 4, cudaMemcpyDefault, s));
  if (kv) kv->pos[lane] = seq;
  return ok();
}

TL_API tl_status tl_decode_step(tl_model* model, tl_kv* kv, const int32_t* ids,
                                const uint16_t* h_in, const int* L_per_lane, int n_lanes,
                                float* y_out, float* h_trace, tl_stream stream) {
  TL_CHECK_ARG(model && kv, "NULL model or kv");
  TL_CHECK_ARG(kv->model == model, "kv was created for another model");
  TL_CHECK_ARG((ids == nullptr) != (h_in == nullptr), "give exactly one of ids and h_in");
  TL_CHECK_ARG(ids == nullptr || model->desc.embed != nullptr, "ids given but no embedding");
  TL_CHECK_ARG(n_lanes >= 1 && n_lanes <= kv->n_lanes && n_lanes <= model->desc.max_lanes,
               "n_lanes = %d out of [1, %d]", n_lanes, std::min(kv->n_lanes, model->desc.max_lanes));
  TL_CHECK_ARG(L_per_lane != nullptr && y_out != nullptr, "NULL L_per_lane or y_out");
  for (int b = 0; b < n_lanes; ++b) {
    TL_CHECK_ARG(L_per_lane[b] >= 1 && L_per_lane[b] <= kv->L[b],
                 "L_per_lane[%d] = %d out of [1, %d]", b, L_per_lane[b], kv->L[b]);
    TL_CHECK_ARG(kv->pos[b] + 1 <= kv->max_ctx, "lane %d is full (%d of %d positions)", b,
                 kv->pos[b], kv->max_ctx);
  }
  // sort lanes by L, descending and stable
  int32_t order[kMaxLanes];
  for (int b = 0; b < kMaxLanes; ++b) order[b] = b < n_lanes ? b : 0;
  std::stable_sort(order, order + n_lanes,
                   [&](int a, int b) { return L_per_lane[a] > L_per_lane[b]; });
  int L_sorted[kMaxLanes];
  for (int i = 0; i < n_lanes; ++i) L_sorted[i] = L_per_lane[order[i]];
  // each row's lane and the cache layers before that lane (the cache header's
  // cum_layers), passed to the attention kernel by value
  RowMap rm;
  for (int i = 0; i < kMaxLanes; ++i) {
    rm.off[i] = 0;
    rm.lane[i] = order[i];
    int cum = 0;
    for (int b = 0; b < order[i] && b < kv->n_lanes; ++b) cum += (int)model->pre.size() + kv->L[b];
    rm.cum[i] = cum;
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int d = model->d;
  if (ids) TL_CUDA(cudaMemcpyAsync(model->ids, ids, (size_t)n_lanes * 4, cudaMemcpyDefault, s));
  else TL_CUDA(cudaMemcpyAsync(model->hin, h_in, (size_t)n_lanes * d * 2, cudaMemcpyDefault, s));
  std::string key = "D|" + std::to_string(kv->id) + "|" + std::to_string(n_lanes) + "|" +
                    std::to_string(ids ? 1 : 0) + "|" + std::to_string((uintptr_t)h_trace);
  for (int b = 0; b < n_lanes; ++b) key += "|" + std::to_string(L_per_lane[b]);
  const bool use_ids = ids != nullptr;
  // store-h: the rebuild's row counts change every 128 positions; they are
  // part of the graph key
  if (kv->dtype == TL_KV_H)
    for (int b = 0; b < n_lanes; ++b) key += "|h" + std::to_string(rebuild_rows(kv, b, 0));
  if (model->graphs) {
    TL_TRY(run_graph(
        model, key, kv->id, s,
        [&](cudaStream_t cs, int32_t* lmap) {
          return enqueue_decode(model, kv, use_ids, n_lanes, L_sorted, lmap, &rm, h_trace, cs);
        },
        order));
  } else {
    // without graphs the lane map lives in the model workspace
    TL_CUDA(cudaMemcpyAsync(model->lane_map, order, sizeof(order), cudaMemcpyHostToDevice, s));
    TL_TRY(enqueue_decode(model, kv, use_ids, n_lanes, L_sorted, model->lane_map, &rm, h_trace,
                          s));
  }
  TL_CUDA(cudaMemcpyAsync(y_out, model->y, (size_t)n_lanes * d * 4, cudaMemcpyDefault, s));
  for (int b = 0; b < n_lanes; ++b) kv->pos[b] += 1;
  return ok();
}

namespace {

tl_status check_extend(tl_model* model, tl_kv* kv, int lane, int n, int L) {
  TL_CHECK_ARG(model && kv, "NULL model or kv");
  TL_CHECK_ARG(kv->model == model, "kv was created for another model");
  TL_CHECK_ARG(lane >= 0 && lane < kv->n_lanes, "lane = %d out of [0, %d)", lane, kv->n_lanes);
  TL_CHECK_ARG(n >= 1 && n <= kMaxLanes && n <= model->Tmax, "n = %d out of [1, %d]", n,
               std::min(kMaxLanes, model->Tmax));
  TL_CHECK_ARG(L >= 1 && L <= kv->L[lane], "L = %d out of [1, %d] for lane %d", L, kv->L[lane], lane);
  TL_CHECK_ARG(kv->pos[lane] + n <= kv->max_ctx, "lane %d: %d + %d positions exceed %d", lane,
               kv->pos[lane], n, kv->max_ctx);
  if (kv->dtype == TL_KV_H)
    return set_error(TL_ERR_UNSUPPORTED, "extend and speculative steps need a K/V cache, not store-h");
  return ok();
}

// enqueue an extend of n tokens whose inputs already sit in the model's ids
// (use_ids) or hin buffer; output in model->y [n][d]
tl_status run_extend(tl_model* model, tl_kv* kv, int lane, bool use_ids, int n, int L,
                     float* h_trace, cudaStream_t s) {
  char key[256];
  snprintf(key, sizeof(key), "E|%llu|%d|%d|%d|%d|%p", (unsigned long long)kv->id, lane, n, L,
           use_ids ? 1 : 0, (void*)h_trace);
  TL_TRY(run_graph(model, key, kv->id, s, [&](cudaStream_t cs, int32_t*) {
    return enqueue_extend(model, kv, lane, use_ids, n, L, h_trace, cs);
  }));
  kv->pos[lane] += n;
  return ok();
}

tl_status set_lane_pos(tl_kv* kv, int lane, int pos, cudaStream_t s) {
  TL_TRY(launch_set_pos((KvHeader*)kv->buffer, lane, pos, s));
  kv->pos[lane] = pos;
  return ok();
}

}  // namespace

TL_API tl_status tl_extend(tl_model* model, tl_kv* kv, int lane, const int32_t* ids,
                           const uint16_t* h_in, int n, int L, float* y_out, float* h_trace,
                           tl_stream stream) {
  TL_TRY(check_extend(model, kv, lane, n, L));
  TL_CHECK_ARG((ids == nullptr) != (h_in == nullptr), "give exactly one of ids and h_in");
  TL_CHECK_ARG(ids == nullptr || model->desc.embed != nullptr, "ids given but no embedding");
  TL_CHECK_ARG(y_out != nullptr, "y_out is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  const int d = model->d;
  if (ids) TL_CUDA(cudaMemcpyAsync(model->ids, ids, (size_t)n * 4, cudaMemcpyDefault, s));
  else TL_CUDA(cudaMemcpyAsync(model->hin, h_in, (size_t)n * d * 2, cudaMemcpyDefault, s));
  TL_TRY(run_extend(model, kv, lane, ids != nullptr, n, L, h_trace, s));
  TL_CUDA(cudaMemcpyAsync(y_out, model->y, (size_t)n * d * 4, cudaMemcpyDefault, s));
  return ok();
}

TL_API tl_status tl_greedy_head(tl_model* model, const float* y, int n, int32_t* ids,
                                tl_stream stream) {
  TL_CHECK_ARG(model && y && ids, "NULL argument");
  TL_CHECK_ARG(model->desc.embed != nullptr, "the model has no embedding to use as its head");
  TL_CHECK_ARG(n >= 1 && n <= 8, "n = %d out of [1, 8]", n);
  return launch_greedy_head(y, n, (const __half*)model->desc.embed, model->desc.vocab, model->d,
                            model->head_ps, model->head_pv, ids, (cudaStream_t)stream);
}

TL_API tl_status tl_spec_step(tl_model* model, tl_kv* kv, int lane, int32_t token, int K,
                              int L_draft, int L_verify, int32_t* tokens_out, int* n_out,
                              tl_stream stream) {
  TL_CHECK_ARG(tokens_out && n_out, "NULL output");
  TL_CHECK_ARG(K >= 1 && K <= kMaxLanes - 1, "K = %d out of [1, %d]", K, kMaxLanes - 1);
  TL_TRY(check_extend(model, kv, lane, K + 1, L_verify));
  TL_CHECK_ARG(L_draft >= 1 && L_draft <= kv->L[lane], "L_draft = %d out of [1, %d]", L_draft,
               kv->L[lane]);
  TL_CHECK_ARG(model->desc.embed != nullptr, "the model has no embedding to use as its head");
  TL_CHECK_ARG(token >= 0 && token < model->desc.vocab, "token %d out of the vocabulary", token);
  cudaStream_t s = (cudaStream_t)stream;
  const int p = kv->pos[lane];
  const __half* E = (const __half*)model->desc.embed;
  // draft: K one-token steps at L_draft, each input the previous greedy token
  TL_TRY(launch_set_i32(model->spec_ids, token, s));
  for (int i = 0; i < K; ++i) {
    TL_CUDA(cudaMemcpyAsync(model->ids, model->spec_ids + i, 4, cudaMemcpyDeviceToDevice, s));
    TL_TRY(run_extend(model, kv, lane, true, 1, L_draft, nullptr, s));
    TL_TRY(launch_greedy_head(model->y, 1, E, model->desc.vocab, model->d, model->head_ps,
                              model->head_pv, model->spec_ids + i + 1, s));
  }
  // verify: back to p, the input token and the K drafts at L_verify
  TL_TRY(set_lane_pos(kv, lane, p, s));
  TL_CUDA(cudaMemcpyAsync(model->ids, model->spec_ids, (size_t)(K + 1) * 4,
                          cudaMemcpyDeviceToDevice, s));
  TL_TRY(run_extend(model, kv, lane, true, K + 1, L_verify, nullptr, s));
  TL_TRY(launch_greedy_head(model->y, K + 1, E, model->desc.vocab, model->d, model->head_ps,
                            model->head_pv, model->spec_ver, s));
  int32_t drafts[kMaxLanes + 1], ver[kMaxLanes + 1];
  TL_CUDA(cudaMemcpyAsync(drafts, model->spec_ids, (size_t)(K + 1) * 4, cudaMemcpyDeviceToHost, s));
  TL_CUDA(cudaMemcpyAsync(ver, model->spec_ver, (size_t)(K + 1) * 4, cudaMemcpyDeviceToHost, s));
  TL_CUDA(cudaStreamSynchronize(s));
  // accept the longest matching prefix, then the verify token after it
  int m = 0;
  while (m < K && drafts[m + 1] == ver[m]) ++m;
  for (int i = 0; i < m; ++i) tokens_out[i] = drafts[i + 1];
  tokens_out[m] = ver[m];
  *n_out = m + 1;
  return set_lane_pos(kv, lane, p + m + 1, s);
}

// ============================================================================
// Linear-layer hook
// ============================================================================
namespace tl {
tl_status check_linear(int N, int K, int group, int T) {
  TL_CHECK_ARG(N >= 64 && N % 64 == 0, "N = %d must be a positive multiple of 64", N);
  TL_CHECK_ARG(K >= 64 && K % 64 == 0, "K = %d must be a positive multiple of 64", K);
  if (group != 64 && group != 128)
    return set_error(TL_ERR_UNSUPPORTED, "group = %d: only 64 and 128 are supported", group);
  // every row holds K / group whole scale groups (as tl_pack_weights requires)
  TL_CHECK_ARG(K % group == 0, "K = %d is not a multiple of group %d", K, group);
  TL_CHECK_ARG(T >= 1 && T <= 8192, "T = %d out of [1, 8192]", T);
  return ok();
}
}  // namespace tl

namespace tl {
// Split count of the linear-layer hook: decode-sized calls run the decode
// projection kernel (no split-K), the rest launch_gemm's kernels.
int linear_splits(int N, int K, int T) {
  return dec_gemv_eligible(N, K, T, 4) ? 1 : gemm_splits(N, K, T);
}

tl_status launch_linear(const uint32_t* packed, const uint16_t* scales, int N, int K, int group,
                        const uint16_t* x, int T, float* y, float* scratch, cudaStream_t s) {
  if (dec_gemv_eligible(N, K, T, 4)) {
    DecGemvArgs p;
    memset(&p, 0, sizeof(p));
    p.w0 = packed;
    p.s0 = (const __half*)scales;
    p.N = N;
    p.K = K;
    p.G = group;
    p.bits = 4;
    p.T = T;
    p.x = (const __half*)x;
    p.epi = DEC_EPI_OUT;
    p.out = y;
    return launch_dec_gemv(p, s);
  }
  const int S = gemm_splits(N, K, T);
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.bits = 4;
  a.w0 = a.w1 = packed;
  a.s0 = a.s1 = (const __half*)scales;
  a.n_split = a.N = N;
  a.K = K;
  a.G = group;
  a.x = (const __half*)x;
  a.T = T;
  a.splits = S;
  a.part = S > 1 ? scratch : y;
  TL_TRY(launch_gemm(a, s));
  if (S > 1) TL_TRY(launch_split_sum(scratch, S, (long)T * N, y, s));
  return ok();
}
}  // namespace tl

TL_API tl_status tl_linear_workspace_bytes(int N, int K, int T, size_t* bytes) {
  TL_CHECK_ARG(bytes, "bytes is NULL");
  TL_TRY(check_linear(N, K, 64, T));
  const int S = linear_splits(N, K, T);
  *bytes = S > 1 ? (size_t)S * T * N * 4 : 0;
  return ok();
}

TL_API tl_status tl_linear(const uint32_t* packed, const uint16_t* scales, int N, int K,
                           int group, const uint16_t* x, int T, float* y, void* workspace,
                           tl_stream stream) {
  TL_TRY(check_linear(N, K, group, T));
  TL_CHECK_ARG(packed && scales && x && y, "NULL device pointer");
  TL_TRY(gemm_tc_init());
  const int S = linear_splits(N, K, T);
  TL_CHECK_ARG(S == 1 || workspace, "workspace is NULL but %zu bytes are needed",
               (size_t)S * T * N * 4);
  return launch_linear(packed, scales, N, K, group, x, T, y, (float*)workspace,
                       (cudaStream_t)stream);
}

TL_API tl_status tl_check_bounded_wait(tl_model* model, unsigned limit_us, tl_stream stream) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CHECK_ARG(limit_us >= 1 && limit_us <= 2000000, "limit_us = %u out of [1, 2000000]",
               limit_us);
  return launch_bounded_wait_check(model->status, (uint64_t)limit_us * 1000ull,
                                   (cudaStream_t)stream);
}

TL_API tl_status tl_sync_status(tl_model* model, tl_stream stream) {
  TL_CHECK_ARG(model, "NULL model");
  TL_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  int code = 0;
  TL_CUDA(cudaMemcpy(&code, model->status, 4, cudaMemcpyDeviceToHost));
  TL_CUDA(cudaMemset(model->status, 0, 4));
  if (code == 0) return ok();
  if (code == TL_ERR_TIMEOUT) return set_error(TL_ERR_TIMEOUT, "a bounded device wait ran out");
  if (code == TL_ERR_NUMERIC) return set_error(TL_ERR_NUMERIC, "a non-finite value reached an output");
  if (code == TL_ERR_INVALID_ARG) return set_error(TL_ERR_INVALID_ARG, "a token id was out of range");
  return set_error((tl_status)code, "device status %d", code);
}
