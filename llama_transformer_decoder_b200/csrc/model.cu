// C-ABI host library: model handle, weights, KV cache, workspace, the layer
// loop of prefill and decode, CUDA-graph replay of prefill and decode steps, and the
// stateless entry points used by tests and benchmarks.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "epilogue.cuh"
#include "kernels.h"
#include "llama_b200.h"

using namespace llama;

namespace {

constexpr uint64_t kStreamKvBase = 1ull << 21;

inline cudaStream_t S_(void* s) { return static_cast<cudaStream_t>(s); }

#define CK(call)                                   \
  do {                                             \
    if ((call) != cudaSuccess) {                   \
      cudaGetLastError();                          \
      return LLAMA_ERR_CUDA;                       \
    }                                              \
  } while (0)
#define RC(call)                  \
  do {                            \
    int rc__ = (call);            \
    if (rc__ != LLAMA_OK) return rc__; \
  } while (0)

struct LayerW {
  void* wqkv;   // [(H+2Hk)*d][D]: wq rows, then wk, then wv
  void* wo;     // [D][H*d]
  void* w13;    // [2F][D]: row 2f = w1[f], row 2f+1 = w3[f]
  void* w2;     // [D][F]
  float* attn_norm;
  float* ffn_norm;
};

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

using GraphKey = std::tuple<int, int, int>;
enum GraphKind { G_PREFILL = 0, G_DECODE = 1 };

struct llama_model {
  llama_config cfg{};
  int dev = 0;
  int d = 0, F = 0, qkv_n = 0, Mmax = 0;
  size_t esz = 2;
  // Element type of weights, activations and cache on the device. By default
  // a bf16 model keeps its bf16 weight values in fp16 storage and computes with
  // fp16 activations: fp16 has 3 more mantissa bits, which holds the logits of
  // a 32-layer stack within 2e-2 of the exact result where bf16 activations do
  // not. act_dtype = LLAMA_BF16 keeps everything in bf16 instead.
  int adt = LLAMA_F16;
  // weights
  void* wbase = nullptr;
  void* tok_emb = nullptr;
  void* out_w = nullptr;
  float* norm_w = nullptr;
  std::vector<LayerW> L;
  // cache
  void* kcache = nullptr;
  void* vcache = nullptr;
  size_t layer_cache_elems = 0;
  // paged cache: pool of n_pages pages of KV_PAGE positions, block table
  // [max_batch][max_pages] on the device and its host copy, free pages, and
  // the pages each sequence holds (table row prefix)
  bool paged = false;
  int max_pages = 0, n_pages = 0;
  int32_t* d_table = nullptr;
  std::vector<int32_t> h_table;
  std::vector<int32_t> free_pages;
  std::vector<int> seq_pages;
  int32_t* d_len = nullptr;
  std::vector<int32_t> h_len;
  float2* rope = nullptr;
  // workspace
  float* ss = nullptr;        // [max_tokens][ceil(dim/256)] partial sums of squares (folded RMSNorm)
  bool norm_ready = false;    // xn / ss already hold the next layer's attention-norm inputs
  // Row-block readiness counters of the chained prefill GEMMs (16-bit
  // models): per layer three sets (Wo, w1/w3, w2 outputs) of one counter per
  // 128 rows, zeroed at the start of every prefill step. qkv_ready_layer: the
  // layer whose QKV projection the previous chain already ran (-1: none).
  int* ready = nullptr;
  int ready_rb = 0;
  int qkv_ready_layer = -1;
  float* x = nullptr;
  void* xn = nullptr;
  void* q = nullptr;
  void* attn = nullptr;
  void* g = nullptr;
  float* logits = nullptr;
  int32_t* tok_buf = nullptr;
  int32_t* gen_buf = nullptr;
  size_t gen_cap = 0;
  int last_B = 0;
  GemmScratch gs{};
  DecodeScratch ds{};
  int* d_status = nullptr;
  // CUDA graphs of whole steps, keyed by (kind, B, S or cache bound): the
  // executable, the kernels it launches, and how often the key has been seen.
  std::map<GraphKey, cudaGraphExec_t> graphs;
  std::map<GraphKey, unsigned long long> graph_kernels;
  std::map<GraphKey, int> seen;
  std::set<GraphKey> eager_only;  // shapes whose capture failed: always run eagerly
  size_t bytes = 0;
  std::vector<void*> allocs;
  // per-kernel profiling (eager runs only): an event before every launch
  bool prof_on = false;
  std::vector<std::pair<int, cudaEvent_t>> prof_marks;
  std::vector<cudaEvent_t> prof_pool;
  size_t prof_used = 0;
  cudaStream_t prof_stream = nullptr;

  void* alloc(size_t n) {
    void* p = nullptr;
    if (cudaMalloc(&p, std::max<size_t>(n, 256)) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    allocs.push_back(p);
    bytes += n;
    return p;
  }
  ~llama_model() {
    for (cudaEvent_t e : prof_pool) cudaEventDestroy(e);
    for (auto& kv : graphs) cudaGraphExecDestroy(kv.second);
    for (void* p : allocs) cudaFree(p);
  }
};

namespace {

// ------------------------------------------------------------- config
int resolve(const llama_config* in, llama_config* c) {
  if (!in) return LLAMA_ERR_INVALID_ARG;
  *c = *in;
  if (c->dtype != LLAMA_F32 && c->dtype != LLAMA_BF16 && c->dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  if (c->dim <= 0 || c->n_layers <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->vocab_size <= 0 ||
      c->max_batch <= 0 || c->max_seq <= 0)
    return LLAMA_ERR_SHAPE;
  if (c->dim % c->n_heads != 0 || c->n_heads % c->n_kv_heads != 0) return LLAMA_ERR_SHAPE;
  const int d = c->dim / c->n_heads;
  if (d % 2 != 0 || d % 32 != 0) return LLAMA_ERR_SHAPE;
  if (c->n_heads / c->n_kv_heads > 8) return LLAMA_ERR_UNSUPPORTED;
  if (c->ffn_hidden <= 0) {
    if (c->multiple_of <= 0) return LLAMA_ERR_SHAPE;
    c->ffn_hidden = llama_ffn_hidden(c->dim, c->multiple_of, c->ffn_dim_multiplier);
  }
  if (c->dtype != LLAMA_F32) {
    if (d != 128) return LLAMA_ERR_UNSUPPORTED;
    if (c->dim % 64 != 0 || c->ffn_hidden % 64 != 0) return LLAMA_ERR_SHAPE;
  }
  if (c->kv_page_size != 0) {
    if (c->kv_page_size != KV_PAGE) return LLAMA_ERR_UNSUPPORTED;
    if (c->dtype == LLAMA_F32) return LLAMA_ERR_UNSUPPORTED;   // paged attention kernels are 16-bit
    if (c->kv_pages < 0) return LLAMA_ERR_SHAPE;
    if (c->kv_pages == 0)
      c->kv_pages = (int32_t)std::min<int64_t>((int64_t)c->max_batch * ((c->max_seq + KV_PAGE - 1) / KV_PAGE),
                                               INT32_MAX);
  } else {
    c->kv_pages = 0;
  }
  if (c->act_dtype != 0 && c->act_dtype != LLAMA_F16 && c->act_dtype != LLAMA_BF16) return LLAMA_ERR_INVALID_ARG;
  if (c->act_dtype == LLAMA_BF16 && c->dtype != LLAMA_BF16) return LLAMA_ERR_UNSUPPORTED;
  if (c->act_dtype == LLAMA_F16 && c->dtype == LLAMA_F32) return LLAMA_ERR_UNSUPPORTED;
  if (c->dtype != LLAMA_F32 && c->act_dtype == 0) c->act_dtype = LLAMA_F16;
  if (c->max_tokens <= 0) {
    const int64_t mt = (int64_t)c->max_batch * c->max_seq;
    c->max_tokens = (int32_t)std::min<int64_t>(mt, 16384);
  }
  c->max_tokens = std::max(c->max_tokens, c->max_batch);
  if (!(c->norm_eps >= 0.f) || !(c->rope_theta > 0.f)) return LLAMA_ERR_INVALID_ARG;
  return LLAMA_OK;
}

// Tensor placement inside the model for a checkpoint name.
struct Place {
  char* base = nullptr;  // first element of row 0
  int64_t rows = 0, cols = 0;
  int row_mult = 1;      // destination row = src row * row_mult (+ base offset)
  size_t esz = 2;
  uint64_t stream = 0;
  bool is_norm = false;
};

int locate(llama_model* m, const std::string& name, Place* p) {
  const llama_config& c = m->cfg;
  const int d = m->d, H = c.n_heads, Hk = c.n_kv_heads, D = c.dim;
  p->esz = m->esz;
  if (name == "tok_embeddings.weight") {
    *p = Place{static_cast<char*>(m->tok_emb), c.vocab_size, D, 1, m->esz, 0, false};
    return LLAMA_OK;
  }
  if (name == "norm.weight") {
    *p = Place{reinterpret_cast<char*>(m->norm_w), 1, D, 1, 4, (uint64_t)(1 + 9 * c.n_layers), true};
    return LLAMA_OK;
  }
  if (name == "output.weight") {
    *p = Place{static_cast<char*>(m->out_w), c.vocab_size, D, 1, m->esz, (uint64_t)(2 + 9 * c.n_layers), false};
    return LLAMA_OK;
  }
  int li = -1, consumed = 0;
  char leaf[64] = {0};
  if (sscanf(name.c_str(), "layers.%d.%63s%n", &li, leaf, &consumed) != 2 || li < 0 || li >= c.n_layers)
    return LLAMA_ERR_INVALID_ARG;
  const std::string lf(leaf);
  const LayerW& w = m->L[li];
  const uint64_t base = 1 + 9 * (uint64_t)li;
  const size_t es = m->esz;
  if (lf == "attention.wq.weight") *p = Place{static_cast<char*>(w.wqkv), (int64_t)H * d, D, 1, es, base + 0, false};
  else if (lf == "attention.wk.weight")
    *p = Place{static_cast<char*>(w.wqkv) + (size_t)H * d * D * es, (int64_t)Hk * d, D, 1, es, base + 1, false};
  else if (lf == "attention.wv.weight")
    *p = Place{static_cast<char*>(w.wqkv) + (size_t)(H + Hk) * d * D * es, (int64_t)Hk * d, D, 1, es, base + 2, false};
  else if (lf == "attention.wo.weight") *p = Place{static_cast<char*>(w.wo), D, (int64_t)H * d, 1, es, base + 3, false};
  else if (lf == "feed_forward.w1.weight") *p = Place{static_cast<char*>(w.w13), m->F, D, 2, es, base + 4, false};
  else if (lf == "feed_forward.w3.weight")
    *p = Place{static_cast<char*>(w.w13) + (size_t)D * es, m->F, D, 2, es, base + 5, false};
  else if (lf == "feed_forward.w2.weight") *p = Place{static_cast<char*>(w.w2), D, m->F, 1, es, base + 6, false};
  else if (lf == "attention_norm.weight")
    *p = Place{reinterpret_cast<char*>(w.attn_norm), 1, D, 1, 4, base + 7, true};
  else if (lf == "ffn_norm.weight") *p = Place{reinterpret_cast<char*>(w.ffn_norm), 1, D, 1, 4, base + 8, true};
  else return LLAMA_ERR_INVALID_ARG;
  return LLAMA_OK;
}

// ------------------------------------------------- stateless device context
struct DevCtx {
  int* status = nullptr;
  GemmScratch gs{};
  DecodeScratch ds{};
};
std::mutex g_mu;
std::map<uint64_t, DevCtx> g_ctx;

// The stateless context of the current device, created on first use
// (create == false: nullptr if it does not exist yet).
// Keyed by the current context, so that the scratch of a context destroyed by
// a device reset (whose memory went with it) is not reused.
DevCtx* dev_ctx(bool create = true) {
  const uint64_t dev = context_key();
  std::lock_guard<std::mutex> lk(g_mu);
  if (!create) {
    auto it = g_ctx.find(dev);
    return it == g_ctx.end() || !it->second.status ? nullptr : &it->second;
  }
  DevCtx& c = g_ctx[dev];
  if (!c.status) {
    if (cudaMalloc(&c.status, sizeof(int)) != cudaSuccess) { cudaGetLastError(); c.status = nullptr; return nullptr; }
    cudaMemset(c.status, 0, sizeof(int));
  }
  return &c;
}

int grow_gemm_scratch(GemmScratch* gs, size_t floats, int tickets) {
  if (gs->ws_floats < floats) {
    cudaDeviceSynchronize();
    if (gs->ws) cudaFree(gs->ws);
    gs->ws = nullptr;
    gs->ws_floats = 0;
    if (cudaMalloc(&gs->ws, floats * sizeof(float)) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_OOM; }
    gs->ws_floats = floats;
  }
  if (gs->n_tickets < tickets) {
    cudaDeviceSynchronize();
    if (gs->tickets) cudaFree(gs->tickets);
    gs->tickets = nullptr;
    gs->n_tickets = 0;
    if (cudaMalloc(&gs->tickets, tickets * sizeof(int)) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_OOM; }
    cudaMemset(gs->tickets, 0, tickets * sizeof(int));
    gs->n_tickets = tickets;
  }
  return LLAMA_OK;
}

int grow_decode_scratch(DecodeScratch* ds, size_t floats) {
  if (ds->floats >= floats) return LLAMA_OK;
  cudaDeviceSynchronize();
  if (ds->part) cudaFree(ds->part);
  ds->part = nullptr;
  ds->floats = 0;
  if (cudaMalloc(&ds->part, floats * sizeof(float)) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_OOM; }
  // the decode kernel's work counters in the last 16 bytes start at zero (it re-arms them itself)
  if (cudaMemset(ds->part + floats - 4, 0, 4 * sizeof(float)) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(ds->part);
    ds->part = nullptr;
    return LLAMA_ERR_CUDA;
  }
  ds->floats = floats;
  return LLAMA_OK;
}

// ------------------------------------------------------------ profiling
enum ProfKind { K_EMBED = 0, K_RMSNORM, K_GEMM_QKV, K_ATTN_PREFILL, K_ATTN_DECODE, K_GEMM_WO, K_GEMM_W13, K_GEMM_W2,
                K_GEMM_LMHEAD, K_OTHER, K_GEMM_CHAIN, K_END, K_COUNT };
const char* kProfNames[K_COUNT] = {"embed", "rmsnorm", "gemm_qkv_rope", "attention_prefill", "attention_decode",
                                   "gemm_wo_residual", "gemm_w13_swiglu", "gemm_w2_residual", "gemm_lm_head",
                                   "other", "gemm_chain", "end"};
std::atomic<unsigned long long> g_launches{0};

void mark(llama_model* m, int kind, cudaStream_t st) {
  if (!m->prof_on) return;
  if (m->prof_used == m->prof_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) { cudaGetLastError(); return; }
    m->prof_pool.push_back(e);
  }
  cudaEvent_t e = m->prof_pool[m->prof_used++];
  cudaEventRecord(e, st);
  m->prof_marks.emplace_back(kind, e);
  m->prof_stream = st;
}

// ---------------------------------------------------------------- forward
int gemm(llama_model* m, const void* A, int M, int K, const void* W, int N, int kind, const EpiArgs& e,
         cudaStream_t st) {
  if (m->adt != LLAMA_F32)
    return gemm16(A, M, K, K, W, N, K, m->adt, kind, e, GEMM_AUTO, &m->gs, m->d_status, st);
  return gemm_f32(static_cast<const float*>(A), M, K, K, static_cast<const float*>(W), N, K, kind, e, m->d_status,
                  st);
}

EpiArgs epi_base(int M, int N, int* status = nullptr) {
  EpiArgs e;
  memset(&e, 0, sizeof(e));
  e.M = M;
  e.N = N;
  e.status = status;
  return e;
}

// One decoder block on m->x ([M][D], M = B*S) for sequences 0..B-1 whose
// first new token sits at position d_len[b]. decode: S == 1 and attention
// reads keys 0..d_len[b] through the split-K kernel.
//
// Prefill-sized GEMMs (M > 128) fold the RMSNorms in: the residual GEMMs'
// epilogues leave y = x * g and per-tile sums of squares for the next norm,
// and the QKV / w1-w3 epilogues scale by rsqrt(mean(x^2) + eps). When all
// four projections run on the CTA-pair kernel, the layer's Wo, w1/w3 and w2
// and the next layer's QKV run as one chained launch (gemm16_chain): each
// projection's tiles wait only for the 128-row blocks of the previous one
// they read, so the partial last waves of one projection fill with the next
// one's tiles and three launches per layer disappear. The next layer then
// starts at its attention.
int run_layer(llama_model* m, int l, int B, int S, bool decode, int cmax, cudaStream_t st, bool alone = false) {
  const llama_config& c = m->cfg;
  const int D = c.dim, H = c.n_heads, Hk = c.n_kv_heads, d = m->d, M = B * S;
  const LayerW& w = m->L[l];
  char* kc = static_cast<char*>(m->kcache) + (size_t)l * m->layer_cache_elems * m->esz;
  char* vc = static_cast<char*>(m->vcache) + (size_t)l * m->layer_cache_elems * m->esz;

  const bool fuse = m->adt != LLAMA_F32 && M > 128;
  const int ss_n = (D + 255) / 256;
  const bool chain = fuse && m->ready != nullptr && gemm16_uses_pair(M, m->qkv_n, D) &&
                     gemm16_uses_pair(M, D, H * d) && gemm16_uses_pair(M, 2 * m->F, D) &&
                     gemm16_uses_pair(M, D, m->F);
  auto norm_in = [&](EpiArgs& a) {
    if (!fuse) return;
    a.ss_in = m->ss;
    a.ss_n = ss_n;
    a.norm_inv_d = 1.f / (float)D;
    a.norm_eps = c.norm_eps;
  };
  auto norm_out = [&](EpiArgs& a, const float* g_next) {
    if (!fuse || !g_next) return;
    a.g_next = g_next;
    a.y_out = m->xn;
    a.ss_out = m->ss;
    a.ss_n = ss_n;
  };
  auto qkv_args = [&](int layer) {
    EpiArgs e = epi_base(M, m->qkv_n, m->d_status);
    norm_in(e);
    e.q = m->q;
    e.kc = static_cast<char*>(m->kcache) + (size_t)layer * m->layer_cache_elems * m->esz;
    e.vc = static_cast<char*>(m->vcache) + (size_t)layer * m->layer_cache_elems * m->esz;
    e.rope = m->rope;
    e.pos0 = m->d_len;
    e.S = S;
    e.H = H;
    e.Hk = Hk;
    e.d = d;
    e.Smax = c.max_seq;
    e.kv_table = m->paged ? m->d_table : nullptr;
    e.kv_max_pages = m->max_pages;
    e.kv_pages = m->n_pages;
    return e;
  };

  // ---- attention norm and QKV (unless the previous layer's chain ran it)
  if (!(chain && m->qkv_ready_layer == l)) {
    if (fuse) {
      if (!m->norm_ready) {
        mark(m, K_RMSNORM, st);
        RC(launch_norm_prep(m->x, w.attn_norm, m->xn, m->ss, M, D, ss_n, m->adt, st, m->d_status));
      }
    } else {
      mark(m, K_RMSNORM, st);
      RC(launch_rmsnorm(m->x, w.attn_norm, m->xn, M, D, c.norm_eps, 0, m->adt, st, m->d_status));
    }
    const EpiArgs e = qkv_args(l);
    mark(m, K_GEMM_QKV, st);
    RC(gemm(m, m->xn, M, D, w.wqkv, m->qkv_n, EPI_QKV_ROPE, e, st));
  }
  m->norm_ready = false;
  m->qkv_ready_layer = -1;
  const int32_t* kv_table = m->paged ? m->d_table : nullptr;
  if (decode) {
    mark(m, K_ATTN_DECODE, st);
    RC(attention_decode(m->q, kc, vc, m->d_len, 1, m->attn, B, cmax, H, Hk, d, c.max_seq, m->adt, &m->ds,
                        m->d_status, st, kv_table, m->max_pages, m->n_pages));
  } else {
    mark(m, K_ATTN_PREFILL, st);
    RC(attention_prefill(m->q, kc, vc, m->attn, m->d_len, B, S, H, Hk, d, c.max_seq, m->adt, m->d_status, st,
                         kv_table, m->max_pages, m->n_pages));
  }
  const bool has_next = !alone && l + 1 < c.n_layers;   // alone: one block on its own (no next layer)
  EpiArgs r = epi_base(M, D, m->d_status);
  r.out = m->x;
  r.ldo = D;
  norm_out(r, w.ffn_norm);
  EpiArgs sg = epi_base(M, 2 * m->F, m->d_status);
  sg.g = m->g;
  sg.ldg = m->F;
  norm_in(sg);
  EpiArgs r2 = epi_base(M, D, m->d_status);
  r2.out = m->x;
  r2.ldo = D;
  if (has_next) norm_out(r2, m->L[l + 1].attn_norm);   // the final norm takes the last rows only

  if (chain) {
    const int m_tiles = (M + 255) / 256;
    int* rs = m->ready + (size_t)l * 3 * m->ready_rb;
    ChainJobDesc jobs[4] = {
        {m->attn, H * d, w.wo, H * d, M, D, H * d, EPI_RESIDUAL, 1, -1, rs, r},
        {m->xn, D, w.w13, D, M, 2 * m->F, D, EPI_SWIGLU, (m_tiles + 1) / 2, 0, rs + m->ready_rb, sg},
        {m->g, m->F, w.w2, m->F, M, D, m->F, EPI_RESIDUAL, 1, 1, has_next ? rs + 2 * m->ready_rb : nullptr, r2},
        {}};
    int n = 3;
    if (has_next) {
      jobs[3] = ChainJobDesc{m->xn, D, m->L[l + 1].wqkv, D, M, m->qkv_n, D, EPI_QKV_ROPE, 1, 2, nullptr, qkv_args(l + 1)};
      n = 4;
      m->qkv_ready_layer = l + 1;
    }
    mark(m, K_GEMM_CHAIN, st);
    RC(gemm16_chain(jobs, n, m->adt, m->d_status, st));
    m->norm_ready = has_next;
    return LLAMA_OK;
  }
  mark(m, K_GEMM_WO, st);
  RC(gemm(m, m->attn, M, H * d, w.wo, D, EPI_RESIDUAL, r, st));
  if (!fuse) {
    mark(m, K_RMSNORM, st);
    RC(launch_rmsnorm(m->x, w.ffn_norm, m->xn, M, D, c.norm_eps, 0, m->adt, st, m->d_status));
  }
  mark(m, K_GEMM_W13, st);
  RC(gemm(m, m->xn, M, D, w.w13, 2 * m->F, EPI_SWIGLU, sg, st));
  mark(m, K_GEMM_W2, st);
  RC(gemm(m, m->g, M, m->F, w.w2, D, EPI_RESIDUAL, r2, st));
  m->norm_ready = fuse && has_next;
  return LLAMA_OK;
}

// Final norm of the last row of every sequence, then logits = xf output^T.
int run_head(llama_model* m, int B, int S, cudaStream_t st) {
  const llama_config& c = m->cfg;
  mark(m, K_RMSNORM, st);
  RC(launch_rmsnorm(m->x, m->norm_w, m->xn, B, c.dim, c.norm_eps, S, m->adt, st, m->d_status));
  EpiArgs e = epi_base(B, c.vocab_size, m->d_status);
  e.out = m->logits;
  e.ldo = c.vocab_size;
  mark(m, K_GEMM_LMHEAD, st);
  RC(gemm(m, m->xn, B, c.dim, m->out_w, c.vocab_size, EPI_STORE_F32, e, st));
  m->last_B = B;
  return LLAMA_OK;
}

// Zeroes the row-block counters of the prefill GEMMs (part of the step, so a
// graph replay zeroes them too).
int reset_ready(llama_model* m, int M, cudaStream_t st) {
  m->qkv_ready_layer = -1;
  if (!m->ready || M <= 128) return LLAMA_OK;
  CK(cudaMemsetAsync(m->ready, 0, (size_t)3 * m->cfg.n_layers * m->ready_rb * sizeof(int), st));
  return LLAMA_OK;
}

int prefill_body(llama_model* m, int B, int S, cudaStream_t st) {
  m->norm_ready = false;
  RC(reset_ready(m, B * S, st));
  mark(m, K_EMBED, st);
  RC(launch_embed(m->tok_buf, B * S, m->tok_emb, m->cfg.vocab_size, m->cfg.dim, m->adt, m->x, m->d_status, st));
  for (int l = 0; l < m->cfg.n_layers; ++l) RC(run_layer(m, l, B, S, false, 0, st));
  RC(run_head(m, B, S, st));
  mark(m, K_OTHER, st);
  RC(launch_add_lengths(m->d_len, B, S, st));
  return LLAMA_OK;
}

int decode_body(llama_model* m, int B, int cmax, cudaStream_t st) {
  m->norm_ready = false;
  m->qkv_ready_layer = -1;
  mark(m, K_EMBED, st);
  RC(launch_embed(m->tok_buf, B, m->tok_emb, m->cfg.vocab_size, m->cfg.dim, m->adt, m->x, m->d_status, st));
  for (int l = 0; l < m->cfg.n_layers; ++l) RC(run_layer(m, l, B, 1, true, cmax, st));
  RC(run_head(m, B, 1, st));
  mark(m, K_OTHER, st);
  RC(launch_add_lengths(m->d_len, B, 1, st));
  return LLAMA_OK;
}

// Runs one step through a CUDA graph cached under `key`. The first call per key
// runs eagerly (it also sets the kernels' attributes), the second captures the
// step and replays it, later calls replay. A step only reads device state whose
// addresses are fixed per model (tokens are staged in tok_buf; positions, lengths
// and the block table are read from device memory), so a replay recomputes the
// step for the current inputs. Profiling, the default stream and LLAMA_NO_GRAPH
// keep every call eager. If a capture or its instantiation fails, the step
// runs eagerly instead, and so does every later call with that key.
template <typename Body>
int run_graphed(llama_model* m, const GraphKey& key, cudaStream_t st, Body&& body) {
  static const bool no_graph = getenv("LLAMA_NO_GRAPH") != nullptr;
  auto it = m->graphs.find(key);
  if (it != m->graphs.end() && !m->prof_on) {
    g_launches += m->graph_kernels[key];
    CK(cudaGraphLaunch(it->second, st));
    m->norm_ready = false;
    return LLAMA_OK;
  }
  if (st == nullptr || no_graph || m->prof_on || m->eager_only.count(key) || m->seen[key]++ == 0) return body();
  auto run_eagerly = [&] {
    cudaGetLastError();
    m->eager_only.insert(key);
    return body();
  };
  if (cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return run_eagerly();
  cudaGraph_t graph = nullptr;
  const unsigned long long before = g_launches.load();
  const int rc = body();
  const unsigned long long captured = g_launches.load() - before;
  g_launches -= captured;  // counted again at every replay
  const cudaError_t ce = cudaStreamEndCapture(st, &graph);
  if (ce != cudaSuccess) {  // capture broken (launches inside it failed too): nothing ran
    if (graph) cudaGraphDestroy(graph);
    return run_eagerly();
  }
  if (rc != LLAMA_OK) { cudaGraphDestroy(graph); return rc; }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (ie != cudaSuccess) return run_eagerly();
  m->graphs[key] = exec;
  m->graph_kernels[key] = captured;
  g_launches += captured;
  CK(cudaGraphLaunch(exec, st));
  m->norm_ready = false;
  return LLAMA_OK;
}

KvLayout kv_layout(const llama_model* m) {
  return KvLayout{m->paged ? m->d_table : nullptr, m->max_pages, m->cfg.max_seq, m->n_pages};
}

// Give sequence b exactly the pages that positions [0, len) need, taking
// pages from (or returning them to) the pool, and upload the changed part of
// its block-table row on `st`. Contiguous caches need nothing.
int fit_pages(llama_model* m, int b, int len, cudaStream_t st) {
  if (!m->paged) return LLAMA_OK;
  const int need = (len + KV_PAGE - 1) / KV_PAGE;
  int& have = m->seq_pages[b];
  if (need > m->max_pages) return LLAMA_ERR_SHAPE;
  if (need - have > (int)m->free_pages.size()) return LLAMA_ERR_SHAPE;   // pool exhausted
  const int first = have;
  while (have < need) {
    m->h_table[(size_t)b * m->max_pages + have] = m->free_pages.back();
    m->free_pages.pop_back();
    ++have;
  }
  while (have > need) {
    --have;
    m->free_pages.push_back(m->h_table[(size_t)b * m->max_pages + have]);
    m->h_table[(size_t)b * m->max_pages + have] = 0;
  }
  if (need > first) {
    const size_t off = (size_t)b * m->max_pages + first;
    CK(cudaMemcpyAsync(m->d_table + off, m->h_table.data() + off, (size_t)(need - first) * sizeof(int32_t),
                       cudaMemcpyHostToDevice, st));
  }
  return LLAMA_OK;
}

int fit_pages_all(llama_model* m, int B, int add, cudaStream_t st) {
  for (int b = 0; b < B; ++b) RC(fit_pages(m, b, m->h_len[b] + add, st));
  return LLAMA_OK;
}

int check_lengths(llama_model* m, int B, int S) {
  if (B <= 0 || B > m->cfg.max_batch || S <= 0) return LLAMA_ERR_SHAPE;
  for (int b = 0; b < B; ++b)
    if ((int64_t)m->h_len[b] + S > m->cfg.max_seq) return LLAMA_ERR_SHAPE;
  return LLAMA_OK;
}

}  // namespace

void llama::count_launches(unsigned long long n) { g_launches += n; }

// ======================================================================= ABI
extern "C" {

int32_t llama_ffn_hidden(int32_t dim, int32_t multiple_of, float ffn_dim_multiplier) {
  if (dim <= 0 || multiple_of <= 0) return 0;
  int64_t hidden = (8 * (int64_t)dim) / 3;
  if (ffn_dim_multiplier > 0.f) hidden = (int64_t)((double)ffn_dim_multiplier * (double)hidden);
  return (int32_t)(multiple_of * ((hidden + multiple_of - 1) / multiple_of));
}

const char* llama_status_string(int status) {
  switch (status) {
    case LLAMA_OK: return "ok";
    case LLAMA_ERR_INVALID_ARG: return "invalid argument";
    case LLAMA_ERR_SHAPE: return "shape outside the model or call limits";
    case LLAMA_ERR_OOM: return "device allocation failed";
    case LLAMA_ERR_CUDA: return "CUDA call failed";
    case LLAMA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case LLAMA_ERR_DEVICE_BOUNDS: return "device-side index out of range";
    case LLAMA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LLAMA_ERR_RANGE: return "16-bit activation out of range (not finite after rounding)";
  }
  return "unknown status";
}

int llama_create(const llama_config* cfg, llama_model** out) {
  if (!out) return LLAMA_ERR_INVALID_ARG;
  *out = nullptr;
  llama_config c;
  RC(resolve(cfg, &c));
  llama_model* m = new (std::nothrow) llama_model();
  if (!m) return LLAMA_ERR_OOM;
  m->cfg = c;
  cudaGetDevice(&m->dev);
  m->esz = c.dtype == LLAMA_F32 ? 4 : 2;
  m->adt = c.dtype == LLAMA_F32 ? LLAMA_F32 : c.act_dtype;
  m->d = c.dim / c.n_heads;
  m->F = c.ffn_hidden;
  m->qkv_n = (c.n_heads + 2 * c.n_kv_heads) * m->d;
  m->Mmax = c.max_tokens;
  const size_t es = m->esz, D = c.dim, V = c.vocab_size, F = m->F, Hd = (size_t)c.n_heads * m->d;
  // ---- weights (one allocation)
  const size_t per_layer = align256((size_t)m->qkv_n * D * es) + align256(D * Hd * es) + align256(2 * F * D * es) +
                           align256(D * F * es) + 2 * align256(D * 4);
  const size_t wbytes = 2 * align256(V * D * es) + align256(D * 4) + per_layer * c.n_layers;
  char* wb = static_cast<char*>(m->alloc(wbytes));
  if (!wb) { delete m; return LLAMA_ERR_OOM; }
  cudaMemset(wb, 0, wbytes);
  m->wbase = wb;
  m->tok_emb = wb; wb += align256(V * D * es);
  m->out_w = wb; wb += align256(V * D * es);
  m->norm_w = reinterpret_cast<float*>(wb); wb += align256(D * 4);
  m->L.resize(c.n_layers);
  for (auto& w : m->L) {
    w.wqkv = wb; wb += align256((size_t)m->qkv_n * D * es);
    w.wo = wb; wb += align256(D * Hd * es);
    w.w13 = wb; wb += align256(2 * F * D * es);
    w.w2 = wb; wb += align256(D * F * es);
    w.attn_norm = reinterpret_cast<float*>(wb); wb += align256(D * 4);
    w.ffn_norm = reinterpret_cast<float*>(wb); wb += align256(D * 4);
  }
  // ---- KV cache
  m->paged = c.kv_page_size != 0;
  if (m->paged) {
    m->max_pages = (c.max_seq + KV_PAGE - 1) / KV_PAGE;
    m->n_pages = c.kv_pages;
    m->layer_cache_elems = (size_t)m->n_pages * c.n_kv_heads * KV_PAGE * m->d;
    m->d_table = static_cast<int32_t*>(m->alloc((size_t)c.max_batch * m->max_pages * sizeof(int32_t)));
    if (!m->d_table) { delete m; return LLAMA_ERR_OOM; }
    cudaMemset(m->d_table, 0, (size_t)c.max_batch * m->max_pages * sizeof(int32_t));
    m->h_table.assign((size_t)c.max_batch * m->max_pages, 0);
    m->seq_pages.assign(c.max_batch, 0);
    // The pool hands pages out in a scattered order (stride coprime with the
    // pool size), so consecutive pages of a sequence are not neighbours.
    int stride = 7919 % m->n_pages;
    auto gcd = [](int a, int b) { while (b) { const int t = a % b; a = b; b = t; } return a; };
    while (stride <= 0 || gcd(stride, m->n_pages) != 1) stride = (stride + 1) % std::max(m->n_pages, 2);
    if (m->n_pages == 1) stride = 1;
    m->free_pages.resize(m->n_pages);
    for (int i = 0; i < m->n_pages; ++i)   // back of the vector is handed out first
      m->free_pages[m->n_pages - 1 - i] = (int32_t)(((int64_t)i * stride) % m->n_pages);
  } else {
    m->layer_cache_elems = (size_t)c.max_batch * c.n_kv_heads * c.max_seq * m->d;
  }
  m->kcache = m->alloc(m->layer_cache_elems * c.n_layers * es);
  m->vcache = m->alloc(m->layer_cache_elems * c.n_layers * es);
  m->d_len = static_cast<int32_t*>(m->alloc(c.max_batch * sizeof(int32_t)));
  m->h_len.assign(c.max_batch, 0);
  // ---- RoPE table: angle pos * theta^(-2i/d), computed in double, stored as fp32 (cos, sin)
  m->rope = static_cast<float2*>(m->alloc((size_t)c.max_seq * (m->d / 2) * sizeof(float2)));
  // ---- workspace
  const size_t Mx = m->Mmax;
  m->x = static_cast<float*>(m->alloc(Mx * D * 4));
  m->ss = static_cast<float*>(m->alloc(Mx * ((D + 255) / 256) * 4));
  m->xn = m->alloc(Mx * D * es);
  m->q = m->alloc(Mx * Hd * es);
  m->attn = m->alloc(Mx * Hd * es);
  m->g = m->alloc(Mx * F * es);
  m->logits = static_cast<float*>(m->alloc((size_t)c.max_batch * V * 4));
  m->tok_buf = static_cast<int32_t*>(m->alloc(Mx * sizeof(int32_t)));
  m->d_status = static_cast<int*>(m->alloc(sizeof(int)));
  if (m->adt != LLAMA_F32 && Mx > 128 && getenv("LLAMA_NO_GEMM_CHAIN") == nullptr) {
    m->ready_rb = (int)(2 * ((Mx + 255) / 256));
    m->ready = static_cast<int*>(m->alloc((size_t)3 * c.n_layers * m->ready_rb * sizeof(int)));
    if (!m->ready) { delete m; return LLAMA_ERR_OOM; }
    cudaMemset(m->ready, 0, (size_t)3 * c.n_layers * m->ready_rb * sizeof(int));
  }
  if (!m->kcache || !m->vcache || !m->d_len || !m->rope || !m->x || !m->ss || !m->xn || !m->q || !m->attn || !m->g ||
      !m->logits || !m->tok_buf || !m->d_status) {
    delete m;
    return LLAMA_ERR_OOM;
  }
  cudaMemset(m->kcache, 0, m->layer_cache_elems * c.n_layers * es);
  cudaMemset(m->vcache, 0, m->layer_cache_elems * c.n_layers * es);
  cudaMemset(m->d_len, 0, c.max_batch * sizeof(int32_t));
  cudaMemset(m->d_status, 0, sizeof(int));
  {
    const int half = m->d / 2;
    std::vector<float2> tab((size_t)c.max_seq * half);
    for (int p = 0; p < c.max_seq; ++p)
      for (int i = 0; i < half; ++i) {
        const double inv = 1.0 / std::pow((double)c.rope_theta, (double)i / (double)half);
        const double a = (double)p * inv;
        tab[(size_t)p * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    if (cudaMemcpy(m->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      delete m;
      return LLAMA_ERR_CUDA;
    }
  }
  // ---- split-K scratch for every skinny GEMM shape the model can issue
  if (m->adt != LLAMA_F32) {
    size_t ws = 0;
    int tickets = 0;
    const int shapes[5][2] = {{m->qkv_n, c.dim}, {c.dim, (int)Hd}, {2 * m->F, c.dim}, {c.dim, m->F}, {c.vocab_size, c.dim}};
    for (auto& sh : shapes) {
      ws = std::max(ws, skinny_workspace_floats(std::min(128, m->Mmax)));
      tickets = std::max(tickets, (sh[0] + 127) / 128);
    }
    // the wide GEMM's stream-K tiles: fewer than 1.5 waves
    const int sk_max = m->Mmax > 128 ? 3 * num_sms() / 2 + 1 : 0;
    tickets = std::max(tickets, sk_max);
    if (sk_max) ws = std::max(ws, wide_workspace_floats());
    if (grow_gemm_scratch(&m->gs, std::max<size_t>(ws, 1), tickets) != LLAMA_OK) { delete m; return LLAMA_ERR_OOM; }
    m->allocs.push_back(m->gs.ws);
    m->allocs.push_back(m->gs.tickets);

  }
  {
    size_t need = 0;
    for (int B = 1; B <= c.max_batch; ++B)
      need = std::max(need, decode_scratch_floats(c.max_seq, B, c.n_heads, c.n_kv_heads, m->d, m->adt));
    if (grow_decode_scratch(&m->ds, need) != LLAMA_OK) { delete m; return LLAMA_ERR_OOM; }
    m->allocs.push_back(m->ds.part);
  }
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); delete m; return LLAMA_ERR_CUDA; }
  *out = m;
  return LLAMA_OK;
}

void llama_destroy(llama_model* m) {
  if (!m) return;
  cudaDeviceSynchronize();
  delete m;
}

int llama_get_config(const llama_model* m, llama_config* out) {
  if (!m || !out) return LLAMA_ERR_INVALID_ARG;
  *out = m->cfg;
  return LLAMA_OK;
}

size_t llama_device_bytes(const llama_model* m) { return m ? m->bytes : 0; }

int llama_init_weights(llama_model* m, uint64_t seed, float std, void* stream) {
  if (!m) return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = S_(stream);
  std::vector<std::string> names{"tok_embeddings.weight"};
  static const char* keys[9] = {"attention.wq.weight", "attention.wk.weight", "attention.wv.weight",
                                "attention.wo.weight", "feed_forward.w1.weight", "feed_forward.w3.weight",
                                "feed_forward.w2.weight", "attention_norm.weight", "ffn_norm.weight"};
  for (int i = 0; i < m->cfg.n_layers; ++i)
    for (auto k : keys) names.push_back("layers." + std::to_string(i) + "." + k);
  names.push_back("norm.weight");
  names.push_back("output.weight");
  for (const auto& n : names) {
    Place p;
    RC(locate(m, n, &p));
    if (p.is_norm) {
      RC(launch_fill_const(reinterpret_cast<float*>(p.base), p.cols, 1.0f, st));
      continue;
    }
    // destination row r*row_mult; w3 rows start one row further through p.base
    const FillLayout fl{1, p.rows, p.cols, 0, p.cols, p.row_mult, 0};
    RC(launch_fill_normal(p.base, fl, seed, p.stream, std, m->adt, st, m->cfg.dtype == LLAMA_BF16));
  }
  return LLAMA_OK;
}

static int copy_weight(llama_model* m, const char* name, void* host_or_dev, size_t nbytes, int on_device,
                       void* stream, bool to_model) {
  if (!m || !name || !host_or_dev) return LLAMA_ERR_INVALID_ARG;
  Place p;
  RC(locate(m, name, &p));
  const size_t row_bytes = (size_t)p.cols * p.esz;
  if (nbytes != row_bytes * (size_t)p.rows) return LLAMA_ERR_SHAPE;
  const size_t model_pitch = row_bytes * p.row_mult;
  cudaStream_t st = S_(stream);
  if (m->cfg.dtype == LLAMA_BF16 && m->adt == LLAMA_F16 && !p.is_norm) {
    // bf16 in the caller's buffer, fp16 in the model: convert on the device.
    void* dev = host_or_dev;
    if (!on_device) {
      if (cudaMalloc(&dev, nbytes) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_OOM; }
      if (to_model && cudaMemcpyAsync(dev, host_or_dev, nbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(dev);
        return LLAMA_ERR_CUDA;
      }
    }
    const int64_t mp = (int64_t)p.cols * p.row_mult;
    int rc = to_model ? launch_convert_2d(p.base, mp, LLAMA_F16, dev, p.cols, LLAMA_BF16, p.rows, p.cols, st)
                      : launch_convert_2d(dev, p.cols, LLAMA_BF16, p.base, mp, LLAMA_F16, p.rows, p.cols, st);
    if (!on_device) {
      if (rc == LLAMA_OK && !to_model &&
          cudaMemcpyAsync(host_or_dev, dev, nbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        rc = LLAMA_ERR_CUDA;
      if (cudaStreamSynchronize(st) != cudaSuccess) rc = LLAMA_ERR_CUDA;
      cudaGetLastError();
      cudaFree(dev);
    }
    return rc;
  }
  cudaMemcpyKind kind = on_device ? cudaMemcpyDeviceToDevice : (to_model ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost);
  if (to_model)
    CK(cudaMemcpy2DAsync(p.base, model_pitch, host_or_dev, row_bytes, row_bytes, p.rows, kind, st));
  else
    CK(cudaMemcpy2DAsync(host_or_dev, row_bytes, p.base, model_pitch, row_bytes, p.rows, kind, st));
  if (!on_device) CK(cudaStreamSynchronize(st));
  return LLAMA_OK;
}

int llama_set_weight(llama_model* m, const char* name, const void* src, size_t nbytes, int on_device, void* stream) {
  return copy_weight(m, name, const_cast<void*>(src), nbytes, on_device, stream, true);
}
int llama_get_weight(llama_model* m, const char* name, void* dst, size_t nbytes, int on_device, void* stream) {
  return copy_weight(m, name, dst, nbytes, on_device, stream, false);
}

int llama_prefill(llama_model* m, const int32_t* tokens, int32_t B, int32_t S, void* stream) {
  if (!m || !tokens) return LLAMA_ERR_INVALID_ARG;
  RC(check_lengths(m, B, S));
  if ((int64_t)B * S > m->Mmax) return LLAMA_ERR_SHAPE;
  cudaStream_t st = S_(stream);
  RC(fit_pages_all(m, B, S, st));  // before the (possibly graph-replayed) step reads the table
  CK(cudaMemcpyAsync(m->tok_buf, tokens, (size_t)B * S * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  RC(run_graphed(m, GraphKey(G_PREFILL, B, S), st, [&] { return prefill_body(m, B, S, st); }));
  m->last_B = B;
  for (int b = 0; b < B; ++b) m->h_len[b] += S;
  return LLAMA_OK;
}

int llama_decode_step(llama_model* m, const int32_t* tokens, int32_t B, void* stream) {
  if (!m || !tokens) return LLAMA_ERR_INVALID_ARG;
  RC(check_lengths(m, B, 1));
  cudaStream_t st = S_(stream);
  RC(fit_pages_all(m, B, 1, st));   // before the (possibly graph-replayed) step reads the table
  int maxlen = 0;
  for (int b = 0; b < B; ++b) maxlen = std::max(maxlen, m->h_len[b] + 1);
  const int cmax = std::min(m->cfg.max_seq, (maxlen + 511) / 512 * 512);
  CK(cudaMemcpyAsync(m->tok_buf, tokens, B * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  RC(run_graphed(m, GraphKey(G_DECODE, B, cmax), st, [&] { return decode_body(m, B, cmax, st); }));
  m->last_B = B;
  for (int b = 0; b < B; ++b) m->h_len[b] += 1;
  return LLAMA_OK;
}

int llama_logits(llama_model* m, float* dst, void* stream) {
  if (!m || !dst) return LLAMA_ERR_INVALID_ARG;
  if (m->last_B <= 0) return LLAMA_ERR_SHAPE;
  CK(cudaMemcpyAsync(dst, m->logits, (size_t)m->last_B * m->cfg.vocab_size * sizeof(float), cudaMemcpyDeviceToDevice,
                     S_(stream)));
  return LLAMA_OK;
}

int llama_argmax(llama_model* m, int32_t* dst, void* stream) {
  if (!m || !dst) return LLAMA_ERR_INVALID_ARG;
  if (m->last_B <= 0) return LLAMA_ERR_SHAPE;
  mark(m, K_OTHER, S_(stream));
  return launch_argmax(m->logits, dst, m->last_B, m->cfg.vocab_size, S_(stream));
}

int llama_generate(llama_model* m, const int32_t* host_tokens, int32_t B, int32_t S, int32_t n_new,
                   int32_t* host_out, void* stream) {
  if (!m || !host_tokens || !host_out || n_new < 0) return LLAMA_ERR_INVALID_ARG;
  RC(check_lengths(m, B, S + n_new));
  if ((int64_t)B * S > m->Mmax) return LLAMA_ERR_SHAPE;
  cudaStream_t st = S_(stream);
  const size_t need = (size_t)B * S + (size_t)B * (n_new + 1);
  if (m->gen_cap < need) {
    CK(cudaStreamSynchronize(st));
    if (m->gen_buf) cudaFree(m->gen_buf);
    m->gen_buf = nullptr;
    m->gen_cap = 0;
    if (cudaMalloc(&m->gen_buf, need * sizeof(int32_t)) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_OOM; }
    m->gen_cap = need;
  }
  int32_t* prompt = m->gen_buf;
  int32_t* outs = m->gen_buf + (size_t)B * S;  // [n_new+1][B]
  CK(cudaMemcpyAsync(prompt, host_tokens, (size_t)B * S * sizeof(int32_t), cudaMemcpyHostToDevice, st));
  RC(llama_prefill(m, prompt, B, S, stream));
  RC(llama_argmax(m, outs, stream));
  for (int i = 1; i <= n_new; ++i) {
    RC(llama_decode_step(m, outs + (size_t)(i - 1) * B, B, stream));
    RC(llama_argmax(m, outs + (size_t)i * B, stream));
  }
  std::vector<int32_t> tmp((size_t)B * (n_new + 1));
  CK(cudaMemcpyAsync(tmp.data(), outs, tmp.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  for (int b = 0; b < B; ++b)
    for (int i = 0; i <= n_new; ++i) host_out[(size_t)b * (n_new + 1) + i] = tmp[(size_t)i * B + b];
  return LLAMA_OK;
}

int llama_block_forward(llama_model* m, int32_t layer, const float* x, float* y, int32_t B, int32_t S,
                        void* stream) {
  if (!m || !x || !y) return LLAMA_ERR_INVALID_ARG;
  if (layer < 0 || layer >= m->cfg.n_layers) return LLAMA_ERR_INVALID_ARG;
  RC(check_lengths(m, B, S));
  if ((int64_t)B * S > m->Mmax) return LLAMA_ERR_SHAPE;
  cudaStream_t st = S_(stream);
  RC(fit_pages_all(m, B, S, st));
  const size_t bytes = (size_t)B * S * m->cfg.dim * sizeof(float);
  CK(cudaMemcpyAsync(m->x, x, bytes, cudaMemcpyDeviceToDevice, st));
  m->norm_ready = false;
  RC(reset_ready(m, B * S, st));
  RC(run_layer(m, layer, B, S, false, 0, st, true));
  m->norm_ready = false;
  CK(cudaMemcpyAsync(y, m->x, bytes, cudaMemcpyDeviceToDevice, st));
  return LLAMA_OK;
}

int llama_fill_kv_random(llama_model* m, uint64_t seed, int32_t c, void* stream) {
  if (!m) return LLAMA_ERR_INVALID_ARG;
  if (c < 0 || c > m->cfg.max_seq) return LLAMA_ERR_SHAPE;
  cudaStream_t st = S_(stream);
  const llama_config& cf = m->cfg;
  for (int b = 0; b < cf.max_batch; ++b) RC(fit_pages(m, b, c, st));   // pages first: the fill writes through them
  const KvLayout L = kv_layout(m);
  for (int l = 0; l < cf.n_layers; ++l) {
    char* kc = static_cast<char*>(m->kcache) + (size_t)l * m->layer_cache_elems * m->esz;
    char* vc = static_cast<char*>(m->vcache) + (size_t)l * m->layer_cache_elems * m->esz;
    const bool rb = cf.dtype == LLAMA_BF16;
    RC(launch_fill_kv(kc, L, cf.max_batch, cf.n_kv_heads, c, m->d, seed, kStreamKvBase + 2 * (uint64_t)l, 1.0f,
                      m->adt, rb, st));
    RC(launch_fill_kv(vc, L, cf.max_batch, cf.n_kv_heads, c, m->d, seed, kStreamKvBase + 2 * (uint64_t)l + 1, 1.0f,
                      m->adt, rb, st));
  }
  std::vector<int32_t> lens(cf.max_batch, c);
  return llama_set_lengths(m, lens.data(), cf.max_batch, stream);
}

int llama_set_kv(llama_model* m, int32_t layer, const void* k, const void* v, int32_t B, int32_t c, void* stream) {
  if (!m || !k || !v) return LLAMA_ERR_INVALID_ARG;
  if (layer < 0 || layer >= m->cfg.n_layers) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || B > m->cfg.max_batch || c <= 0 || c > m->cfg.max_seq) return LLAMA_ERR_SHAPE;
  cudaStream_t st = S_(stream);
  for (int b = 0; b < B; ++b) RC(fit_pages(m, b, std::max(m->h_len[b], (int)c), st));
  char* kc = static_cast<char*>(m->kcache) + (size_t)layer * m->layer_cache_elems * m->esz;
  char* vc = static_cast<char*>(m->vcache) + (size_t)layer * m->layer_cache_elems * m->esz;
  // caller's dtype in, the model's storage type (fp16 for bf16 models) in the cache
  const KvLayout L = kv_layout(m);
  RC(launch_kv_scatter(kc, m->adt, L, B, m->cfg.n_kv_heads, c, m->d, k, m->cfg.dtype, st));
  return launch_kv_scatter(vc, m->adt, L, B, m->cfg.n_kv_heads, c, m->d, v, m->cfg.dtype, st);
}

int llama_set_lengths(llama_model* m, const int32_t* host_len, int32_t B, void* stream) {
  if (!m || !host_len) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || B > m->cfg.max_batch) return LLAMA_ERR_SHAPE;
  for (int b = 0; b < B; ++b)
    if (host_len[b] < 0 || host_len[b] > m->cfg.max_seq) return LLAMA_ERR_SHAPE;
  for (int b = 0; b < B; ++b) m->h_len[b] = host_len[b];
  for (int b = 0; b < B; ++b) RC(fit_pages(m, b, m->h_len[b], S_(stream)));
  CK(cudaMemcpyAsync(m->d_len, m->h_len.data(), B * sizeof(int32_t), cudaMemcpyHostToDevice, S_(stream)));
  CK(cudaStreamSynchronize(S_(stream)));
  return LLAMA_OK;
}

int llama_get_block_table(const llama_model* m, int32_t* host_table, int32_t B) {
  if (!m || !host_table) return LLAMA_ERR_INVALID_ARG;
  if (!m->paged) return LLAMA_ERR_UNSUPPORTED;
  if (B <= 0 || B > m->cfg.max_batch) return LLAMA_ERR_SHAPE;
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < m->max_pages; ++j)
      host_table[(size_t)b * m->max_pages + j] = j < m->seq_pages[b] ? m->h_table[(size_t)b * m->max_pages + j] : -1;
  return LLAMA_OK;
}

int llama_get_lengths(const llama_model* m, int32_t* host_len, int32_t B) {
  if (!m || !host_len) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || B > m->cfg.max_batch) return LLAMA_ERR_SHAPE;
  for (int b = 0; b < B; ++b) host_len[b] = m->h_len[b];
  return LLAMA_OK;
}

int llama_reset(llama_model* m, void* stream) {
  if (!m) return LLAMA_ERR_INVALID_ARG;
  std::fill(m->h_len.begin(), m->h_len.end(), 0);
  for (int b = 0; b < m->cfg.max_batch; ++b) RC(fit_pages(m, b, 0, S_(stream)));   // every page back to the pool
  m->last_B = 0;
  CK(cudaMemsetAsync(m->d_len, 0, m->cfg.max_batch * sizeof(int32_t), S_(stream)));
  return LLAMA_OK;
}

int llama_profile(llama_model* m, int enable) {
  if (!m) return LLAMA_ERR_INVALID_ARG;
  m->prof_on = enable != 0;
  return LLAMA_OK;
}

int llama_profile_read(llama_model* m, double* ms, int64_t* launches, int n_kinds) {
  if (!m || !ms || !launches || n_kinds <= 0) return LLAMA_ERR_INVALID_ARG;
  const int n = std::min(n_kinds, (int)K_END);
  for (int i = 0; i < n; ++i) { ms[i] = 0.0; launches[i] = 0; }
  if (!m->prof_marks.empty()) {
    cudaEvent_t end = nullptr;
    if (cudaEventCreate(&end) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_CUDA; }
    cudaEventRecord(end, m->prof_stream);
    if (cudaEventSynchronize(end) != cudaSuccess) { cudaGetLastError(); cudaEventDestroy(end); return LLAMA_ERR_CUDA; }
    for (size_t i = 0; i < m->prof_marks.size(); ++i) {
      cudaEvent_t next = i + 1 < m->prof_marks.size() ? m->prof_marks[i + 1].second : end;
      float t = 0.f;
      cudaEventElapsedTime(&t, m->prof_marks[i].second, next);
      const int k = m->prof_marks[i].first;
      if (k < n) { ms[k] += t; launches[k] += 1; }
    }
    cudaEventDestroy(end);
  }
  m->prof_marks.clear();
  m->prof_used = 0;
  return n;
}

const char* llama_profile_kind_name(int kind) {
  return (kind >= 0 && kind < K_COUNT) ? kProfNames[kind] : "";
}

uint64_t llama_kernel_launches(void) { return g_launches.load(); }

int llama_sync_status(llama_model* m, void* stream) {
  if (!m) return LLAMA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(S_(stream)) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_CUDA; }
  int s = 0;
  CK(cudaMemcpy(&s, m->d_status, sizeof(int), cudaMemcpyDeviceToHost));
  CK(cudaMemset(m->d_status, 0, sizeof(int)));
  return s;
}

// ------------------------------------------------------------- stateless
int llama_status(void* stream) {
  if (cudaStreamSynchronize(S_(stream)) != cudaSuccess) { cudaGetLastError(); return LLAMA_ERR_CUDA; }
  int s = 0;
  if (DevCtx* c = dev_ctx(false)) {   // no context yet: no stateless call has run, nothing to allocate
    CK(cudaMemcpy(&s, c->status, sizeof(int), cudaMemcpyDeviceToHost));
    CK(cudaMemset(c->status, 0, sizeof(int)));
  }
  int s2 = 0;
  RC(noalloc_take_status(&s2));
  return s != 0 ? s : s2;
}

int llama_attention_prefill(const void* q, const void* k, const void* v, void* o, int32_t B, int32_t S, int32_t H,
                            int32_t Hk, int32_t d, int32_t dtype, void* stream) {
  if (!q || !k || !v || !o) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0 || H <= 0 || Hk <= 0 || H % Hk != 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_F32 && dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  return attention_prefill(q, k, v, o, nullptr, B, S, H, Hk, d, S, dtype, c->status, S_(stream));
}

int llama_attention_decode(const void* q, const void* kc, const void* vc, const int32_t* len, void* o, int32_t B,
                           int32_t cmax, int32_t H, int32_t Hk, int32_t d, int32_t dtype, void* stream) {
  if (!q || !kc || !vc || !len || !o) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || cmax <= 0 || H <= 0 || Hk <= 0 || H % Hk != 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_F32 && dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  RC(grow_decode_scratch(&c->ds, decode_scratch_floats(cmax, B, H, Hk, d, dtype)));
  return attention_decode(q, kc, vc, len, 0, o, B, cmax, H, Hk, d, cmax, dtype, &c->ds, c->status, S_(stream));
}

// Validates a caller's block table (device [B][max_pages]): every entry in
// [-1, n_pages) (-1 marks an unused slot).
static int check_block_table(const int32_t* table, int B, int max_pages, int n_pages, cudaStream_t st) {
  std::vector<int32_t> h((size_t)B * max_pages);
  CK(cudaMemcpyAsync(h.data(), table, h.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  CK(cudaStreamSynchronize(st));
  for (int32_t p : h)
    if (p < -1 || p >= n_pages) return LLAMA_ERR_SHAPE;
  return LLAMA_OK;
}

int llama_attention_prefill_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* table,
                                  int32_t max_pages, int32_t n_pages, const int32_t* pos0, void* o, int32_t B,
                                  int32_t S, int32_t H, int32_t Hk, int32_t d, int32_t dtype, void* stream) {
  if (!q || !k_pages || !v_pages || !table || !o) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || max_pages <= 0 || n_pages <= 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_UNSUPPORTED;
  if (d != 128) return LLAMA_ERR_UNSUPPORTED;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  RC(check_block_table(table, B, max_pages, n_pages, S_(stream)));
  return attention_prefill(q, k_pages, v_pages, o, pos0, B, S, H, Hk, d, max_pages * KV_PAGE, dtype, c->status,
                           S_(stream), table, max_pages, n_pages);
}

int llama_attention_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* table,
                                 int32_t max_pages, int32_t n_pages, const int32_t* len, void* o, int32_t B,
                                 int32_t H, int32_t Hk, int32_t d, int32_t dtype, void* stream) {
  if (!q || !k_pages || !v_pages || !table || !len || !o) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || max_pages <= 0 || n_pages <= 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_UNSUPPORTED;
  if (d != 128) return LLAMA_ERR_UNSUPPORTED;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  RC(check_block_table(table, B, max_pages, n_pages, S_(stream)));
  const int cmax = max_pages * KV_PAGE;
  RC(grow_decode_scratch(&c->ds, decode_scratch_floats(cmax, B, H, Hk, d, dtype)));
  return attention_decode(q, k_pages, v_pages, len, 0, o, B, cmax, H, Hk, d, cmax, dtype, &c->ds, c->status,
                          S_(stream), table, max_pages, n_pages);
}

int llama_linear(const void* x, const void* w, float* y, int32_t M, int32_t N, int32_t K, int32_t dtype,
                 int32_t variant, void* stream) {
  if (!x || !w || !y) return LLAMA_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return LLAMA_ERR_SHAPE;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  EpiArgs e = epi_base(M, N);
  e.out = y;
  e.ldo = N;
  if (dtype == LLAMA_F32)
    return gemm_f32(static_cast<const float*>(x), M, K, K, static_cast<const float*>(w), N, K, EPI_STORE_F32, e,
                    c->status, S_(stream));
  if ((dtype != LLAMA_BF16 && dtype != LLAMA_F16) || variant < 0 || variant > 2) return LLAMA_ERR_INVALID_ARG;
  const bool skinny = variant == GEMM_SKINNY || (variant == GEMM_AUTO && M <= 128);
  if (skinny) {
    if (M > 256) return LLAMA_ERR_SHAPE;
    RC(grow_gemm_scratch(&c->gs, skinny_workspace_floats(M), (N + 127) / 128));
  } else {
    const WideSplit w = wide_split(M, N, K);
    RC(grow_gemm_scratch(&c->gs, wide_workspace_floats(), std::max(w.sk_tiles, 1)));
  }
  return gemm16(x, M, K, K, w, N, K, dtype, EPI_STORE_F32, e, variant, &c->gs, c->status, S_(stream));
}

int llama_rmsnorm(const float* x, const float* g, void* y, int32_t M, int32_t D, float eps, int32_t dtype,
                  void* stream) {
  if (!x || !g || !y) return LLAMA_ERR_INVALID_ARG;
  if (M <= 0 || D <= 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_F32 && dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  return launch_rmsnorm(x, g, y, M, D, eps, 0, dtype, S_(stream), c->status);
}

int llama_argmax_rows(const float* logits, int32_t* out, int32_t B, int32_t V, void* stream) {
  if (!logits || !out) return LLAMA_ERR_INVALID_ARG;
  if (B <= 0 || V <= 0) return LLAMA_ERR_SHAPE;
  return launch_argmax(logits, out, B, V, S_(stream));
}

int llama_wait_selftest(int32_t kind, uint64_t limit_ns, void* stream) {
  if (kind != 0 && kind != 1) return LLAMA_ERR_INVALID_ARG;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return LLAMA_ERR_INVALID_ARG;
  DevCtx* c = dev_ctx();
  if (!c) return LLAMA_ERR_OOM;
  return launch_wait_selftest(kind, limit_ns, c->status, S_(stream));
}

int llama_fill_normal(void* dst, int64_t n, uint64_t seed, uint64_t stream_id, float std, int32_t dtype,
                      void* stream) {
  if (!dst) return LLAMA_ERR_INVALID_ARG;
  if (n < 0) return LLAMA_ERR_SHAPE;
  if (dtype != LLAMA_F32 && dtype != LLAMA_BF16 && dtype != LLAMA_F16) return LLAMA_ERR_INVALID_ARG;
  FillLayout fl{1, 1, n, 0, n, 1, 0};
  return launch_fill_normal(dst, fl, seed, stream_id, std, dtype, S_(stream));
}

}  // extern "C"
