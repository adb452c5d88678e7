// The exported C ABI (include/csa.h): host-side validation, workspace
// layout, and dispatch to the kernels.  Nothing here allocates device memory.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "pool.cuh"

namespace csa {

csa_status_t launch_compress(const csa_tensor_t* C, const csa_tensor_t* Z, int batch, int64_t n_tokens, int d,
                             int m, const csa_tensor_t* out, int64_t out_rows, const csa_tensor_t* w_ik,
                             int d_idx, const csa_tensor_t* kidx_out, cudaStream_t stream);
csa_status_t launch_decode_append(const csa_params_t* p, int batch, const csa_decode_caches_t* cc,
                                  const csa_decode_token_t* tok, const int64_t* pos, int32_t* n_visible,
                                  int64_t* q_pos, int32_t* q_req, void* zero, size_t zero_bytes,
                                  cudaStream_t stream);
bool index_tc_supported(const csa_params_t* p, int batch, int64_t cap, int q_dtype, int k_dtype);
bool index_tc_append_supported(const csa_params_t* p, int w_dtype);
size_t index_tc_control_bytes(int batch);
size_t index_tc_workspace_bytes(int batch, int64_t cap, int k);
csa_status_t launch_index_topk_tc(const csa_params_t* p, int batch, const csa_tensor_t* q_idx, const float* w,
                                  const csa_tensor_t* k_idx, int64_t cap, const int32_t* n_visible, int32_t* out_idx,
                                  float* out_score, void* ws, cudaStream_t stream, const AppendArgs* ap = nullptr,
                                  float* bmax = nullptr, int64_t ldb = 0, int block = 1,
                                  const int32_t* pool = nullptr, int pool_blocks = 0, int pblock = 0);
bool index_tc_pool_supported(const csa_params_t* p, int batch, int64_t cap, int block, int pool_blocks, int q_dtype,
                             int k_dtype);
uint32_t index_tc_take_error();
csa_status_t test_expire_next_barrier(int cta, uint32_t polls);
uint32_t attn_tc_take_error();
csa_status_t launch_index_score(const csa_params_t* p, int nq, const csa_tensor_t* q_idx, const float* w,
                                const csa_tensor_t* k_idx, int batch, int64_t cap, const int32_t* q_req,
                                const int32_t* n_visible, float* scores, int64_t ld, int64_t max_entries,
                                cudaStream_t stream, const int32_t* pool = nullptr, int block = 1,
                                int pool_blocks = 0);
csa_status_t launch_topk(const float* scores, int n_rows, int64_t ld, const int32_t* n_valid, int64_t max_n, int k,
                         int32_t* out_idx, float* out_score, cudaStream_t stream, int nv_div = 1, int ordered = 0);
csa_status_t launch_block_max(const float* scores, int nq, int64_t ld, const int32_t* n_visible, int64_t cap,
                              int block, float* out, int64_t ld_out, cudaStream_t stream);
int topk_multi_ctas(int n_rows, int64_t max_n);
size_t topk_multi_ctl_bytes(int n_rows);
csa_status_t launch_topk_multi(const float* scores, int n_rows, int64_t ld, const int32_t* n_valid, int nv_div,
                               int64_t max_n, int k, int32_t* out_idx, float* out_score, int ordered, int G,
                               void* ctl, cudaStream_t stream);
uint32_t topk_multi_take_error();
bool index_many_tc_supported(const csa_params_t* p, int q_dtype, int k_dtype);
size_t index_many_tc_table_bytes(int nq);
csa_status_t launch_index_many_tc(const csa_params_t* p, int nq, const csa_tensor_t* q_idx, const float* w,
                                  const csa_tensor_t* k_idx, int batch, int64_t cap, const int32_t* q_req,
                                  const int32_t* n_visible, float* scores, int64_t ld, int32_t* table,
                                  cudaStream_t stream);
uint32_t index_many_take_error();
uint32_t attn_many_take_error();
csa_status_t launch_pool_map(const int32_t* pos, const float* pos_score, int nq, int k, const int32_t* pool, int block,
                             int pool_blocks, int32_t* out_idx, cudaStream_t stream);
csa_status_t launch_attention(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                              int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible, const int32_t* q_req,
                              const csa_tensor_t* swa_k, const csa_tensor_t* swa_v, const int64_t* q_pos,
                              const int64_t* swa_lo, const float* sink, const csa_tensor_t* out, float* lse,
                              void* workspace, int max_keys, cudaStream_t stream, bool pdl = false);
size_t attn_workspace_bytes(int nq, int hq, int d, int max_keys, int window);

csa_status_t set_error(csa_status_t st, const char* fmt, ...);

namespace {
thread_local char g_msg[512] = "";
}  // namespace

namespace {

// Workspace carve-up: consecutive 256-byte aligned regions.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t n) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// allow_mx4: MXFP4 main-KV rows (scale_group 16, E4M3 scale bytes).
csa_status_t check_tensor(const char* name, const csa_tensor_t* t, int row_elems, bool allow_f32, bool allow_bf16,
                          bool allow_fp8, int fp8_group, bool allow_mx4 = false) {
  if (t == nullptr || t->data == nullptr) return set_error(CSA_ERR_INVALID_ARG, "%s: null tensor", name);
  const int dt = t->dtype;
  if ((dt == kF32 && !allow_f32) || (dt == kBF16 && !allow_bf16) || (dt == kFP8 && !allow_fp8) ||
      (dt == kMXFP4 && !allow_mx4) || (dt != kF32 && dt != kBF16 && dt != kFP8 && dt != kMXFP4))
    return set_error(CSA_ERR_INVALID_ARG, "%s: dtype %d not accepted here", name, dt);
  if (!aligned16(t->data)) return set_error(CSA_ERR_INVALID_ARG, "%s: data not 16-byte aligned", name);
  if (row_bytes(dt, row_elems) % 16 != 0 || (dt == kMXFP4 && row_elems % 32 != 0))
    return set_error(CSA_ERR_INVALID_ARG, "%s: rows of %d elements are not a multiple of 16 bytes", name, row_elems);
  if (dt == kMXFP4) {
    if (t->scale == nullptr || !aligned16(t->scale))
      return set_error(CSA_ERR_INVALID_ARG, "%s: MXFP4 tensor without 16-byte aligned scales", name);
    if (t->scale_group != 16)
      return set_error(CSA_ERR_INVALID_ARG, "%s: MXFP4 scale_group must be 16 (got %d)", name, t->scale_group);
  }
  if (dt == kFP8) {
    if (t->scale == nullptr) return set_error(CSA_ERR_INVALID_ARG, "%s: FP8 tensor without scales", name);
    if (fp8_group > 0 && t->scale_group != fp8_group)
      return set_error(CSA_ERR_INVALID_ARG, "%s: FP8 scale_group must be %d (got %d)", name, fp8_group,
                       t->scale_group);
    if (t->scale_group <= 0 || t->scale_group % 8 != 0 || row_elems % t->scale_group != 0)
      return set_error(CSA_ERR_INVALID_ARG, "%s: bad FP8 scale_group %d", name, t->scale_group);
  }
  return CSA_OK;
}

}  // namespace

csa_status_t check_params(const csa_params_t* p, bool need_idx) {
  if (p == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null params");
  if (p->m < 1 || p->d < 8 || p->h_q < 1 || p->window < 0)
    return set_error(CSA_ERR_INVALID_ARG, "bad params (m=%d d=%d h_q=%d window=%d)", p->m, p->d, p->h_q, p->window);
  if (p->d % 8 != 0) return set_error(CSA_ERR_INVALID_ARG, "d=%d must be a multiple of 8", p->d);
  if (p->window > 0 && p->swa_cap < p->window)
    return set_error(CSA_ERR_INVALID_ARG, "swa_cap=%d smaller than window=%d", p->swa_cap, p->window);
  if (need_idx && (p->h_idx < 1 || p->d_idx < 8 || p->d_idx % 8 != 0))
    return set_error(CSA_ERR_INVALID_ARG, "bad indexer shape h_idx=%d d_idx=%d", p->h_idx, p->d_idx);
  return CSA_OK;
}

// Keys one query's attention covers: its selection (or, dense, the cache's
// rows) plus the window.  Computed in 64 bits; a count beyond INT_MAX is an
// invalid argument (the kernels index keys with 32-bit ints).
csa_status_t attention_max_keys(const csa_params_t* p, bool sparse, int64_t cap, int* out) {
  const int64_t mk = (sparse ? static_cast<int64_t>(p->topk) : cap) + p->window;
  if (mk < 0 || mk > static_cast<int64_t>(INT32_MAX))
    return set_error(CSA_ERR_INVALID_ARG, "attention over %lld keys per query (more than 2^31 - 1)",
                     static_cast<long long>(mk));
  *out = static_cast<int>(mk);
  return CSA_OK;
}

void clear_error() { g_msg[0] = 0; }

namespace {

size_t index_ws_bytes(int nq, int64_t cap) {
  Carver c(nullptr);
  c.take<float>(static_cast<size_t>(nq) * round_up(cap, 4));
  c.take<char>(index_many_tc_table_bytes(nq));
  return c.off;
}

// Scores of many queries per request: the tensor-core contraction where the
// shapes allow it (64 x 128 bf16 indexer, 16-byte aligned head weights),
// else the CUDA-core scorer.
csa_status_t score_many(const csa_params_t* p, int nq, const csa_tensor_t* q_idx, const float* w,
                        const csa_tensor_t* k_idx, int batch, int64_t cap, const int32_t* q_req,
                        const int32_t* n_visible, float* scores, int64_t ld, int32_t* table, cudaStream_t s) {
  if (index_many_tc_supported(p, q_idx->dtype, k_idx->dtype) && aligned16(w))
    return launch_index_many_tc(p, nq, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, table, s);
  return launch_index_score(p, nq, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, cap, s);
}

// Full layer of the hierarchical indexer: the block maxima, then either all
// scores (CUDA-core scoring) or the fused indexer's workspace and a top-k
// scratch for a caller that wants the pool alone.
size_t pool_ws_bytes(const csa_params_t* p, int nq, int64_t cap, int block) {
  Carver c(nullptr);
  c.take<float>(static_cast<size_t>(nq) * round_up((cap + block - 1) / block, 4));
  c.take<char>(topk_multi_ctl_bytes(nq));
  const size_t head = c.off;
  c.take<float>(static_cast<size_t>(nq) * round_up(cap, 4));
  size_t need = c.off;
  if (p->topk >= 1 && p->h_idx > 0 && p->d_idx > 0) {
    Carver t(nullptr);
    t.off = head;
    t.take<int32_t>(static_cast<size_t>(nq) * p->topk);
    t.take<char>(index_tc_workspace_bytes(nq, cap, p->topk));
    if (t.off > need) need = t.off;
  }
  return need;
}

// Reindex layer: the pool's scores, the selected pool positions and their scores.
size_t reindex_ws_bytes(int nq, int block, int pool_blocks, int k) {
  Carver c(nullptr);
  c.take<float>(static_cast<size_t>(nq) * round_up(static_cast<int64_t>(block) * pool_blocks, 4));
  c.take<int32_t>(static_cast<size_t>(nq) * k);
  c.take<float>(static_cast<size_t>(nq) * k);
  return c.off;
}

csa_status_t check_pool_shape(int32_t block, int32_t pool_blocks) {
  if (block < 1 || block > 128 || (block & (block - 1)) != 0)
    return set_error(CSA_ERR_INVALID_ARG, "block=%d must be a power of two in [1, 128]", block);
  if (pool_blocks < 1 || static_cast<int64_t>(block) * pool_blocks > (int64_t(1) << 30))
    return set_error(CSA_ERR_INVALID_ARG, "bad pool_blocks=%d", pool_blocks);
  return CSA_OK;
}

}  // namespace

csa_status_t set_error(csa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

// ---- per-launch event profiler (csa_profile_*) ----
namespace {
std::mutex g_prof_mu;
bool g_prof_on = false;
bool g_prof_open = false;            // a begin event is recorded, its end is not
int g_prof_n = 0;
std::vector<cudaEvent_t> g_prof_ev;  // 2 per record
std::vector<const char*> g_prof_name;
}  // namespace

void prof_begin(cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on || 2 * (g_prof_n + 1) > static_cast<int>(g_prof_ev.size())) return;
  cudaEventRecord(g_prof_ev[2 * g_prof_n], stream);
  g_prof_open = true;
}

csa_status_t check_launch(const char* what, cudaStream_t stream) {
  cudaError_t e = cudaGetLastError();
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof_open) {
      cudaEventRecord(g_prof_ev[2 * g_prof_n + 1], stream);
      g_prof_name[g_prof_n] = what;
      ++g_prof_n;
      g_prof_open = false;
    }
  }
  if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return CSA_OK;
}

}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_last_error(void) { return g_msg; }

size_t csa_workspace_size(const csa_params_t* p, int32_t n_queries, int64_t max_entries) {
  if (p == nullptr || n_queries < 0 || max_entries < 0) return 0;
  const int64_t mk = (p->topk > 0 ? static_cast<int64_t>(p->topk) : max_entries) + p->window;
  if (mk < 0 || mk > static_cast<int64_t>(INT32_MAX)) return 0;
  const int max_keys = static_cast<int>(mk);
  Carver c(nullptr);
  // decode-step bookkeeping
  c.take<int32_t>(n_queries);
  c.take<int64_t>(n_queries);
  c.take<int32_t>(n_queries);
  if (p->topk > 0) {
    c.take<int32_t>(static_cast<size_t>(n_queries) * p->topk);
    size_t ib = index_ws_bytes(n_queries, max_entries);
    if (p->h_idx > 0 && p->d_idx > 0) {
      const size_t tb = index_tc_workspace_bytes(n_queries, max_entries, p->topk);
      if (tb > ib) ib = tb;
    }
    c.take<char>(ib);
  }
  const size_t attn = attn_workspace_bytes(n_queries, p->h_q, p->d, max_keys, p->window);
  return c.off + attn + 256;
}

csa_status_t csa_compress(const csa_tensor_t* C, const csa_tensor_t* Z, int32_t batch, int64_t n_tokens, int32_t d,
                          int32_t m, const csa_tensor_t* out, int64_t out_rows, const csa_tensor_t* w_ik,
                          int32_t d_idx, const csa_tensor_t* kidx_out, csa_stream_t stream) {
  g_msg[0] = 0;
  if (batch < 0 || n_tokens < 0 || m < 1 || d < 8 || d % 8 != 0)
    return set_error(CSA_ERR_INVALID_ARG, "bad shape batch=%d n_tokens=%lld d=%d m=%d", batch,
                     static_cast<long long>(n_tokens), d, m);
  if (out_rows < n_tokens / m) return set_error(CSA_ERR_INVALID_ARG, "out_rows smaller than n_tokens / m");
  csa_status_t st;
  if ((st = check_tensor("C", C, d, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("Z", Z, d, true, true, false, 0)) != CSA_OK) return st;
  if (Z->dtype != C->dtype) return set_error(CSA_ERR_INVALID_ARG, "C and Z dtypes differ");
  if ((st = check_tensor("out", out, d, true, true, true, 64, true)) != CSA_OK) return st;
  if (w_ik != nullptr) {
    if (d_idx < 32 || d_idx > 256 || d_idx % 32 != 0)
      return set_error(CSA_ERR_UNSUPPORTED, "d_idx=%d: projection needs a multiple of 32 in [32, 256]", d_idx);
    if ((st = check_tensor("w_ik", w_ik, d_idx, true, true, false, 0)) != CSA_OK) return st;
    if ((st = check_tensor("kidx_out", kidx_out, d_idx, true, true, true, d_idx)) != CSA_OK) return st;
    if (static_cast<size_t>(8) * d * sizeof(float) > 200 * 1024)
      return set_error(CSA_ERR_UNSUPPORTED, "d=%d too large for the projection stage", d);
  }
  return launch_compress(C, Z, batch, n_tokens, d, m, out, out_rows, w_ik, d_idx, kidx_out,
                         reinterpret_cast<cudaStream_t>(stream));
}

size_t csa_topk_workspace_size(int32_t n_rows) { return n_rows > 0 ? topk_multi_ctl_bytes(n_rows) : 0; }

csa_status_t csa_topk(const float* scores, int32_t n_rows, int64_t ld, const int32_t* n_valid, int32_t k,
                      int32_t* out_idx, float* out_score, void* workspace, size_t workspace_bytes,
                      csa_stream_t stream) {
  g_msg[0] = 0;
  if (n_rows < 0 || k < 1 || ld < 0) return set_error(CSA_ERR_INVALID_ARG, "bad shape n_rows=%d k=%d", n_rows, k);
  if (n_rows == 0) return CSA_OK;
  if (scores == nullptr || n_valid == nullptr || out_idx == nullptr)
    return set_error(CSA_ERR_INVALID_ARG, "null pointer");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int G = topk_multi_ctas(n_rows, ld);
  if (G > 0 && workspace != nullptr && workspace_bytes >= topk_multi_ctl_bytes(n_rows))
    return launch_topk_multi(scores, n_rows, ld, n_valid, 1, ld, k, out_idx, out_score, 0, G, workspace, s);
  return launch_topk(scores, n_rows, ld, n_valid, ld, k, out_idx, out_score, s);
}

csa_status_t csa_index_topk(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx, const float* w,
                            const csa_tensor_t* k_idx, int32_t batch, int64_t cap, const int32_t* q_req, const int32_t* n_visible,
                            int32_t* out_idx, float* out_score, void* workspace, size_t workspace_bytes,
                            csa_stream_t stream) {
  g_msg[0] = 0;
  csa_status_t st;
  if ((st = check_params(p, true)) != CSA_OK) return st;
  if (p->topk < 1) return set_error(CSA_ERR_INVALID_ARG, "csa_index_topk needs topk >= 1");
  if (n_queries < 0 || cap < 0 || batch < 1) return set_error(CSA_ERR_INVALID_ARG, "bad n_queries / batch / cap");
  if (n_queries == 0) return CSA_OK;
  if ((st = check_tensor("q_idx", q_idx, p->d_idx, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("k_idx", k_idx, p->d_idx, true, true, true, p->d_idx)) != CSA_OK) return st;
  if (w == nullptr || n_visible == nullptr || out_idx == nullptr)
    return set_error(CSA_ERR_INVALID_ARG, "null w / n_visible / out_idx");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (q_req == nullptr && n_queries == batch && index_tc_supported(p, batch, cap, q_idx->dtype, k_idx->dtype)) {
    // one query per request: the fused tensor-core kernel
    const size_t need = index_tc_workspace_bytes(batch, cap, p->topk);
    if (workspace == nullptr || workspace_bytes < need)
      return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);
    cudaError_t e = cudaMemsetAsync(workspace, 0, index_tc_control_bytes(batch), s);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    return launch_index_topk_tc(p, batch, q_idx, w, k_idx, cap, n_visible, out_idx, out_score, workspace, s);
  }
  const size_t need = index_ws_bytes(n_queries, cap);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  Carver c(workspace);
  const int64_t ld = round_up(cap, 4);
  float* scores = c.take<float>(static_cast<size_t>(n_queries) * ld);
  int32_t* table = reinterpret_cast<int32_t*>(c.take<char>(index_many_tc_table_bytes(n_queries)));
  if ((st = score_many(p, n_queries, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, table, s)) != CSA_OK)
    return st;
  return launch_topk(scores, n_queries, ld, n_visible, cap, p->topk, out_idx, out_score, s);
}

namespace {

csa_status_t check_index_args(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx, const float* w,
                              const csa_tensor_t* k_idx, int32_t batch, int64_t cap, const int32_t* n_visible) {
  csa_status_t st;
  if ((st = check_params(p, true)) != CSA_OK) return st;
  if (n_queries < 0 || cap < 0 || batch < 1) return set_error(CSA_ERR_INVALID_ARG, "bad n_queries / batch / cap");
  if (n_queries == 0) return CSA_OK;
  if ((st = check_tensor("q_idx", q_idx, p->d_idx, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("k_idx", k_idx, p->d_idx, true, true, true, p->d_idx)) != CSA_OK) return st;
  if (w == nullptr || n_visible == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null w / n_visible");
  return CSA_OK;
}

}  // namespace

size_t csa_index_pool_workspace_size(const csa_params_t* p, int32_t n_queries, int64_t max_entries, int32_t block,
                                     int32_t pool_blocks) {
  if (p == nullptr || n_queries < 0 || max_entries < 0 || block < 1 || pool_blocks < 1) return 0;
  const size_t a = pool_ws_bytes(p, n_queries, max_entries, block);
  size_t b = reindex_ws_bytes(n_queries, block, pool_blocks, p->topk > 0 ? p->topk : 1);
  if (p->topk >= 1 && p->h_idx > 0 && p->d_idx > 0) {
    const size_t t = index_tc_workspace_bytes(n_queries, static_cast<int64_t>(block) * pool_blocks, p->topk);
    if (t > b) b = t;
  }
  return (a > b ? a : b) + 256;
}

csa_status_t csa_index_topk_pool(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx, const float* w,
                                 const csa_tensor_t* k_idx, int32_t batch, int64_t cap, const int32_t* q_req,
                                 const int32_t* n_visible, int32_t block, int32_t pool_blocks, int32_t* out_pool,
                                 int32_t* out_idx, float* out_score, void* workspace, size_t workspace_bytes,
                                 csa_stream_t stream) {
  g_msg[0] = 0;
  csa_status_t st;
  if ((st = check_index_args(p, n_queries, q_idx, w, k_idx, batch, cap, n_visible)) != CSA_OK) return st;
  if ((st = check_pool_shape(block, pool_blocks)) != CSA_OK) return st;
  if (out_idx != nullptr && p->topk < 1) return set_error(CSA_ERR_INVALID_ARG, "out_idx needs topk >= 1");
  if (n_queries == 0) return CSA_OK;
  if (out_pool == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null out_pool");
  const size_t need = pool_ws_bytes(p, n_queries, cap, block);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carver c(workspace);
  const int64_t ld = round_up(cap, 4);
  const int64_t nb = (cap + block - 1) / block, ldb = round_up(nb, 4);
  float* bmax = c.take<float>(static_cast<size_t>(n_queries) * ldb);
  void* mctl = c.take<char>(topk_multi_ctl_bytes(n_queries));
  // the pool: the best blocks in ascending order, several CTAs per query when
  // the rows are long (one SM would take ~100 us over 131,072 maxima)
  auto select_pool = [&]() -> csa_status_t {
    const int G = topk_multi_ctas(n_queries, nb);
    if (G > 0)
      return launch_topk_multi(bmax, n_queries, ldb, n_visible, block, nb, pool_blocks, out_pool, nullptr, 1, G, mctl,
                               s);
    return launch_topk(bmax, n_queries, ldb, n_visible, nb, pool_blocks, out_pool, nullptr, s, block, 1);
  };
  if (q_req == nullptr && n_queries == batch && p->topk >= 1 &&
      index_tc_supported(p, batch, cap, q_idx->dtype, k_idx->dtype)) {
    // the fused tensor-core indexer writes its top-k and the block maxima
    int32_t* idx = c.take<int32_t>(static_cast<size_t>(n_queries) * p->topk);
    void* tws = c.take<char>(index_tc_workspace_bytes(batch, cap, p->topk));
    cudaError_t e = cudaMemsetAsync(tws, 0, index_tc_control_bytes(batch), s);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    if ((st = launch_index_topk_tc(p, batch, q_idx, w, k_idx, cap, n_visible, out_idx ? out_idx : idx, out_score,
                                   tws, s, nullptr, bmax, ldb, block)) != CSA_OK)
      return st;
    return select_pool();
  }
  float* scores = c.take<float>(static_cast<size_t>(n_queries) * ld);
  if ((st = launch_index_score(p, n_queries, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, cap, s)) !=
      CSA_OK)
    return st;
  if (out_idx != nullptr &&
      (st = launch_topk(scores, n_queries, ld, n_visible, cap, p->topk, out_idx, out_score, s)) != CSA_OK)
    return st;
  if ((st = launch_block_max(scores, n_queries, ld, n_visible, cap, block, bmax, ldb, s)) != CSA_OK) return st;
  return select_pool();
}

csa_status_t csa_index_topk_reindex(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx,
                                    const float* w, const csa_tensor_t* k_idx, int32_t batch, int64_t cap,
                                    const int32_t* q_req, const int32_t* n_visible, const int32_t* pool, int32_t block,
                                    int32_t pool_blocks, int32_t* out_idx, float* out_score, void* workspace,
                                    size_t workspace_bytes, csa_stream_t stream) {
  g_msg[0] = 0;
  csa_status_t st;
  if ((st = check_index_args(p, n_queries, q_idx, w, k_idx, batch, cap, n_visible)) != CSA_OK) return st;
  if ((st = check_pool_shape(block, pool_blocks)) != CSA_OK) return st;
  if (p->topk < 1) return set_error(CSA_ERR_INVALID_ARG, "csa_index_topk_reindex needs topk >= 1");
  if (n_queries == 0) return CSA_OK;
  if (pool == nullptr || out_idx == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null pool / out_idx");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (q_req == nullptr && n_queries == batch &&
      index_tc_pool_supported(p, batch, cap, block, pool_blocks, q_idx->dtype, k_idx->dtype)) {
    // one query per request: the fused tensor-core indexer over the pool
    const size_t need = index_tc_workspace_bytes(batch, static_cast<int64_t>(block) * pool_blocks, p->topk);
    if (workspace == nullptr || workspace_bytes < need)
      return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);
    cudaError_t e = cudaMemsetAsync(workspace, 0, index_tc_control_bytes(batch), s);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    return launch_index_topk_tc(p, batch, q_idx, w, k_idx, cap, n_visible, out_idx, out_score, workspace, s, nullptr,
                                nullptr, 0, 1, pool, pool_blocks, block);
  }
  const size_t need = reindex_ws_bytes(n_queries, block, pool_blocks, p->topk);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  Carver c(workspace);
  const int64_t np = static_cast<int64_t>(block) * pool_blocks, ld = round_up(np, 4);
  float* scores = c.take<float>(static_cast<size_t>(n_queries) * ld);
  int32_t* pos = c.take<int32_t>(static_cast<size_t>(n_queries) * p->topk);
  float* pos_score = c.take<float>(static_cast<size_t>(n_queries) * p->topk);
  if ((st = launch_index_score(p, n_queries, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, np, s, pool,
                               block, pool_blocks)) != CSA_OK)
    return st;
  if ((st = launch_topk(scores, n_queries, ld, nullptr, np, p->topk, pos, pos_score, s)) != CSA_OK) return st;
  if (out_score != nullptr) {
    cudaError_t e = cudaMemcpyAsync(out_score, pos_score, static_cast<size_t>(n_queries) * p->topk * sizeof(float),
                                    cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
  }
  return launch_pool_map(pos, pos_score, n_queries, p->topk, pool, block, pool_blocks, out_idx, s);
}

csa_status_t csa_sparse_swa_attention(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q,
                                      const csa_tensor_t* kv, int32_t batch, int64_t cap, const int32_t* idx,
                                      const int32_t* n_visible, const int32_t* q_req, const csa_tensor_t* swa_k,
                                      const csa_tensor_t* swa_v, const int64_t* q_pos, const int64_t* swa_lo,
                                      const float* sink, const csa_tensor_t* out, float* lse, void* workspace,
                                      size_t workspace_bytes, csa_stream_t stream) {
  g_msg[0] = 0;
  csa_status_t st;
  if ((st = check_params(p, false)) != CSA_OK) return st;
  if (n_queries < 0 || cap < 0 || batch < 1) return set_error(CSA_ERR_INVALID_ARG, "bad n_queries / batch / cap");
  if (n_queries == 0) return CSA_OK;
  if ((st = check_tensor("q", q, p->d, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("kv", kv, p->d, true, true, true, 64, true)) != CSA_OK) return st;
  if ((st = check_tensor("out", out, p->d, true, true, false, 0)) != CSA_OK) return st;
  if (p->window > 0) {
    if ((st = check_tensor("swa_k", swa_k, p->d, true, true, false, 0)) != CSA_OK) return st;
    if ((st = check_tensor("swa_v", swa_v, p->d, true, true, false, 0)) != CSA_OK) return st;
    if (swa_k->dtype != swa_v->dtype) return set_error(CSA_ERR_INVALID_ARG, "swa_k / swa_v dtypes differ");
  }
  if (n_visible == nullptr || q_pos == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null n_visible / q_pos");
  if (idx != nullptr && p->topk < 1) return set_error(CSA_ERR_INVALID_ARG, "idx given with topk < 1");
  int max_keys = 0;
  if ((st = attention_max_keys(p, idx != nullptr, cap, &max_keys)) != CSA_OK) return st;
  const size_t need = attn_workspace_bytes(n_queries, p->h_q, p->d, max_keys, p->window);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  return launch_attention(p, n_queries, q, kv, batch, cap, idx, n_visible, q_req, swa_k, swa_v, q_pos, swa_lo, sink, out,
                          lse, workspace, max_keys, reinterpret_cast<cudaStream_t>(stream));
}

csa_status_t csa_decode_step(const csa_params_t* p, int32_t batch, const csa_decode_caches_t* cc,
                             const csa_decode_token_t* tok, const int64_t* pos, const csa_tensor_t* out, float* lse,
                             int32_t* out_idx, void* workspace, size_t workspace_bytes, csa_stream_t stream) {
  g_msg[0] = 0;
  csa_status_t st;
  const bool sparse = p && p->topk > 0;
  // the indexer-key projection runs when the caller passes a projection (always for CSA)
  const bool project = tok && tok->w_ik.data != nullptr;
  if ((st = check_params(p, sparse || project)) != CSA_OK) return st;
  if (cc == nullptr || tok == nullptr || pos == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null caches / token / pos");
  if (batch < 0) return set_error(CSA_ERR_INVALID_ARG, "bad batch");
  if (batch == 0) return CSA_OK;
  if (p->window < 1) return set_error(CSA_ERR_INVALID_ARG, "decode step needs window >= 1 (the token's own SWA slot)");
  if (sparse && !project) return set_error(CSA_ERR_INVALID_ARG, "a sparse (topk >= 1) step needs w_ik");
  if (project && (p->d_idx < 32 || p->d_idx > 256 || p->d_idx % 32 != 0))
    return set_error(CSA_ERR_UNSUPPORTED, "d_idx=%d: projection needs a multiple of 32 in [32, 256]", p->d_idx);
  if ((st = check_tensor("kv", &cc->kv, p->d, true, true, true, 64, true)) != CSA_OK) return st;
  if (project && (st = check_tensor("kidx", &cc->kidx, p->d_idx, true, true, true, p->d_idx)) != CSA_OK) return st;
  if ((st = check_tensor("swa_k", &cc->swa_k, p->d, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("swa_v", &cc->swa_v, p->d, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("open_c", &cc->open_c, p->d, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("open_z", &cc->open_z, p->d, true, true, false, 0)) != CSA_OK) return st;
  const int act = tok->c.dtype;
  const csa_tensor_t* acts[] = {&tok->c, &tok->z, &tok->k_swa, &tok->v_swa};
  const char* names[] = {"c", "z", "k_swa", "v_swa"};
  for (int i = 0; i < 4; ++i) {
    if ((st = check_tensor(names[i], acts[i], p->d, true, true, false, 0)) != CSA_OK) return st;
    if (acts[i]->dtype != act) return set_error(CSA_ERR_INVALID_ARG, "token rows must share one dtype");
  }
  if (cc->open_c.dtype != act || cc->open_z.dtype != act)
    return set_error(CSA_ERR_INVALID_ARG, "open-block buffers must have the token rows' dtype");
  if (cc->swa_k.dtype != cc->swa_v.dtype) return set_error(CSA_ERR_INVALID_ARG, "swa_k / swa_v dtypes differ");
  if ((st = check_tensor("q", &tok->q, p->d, true, true, false, 0)) != CSA_OK) return st;
  if (project && (st = check_tensor("w_ik", &tok->w_ik, p->d_idx, true, true, false, 0)) != CSA_OK) return st;
  if (sparse) {
    if ((st = check_tensor("q_idx", &tok->q_idx, p->d_idx, true, true, false, 0)) != CSA_OK) return st;
    if (tok->w == nullptr) return set_error(CSA_ERR_INVALID_ARG, "null indexer weights");
  }
  if ((st = check_tensor("out", out, p->d, true, true, false, 0)) != CSA_OK) return st;
  int max_keys = 0;
  if ((st = attention_max_keys(p, sparse, cc->cap, &max_keys)) != CSA_OK) return st;
  const size_t need = csa_workspace_size(p, batch, cc->cap);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(CSA_ERR_CAPACITY, "workspace of %zu bytes, need %zu", workspace_bytes, need);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carver c(workspace);
  int32_t* n_vis = c.take<int32_t>(batch);
  int64_t* q_pos = c.take<int64_t>(batch);
  int32_t* q_req = c.take<int32_t>(batch);
  int32_t* idx = nullptr;
  void* index_ws = nullptr;
  const bool tc = sparse && index_tc_supported(p, batch, cc->cap, tok->q_idx.dtype, cc->kidx.dtype);
  if (sparse) {
    idx = c.take<int32_t>(static_cast<size_t>(batch) * p->topk);
    if (out_idx != nullptr) idx = out_idx;  // the caller keeps the selection
    size_t ib = index_ws_bytes(batch, cc->cap);
    const size_t tb = index_tc_workspace_bytes(batch, cc->cap, p->topk);
    index_ws = c.take<char>(ib > tb ? ib : tb);
  }
  void* attn_ws = c.take<char>(attn_workspace_bytes(batch, p->h_q, p->d, max_keys, p->window));

  // CSA on the tensor-core indexer: the token is appended inside the indexer
  // (by the CTA that owns each request's last chunk); otherwise by its own kernel
  const bool fused = tc && index_tc_append_supported(p, tok->w_ik.dtype);
  if (fused) {
    const cudaError_t e = cudaMemsetAsync(index_ws, 0, index_tc_control_bytes(batch), s);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
    AppendArgs ap;
    ap.pos = pos;
    ap.m = p->m;
    ap.d = p->d;
    ap.act_dtype = tok->c.dtype;
    ap.c_t = tok->c.data;
    ap.z_t = tok->z.data;
    ap.k_t = tok->k_swa.data;
    ap.v_t = tok->v_swa.data;
    ap.open_c = cc->open_c.data;
    ap.open_z = cc->open_z.data;
    ap.swa_k = cc->swa_k.data;
    ap.swa_v = cc->swa_v.data;
    ap.swa_dtype = cc->swa_k.dtype;
    ap.swa_cap = p->swa_cap;
    ap.kv = make_out_spec(&cc->kv, p->d);
    ap.w_ik = tok->w_ik.data;
    ap.w_dtype = tok->w_ik.dtype;
    ap.kidx = make_out_spec(&cc->kidx, p->d_idx);
    ap.n_vis_out = n_vis;
    ap.q_pos_out = q_pos;
    ap.q_req_out = q_req;
    ap.shrink = 0;
    if ((st = launch_index_topk_tc(p, batch, &tok->q_idx, tok->w, &cc->kidx, cc->cap, n_vis, idx, nullptr, index_ws,
                                   s, &ap)) != CSA_OK)
      return st;
  } else if ((st = launch_decode_append(p, batch, cc, tok, pos, n_vis, q_pos, q_req, tc ? index_ws : nullptr,
                                        tc ? index_tc_control_bytes(batch) : 0, s)) != CSA_OK) {
    return st;
  }
  if (tc && !fused) {
    if ((st = launch_index_topk_tc(p, batch, &tok->q_idx, tok->w, &cc->kidx, cc->cap, n_vis, idx, nullptr, index_ws,
                                   s)) != CSA_OK)
      return st;
  } else if (sparse && !tc) {
    const int64_t ld = round_up(cc->cap, 4);
    float* scores = static_cast<float*>(index_ws);
    if ((st = launch_index_score(p, batch, &tok->q_idx, tok->w, &cc->kidx, batch, cc->cap, q_req, n_vis, scores, ld,
                                 cc->cap, s)) != CSA_OK)
      return st;
    if ((st = launch_topk(scores, batch, ld, n_vis, cc->cap, p->topk, idx, nullptr, s)) != CSA_OK) return st;
  }
  // a programmatic launch: the attention's prologue overlaps the tail of the
  // kernel before it (this step's indexer or append), whose outputs it
  // reads only after a grid-dependency wait
  return launch_attention(p, batch, &tok->q, &cc->kv, batch, cc->cap, idx, n_vis, q_req, &cc->swa_k, &cc->swa_v, q_pos,
                          nullptr, tok->sink, out, lse, attn_ws, max_keys, s, /*pdl=*/true);
}

csa_status_t csa_index_score(const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q_idx, const float* w,
                             const csa_tensor_t* k_idx, int32_t batch, int64_t cap, const int32_t* q_req,
                             const int32_t* n_visible, float* scores, int64_t ld, csa_stream_t stream) {
  g_msg[0] = 0;
  csa_status_t st;
  if ((st = check_params(p, true)) != CSA_OK) return st;
  if (n_queries < 0 || cap < 0 || batch < 1 || ld < cap)
    return set_error(CSA_ERR_INVALID_ARG, "bad n_queries / batch / cap / ld");
  if (n_queries == 0) return CSA_OK;
  if ((st = check_tensor("q_idx", q_idx, p->d_idx, true, true, false, 0)) != CSA_OK) return st;
  if ((st = check_tensor("k_idx", k_idx, p->d_idx, true, true, true, p->d_idx)) != CSA_OK) return st;
  if (w == nullptr || n_visible == nullptr || scores == nullptr)
    return set_error(CSA_ERR_INVALID_ARG, "null w / n_visible / scores");
  return launch_index_score(p, n_queries, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, cap,
                            reinterpret_cast<cudaStream_t>(stream));
}

csa_status_t csa_profile_start(int32_t max_launches) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (max_launches < 1) return set_error(CSA_ERR_INVALID_ARG, "max_launches must be >= 1");
  for (cudaEvent_t e : g_prof_ev) cudaEventDestroy(e);
  g_prof_ev.assign(2 * static_cast<size_t>(max_launches), nullptr);
  g_prof_name.assign(max_launches, nullptr);
  for (auto& e : g_prof_ev) {
    cudaError_t err = cudaEventCreate(&e);
    if (err != cudaSuccess) {
      g_prof_on = false;
      return set_error(CSA_ERR_CUDA, "cudaEventCreate: %s", cudaGetErrorString(err));
    }
  }
  g_prof_n = 0;
  g_prof_open = false;
  g_prof_on = true;
  return CSA_OK;
}

csa_status_t csa_profile_stop(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  g_prof_open = false;
  return CSA_OK;
}

int32_t csa_profile_count(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return g_prof_n;
}

csa_status_t csa_profile_get(int32_t i, const char** name, float* ms) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (i < 0 || i >= g_prof_n) return set_error(CSA_ERR_INVALID_ARG, "no profile record %d", i);
  cudaError_t e = cudaEventSynchronize(g_prof_ev[2 * i + 1]);
  if (e == cudaSuccess) e = cudaEventElapsedTime(ms, g_prof_ev[2 * i], g_prof_ev[2 * i + 1]);
  if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "profile record %d: %s", i, cudaGetErrorString(e));
  if (name) *name = g_prof_name[i];
  return CSA_OK;
}

csa_status_t csa_test_expire_next_barrier(int32_t cta, uint32_t polls) {
  g_msg[0] = 0;
  return test_expire_next_barrier(cta < 0 ? -1 : cta, polls);
}

csa_status_t csa_sync_status(csa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  if (index_tc_take_error() != 0)
    return set_error(CSA_ERR_TIMEOUT, "a bounded device-side wait of the indexer gave up");
  if (attn_tc_take_error() != 0)
    return set_error(CSA_ERR_TIMEOUT, "a bounded device-side wait of the attention gave up");
  if (topk_multi_take_error() != 0)
    return set_error(CSA_ERR_TIMEOUT, "a bounded device-side wait of the multi-CTA top-k gave up");
  if (index_many_take_error() != 0)
    return set_error(CSA_ERR_TIMEOUT, "a bounded device-side wait of the many-query indexer gave up");
  if (attn_many_take_error() != 0)
    return set_error(CSA_ERR_TIMEOUT, "a bounded device-side wait of the many-query attention gave up");
  return CSA_OK;
}

}  // extern "C"
