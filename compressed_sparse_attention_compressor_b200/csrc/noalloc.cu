// csa_sparse_swa_attention_noalloc: the attention entry point with its
// scratch space in a fixed device array owned by this library, for callers
// that cannot allocate device memory themselves.
//
// Some callers cannot call cudaMalloc or keep a caching allocator: a plugin
// whose host application owns every byte of device memory, or a tight serving
// loop in which cudaMalloc's implicit device-wide synchronisation is not
// acceptable.  This entry point takes the same inputs and outputs as
// csa_sparse_swa_attention but no workspace: the per-split partial softmax
// states it needs live in g_attn_scratch below, which every GPU that loads
// the library keeps until the process exits.
#include <mutex>

#include "common.cuh"

// 16 MiB of scratch per device.  In host code this name is only a stand-in
// for the device symbol: its device address comes from cudaGetSymbolAddress,
// once per device.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_attn_scratch[kNoAllocScratchBytes];

namespace csa {

size_t attn_workspace_bytes(int nq, int hq, int d, int max_keys, int window);
csa_status_t check_params(const csa_params_t* p, bool need_idx);
csa_status_t attention_max_keys(const csa_params_t* p, bool sparse, int64_t cap, int* out);
void clear_error();

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device, looked up on the
// first call made with that device current.
csa_status_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(CSA_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(CSA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return CSA_OK;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" csa_status_t csa_sparse_swa_attention_noalloc(
    const csa_params_t* p, int32_t n_queries, const csa_tensor_t* q, const csa_tensor_t* kv, int32_t batch,
    int64_t cap, const int32_t* idx, const int32_t* n_visible, const int32_t* q_req, const csa_tensor_t* swa_k,
    const csa_tensor_t* swa_v, const int64_t* q_pos, const int64_t* swa_lo, const float* sink,
    const csa_tensor_t* out, float* lse, csa_stream_t stream) {
  clear_error();
  // the same checks as csa_sparse_swa_attention before the scratch is sized,
  // so that bad parameters give the same status from both entry points
  csa_status_t st = check_params(p, false);
  if (st != CSA_OK) return st;
  if (n_queries < 0 || cap < 0 || batch < 1) return set_error(CSA_ERR_INVALID_ARG, "bad n_queries / batch / cap");
  if (idx != nullptr && p->topk < 1) return set_error(CSA_ERR_INVALID_ARG, "idx given with topk < 1");
  int max_keys = 0;
  if ((st = attention_max_keys(p, idx != nullptr, cap, &max_keys)) != CSA_OK) return st;
  const size_t need = attn_workspace_bytes(n_queries, p->h_q, p->d, max_keys, p->window);
  if (need > kNoAllocScratchBytes)
    return set_error(CSA_ERR_CAPACITY,
                     "csa_sparse_swa_attention_noalloc: this problem needs %zu bytes of scratch, more than the "
                     "library's fixed %zu; use csa_sparse_swa_attention with a caller workspace",
                     need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != CSA_OK) return st;
  // Nothing in the scratch needs clearing: every split state the merge reads
  // is written by this call first.
  return csa_sparse_swa_attention(p, n_queries, q, kv, batch, cap, idx, n_visible, q_req, swa_k, swa_v, q_pos, swa_lo,
                                  sink, out, lse, scratch, kNoAllocScratchBytes, stream);
}
