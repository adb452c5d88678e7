// K4 -- sparse (CSA) or dense (HCA) attention over compressed entries,
// continued over the sliding window and closed with the sink, in one online
// softmax.
//
// Atlas "Model architectures": "compressed KV" entry (top-k selected
// compressed entries plus a sliding window for CSA; dense attention over all
// compressed entries for HCA), "Sliding-window attention" entry (rolling
// buffer), "MLA" entry (attention over the latent directly, so the entry is
// both key and value).  Tech-report tour, "The indexer selects, SWA covers
// the rest" (the query attends to the selected entries together with the
// layer-local sliding-window KV); "Replay only the window" (keys in
// [max(s, i-W+1), i]).
//
// Work split: the list of keys of a query -- its selected entries followed
// by its window positions -- is cut into `n_splits` ranges; one CTA handles
// one range of one query for all heads, keeping a running (max, sum, acc[d])
// per head.  With one split the CTA finishes the softmax itself (sink,
// normalisation, lse); otherwise every CTA writes its partial state and a
// merge kernel combines the partials by their log-sum-exp.
#include "common.cuh"

namespace csa {

namespace {

constexpr int kAttnThreads = 256;

__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }

template <int HQ, int D>
struct AttnCfg {
  static constexpr int TE = (D >= 512) ? 16 : 32;     // keys per tile
  static constexpr int LDS = D + 4;                  // padded smem row (floats)
  static constexpr int PP = HQ * TE / kAttnThreads;  // logits per thread
  static constexpr int RE = cmin(PP, 4);
  static constexpr int RH = PP / RE;
  static constexpr int TPH = kAttnThreads / HQ;      // threads per head (accumulate)
  static constexpr int ACC4 = D / 4 / TPH;           // float4 accumulators per thread
  static_assert(PP >= 1 && RE * RH == PP, "tile shape");
  static_assert((HQ / RH) * (TE / RE) == kAttnThreads, "thread map");
  static_assert(ACC4 >= 1 && ACC4 * TPH * 4 == D, "accumulator map");
  static constexpr size_t smem_floats =
      static_cast<size_t>(HQ) * LDS + 2 * static_cast<size_t>(TE) * LDS + static_cast<size_t>(HQ) * TE + 3 * HQ;
};

struct AttnArgs {
  const void* q; int q_dtype;
  const void* kv; const void* kv_scale; int kv_dtype; int kv_group; int batch; int64_t cap;
  const int32_t* idx; int topk;           // idx == nullptr: dense over n_visible
  const int32_t* n_visible; const int32_t* q_req;
  const void* swa_k; const void* swa_v; int swa_dtype; int swa_cap; int window;
  const int64_t* q_pos; const int64_t* swa_lo;
  const float* sink; float tau;
  void* out; int out_dtype; float* lse;
  float* part;        // [nq][n_splits][HQ][D + 2] (m, l, acc) when n_splits > 1
  int n_splits; int per_split;
};

template <int HQ, int D>
__global__ void __launch_bounds__(kAttnThreads)
attn_simt_kernel(AttnArgs a) {
  using Cfg = AttnCfg<HQ, D>;
  constexpr int TE = Cfg::TE, LDS = Cfg::LDS, RE = Cfg::RE, RH = Cfg::RH, TPH = Cfg::TPH, ACC4 = Cfg::ACC4;
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;                      // [HQ][LDS]   tau * q
  float* ks = qs + HQ * LDS;             // [TE][LDS]   key rows
  float* vs = ks + TE * LDS;             // [TE][LDS]   value rows (window entries only)
  float* ps = vs + TE * LDS;             // [HQ][TE]    logits, then probabilities
  float* m_run = ps + HQ * TE;           // [HQ]
  float* l_run = m_run + HQ;             // [HQ]
  float* alpha = l_run + HQ;             // [HQ]
  __shared__ int32_t ent[32];            // per tile: entry row (>=0), window slot (-2 - slot), or -1 (skip)

  const int qi = blockIdx.y, split = blockIdx.x, tid = threadIdx.x;
  const int r = a.q_req ? a.q_req[qi] : qi;
  const bool live = r >= 0 && r < a.batch;   // a request outside the batch attends to nothing
  const int nv = static_cast<int>(min(max(static_cast<int64_t>(a.n_visible[qi]), int64_t(0)), a.cap));
  const int n_sel = a.idx ? a.topk : nv;
  const int64_t t = a.q_pos[qi];
  int64_t p_lo = t - a.window + 1;
  if (a.swa_lo && a.swa_lo[qi] > p_lo) p_lo = a.swa_lo[qi];
  if (p_lo < 0) p_lo = 0;
  const int n_win = (a.window > 0 && t >= p_lo) ? static_cast<int>(t - p_lo + 1) : 0;
  const int total = live ? n_sel + n_win : 0;
  const int x_begin = split * a.per_split;
  const int x_end = min(total, x_begin + a.per_split);

  // query rows, pre-scaled by tau
  const int qeb = elem_bytes(a.q_dtype);
  const char* qbase = static_cast<const char*>(a.q) + static_cast<int64_t>(qi) * HQ * D * qeb;
  for (int v = tid; v < HQ * D / 8; v += kAttnThreads) {
    const int h = v / (D / 8), col = (v % (D / 8)) * 8;
    float x[8];
    load8(qbase + static_cast<int64_t>(h) * D * qeb, a.q_dtype, col, nullptr, 1, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) qs[h * LDS + col + e] = x[e] * a.tau;
  }
  for (int h = tid; h < HQ; h += kAttnThreads) { m_run[h] = -INFINITY; l_run[h] = 0.f; }

  float4 acc[ACC4];
#pragma unroll
  for (int i = 0; i < ACC4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int hh = tid / TPH;          // head owned in the accumulate phase
  const int c4 = tid % TPH;          // first float4 column owned

  const int sweb = elem_bytes(a.swa_dtype);
  const int64_t kv_row0 = live ? static_cast<int64_t>(r) * a.cap : 0;
  const int64_t sw_row0 = live ? static_cast<int64_t>(r) * a.swa_cap : 0;

  for (int x0 = x_begin; x0 < x_end; x0 += TE) {
    __syncthreads();
    if (tid < TE) {
      const int x = x0 + tid;
      int32_t e = -1;
      if (x < x_end) {
        if (x < n_sel) {
          const int32_t j = a.idx ? a.idx[static_cast<int64_t>(qi) * a.topk + x] : x;
          e = (j >= 0 && j < nv) ? j : -1;
        } else {
          const int64_t pos = p_lo + (x - n_sel);
          e = -2 - static_cast<int32_t>(pos % a.swa_cap);
        }
      }
      ent[tid] = e;
    }
    __syncthreads();
    // gather key (and window value) rows into shared memory as fp32
    for (int v = tid; v < TE * (D / 8); v += kAttnThreads) {
      const int row = v / (D / 8), col = (v % (D / 8)) * 8;
      const int32_t e = ent[row];
      float x[8], y[8];
      if (e >= 0) {
        const int64_t gr = kv_row0 + e;
        // FP8: fp32 scales; MXFP4: E4M3 scale bytes
        const void* srow = a.kv_scale == nullptr ? nullptr
                           : a.kv_dtype == kMXFP4
                               ? static_cast<const void*>(static_cast<const uint8_t*>(a.kv_scale) + gr * (D / 16))
                               : static_cast<const void*>(static_cast<const float*>(a.kv_scale) + gr * (D / a.kv_group));
        load8_kv(static_cast<const char*>(a.kv) + row_bytes(a.kv_dtype, gr * D), a.kv_dtype, col, srow, a.kv_group,
                 x);
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = x[i];
      } else if (e <= -2) {
        const int64_t gr = sw_row0 + (-2 - e);
        load8(static_cast<const char*>(a.swa_k) + gr * D * sweb, a.swa_dtype, col, nullptr, 1, x);
        load8(static_cast<const char*>(a.swa_v) + gr * D * sweb, a.swa_dtype, col, nullptr, 1, y);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) { x[i] = 0.f; y[i] = 0.f; }
      }
#pragma unroll
      for (int i = 0; i < 8; i += 4) {
        *reinterpret_cast<float4*>(&ks[row * LDS + col + i]) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        *reinterpret_cast<float4*>(&vs[row * LDS + col + i]) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
      }
    }
    __syncthreads();
    // logits: thread owns RH heads x RE keys
    {
      const int eb = tid % (TE / RE), hb = tid / (TE / RE);
      float s[RH][RE];
#pragma unroll
      for (int i = 0; i < RH; ++i)
#pragma unroll
        for (int j = 0; j < RE; ++j) s[i][j] = 0.f;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        float4 qv[RH], kv4[RE];
#pragma unroll
        for (int i = 0; i < RH; ++i) qv[i] = *reinterpret_cast<const float4*>(&qs[(hb * RH + i) * LDS + c]);
#pragma unroll
        for (int j = 0; j < RE; ++j) kv4[j] = *reinterpret_cast<const float4*>(&ks[(eb + j * (TE / RE)) * LDS + c]);
#pragma unroll
        for (int i = 0; i < RH; ++i)
#pragma unroll
          for (int j = 0; j < RE; ++j) {
            s[i][j] = fmaf(qv[i].x, kv4[j].x, s[i][j]);
            s[i][j] = fmaf(qv[i].y, kv4[j].y, s[i][j]);
            s[i][j] = fmaf(qv[i].z, kv4[j].z, s[i][j]);
            s[i][j] = fmaf(qv[i].w, kv4[j].w, s[i][j]);
          }
      }
#pragma unroll
      for (int i = 0; i < RH; ++i)
#pragma unroll
        for (int j = 0; j < RE; ++j) {
          const int e = eb + j * (TE / RE);
          ps[(hb * RH + i) * TE + e] = (ent[e] == -1) ? -INFINITY : s[i][j];
        }
    }
    __syncthreads();
    // online-softmax update, one warp per head (lanes over keys)
    for (int h = tid >> 5; h < HQ; h += kAttnThreads / 32) {
      const int lane = tid & 31;
      const float v = lane < TE ? ps[h * TE + lane] : -INFINITY;
      const float mt = warp_max(v);
      const float m_old = m_run[h];
      const float m_new = fmaxf(m_old, mt);
      const float pr = (m_new == -INFINITY) ? 0.f : __expf(v - m_new);
      const float st = warp_sum(pr);
      if (lane < TE) ps[h * TE + lane] = pr;
      if (lane == 0) {
        const float al = (m_old == -INFINITY) ? 0.f : __expf(m_old - m_new);
        alpha[h] = al;
        l_run[h] = l_run[h] * al + st;
        m_run[h] = m_new;
      }
    }
    __syncthreads();
    // accumulate: thread owns head hh, float4 columns c4 + TPH*i
    {
      const float al = alpha[hh];
#pragma unroll
      for (int i = 0; i < ACC4; ++i) {
        acc[i].x *= al; acc[i].y *= al; acc[i].z *= al; acc[i].w *= al;
      }
      for (int e = 0; e < TE; ++e) {
        const float pr = ps[hh * TE + e];
        if (pr == 0.f) continue;
        const float* vrow = (ent[e] <= -2 ? vs : ks) + e * LDS;
#pragma unroll
        for (int i = 0; i < ACC4; ++i) {
          const float4 v = *reinterpret_cast<const float4*>(&vrow[(c4 + TPH * i) * 4]);
          acc[i].x = fmaf(pr, v.x, acc[i].x);
          acc[i].y = fmaf(pr, v.y, acc[i].y);
          acc[i].z = fmaf(pr, v.z, acc[i].z);
          acc[i].w = fmaf(pr, v.w, acc[i].w);
        }
      }
    }
  }
  __syncthreads();

  if (a.n_splits == 1) {
    // finish: add the sink to the denominator, normalise, write out and lse
    const float m = m_run[hh], l = l_run[hh];
    const float sk = a.sink ? a.sink[hh] : -INFINITY;
    const float M = fmaxf(m, sk);
    float scale_acc = 0.f, L = 0.f;
    if (M != -INFINITY) {
      const float am = (m == -INFINITY) ? 0.f : __expf(m - M);
      L = l * am + ((sk == -INFINITY) ? 0.f : __expf(sk - M));
      scale_acc = am / L;
    }
    const int oeb = elem_bytes(a.out_dtype);
    char* orow = static_cast<char*>(a.out) + (static_cast<int64_t>(qi) * HQ + hh) * D * oeb;
#pragma unroll
    for (int i = 0; i < ACC4; ++i) {
      const int col = (c4 + TPH * i) * 4;
      const float v0 = acc[i].x * scale_acc, v1 = acc[i].y * scale_acc, v2 = acc[i].z * scale_acc,
                  v3 = acc[i].w * scale_acc;
      if (a.out_dtype == kF32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(orow) + col) = make_float4(v0, v1, v2, v3);
      } else {
        uint2 u;
        u.x = f32_to_bf16_bits(v0) | (static_cast<uint32_t>(f32_to_bf16_bits(v1)) << 16);
        u.y = f32_to_bf16_bits(v2) | (static_cast<uint32_t>(f32_to_bf16_bits(v3)) << 16);
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(orow) + col) = u;
      }
    }
    if (a.lse && c4 == 0) a.lse[static_cast<int64_t>(qi) * HQ + hh] = (M == -INFINITY) ? -INFINITY : M + __logf(L);
    return;
  }
  float* pp = a.part + ((static_cast<int64_t>(qi) * a.n_splits + split) * HQ + hh) * (D + 2);
  if (c4 == 0) { pp[0] = m_run[hh]; pp[1] = l_run[hh]; }
#pragma unroll
  for (int i = 0; i < ACC4; ++i) {
    const int col = (c4 + TPH * i) * 4;
    pp[2 + col + 0] = acc[i].x; pp[2 + col + 1] = acc[i].y;
    pp[2 + col + 2] = acc[i].z; pp[2 + col + 3] = acc[i].w;
  }
}

// Combines the per-split partial states of one (query, head): one CTA each.
constexpr int kMaxSplits = 256;
__global__ void __launch_bounds__(128)
attn_merge_kernel(const float* __restrict__ part, int n_splits, int hq, int d, const float* __restrict__ sink,
                  void* out, int out_dtype, float* lse) {
  __shared__ float wgt[kMaxSplits];
  __shared__ float s_ml[2];
  const int qi = blockIdx.x / hq, h = blockIdx.x % hq;
  const float* base = part + (static_cast<int64_t>(qi) * n_splits * hq + h) * (d + 2);
  const int64_t sstride = static_cast<int64_t>(hq) * (d + 2);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const float sk = sink ? sink[h] : -INFINITY;
    float M = sk;
    for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, __ldg(base + s * sstride));
    M = warp_max(M);
    float L = 0.f;
    if (M != -INFINITY) {
      for (int s = lane; s < n_splits; s += 32) {
        const float ms = __ldg(base + s * sstride);
        const float wv = (ms == -INFINITY) ? 0.f : __expf(ms - M);
        wgt[s] = wv;
        L += wv * __ldg(base + s * sstride + 1);
      }
      L = warp_sum(L);
      if (sk != -INFINITY) L += __expf(sk - M);
    }
    if (lane == 0) { s_ml[0] = M; s_ml[1] = L; }
  }
  __syncthreads();
  const float M = s_ml[0], L = s_ml[1];
  const int oeb = elem_bytes(out_dtype);
  char* orow = static_cast<char*>(out) + (static_cast<int64_t>(qi) * hq + h) * d * oeb;
  const float inv = (M != -INFINITY) ? 1.f / L : 0.f;
  // columns c, c+128, ... of this thread; the split states are read in
  // batches of 8 splits, all loads of a batch issued before use
  for (int c0 = threadIdx.x; c0 < d; c0 += 128 * 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
      for (int s0 = 0; s0 < n_splits; s0 += 8) {
        float v[8][4];
#pragma unroll
        for (int b = 0; b < 8; ++b)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int s = s0 + b, c = c0 + q * 128;
            v[b][q] = (s < n_splits && c < d) ? __ldg(base + s * sstride + 2 + c) : 0.f;
          }
#pragma unroll
        for (int b = 0; b < 8; ++b)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (s0 + b < n_splits) acc[q] = fmaf(wgt[s0 + b], v[b][q], acc[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * 128;
      if (c >= d) continue;
      const float o = acc[q] * inv;
      if (out_dtype == kF32) reinterpret_cast<float*>(orow)[c] = o;
      else reinterpret_cast<uint16_t*>(orow)[c] = f32_to_bf16_bits(o);
    }
  }
  if (lse && threadIdx.x == 0) lse[static_cast<int64_t>(qi) * hq + h] = (M == -INFINITY) ? -INFINITY : M + __logf(L);
}

template <int HQ, int D>
csa_status_t launch_attn_t(AttnArgs a, int nq, cudaStream_t stream) {
  using Cfg = AttnCfg<HQ, D>;
  const size_t smem = Cfg::smem_floats * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<HQ, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  dim3 grid(a.n_splits, nq);
  prof_begin(stream);
  attn_simt_kernel<HQ, D><<<grid, kAttnThreads, smem, stream>>>(a);
  csa_status_t st = check_launch("attn_simt_kernel", stream);
  if (st != CSA_OK || a.n_splits == 1) return st;
  prof_begin(stream);
  attn_merge_kernel<<<nq * HQ, 128, 0, stream>>>(a.part, a.n_splits, HQ, D, a.sink, a.out, a.out_dtype, a.lse);
  return check_launch("attn_merge_kernel", stream);
}

}  // namespace

csa_status_t launch_attn_merge(const float* part, int nq, int n_splits, int hq, int d, const float* sink, void* out,
                               int out_dtype, float* lse, cudaStream_t stream) {
  if (n_splits > kMaxSplits) return set_error(CSA_ERR_UNSUPPORTED, "%d attention splits (max %d)", n_splits, kMaxSplits);
  prof_begin(stream);
  attn_merge_kernel<<<nq * hq, 128, 0, stream>>>(part, n_splits, hq, d, sink, out, out_dtype, lse);
  return check_launch("attn_merge_kernel", stream);
}

// Splits per query: enough CTAs to cover the GPU twice for small query
// counts; one split (no merge pass) once the queries alone fill it.
int attn_splits(int nq, int max_keys) {
  const int target = 2 * 148;
  int s = (target + nq - 1) / nq;
  const int max_s = (max_keys + 63) / 64;  // a partial state costs as much as ~128 bf16 rows
  if (s > max_s) s = max_s;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < 1) s = 1;
  return s;
}

bool attn_tc_supported(const csa_params_t* p, int q_dtype, int kv_dtype, int swa_dtype, bool has_window);
size_t attn_tc_workspace_bytes(int nq, int max_keys);
int attn_tc_splits(int max_keys);
int attn_cluster_min(int sel_max, int window);
csa_status_t launch_attention_tc(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                                 int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible,
                                 const int32_t* q_req, const csa_tensor_t* swa_k, const csa_tensor_t* swa_v,
                                 const int64_t* q_pos, const int64_t* swa_lo, const float* sink,
                                 const csa_tensor_t* out, float* lse, void* workspace, int max_keys,
                                 cudaStream_t stream, bool pdl);

csa_status_t launch_attention_many_tc(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                                      int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible,
                                      const int32_t* q_req, const csa_tensor_t* swa_k, const csa_tensor_t* swa_v,
                                      const int64_t* q_pos, const int64_t* swa_lo, const float* sink,
                                      const csa_tensor_t* out, float* lse, cudaStream_t stream);

// Tensor-core attention (64 heads of 512): few queries (decode) are each
// cut over the CTAs of a cluster, or into 128-key splits merged by a second
// kernel; many queries (prefill) take one CTA each that loops over the
// query's keys (no workspace).
constexpr int kManyQueries = 64;
static bool attn_tc_shape(int nq, int hq, int d, int max_keys, int window) {
  (void)window;
  if (hq != 64 || d != 512) return false;
  return nq > kManyQueries || attn_tc_splits(max_keys) <= kMaxSplits;
}

size_t attn_workspace_bytes(int nq, int hq, int d, int max_keys, int window) {
  const int s = attn_splits(nq, max_keys);
  size_t b = s <= 1 ? 0 : static_cast<size_t>(nq) * s * hq * (d + 2) * sizeof(float);
  if (attn_tc_shape(nq, hq, d, max_keys, window) && nq <= kManyQueries) {
    const size_t t = attn_tc_workspace_bytes(nq, max_keys);
    if (t > b) b = t;
  }
  return b;
}

csa_status_t launch_attention(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                              int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible, const int32_t* q_req,
                              const csa_tensor_t* swa_k, const csa_tensor_t* swa_v, const int64_t* q_pos,
                              const int64_t* swa_lo, const float* sink, const csa_tensor_t* out, float* lse,
                              void* workspace, int max_keys, cudaStream_t stream, bool pdl) {
  if (nq == 0) return CSA_OK;
  if (attn_tc_shape(nq, p->h_q, p->d, max_keys, p->window) &&
      attn_tc_supported(p, q->dtype, kv->dtype, swa_k ? swa_k->dtype : kBF16, p->window > 0)) {
    if (nq > kManyQueries)
      return launch_attention_many_tc(p, nq, q, kv, batch, cap, idx, n_visible, q_req, swa_k, swa_v, q_pos, swa_lo,
                                      sink, out, lse, stream);
    return launch_attention_tc(p, nq, q, kv, batch, cap, idx, n_visible, q_req, swa_k, swa_v, q_pos, swa_lo, sink,
                               out, lse, workspace, max_keys, stream, pdl);
  }
  AttnArgs a;
  a.q = q->data; a.q_dtype = q->dtype;
  a.kv = kv->data; a.kv_scale = kv->scale; a.kv_dtype = kv->dtype;
  a.kv_group = (kv->dtype == kFP8 || kv->dtype == kMXFP4) ? kv->scale_group : 1; a.batch = batch; a.cap = cap;
  a.idx = idx; a.topk = p->topk;
  a.n_visible = n_visible; a.q_req = q_req;
  a.swa_k = swa_k ? swa_k->data : nullptr; a.swa_v = swa_v ? swa_v->data : nullptr;
  a.swa_dtype = swa_k ? swa_k->dtype : kF32; a.swa_cap = p->swa_cap > 0 ? p->swa_cap : 1; a.window = p->window;
  a.q_pos = q_pos; a.swa_lo = swa_lo; a.sink = sink; a.tau = p->softmax_scale;
  a.out = out->data; a.out_dtype = out->dtype; a.lse = lse;
  a.part = static_cast<float*>(workspace);
  a.n_splits = attn_splits(nq, max_keys);
  const int per = (max_keys + a.n_splits - 1) / a.n_splits;
  a.per_split = per < 1 ? 1 : per;
#define CSA_ATTN_CASE(HQ, D) \
  if (p->h_q == HQ && p->d == D) return launch_attn_t<HQ, D>(a, nq, stream);
  CSA_ATTN_CASE(8, 128)
  CSA_ATTN_CASE(16, 128)
  CSA_ATTN_CASE(64, 128)
  CSA_ATTN_CASE(64, 512)
#undef CSA_ATTN_CASE
  return set_error(CSA_ERR_UNSUPPORTED, "attention shape h_q=%d d=%d is not built", p->h_q, p->d);
}

}  // namespace csa
