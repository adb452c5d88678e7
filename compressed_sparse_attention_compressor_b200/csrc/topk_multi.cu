// Top-k of long score rows with several CTAs per row (a cooperative launch):
// each CTA holds a contiguous segment of its row in shared memory, the CTAs
// of a row agree on the k-th largest key through histograms merged in global
// memory (a radix select over the keys' own range), then write their entries
// -- optionally in ascending index order -- at offsets from an exchange of
// per-CTA counts.  Same result as topk_row_kernel (score descending, lower
// index first among exactly equal scores, -0 == +0), for rows too long for
// one CTA to go through quickly (the candidate pool's block maxima:
// 131,072 per query at one million tokens).  Tech-report tour, "The
// Hierarchical Sparse Indexer" (2,048 blocks of 8 positions form the pool)
// and "The indexer selects, SWA covers the rest" (the top-k selection).
#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

constexpr int kMT = 512;           // threads per CTA
constexpr int kMW = kMT / 32;
constexpr int kMBins = 2048;
constexpr int kMLevels = 3;        // a 32-bit key range takes at most three 11-bit levels
constexpr int kMSeg = 8192;        // scores of one CTA (32 KB of shared memory)
constexpr int kMMaxG = 148;
constexpr uint32_t kMSpin = 1u << 22;  // barrier polls (~64 ns apart)

__device__ uint32_t g_topk_multi_error = 0;  // bit 0: a bounded barrier wait gave up

struct MultiArgs {
  const float* scores;
  int64_t ld;
  const int32_t* n_valid;  // valid columns ceil(n_valid / nv_div), or max_n when null
  int nv_div;
  int64_t max_n;
  int k;
  int32_t* out_idx;
  float* out_score;
  int ordered;
  int G;                   // CTAs per row
  uint32_t* ctl;           // per row ctl_words words, zero on entry
};

// per-row control words
constexpr int kCMin = 0;   // max of ~key (so that zero is the identity)
constexpr int kCMax = 1;
constexpr int kCBar = 2;
constexpr int kCHist = 4;  // [kMLevels][kMBins]
constexpr int kCCnt = kCHist + kMLevels * kMBins;  // [G][2] entries above / at the k-th key per CTA
constexpr int kCtlWords = kCCnt + 2 * kMMaxG;

// All threads: one arrival of this CTA at the row's barrier, then a bounded
// wait for `target` arrivals; false on a timeout.
__device__ bool row_barrier(uint32_t* ctr, uint32_t target, int* flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    int ok = 1;
    uint32_t it = 0;
    while (sm100::ld_acquire_gpu(ctr) < target) {
      if (++it > kMSpin) {
        atomicOr(&g_topk_multi_error, 1u);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    *flag = ok;
  }
  __syncthreads();
  return *flag != 0;
}

// Warp 0: the bin b of hist[0..kMBins) (from the top) with
// above(b) < need <= above(b) + hist[b]; bc[0] = b, bc[1] = above(b).
__device__ void find_bin_warp(const uint32_t* hist, uint32_t need, uint32_t* bc) {
  const int lane = threadIdx.x & 31;
  constexpr int per = kMBins / 32;
  const int lo = lane * per;
  uint32_t mine = 0;
  for (int i = 0; i < per; ++i) mine += hist[lo + i];
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += v;
  }
  const uint32_t excl = incl - mine;
  if (excl < need && need <= incl) {
    uint32_t above = excl;
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t c = hist[lo + i];
      if (above + c >= need) {
        bc[0] = lo + i;
        bc[1] = above;
        break;
      }
      above += c;
    }
  }
}

__global__ void __launch_bounds__(kMT) topk_multi_kernel(MultiArgs a) {
  __shared__ __align__(16) float sv[kMSeg];
  __shared__ uint32_t hist[kMBins];
  __shared__ uint32_t wr[2 * kMW];
  __shared__ uint32_t bc[2];
  __shared__ int flag;
  const int row = blockIdx.x / a.G, g = blockIdx.x % a.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nv = a.n_valid ? (static_cast<int64_t>(a.n_valid[row]) + a.nv_div - 1) / a.nv_div : a.max_n;
  const int64_t n = min(max(nv, int64_t(0)), a.max_n);
  const float* s = a.scores + static_cast<int64_t>(row) * a.ld;
  const int k = a.k;
  int32_t* oi = a.out_idx + static_cast<int64_t>(row) * k;
  float* os = a.out_score ? a.out_score + static_cast<int64_t>(row) * k : nullptr;
  uint32_t* ctl = a.ctl + static_cast<int64_t>(row) * kCtlWords;

  if (n <= k) {  // every entry, in index order; the row's CTAs share [0, k)
    for (int64_t j = static_cast<int64_t>(g) * kMT + tid; j < k; j += static_cast<int64_t>(a.G) * kMT) {
      oi[j] = j < n ? static_cast<int32_t>(j) : -1;
      if (os) os[j] = j < n ? s[j] : -INFINITY;
    }
    return;
  }

  // this CTA's contiguous segment (the host keeps it within kMSeg)
  const int64_t seg = (n + a.G - 1) / a.G;
  const int64_t b0 = min(n, static_cast<int64_t>(g) * seg), b1 = min(n, b0 + seg);
  const int len = static_cast<int>(b1 - b0);
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int i = tid; i < len; i += kMT) {
    const float v = __ldg(s + b0 + i);
    sv[i] = v;
    const uint32_t key = score_key(v);
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  }
  kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
  kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
  if (lane == 0 && len > 0) {
    atomicMax(&ctl[kCMin], ~kmin);
    atomicMax(&ctl[kCMax], kmax);
  }
  uint32_t nbar = 1;
  if (!row_barrier(&ctl[kCBar], nbar * a.G, &flag)) return;
  uint32_t lo = ~__ldcg(&ctl[kCMin]);
  const uint32_t hi = __ldcg(&ctl[kCMax]);

  // radix select over [lo, lo + span): levels of <= 2048 bins of 2^shift keys
  uint64_t span = static_cast<uint64_t>(hi - lo) + 1;
  uint32_t need = static_cast<uint32_t>(k);
  int shift = max(0, 64 - __clzll(static_cast<long long>(span - 1)) - 11);
  for (int level = 0;; ++level) {
    for (int i = tid; i < kMBins; i += kMT) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < len; i += kMT) {
      const uint32_t d = score_key(sv[i]) - lo;
      if (static_cast<uint64_t>(d) < span) atomicAdd(&hist[d >> shift], 1u);
    }
    __syncthreads();
    uint32_t* gh = ctl + kCHist + level * kMBins;
    for (int i = tid; i < kMBins; i += kMT)
      if (hist[i]) atomicAdd(&gh[i], hist[i]);
    ++nbar;
    if (!row_barrier(&ctl[kCBar], nbar * a.G, &flag)) return;
    for (int i = tid; i < kMBins; i += kMT) hist[i] = __ldcg(&gh[i]);
    if (tid == 0) {
      bc[0] = 0;
      bc[1] = 0;
    }
    __syncthreads();
    if (warp == 0) find_bin_warp(hist, need, bc);
    __syncthreads();
    const uint32_t b = bc[0];
    need -= bc[1];
    lo += b << shift;
    span = min(span - (static_cast<uint64_t>(b) << shift), static_cast<uint64_t>(1) << shift);
    if (shift == 0) break;
    shift = max(0, shift - 11);
  }
  const uint32_t T = lo;           // exact key of the k-th largest score
  const uint32_t take_eq = need;   // entries equal to T that are kept
  const uint32_t n_gt = static_cast<uint32_t>(k) - take_eq;

  // this CTA's counts above / at T, exchanged for the output offsets
  uint32_t cg = 0, ce = 0;
  for (int i = tid; i < len; i += kMT) {
    const uint32_t key = score_key(sv[i]);
    cg += key > T;
    ce += key == T;
  }
  cg = __reduce_add_sync(0xFFFFFFFFu, cg);
  ce = __reduce_add_sync(0xFFFFFFFFu, ce);
  if (lane == 0) {
    wr[warp] = cg;
    wr[kMW + warp] = ce;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t tg = 0, te = 0;
    for (int w = 0; w < kMW; ++w) {
      tg += wr[w];
      te += wr[kMW + w];
    }
    reinterpret_cast<uint2*>(ctl + kCCnt)[g] = make_uint2(tg, te);
  }
  ++nbar;
  if (!row_barrier(&ctl[kCBar], nbar * a.G, &flag)) return;
  uint32_t og = 0, oe = 0;  // above / at T in the row's earlier CTAs
  for (int c = 0; c < g; ++c) {
    const uint2 ce2 = __ldcg(reinterpret_cast<const uint2*>(ctl + kCCnt) + c);
    og += ce2.x;
    oe += ce2.y;
  }
  // warp-contiguous sub-segments walked 32 entries at a time: ballots rank
  // the entries inside a warp, a scan of the per-warp counts places the warps
  const int wseg = (((len + kMW - 1) / kMW) + 31) & ~31;
  const int w0 = min(len, warp * wseg), w1 = min(len, w0 + wseg);
  uint32_t mg = 0, me = 0;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < w1 ? score_key(sv[i]) : 0u;
    mg += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && key > T));
    me += __popc(__ballot_sync(0xFFFFFFFFu, i < w1 && key == T));
  }
  __syncthreads();  // wr reused
  if (lane == 0) {
    wr[warp] = mg;
    wr[kMW + warp] = me;
  }
  __syncthreads();
  for (int w = 0; w < warp; ++w) {
    og += wr[w];
    oe += wr[kMW + w];
  }
  const uint32_t lm = (1u << lane) - 1u;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    float v = 0.f;
    uint32_t key = 0u;
    if (i < w1) {
      v = sv[i];
      key = score_key(v);
    }
    const bool gt = i < w1 && key > T, eq = i < w1 && key == T;
    const uint32_t bgt = __ballot_sync(0xFFFFFFFFu, gt), beq = __ballot_sync(0xFFFFFFFFu, eq);
    const uint32_t rg = og + __popc(bgt & lm), re = oe + __popc(beq & lm);  // before entry i
    const int32_t j = static_cast<int32_t>(b0 + i);
    if (gt) {
      const uint32_t p = a.ordered ? rg + min(re, take_eq) : rg;
      oi[p] = j;
      if (os) os[p] = v;
    } else if (eq && re < take_eq) {
      const uint32_t p = a.ordered ? rg + re : n_gt + re;
      oi[p] = j;
      if (os) os[p] = v;
    }
    og += __popc(bgt);
    oe += __popc(beq);
  }
}

}  // namespace

// CTAs per row for rows of up to max_n scores (0: use the one-CTA kernel):
// about 4,096 scores per CTA, at least enough CTAs that a segment fits in
// shared memory, and every row's CTAs co-resident (one per SM at most).
int topk_multi_ctas(int n_rows, int64_t max_n) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  // rows of up to 65,536 scores: one CTA per row (its candidate form) is faster
  if (n_rows < 1 || max_n <= 65536) return 0;
  const int64_t need = (max_n + kMSeg - 1) / kMSeg;
  int64_t G = (max_n + 4095) / 4096;
  if (G < need) G = need;
  const int64_t cap = min(static_cast<int64_t>(kMMaxG), static_cast<int64_t>(sms / n_rows));
  if (G > cap) G = cap;
  return G >= need && G >= 2 ? static_cast<int>(G) : 0;
}

size_t topk_multi_ctl_bytes(int n_rows) { return static_cast<size_t>(n_rows) * kCtlWords * 4; }

// ctl: topk_multi_ctl_bytes(n_rows) bytes; zeroed here.
csa_status_t launch_topk_multi(const float* scores, int n_rows, int64_t ld, const int32_t* n_valid, int nv_div,
                               int64_t max_n, int k, int32_t* out_idx, float* out_score, int ordered, int G,
                               void* ctl, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(ctl, 0, topk_multi_ctl_bytes(n_rows), stream);
  if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  MultiArgs a;
  a.scores = scores;
  a.ld = ld;
  a.n_valid = n_valid;
  a.nv_div = nv_div;
  a.max_n = max_n;
  a.k = k;
  a.out_idx = out_idx;
  a.out_score = out_score;
  a.ordered = ordered;
  a.G = G;
  a.ctl = static_cast<uint32_t*>(ctl);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_rows * G);
  cfg.blockDim = dim3(kMT);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(stream);
  e = cudaLaunchKernelEx(&cfg, topk_multi_kernel, a);
  if (e != cudaSuccess) {
    check_launch("topk_multi_kernel", stream);
    return set_error(CSA_ERR_CUDA, "topk_multi_kernel launch: %s", cudaGetErrorString(e));
  }
  return check_launch("topk_multi_kernel", stream);
}

uint32_t topk_multi_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_topk_multi_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_topk_multi_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
