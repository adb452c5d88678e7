// K2 -- lightning-indexer scores, and K3 -- exact per-query top-k.
//
// Atlas "Model architectures", "Trained sparse attention" entry (DSA: a
// lightning indexer followed by fine-grained top-k selection) and
// "compressed KV" entry (top-k over compressed entries); tech-report tour,
// "The indexer selects, SWA covers the rest" (the indexer scores main-KV
// entries with indexer query and indexer key and keeps the top entries of
// every query).
//
//   s_j = sum_h w_h * max(0, q_h . k_j)       (FP8 keys: k_j = codes * scale_j)
//
// Top-k order: score descending; among exactly equal scores the lower index
// wins (-0 == +0).  The selection is a radix select on the ordered 32-bit
// key of each fp32 score (histogram levels of up to 2,048 bins over the
// keys' own range), which yields the exact k-th key T and the number r of
// entries equal to T that are kept; an index-ordered pass then takes every
// entry above T and the r lowest-index entries equal to T.  The row kernel
// first keeps, in shared memory, the candidates that reach a threshold
// taken from a sample of the row and runs the levels over them; a row whose
// candidates do not fit (or fall short of k) takes them over the whole row.
#include "common.cuh"

namespace csa {

namespace {

// ---------------------------------------------------------------------------
// K2, CUDA-core form: one thread per key, all heads accumulated in registers.
// ---------------------------------------------------------------------------
constexpr int kScoreThreads = 256;

// pool != nullptr (re-indexing inside a candidate pool): score j of query
// qi is that of entry pool[qi][j / block] * block + j % block for j <
// pool_blocks * block, -inf where the pool slot is -1 or the entry is not
// visible.
template <int H, int DI>
__global__ void __launch_bounds__(kScoreThreads)
index_score_simt_kernel(const void* __restrict__ q_idx, int q_dtype, const float* __restrict__ w,
                        const void* __restrict__ keys, const float* __restrict__ kscale, int k_dtype,
                        int batch, int64_t cap, const int32_t* __restrict__ q_req,
                        const int32_t* __restrict__ n_visible, float* __restrict__ scores, int64_t ld,
                        const int32_t* __restrict__ pool, int block, int pool_blocks) {
  __shared__ __align__(16) float qs[H * DI];
  __shared__ float ws[H];
  const int qi = blockIdx.y;
  const int r = q_req ? q_req[qi] : qi;
  const int64_t nvis = (r < 0 || r >= batch) ? 0 : min(max(static_cast<int64_t>(n_visible[qi]), int64_t(0)), cap);
  const int64_t n = pool ? static_cast<int64_t>(pool_blocks) * block : nvis;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kScoreThreads;
  if (j0 >= n) return;  // uniform over the CTA
  const char* qrow = static_cast<const char*>(q_idx) + static_cast<int64_t>(qi) * H * DI * elem_bytes(q_dtype);
  for (int i = threadIdx.x; i < H * DI; i += kScoreThreads) qs[i] = load1(qrow, q_dtype, i, nullptr, 1);
  for (int i = threadIdx.x; i < H; i += kScoreThreads) ws[i] = w[static_cast<int64_t>(qi) * H + i];
  __syncthreads();
  const int64_t j = j0 + threadIdx.x;
  if (j >= n) return;
  int64_t e = j;  // the entry scored
  if (pool) {
    const int32_t b = pool[static_cast<int64_t>(qi) * pool_blocks + j / block];
    e = b < 0 ? -1 : static_cast<int64_t>(b) * block + j % block;
    if (e < 0 || e >= nvis) {
      scores[static_cast<int64_t>(qi) * ld + j] = -INFINITY;
      return;
    }
  }
  const int64_t krow = static_cast<int64_t>(r) * cap + e;
  const char* kp = static_cast<const char*>(keys) + krow * DI * elem_bytes(k_dtype);
  const float* sp = (k_dtype == kFP8) ? kscale + krow : nullptr;
  float acc[H];
#pragma unroll
  for (int h = 0; h < H; ++h) acc[h] = 0.f;
#pragma unroll 1
  for (int c0 = 0; c0 < DI; c0 += 8) {
    float k[8];
    if (k_dtype == kFP8) {
      // the row scale multiplies the whole score (ReLU(s*x) = s*ReLU(x), s > 0)
      uint2 u = __ldg(reinterpret_cast<const uint2*>(kp + c0));
      float2 a = e4m3x2_to_f32x2(static_cast<uint16_t>(u.x & 0xFFFF));
      float2 b = e4m3x2_to_f32x2(static_cast<uint16_t>(u.x >> 16));
      float2 c = e4m3x2_to_f32x2(static_cast<uint16_t>(u.y & 0xFFFF));
      float2 d = e4m3x2_to_f32x2(static_cast<uint16_t>(u.y >> 16));
      k[0] = a.x; k[1] = a.y; k[2] = b.x; k[3] = b.y; k[4] = c.x; k[5] = c.y; k[6] = d.x; k[7] = d.y;
    } else {
      load8(kp, k_dtype, c0, nullptr, 1, k);
    }
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float4 qa = *reinterpret_cast<const float4*>(&qs[h * DI + c0]);
      const float4 qb = *reinterpret_cast<const float4*>(&qs[h * DI + c0 + 4]);
      float a = acc[h];
      a = fmaf(qa.x, k[0], a); a = fmaf(qa.y, k[1], a); a = fmaf(qa.z, k[2], a); a = fmaf(qa.w, k[3], a);
      a = fmaf(qb.x, k[4], a); a = fmaf(qb.y, k[5], a); a = fmaf(qb.z, k[6], a); a = fmaf(qb.w, k[7], a);
      acc[h] = a;
    }
  }
  float s = 0.f;
#pragma unroll
  for (int h = 0; h < H; ++h) s = fmaf(ws[h], fmaxf(acc[h], 0.f), s);
  if (sp) s *= __ldg(sp);
  scores[static_cast<int64_t>(qi) * ld + j] = s;
}

// ---------------------------------------------------------------------------
// K3: one CTA per row.
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kU = 4;  // 16-byte loads in flight per thread

struct TopkShared {
  uint32_t hist[2048];
  uint32_t warp_gt[kTopkWarps];
  uint32_t warp_eq[kTopkWarps];
  uint32_t wsum[kTopkWarps];
  uint32_t sel_bin;
  uint32_t above;
};

// All threads (two bins each): the bin b of hist[0..2048), scanned from the
// top, with above(b) < need <= above(b) + hist[b], where above(b) counts the
// entries of the bins over b; writes (b, above(b)) to sel_bin / above, read
// after the caller's next barrier.  Needs 1 <= need <= the histogram total.
__device__ void find_bin_all(TopkShared& sh, uint32_t need) {
  static_assert(2 * kTopkThreads == 2048, "two bins per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint2 c = *reinterpret_cast<const uint2*>(sh.hist + 2 * tid);  // bins 2 tid, 2 tid + 1
  const uint32_t v = c.x + c.y;
  uint32_t incl = v;  // this lane's bins and those of the lanes above it
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += x;
  }
  if (lane == 0) sh.wsum[warp] = incl;
  __syncthreads();
  const uint32_t ws = sh.wsum[lane];  // lane l: the total of warp l
  uint32_t wi = ws;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_down_sync(0xFFFFFFFFu, wi, o);
    if (lane + o < 32) wi += x;
  }
  const uint32_t above = __shfl_sync(0xFFFFFFFFu, wi - ws, warp) + incl - v;  // entries over bin 2 tid + 1
  if (above < need && need <= above + c.y) {
    sh.sel_bin = 2 * tid + 1;
    sh.above = above;
  } else if (above + c.y < need && need <= above + v) {
    sh.sel_bin = 2 * tid;
    sh.above = above + c.y;
  }
}

// Four consecutive scores of a row (zero past n), as one 16-byte load when
// the row start allows it: each thread keeps several loads in flight.
struct Row4 {
  const float* s;
  int64_t n;
  bool vec;
  __device__ __forceinline__ void load(int64_t j, float (&v)[4]) const {  // j % 4 == 0
    if (vec && j + 3 < n) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(s + j));
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[c] = j + c < n ? __ldg(s + j + c) : 0.f;
    }
  }
};

// The whole row (any distribution): a min / max pass, then the radix select
// of the k-th key over the keys' own range, then the index-ordered pass.
__device__ void topk_row_full(TopkShared& sh, const float* s, int64_t n, int k, int32_t* oi, float* os,
                              int ordered) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Row4 rs4{s, n, (reinterpret_cast<uintptr_t>(s) & 15) == 0};
  // radix select of the k-th largest key over the keys' own range: the
  // range [lo, lo + span) is cut into <= 2048 bins of 2^shift keys and
  // narrowed to the bin holding the k-th key until a bin is one key wide.
  // Bins that follow the data keep shared-memory atomics on distinct words.
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int64_t j0 = 0; j0 < n; j0 += kU * 4 * kTopkThreads) {
    float v[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) rs4.load(j0 + 4 * (u * kTopkThreads + tid), v[u]);
#pragma unroll
    for (int u = 0; u < kU; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (j0 + 4 * (u * kTopkThreads + tid) + c < n) {
          const uint32_t key = score_key(v[u][c]);
          kmin = min(kmin, key);
          kmax = max(kmax, key);
        }
  }
  kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
  kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
  if (lane == 0) { sh.warp_gt[warp] = kmin; sh.warp_eq[warp] = kmax; }
  __syncthreads();
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int w2 = 0; w2 < kTopkWarps; ++w2) { lo = min(lo, sh.warp_gt[w2]); hi = max(hi, sh.warp_eq[w2]); }
  __syncthreads();
  uint64_t span = static_cast<uint64_t>(hi - lo) + 1;
  uint32_t need = static_cast<uint32_t>(k);
  int shift = max(0, 64 - __clzll(static_cast<long long>(span - 1)) - 11);
  for (;;) {
    for (int i = tid; i < 2048; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    for (int64_t j0 = 0; j0 < n; j0 += kU * 4 * kTopkThreads) {
      float v[kU][4];
#pragma unroll
      for (int u = 0; u < kU; ++u) rs4.load(j0 + 4 * (u * kTopkThreads + tid), v[u]);
#pragma unroll
      for (int u = 0; u < kU; ++u)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t d = score_key(v[u][c]) - lo;
          if (j0 + 4 * (u * kTopkThreads + tid) + c < n && static_cast<uint64_t>(d) < span)
            atomicAdd(&sh.hist[d >> shift], 1u);
        }
    }
    __syncthreads();
    find_bin_all(sh, need);
    __syncthreads();
    const uint32_t b = sh.sel_bin;
    need -= sh.above;
    lo += b << shift;
    span = min(span - (static_cast<uint64_t>(b) << shift), static_cast<uint64_t>(1) << shift);
    __syncthreads();
    if (shift == 0) break;
    shift = max(0, shift - 11);
  }
  const uint32_t prefix = lo;
  const uint32_t T = prefix;        // exact key of the k-th largest score
  const uint32_t take_eq = need;    // entries equal to T that are kept
  const uint32_t n_gt = static_cast<uint32_t>(k) - take_eq;

  // selection: every warp owns a contiguous segment that it walks 128
  // entries (four per lane) at a time; a scan over the lanes ranks the
  // entries inside the warp and one scan of the per-warp counts gives every
  // entry its output slot
  const int64_t segw = ((n + kTopkWarps - 1) / kTopkWarps + 127) & ~int64_t(127);
  const int64_t a0 = min(n, warp * segw), a1 = min(n, a0 + segw);
  uint32_t cg = 0, ce = 0;
  for (int64_t j1 = a0; j1 < a1; j1 += kU * 128) {
    float v[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) rs4.load(j1 + u * 128 + 4 * lane, v[u]);
#pragma unroll
    for (int u = 0; u < kU; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool ok = j1 + u * 128 + 4 * lane + c < a1;
        const uint32_t key = score_key(v[u][c]);
        cg += ok && key > T;
        ce += ok && key == T;
      }
  }
  cg = __reduce_add_sync(0xFFFFFFFFu, cg);
  ce = __reduce_add_sync(0xFFFFFFFFu, ce);
  if (lane == 0) { sh.warp_gt[warp] = cg; sh.warp_eq[warp] = ce; }
  __syncthreads();
  uint32_t og = 0, oe = 0;  // entries above / at T before the current step
  for (int w2 = 0; w2 < warp; ++w2) { og += sh.warp_gt[w2]; oe += sh.warp_eq[w2]; }
  for (int64_t j1 = a0; j1 < a1; j1 += kU * 128) {
    float vv[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) rs4.load(j1 + u * 128 + 4 * lane, vv[u]);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t j0 = j1 + u * 128;
      if (j0 >= a1) break;
      const float* v = vv[u];
      uint32_t key[4], lg = 0, le = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool ok = j0 + 4 * lane + c < a1;
        key[c] = score_key(v[c]);
        lg += ok && key[c] > T;
        le += ok && key[c] == T;
      }
      uint32_t ig = lg, ie = le;  // inclusive scans over the lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t vg = __shfl_up_sync(0xFFFFFFFFu, ig, o), ve = __shfl_up_sync(0xFFFFFFFFu, ie, o);
        if (lane >= o) { ig += vg; ie += ve; }
      }
      uint32_t g = og + ig - lg, e = oe + ie - le;  // before this lane's first entry
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int64_t j = j0 + 4 * lane + c;
        if (j >= a1) break;
        if (key[c] > T) {
          // ordered: the kept entries before j are g above T and min(e, take_eq) at T
          const uint32_t p = ordered ? g + min(e, take_eq) : g;
          oi[p] = static_cast<int32_t>(j);
          if (os) os[p] = v[c];
          ++g;
        } else if (key[c] == T) {
          if (e < take_eq) {
            const uint32_t p = ordered ? g + e : n_gt + e;
            oi[p] = static_cast<int32_t>(j);
            if (os) os[p] = v[c];
          }
          ++e;
        }
      }
      og += __shfl_sync(0xFFFFFFFFu, ig, 31);
      oe += __shfl_sync(0xFFFFFFFFu, ie, 31);
    }
  }
}

// Candidate form of the same selection.  A strided sample of 2,048 scores
// gives a key t that at least k entries of the row reach with high
// probability (the sample's r-th largest, r a few standard deviations above
// the k / n share of the sample, rounded down to a bin of 2^10 keys); one
// pass over the row copies every entry with key >= t into shared memory, in
// index order per warp segment.  When at least k entries reached t, the k
// best of the row are all among them (ties at the k-th key included), and
// the radix select and the index-ordered pass run over the candidates.
// Returns false (uniformly over the CTA) when the candidates do not fit in
// kCandR slots per warp or fewer than k entries reached t: the caller then
// runs topk_row_full, so the result never depends on the sample.
constexpr int kCandR = 256;      // candidate slots per warp
constexpr int kSamples = 2 * kTopkThreads;
constexpr int kTopkDynSmem = 2 * kTopkWarps * kCandR * 4;  // keys, then indices

__device__ bool topk_row_candidates(TopkShared& sh, uint32_t* cand, const float* s, int64_t n, int k, int32_t* oi,
                                    float* os, int ordered) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t below = (1u << lane) - 1u;  // lanes under this one
  // ---- t from the sample (every entry is a candidate when the row fits) ----
  uint32_t t = 0;
  if (n > static_cast<int64_t>(kTopkWarps) * kCandR) {
    const uint32_t s0 = score_key(__ldg(s + static_cast<int64_t>(tid) * n / kSamples));
    const uint32_t s1 = score_key(__ldg(s + static_cast<int64_t>(tid + kTopkThreads) * n / kSamples));
    const float mu = static_cast<float>(k) * kSamples / static_cast<float>(n);
    uint32_t need = static_cast<uint32_t>(min(static_cast<float>(kSamples), ceilf(mu + 4.f * sqrtf(mu) + 4.f)));
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 21 : 10;  // bits 21..31, then 10..20
      for (int i = tid; i < 2048; i += kTopkThreads) sh.hist[i] = 0;
      __syncthreads();
      if (pass == 0 || (s0 >> 21) == (t >> 21)) atomicAdd(&sh.hist[(s0 >> shift) & 2047u], 1u);
      if (pass == 0 || (s1 >> 21) == (t >> 21)) atomicAdd(&sh.hist[(s1 >> shift) & 2047u], 1u);
      __syncthreads();
      find_bin_all(sh, need);
      __syncthreads();
      t |= sh.sel_bin << shift;
      need -= sh.above;
    }
  }
  // ---- candidates: key >= t, per warp segment in index order ----
  uint32_t* ckey = cand + warp * kCandR;
  uint32_t* cidx = cand + kTopkWarps * kCandR + warp * kCandR;
  const Row4 rs4{s, n, (reinterpret_cast<uintptr_t>(s) & 15) == 0};
  const int64_t segw = ((n + kTopkWarps - 1) / kTopkWarps + 127) & ~int64_t(127);
  const int64_t a0 = min(n, warp * segw), a1 = min(n, a0 + segw);
  uint32_t cnt = 0;  // candidates of this warp so far (warp-uniform)
  for (int64_t j1 = a0; j1 < a1; j1 += kU * 128) {
    float v[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) rs4.load(j1 + u * 128 + 4 * lane, v[u]);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int64_t j0 = j1 + u * 128 + 4 * lane;
      if (j1 + u * 128 >= a1) break;
      uint32_t key[4], b[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        key[c] = score_key(v[u][c]);
        b[c] = __ballot_sync(0xFFFFFFFFu, j0 + c < a1 && key[c] >= t);
      }
      const uint32_t tot = __popc(b[0]) + __popc(b[1]) + __popc(b[2]) + __popc(b[3]);
      if (tot == 0) continue;
      uint32_t pos = cnt + __popc(b[0] & below) + __popc(b[1] & below) + __popc(b[2] & below) + __popc(b[3] & below);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if ((b[c] >> lane) & 1u) {
          if (pos < kCandR) {
            ckey[pos] = key[c];
            cidx[pos] = static_cast<uint32_t>(j0 + c);
          }
          ++pos;
        }
      cnt += tot;
    }
  }
  if (lane == 0) sh.warp_gt[warp] = cnt;
  __syncthreads();
  uint32_t total = 0;
  bool fits = true;
  for (int w2 = 0; w2 < kTopkWarps; ++w2) {
    total += sh.warp_gt[w2];
    fits = fits && sh.warp_gt[w2] <= static_cast<uint32_t>(kCandR);
  }
  __syncthreads();
  if (!fits || total < static_cast<uint32_t>(k)) return false;

  // ---- radix select of the k-th key among the candidates (range [t, max]) ----
  uint32_t kmax = 0u;
  for (uint32_t i = lane; i < cnt; i += 32) kmax = max(kmax, ckey[i]);
  kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
  if (lane == 0) sh.warp_eq[warp] = kmax;
  __syncthreads();
  uint32_t hi = 0u;
  for (int w2 = 0; w2 < kTopkWarps; ++w2) hi = max(hi, sh.warp_eq[w2]);
  uint32_t lo = t;
  uint64_t span = static_cast<uint64_t>(hi - lo) + 1;
  uint32_t need = static_cast<uint32_t>(k);
  int shift = max(0, 64 - __clzll(static_cast<long long>(span - 1)) - 11);
  // a level whose chosen bin is taken whole (usual: ~1,000 candidates over
  // 2,048 bins) ends the search with T just below that bin
  bool whole = false;
  for (;;) {
    for (int i = tid; i < 2048; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = lane; i < cnt; i += 32) {
      const uint32_t d = ckey[i] - lo;
      if (static_cast<uint64_t>(d) < span) atomicAdd(&sh.hist[d >> shift], 1u);
    }
    __syncthreads();
    find_bin_all(sh, need);
    __syncthreads();
    const uint32_t b = sh.sel_bin;
    const uint32_t cb = sh.hist[b];  // entries in the chosen bin
    need -= sh.above;
    lo += b << shift;
    span = min(span - (static_cast<uint64_t>(b) << shift), static_cast<uint64_t>(1) << shift);
    __syncthreads();
    if (shift == 0) break;
    if (cb == need && lo != 0u) {
      whole = true;
      break;
    }
    shift = max(0, shift - 11);
  }
  const uint32_t T = whole ? lo - 1u : lo;  // the k-th largest key, or the key below the whole bin
  const uint32_t take_eq = whole ? 0u : need;  // entries equal to T that are kept
  const uint32_t n_gt = static_cast<uint32_t>(k) - take_eq;

  // ---- index-ordered output over the candidates ----
  uint32_t cg = 0, ce = 0;
  for (uint32_t i = lane; i < cnt; i += 32) {
    const uint32_t key = ckey[i];
    cg += key > T;
    ce += key == T;
  }
  cg = __reduce_add_sync(0xFFFFFFFFu, cg);
  ce = __reduce_add_sync(0xFFFFFFFFu, ce);
  if (lane == 0) { sh.warp_gt[warp] = cg; sh.warp_eq[warp] = ce; }
  __syncthreads();
  uint32_t og = 0, oe = 0;  // entries above / at T before the current step
  for (int w2 = 0; w2 < warp; ++w2) { og += sh.warp_gt[w2]; oe += sh.warp_eq[w2]; }
  for (uint32_t i0 = 0; i0 < cnt; i0 += 32) {
    const uint32_t i = i0 + lane;
    const uint32_t key = i < cnt ? ckey[i] : 0u;
    const bool pg = i < cnt && key > T, pe = i < cnt && key == T;
    const uint32_t bg = __ballot_sync(0xFFFFFFFFu, pg), be = __ballot_sync(0xFFFFFFFFu, pe);
    const uint32_t g = og + __popc(bg & below), e = oe + __popc(be & below);
    if (pg || (pe && e < take_eq)) {
      // ordered: the kept entries before this one are g above T and min(e, take_eq) at T
      const uint32_t p = pg ? (ordered ? g + min(e, take_eq) : g) : (ordered ? g + e : n_gt + e);
      const uint32_t j = cidx[i];
      oi[p] = static_cast<int32_t>(j);
      if (os) os[p] = __ldg(s + j);
    }
    og += __popc(bg);
    oe += __popc(be);
  }
  return true;
}

__global__ void __launch_bounds__(kTopkThreads)
topk_row_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_valid, int64_t max_n,
                int k, int32_t* __restrict__ out_idx, float* __restrict__ out_score, int nv_div, int ordered) {
  __shared__ TopkShared sh;
  extern __shared__ uint32_t cand[];
  const int row = blockIdx.x;
  // valid columns: ceil(n_valid / nv_div), or max_n without n_valid
  const int64_t nv = n_valid ? (static_cast<int64_t>(n_valid[row]) + nv_div - 1) / nv_div : max_n;
  const int64_t n = min(max(nv, int64_t(0)), max_n);
  const float* s = scores + static_cast<int64_t>(row) * ld;
  int32_t* oi = out_idx + static_cast<int64_t>(row) * k;
  float* os = out_score ? out_score + static_cast<int64_t>(row) * k : nullptr;

  if (n <= k) {
    for (int64_t j = threadIdx.x; j < k; j += kTopkThreads) {
      oi[j] = j < n ? static_cast<int32_t>(j) : -1;
      if (os) os[j] = j < n ? s[j] : -INFINITY;
    }
    return;
  }
  if (!topk_row_candidates(sh, cand, s, n, k, oi, os, ordered)) topk_row_full(sh, s, n, k, oi, os, ordered);
}

template <int H, int DI>
csa_status_t launch_score_t(const csa_params_t* p, int nq, const csa_tensor_t* q_idx, const float* w,
                            const csa_tensor_t* k_idx, int batch, int64_t cap, const int32_t* q_req,
                            const int32_t* n_visible, float* scores, int64_t ld, int64_t max_entries,
                            cudaStream_t stream, const int32_t* pool, int block, int pool_blocks) {
  dim3 grid(static_cast<unsigned>((max_entries + kScoreThreads - 1) / kScoreThreads), nq);
  prof_begin(stream);
  index_score_simt_kernel<H, DI><<<grid, kScoreThreads, 0, stream>>>(
      q_idx->data, q_idx->dtype, w, k_idx->data, static_cast<const float*>(k_idx->scale), k_idx->dtype, batch, cap,
      q_req, n_visible, scores,
      ld, pool, block, pool_blocks);
  return check_launch("index_score_simt_kernel", stream);
}

}  // namespace

csa_status_t launch_index_score(const csa_params_t* p, int nq, const csa_tensor_t* q_idx, const float* w,
                                const csa_tensor_t* k_idx, int batch, int64_t cap, const int32_t* q_req,
                                const int32_t* n_visible, float* scores, int64_t ld, int64_t max_entries,
                                cudaStream_t stream, const int32_t* pool, int block, int pool_blocks) {
  if (nq == 0 || max_entries == 0) return CSA_OK;
#define CSA_SCORE_CASE(H, DI)                                                                                  \
  if (p->h_idx == H && p->d_idx == DI)                                                                         \
    return launch_score_t<H, DI>(p, nq, q_idx, w, k_idx, batch, cap, q_req, n_visible, scores, ld, max_entries, \
                                 stream, pool, block, pool_blocks);
  CSA_SCORE_CASE(4, 32)
  CSA_SCORE_CASE(8, 32)
  CSA_SCORE_CASE(16, 64)
  CSA_SCORE_CASE(32, 128)
  CSA_SCORE_CASE(64, 128)
#undef CSA_SCORE_CASE
  return set_error(CSA_ERR_UNSUPPORTED, "indexer shape h_idx=%d d_idx=%d is not built", p->h_idx, p->d_idx);
}

csa_status_t launch_topk(const float* scores, int n_rows, int64_t ld, const int32_t* n_valid, int64_t max_n, int k,
                         int32_t* out_idx, float* out_score, cudaStream_t stream, int nv_div, int ordered) {
  if (n_rows == 0) return CSA_OK;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(topk_row_kernel),
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kTopkDynSmem);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  prof_begin(stream);
  topk_row_kernel<<<n_rows, kTopkThreads, kTopkDynSmem, stream>>>(scores, ld, n_valid, max_n, k, out_idx, out_score,
                                                                  nv_div, ordered);
  return check_launch("topk_row_kernel", stream);
}

namespace {

// Block maxima of score rows: out[q][b] = max of scores[q][b*block ..
// min(n, (b+1)*block)) for the n = n_visible[q] valid scores of row q.
__global__ void block_max_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_visible,
                                 int64_t cap, int block, float* __restrict__ out, int64_t ld_out) {
  const int q = blockIdx.y;
  const int64_t n = min(max(static_cast<int64_t>(n_visible[q]), int64_t(0)), cap);
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b * block >= n) return;
  const float* s = scores + static_cast<int64_t>(q) * ld + b * block;
  float m = s[0];
  for (int i = 1; i < block && b * block + i < n; ++i) m = fmaxf(m, s[i]);
  out[static_cast<int64_t>(q) * ld_out + b] = m;
}

// Pool positions -> entry ids: pos -> pool[q][pos / block] * block + pos % block;
// -1 for padding and for positions whose score is -inf (not a visible entry).
__global__ void pool_map_kernel(const int32_t* __restrict__ pos, const float* __restrict__ pos_score, int k,
                                const int32_t* __restrict__ pool, int block, int pool_blocks,
                                int32_t* __restrict__ out_idx) {
  const int q = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= k) return;
  const int32_t p = pos[static_cast<int64_t>(q) * k + i];
  int32_t e = -1;
  if (p >= 0 && pos_score[static_cast<int64_t>(q) * k + i] != -INFINITY) {
    const int32_t b = pool[static_cast<int64_t>(q) * pool_blocks + p / block];
    if (b >= 0) e = b * block + p % block;
  }
  out_idx[static_cast<int64_t>(q) * k + i] = e;
}

}  // namespace

csa_status_t launch_block_max(const float* scores, int nq, int64_t ld, const int32_t* n_visible, int64_t cap,
                              int block, float* out, int64_t ld_out, cudaStream_t stream) {
  if (nq == 0) return CSA_OK;
  const int64_t nb = (cap + block - 1) / block;
  dim3 grid(static_cast<unsigned>((nb + 255) / 256), nq);
  prof_begin(stream);
  block_max_kernel<<<grid, 256, 0, stream>>>(scores, ld, n_visible, cap, block, out, ld_out);
  return check_launch("block_max_kernel", stream);
}

csa_status_t launch_pool_map(const int32_t* pos, const float* pos_score, int nq, int k, const int32_t* pool, int block,
                             int pool_blocks, int32_t* out_idx, cudaStream_t stream) {
  if (nq == 0) return CSA_OK;
  dim3 grid(static_cast<unsigned>((k + 255) / 256), nq);
  prof_begin(stream);
  pool_map_kernel<<<grid, 256, 0, stream>>>(pos, pos_score, k, pool, block, pool_blocks, out_idx);
  return check_launch("pool_map_kernel", stream);
}

}  // namespace csa
