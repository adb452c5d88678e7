// K2 + K3 on the tensor cores: lightning-indexer scores and the exact
// per-query top-k of one decode query per request, in one persistent
// cooperative kernel.
//
// Atlas "Model architectures", "Trained sparse attention" entry (DSA:
// lightning indexer + fine-grained top-k) and "compressed KV" entry;
// tech-report tour, "The indexer selects, SWA covers the rest" and "The
// Hierarchical Sparse Indexer" (the full-range scan over the causally
// visible context is the cost that dominates at long context).
//
//   s_j = sum_h w_h * max(0, q_h . k_j)
//
// Layout: request r's visible keys are cut into `chunks` contiguous ranges
// of 128-key tiles, one CTA per range (grid = batch * chunks <= #SMs, all
// resident: cooperative launch).  Inside a CTA:
//   warp 0     TMA producer: key tiles (128 rows x 128 B, 128B swizzle)
//              into a ring of shared-memory stages;
//   warp 1     MMA issuer: D[128 keys][64 heads] (fp32, TMEM, two buffers)
//              = keys x q^T with tcgen05.mma, M=128, N=64;
//   warps 2-5  epilogue: TMEM -> registers, s = sum_h w_h ReLU(D_h),
//              scores kept in shared memory.
// FP8 keys are consumed as stored (kind::f8f6f4, E4M3 x E4M3): the bf16
// query, scaled by a power of two 2^e so that max|q| 2^e lies in [128, 256),
// is split into two E4M3 terms q1 = e4m3(q 2^e), q2 = e4m3(q 2^e - q1) and
// both are accumulated into the same D; q1 + q2 equals q 2^e exactly for
// every element with |q 2^e| >= 2^-2 (smaller elements keep an absolute
// error below 2^-10 / 2^e).  The score is then multiplied by 2^-e and by
// the key row's fp32 scale (ReLU(c x) = c ReLU(x) for c > 0).  bf16 keys use
// kind::f16 with the bf16 query directly.
//
// Top-k (score descending, lower index first on exact ties): a radix select
// on the ordered 32-bit key of each fp32 score, distributed over the CTAs
// of a request: pass 1 histograms bits 31..20, pass 2 bits 19..8 of the keys
// in the boundary bin, each CTA adding its shared-memory histogram into a
// global one, separated by bounded per-request grid barriers.  Every CTA
// then stages, in index order, its keys above the 24-bit boundary prefix and
// those equal to it; the last CTA of the request to finish (atomic counter,
// no waiting) concatenates them in chunk order -- which is index order --
// and resolves the remaining boundary entries exactly (low 8 bits, then
// lowest indices), so the output order is deterministic.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr int kHeads = 64;
constexpr int kDI = 128;
constexpr int kThreads = 192;
constexpr int kMaxChunkTiles = 128;
constexpr int kHistBins = 4096;
constexpr int kEqCache = 8192;   // boundary entries the last CTA resolves in shared memory
constexpr uint32_t kWaitLimit = 1u << 22;     // mbarrier polls
constexpr uint32_t kSpinLimit = 1u << 22;     // grid-barrier polls (~64 ns apart)

__device__ uint32_t g_index_tc_error = 0;   // bit 0: wait timed out

template <bool FP8>
struct Cfg {
  static constexpr int kStageBytes = FP8 ? 16384 : 32768;
  static constexpr int kStages = FP8 ? 6 : 4;
  static constexpr int kBBytes = 16384;
  static constexpr int oStages = 0;
  static constexpr int oB = kStages * kStageBytes;
  static constexpr int oScores = oB + kBBytes;
  static constexpr int oW = oScores + kMaxChunkTiles * kTileM * 4;
  static constexpr int oBars = oW + kHeads * 4;
  static constexpr int oMisc = oBars + 256;
  static constexpr int kSmem = oMisc + 256 + 1024;
  static constexpr uint32_t kIdesc = FP8 ? idesc(0, 0, kTileM, kHeads) : idesc(1, 1, kTileM, kHeads);
};

struct IdxArgs {
  const uint16_t* q_idx;   // [batch][64][128] bf16 bits
  const float* w;          // [batch][64]
  const float* kscale;     // FP8: [batch][cap] row scales
  int batch;
  int64_t cap;
  const int32_t* n_visible;
  int chunks;
  int k;
  int32_t* out_idx;
  float* out_score;
  uint32_t* ghist;         // [batch][2][4096]  (zero on entry)
  uint32_t* sync;          // [batch][4]        (zero on entry): barrier, done
  uint32_t* cnt;           // [batch][chunks][2]
  int32_t* st_idx;         // [batch][chunks][k]
  float* st_score;
  int32_t* eq_idx;         // [batch][chunks][kMaxChunkTiles * 128]
  float* eq_score;
};

struct Shared {
  uint32_t tmem_base;
  uint32_t bcast[8];
  int fail;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Bounded per-request grid barrier; returns false on timeout.
__device__ bool request_barrier(uint32_t* ctr, uint32_t target, Shared& sh) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(ctr, 1u);
    uint32_t it = 0;
    while (ld_acquire_gpu(ctr) < target) {
      if (++it > kSpinLimit) {
        atomicOr(&g_index_tc_error, 1u);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    sh.bcast[7] = ok;
  }
  __syncthreads();
  return sh.bcast[7] != 0;
}

// Whole block: bin b of a shared-memory histogram of kHistBins bins,
// scanned from the top, with above(b) < need <= above(b) + hist[b]; writes
// (b, above) to bcast[0..1].  Threads 0..127 own 32 consecutive bins each.
__device__ void find_bin_block(const uint32_t* hist, uint32_t need, Shared& sh, uint32_t* scratch) {
  const int tid = threadIdx.x;
  constexpr int per = kHistBins / 128;
  uint32_t mine = 0;
  if (tid < 128) {
#pragma unroll
    for (int i = 0; i < per; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(hist + tid * per + i);
      mine += v.x + v.y + v.z + v.w;
    }
    scratch[tid] = mine;
  }
  __syncthreads();
  if (tid < 32) {
    // suffix sums of the 128 thread totals, four per lane
    uint32_t t4[4], s4 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) { t4[q] = scratch[tid * 4 + q]; s4 += t4[q]; }
    uint32_t incl = s4;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
      if (tid + o < 32) incl += v;
    }
    uint32_t above = incl - s4;  // totals of lanes above this one
#pragma unroll
    for (int q = 3; q >= 0; --q) {
      scratch[128 + tid * 4 + q] = above;  // above(thread) = totals of higher threads
      above += t4[q];
    }
  }
  __syncthreads();
  if (tid < 128) {
    const uint32_t excl = scratch[128 + tid];
    if (excl < need && need <= excl + mine) {
      uint32_t above = excl;
      for (int i = per - 1; i >= 0; --i) {
        const uint32_t c = hist[tid * per + i];
        if (above + c >= need) {
          sh.bcast[0] = tid * per + i;
          sh.bcast[1] = above;
          break;
        }
        above += c;
      }
    }
  }
  __syncthreads();
}

// Copies a global histogram (written by other CTAs) into shared memory.
__device__ __forceinline__ void load_hist(uint32_t* dst, const uint32_t* src) {
  for (int i = threadIdx.x; i < kHistBins / 4; i += kThreads)
    reinterpret_cast<uint4*>(dst)[i] = __ldcg(reinterpret_cast<const uint4*>(src) + i);
  __syncthreads();
}

// Block-wide index-ordered compaction step over `cnt` items: returns the
// rank of this thread's flagged item among flagged items of the block and
// the block total, for two flags at once.
__device__ __forceinline__ void block_rank2(bool f0, bool f1, uint32_t& r0, uint32_t& r1, uint32_t& t0,
                                            uint32_t& t1, uint32_t* scratch /* 2 * warps */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int W = kThreads / 32;
  const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, f0), b1 = __ballot_sync(0xFFFFFFFFu, f1);
  if (lane == 0) {
    scratch[warp] = __popc(b0);
    scratch[W + warp] = __popc(b1);
  }
  __syncthreads();
  uint32_t o0 = 0, o1 = 0, s0 = 0, s1 = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const uint32_t a = scratch[w], b = scratch[W + w];
    if (w < warp) { o0 += a; o1 += b; }
    s0 += a; s1 += b;
  }
  const uint32_t lm = (1u << lane) - 1u;
  r0 = o0 + __popc(b0 & lm);
  r1 = o1 + __popc(b1 & lm);
  t0 = s0;
  t1 = s1;
  __syncthreads();
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
index_topk_tc_kernel(const __grid_constant__ CUtensorMap kmap, IdxArgs a) {
  using C = Cfg<FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Shared& sh = *reinterpret_cast<Shared*>(smem + C::oMisc);
  float* scores = reinterpret_cast<float*>(smem + C::oScores);
  float* ws = reinterpret_cast<float*>(smem + C::oW);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::oBars);
  uint64_t* empty = full + 8;
  uint64_t* tfull = full + 16;
  uint64_t* tempty = full + 18;
  uint64_t* mdone = full + 20;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x / a.chunks, c = blockIdx.x % a.chunks;
  const int64_t n = min(max(static_cast<int64_t>(a.n_visible[r]), int64_t(0)), a.cap);
  const int tiles_req = static_cast<int>((n + kTileM - 1) / kTileM);
  const int t0 = static_cast<int>(static_cast<int64_t>(c) * tiles_req / a.chunks);
  const int t1 = static_cast<int>(static_cast<int64_t>(c + 1) * tiles_req / a.chunks);
  const int nt = min(t1 - t0, kMaxChunkTiles);

  // ---------------- prologue ----------------
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(mdone, 1);
    sh.fail = 0;
    fence_barrier_init();
    prefetch_tensormap(&kmap);
  }
  if (warp == 1) tmem_alloc(&sh.tmem_base, 128);

  // query operand: bf16 [64 heads][128] -> swizzled K-major blocks
  const uint16_t* q = a.q_idx + static_cast<int64_t>(r) * kHeads * kDI;
  uint8_t* Bs = smem + C::oB;
  float qinv = 1.f;
  if constexpr (FP8) {
    float m = 0.f;
    for (int i = tid; i < kHeads * kDI / 8; i += kThreads) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(q) + i);
      const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        m = fmaxf(m, fabsf(__uint_as_float(wds[e] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(wds[e] & 0xFFFF0000u)));
      }
    }
    m = warp_max(m);
    if (lane == 0) sh.bcast[warp] = __float_as_uint(m);
    __syncthreads();
    m = 0.f;
    for (int i = 0; i < kThreads / 32; ++i) m = fmaxf(m, __uint_as_float(sh.bcast[i]));
    int e = 0;
    if (m > 0.f) {
      frexpf(m, &e);  // m = f 2^e, f in [0.5, 1)
      e = min(8 - e, 126);  // m 2^e in [128, 256)
    }
    const float S = ldexpf(1.f, e);
    qinv = ldexpf(1.f, -e);
    // 16 elements (one 16-byte chunk of a 128-byte row) per task
    for (int task = tid; task < kHeads * 8; task += kThreads) {
      const int h = task >> 3, ch = task & 7;
      const uint4* src = reinterpret_cast<const uint4*>(q + h * kDI + ch * 16);
      const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
      const uint32_t wds[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      uint32_t p1[4] = {0, 0, 0, 0}, p2[4] = {0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t wv = wds[i >> 1];
        const float x = __uint_as_float((i & 1) ? (wv & 0xFFFF0000u) : (wv << 16)) * S;
        const uint8_t c1 = f32_to_e4m3(x);
        const float r1 = x - e4m3_to_f32(c1);
        const uint8_t c2 = f32_to_e4m3(r1);
        p1[i >> 2] |= static_cast<uint32_t>(c1) << (8 * (i & 3));
        p2[i >> 2] |= static_cast<uint32_t>(c2) << (8 * (i & 3));
      }
      const uint32_t off = sw128_offset(h, ch);
      *reinterpret_cast<uint4*>(Bs + off) = make_uint4(p1[0], p1[1], p1[2], p1[3]);
      *reinterpret_cast<uint4*>(Bs + 8192 + off) = make_uint4(p2[0], p2[1], p2[2], p2[3]);
    }
  } else {
    // two 64-element K halves, 8 bf16 per 16-byte chunk
    for (int task = tid; task < 2 * kHeads * 8; task += kThreads) {
      const int half = task / (kHeads * 8), h = (task / 8) % kHeads, ch = task & 7;
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(q + h * kDI + half * 64 + ch * 8));
      *reinterpret_cast<uint4*>(Bs + half * 8192 + sw128_offset(h, ch)) = u;
    }
  }
  for (int i = tid; i < kHeads; i += kThreads) ws[i] = a.w[static_cast<int64_t>(r) * kHeads + i];
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  // ---------------- phase 1: scores ----------------
  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % C::kStages;
        const uint32_t ph = (t / C::kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, kWaitLimit)) {
          atomicOr(&g_index_tc_error, 1u);
          sh.fail = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        const int y = static_cast<int>(r * a.cap + static_cast<int64_t>(t0 + t) * kTileM);
        uint8_t* dst = smem + C::oStages + s * C::kStageBytes;
        tma_load_2d(dst, &kmap, &full[s], 0, y);
        if constexpr (!FP8) tma_load_2d(dst + 16384, &kmap, &full[s], 64, y);
        issued = t + 1;
      }
      // on failure, let the copies still in flight land before the CTA exits
      if (sh.fail)
        for (int t = max(0, issued - C::kStages); t < issued; ++t)
          mbar_wait(&full[t % C::kStages], (t / C::kStages) & 1, kWaitLimit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t b_base = smem_u32(Bs);
      for (int t = 0; t < nt; ++t) {
        const int s = t % C::kStages;
        const uint32_t ph = (t / C::kStages) & 1;
        const int acc = t & 1;
        const uint32_t aph = (t >> 1) & 1;
        if (!mbar_wait(&full[s], ph, kWaitLimit) || !mbar_wait(&tempty[acc], aph ^ 1, kWaitLimit)) {
          atomicOr(&g_index_tc_error, 1u);
          sh.fail = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + acc * kHeads;
        const uint32_t a_base = smem_u32(smem + C::oStages + s * C::kStageBytes);
        if constexpr (FP8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = desc_k_sw128(a_base + kk * 32);
            mma_f8f6f4(d, ad, desc_k_sw128(b_base + kk * 32), C::kIdesc, kk > 0 ? 1u : 0u);
            mma_f8f6f4(d, ad, desc_k_sw128(b_base + 8192 + kk * 32), C::kIdesc, 1u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t half = kk >> 2, off = (kk & 3) * 32;
            mma_f16(d, desc_k_sw128(a_base + half * 16384 + off), desc_k_sw128(b_base + half * 8192 + off),
                    C::kIdesc, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[acc]);
      }
      // every MMA of this CTA has completed before TMEM is released
      mma_commit(mdone);
      mbar_wait(mdone, 0, kWaitLimit);
    }
  } else {
    const int sub = warp & 3;  // TMEM lanes 32*sub .. 32*sub+31
    const int row = sub * 32 + lane;
    // FP8 key scales are loaded four tiles ahead so their latency hides
    // behind the MMA pipeline
    auto load_ks = [&](int t) -> float {
      if constexpr (FP8) {
        const int64_t j = static_cast<int64_t>(t0 + t) * kTileM + row;
        if (t < nt && j < n) return __ldg(a.kscale + r * a.cap + j);
      }
      return 1.f;
    };
    float ks[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) ks[u] = load_ks(u);
    bool ok = true;
    for (int tb = 0; tb < nt && ok; tb += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = tb + u;
        if (t < nt && ok) {
          const int acc = t & 1;
          const uint32_t aph = (t >> 1) & 1;
          const int64_t j = static_cast<int64_t>(t0 + t) * kTileM + row;
          if (!mbar_wait(&tfull[acc], aph, kWaitLimit)) {
            atomicOr(&g_index_tc_error, 1u);
            sh.fail = 1;
            ok = false;
          } else {
            tc_fence_after();
            uint32_t v0[32], v1[32];
            const uint32_t ta = tmem + (static_cast<uint32_t>(sub * 32) << 16) + acc * kHeads;
            tmem_ld32(ta, v0);
            tmem_ld32(ta + 32, v1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int h = 0; h < 32; ++h) {
              s0 = fmaf(ws[h], fmaxf(__uint_as_float(v0[h]), 0.f), s0);
              s1 = fmaf(ws[32 + h], fmaxf(__uint_as_float(v1[h]), 0.f), s1);
            }
            float sc = s0 + s1;
            if constexpr (FP8) sc = sc * qinv * ks[u];
            if (j < n) scores[t * kTileM + row] = sc;
            ks[u] = load_ks(t + 4);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
  if (sh.fail) return;

  // ---------------- phase 2: top-k ----------------
  const int64_t base = static_cast<int64_t>(t0) * kTileM;          // first key of the chunk
  const int nloc = static_cast<int>(max(int64_t(0), min(n, static_cast<int64_t>(t0 + nt) * kTileM) - base));
  const int k = a.k;
  int32_t* oi = a.out_idx + static_cast<int64_t>(r) * k;
  float* os = a.out_score ? a.out_score + static_cast<int64_t>(r) * k : nullptr;

  if (n <= k) {
    for (int i = tid; i < nloc; i += kThreads) {
      oi[base + i] = static_cast<int32_t>(base + i);
      if (os) os[base + i] = scores[i];
    }
    if (c == 0)
      for (int64_t j = n + tid; j < k; j += kThreads) {
        oi[j] = -1;
        if (os) os[j] = -INFINITY;
      }
    return;
  }

  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::oStages);      // stages are free now
  uint32_t* scratch = hist + kHistBins;             // 256 words
  uint32_t* cpre = scratch + 256;                    // per-chunk prefixes (above, boundary)
  int32_t* eq_cache_i = reinterpret_cast<int32_t*>(cpre + 2 * 160);
  float* eq_cache_s = reinterpret_cast<float*>(eq_cache_i + kEqCache);
  uint32_t* gh1 = a.ghist + static_cast<int64_t>(r) * 2 * kHistBins;
  uint32_t* gh2 = gh1 + kHistBins;
  uint32_t* bar = a.sync + r * 4;

  // pass 1: bits 31..20
  for (int i = tid; i < kHistBins; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < nloc; i += kThreads) atomicAdd(&hist[score_key(scores[i]) >> 20], 1u);
  __syncthreads();
  for (int i = tid; i < kHistBins; i += kThreads)
    if (hist[i]) atomicAdd(&gh1[i], hist[i]);
  if (!request_barrier(&bar[0], a.chunks, sh)) return;
  load_hist(hist, gh1);
  find_bin_block(hist, static_cast<uint32_t>(k), sh, scratch);
  const uint32_t b1 = sh.bcast[0];
  const uint32_t need1 = static_cast<uint32_t>(k) - sh.bcast[1];

  // pass 2: bits 19..8 of the keys in bin b1
  for (int i = tid; i < kHistBins; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < nloc; i += kThreads) {
    const uint32_t key = score_key(scores[i]);
    if ((key >> 20) == b1) atomicAdd(&hist[(key >> 8) & 0xFFFu], 1u);
  }
  __syncthreads();
  for (int i = tid; i < kHistBins; i += kThreads)
    if (hist[i]) atomicAdd(&gh2[i], hist[i]);
  if (!request_barrier(&bar[0], 2u * a.chunks, sh)) return;
  load_hist(hist, gh2);
  find_bin_block(hist, need1, sh, scratch);
  const uint32_t prefix = (b1 << 12) | sh.bcast[0];  // 24-bit boundary prefix
  const uint32_t need2 = need1 - sh.bcast[1];          // still to take from the boundary

  // stage this chunk's entries above / at the boundary prefix, index order
  const int64_t slot = static_cast<int64_t>(r) * a.chunks + c;
  int32_t* sti = a.st_idx + slot * k;
  float* sts = a.st_score + slot * k;
  int32_t* eqi = a.eq_idx + slot * (kMaxChunkTiles * kTileM);
  float* eqs = a.eq_score + slot * (kMaxChunkTiles * kTileM);
  uint32_t n_above = 0, n_eq = 0;
  for (int i0 = 0; i0 < nloc; i0 += kThreads) {
    const int i = i0 + tid;
    float v = 0.f;
    uint32_t kp = 0;
    if (i < nloc) {
      v = scores[i];
      kp = score_key(v) >> 8;
    }
    const bool above = i < nloc && kp > prefix, eq = i < nloc && kp == prefix;
    uint32_t ra, re, ta, te;
    block_rank2(above, eq, ra, re, ta, te, scratch);
    if (above && n_above + ra < static_cast<uint32_t>(k)) {
      sti[n_above + ra] = static_cast<int32_t>(base + i);
      sts[n_above + ra] = v;
    }
    if (eq) { eqi[n_eq + re] = static_cast<int32_t>(base + i); eqs[n_eq + re] = v; }
    n_above += ta;
    n_eq += te;
  }
  if (tid == 0) {
    a.cnt[slot * 2] = n_above;
    a.cnt[slot * 2 + 1] = n_eq;
    __threadfence();
    const uint32_t prev = atomicAdd(&bar[1], 1u);
    sh.bcast[2] = (prev == static_cast<uint32_t>(a.chunks) - 1) ? 1u : 0u;
  }
  __syncthreads();
  if (!sh.bcast[2]) return;

  // ---------------- last CTA of the request: assemble ----------------
  __threadfence();
  const uint32_t* cnt = a.cnt + static_cast<int64_t>(r) * a.chunks * 2;
  const int nch = a.chunks;
  for (int cc = tid; cc < nch; cc += kThreads) {
    cpre[cc] = __ldcg(cnt + cc * 2);
    cpre[160 + cc] = __ldcg(cnt + cc * 2 + 1);
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t sa = 0, se = 0;
    for (int cc = 0; cc < nch; ++cc) {
      const uint32_t x = cpre[cc], y = cpre[160 + cc];
      cpre[cc] = sa;
      cpre[160 + cc] = se;
      sa += x;
      se += y;
    }
    cpre[nch] = sa;
    cpre[160 + nch] = se;
  }
  __syncthreads();
  const uint32_t A = min(cpre[nch], static_cast<uint32_t>(k));
  const uint32_t E = cpre[160 + nch];
  const int64_t eq_stride = kMaxChunkTiles * kTileM;
  // chunk of the i-th entry of a concatenation with exclusive prefixes pre[]
  auto chunk_of = [&](const uint32_t* pre, uint32_t i) {
    int lo = 0, hi = nch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  for (uint32_t i = tid; i < A; i += kThreads) {
    const int cc = chunk_of(cpre, i);
    const int64_t src = (static_cast<int64_t>(r) * nch + cc) * k + (i - cpre[cc]);
    oi[i] = __ldcg(a.st_idx + src);
    if (os) os[i] = __ldcg(a.st_score + src);
  }
  const uint32_t room = static_cast<uint32_t>(k) - A;  // == need2 when the counts agree
  const uint32_t take = min(need2, room);
  if (E <= take) {
    for (uint32_t i = tid; i < E; i += kThreads) {
      const int cc = chunk_of(cpre + 160, i);
      const int64_t src = (static_cast<int64_t>(r) * nch + cc) * eq_stride + (i - cpre[160 + cc]);
      oi[A + i] = __ldcg(a.eq_idx + src);
      if (os) os[A + i] = __ldcg(a.eq_score + src);
    }
    return;
  }
  // more boundary entries than places left: the low 8 bits of the key
  // decide, then the lowest indices (entries are in index order)
  const uint32_t ncache = min(E, static_cast<uint32_t>(kEqCache));
  for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
  for (uint32_t i = tid; i < ncache; i += kThreads) {
    const int cc = chunk_of(cpre + 160, i);
    const int64_t src = (static_cast<int64_t>(r) * nch + cc) * eq_stride + (i - cpre[160 + cc]);
    eq_cache_i[i] = __ldcg(a.eq_idx + src);
    eq_cache_s[i] = __ldcg(a.eq_score + src);
  }
  __syncthreads();
  auto eq_at = [&](uint32_t i, int32_t& j, float& v) {
    if (i < ncache) {
      j = eq_cache_i[i];
      v = eq_cache_s[i];
    } else {
      const int cc = chunk_of(cpre + 160, i);
      const int64_t src = (static_cast<int64_t>(r) * nch + cc) * eq_stride + (i - cpre[160 + cc]);
      j = __ldcg(a.eq_idx + src);
      v = __ldcg(a.eq_score + src);
    }
  };
  for (uint32_t i = tid; i < E; i += kThreads) {
    int32_t j;
    float v;
    eq_at(i, j, v);
    atomicAdd(&hist[score_key(v) & 0xFFu], 1u);
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t above = 0;
    for (int b = 255; b >= 0; --b) {
      if (above + hist[b] >= take) {
        sh.bcast[3] = (prefix << 8) | b;
        sh.bcast[4] = take - above;
        break;
      }
      above += hist[b];
    }
  }
  __syncthreads();
  const uint32_t T = sh.bcast[3], take_eq = sh.bcast[4];
  uint32_t out = A, got_eq = 0;
  for (uint32_t i0 = 0; i0 < E; i0 += kThreads) {
    const uint32_t i = i0 + tid;
    int32_t j = 0;
    float v = 0.f;
    uint32_t key = 0;
    if (i < E) {
      eq_at(i, j, v);
      key = score_key(v);
    }
    const bool gt = i < E && key > T, eq = i < E && key == T;
    uint32_t rg, re, tg, te;
    block_rank2(gt, eq, rg, re, tg, te, scratch);
    if (gt && out + rg < static_cast<uint32_t>(k)) {
      oi[out + rg] = j;
      if (os) os[out + rg] = v;
    }
    out += tg;
    if (eq && got_eq + re < take_eq && out + re < static_cast<uint32_t>(k)) {
      oi[out + re] = j;
      if (os) os[out + re] = v;
    }
    const uint32_t add = min(te, take_eq - got_eq);
    got_eq += add;
    out += add;
  }
}

struct Launcher {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  int sms = 0;
  bool attr_set[2] = {false, false};
};

Launcher& launcher() {
  static Launcher L;
  if (!L.encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      L.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&L.sms, cudaDevAttrMultiProcessorCount, dev);
  }
  return L;
}

}  // namespace

// Host-side plan: chunks per request and workspace carve-up of the fused
// kernel (shared with csa_api.cu through these functions).
int index_tc_chunks(int batch, int64_t cap) {
  const int sms = launcher().sms > 0 ? launcher().sms : 148;
  const int64_t tiles = (cap + kTileM - 1) / kTileM;
  int ch = sms / (batch > 0 ? batch : 1);
  if (ch > tiles) ch = static_cast<int>(tiles > 0 ? tiles : 1);
  return ch;
}

bool index_tc_supported(const csa_params_t* p, int batch, int64_t cap, int q_dtype, int k_dtype) {
  if (p->h_idx != kHeads || p->d_idx != kDI || q_dtype != kBF16) return false;
  if (k_dtype != kFP8 && k_dtype != kBF16) return false;
  if (batch < 1 || batch > (launcher().sms > 0 ? launcher().sms : 148)) return false;
  if (static_cast<int64_t>(batch) * cap >= (int64_t(1) << 31)) return false;
  const int ch = index_tc_chunks(batch, cap);
  const int64_t tiles = (cap + kTileM - 1) / kTileM;
  return (tiles + ch - 1) / ch <= kMaxChunkTiles && p->topk >= 1;
}

size_t index_tc_control_bytes(int batch) { return static_cast<size_t>(batch) * (2 * kHistBins + 4) * 4; }

size_t index_tc_workspace_bytes(int batch, int64_t cap, int k) {
  const int ch = index_tc_chunks(batch, cap);
  size_t b = index_tc_control_bytes(batch);
  b += static_cast<size_t>(batch) * ch * 2 * 4;                       // cnt
  b += static_cast<size_t>(batch) * ch * k * 8;                       // staging above
  b += static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 8;  // staging boundary
  return b + 4 * 256;
}

// `ws` must hold index_tc_workspace_bytes; its first index_tc_control_bytes
// must be zero on entry (the caller zeroes them).
csa_status_t launch_index_topk_tc(const csa_params_t* p, int batch, const csa_tensor_t* q_idx, const float* w,
                                  const csa_tensor_t* k_idx, int64_t cap, const int32_t* n_visible, int32_t* out_idx,
                                  float* out_score, void* ws, cudaStream_t stream) {
  Launcher& L = launcher();
  if (!L.encode) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const bool fp8 = k_idx->dtype == kFP8;
  const int ch = index_tc_chunks(batch, cap);
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDI), static_cast<cuuint64_t>(batch) * cap};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDI) * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(fp8 ? 128 : 64), static_cast<cuuint32_t>(kTileM)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = L.encode(&map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                         k_idx->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(cr));

  IdxArgs a;
  a.q_idx = static_cast<const uint16_t*>(q_idx->data);
  a.w = w;
  a.kscale = fp8 ? k_idx->scale : nullptr;
  a.batch = batch;
  a.cap = cap;
  a.n_visible = n_visible;
  a.chunks = ch;
  a.k = p->topk;
  a.out_idx = out_idx;
  a.out_score = out_score;
  char* base = static_cast<char*>(ws);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = base + off;
    off = (off + bytes + 255) & ~static_cast<size_t>(255);
    return q;
  };
  a.ghist = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(batch) * 2 * kHistBins * 4));
  a.sync = reinterpret_cast<uint32_t*>(base + static_cast<size_t>(batch) * 2 * kHistBins * 4);
  off = (index_tc_control_bytes(batch) + 255) & ~static_cast<size_t>(255);
  a.cnt = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(batch) * ch * 2 * 4));
  a.st_idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(batch) * ch * p->topk * 4));
  a.st_score = reinterpret_cast<float*>(take(static_cast<size_t>(batch) * ch * p->topk * 4));
  a.eq_idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 4));
  a.eq_score = reinterpret_cast<float*>(take(static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 4));

  const int smem = fp8 ? Cfg<true>::kSmem : Cfg<false>::kSmem;
  void* fn = fp8 ? reinterpret_cast<void*>(index_topk_tc_kernel<true>) : reinterpret_cast<void*>(index_topk_tc_kernel<false>);
  if (!L.attr_set[fp8 ? 1 : 0]) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    L.attr_set[fp8 ? 1 : 0] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch * ch);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  prof_begin(stream);
  cudaError_t e = fp8 ? cudaLaunchKernelEx(&cfg, index_topk_tc_kernel<true>, map, a)
                      : cudaLaunchKernelEx(&cfg, index_topk_tc_kernel<false>, map, a);
  if (e != cudaSuccess) {
    check_launch("index_topk_tc_kernel", stream);
    return set_error(CSA_ERR_CUDA, "index_topk_tc_kernel launch: %s", cudaGetErrorString(e));
  }
  return check_launch("index_topk_tc_kernel", stream);
}

// Reads and clears the device error word of this kernel (bounded waits).
uint32_t index_tc_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_index_tc_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_index_tc_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
