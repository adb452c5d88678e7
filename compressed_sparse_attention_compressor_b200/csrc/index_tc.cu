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

#include <cstring>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

using namespace sm100;

constexpr int kTileM = 128;
constexpr int kHeads = 64;
constexpr int kDI = 128;
constexpr int kEpiWarps = 8;                     // two groups of four, alternating tiles
constexpr int kThreads = 32 * (2 + kEpiWarps);   // producer, MMA, epilogue
constexpr int kPrep = kThreads - 32;             // threads preparing the query (warps 1..)
constexpr int kNAcc = 4;                         // accumulator buffers (64 TMEM columns each)
constexpr int kScoreCol = kNAcc * kHeads;        // first TMEM column holding scores (one per tile)
constexpr int kMaxChunkTiles = 512 - kScoreCol;
constexpr int kTmemCols = 512;
constexpr int kHistBins = 4096;
constexpr int kEqCache = 8192;                   // boundary entries resolved in shared memory
constexpr uint32_t kWaitLimit = 1u << 22;        // mbarrier polls
constexpr uint32_t kSpinLimit = 1u << 22;        // grid-barrier polls (~64 ns apart)

__device__ uint32_t g_index_tc_error = 0;  // bit 0: a bounded wait gave up

template <bool FP8>
struct Cfg {
  static constexpr int kStageBytes = FP8 ? 16384 : 32768;
  static constexpr int kStages = FP8 ? 9 : 5;
  static constexpr int kScaleBytes = FP8 ? kTileM * 4 : 0;  // per stage
  static constexpr int oStages = 0;
  static constexpr int oScales = kStages * kStageBytes;
  static constexpr int oB = oScales + (kStages * kScaleBytes + 1023) / 1024 * 1024;
  static constexpr int oQ = oB + 16384;            // raw query staging (bf16)
  static constexpr int oHist = oQ + 16384;          // two group histograms
  static constexpr int oW = oHist + 2 * kHistBins * 4;
  static constexpr int oBars = oW + kHeads * 4;
  static constexpr int oMisc = oBars + 512;
  static constexpr int kSmem = oMisc + 256 + 1024;
  static constexpr uint32_t kIdesc = FP8 ? idesc(0, 0, kTileM, kHeads) : idesc(1, 1, kTileM, kHeads);
  static constexpr uint32_t kEmptyCount = FP8 ? 1 + 128 : 1;  // MMA commit (+ epilogue scale reads)
  static_assert(sizeof(uint64_t) * (2 * kStages + 2 * kNAcc + 2) <= 512, "mbarrier area");
  static_assert(oB % 1024 == 0, "operand alignment");
  // phase-2 scratch, inside the (then idle) stage ring
  static constexpr int pHist = 0;                         // merged histogram
  static constexpr int pScratch = kHistBins * 4;          // 256 words
  static constexpr int pCpre = pScratch + 1024;           // 320 words
  static constexpr int pCntA = pCpre + 1536;              // [kMaxChunkTiles][4] words each
  static constexpr int pCntE = pCntA + kMaxChunkTiles * 16;
  static constexpr int pOffA = pCntE + kMaxChunkTiles * 16;
  static constexpr int pOffE = pOffA + kMaxChunkTiles * 16;
  static constexpr int pEq = pOffE + kMaxChunkTiles * 16;
  static_assert(pEq + kEqCache * 8 <= oScales, "phase-2 scratch must fit in the stage ring");
};

struct IdxArgs {
  const uint16_t* q_idx;   // [batch][64][128] bf16 bits
  const float* w;          // [batch][64]
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
  uint32_t qmax[kThreads / 32];
  float qinv;
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
      __nanosleep(32);
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
    uint32_t t4[4], s4 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      t4[q] = scratch[tid * 4 + q];
      s4 += t4[q];
    }
    uint32_t incl = s4;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
      if (tid + o < 32) incl += v;
    }
    uint32_t above = incl - s4;
#pragma unroll
    for (int q = 3; q >= 0; --q) {
      scratch[128 + tid * 4 + q] = above;
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

// Block-wide index-ordered compaction step: rank of this thread's flagged
// item among the block's flagged items, and the block totals, for two flags.
__device__ __forceinline__ void block_rank2(bool f0, bool f1, uint32_t& r0, uint32_t& r1, uint32_t& t0,
                                            uint32_t& t1, uint32_t* scratch) {
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
    s0 += a;
    s1 += b;
  }
  const uint32_t lm = (1u << lane) - 1u;
  r0 = o0 + __popc(b0 & lm);
  r1 = o1 + __popc(b1 & lm);
  t0 = s0;
  t1 = s1;
  __syncthreads();
}

// One warp: exclusive prefix sums of cnt[0..n) into off[0..n); returns the
// total (valid in every lane).
__device__ uint32_t warp_exclusive_scan(const uint32_t* cnt, uint32_t* off, int n) {
  const int lane = threadIdx.x & 31;
  const int seg = (n + 31) / 32;
  const int lo = min(n, lane * seg), hi = min(n, lo + seg);
  uint32_t mine = 0;
  for (int i = lo; i < hi; ++i) mine += cnt[i];
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  uint32_t run = incl - mine;
  for (int i = lo; i < hi; ++i) {
    off[i] = run;
    run += cnt[i];
  }
  return __shfl_sync(0xFFFFFFFFu, incl, 31);
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
index_topk_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap smap,
                     IdxArgs a) {
  using C = Cfg<FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Shared& sh = *reinterpret_cast<Shared*>(smem + C::oMisc);
  uint32_t* ghist0 = reinterpret_cast<uint32_t*>(smem + C::oHist);  // group 0; group 1 follows
  float* ws = reinterpret_cast<float*>(smem + C::oW);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::oBars);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + kNAcc;
  uint64_t* qbar = tempty + kNAcc;
  uint64_t* mdone = qbar + 1;
  uint8_t* Bs = smem + C::oB;
  const float* scale_ring = reinterpret_cast<const float*>(smem + C::oScales);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x / a.chunks, c = blockIdx.x % a.chunks;
  const int64_t n = min(max(static_cast<int64_t>(a.n_visible[r]), int64_t(0)), a.cap);
  const int tiles_req = static_cast<int>((n + kTileM - 1) / kTileM);
  const int t0 = static_cast<int>(static_cast<int64_t>(c) * tiles_req / a.chunks);
  const int t1 = static_cast<int>(static_cast<int64_t>(c + 1) * tiles_req / a.chunks);
  const int nt = min(t1 - t0, kMaxChunkTiles);
  const int64_t base = static_cast<int64_t>(t0) * kTileM;  // first key of the chunk
  const int nloc = static_cast<int>(max(int64_t(0), min(n, static_cast<int64_t>(t0 + nt) * kTileM) - base));

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kEmptyCount);
    }
    for (int b = 0; b < kNAcc; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(qbar, 1);
    mbar_init(mdone, 1);
    sh.fail = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < 2 * kHistBins; i += kThreads) ghist0[i] = 0;
  __syncthreads();

  // ================= phase 1: stream the keys, scores into TMEM =================
  if (warp == 0) {
    if (lane == 0) {
      // the query first, so that it is not queued behind the key stream
      mbar_arrive_expect_tx(qbar, kHeads * kDI * 2);
      bulk_load(smem + C::oQ, a.q_idx + static_cast<int64_t>(r) * kHeads * kDI, kHeads * kDI * 2, qbar);
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % C::kStages;
        const uint32_t ph = (t / C::kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, kWaitLimit)) {
          atomicOr(&g_index_tc_error, 1u);
          sh.fail = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[s], C::kStageBytes + C::kScaleBytes);
        const int64_t row0 = static_cast<int64_t>(t0 + t) * kTileM;
        const int y = static_cast<int>(r * a.cap + row0);
        uint8_t* dst = smem + C::oStages + s * C::kStageBytes;
        tma_load_2d(dst, &kmap, &full[s], 0, y);
        if constexpr (FP8) {
          tma_load_2d(smem + C::oScales + s * C::kScaleBytes, &smap, &full[s], static_cast<int>(row0), r);
        } else {
          tma_load_2d(dst + 16384, &kmap, &full[s], 64, y);
        }
        issued = t + 1;
      }
      if (sh.fail)  // let the copies still in flight land before the CTA winds down
        for (int t = max(0, issued - C::kStages); t < issued; ++t)
          mbar_wait(&full[t % C::kStages], (t / C::kStages) & 1, kWaitLimit);
    }
  } else {
    // warps 1..: TMEM, head weights, query operand
    const int ptid = tid - 32;
    if (warp == 1) tmem_alloc(&sh.tmem_base, kTmemCols);
    if (ptid < kHeads) ws[ptid] = __ldg(a.w + static_cast<int64_t>(r) * kHeads + ptid);
    const bool qok = __all_sync(0xFFFFFFFFu, mbar_wait(qbar, 0, kWaitLimit));
    if (!qok) {
      atomicOr(&g_index_tc_error, 1u);
      sh.fail = 1;
    }
    const uint4* q4 = reinterpret_cast<const uint4*>(smem + C::oQ);
    if constexpr (FP8) {
      float m = 0.f;
      for (int i = ptid; i < kHeads * kDI / 8; i += kPrep) {
        const uint4 u = q4[i];
        const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          m = fmaxf(m, fabsf(__uint_as_float(wds[e] << 16)));
          m = fmaxf(m, fabsf(__uint_as_float(wds[e] & 0xFFFF0000u)));
        }
      }
      m = warp_max(m);
      if (lane == 0) sh.qmax[warp - 1] = __float_as_uint(m);
      named_barrier(2, kPrep);
      m = 0.f;
      for (int i = 0; i < kPrep / 32; ++i) m = fmaxf(m, __uint_as_float(sh.qmax[i]));
      int e = 0;
      if (m > 0.f) {
        frexpf(m, &e);        // m = f 2^e, f in [0.5, 1)
        e = min(8 - e, 126);  // m 2^e in [128, 256)
      }
      const float S = ldexpf(1.f, e);
      if (ptid == 0) sh.qinv = ldexpf(1.f, -e);
      for (int task = ptid; task < kHeads * 8; task += kPrep) {
        const int h = task >> 3, ch = task & 7;
        const uint4 u0 = q4[(h * kDI + ch * 16) / 8], u1 = q4[(h * kDI + ch * 16) / 8 + 1];
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
      if (ptid == 0) sh.qinv = 1.f;
      for (int task = ptid; task < 2 * kHeads * 8; task += kPrep) {
        const int half = task / (kHeads * 8), h = (task / 8) % kHeads, ch = task & 7;
        *reinterpret_cast<uint4*>(Bs + half * 8192 + sw128_offset(h, ch)) = q4[(h * kDI + half * 64 + ch * 8) / 8];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_barrier(1, kPrep);
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    if (warp == 1) {
      // MMA issuer
      if (lane == 0 && !sh.fail) {
        const uint32_t b_base = smem_u32(Bs);
        for (int t = 0; t < nt; ++t) {
          const int s = t % C::kStages;
          const uint32_t ph = (t / C::kStages) & 1;
          const int acc = t % kNAcc;
          const uint32_t aph = (t / kNAcc) & 1;
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
        // every MMA of this CTA has completed before TMEM is read back or released
        mma_commit(mdone);
        mbar_wait(mdone, 0, kWaitLimit);
      }
    } else if (!sh.fail) {
      // epilogue: two groups of four warps take alternate tiles; warp w owns
      // TMEM lanes 32 (w % 4) .. +31
      const int grp = (warp - 2) >> 2;
      const int sub = warp & 3;
      const int row = sub * 32 + lane;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(sub * 32) << 16);
      const float qinv = sh.qinv;
      uint32_t* hist = ghist0 + grp * kHistBins;
      float w_r[kHeads];
#pragma unroll
      for (int h = 0; h < kHeads; ++h) w_r[h] = ws[h];
      for (int t = grp; t < nt; t += 2) {
        const int acc = t % kNAcc;
        const uint32_t aph = (t / kNAcc) & 1;
        // the whole warp takes the same branch (warp-wide TMEM ops below)
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], aph, kWaitLimit))) {
          atomicOr(&g_index_tc_error, 1u);
          sh.fail = 1;
          break;
        }
        tc_fence_after();
        float ks = 1.f;
        if constexpr (FP8) {
          const int s = t % C::kStages;
          mbar_wait(&full[s], (t / C::kStages) & 1, kWaitLimit);  // complete: makes the scales visible
          ks = scale_ring[s * kTileM + row] * qinv;
          mbar_arrive(&empty[s]);
        }
        uint32_t v0[32], v1[32];
        tmem_ld32(lane_addr + acc * kHeads, v0);
        tmem_ld32(lane_addr + acc * kHeads + 32, v1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
        for (int h = 0; h < 32; h += 2) {
          s0 = fmaf(w_r[h], fmaxf(__uint_as_float(v0[h]), 0.f), s0);
          s1 = fmaf(w_r[h + 1], fmaxf(__uint_as_float(v0[h + 1]), 0.f), s1);
          s2 = fmaf(w_r[32 + h], fmaxf(__uint_as_float(v1[h]), 0.f), s2);
          s3 = fmaf(w_r[33 + h], fmaxf(__uint_as_float(v1[h + 1]), 0.f), s3);
        }
        const float sc = ((s0 + s1) + (s2 + s3)) * ks;
        tmem_st1(lane_addr + kScoreCol + t, __float_as_uint(sc));
        if (static_cast<int64_t>(t0 + t) * kTileM + row < n) atomicAdd(&hist[score_key(sc) >> 20], 1u);
      }
      tmem_wait_st();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (!sh.fail) {
    // ================= phase 2: exact top-k over the request =================
    const int k = a.k;
    int32_t* oi = a.out_idx + static_cast<int64_t>(r) * k;
    float* os = a.out_score ? a.out_score + static_cast<int64_t>(r) * k : nullptr;
    uint8_t* p2 = smem + C::oStages;  // the stage ring is idle now
    uint32_t* hist = reinterpret_cast<uint32_t*>(p2 + C::pHist);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(p2 + C::pScratch);
    uint32_t* cpre = reinterpret_cast<uint32_t*>(p2 + C::pCpre);
    uint32_t* cntA = reinterpret_cast<uint32_t*>(p2 + C::pCntA);
    uint32_t* cntE = reinterpret_cast<uint32_t*>(p2 + C::pCntE);
    uint32_t* offA = reinterpret_cast<uint32_t*>(p2 + C::pOffA);
    uint32_t* offE = reinterpret_cast<uint32_t*>(p2 + C::pOffE);
    int32_t* eq_cache_i = reinterpret_cast<int32_t*>(p2 + C::pEq);
    float* eq_cache_s = reinterpret_cast<float*>(eq_cache_i + kEqCache);
    uint32_t* gh_g = ghist0;  // the two group histograms
    // TMEM readers in phase 2: the four warps 2..5 (one per lane quarter)
    const bool rd = warp >= 2 && warp < 6;
    const int sub = warp & 3;
    const uint32_t score_addr = tmem + (static_cast<uint32_t>(sub * 32) << 16) + kScoreCol;
    auto local_of = [&](int t) { return t * kTileM + sub * 32 + lane; };

    if (n <= k) {
      if (rd)
        for (int tb = 0; tb < nt; tb += 32) {
          uint32_t v[32];
          tmem_ld32(score_addr + tb, v);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int t = tb + u, loc = local_of(t);
            if (t < nt && loc < nloc) {
              oi[base + loc] = static_cast<int32_t>(base + loc);
              if (os) os[base + loc] = __uint_as_float(v[u]);
            }
          }
        }
      if (c == 0)
        for (int64_t j = n + tid; j < k; j += kThreads) {
          oi[j] = -1;
          if (os) os[j] = -INFINITY;
        }
    } else {
      uint32_t* gh1 = a.ghist + static_cast<int64_t>(r) * 2 * kHistBins;
      uint32_t* gh2 = gh1 + kHistBins;
      uint32_t* bar = a.sync + r * 4;
      // pass 1 (bits 31..20): built while streaming
      for (int i = tid; i < kHistBins; i += kThreads) {
        const uint32_t v = gh_g[i] + gh_g[kHistBins + i];
        if (v) atomicAdd(&gh1[i], v);
      }
      bool alive = request_barrier(&bar[0], a.chunks, sh);
      uint32_t shift = 20, prefix = 0, need = 0;
      if (alive) {
        for (int i = tid; i < kHistBins / 4; i += kThreads)
          reinterpret_cast<uint4*>(hist)[i] = __ldcg(reinterpret_cast<const uint4*>(gh1) + i);
        __syncthreads();
        find_bin_block(hist, static_cast<uint32_t>(k), sh, scratch);
        prefix = sh.bcast[0];
        need = static_cast<uint32_t>(k) - sh.bcast[1];
        if (hist[prefix] > static_cast<uint32_t>(kEqCache)) {
          // a crowded boundary bin: one more distributed pass (bits 19..8)
          for (int i = tid; i < 2 * kHistBins; i += kThreads) gh_g[i] = 0;
          __syncthreads();
          if (rd)
            for (int tb = 0; tb < nt; tb += 32) {
              uint32_t v[32];
              tmem_ld32(score_addr + tb, v);
              tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const uint32_t key = score_key(__uint_as_float(v[u]));
                if (tb + u < nt && local_of(tb + u) < nloc && (key >> 20) == prefix)
                  atomicAdd(&gh_g[(key >> 8) & 0xFFFu], 1u);
              }
            }
          __syncthreads();
          for (int i = tid; i < kHistBins; i += kThreads)
            if (gh_g[i]) atomicAdd(&gh2[i], gh_g[i]);
          alive = request_barrier(&bar[0], 2u * a.chunks, sh);
          if (alive) {
            for (int i = tid; i < kHistBins / 4; i += kThreads)
              reinterpret_cast<uint4*>(hist)[i] = __ldcg(reinterpret_cast<const uint4*>(gh2) + i);
            __syncthreads();
            find_bin_block(hist, need, sh, scratch);
            prefix = (prefix << 12) | sh.bcast[0];
            need -= sh.bcast[1];
            shift = 8;
          }
        }
      }
      if (alive) {
        // stage this chunk's keys above the boundary prefix and at it, in
        // index order: per (tile, quarter) counts, prefix sums, then writes
        const int64_t slot = static_cast<int64_t>(r) * a.chunks + c;
        int32_t* sti = a.st_idx + slot * k;
        float* sts = a.st_score + slot * k;
        int32_t* eqi = a.eq_idx + slot * (kMaxChunkTiles * kTileM);
        float* eqs = a.eq_score + slot * (kMaxChunkTiles * kTileM);
        for (int pass = 0; pass < 2; ++pass) {
          if (rd)
            for (int tb = 0; tb < nt; tb += 32) {
              uint32_t v[32];
              tmem_ld32(score_addr + tb, v);
              tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 32; ++u) {
                const int t = tb + u;
                const int loc = local_of(t);
                const bool valid = t < nt && loc < nloc;
                const float sv = __uint_as_float(v[u]);
                const uint32_t kp = score_key(sv) >> shift;
                const bool above = valid && kp > prefix, eq = valid && kp == prefix;
                const uint32_t ba = __ballot_sync(0xFFFFFFFFu, above), be = __ballot_sync(0xFFFFFFFFu, eq);
                if (t < nt) {
                  if (pass == 0) {
                    if (lane == 0) {
                      cntA[t * 4 + sub] = __popc(ba);
                      cntE[t * 4 + sub] = __popc(be);
                    }
                  } else {
                    const uint32_t lm = (1u << lane) - 1u;
                    if (above) {
                      const uint32_t pos = offA[t * 4 + sub] + __popc(ba & lm);
                      if (pos < static_cast<uint32_t>(k)) {
                        sti[pos] = static_cast<int32_t>(base + loc);
                        sts[pos] = sv;
                      }
                    }
                    if (eq) {
                      const uint32_t pos = offE[t * 4 + sub] + __popc(be & lm);
                      eqi[pos] = static_cast<int32_t>(base + loc);
                      eqs[pos] = sv;
                    }
                  }
                }
              }
            }
          __syncthreads();
          if (pass == 0) {
            if (warp == 0) {
              const uint32_t ta = warp_exclusive_scan(cntA, offA, nt * 4);
              const uint32_t te = warp_exclusive_scan(cntE, offE, nt * 4);
              if (lane == 0) {
                sh.bcast[5] = ta;
                sh.bcast[6] = te;
              }
            }
            __syncthreads();
          }
        }
        if (tid == 0) {
          a.cnt[slot * 2] = sh.bcast[5];
          a.cnt[slot * 2 + 1] = sh.bcast[6];
          __threadfence();
          const uint32_t prev = atomicAdd(&bar[1], 1u);
          sh.bcast[2] = (prev == static_cast<uint32_t>(a.chunks) - 1) ? 1u : 0u;
        }
        __syncthreads();
        if (sh.bcast[2]) {
          // ---------- last CTA of the request: assemble in chunk (= index) order ----------
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
          const uint32_t take = min(need, static_cast<uint32_t>(k) - A);
          if (E <= take) {
            for (uint32_t i = tid; i < E; i += kThreads) {
              const int cc = chunk_of(cpre + 160, i);
              const int64_t src = (static_cast<int64_t>(r) * nch + cc) * eq_stride + (i - cpre[160 + cc]);
              oi[A + i] = __ldcg(a.eq_idx + src);
              if (os) os[A + i] = __ldcg(a.eq_score + src);
            }
          } else {
            // more boundary entries than places left: radix passes over the
            // low `shift` bits of their keys, then the lowest indices
            // (entries are in index order)
            const uint32_t ncache = min(E, static_cast<uint32_t>(kEqCache));
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
            uint32_t pfx = prefix, rb = shift, tk = take;
            while (rb > 0) {
              const uint32_t nb = rb > 12 ? 12 : rb;
              const uint32_t sft = rb - nb;
              for (int i = tid; i < kHistBins; i += kThreads) hist[i] = 0;
              __syncthreads();
              for (uint32_t i = tid; i < E; i += kThreads) {
                int32_t j;
                float v;
                eq_at(i, j, v);
                const uint32_t key = score_key(v);
                if ((key >> rb) == pfx) atomicAdd(&hist[(key >> sft) & ((1u << nb) - 1u)], 1u);
              }
              __syncthreads();
              find_bin_block(hist, tk, sh, scratch);
              pfx = (pfx << nb) | sh.bcast[0];
              tk -= sh.bcast[1];
              rb = sft;
            }
            // every boundary entry with key > T, then the first tk equal to T
            const uint32_t T = pfx, take_eq = tk;
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
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
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
  if (k_dtype == kFP8 && cap % 4 != 0) return false;  // row-scale tiles: 16-byte row stride
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

  // FP8 row scales as a [batch][cap] fp32 tensor, one 128-wide box per tile
  CUtensorMap smap;
  memset(&smap, 0, sizeof(smap));
  if (fp8) {
    const cuuint64_t sdims[2] = {static_cast<cuuint64_t>(cap), static_cast<cuuint64_t>(batch)};
    const cuuint64_t sstrides[1] = {static_cast<cuuint64_t>(cap) * 4};
    const cuuint32_t sbox[2] = {static_cast<cuuint32_t>(kTileM), 1};
    cr = L.encode(&smap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, k_idx->scale, sdims, sstrides, sbox, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS)
      return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", static_cast<int>(cr));
  }

  IdxArgs a;
  a.q_idx = static_cast<const uint16_t*>(q_idx->data);
  a.w = w;
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
  cudaError_t e = fp8 ? cudaLaunchKernelEx(&cfg, index_topk_tc_kernel<true>, map, smap, a)
                      : cudaLaunchKernelEx(&cfg, index_topk_tc_kernel<false>, map, smap, a);
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
