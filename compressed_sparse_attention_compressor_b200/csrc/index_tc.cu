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
//              into a ring of shared-memory stages (FP8: one 256-row box =
//              two tiles per stage);
//   warp 1     MMA issuer: D[128 keys][N] (fp32, TMEM, two accumulators of
//              128 columns, tiles taken in pairs) = keys x q^T with
//              tcgen05.mma, M = 128; N = 128 for FP8 keys (both E4M3 terms
//              of the split query, 64 heads each), N = 64 for bf16 keys;
//   warps 2-9  epilogue, two groups of four warps on alternate tiles of a
//              pair: TMEM -> registers, s = sum_h w_h ReLU(D_h) (FP8: the
//              two query terms summed first), one score per key written
//              back to a TMEM column and counted in the key histogram.
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
// of a request.  The histogram of key bits 31..20 is built while the keys
// stream; each CTA adds it into a global per-request histogram, and after a
// bounded per-request grid barrier every CTA finds the boundary bin (a
// crowded bin takes one more distributed level, bits 19..8).  Each CTA then
// classifies its scores once: entries above the boundary prefix stay in its
// shared memory, entries at the prefix are published to global memory, both
// lists in index order; the per-chunk counts are exchanged at a second
// barrier.  From the chunk prefix sums every CTA writes its own entries
// above the boundary straight to their output slots, loads the request's
// boundary entries (a few thousand) into shared memory, resolves the
// remaining key bits with shared-memory radix levels -- all CTAs reach the
// same threshold key T and count -- and writes its own selected boundary
// entries.  The output is deterministic: entries above the boundary in
// index order, then the selected boundary entries in index order.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "pool.cuh"
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
constexpr int kNAcc = 4;                         // accumulators: two pair slots x one per epilogue group
constexpr int kAccCols = 128;                    // TMEM columns per accumulator
constexpr int kMaxChunkTiles = 224;              // tiles of one CTA (TMEM columns, shared-memory scores)
constexpr int kTmemCols = 512;
constexpr int kHistBins = 4096;
constexpr int kEqCache = 8192;                   // boundary entries resolved in shared memory
constexpr int kACache = 2048;                    // entries above the boundary kept in shared memory
constexpr int kMaxChunks = 148;                  // CTAs of one request (<= SMs)
constexpr int kSStages = 16;                     // FP8 row-scale ring (one 512-byte tile each)
constexpr int kAppendShrink = 26;                // tiles the appending CTA's chunk gives up
constexpr uint32_t kWaitLimit = 1u << 22;        // mbarrier polls
constexpr uint32_t kSpinLimit = 1u << 22;        // grid-barrier polls (~64 ns apart)
static_assert(kNAcc * kAccCols <= kTmemCols, "TMEM columns");

__device__ uint32_t g_index_tc_error = 0;  // bit 0: a bounded wait gave up

template <bool FP8>
struct Cfg {
  // one TMA stage = 32 KB: two FP8 key tiles (one 256-row box) or one bf16 tile
  static constexpr int kTPS = FP8 ? 2 : 1;
  static constexpr int kStageBytes = 32768;
  static constexpr int kStages = 5;
  static constexpr int oStages = 0;
  static constexpr int oScales = kStages * kStageBytes;                 // FP8: [kSStages][128] fp32
  static constexpr int oB = oScales + (FP8 ? kSStages * kTileM * 4 : 0);
  static constexpr int oHist = oB + 16384;          // two group histograms; the raw query before them
  static constexpr int oQ = oHist;
  static constexpr int oW = oHist + 2 * kHistBins * 4;
  static constexpr int oBars = oW + kHeads * 4;
  static constexpr int oMisc = oBars + 512;
  static constexpr int kSmem = oMisc + 256 + 1024;
  // FP8: N = 128 = both E4M3 terms of the split query (rows 0..63 and 64..127 of B)
  static constexpr uint32_t kIdesc = FP8 ? idesc(0, 0, kTileM, 2 * kHeads) : idesc(1, 1, kTileM, kHeads);
  static_assert(sizeof(uint64_t) * (2 * kStages + 2 * kSStages + 8) <= 512, "mbarrier area");
  static_assert(oB % 1024 == 0, "operand alignment");
  static_assert(kSmem <= 232448, "shared memory");
  // phase-2 scratch, inside the (then idle) stage and scale rings
  static constexpr int pHist = 0;                              // [kHistBins] histogram
  static constexpr int pScratch = pHist + kHistBins * 4;       // 512 words
  static constexpr int pCpre = pScratch + 2048;                // [2][kMaxChunks + 4] chunk prefixes
  static constexpr int pACache = pCpre + 2 * (kMaxChunks + 4) * 4;   // this chunk's entries above the boundary
  static constexpr int pScores = pACache + kACache * 8;        // this chunk's scores, index order
  static constexpr int pEq = pScores;                          // later: the request's boundary entries
  static_assert(pScores + kMaxChunkTiles * kTileM * 4 <= oB, "phase-2 scores must fit in the rings");
  static_assert(pEq + kEqCache * 8 <= oB, "phase-2 boundary list must fit in the rings");
  static_assert(pACache % 16 == 0 && pScores % 16 == 0, "phase-2 alignment");
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
  uint32_t* sync;          // [batch][4]        (zero on entry): barrier counter
  uint32_t* cnt;           // [batch][chunks][2] entries above / at the boundary per chunk
  uint2* st;               // [batch][chunks][k] (index, score bits) above the boundary, beyond kACache
  uint2* eq;               // [batch][chunks][kMaxChunkTiles * 128] (index, score bits) at the boundary
  float* scg;              // [batch][chunks][kMaxChunkTiles * 128] the chunk's scores, tile by tile
  int append;              // 1: n = (pos + 1) / m and the last chunk's CTA appends the token
  AppendArgs ap;
  float* bmax;             // optional [batch][ldb]: max score of each block of `block` entries
  int64_t ldb;
  int block;               // power of two <= kTileM, so no block straddles two chunks
  // candidate-pool mode: position j of request r is entry
  // pool[r][j / pblock] * pblock + j % pblock; the keys come in pblock-row boxes
  const int32_t* pool;     // [batch][pool_blocks] ascending block ids, -1 padded (or null)
  int pool_blocks;
  int pblock;              // 8 .. 128, a power of two
  const float* kscale;     // FP8 row scales [batch][cap] (pool mode)
  uint32_t spin_limit;     // grid-barrier polls before a wait gives up (kSpinLimit)
  int skip_arrive;         // CTA that does not arrive at the first barrier (-1: none; test hook)
};

struct Shared {
  uint32_t tmem_base;
  uint32_t bcast[8];
  uint32_t qmax[kThreads / 32];
  float qinv;
  int fail;
  int red[kThreads / 32];
};

// Candidate-pool mode: the positions of request r that hold visible
// entries.  The pool's valid slots (block id >= 0, block start < n_vis) form
// its leading run when the pool ascends with -1 padding at the end; the run
// ends at the first other slot, and the positions are the entries of the
// run's blocks, the last of which may be partial.  Called by every thread.
__device__ int64_t pool_positions(const IdxArgs& a, int r, Shared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* prow = a.pool + static_cast<int64_t>(r) * a.pool_blocks;
  const int64_t nv = min(max(static_cast<int64_t>(a.n_visible[r]), int64_t(0)), a.cap);
  const int bs = a.pblock;
  int first_bad = a.pool_blocks;
  for (int q = tid; q < a.pool_blocks; q += kThreads) {
    const int32_t b = __ldg(prow + q);
    if (b < 0 || static_cast<int64_t>(b) * bs >= nv) {
      first_bad = q;
      break;
    }
  }
  first_bad = static_cast<int>(__reduce_min_sync(0xFFFFFFFFu, static_cast<uint32_t>(first_bad)));
  if (lane == 0) sh.red[warp] = first_bad;
  __syncthreads();
  int end = a.pool_blocks;
  for (int w2 = 0; w2 < kThreads / 32; ++w2) end = min(end, sh.red[w2]);
  __syncthreads();
  uint32_t cnt = 0;
  for (int q = tid; q < end; q += kThreads)
    cnt += static_cast<uint32_t>(min(static_cast<int64_t>(bs), nv - static_cast<int64_t>(__ldg(prow + q)) * bs));
  cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
  if (lane == 0) sh.red[warp] = static_cast<int>(cnt);
  __syncthreads();
  int64_t np = 0;
  for (int w2 = 0; w2 < kThreads / 32; ++w2) np += sh.red[w2];
  __syncthreads();
  return np;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Bounded per-request grid barrier in two halves, so that local work can
// run between the arrival and the wait.  request_arrive: the CTA's earlier
// writes, then one arrival.  request_wait: until `target` arrivals; false on
// a timeout.
// `skip`: this CTA does not arrive (the test hook that makes the request's
// waits run out; false in every normal launch).
__device__ void request_arrive(uint32_t* ctr, bool skip) {
  __syncthreads();
  if (threadIdx.x == 0 && !skip) {
    __threadfence();
    atomicAdd(ctr, 1u);
  }
}

__device__ bool request_wait(uint32_t* ctr, uint32_t target, uint32_t limit, Shared& sh) {
  if (threadIdx.x == 0) {
    int ok = 1;
    uint32_t it = 0;
    while (ld_acquire_gpu(ctr) < target) {
      if (++it > limit) {
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

// Bounded per-request grid barrier; returns false on timeout.
__device__ bool request_barrier(uint32_t* ctr, uint32_t target, uint32_t limit, Shared& sh) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(ctr, 1u);
    uint32_t it = 0;
    while (ld_acquire_gpu(ctr) < target) {
      if (++it > limit) {
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

// Whole block: bin b of a shared-memory histogram of `nbins` bins (a power
// of two, 256..kHistBins), scanned from the top, with
// above(b) < need <= above(b) + hist[b]; writes (b, above, hist[b]) to
// bcast[0..2].
// Threads 0..255 own nbins / 256 consecutive bins each (read at once, kept
// in registers); a suffix scan over the lanes and the eight warps' totals
// gives each thread the entries above its bins.
__device__ void find_bin_block(const uint32_t* hist, int nbins, uint32_t need, Shared& sh, uint32_t* scratch) {
  constexpr int kT = 256, kMaxPer = kHistBins / kT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins / kT;  // 1, 4 or 16
  // a histogram that holds fewer than `need` entries (never produced by the
  // kernel: the counts add up to the visible entries) selects bin 0
  if (tid == 0) {
    sh.bcast[0] = 0;
    sh.bcast[1] = 0;
    sh.bcast[2] = 0;
  }
  uint32_t c[kMaxPer];
  uint32_t mine = 0;
  if (tid < kT) {
    if (per >= 4) {
#pragma unroll
      for (int i = 0; i < kMaxPer; i += 4)
        if (i < per) {
          const uint4 v = *reinterpret_cast<const uint4*>(hist + tid * per + i);
          c[i] = v.x; c[i + 1] = v.y; c[i + 2] = v.z; c[i + 3] = v.w;
        }
    } else {
      c[0] = hist[tid];
    }
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i)
      if (i < per) mine += c[i];
  }
  uint32_t incl = mine;  // this thread's bins and those of the lanes above it
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += x;
  }
  if (tid < kT && lane == 0) scratch[warp] = incl;
  __syncthreads();
  if (tid < kT) {
    uint32_t above = incl - mine;
    for (int w = warp + 1; w < kT / 32; ++w) above += scratch[w];
    if (above < need && need <= above + mine) {
#pragma unroll
      for (int i = kMaxPer - 1; i >= 0; --i) {
        if (i >= per) continue;
        if (above + c[i] >= need) {
          sh.bcast[0] = tid * per + i;
          sh.bcast[1] = above;
          sh.bcast[2] = c[i];
          break;
        }
        above += c[i];
      }
    }
  }
  __syncthreads();
}

// Whole block: exclusive prefix sums over the block (thread order) of two
// per-thread counts, and their totals.  scratch: 2 * warps words.
__device__ __forceinline__ void block_scan2(uint32_t a, uint32_t b, uint32_t& oa, uint32_t& ob, uint32_t& ta,
                                            uint32_t& tb, uint32_t* scratch) {
  constexpr int W = kThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t xa = __shfl_up_sync(0xFFFFFFFFu, ia, o), xb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
    if (lane >= o) {
      ia += xa;
      ib += xb;
    }
  }
  if (lane == 31) {
    scratch[warp] = ia;
    scratch[W + warp] = ib;
  }
  __syncthreads();
  uint32_t pa = 0, pb = 0, sa = 0, sb = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const uint32_t x = scratch[w], y = scratch[W + w];
    if (w < warp) {
      pa += x;
      pb += y;
    }
    sa += x;
    sb += y;
  }
  oa = pa + ia - a;
  ob = pb + ib - b;
  ta = sa;
  tb = sb;
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

// Whole block: a global histogram of kHistBins words into shared memory,
// every load issued before the first store.
__device__ __forceinline__ void load_hist(uint32_t* dst, const uint32_t* src) {
  constexpr int N4 = kHistBins / 4, R = (N4 + kThreads - 1) / kThreads;
  uint4 v[R];
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const int i = threadIdx.x + j * kThreads;
    if (i < N4) v[j] = __ldcg(reinterpret_cast<const uint4*>(src) + i);
  }
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const int i = threadIdx.x + j * kThreads;
    if (i < N4) reinterpret_cast<uint4*>(dst)[i] = v[j];
  }
}

// Whole block: sum of two per-thread counts over the block (scratch: 2 * warps words).
__device__ __forceinline__ void block_sum2(uint32_t& a, uint32_t& b, uint32_t* scratch) {
  constexpr int W = kThreads / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
    b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
  }
  if ((threadIdx.x & 31) == 0) {
    scratch[threadIdx.x >> 5] = a;
    scratch[W + (threadIdx.x >> 5)] = b;
  }
  __syncthreads();
  a = 0;
  b = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    a += scratch[w];
    b += scratch[W + w];
  }
  __syncthreads();
}

// All threads of one CTA: the decode-step append of request r.  wbuf: room
// for W_IK (d x 128, 16-aligned; the idle stage ring); scratch: d + 256
// floats; wbar: an initialised mbarrier.  The stores are visible to this
// CTA's later TMA loads (and to every later kernel) when it returns.
template <bool KV_MX4>
__device__ void append_block(const AppendArgs& p, int r, int64_t cap, uint8_t* wbuf, float* scratch,
                             uint64_t* wbar, Shared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d, m = p.m;
  const int64_t t = p.pos[r];
  const bool closes = (t + 1) % m == 0;
  const int wbytes = d * kDI * elem_bytes(p.w_dtype);
  if (closes && tid == 0) {  // W_IK by bulk copies, in flight while the block is pooled
    mbar_arrive_expect_tx(wbar, wbytes);
    for (int off = 0; off < wbytes; off += 32768)
      bulk_load(wbuf + off, static_cast<const uint8_t*>(p.w_ik) + off, min(32768, wbytes - off), wbar);
  }
  const int ea = elem_bytes(p.act_dtype), es = elem_bytes(p.swa_dtype);
  const int vecs = d / 8;
  const int slot_m = static_cast<int>(t % m);
  const int64_t slot_w = t % p.swa_cap;
  const char* crow = static_cast<const char*>(p.c_t) + static_cast<int64_t>(r) * d * ea;
  const char* zrow = static_cast<const char*>(p.z_t) + static_cast<int64_t>(r) * d * ea;
  char* ocb = static_cast<char*>(p.open_c) + static_cast<int64_t>(r) * m * d * ea;
  char* ozb = static_cast<char*>(p.open_z) + static_cast<int64_t>(r) * m * d * ea;
  // the token's rows into their slots: SWA key / value, open-block C / Z
  for (int task = tid; task < 4 * vecs; task += kThreads) {
    const int row = task / vecs, col = (task % vecs) * 8;
    float v[8];
    const char* src = row == 0 ? static_cast<const char*>(p.k_t) + static_cast<int64_t>(r) * d * ea
                    : row == 1 ? static_cast<const char*>(p.v_t) + static_cast<int64_t>(r) * d * ea
                    : row == 2 ? crow : zrow;
    load8(src, p.act_dtype, col, nullptr, 1, v);
    char* dst = row == 0 ? static_cast<char*>(p.swa_k) + (static_cast<int64_t>(r) * p.swa_cap + slot_w) * d * es
              : row == 1 ? static_cast<char*>(p.swa_v) + (static_cast<int64_t>(r) * p.swa_cap + slot_w) * d * es
              : (row == 2 ? ocb : ozb) + static_cast<int64_t>(slot_m) * d * ea;
    store8(dst, row < 2 ? p.swa_dtype : p.act_dtype, col, v);
  }
  if (tid == 0) {
    p.n_vis_out[r] = static_cast<int32_t>((t + 1) / m);
    p.q_pos_out[r] = t;
    p.q_req_out[r] = r;
  }
  if (closes) {  // uniform over the CTA
    const int64_t row = static_cast<int64_t>(r) * cap + (t + 1) / m - 1;
    float* pooled = scratch;  // [d]
    float* red = scratch + d;  // [2][128]
    // every thread of a warp pools 8 channels (FP8: 8 lanes = one 64-channel scale group)
    const int nvt = (vecs + 31) / 32 * 32;
    for (int vec = tid; vec < nvt; vec += kThreads) {  // warp-uniform trip count
      const bool valid = vec < vecs;
      const int col = valid ? vec * 8 : 0;
      float v[8];
      if (valid) {
        auto rowC = [&](int i) -> const char* { return i == slot_m ? crow : ocb + static_cast<int64_t>(i) * d * ea; };
        auto rowZ = [&](int i) -> const char* { return i == slot_m ? zrow : ozb + static_cast<int64_t>(i) * d * ea; };
        pool8(rowC, rowZ, p.act_dtype, m, col, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) pooled[col + e] = v[e];
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = 0.f;
      }
      store_pooled8<KV_MX4>(p.kv, row, col, v, valid);
    }
    // indexer key = pooled . W_IK (fp32 pooled row, before storage rounding):
    // thread (j, half) sums half of the d channels of output j
    if (tid == 0 && !mbar_wait(wbar, 0, kWaitLimit)) {
      atomicOr(&g_index_tc_error, 1u);
      sh.fail = 1;
    }
    __syncthreads();  // pooled row complete; W_IK landed (or the wait gave up)
    const bool wok = !sh.fail;
    if (tid < 2 * kDI) {
      const int j = tid & (kDI - 1), half = tid / kDI;
      const int c0 = half * (d / 2), c1 = c0 + d / 2;
      float acc = 0.f;
      if (wok) {
        if (p.w_dtype == kBF16) {
          const uint16_t* w = reinterpret_cast<const uint16_t*>(wbuf) + j;
          for (int c = c0; c < c1; ++c) acc = fmaf(pooled[c], bf16_bits_to_f32(w[c * kDI]), acc);
        } else {
          const float* w = reinterpret_cast<const float*>(wbuf) + j;
          for (int c = c0; c < c1; ++c) acc = fmaf(pooled[c], w[c * kDI], acc);
        }
      }
      red[half * kDI + j] = acc;
    }
    __syncthreads();
    float key = 0.f;
    if (tid < kDI) key = red[tid] + red[kDI + tid];
    if (wok) {
      if (p.kidx.dtype == kFP8) {
        float a = tid < kDI ? fabsf(key) : 0.f;
        a = warp_max(a);
        if (lane == 0 && warp < kDI / 32) red[2 * kDI + warp] = a;
        __syncthreads();
        float amax = 0.f;
#pragma unroll
        for (int w = 0; w < kDI / 32; ++w) amax = fmaxf(amax, red[2 * kDI + w]);
        const float sc = amax > 0.f ? amax / 448.f : 1.f;
        if (tid < kDI) static_cast<uint8_t*>(p.kidx.data)[row * p.kidx.row_stride + tid] = f32_to_e4m3(key / sc);
        if (tid == 0) static_cast<float*>(p.kidx.scale)[row * p.kidx.scale_stride] = sc;
      } else if (tid < kDI) {
        if (p.kidx.dtype == kBF16) static_cast<uint16_t*>(p.kidx.data)[row * p.kidx.row_stride + tid] = f32_to_bf16_bits(key);
        else static_cast<float*>(p.kidx.data)[row * p.kidx.row_stride + tid] = key;
      }
    }
  }
  // the generic-proxy stores above, before this CTA's TMA (async-proxy) loads
  // of the same rows; W_IK's shared memory, before TMA writes it again
  asm volatile("fence.proxy.async.global;" ::: "memory");
  fence_proxy_async_smem();
  __threadfence();
  __syncthreads();
}

// Launch modes.  Each is its own instantiation, so that a launch carries
// only its own code: every CTA fetches the kernel's instructions cold.
constexpr int kModePlain = 0;      // top-k of the visible entries
constexpr int kModeBmax = 1;       // ... and the block maxima (a.bmax)
constexpr int kModePool = 2;       // top-k inside a candidate pool (a.pool)
constexpr int kModeAppend = 3;     // decode step: append the token first (a.ap), main KV not MXFP4
constexpr int kModeAppendMx4 = 4;  // ... main KV in MXFP4
constexpr int kModes = 5;

template <bool FP8, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
index_topk_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap smap,
                     IdxArgs a) {
  using C = Cfg<FP8>;
  constexpr bool POOL = MODE == kModePool, BMAX = MODE == kModeBmax;
  constexpr bool APPEND = MODE == kModeAppend || MODE == kModeAppendMx4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Shared& sh = *reinterpret_cast<Shared*>(smem + C::oMisc);
  uint32_t* ghist0 = reinterpret_cast<uint32_t*>(smem + C::oHist);  // group 0; group 1 follows
  float* ws = reinterpret_cast<float*>(smem + C::oW);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::oBars);
  uint64_t* empty = full + C::kStages;
  uint64_t* sfull = empty + C::kStages;
  uint64_t* sempty = sfull + kSStages;
  uint64_t* tfull = sempty + kSStages;  // [2] pair slot s: its two tiles' accumulators are ready
  uint64_t* tempty = tfull + 2;          // [2] ... and have been read back
  uint64_t* qbar = tempty + 2;
  uint64_t* mdone = qbar + 1;
  uint64_t* abar = mdone + 1;  // W_IK of the in-kernel append
  uint64_t* cbar = abar + 1;   // the chunk's scores, workspace -> shared memory (phase 2)
  uint8_t* Bs = smem + C::oB;
  const float* scale_ring = reinterpret_cast<const float*>(smem + C::oScales);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x / a.chunks, c = blockIdx.x % a.chunks;
  int64_t n_raw;
  if constexpr (POOL)
    n_raw = pool_positions(a, r, sh);
  else
    n_raw = APPEND ? (a.ap.pos[r] + 1) / a.ap.m : static_cast<int64_t>(a.n_visible[r]);
  const int64_t n = min(max(n_raw, int64_t(0)), POOL ? static_cast<int64_t>(a.pool_blocks) * a.pblock : a.cap);
  const int32_t* prow = POOL ? a.pool + static_cast<int64_t>(r) * a.pool_blocks : nullptr;
  // pool position -> entry id (identity without a pool)
  auto entry_of = [&](uint32_t j) -> int32_t {
    if constexpr (!POOL) return static_cast<int32_t>(j);
    return __ldg(prow + j / a.pblock) * a.pblock + static_cast<int32_t>(j % a.pblock);
  };
  const int tiles_req = static_cast<int>((n + kTileM - 1) / kTileM);
  int t0, t1;
  if (APPEND && a.chunks > 1) {
    // the last chunk (whose CTA appends the token first) is shorter by `shrink` tiles
    const int per = (tiles_req + a.chunks - 1) / a.chunks;
    const int last = min(tiles_req, max(1, per - a.ap.shrink));
    const int rest = tiles_req - last;
    t0 = c < a.chunks - 1 ? c * rest / (a.chunks - 1) : rest;
    t1 = c < a.chunks - 1 ? (c + 1) * rest / (a.chunks - 1) : tiles_req;
  } else {
    t0 = static_cast<int>(static_cast<int64_t>(c) * tiles_req / a.chunks);
    t1 = static_cast<int>(static_cast<int64_t>(c + 1) * tiles_req / a.chunks);
  }
  const int nt = min(t1 - t0, kMaxChunkTiles);
  const int64_t base = static_cast<int64_t>(t0) * kTileM;  // first key of the chunk
  const int nloc = static_cast<int>(max(int64_t(0), min(n, static_cast<int64_t>(t0 + nt) * kTileM) - base));

  if (tid == 0) {
    prefetch_tensormap(&kmap);
    if constexpr (FP8) prefetch_tensormap(&smap);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);  // the MMA commit
    }
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 128);  // the epilogue group that read the scales
    }
    for (int ps = 0; ps < 2; ++ps) {
      mbar_init(&tfull[ps], 1);
      mbar_init(&tempty[ps], 2 * 128);  // both epilogue groups
    }
    mbar_init(qbar, 1);
    mbar_init(mdone, 1);
    mbar_init(abar, 1);
    mbar_init(cbar, 1);
    sh.fail = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if constexpr (APPEND)
    if (c == a.chunks - 1)
      append_block<MODE == kModeAppendMx4>(a.ap, r, a.cap, smem + C::oStages,
                                           reinterpret_cast<float*>(smem + C::oHist), abar, sh);

  // ================= phase 1: stream the keys, scores into TMEM =================
  if (POOL && warp == 0) {
    // candidate-pool mode: per stage, lane l loads the pblock-row box of
    // slot q0 + l (and, FP8, its row scales); a stage's slots are <= 32
    if (lane == 0) {
      mbar_arrive_expect_tx(qbar, kHeads * kDI * 2);
      bulk_load(smem + C::oQ, a.q_idx + static_cast<int64_t>(r) * kHeads * kDI, kHeads * kDI * 2, qbar);
    }
    const int bs = a.pblock, spt = kTileM / bs, sps = C::kTPS * spt;
    const int nst = (nt + C::kTPS - 1) / C::kTPS;
    const int64_t end_slot = (n + bs - 1) / bs;  // slots that hold positions
    const uint64_t l2_stream = l2_policy_evict_first();
    int issued = 0, sissued = 0;
    for (int p = 0; p < nst; ++p) {
      if (__shfl_sync(0xFFFFFFFFu, sh.fail, 0)) break;
      const int s = p % C::kStages;
      const int t = p * C::kTPS;
      const int64_t q0 = static_cast<int64_t>(t0 + t) * kTileM / bs;
      // slots past the run re-read the first block: those positions are >= n
      int32_t b = 0;
      if (lane < sps) b = __ldg(prow + (q0 + lane < end_slot ? q0 + lane : 0));
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[s], ((p / C::kStages) & 1) ^ 1, kWaitLimit);
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
        if (lane == 0) {
          atomicOr(&g_index_tc_error, 1u);
          sh.fail = 1;
        }
        break;
      }
      uint8_t* dst = smem + C::oStages + s * C::kStageBytes;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], C::kStageBytes);
      __syncwarp();
      if (lane < sps) {
        const int y = static_cast<int>(r * a.cap + static_cast<int64_t>(b) * bs);
        tma_load_2d_hint(dst + lane * bs * 128, &kmap, &full[s], 0, y, l2_stream);
        if constexpr (!FP8) tma_load_2d_hint(dst + 16384 + lane * bs * 128, &kmap, &full[s], 64, y, l2_stream);
      }
      issued = p + 1;
      if constexpr (FP8) {
        bool sfail = false;
        for (int j = 0; j < C::kTPS && t + j < nt; ++j) {
          const int u = t + j, ss = u % kSStages;
          bool sok = true;
          if (lane == 0) sok = mbar_wait(&sempty[ss], ((u / kSStages) & 1) ^ 1, kWaitLimit);
          if (!__shfl_sync(0xFFFFFFFFu, sok, 0)) {
            if (lane == 0) {
              atomicOr(&g_index_tc_error, 1u);
              sh.fail = 1;
            }
            sfail = true;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(&sfull[ss], kTileM * 4);
          __syncwarp();
          if (lane >= j * spt && lane < (j + 1) * spt)
            bulk_load(smem + C::oScales + ss * kTileM * 4 + (lane - j * spt) * bs * 4,
                      a.kscale + r * a.cap + static_cast<int64_t>(b) * bs, bs * 4, &sfull[ss]);
          sissued = u + 1;
        }
        if (sfail) break;
      }
    }
    if (lane == 0 && sh.fail) {  // let the copies still in flight land before the CTA winds down
      for (int p = max(0, issued - C::kStages); p < issued; ++p)
        mbar_wait(&full[p % C::kStages], (p / C::kStages) & 1, kWaitLimit);
      for (int u = max(0, sissued - kSStages); u < sissued; ++u)
        mbar_wait(&sfull[u % kSStages], (u / kSStages) & 1, kWaitLimit);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // the query first, so that it is not queued behind the key stream
      mbar_arrive_expect_tx(qbar, kHeads * kDI * 2);
      bulk_load(smem + C::oQ, a.q_idx + static_cast<int64_t>(r) * kHeads * kDI, kHeads * kDI * 2, qbar);
      int issued = 0, sissued = 0;
      const int nst = (nt + C::kTPS - 1) / C::kTPS;
      const uint64_t l2_stream = l2_policy_evict_first();
      for (int p = 0; p < nst && !sh.fail; ++p) {
        const int s = p % C::kStages;
        if (!mbar_wait(&empty[s], ((p / C::kStages) & 1) ^ 1, kWaitLimit)) {
          atomicOr(&g_index_tc_error, 1u);
          sh.fail = 1;
          break;
        }
        const int t = p * C::kTPS;
        const int y = static_cast<int>(r * a.cap + static_cast<int64_t>(t0 + t) * kTileM);
        uint8_t* dst = smem + C::oStages + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        // the keys are read once: evict them from L2 first, so that the stream
        // does not push out the code and the small data of the later phases
        if constexpr (FP8) {
          tma_load_2d_hint(dst, &kmap, &full[s], 0, y, l2_stream);  // 256 rows: tiles t and t + 1
        } else {
          tma_load_2d_hint(dst, &kmap, &full[s], 0, y, l2_stream);
          tma_load_2d_hint(dst + 16384, &kmap, &full[s], 64, y, l2_stream);
        }
        issued = p + 1;
        if constexpr (FP8) {
          for (int j = 0; j < C::kTPS && t + j < nt; ++j) {
            const int u = t + j, ss = u % kSStages;
            if (!mbar_wait(&sempty[ss], ((u / kSStages) & 1) ^ 1, kWaitLimit)) {
              atomicOr(&g_index_tc_error, 1u);
              sh.fail = 1;
              break;
            }
            mbar_arrive_expect_tx(&sfull[ss], kTileM * 4);
            tma_load_2d(smem + C::oScales + ss * kTileM * 4, &smap, &sfull[ss],
                        static_cast<int>(static_cast<int64_t>(t0 + u) * kTileM), r);
            sissued = u + 1;
          }
        }
      }
      if (sh.fail) {  // let the copies still in flight land before the CTA winds down
        for (int p = max(0, issued - C::kStages); p < issued; ++p)
          mbar_wait(&full[p % C::kStages], (p / C::kStages) & 1, kWaitLimit);
        for (int u = max(0, sissued - kSStages); u < sissued; ++u)
          mbar_wait(&sfull[u % kSStages], (u / kSStages) & 1, kWaitLimit);
      }
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
      // MMA issuer.  Tiles go in pairs (2p -> accumulator 0, 2p + 1 -> 1)
      // with their K steps interleaved; per pair it polls one barrier for
      // the keys (FP8) and one for the accumulators, and commits twice (an
      // mbarrier poll in this thread stalls the MMA issue for ~150 cycles).
      if (lane == 0 && !sh.fail) {
        const uint32_t b_base = smem_u32(Bs);
        for (int p = 0; 2 * p < nt; ++p) {
          const int ta = 2 * p;
          const bool two = ta + 1 < nt;
          int sa, sb;
          bool ok;
          if constexpr (FP8) {
            sa = sb = p % C::kStages;
            ok = mbar_wait(&full[sa], (p / C::kStages) & 1, kWaitLimit);
          } else {
            sa = ta % C::kStages;
            sb = (ta + 1) % C::kStages;
            ok = mbar_wait(&full[sa], (ta / C::kStages) & 1, kWaitLimit);
            if (ok && two) ok = mbar_wait(&full[sb], ((ta + 1) / C::kStages) & 1, kWaitLimit);
          }
          // pair slot p % 2: its previous use (pair p - 2) has been read back
          const int ps = p & 1;
          if (ok) ok = mbar_wait(&tempty[ps], ((p >> 1) & 1) ^ 1, kWaitLimit);
          if (!ok) {
            atomicOr(&g_index_tc_error, 1u);
            sh.fail = 1;
            break;
          }
          tc_fence_after();
          const uint32_t d0 = tmem + ps * 2 * kAccCols, d1 = d0 + kAccCols;
          const uint32_t a0 = smem_u32(smem + C::oStages + sa * C::kStageBytes);
          const uint32_t a1 = FP8 ? a0 + 16384 : smem_u32(smem + C::oStages + sb * C::kStageBytes);
          if constexpr (FP8) {
            // N = 128: the key tile is read once for both query terms
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = desc_k_sw128(b_base + kk * 32);
              mma_f8f6f4(d0, desc_k_sw128(a0 + kk * 32), bd, C::kIdesc, kk > 0 ? 1u : 0u);
              if (two) mma_f8f6f4(d1, desc_k_sw128(a1 + kk * 32), bd, C::kIdesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(&empty[sa]);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t half = kk >> 2, off = (kk & 3) * 32;
              const uint64_t bd = desc_k_sw128(b_base + half * 8192 + off);
              mma_f16(d0, desc_k_sw128(a0 + half * 16384 + off), bd, C::kIdesc, kk > 0 ? 1u : 0u);
              if (two) mma_f16(d1, desc_k_sw128(a1 + half * 16384 + off), bd, C::kIdesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(&empty[sa]);
            if (two) mma_commit(&empty[sb]);
          }
          mma_commit(&tfull[ps]);
        }
        // every MMA of this CTA has completed before TMEM is read back or released
        mma_commit(mdone);
        mbar_wait(mdone, 0, kWaitLimit);
      }
    } else {
      // epilogue: the raw query is consumed, its space becomes the histograms
      for (int i = tid - 64; i < 2 * kHistBins; i += kEpiWarps * 32) ghist0[i] = 0;
      named_barrier(3, kEpiWarps * 32);
      if (!sh.fail) {
        // two groups of four warps take alternate tiles; warp w owns TMEM
        // lanes 32 (w % 4) .. +31
        const int grp = (warp - 2) >> 2;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(sub * 32) << 16);
        const float qinv = sh.qinv;
        uint32_t* hist = ghist0 + grp * kHistBins;
        float w_r[kHeads];
#pragma unroll
        for (int h = 0; h < kHeads; ++h) w_r[h] = ws[h];
        // this chunk's scores in the workspace, tile by tile (lane = key)
        float* scg = a.scg + (static_cast<int64_t>(r) * a.chunks + c) * (kMaxChunkTiles * kTileM);
        for (int t = grp; t < nt; t += 2) {
          // tile t = 2p + grp sits in pair slot ps = p % 2, accumulator 2 ps + grp
          const int ps = (t >> 1) & 1;
          const int acc = 2 * ps + grp;
          // lane 0 polls, the warp follows its verdict (warp-wide TMEM ops below)
          bool tok = true;
          if (lane == 0) tok = mbar_wait(&tfull[ps], (t >> 2) & 1, kWaitLimit);
          __syncwarp();  // orders the other lanes after lane 0's acquire
          if (!__shfl_sync(0xFFFFFFFFu, tok, 0)) {
            atomicOr(&g_index_tc_error, 1u);
            sh.fail = 1;
            break;
          }
          tc_fence_after();
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
          const uint32_t acc_addr = lane_addr + acc * kAccCols;
#pragma unroll
          for (int hh = 0; hh < kHeads; hh += 32) {
            // heads hh..hh+31: FP8 adds the two query terms (columns h and 64 + h)
            uint32_t v0[32], v1[32];
            tmem_ld32(acc_addr + hh, v0);
            if constexpr (FP8) tmem_ld32(acc_addr + kHeads + hh, v1);
            tmem_wait_ld();
            if (hh + 32 == kHeads) {
              tc_fence_before();
              mbar_arrive(&tempty[ps]);
            }
#pragma unroll
            for (int h = 0; h < 32; h += 2) {
              float x0 = __uint_as_float(v0[h]), x1 = __uint_as_float(v0[h + 1]);
              if constexpr (FP8) {
                x0 += __uint_as_float(v1[h]);
                x1 += __uint_as_float(v1[h + 1]);
              }
              if (hh == 0) {
                s0 = fmaf(w_r[h], fmaxf(x0, 0.f), s0);
                s1 = fmaf(w_r[h + 1], fmaxf(x1, 0.f), s1);
              } else {
                s2 = fmaf(w_r[hh + h], fmaxf(x0, 0.f), s2);
                s3 = fmaf(w_r[hh + h + 1], fmaxf(x1, 0.f), s3);
              }
            }
          }
          // the row scale after the accumulator is released: its wait is off
          // the MMA -> epilogue -> MMA chain that paces the key stream
          float ks = 1.f;
          if constexpr (FP8) {
            const int ss = t % kSStages;
            bool sok = true;
            if (lane == 0) sok = mbar_wait(&sfull[ss], (t / kSStages) & 1, kWaitLimit);
            __syncwarp();
            if (!__shfl_sync(0xFFFFFFFFu, sok, 0)) {
              atomicOr(&g_index_tc_error, 1u);
              sh.fail = 1;
              break;
            }
            ks = scale_ring[ss * kTileM + row] * qinv;
            mbar_arrive(&sempty[ss]);
          }
          const float sc = ((s0 + s1) + (s2 + s3)) * ks;
          scg[t * kTileM + row] = sc;
          if (static_cast<int64_t>(t0 + t) * kTileM + row < n) atomicAdd(&hist[score_key(sc) >> 20], 1u);
        }
      }
    }
  }
  // the staged scores come back by a bulk copy (the async proxy) in phase 2
  asm volatile("fence.proxy.async.global;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // a kernel launched programmatically after this one (the decode step's
  // attention) may start its prologue on the SMs this grid frees; it reads
  // this grid's outputs only after waiting for its completion
  grid_launch_dependents();

  if (!sh.fail) {
    // ================= phase 2: exact top-k over the request =================
    const int k = a.k;
    const int nch = a.chunks;
    int32_t* oi = a.out_idx + static_cast<int64_t>(r) * k;
    float* os = a.out_score ? a.out_score + static_cast<int64_t>(r) * k : nullptr;
    uint8_t* p2 = smem + C::oStages;  // the rings are idle now
    uint32_t* hist = reinterpret_cast<uint32_t*>(p2 + C::pHist);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(p2 + C::pScratch);
    uint32_t* preA = reinterpret_cast<uint32_t*>(p2 + C::pCpre);  // [nch + 1] chunk prefixes
    uint32_t* preE = preA + kMaxChunks + 4;
    uint2* acache = reinterpret_cast<uint2*>(p2 + C::pACache);
    float* sc = reinterpret_cast<float*>(p2 + C::pScores);
    uint2* ecache = reinterpret_cast<uint2*>(p2 + C::pEq);
    auto put = [&](uint32_t pos, uint2 e) {
      if (pos < static_cast<uint32_t>(k)) {
        oi[pos] = entry_of(e.x);
        if (os) os[pos] = __uint_as_float(e.y);
      }
    };

    // scores TMEM -> shared memory in index order: warps 2..9, two per lane quarter
    // the chunk's scores, workspace -> shared memory in index order (the
    // block's own writes of phase 1, ordered by the barrier after it)
    // (one bulk copy of the chunk's nt x 512 contiguous bytes, waited for by
    // every thread)
    auto copy_scores = [&]() {
      if (nt <= 0) return;
      if (tid == 0) {
        const uint32_t bytes = static_cast<uint32_t>(nt) * kTileM * 4;
        mbar_arrive_expect_tx(cbar, bytes);
        bulk_load(sc, a.scg + (static_cast<int64_t>(r) * a.chunks + c) * (kMaxChunkTiles * kTileM), bytes, cbar);
      }
      if (!mbar_wait(cbar, 0, kWaitLimit)) atomicOr(&g_index_tc_error, 1u);
    };
    // block maxima of the chunk (the chunk starts on a tile, so on a block)
    auto write_block_max = [&]() {
      __syncthreads();
      const int bs = a.block, nb = (nloc + bs - 1) / bs;
      float* bm = a.bmax + static_cast<int64_t>(r) * a.ldb + base / bs;
      for (int b = tid; b < nb; b += kThreads) {
        const int e0 = b * bs, e1 = min(nloc, e0 + bs);
        float m = sc[e0];
        for (int e = e0 + 1; e < e1; ++e) m = fmaxf(m, sc[e]);
        bm[b] = m;
      }
    };
    // every thread owns a contiguous, 4-aligned segment of the chunk's entries
    const int seg = ((nloc + kThreads - 1) / kThreads + 3) & ~3;
    const int i0 = min(nloc, tid * seg), i1 = min(nloc, i0 + seg);

    if (n <= k) {
      copy_scores();
      if constexpr (BMAX) write_block_max();
      __syncthreads();
      for (int i = tid; i < nloc; i += kThreads) {
        oi[base + i] = entry_of(static_cast<uint32_t>(base + i));
        if (os) os[base + i] = sc[i];
      }
      if (c == 0)
        for (int64_t j = n + tid; j < k; j += kThreads) {
          oi[j] = -1;
          if (os) os[j] = -INFINITY;
        }
    } else {
      uint32_t* gh_g = ghist0;  // the two group histograms
      uint32_t* gh1 = a.ghist + static_cast<int64_t>(r) * 2 * kHistBins;
      uint32_t* gh2 = gh1 + kHistBins;
      uint32_t* bar = a.sync + r * 4;
      uint32_t nbar = 1;
      // level 1 (bits 31..20): the histogram built while streaming
      for (int i = tid; i < kHistBins / 4; i += kThreads) {
        const uint4 x = reinterpret_cast<const uint4*>(gh_g)[i];
        const uint4 y = reinterpret_cast<const uint4*>(gh_g + kHistBins)[i];
        const uint32_t v[4] = {x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (v[e]) atomicAdd(&gh1[4 * i + e], v[e]);
      }
      // arrive, copy the scores while the request's slower CTAs finish, wait
      request_arrive(&bar[0], static_cast<int>(blockIdx.x) == a.skip_arrive);
      copy_scores();
      if constexpr (BMAX) write_block_max();
      bool alive = request_wait(&bar[0], a.chunks, a.spin_limit, sh);
      uint32_t shift = 20, prefix = 0;
      if (alive) {
        load_hist(hist, gh1);
        __syncthreads();
        find_bin_block(hist, kHistBins, static_cast<uint32_t>(k), sh, scratch);
        prefix = sh.bcast[0];
        if (hist[prefix] > static_cast<uint32_t>(kEqCache)) {
          // a crowded boundary bin: one more distributed level (bits 19..8)
          const uint32_t need = static_cast<uint32_t>(k) - sh.bcast[1];
          for (int i = tid; i < kHistBins; i += kThreads) gh_g[i] = 0;
          __syncthreads();
          for (int i = i0; i < i1; ++i) {
            const uint32_t key = score_key(sc[i]);
            if ((key >> 20) == prefix) atomicAdd(&gh_g[(key >> 8) & 0xFFFu], 1u);
          }
          __syncthreads();
          for (int i = tid; i < kHistBins; i += kThreads)
            if (gh_g[i]) atomicAdd(&gh2[i], gh_g[i]);
          nbar = 2;
          alive = request_barrier(&bar[0], 2u * a.chunks, a.spin_limit, sh);
          if (alive) {
            load_hist(hist, gh2);
            __syncthreads();
            find_bin_block(hist, kHistBins, need, sh, scratch);
            prefix = (prefix << 12) | sh.bcast[0];
            shift = 8;
          }
        }
      }
      const int64_t slot = static_cast<int64_t>(r) * nch + c;
      uint2* st = a.st + slot * k;
      uint2* eqg = a.eq + slot * (kMaxChunkTiles * kTileM);
      uint32_t my_a = 0, my_e = 0;
      if (alive) {
        // this chunk's entries above the boundary prefix (kept here) and at
        // it (published), both lists in index order: counts per segment,
        // block prefix sums, writes
        uint32_t na = 0, ne = 0;
        for (int i = i0; i < i1; i += 4) {
          const float4 f = *reinterpret_cast<const float4*>(sc + i);
          const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t kp = score_key(fv[e]) >> shift;
            const bool ok = i + e < i1;
            na += ok && kp > prefix;
            ne += ok && kp == prefix;
          }
        }
        uint32_t pa, pe;
        block_scan2(na, ne, pa, pe, my_a, my_e, scratch);
        for (int i = i0; i < i1; i += 4) {
          const float4 f = *reinterpret_cast<const float4*>(sc + i);
          const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (i + e >= i1) break;
            const uint32_t kp = score_key(fv[e]) >> shift;
            const uint2 en = make_uint2(static_cast<uint32_t>(base + i + e), __float_as_uint(fv[e]));
            if (kp > prefix) {
              if (pa < static_cast<uint32_t>(kACache)) acache[pa] = en;
              else if (pa < static_cast<uint32_t>(k)) st[pa] = en;
              ++pa;
            } else if (kp == prefix) {
              eqg[pe++] = en;
            }
          }
        }
        if (tid == 0) reinterpret_cast<uint2*>(a.cnt)[slot] = make_uint2(my_a, my_e);
        ++nbar;
        alive = request_barrier(&bar[0], nbar * a.chunks, a.spin_limit, sh);
      }
      if (alive) {
        // ---- every CTA: chunk offsets, then its own share of the output ----
        // chunk counts straight into registers (warp 0: above, warp 1: at
        // the boundary; lane l holds chunks 5 l .. 5 l + 4), exclusive prefix
        // sums by a lane scan, written with the total at [nch]
        const uint2* cnt = reinterpret_cast<const uint2*>(a.cnt) + static_cast<int64_t>(r) * nch;
        static_assert(kMaxChunks <= 5 * 32, "five chunks per lane");
        if (warp < 2) {
          uint32_t v[5], mine = 0;
#pragma unroll
          for (int u = 0; u < 5; ++u) {
            const int i = lane * 5 + u;
            v[u] = 0u;
            if (i < nch) {
              const uint2 ce = __ldcg(cnt + i);
              v[u] = warp == 0 ? ce.x : ce.y;
            }
            mine += v[u];
          }
          uint32_t incl = mine;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += x;
          }
          uint32_t* pre = warp == 0 ? preA : preE;
          uint32_t run = incl - mine;
#pragma unroll
          for (int u = 0; u < 5; ++u) {
            const int i = lane * 5 + u;
            if (i < nch) pre[i] = run;
            run += v[u];
          }
          if (lane == 31) pre[nch] = incl;
        }
        __syncthreads();
        const uint32_t A_tot = preA[nch], E_tot = preE[nch];
        // entries above the boundary: straight to their place
        for (uint32_t i = tid; i < my_a; i += kThreads)
          put(preA[c] + i, i < static_cast<uint32_t>(kACache) ? acache[i] : __ldcg(st + i));
        const uint32_t take = A_tot < static_cast<uint32_t>(k) ? static_cast<uint32_t>(k) - A_tot : 0u;
        // chunk of boundary entry i (i < E_tot): fixed-step binary search
        auto eq_src = [&](uint32_t i) {
          int lo = 0;
#pragma unroll
          for (int step = 128; step > 0; step >>= 1) {
            const int m = lo + step;
            if (m < nch && preE[m] <= i) lo = m;
          }
          return a.eq + (static_cast<int64_t>(r) * nch + lo) * (kMaxChunkTiles * kTileM) + (i - preE[lo]);
        };
        if (E_tot <= take) {
          // every boundary entry is taken
          for (uint32_t i = tid; i < my_e; i += kThreads) put(A_tot + preE[c] + i, __ldcg(eqg + i));
        } else if (E_tot <= static_cast<uint32_t>(kEqCache)) {
          // the request's boundary entries, in index order, into shared
          // memory: warp w copies the lists of chunks w, w + 10, ... (each
          // list is contiguous in its chunk's staging), four loads in flight
          // per lane
          for (int cc = warp; cc < nch; cc += kThreads / 32) {
            const uint2* src = a.eq + (static_cast<int64_t>(r) * nch + cc) * (kMaxChunkTiles * kTileM);
            const uint32_t o = preE[cc], len = preE[cc + 1] - o;
            for (uint32_t j0 = 0; j0 < len; j0 += 128) {
              uint2 e[4];
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (j0 + b * 32 + lane < len) e[b] = __ldcg(src + j0 + b * 32 + lane);
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (j0 + b * 32 + lane < len) ecache[o + j0 + b * 32 + lane] = e[b];
            }
          }
          __syncthreads();
          // radix levels over the low `shift` key bits (12 + 8, or 8): the
          // take-th largest key T and how many entries equal to T are taken.
          // A level whose chosen bin is taken whole (usual after 12 bits: a
          // few thousand entries over 4,096 bins) ends the search: T is then
          // the key just below that bin and no entry equal to T is taken
          uint32_t pfx = prefix, rb = shift, tk = take;
          bool whole = false;
          while (rb > 0) {
            const uint32_t nb = rb > 12 ? 12 : rb;
            const uint32_t sft = rb - nb;
            for (int i = tid; i < (1 << nb); i += kThreads) hist[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < E_tot; i += kThreads) {
              const uint32_t key = score_key(__uint_as_float(ecache[i].y));
              if ((key >> rb) == pfx) atomicAdd(&hist[(key >> sft) & ((1u << nb) - 1u)], 1u);
            }
            __syncthreads();
            find_bin_block(hist, 1 << nb, tk, sh, scratch);
            const uint32_t bsel = sh.bcast[0];
            pfx = (pfx << nb) | bsel;
            tk -= sh.bcast[1];
            rb = sft;
            if (rb > 0 && sh.bcast[2] == tk && (pfx << rb) != 0u) {
              whole = true;
              break;
            }
          }
          const uint32_t T = whole ? (pfx << rb) - 1u : pfx;
          if (whole) tk = 0;
          // taken: key > T, and the first tk (lowest indices) with key == T
          const uint32_t e0 = preE[c], e1 = preE[c + 1];
          uint32_t g = 0, q = 0;
          for (uint32_t i = tid; i < e0; i += kThreads) {
            const uint32_t key = score_key(__uint_as_float(ecache[i].y));
            g += key > T;
            q += key == T;
          }
          block_sum2(g, q, scratch);
          uint32_t out = A_tot + g + min(q, tk), eq_seen = q;
          for (uint32_t j0 = e0; j0 < e1; j0 += kThreads) {
            const uint32_t i = j0 + tid;
            const uint2 e = i < e1 ? ecache[i] : make_uint2(0u, 0u);
            const uint32_t key = score_key(__uint_as_float(e.y));
            const bool gt = i < e1 && key > T, eq = i < e1 && key == T;
            uint32_t re, rz, te, tz;
            block_rank2(eq, false, re, rz, te, tz, scratch);
            const bool sel = gt || (eq && eq_seen + re < tk);
            uint32_t rs, ts;
            block_rank2(sel, false, rs, rz, ts, tz, scratch);
            if (sel) put(out + rs, e);
            out += ts;
            eq_seen += te;
          }
        } else if (c == 0) {
          // very many boundary entries (massive ties): one CTA streams them
          // from global memory through the same radix levels and writes the
          // whole boundary part of the output
          uint32_t pfx = prefix, rb = shift, tk = take;
          while (rb > 0) {
            const uint32_t nb = rb > 10 ? 10 : rb;
            const uint32_t sft = rb - nb;
            for (int i = tid; i < (1 << nb); i += kThreads) hist[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < E_tot; i += kThreads) {
              const uint32_t key = score_key(__uint_as_float(__ldcg(eq_src(i)).y));
              if ((key >> rb) == pfx) atomicAdd(&hist[(key >> sft) & ((1u << nb) - 1u)], 1u);
            }
            __syncthreads();
            find_bin_block(hist, 1 << nb, tk, sh, scratch);
            pfx = (pfx << nb) | sh.bcast[0];
            tk -= sh.bcast[1];
            rb = sft;
          }
          const uint32_t T = pfx;
          uint32_t out = A_tot, eq_seen = 0;
          for (uint32_t j0 = 0; j0 < E_tot; j0 += kThreads) {
            const uint32_t i = j0 + tid;
            const uint2 e = i < E_tot ? __ldcg(eq_src(i)) : make_uint2(0u, 0u);
            const uint32_t key = score_key(__uint_as_float(e.y));
            const bool gt = i < E_tot && key > T, eq = i < E_tot && key == T;
            uint32_t re, rz, te, tz;
            block_rank2(eq, false, re, rz, te, tz, scratch);
            const bool sel = gt || (eq && eq_seen + re < tk);
            uint32_t rs, ts;
            block_rank2(sel, false, rs, rz, ts, tz, scratch);
            if (sel) put(out + rs, e);
            out += ts;
            eq_seen += te;
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

// A pending test request (csa_test_expire_next_barrier): consumed by the
// next launch of this kernel.
std::mutex g_test_mu;
int g_test_skip_cta = -1;
uint32_t g_test_polls = kSpinLimit;

struct Launcher {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  int sms = 0;
  bool attr_set[2][kModes] = {};  // per key format and launch mode
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
  return ch > 0 ? ch : 1;  // more requests than SMs: not run by this kernel, sized as one chunk
}

bool index_tc_supported(const csa_params_t* p, int batch, int64_t cap, int q_dtype, int k_dtype) {
  if (p->h_idx != kHeads || p->d_idx != kDI || q_dtype != kBF16) return false;
  if (k_dtype != kFP8 && k_dtype != kBF16) return false;
  if (k_dtype == kFP8 && cap % 4 != 0) return false;  // row-scale tiles: 16-byte row stride
  if (batch < 1 || batch > (launcher().sms > 0 ? launcher().sms : 148)) return false;
  if (static_cast<int64_t>(batch) * cap >= (int64_t(1) << 31)) return false;
  const int ch = index_tc_chunks(batch, cap);
  const int64_t tiles = (cap + kTileM - 1) / kTileM;
  // room for the in-kernel append's shorter last chunk
  const int64_t per = (tiles + ch - 1) / ch + (ch > 1 ? (kAppendShrink + ch - 2) / (ch - 1) + 1 : 0);
  return ch <= kMaxChunks && per <= kMaxChunkTiles && p->topk >= 1;
}

// Candidate-pool mode (a Reindex layer): positions are the pool's entries,
// loaded as `block`-row boxes of whole 1 KB swizzle atoms (block >= 8).
bool index_tc_pool_supported(const csa_params_t* p, int batch, int64_t cap, int block, int pool_blocks, int q_dtype,
                             int k_dtype) {
  if (block < 8 || block > kTileM || (block & (block - 1)) != 0) return false;
  if (p->h_idx != kHeads || p->d_idx != kDI || q_dtype != kBF16) return false;
  if (k_dtype != kFP8 && k_dtype != kBF16) return false;
  // FP8: whole blocks of row scales, so that no block's scales run past the tensor
  if (k_dtype == kFP8 && cap % block != 0) return false;
  if (batch < 1 || batch > (launcher().sms > 0 ? launcher().sms : 148)) return false;
  if (static_cast<int64_t>(batch) * cap >= (int64_t(1) << 31)) return false;
  const int64_t np = static_cast<int64_t>(block) * pool_blocks;
  const int ch = index_tc_chunks(batch, np);
  const int64_t tiles = (np + kTileM - 1) / kTileM;
  return ch <= kMaxChunks && (tiles + ch - 1) / ch <= kMaxChunkTiles && p->topk >= 1;
}

// The decode step can append inside the indexer: W_IK (d x 128) fits the
// idle stage ring and the pooled row the shared scratch.
bool index_tc_append_supported(const csa_params_t* p, int w_dtype) {
  const int wb = w_dtype == kBF16 ? 2 : 4;
  return p->d % 8 == 0 && static_cast<size_t>(p->d) * kDI * wb <= static_cast<size_t>(Cfg<true>::oScales) &&
         static_cast<size_t>(p->d + 3 * kDI) * 4 <= 2 * kHistBins * 4;
}

size_t index_tc_control_bytes(int batch) { return static_cast<size_t>(batch) * (2 * kHistBins + 4) * 4; }

size_t index_tc_workspace_bytes(int batch, int64_t cap, int k) {
  const int ch = index_tc_chunks(batch, cap);
  size_t b = index_tc_control_bytes(batch);
  b += static_cast<size_t>(batch) * ch * 2 * 4;                       // cnt
  b += static_cast<size_t>(batch) * ch * k * 8;                       // staging above
  b += static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 8;  // staging boundary
  b += static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 4;  // scores
  return b + 5 * 256;
}

// `ws` must hold index_tc_workspace_bytes; its first index_tc_control_bytes
// must be zero on entry (the caller zeroes them).
csa_status_t launch_index_topk_tc(const csa_params_t* p, int batch, const csa_tensor_t* q_idx, const float* w,
                                  const csa_tensor_t* k_idx, int64_t cap, const int32_t* n_visible, int32_t* out_idx,
                                  float* out_score, void* ws, cudaStream_t stream, const AppendArgs* ap,
                                  float* bmax, int64_t ldb, int block, const int32_t* pool,
                                  int pool_blocks, int pblock) {
  Launcher& L = launcher();
  if (!L.encode) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const bool fp8 = k_idx->dtype == kFP8;
  // pool mode chunks the pool's positions, not the cache
  const int64_t npos = pool ? static_cast<int64_t>(pool_blocks) * pblock : cap;
  const int ch = index_tc_chunks(batch, npos);
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDI), static_cast<cuuint64_t>(batch) * cap};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDI) * (fp8 ? 1 : 2)};
  // FP8: one 256-row box = two key tiles per stage; bf16: two 64-column boxes
  // per tile; pool mode: one box per pool block
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(fp8 ? 128 : 64),
                             static_cast<cuuint32_t>(pool ? pblock : fp8 ? 2 * kTileM : kTileM)};
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
  a.append = ap != nullptr;
  a.bmax = bmax;
  a.ldb = ldb;
  a.block = block;
  a.pool = pool;
  a.pool_blocks = pool_blocks;
  a.pblock = pblock;
  a.kscale = fp8 ? static_cast<const float*>(k_idx->scale) : nullptr;
  a.spin_limit = kSpinLimit;
  a.skip_arrive = -1;
  {
    std::lock_guard<std::mutex> lk(g_test_mu);
    if (g_test_skip_cta >= 0) {
      a.skip_arrive = g_test_skip_cta;
      a.spin_limit = g_test_polls;
      g_test_skip_cta = -1;
      g_test_polls = kSpinLimit;
    }
  }
  if (ap) {
    a.ap = *ap;
    a.ap.shrink = kAppendShrink;
  } else {
    memset(&a.ap, 0, sizeof(a.ap));
  }
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
  a.st = reinterpret_cast<uint2*>(take(static_cast<size_t>(batch) * ch * p->topk * 8));
  a.eq = reinterpret_cast<uint2*>(take(static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 8));
  a.scg = reinterpret_cast<float*>(take(static_cast<size_t>(batch) * ch * kMaxChunkTiles * kTileM * 4));

  const int smem = fp8 ? Cfg<true>::kSmem : Cfg<false>::kSmem;
  const int mode = pool ? kModePool : bmax ? kModeBmax
                   : ap ? (ap->kv.dtype == kMXFP4 ? kModeAppendMx4 : kModeAppend) : kModePlain;
  using Kern = void (*)(CUtensorMap, CUtensorMap, IdxArgs);
  const Kern kerns[2][kModes] = {
      {index_topk_tc_kernel<false, 0>, index_topk_tc_kernel<false, 1>, index_topk_tc_kernel<false, 2>,
       index_topk_tc_kernel<false, 3>, index_topk_tc_kernel<false, 4>},
      {index_topk_tc_kernel<true, 0>, index_topk_tc_kernel<true, 1>, index_topk_tc_kernel<true, 2>,
       index_topk_tc_kernel<true, 3>, index_topk_tc_kernel<true, 4>}};
  const Kern fn = kerns[fp8 ? 1 : 0][mode];
  if (!L.attr_set[fp8 ? 1 : 0][mode]) {
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    L.attr_set[fp8 ? 1 : 0][mode] = true;
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, map, smap, a);
  if (e != cudaSuccess) {
    check_launch("index_topk_tc_kernel", stream);
    return set_error(CSA_ERR_CUDA, "index_topk_tc_kernel launch: %s", cudaGetErrorString(e));
  }
  return check_launch("index_topk_tc_kernel", stream);
}

csa_status_t test_expire_next_barrier(int cta, uint32_t polls) {
  std::lock_guard<std::mutex> lk(g_test_mu);
  g_test_skip_cta = cta;
  g_test_polls = polls < 1 ? 1 : polls;
  return CSA_OK;
}

// Reads and clears the device error word of this kernel (bounded waits).
uint32_t index_tc_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_index_tc_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_index_tc_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
