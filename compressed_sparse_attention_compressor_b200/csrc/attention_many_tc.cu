// K4 + K5 on the tensor cores for many query tokens (chunked prefill): one
// CTA per query, 64 heads of d = 512, looping over the query's key list --
// its selected compressed entries (CSA) or every visible entry (HCA), then
// its window positions -- in tiles of 128 keys, with one online softmax
// whose running sums stay on chip for the whole list.
//
// Atlas "Model architectures", "compressed KV" (CSA top-k entries plus a
// sliding window; HCA dense) and "MLA" (the latent is key and value);
// tech-report tour, "The indexer selects, SWA covers the rest" (the query
// attends to the selected entries together with the sliding-window KV).
//
// Per tile (attn_tile.cuh's layouts):
//   1. gather: key rows -> bf16, K-major 128-byte swizzled tile, in eight
//      64-dim column blocks (all warps, asynchronous copies);
//   2. S^T[128 keys][64 heads] = K Q^T (tcgen05, M = 128, N = 64, K = 512),
//      each block's four MMAs issued as soon as every thread's copies of the
//      block have landed; the query (64 KB) was loaded once by TMA;
//   3. all eight warps read S^T from TMEM (warp w: keys 32 (w % 4) .. + 31,
//      heads 32 (w / 4) .. + 31, a key per thread), and write
//      P^T = exp(S - m) as bf16; the window rows' values replace their keys
//      by asynchronous copies meanwhile;
//   4. O^T[512][64] += V^T P^T (tcgen05, the tile as an MN-major A operand),
//      accumulated in TMEM over all tiles.
// The running maximum m is updated lazily: a head's m moves only when a
// logit exceeds it by more than kLazy (P <= e^kLazy meanwhile, exact in
// bf16's range; the tile's per-head maxima are reduced across the keys, by
// a transposing warp butterfly, only in tiles where some logit does), and
// only then is its column of O rescaled in TMEM.  The sink enters the
// denominator once at the end; out = O / L and lse = M + log L exactly as
// in the single-tile kernels; the output block is staged in shared memory
// and leaves by bulk stores.
#include <cudaTypedefs.h>

#include "attn_tile.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

using namespace sm100;
using namespace attn;

constexpr uint32_t kTmemColsM = 512;  // S^T 64 columns + O^T 256 columns
constexpr float kLazy = 8.f;          // nats a tile maximum may exceed m before m moves
constexpr float kLog2e = 1.4426950408889634f;

// shared memory, from a 1024-byte aligned base
constexpr int mK = 0;                       // 8 x 16 KB key / value tile
constexpr int mQ = mK + 8 * kTK * 128;      // 8 x 8 KB query
constexpr int mP = mQ + 8 * kH * 128;       // 2 x 8 KB P^T (bf16, K-major over keys)
constexpr int mRed = mP + 2 * kH * 128;     // [4][64] per-warp partial maxima / sums
constexpr int mStat = mRed + 4 * kH * 4;    // m, l, rescale factor, final scale, m + kLazy, m log2 e: [64] each
constexpr int mEnt = mStat + 6 * kH * 4;    // [128] entry codes of the tile
constexpr int mBars = mEnt + kTK * 4;
constexpr int mMisc = mBars + 64;
constexpr int mLut = mMisc + 64;            // MXFP4 code-byte table, 256 x bf16x2
constexpr int kSmemM = mLut + 1024 + 1024;  // + alignment slack
static_assert(kSmemM <= 232448, "shared memory");
static_assert(mP % 1024 == 0, "operand alignment");

__device__ uint32_t g_attn_many_error = 0;

struct AttnManyArgs {
  const void* kv; const void* kv_scale; int batch; int64_t cap;
  const int32_t* idx; int topk;   // idx == nullptr: dense over n_visible
  const int32_t* n_visible; const int32_t* q_req;
  const uint16_t* swa_k; const uint16_t* swa_v; int swa_cap; int window;
  const int64_t* q_pos; const int64_t* swa_lo;
  float tau;
  const float* sink; void* out; int out_dtype; float* lse;
  int out_bulk;  // out is 16-byte aligned: the block leaves by bulk stores
};

__device__ __forceinline__ uint8_t* align1024m(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Butterfly over the warp's 32 lanes that reduces 32 per-lane values (one
// per head of a half) with `op` while transposing them: afterwards lane l
// holds the warp's result for head l of the half in v[0].  31 shuffles.
template <class Op>
__device__ __forceinline__ void warp_reduce32(float (&v)[32], Op op) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int o = 16 >> r;   // partner distance
    const int n = 32 >> r;   // values still held
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      v[i] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, o));
    }
  }
}

struct MaxOp {
  __device__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct SumOp {
  __device__ float operator()(float a, float b) const { return a + b; }
};

// Shared-memory address of 16-byte chunk c8 (elements 8 c8 .. 8 c8 + 7) of
// tile row r (put_chunk's layout).
__device__ __forceinline__ uint8_t* chunk_addr(uint8_t* tile, int r, int c8) {
  return tile + (c8 >> 3) * (kTK * 128) + sw128_offset(r, c8 & 7);
}

// All threads: the tile's window rows (entry codes <= -2) take their value
// rows (compressed entries are their own values), by asynchronous 16-byte
// copies; the caller waits for them (cp_async_wait_all) before P V.
__device__ void issue_window_values(uint8_t* tile, const int32_t* ent, const Src& a) {
  for (int task = static_cast<int>(threadIdx.x); task < kTK * 64; task += kNT) {
    const int32_t e = ent[task >> 6];
    if (e <= -2)
      cp_async16(chunk_addr(tile, task >> 6, task & 63),
                 reinterpret_cast<const uint4*>(a.swa_v + (a.sw_row0 + (-2 - e)) * kD) + (task & 63));
  }
}

// Named barriers 2 .. 9: column block b (dims 64 b .. 64 b + 63) of the key
// tile is in shared memory.  Barrier 1 is free; 0 is __syncthreads.
constexpr uint32_t kBarBlock = 2;

// All threads: the tile's key rows, column block by column block.  bf16
// rows (compressed bf16 entries, window keys) by asynchronous 16-byte
// copies, one commit group per block: thread t copies chunks q = i kNT + t
// (i < 4) of every block, row q / 8, chunk q % 8 of the block; FP8 / MXFP4
// compressed rows go through registers (dequantised to bf16) before any
// block is released; rows without a key (-1) are zeroed.  A thread releases
// block b once its own copies of it have landed (and are fenced for the
// tensor cores): warp 1, which issues the S MMAs, waits for the block's
// barrier instead and issues the block's four MMAs as soon as every thread
// has released it, so the MMAs follow the copies block by block.
template <int FMT>
__device__ bool gather_keys_issue_s(uint8_t* tile, const int32_t* ent, const Src& a, uint32_t dS, uint32_t qb,
                                    uint64_t* qbar, bool first) {
  const int tid = static_cast<int>(threadIdx.x), warp = tid >> 5, lane = tid & 31;
  if constexpr (FMT != kKvBF16) {
    gather_rows<FMT>(tile, ent, a, 0);  // quantised rows (and the rest), through registers
  } else {
#pragma unroll
    for (int b = 0; b < 8; ++b) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = i * kNT + tid;
        const int r = q >> 3, c8 = b * 8 + (q & 7);
        const int32_t e = ent[r];
        uint8_t* dst = chunk_addr(tile, r, c8);
        if (e >= 0)
          cp_async16(dst, reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.kv) + (a.kv_row0 + e) * kD) + c8);
        else if (e <= -2)
          cp_async16(dst, reinterpret_cast<const uint4*>(a.swa_k + (a.sw_row0 + (-2 - e)) * kD) + c8);
        else
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
      cp_async_commit();
    }
  }
  bool ok = true;
  const uint32_t kb = smem_u32(tile);
  auto release = [&](int b) {
    fence_proxy_async_smem();
    if (warp != 1) {
      named_barrier_arrive(kBarBlock + b, kNT);
      return;
    }
    named_barrier(kBarBlock + b, kNT);
    if (lane == 0) {
      if (b == 0 && first) ok = mbar_wait(qbar, 0, kWaitLimit);
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(dS, desc_k_sw128(kb + b * kTK * 128 + kk * 32), desc_k_sw128(qb + b * kH * 128 + kk * 32), kIdescS,
                  (b | kk) ? 1u : 0u);
      }
    }
    __syncwarp();
  };
  if constexpr (FMT != kKvBF16) {
#pragma unroll
    for (int b = 0; b < 8; ++b) release(b);
  } else {
    cp_async_wait_group<7>(); release(0);
    cp_async_wait_group<6>(); release(1);
    cp_async_wait_group<5>(); release(2);
    cp_async_wait_group<4>(); release(3);
    cp_async_wait_group<3>(); release(4);
    cp_async_wait_group<2>(); release(5);
    cp_async_wait_group<1>(); release(6);
    cp_async_wait_group<0>(); release(7);
  }
  return ok;
}

template <int FMT>
__global__ void __launch_bounds__(kNT, 1)
attn_many_tc_kernel(const __grid_constant__ CUtensorMap qmap, AttnManyArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024m(smem_raw);
  uint8_t* Kt = smem + mK;
  uint8_t* Pt = smem + mP;
  float* red = reinterpret_cast<float*>(smem + mRed);
  float* m_run = reinterpret_cast<float*>(smem + mStat);
  float* l_run = m_run + kH;
  float* fac = l_run + kH;
  float* fin = fac + kH;
  float* thr = fin + kH;  // m + kLazy (-inf while a head has no mass)
  float* ml2 = thr + kH;  // m log2(e) (0 while a head has no mass)
  int32_t* ent = reinterpret_cast<int32_t*>(smem + mEnt);
  uint64_t* qbar = reinterpret_cast<uint64_t*>(smem + mBars);
  uint64_t* sbar = qbar + 1;
  uint64_t* obar = qbar + 2;
  uint64_t* mdone = qbar + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + mMisc);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + mMisc + 16);  // [0] rescale, [1] failed

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qi = blockIdx.x;
  const int r = a.q_req ? a.q_req[qi] : qi;
  const bool live = r >= 0 && r < a.batch;
  const int nv = static_cast<int>(min(max(static_cast<int64_t>(a.n_visible[qi]), int64_t(0)), a.cap));
  const int n_sel = a.idx ? a.topk : nv;
  const int64_t t = a.q_pos[qi];
  int64_t p_lo = t - a.window + 1;
  if (a.swa_lo && a.swa_lo[qi] > p_lo) p_lo = a.swa_lo[qi];
  if (p_lo < 0) p_lo = 0;
  const int n_win = (a.window > 0 && t >= p_lo) ? static_cast<int>(t - p_lo + 1) : 0;
  const int total = live ? n_sel + n_win : 0;
  const int ntiles = (total + kTK - 1) / kTK;
  // entry code of key-list position x: selected entry (>= 0), window slot
  // (-2 - slot), nothing (-1); the selection's index is loaded apart
  // (idx_at), so that its load can be issued well before the code is formed
  auto idx_at = [&](int x) -> int32_t {
    return (a.idx && x < total && x < n_sel) ? a.idx[static_cast<int64_t>(qi) * a.topk + x] : x;
  };
  auto code = [&](int x, int32_t jj) -> int32_t {
    int32_t e = -1;
    if (x < total) {
      if (x < n_sel) e = (jj >= 0 && jj < nv) ? jj : -1;
      else e = -2 - static_cast<int32_t>((p_lo + (x - n_sel)) % a.swa_cap);
    }
    return e;
  };

  if (tid == 0) {
    prefetch_tensormap(&qmap);
    mbar_init(qbar, 1);
    mbar_init(sbar, 1);
    mbar_init(obar, 1);
    mbar_init(mdone, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
    if (ntiles > 0) {  // the query, once; its load overlaps the first gather
      mbar_arrive_expect_tx(qbar, kH * kD * 2);
      for (int blk = 0; blk < 8; ++blk) tma_load_2d(smem + mQ + blk * kH * 128, &qmap, qbar, blk * 64, qi * kH);
    }
  }
  if (tid < kH) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
    thr[tid] = -INFINITY;
    ml2[tid] = 0.f;
  }
  if (tid < kTK) ent[tid] = code(tid, idx_at(tid));
  if (warp == 1) tmem_alloc(tmem_slot, kTmemColsM);
  if constexpr (FMT == kKvMX4) fill_mx4_lut(reinterpret_cast<uint32_t*>(smem + mLut));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t dS = tmem, dO = tmem + kH;
  Src src;
  src.kv = a.kv;
  src.kv_scale = a.kv_scale;
  src.lut = reinterpret_cast<const uint32_t*>(smem + mLut);
  src.swa_k = a.swa_k;
  src.swa_v = a.swa_v;
  src.kv_row0 = live ? static_cast<int64_t>(r) * a.cap : 0;
  src.sw_row0 = live ? static_cast<int64_t>(r) * a.swa_cap : 0;
  src.tau = a.tau;
  // softmax split: warp w reads TMEM lanes (keys) 32 (w % 4) .. + 31 and
  // takes heads hb .. hb + 31 of them
  const int q4 = warp & 3, hb = (warp >> 2) * 32;
  const int row = q4 * 32 + lane;  // key of the tile this thread reads
  const uint32_t taS = dS + (static_cast<uint32_t>(q4 * 32) << 16) + hb;

  for (int j = 0; j < ntiles; ++j) {
    // the next tile's entry codes: index loads issued now, codes stored while P V runs
    const int x_next = (j + 1) * kTK + tid;
    const int32_t jj_next = (tid < kTK && j + 1 < ntiles) ? idx_at(x_next) : 0;
    // ---- gather, and S^T = K Q^T block by block behind it ----
    if (!gather_keys_issue_s<FMT>(Kt, ent, src, dS, smem_u32(smem + mQ), qbar, j == 0)) {
      atomicOr(&g_attn_many_error, 1u);
      flags[1] = 1;
    }
    if (tid == 32) mma_commit(sbar);
    if (tid == 0 && !mbar_wait(sbar, j & 1, kWaitLimit)) {
      atomicOr(&g_attn_many_error, 1u);
      flags[1] = 1;
    }
    __syncthreads();
    tc_fence_after();
    if (flags[1]) break;
    const int x0 = j * kTK;
    // window rows: values replace keys in the tile (S has read it); the
    // copies fly during the softmax
    if (n_win > 0 && x0 + kTK > n_sel && x0 < total) issue_window_values(Kt, ent, src);

    // ---- softmax over the tile: P = exp(S - m), m moving lazily ----
    const bool row_ok = ent[row] != -1;
    float s[32];
    auto load_logits = [&]() {
      uint32_t v[32];
      tmem_ld32(taS, v);
      tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < 32; ++h) s[h] = __uint_as_float(v[h]) * a.tau;
    };
    load_logits();
    // m stays unless a logit passes m + kLazy (or a head has no mass yet)
    bool pass = false;
    if (row_ok) {
#pragma unroll
      for (int h = 0; h < 32; h += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(thr + hb + h);
        pass = pass || (s[h] > t4.x) || (s[h + 1] > t4.y) || (s[h + 2] > t4.z) || (s[h + 3] > t4.w);
      }
    }
    const bool moved = __syncthreads_or(pass) != 0;
    if (moved) {
      // the tile's maximum of every head: per warp (lane l: head hb + l), then over the 4 key quarters
#pragma unroll
      for (int h = 0; h < 32; ++h) s[h] = row_ok ? s[h] : -INFINITY;
      warp_reduce32(s, MaxOp());
      red[q4 * kH + hb + lane] = s[0];
      __syncthreads();
      if (tid < kH) {
        const int h = tid;
        const float mt = fmaxf(fmaxf(red[h], red[kH + h]), fmaxf(red[2 * kH + h], red[3 * kH + h]));
        const float mo = m_run[h];
        float f = 1.f, mu = mo;
        if (mt != -INFINITY) {
          if (mo == -INFINITY) {
            mu = mt;  // no mass yet: this head's O and l are zero
          } else if (mt > mo + kLazy) {
            f = __expf(mo - mt);
            mu = mt;
            flags[0] = 1;
          }
        }
        m_run[h] = mu;
        fac[h] = f;
        thr[h] = mu == -INFINITY ? -INFINITY : mu + kLazy;
        ml2[h] = mu == -INFINITY ? 0.f : mu * kLog2e;
      }
      __syncthreads();
      load_logits();
    }
    // P^T [head][key] as bf16 (rows without a key: 0); the sums in fp32
    {
      uint8_t* prow = Pt + (row >> 6) * (kH * 128) + (row & 7) * 2;
      const uint32_t ch = (row & 63) >> 3;
      // P for 16 heads at a time: their m log2 e into registers before the
      // stores (a shared-memory load after a shared-memory store waits for it)
#pragma unroll
      for (int h0 = 0; h0 < 32; h0 += 16) {
        float mm[16];
#pragma unroll
        for (int h = 0; h < 16; h += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(ml2 + hb + h0 + h);
          mm[h] = m4.x; mm[h + 1] = m4.y; mm[h + 2] = m4.z; mm[h + 3] = m4.w;
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float p = row_ok ? ex2_approx(fmaf(s[h0 + h], kLog2e, -mm[h])) : 0.f;
          s[h0 + h] = p;
          *reinterpret_cast<uint16_t*>(prow + sw128_offset(hb + h0 + h, ch)) = f32_to_bf16_bits(p);
        }
      }
    }
    warp_reduce32(s, SumOp());
    red[q4 * kH + hb + lane] = s[0];
    __syncthreads();
    if (tid < kH) {
      const int h = tid;
      const float f = moved ? fac[h] : 1.f;
      l_run[h] = l_run[h] * f + ((red[h] + red[kH + h]) + (red[2 * kH + h] + red[3 * kH + h]));
    }
    // a head whose m moved: its column of O (all 512 dims) by the factor;
    // warp w rescales dims 32 (w % 4) .. + 31 of the blocks 2 (w / 4), + 1
    if (moved && j > 0 && flags[0]) {
#pragma unroll 1
      for (int mt = 2 * (warp >> 2); mt < 2 * (warp >> 2) + 2; ++mt) {
        const uint32_t ta = dO + mt * kH + (static_cast<uint32_t>(q4 * 32) << 16);
        uint32_t v0[32], v1[32];
        tmem_ld32(ta, v0);
        tmem_ld32(ta + 32, v1);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          v0[h] = __float_as_uint(__uint_as_float(v0[h]) * fac[h]);
          v1[h] = __float_as_uint(__uint_as_float(v1[h]) * fac[32 + h]);
        }
        tmem_st32(ta, v0);
        tmem_st32(ta + 32, v1);
      }
      tmem_wait_st();
    }
    cp_async_wait_all();  // window values
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- O^T += V^T P^T ----
    if (tid == 32) {
      const uint32_t kb = smem_u32(Kt), pb = smem_u32(Pt);
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          mma_f16(dO + mt * kH, desc_mn_sw128(kb + (2 * mt) * kTK * 128 + kk * 16 * 128, kTK * 128),
                  desc_k_sw128(pb + (kk >> 2) * kH * 128 + (kk & 3) * 32), kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit(obar);
    }
    if (tid < kTK) ent[tid] = j + 1 < ntiles ? code(x_next, jj_next) : -1;  // this tile's were last read before the barrier
    if (tid == 128) flags[0] = 0;
    if (tid == 0 && !mbar_wait(obar, j & 1, kWaitLimit)) {
      atomicOr(&g_attn_many_error, 1u);
      flags[1] = 1;
    }
    __syncthreads();  // the next tile may overwrite the key tile and P^T
    tc_fence_after();
    if (flags[1]) break;
  }

  // ---- out = O / L with the sink in L; lse = M + log L ----
  const bool done = !flags[1];
  if (tid < kH) {
    const int h = tid;
    const float m = m_run[h], l = l_run[h];
    const float sk = a.sink ? a.sink[h] : -INFINITY;
    const float M = fmaxf(m, sk);
    float scale = 0.f, L = 0.f;
    if (M != -INFINITY) {
      const float am = (m == -INFINITY) ? 0.f : __expf(m - M);
      L = l * am + ((sk == -INFINITY) ? 0.f : __expf(sk - M));
      scale = am / L;
    }
    fin[h] = (ntiles > 0 && done) ? scale : 0.f;
    if (a.lse) a.lse[static_cast<int64_t>(qi) * kH + h] = (M == -INFINITY) ? -INFINITY : M + __logf(L);
  }
  __syncthreads();
  {
    // O / L into shared memory as the output rows [head][dim] (the key tile
    // is idle now: every MMA has completed), then one bulk store of the
    // query's 64 x 512 block; warp w takes dims 32 (w % 4) .. + 31 of the
    // blocks 2 (w / 4), + 1
    const bool f32 = a.out_dtype == kF32;
    const int oeb = f32 ? 4 : 2;
    uint8_t* ost = Kt;  // 64 KB (bf16) or 128 KB (fp32)
    // rolled over (block, head half) and one loop body per output type: this
    // code runs once per CTA, and its instructions are fetched cold
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
      const int mt = 2 * (warp >> 2) + (i >> 1), hh = (i & 1) * 32;
      const int dim = mt * 128 + q4 * 32 + lane;
      uint32_t v[32];
      if (ntiles > 0) {
        tmem_ld32(dO + mt * kH + hh + (static_cast<uint32_t>(q4 * 32) << 16), v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int h = 0; h < 32; ++h) v[h] = 0u;
      }
      // the scales into registers before the first store (a shared-memory
      // load after a shared-memory store waits for it)
      float o[32];
#pragma unroll
      for (int h = 0; h < 32; h += 4) {
        const float4 f4 = *reinterpret_cast<const float4*>(fin + hh + h);
        o[h] = __uint_as_float(v[h]) * f4.x;
        o[h + 1] = __uint_as_float(v[h + 1]) * f4.y;
        o[h + 2] = __uint_as_float(v[h + 2]) * f4.z;
        o[h + 3] = __uint_as_float(v[h + 3]) * f4.w;
      }
      if (f32) {
#pragma unroll
        for (int h = 0; h < 32; ++h) reinterpret_cast<float*>(ost)[(hh + h) * kD + dim] = o[h];
      } else {
#pragma unroll
        for (int h = 0; h < 32; ++h) reinterpret_cast<uint16_t*>(ost)[(hh + h) * kD + dim] = f32_to_bf16_bits(o[h]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    char* obase = static_cast<char*>(a.out) + static_cast<int64_t>(qi) * kH * kD * oeb;
    if (a.out_bulk) {
      if (tid == 0) {
        const uint32_t bytes = static_cast<uint32_t>(kH * kD * oeb);
        for (uint32_t o = 0; o < bytes; o += 32768) bulk_store(obase + o, ost + o, 32768);
        bulk_store_wait_read();
      }
    } else if (f32) {
      for (int i = tid; i < kH * kD; i += kNT) reinterpret_cast<float*>(obase)[i] = reinterpret_cast<float*>(ost)[i];
    } else {
      for (int i = tid; i < kH * kD; i += kNT)
        reinterpret_cast<uint16_t*>(obase)[i] = reinterpret_cast<uint16_t*>(ost)[i];
    }
  }
  // every MMA of this CTA and the query's copy have completed before TMEM
  // is released and the CTA exits
  if (tid == 32) {
    mma_commit(mdone);
    mbar_wait(mdone, 0, kWaitLimit);
    if (ntiles > 0) mbar_wait(qbar, 0, kWaitLimit);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemColsM);
}

PFN_cuTensorMapEncodeTiled_v12000 many_attn_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

template <int FMT>
csa_status_t launch_many_fmt(const CUtensorMap& qmap, const AttnManyArgs& a, int nq, cudaStream_t stream) {
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(attn_many_tc_kernel<FMT>),
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemM);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  prof_begin(stream);
  attn_many_tc_kernel<FMT><<<nq, kNT, kSmemM, stream>>>(qmap, a);
  return check_launch("attn_many_tc_kernel", stream);
}

}  // namespace

// Many queries (no workspace): h_q = 64, d = 512, bf16 queries, bf16 window,
// main KV in bf16, FP8 (scale per 64) or MXFP4; the caller checked them.
csa_status_t launch_attention_many_tc(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                                      int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible,
                                      const int32_t* q_req, const csa_tensor_t* swa_k, const csa_tensor_t* swa_v,
                                      const int64_t* q_pos, const int64_t* swa_lo, const float* sink,
                                      const csa_tensor_t* out, float* lse, cudaStream_t stream) {
  if (nq == 0) return CSA_OK;
  if (!many_attn_encoder()) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap qmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(nq) * kH};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kH)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult cr = many_attn_encoder()(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q->data, dims, strides, box, estr,
                                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled (query) failed (%d)", (int)cr);
  AttnManyArgs a;
  a.kv = kv->data;
  a.kv_scale = kv->scale;
  a.batch = batch;
  a.cap = cap;
  a.idx = idx;
  a.topk = p->topk;
  a.n_visible = n_visible;
  a.q_req = q_req;
  a.swa_k = swa_k ? static_cast<const uint16_t*>(swa_k->data) : nullptr;
  a.swa_v = swa_v ? static_cast<const uint16_t*>(swa_v->data) : nullptr;
  a.swa_cap = p->swa_cap > 0 ? p->swa_cap : 1;
  a.window = p->window;
  a.q_pos = q_pos;
  a.swa_lo = swa_lo;
  a.tau = p->softmax_scale;
  a.sink = sink;
  a.out = out->data;
  a.out_dtype = out->dtype;
  a.out_bulk = (reinterpret_cast<uintptr_t>(out->data) & 15) == 0;
  a.lse = lse;
  if (kv->dtype == kMXFP4) return launch_many_fmt<kKvMX4>(qmap, a, nq, stream);
  if (kv->dtype == kFP8) return launch_many_fmt<kKvFP8>(qmap, a, nq, stream);
  return launch_many_fmt<kKvBF16>(qmap, a, nq, stream);
}

uint32_t attn_many_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_many_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_attn_many_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
