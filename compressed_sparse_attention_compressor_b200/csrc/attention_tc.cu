// K4 on the tensor cores: attention of 64 query heads (d = 512) over a list
// of selected compressed entries (CSA) or all visible entries (HCA), plus the
// sliding window, for few query tokens (decode).
//
// Atlas "Model architectures", "compressed KV" (CSA top-k entries plus a
// sliding window; HCA dense over the short stream) and "MLA" (the latent is
// key and value); tech-report tour, "The indexer selects, SWA covers the
// rest".
//
// One CTA takes 128 consecutive keys of one query's key list (selected
// entries, then window positions):
//   1. gather: the key rows are dequantised to bf16 into a K-major tile of
//      8 blocks x (128 rows x 128 B) with the 128-byte swizzle; the query
//      [64][512] arrives by TMA in the same layout;
//   2. S^T[128 keys][64 heads] = K Q^T  (tcgen05, M=128, N=64, K=512);
//   3. softmax statistics per head over the tile (logits transposed through
//      shared memory), P^T written as the bf16 B operand [64][128];
//      window rows of the tile are then overwritten with their value rows
//      (compressed entries are key and value at once);
//   4. O^T[512 dims][64 heads] = V^T P^T: the same tile read as an
//      MN-major A operand (4 M-tiles of 128 dims);
//   5. (max, sum, O) of the tile go to the split-state workspace; a merge
//      kernel combines the tiles of a query by their log-sum-exp and adds
//      the sink.
#include <cudaTypedefs.h>

#include <cstring>

#include <cooperative_groups.h>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

using namespace sm100;

constexpr int kTK = 128;       // keys per CTA
constexpr int kH = 64;         // query heads
constexpr int kD = 512;        // head dim
constexpr int kThreads = 256;  // 8 warps; warps 4..7 read TMEM
constexpr int kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 22;

// shared-memory layout
constexpr int oK = 0;                        // 8 x 16 KB key tile
constexpr int oQ = oK + 8 * kTK * 128;       // 8 x 8 KB query (later: logits, P^T, stats)
constexpr int oS = oQ;                       // fp32 logits [64 heads][4 blocks of 33] (after S is done)
constexpr int kSbStride = 4 * 33;            // padded head row: conflict-free writes and reads
constexpr int oP = oQ + (kH * kSbStride * 4 + 1023) / 1024 * 1024;  // 2 x 8 KB P^T
constexpr int oML = oP + 2 * kH * 128;       // per-head (max, sum)
constexpr int oEnt = oQ + 8 * kH * 128;      // [128] entry codes
constexpr int oBars = oEnt + kTK * 4;
constexpr int oMisc = oBars + 64;
constexpr int kSmem = oMisc + 64 + 1024;

constexpr uint32_t kIdescS = idesc(1, 1, kTK, kH);                     // bf16, K-major A and B
constexpr uint32_t kIdescO = idesc(1, 1, 128, kH) | (1u << 15);        // A MN-major

__device__ uint32_t g_attn_tc_error = 0;

struct AttnTcArgs {
  const void* kv; const float* kv_scale; int kv_fp8; int batch; int64_t cap;
  const int32_t* idx; int topk;   // idx == nullptr: dense over n_visible
  const int32_t* n_visible; const int32_t* q_req;
  const uint16_t* swa_k; const uint16_t* swa_v; int swa_cap; int window;
  const int64_t* q_pos; const int64_t* swa_lo;
  float tau;
  float* part;     // [nq][splits][64][512 + 2]: (m, l, O)
  int splits;
  // cluster path: the merged output
  const float* sink; void* out; int out_dtype; float* lse;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// MN-major, 128-byte swizzled operand: 64-element rows of 128 B along M,
// 8-row groups of K 1024 B apart, next 64 elements of M `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Writes 8 bf16 (one 16-byte chunk) of element block [e, e+8) of tile row r.
__device__ __forceinline__ void put_chunk(uint8_t* tile, int r, int e, uint4 v) {
  const int blk = e >> 6, ch = (e & 63) >> 3;
  *reinterpret_cast<uint4*>(tile + blk * (kTK * 128) + sw128_offset(r, ch)) = v;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return static_cast<uint32_t>(f32_to_bf16_bits(a)) | (static_cast<uint32_t>(f32_to_bf16_bits(b)) << 16);
}

// All threads: rows of the tile from their sources.  which = 0: keys
// (compressed entries and window keys); which = 1: only the window rows,
// from the value ring (compressed rows are their own values).  Loads are
// issued in batches of 8 per thread before any of them is used.
__device__ void gather_rows(uint8_t* tile, const int32_t* ent, const AttnTcArgs& a, int64_t kv_row0,
                            int64_t sw_row0, int which) {
  constexpr int B = 8;
  if (a.kv_fp8 && which == 0) {
    // FP8 entries: 32 tasks of 16 codes per row
    for (int t0 = threadIdx.x; t0 < kTK * 32; t0 += kThreads * B) {
      uint4 u[B];
      float sc[B];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int task = t0 + b * kThreads;
        const int r = task >> 5, c16 = task & 31;
        const int32_t e = task < kTK * 32 ? ent[r] : -1;
        u[b] = make_uint4(0, 0, 0, 0);
        sc[b] = 0.f;
        if (e >= 0) {
          const int64_t gr = kv_row0 + e;
          u[b] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.kv) + gr * kD) + c16);
          sc[b] = __ldg(a.kv_scale + gr * (kD / 64) + (c16 >> 2));
        }
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int task = t0 + b * kThreads;
        const int r = task >> 5, c16 = task & 31;
        if (task >= kTK * 32 || ent[r] < 0) continue;
        const uint32_t w[4] = {u[b].x, u[b].y, u[b].z, u[b].w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 lo = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] & 0xFFFF));
          const float2 hi = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] >> 16));
          o[2 * i] = pack_bf16(lo.x * sc[b], lo.y * sc[b]);
          o[2 * i + 1] = pack_bf16(hi.x * sc[b], hi.y * sc[b]);
        }
        put_chunk(tile, r, c16 * 16, make_uint4(o[0], o[1], o[2], o[3]));
        put_chunk(tile, r, c16 * 16 + 8, make_uint4(o[4], o[5], o[6], o[7]));
      }
    }
  }
  // bf16 rows (compressed bf16 entries, window keys or values): 64 tasks of 8 elements per row
  for (int t0 = threadIdx.x; t0 < kTK * 64; t0 += kThreads * B) {
    uint4 v[B];
    bool put[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kThreads;
      const int r = task >> 6, c8 = task & 63;
      const int32_t e = task < kTK * 64 ? ent[r] : -1;
      v[b] = make_uint4(0, 0, 0, 0);
      put[b] = task < kTK * 64;
      if (e >= 0) {
        if (a.kv_fp8 || which == 1) put[b] = false;  // FP8 rows done above; compressed rows keep their keys
        else v[b] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.kv) + (kv_row0 + e) * kD) + c8);
      } else if (e <= -2) {
        const uint16_t* src = (which == 0 ? a.swa_k : a.swa_v) + (sw_row0 + (-2 - e)) * kD;
        v[b] = __ldg(reinterpret_cast<const uint4*>(src) + c8);
      } else if (which == 1) {
        put[b] = false;
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kThreads;
      if (put[b]) put_chunk(tile, task >> 6, (task & 63) * 8, v[b]);
    }
  }
}

// CLUSTER = false: one CTA per 128-key split of a query's key list, the
// split's (max, sum, O) to the global workspace, merged by another kernel.
// CLUSTER = true: the gridDim.x CTAs of one cluster serve one query; CTA r
// takes the r-th even slice of the selected entries and of the window, keeps
// its (max, sum, O) in its own shared memory, and the cluster merges them
// through distributed shared memory (CTA r finishes heads r, r + R, ...).
// Cluster path, all threads: the tile's rows [0, nsr) from their compressed
// entries (FP8 dequantised to bf16) and rows [nsr, nsr + nwr) from the
// window keys, every load of a batch of 16 per thread issued before any is
// used; the window rows' values go to vw[] (registers) in the same batch
// (nwr <= 16), to replace the keys once the logits are out.  Rows
// [nsr + nwr, nk16) are zeroed (the PV product reads them with weight 0).
__device__ void gather_cluster(uint8_t* tile, const int32_t* ent, const AttnTcArgs& a, int64_t kv_row0,
                               int64_t sw_row0, int nsr, int nwr, int nk16, uint4 (&vw)[4]) {
  const int per_sel = a.kv_fp8 ? 32 : 64;  // 16-byte chunks per selected row
  const int T1 = nsr * per_sel, T = T1 + nwr * 64;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int task = threadIdx.x + b * kThreads;
    vw[b] = make_uint4(0, 0, 0, 0);
    if (task < nwr * 64) {
      const int e = ent[nsr + (task >> 6)];
      if (e <= -2) vw[b] = __ldg(reinterpret_cast<const uint4*>(a.swa_v + (sw_row0 + (-2 - e)) * kD) + (task & 63));
    }
  }
  constexpr int B = 16;
  for (int t0 = threadIdx.x; t0 < T; t0 += kThreads * B) {
    uint4 u[B];
    float sc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kThreads;
      u[b] = make_uint4(0, 0, 0, 0);
      sc[b] = 0.f;
      if (task < T1) {
        const int r = task / per_sel, c = task % per_sel;
        const int32_t e = ent[r];
        if (e >= 0) {
          const int64_t gr = kv_row0 + e;
          if (a.kv_fp8) {
            u[b] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.kv) + gr * kD) + c);
            sc[b] = __ldg(a.kv_scale + gr * (kD / 64) + (c >> 2));
          } else {
            u[b] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.kv) + gr * kD) + c);
          }
        }
      } else if (task < T) {
        const int w = task - T1;
        const int32_t e = ent[nsr + (w >> 6)];
        if (e <= -2) u[b] = __ldg(reinterpret_cast<const uint4*>(a.swa_k + (sw_row0 + (-2 - e)) * kD) + (w & 63));
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kThreads;
      if (task < T1) {
        const int r = task / per_sel, c = task % per_sel;
        if (a.kv_fp8) {
          const uint32_t w[4] = {u[b].x, u[b].y, u[b].z, u[b].w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 lo = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] & 0xFFFF));
            const float2 hi = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] >> 16));
            const __nv_bfloat162 bl = __floats2bfloat162_rn(lo.x * sc[b], lo.y * sc[b]);
            const __nv_bfloat162 bh = __floats2bfloat162_rn(hi.x * sc[b], hi.y * sc[b]);
            o[2 * i] = *reinterpret_cast<const uint32_t*>(&bl);
            o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&bh);
          }
          put_chunk(tile, r, c * 16, make_uint4(o[0], o[1], o[2], o[3]));
          put_chunk(tile, r, c * 16 + 8, make_uint4(o[4], o[5], o[6], o[7]));
        } else {
          put_chunk(tile, r, c * 8, u[b]);
        }
      } else if (task < T) {
        const int w = task - T1;
        put_chunk(tile, nsr + (w >> 6), (w & 63) * 8, u[b]);
      }
    }
  }
  // zero rows between the last valid key and the next multiple of 16
  for (int task = (nsr + nwr) * 64 + threadIdx.x; task < nk16 * 64; task += kThreads)
    put_chunk(tile, task >> 6, (task & 63) * 8, make_uint4(0, 0, 0, 0));
}

template <bool CLUSTER>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* Kt = smem + oK;
  float* Sb = reinterpret_cast<float*>(smem + oS);
  uint8_t* Pt = smem + oP;
  float* ml = reinterpret_cast<float*>(smem + oML);
  int32_t* ent = reinterpret_cast<int32_t*>(smem + oEnt);
  uint64_t* qbar = reinterpret_cast<uint64_t*>(smem + oBars);
  uint64_t* sbar = qbar + 1;
  uint64_t* obar = qbar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + oMisc);
  int* s_flags = reinterpret_cast<int*>(smem + oMisc + 16);  // [0] any window row, [1] failed

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qi = blockIdx.y, split = blockIdx.x;
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
  const int x0 = split * kTK;
  // cluster slices: selected [s0, s1), window [w0, w1) (window offsets)
  const int R = static_cast<int>(gridDim.x);
  const int s0 = live ? static_cast<int>(static_cast<int64_t>(split) * n_sel / R) : 0;
  const int s1 = live ? static_cast<int>(static_cast<int64_t>(split + 1) * n_sel / R) : 0;
  const int w0 = live ? static_cast<int>(static_cast<int64_t>(split) * n_win / R) : 0;
  const int w1 = live ? static_cast<int>(static_cast<int64_t>(split + 1) * n_win / R) : 0;
  const int64_t kv_row0 = live ? static_cast<int64_t>(r) * a.cap : 0;
  const int64_t sw_row0 = live ? static_cast<int64_t>(r) * a.swa_cap : 0;
  float* pp = a.part + (static_cast<int64_t>(qi) * a.splits + split) * kH * (kD + 2);

  if (!CLUSTER && x0 >= total) {  // an empty split: m = -inf
    for (int h = tid; h < kH; h += kThreads) {
      pp[h * (kD + 2)] = -INFINITY;
      pp[h * (kD + 2) + 1] = 0.f;
    }
    return;
  }

  if (tid == 0) {
    mbar_init(qbar, 1);
    mbar_init(sbar, 1);
    mbar_init(obar, 1);
    s_flags[0] = 0;
    s_flags[1] = 0;
    fence_barrier_init();
  }
  if (tid < kTK) {
    int32_t e = -1;
    int xs = -1, xw = -1;  // selected-list position / window offset of this row
    if (CLUSTER) {
      if (tid < s1 - s0) xs = s0 + tid;
      else if (tid < (s1 - s0) + (w1 - w0)) xw = w0 + tid - (s1 - s0);
    } else {
      const int x = x0 + tid;
      if (x < total) {
        if (x < n_sel) xs = x;
        else xw = x - n_sel;
      }
    }
    if (xs >= 0) {
      const int32_t j = a.idx ? a.idx[static_cast<int64_t>(qi) * a.topk + xs] : xs;
      e = (j >= 0 && j < nv) ? j : -1;
    } else if (xw >= 0) {
      e = -2 - static_cast<int32_t>((p_lo + xw) % a.swa_cap);
    }
    ent[tid] = e;
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(qbar, kH * kD * 2);
    for (int blk = 0; blk < 8; ++blk) tma_load_2d(smem + oQ + blk * kH * 128, &qmap, qbar, blk * 64, qi * kH);
  }
  if (tid < kTK && ent[tid] <= -2) s_flags[0] = 1;
  const int nsr = s1 - s0, nwr = w1 - w0;
  const int nk16 = CLUSTER ? ((nsr + nwr + 15) & ~15) : kTK;  // keys the PV product covers
  const bool vregs = CLUSTER && nwr <= 16;                     // window values held in registers
  uint4 vw[4];
  if (vregs) gather_cluster(Kt, ent, a, kv_row0, sw_row0, nsr, nwr, nk16, vw);
  else gather_rows(Kt, ent, a, kv_row0, sw_row0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t dS = tmem, dO = tmem + kH;

  // ---- S^T = K Q^T ----
  if (tid == 32) {
    if (!mbar_wait(qbar, 0, kWaitLimit)) {
      atomicOr(&g_attn_tc_error, 1u);
      s_flags[1] = 1;
    }
    tc_fence_after();
    const uint32_t kb = smem_u32(Kt), qb = smem_u32(smem + oQ);
#pragma unroll
    for (int blk = 0; blk < 8; ++blk)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f16(dS, desc_k_sw128(kb + blk * kTK * 128 + kk * 32), desc_k_sw128(qb + blk * kH * 128 + kk * 32),
                kIdescS, (blk | kk) ? 1u : 0u);
    mma_commit(sbar);
  }
  // logits -> shared memory, transposed to [head][key]; one thread polls
  // the MMA's barrier and the CTA barrier releases the others
  if (tid == 0 && !mbar_wait(sbar, 0, kWaitLimit)) {
    atomicOr(&g_attn_tc_error, 1u);
    s_flags[1] = 1;
  }
  __syncthreads();
  tc_fence_after();
  if (warp >= 4) {
    const int sub = warp & 3, row = sub * 32 + lane;
    const uint32_t ta = dS + (static_cast<uint32_t>(sub * 32) << 16);
    uint32_t v0[32], v1[32];
    tmem_ld32(ta, v0);
    tmem_ld32(ta + 32, v1);
    tmem_wait_ld();
    const bool ok = ent[row] != -1;
#pragma unroll
    for (int h = 0; h < 32; ++h) {
      Sb[h * kSbStride + sub * 33 + lane] = ok ? __uint_as_float(v0[h]) * a.tau : -INFINITY;
      Sb[(32 + h) * kSbStride + sub * 33 + lane] = ok ? __uint_as_float(v1[h]) * a.tau : -INFINITY;
    }
  }
  __syncthreads();
  // window rows: values replace keys in the tile (the S MMA has read it)
  if (vregs) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int task = tid + b * kThreads;
      if (task < nwr * 64) put_chunk(Kt, nsr + (task >> 6), (task & 63) * 8, vw[b]);
    }
  } else if (s_flags[0]) {
    gather_rows(Kt, ent, a, kv_row0, sw_row0, 1);
  }
  // softmax statistics and P^T: four threads per head, 32 keys each
  {
    const int h = tid >> 2, q4 = tid & 3;
    const float* srow = Sb + h * kSbStride + q4 * 33;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, srow[i]);
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    float sum = 0.f;
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float p0 = (m == -INFINITY) ? 0.f : __expf(srow[i] - m);
      const float p1 = (m == -INFINITY) ? 0.f : __expf(srow[i + 1] - m);
      sum += p0 + p1;
      pk[i >> 1] = pack_bf16(p0, p1);
    }
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    // keys q4*32 .. +31 of row h: K-major blocks of 64 keys
    const int k0 = q4 * 32;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int kk = k0 + c * 8;
      *reinterpret_cast<uint4*>(Pt + (kk >> 6) * (kH * 128) + sw128_offset(h, (kk & 63) >> 3)) =
          make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    }
    if (q4 == 0) {
      ml[2 * h] = m;
      ml[2 * h + 1] = sum;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- O^T = V^T P^T ----
  if (tid == 32) {
    const uint32_t kb = smem_u32(Kt), pb = smem_u32(Pt);
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int kk = 0; kk < nk16 / 16; ++kk)
        mma_f16(dO + mt * kH, desc_mn_sw128(kb + (2 * mt) * kTK * 128 + kk * 16 * 128, kTK * 128),
                desc_k_sw128(pb + (kk >> 2) * kH * 128 + (kk & 3) * 32), kIdescO, kk > 0 ? 1u : 0u);
    mma_commit(obar);
  }
  if (!CLUSTER && tid < kH) {
    pp[tid * (kD + 2)] = ml[2 * tid];
    pp[tid * (kD + 2) + 1] = ml[2 * tid + 1];
  }
  if (tid == 0 && !mbar_wait(obar, 0, kWaitLimit)) {
    atomicOr(&g_attn_tc_error, 1u);
    s_flags[1] = 1;
  }
  __syncthreads();
  tc_fence_after();
  if constexpr (!CLUSTER) {
    if (warp >= 4) {
      const int sub = warp & 3;
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        const uint32_t ta = dO + mt * kH + (static_cast<uint32_t>(sub * 32) << 16);
        uint32_t v0[32], v1[32];
        tmem_ld32(ta, v0);
        tmem_ld32(ta + 32, v1);
        tmem_wait_ld();
        const int dim = mt * 128 + sub * 32 + lane;
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          pp[h * (kD + 2) + 2 + dim] = __uint_as_float(v0[h]);
          pp[(32 + h) * (kD + 2) + 2 + dim] = __uint_as_float(v1[h]);
        }
      }
    }
  } else {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    // this CTA's O (unnormalised) into its own shared memory as [head][dim]
    // fp32, over the key tile (both MMAs have completed)
    float* Osm = reinterpret_cast<float*>(smem + oK);
    {
      const int sub = warp & 3, mh = warp >> 2;  // two warps per TMEM lane quarter
#pragma unroll 1
      for (int mt = mh * 2; mt < mh * 2 + 2; ++mt) {
        const uint32_t ta = dO + mt * kH + (static_cast<uint32_t>(sub * 32) << 16);
        uint32_t v0[32], v1[32];
        tmem_ld32(ta, v0);
        tmem_ld32(ta + 32, v1);
        tmem_wait_ld();
        const int dim = mt * 128 + sub * 32 + lane;
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          Osm[h * kD + dim] = __uint_as_float(v0[h]);
          Osm[(32 + h) * kD + dim] = __uint_as_float(v1[h]);
        }
      }
    }
    cluster.sync();
    // heads split + r * R for r = 0, 1, ...: warp w weighs head split + w R
    float* wgt = reinterpret_cast<float*>(smem + oS);  // [head][16 CTAs], then [head][2] (M, 1/L); logits are dead
    const int nh = (kH - split + R - 1) / R;
    for (int w = warp; w < nh; w += kThreads / 32) {
      const int h = split + w * R;
      float mj = -INFINITY, lj = 0.f;
      if (lane < R) {
        const float* pml = cluster.map_shared_rank(ml, lane);
        mj = pml[2 * h];
        lj = pml[2 * h + 1];
      }
      const float sk = a.sink ? a.sink[h] : -INFINITY;
      const float M = fmaxf(warp_max(mj), sk);
      const float wj = (mj == -INFINITY) ? 0.f : __expf(mj - M);
      float L = warp_sum(wj * lj);
      if (sk != -INFINITY) L += __expf(sk - M);
      if (lane < R) wgt[w * 16 + lane] = wj;
      if (lane == 0) {
        wgt[kH * 16 + w * 2] = M;
        wgt[kH * 16 + w * 2 + 1] = (M == -INFINITY) ? 0.f : 1.f / L;
        if (a.lse) a.lse[static_cast<int64_t>(qi) * kH + h] = (M == -INFINITY) ? -INFINITY : M + __logf(L);
      }
    }
    __syncthreads();
    // two consecutive dims per thread, R peers each
    for (int w = 0; w < nh; ++w) {
      const int h = split + w * R;
      const int dim = tid * 2;
      float2 v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)  // every peer's load in flight before the sums
        if (j < R) v[j] = *reinterpret_cast<const float2*>(cluster.map_shared_rank(Osm, j) + h * kD + dim);
      float o0 = 0.f, o1 = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < R) {
          const float wj = wgt[w * 16 + j];
          o0 = fmaf(wj, v[j].x, o0);
          o1 = fmaf(wj, v[j].y, o1);
        }
      const float inv = wgt[kH * 16 + w * 2 + 1];
      o0 *= inv;
      o1 *= inv;
      const int64_t off = (static_cast<int64_t>(qi) * kH + h) * kD + dim;
      if (a.out_dtype == kF32) {
        *reinterpret_cast<float2*>(static_cast<float*>(a.out) + off) = make_float2(o0, o1);
      } else {
        *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.out) + off) = pack_bf16(o0, o1);
      }
    }
    cluster.sync();  // every peer has read this CTA's partial
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

struct TcLauncher {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  bool attr[2] = {false, false};
  int cluster_ok[17] = {0};  // per cluster size: 0 unknown, else co-resident clusters (-1: none)
};

TcLauncher& tc_launcher() {
  static TcLauncher L;
  if (!L.encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      L.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return L;
}

}  // namespace

int attn_tc_splits(int max_keys) { return (max_keys + kTK - 1) / kTK; }

// Smallest cluster whose even slices of `sel_max` selected entries and
// `window` window positions fit one 128-key tile per CTA; 0 if none <= 16.
int attn_cluster_min(int sel_max, int window) {
  for (int r = 1; r <= 16; ++r)
    if ((sel_max + r - 1) / r + (window + r - 1) / r <= kTK) return r;
  return 0;
}

bool attn_tc_supported(const csa_params_t* p, int q_dtype, int kv_dtype, int swa_dtype, bool has_window) {
  if (p->h_q != kH || p->d != kD || q_dtype != kBF16) return false;
  if (kv_dtype != kBF16 && !(kv_dtype == kFP8)) return false;
  if (has_window && swa_dtype != kBF16) return false;
  return true;
}

size_t attn_tc_workspace_bytes(int nq, int max_keys) {
  return static_cast<size_t>(nq) * attn_tc_splits(max_keys) * kH * (kD + 2) * sizeof(float);
}

csa_status_t launch_attn_merge(const float* part, int nq, int n_splits, int hq, int d, const float* sink, void* out,
                               int out_dtype, float* lse, cudaStream_t stream);

csa_status_t launch_attention_tc(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                                 int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible,
                                 const int32_t* q_req, const csa_tensor_t* swa_k, const csa_tensor_t* swa_v,
                                 const int64_t* q_pos, const int64_t* swa_lo, const float* sink,
                                 const csa_tensor_t* out, float* lse, void* workspace, int max_keys,
                                 cudaStream_t stream) {
  TcLauncher& L = tc_launcher();
  if (!L.encode) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap qmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(nq) * kH};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kH)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = L.encode(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q->data, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled (query) failed (%d)", (int)cr);
  AttnTcArgs a;
  a.kv = kv->data;
  a.kv_scale = kv->scale;
  a.kv_fp8 = kv->dtype == kFP8;
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
  a.part = static_cast<float*>(workspace);
  a.splits = attn_tc_splits(max_keys);
  a.sink = sink;
  a.out = out->data;
  a.out_dtype = out->dtype;
  a.lse = lse;
  for (int c = 0; c < 2; ++c)
    if (!L.attr[c]) {
      void* fn = c ? reinterpret_cast<void*>(attn_tc_kernel<true>) : reinterpret_cast<void*>(attn_tc_kernel<false>);
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
      if (e == cudaSuccess && c) e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      L.attr[c] = true;
    }
  // One cluster per query when its keys fit 16 CTAs of one tile each: the
  // largest size (least work per CTA) whose nq clusters are co-resident.
  const int rmin = attn_cluster_min(max_keys - p->window, p->window);
  int R = 0;
  for (int r = 16; rmin > 0 && r >= rmin && R == 0; --r) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(r, nq);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = r;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (L.cluster_ok[r] == 0) {
      int ncl = 0;
      const cudaError_t e = cudaOccupancyMaxActiveClusters(&ncl, attn_tc_kernel<true>, &cfg);
      L.cluster_ok[r] = (e == cudaSuccess && ncl >= 1) ? ncl : -1;
      cudaGetLastError();
    }
    if (L.cluster_ok[r] >= nq || (r == rmin && L.cluster_ok[r] > 0)) R = r;
  }
  if (R > 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(R, nq);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = R;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
      prof_begin(stream);
      const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<true>, qmap, a);
      if (e != cudaSuccess) {
        check_launch("attn_tc_cluster_kernel", stream);
        return set_error(CSA_ERR_CUDA, "attn_tc_kernel (cluster) launch: %s", cudaGetErrorString(e));
      }
      return check_launch("attn_tc_cluster_kernel", stream);
    }
  }
  prof_begin(stream);
  attn_tc_kernel<false><<<dim3(a.splits, nq), kThreads, kSmem, stream>>>(qmap, a);
  csa_status_t st = check_launch("attn_tc_kernel", stream);
  if (st != CSA_OK) return st;
  return launch_attn_merge(a.part, nq, a.splits, kH, kD, sink, out->data, out->dtype, lse, stream);
}

uint32_t attn_tc_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_tc_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_attn_tc_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
