// One attention tile on the tensor cores: the 64 query heads (d = 512) of
// one query over up to 128 keys -- selected compressed entries (K = V = the
// latent, FP8 or MXFP4 dequantised to bf16) and sliding-window positions (separate K
// and V) -- with the unnormalised result left in TMEM and the per-head
// softmax statistics in shared memory.  Used by the stand-alone attention
// kernels and by the decode step's fused indexer.
//
// Atlas "Model architectures", "compressed KV" (CSA top-k entries plus a
// sliding window) and "MLA" (the latent is key and value); tech-report tour,
// "The indexer selects, SWA covers the rest".
//
//   S^T[128 keys][64 heads] = K Q^T         (tcgen05, M = 128, N = 64, K = 512)
//   logits -> shared memory, softmax statistics per head, P^T in bf16
//   (window rows' keys are then replaced by their values in the tile)
//   O^T[512 dims][64 heads] = V^T P^T       (the tile as an MN-major A operand)
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace attn {
namespace {  // per translation unit

using namespace sm100;

constexpr int kTK = 128;  // keys per tile
constexpr int kH = 64;    // query heads
constexpr int kD = 512;   // head dim
constexpr int kNT = 256;  // threads taking part (warps 0..7; warps 4..7 read TMEM)

// shared-memory layout, relative to a 1024-byte aligned base
constexpr int oK = 0;                        // 8 x 16 KB key / value tile
constexpr int oQ = oK + 8 * kTK * 128;       // 8 x 8 KB query (later: logits, P^T, stats)
constexpr int oS = oQ;                       // fp32 logits [64 heads][4 blocks of 33] (after S is done)
constexpr int kSbStride = 4 * 33;            // padded head row: conflict-free writes and reads
constexpr int oP = oQ + (kH * kSbStride * 4 + 1023) / 1024 * 1024;  // 2 x 8 KB P^T
constexpr int oML = oP + 2 * kH * 128;       // per-head (max, sum)
constexpr int oEnt = oQ + 8 * kH * 128;      // [128] entry codes
constexpr int kTileSmem = oEnt + kTK * 4;    // bytes the tile uses from the base

constexpr uint32_t kIdescS = idesc(1, 1, kTK, kH);               // bf16, K-major A and B
constexpr uint32_t kIdescO = idesc(1, 1, 128, kH) | (1u << 15);  // A MN-major
constexpr uint32_t kWaitLimit = 1u << 22;

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

// Two floats -> two bf16 (round to nearest even), a in the low half: one
// packed conversion.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Storage of the compressed rows.
constexpr int kKvBF16 = 0;
constexpr int kKvFP8 = 1;   // E4M3 codes, one fp32 scale per 64 elements
constexpr int kKvMX4 = 2;   // E2M1 codes (two per byte), one E4M3 scale byte per 16 elements

// Where the tile's rows come from: entry codes e >= 0 name compressed row
// kv_row0 + e, e <= -2 window slot sw_row0 + (-2 - e), e = -1 nothing.
struct Src {
  const void* kv;
  const void* kv_scale;   // FP8: fp32 scales; MXFP4: E4M3 scale bytes
  const uint32_t* lut;    // MXFP4: shared-memory table, code byte -> its two E2M1 values as bf16x2
  const uint16_t* swa_k;
  const uint16_t* swa_v;
  int64_t kv_row0;
  int64_t sw_row0;
  float tau;
};

// One 16-byte chunk of a quantised compressed row with its scale(s): FP8, 16
// codes and their fp32 scale; MXFP4, 32 codes and the two scale bytes of
// their 16-element groups.
struct QChunk {
  uint4 u;
  uint32_t s;
};

// 16-byte chunks of one compressed row: bf16 64, FP8 32, MXFP4 16.
template <int FMT>
constexpr int chunks_per_row() { return FMT == kKvBF16 ? kD / 8 : FMT == kKvFP8 ? kD / 16 : kD / 32; }

template <int FMT>
__device__ __forceinline__ QChunk load_qchunk(const Src& a, int64_t gr, int c) {
  QChunk q;
  if constexpr (FMT == kKvMX4) {
    q.u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.kv) + gr * (kD / 2)) + c);
    q.s = __ldg(reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(a.kv_scale) + gr * (kD / 16)) + c);
  } else {
    q.u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.kv) + gr * kD) + c);
    q.s = __float_as_uint(__ldg(static_cast<const float*>(a.kv_scale) + gr * (kD / 64) + (c >> 2)));
  }
  return q;
}

// The MXFP4 table: byte b -> bf16x2 (E2M1 value of its low nibble, of its
// high nibble).  All threads of the block; visible after the next barrier.
__device__ __forceinline__ void fill_mx4_lut(uint32_t* lut) {
  for (int b = static_cast<int>(threadIdx.x); b < 256; b += static_cast<int>(blockDim.x))
    lut[b] = pack_bf16(e2m1_to_f32(static_cast<uint32_t>(b) & 0xFu), e2m1_to_f32(static_cast<uint32_t>(b) >> 4));
}

// Dequantises chunk c of a row into tile row r as bf16.  MXFP4: a table
// lookup per code byte and one bf16x2 multiply by the group scale, exact (an
// E2M1 value times an E4M3 scale has at most 5 significant bits, and both
// factors are exact in bf16).
template <int FMT>
__device__ __forceinline__ void put_qchunk(uint8_t* tile, int r, int c, const QChunk& q, const uint32_t* lut) {
  const uint32_t w[4] = {q.u.x, q.u.y, q.u.z, q.u.w};
  if constexpr (FMT == kKvMX4) {
    const __nv_bfloat162 s0 = __float2bfloat162_rn(e4m3_to_f32(static_cast<uint8_t>(q.s & 0xFF)));
    const __nv_bfloat162 s1 = __float2bfloat162_rn(e4m3_to_f32(static_cast<uint8_t>(q.s >> 8)));
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // word i: elements 8i .. 8i+7 (byte k: elements 8i+2k, 8i+2k+1)
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t two = lut[(w[i] >> (8 * k)) & 0xFFu];
        const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&two), i < 2 ? s0 : s1);
        o[k] = *reinterpret_cast<const uint32_t*>(&v);
      }
      put_chunk(tile, r, c * 32 + i * 8, make_uint4(o[0], o[1], o[2], o[3]));
    }
  } else {
    const float sc = __uint_as_float(q.s);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 lo = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] & 0xFFFF));
      const float2 hi = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] >> 16));
      o[2 * i] = pack_bf16(lo.x * sc, lo.y * sc);
      o[2 * i + 1] = pack_bf16(hi.x * sc, hi.y * sc);
    }
    put_chunk(tile, r, c * 16, make_uint4(o[0], o[1], o[2], o[3]));
    put_chunk(tile, r, c * 16 + 8, make_uint4(o[4], o[5], o[6], o[7]));
  }
}

// All threads: rows of the tile from their sources.  which = 0: keys
// (compressed entries and window keys); which = 1: only the window rows,
// from the value ring (compressed rows are their own values).  Loads are
// issued in batches of 8 per thread before any of them is used.
template <int FMT>
__device__ void gather_rows(uint8_t* tile, const int32_t* ent, const Src& a, int which) {
  constexpr int B = 8;
  if (FMT != kKvBF16 && which == 0) {
    // quantised entries: tpr tasks of one 16-byte chunk per row
    constexpr int tpr = chunks_per_row<FMT>();
    for (int t0 = static_cast<int>(threadIdx.x); t0 < kTK * tpr; t0 += kNT * B) {
      QChunk q[B];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int task = t0 + b * kNT;
        const int r = task / tpr, c = task % tpr;
        const int32_t e = task < kTK * tpr ? ent[r] : -1;
        q[b].u = make_uint4(0, 0, 0, 0);
        q[b].s = 0u;
        if (e >= 0) q[b] = load_qchunk<FMT>(a, a.kv_row0 + e, c);
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int task = t0 + b * kNT;
        const int r = task / tpr, c = task % tpr;
        if (task >= kTK * tpr || ent[r] < 0) continue;
        put_qchunk<FMT>(tile, r, c, q[b], a.lut);
      }
    }
  }
  // bf16 rows (compressed bf16 entries, window keys or values): 64 tasks of 8 elements per row
  for (int t0 = static_cast<int>(threadIdx.x); t0 < kTK * 64; t0 += kNT * B) {
    uint4 v[B];
    bool put[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kNT;
      const int r = task >> 6, c8 = task & 63;
      const int32_t e = task < kTK * 64 ? ent[r] : -1;
      v[b] = make_uint4(0, 0, 0, 0);
      put[b] = task < kTK * 64;
      if (e >= 0) {
        if (FMT != kKvBF16 || which == 1) put[b] = false;  // quantised rows done above; compressed rows keep their keys
        else v[b] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.kv) + (a.kv_row0 + e) * kD) + c8);
      } else if (e <= -2) {
        const uint16_t* src = (which == 0 ? a.swa_k : a.swa_v) + (a.sw_row0 + (-2 - e)) * kD;
        v[b] = __ldg(reinterpret_cast<const uint4*>(src) + c8);
      } else if (which == 1) {
        put[b] = false;
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kNT;
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
template <int FMT>
__device__ void gather_cluster(uint8_t* tile, const int32_t* ent, const Src& a, int nsr, int nwr, int nk16,
                               uint4 (&vw)[4]) {
  constexpr int per_sel = chunks_per_row<FMT>();  // 16-byte chunks per selected row
  const int T1 = nsr * per_sel, T = T1 + nwr * 64;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int task = static_cast<int>(threadIdx.x) + b * kNT;
    vw[b] = make_uint4(0, 0, 0, 0);
    if (task < nwr * 64) {
      const int e = ent[nsr + (task >> 6)];
      if (e <= -2) vw[b] = __ldg(reinterpret_cast<const uint4*>(a.swa_v + (a.sw_row0 + (-2 - e)) * kD) + (task & 63));
    }
  }
  constexpr int B = 16;
  for (int t0 = static_cast<int>(threadIdx.x); t0 < T; t0 += kNT * B) {
    QChunk q[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kNT;
      q[b].u = make_uint4(0, 0, 0, 0);
      q[b].s = 0u;
      if (task < T1) {
        const int r = task / per_sel, c = task % per_sel;
        const int32_t e = ent[r];
        if (e >= 0) {
          const int64_t gr = a.kv_row0 + e;
          if constexpr (FMT != kKvBF16)
            q[b] = load_qchunk<FMT>(a, gr, c);
          else
            q[b].u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.kv) + gr * kD) + c);
        }
      } else if (task < T) {
        const int w = task - T1;
        const int32_t e = ent[nsr + (w >> 6)];
        if (e <= -2) q[b].u = __ldg(reinterpret_cast<const uint4*>(a.swa_k + (a.sw_row0 + (-2 - e)) * kD) + (w & 63));
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const int task = t0 + b * kNT;
      if (task < T1) {
        const int r = task / per_sel, c = task % per_sel;
        if constexpr (FMT != kKvBF16)
          put_qchunk<FMT>(tile, r, c, q[b], a.lut);
        else
          put_chunk(tile, r, c * 8, q[b].u);
      } else if (task < T) {
        const int w = task - T1;
        put_chunk(tile, nsr + (w >> 6), (w & 63) * 8, q[b].u);
      }
    }
  }
  // zero rows between the last valid key and the next multiple of 16
  for (int task = (nsr + nwr) * 64 + static_cast<int>(threadIdx.x); task < nk16 * 64; task += kNT)
    put_chunk(tile, task >> 6, (task & 63) * 8, make_uint4(0, 0, 0, 0));
}

// Threads 0 .. kNT-1 only (the others must not call it); `bar` is a named
// barrier over exactly those threads.  On entry ent[] (at oEnt) holds the
// tile's entry codes and is visible to all of them, the query's TMA (8 boxes
// into oQ) has been issued on qbar, and sbar / obar are fresh mbarriers.
// contiguous: rows [0, nsr) are selected entries and [nsr, nsr + nwr) window
// positions (one batched gather, window values in registers while nwr <= 16;
// the PV product covers the first nsr + nwr keys rounded up to 16); otherwise
// any layout of the 128 rows (two-pass gather, all 128 keys).  On return,
// ml = (max, sum) per head at oML and O^T in TMEM columns dO .. dO + 255
// (unnormalised, lanes = dims mod 128); on a bounded-wait timeout *fail = 1
// and bit 0 of *err is set.
template <int FMT>
__device__ void attend_tile(uint8_t* smem, const Src& s, bool contiguous, int nsr, int nwr, bool any_window,
                            uint64_t* qbar, uint64_t* sbar, uint64_t* obar, uint32_t dS, uint32_t dO, int bar,
                            int* fail, uint32_t* err) {
  uint8_t* Kt = smem + oK;
  float* Sb = reinterpret_cast<float*>(smem + oS);
  uint8_t* Pt = smem + oP;
  float* ml = reinterpret_cast<float*>(smem + oML);
  const int32_t* ent = reinterpret_cast<const int32_t*>(smem + oEnt);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk16 = contiguous ? ((nsr + nwr + 15) & ~15) : kTK;  // keys the PV product covers
  const bool vregs = contiguous && nwr <= 16;                       // window values held in registers
  uint4 vw[4];
  if (vregs) gather_cluster<FMT>(Kt, ent, s, nsr, nwr, nk16, vw);
  else gather_rows<FMT>(Kt, ent, s, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  named_barrier(bar, kNT);
  tc_fence_after();

  // ---- S^T = K Q^T ----
  if (tid == 32) {
    if (!mbar_wait(qbar, 0, kWaitLimit)) {
      atomicOr(err, 1u);
      *fail = 1;
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
  // the MMA's barrier and the named barrier releases the others
  if (tid == 0 && !mbar_wait(sbar, 0, kWaitLimit)) {
    atomicOr(err, 1u);
    *fail = 1;
  }
  named_barrier(bar, kNT);
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
      Sb[h * kSbStride + sub * 33 + lane] = ok ? __uint_as_float(v0[h]) * s.tau : -INFINITY;
      Sb[(32 + h) * kSbStride + sub * 33 + lane] = ok ? __uint_as_float(v1[h]) * s.tau : -INFINITY;
    }
  }
  named_barrier(bar, kNT);
  // window rows: values replace keys in the tile (the S MMA has read it)
  if (vregs) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int task = tid + b * kNT;
      if (task < nwr * 64) put_chunk(Kt, nsr + (task >> 6), (task & 63) * 8, vw[b]);
    }
  } else if (any_window) {
    gather_rows<FMT>(Kt, ent, s, 1);
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
    // keys q4*32 .. +31 of row h into P^T (K-major blocks of 64 keys), eight
    // at a time: a rolled loop, since this code runs once per launch and
    // every instruction of it is fetched cold
    const int k0 = q4 * 32;
    const float mm = (m == -INFINITY) ? 0.f : m;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float p0 = (m == -INFINITY) ? 0.f : __expf(srow[c * 8 + 2 * u] - mm);
        const float p1 = (m == -INFINITY) ? 0.f : __expf(srow[c * 8 + 2 * u + 1] - mm);
        sum += p0 + p1;
        pk[u] = pack_bf16(p0, p1);
      }
      const int kk = k0 + c * 8;
      *reinterpret_cast<uint4*>(Pt + (kk >> 6) * (kH * 128) + sw128_offset(h, (kk & 63) >> 3)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
    if (q4 == 0) {
      ml[2 * h] = m;
      ml[2 * h + 1] = sum;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  named_barrier(bar, kNT);
  tc_fence_after();
  // ---- O^T = V^T P^T ----
  if (tid == 32) {
    const uint32_t kb = smem_u32(Kt), pb = smem_u32(Pt);
#pragma unroll 1
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll 1
      for (int kk = 0; kk < nk16 / 16; ++kk)
        mma_f16(dO + mt * kH, desc_mn_sw128(kb + (2 * mt) * kTK * 128 + kk * 16 * 128, kTK * 128),
                desc_k_sw128(pb + (kk >> 2) * kH * 128 + (kk & 3) * 32), kIdescO, kk > 0 ? 1u : 0u);
    mma_commit(obar);
  }
  if (tid == 0 && !mbar_wait(obar, 0, kWaitLimit)) {
    atomicOr(err, 1u);
    *fail = 1;
  }
  named_barrier(bar, kNT);
  tc_fence_after();
}

}  // namespace
}  // namespace attn
}  // namespace csa
