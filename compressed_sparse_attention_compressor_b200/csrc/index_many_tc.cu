// K2 on the tensor cores for many queries per request (chunked prefill):
// lightning-indexer scores of every query against every compressed key it
// may see, s[i][j] = sum_h w[i][h] * max(0, q_idx[i][h] . k_idx[r][j]).
//
// Atlas "Model architectures", "Trained sparse attention" entry (DSA:
// lightning indexer + top-k) and "compressed KV" entry; tech-report tour,
// "The Hierarchical Sparse Indexer" (the first Full layer pays for a scan
// over the whole causally visible range) and "The indexer selects, SWA
// covers the rest".
//
// With thousands of queries per request the indexer is a dense contraction,
// [queries x heads] x [keys x d_idx], so it runs on tcgen05 with bf16
// operands and fp32 accumulators:
//   * queries form groups of up to 8 consecutive queries of one request; a
//     group's bf16 query rows (8 x 64 heads x 128 = 128 KB) stay in shared
//     memory and are the MMA's B operand, in two halves of N = 256 columns
//     (4 queries x 64 heads);
//   * the request's keys stream through a 3-stage TMA ring as 128-key tiles
//     (A operand, M = 128, K = 128, 128-byte swizzle);
//   * per tile the MMA issuer writes D_G[128 keys][256] = K_tile Q_G^T into
//     TMEM accumulator G (G = 0, 1; 2 x 256 columns), and the epilogue group
//     G (eight warps: a TMEM lane quarter and two of the half's four queries
//     each) reduces each key's row: s = sum_h w_h ReLU(D[h]) for each of its
//     queries, and stores the score of every key the query sees (causal:
//     j < n_visible[i]).
//     Accumulator G is released as soon as it is read, so the MMAs of the
//     other half run while one half is reduced;
//   * the work -- every (group, key tile) pair, groups in query order and
//     tiles in key order -- is cut into equal contiguous ranges, one per
//     persistent CTA; a CTA reloads its query rows only where its range
//     crosses into the next group.
// Every wait is bounded; a wait that gives up latches an error (reported by
// csa_sync_status) and the CTA winds down without touching TMEM in flight.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace csa {
namespace {

using namespace sm100;

constexpr int kTile = 128;                     // keys per tile (TMEM lanes, MMA M)
constexpr int kHeads = 64;
constexpr int kDI = 128;
constexpr int kQG = 8;                         // queries per group
constexpr int kQH = 4;                         // queries per MMA half
constexpr int kN = kQH * kHeads;               // 256: MMA N, TMEM columns per accumulator
constexpr int kStages = 3;
constexpr int kStageBytes = kTile * kDI * 2;   // 32 KB: two 16 KB K halves of 128 rows x 128 B
constexpr int kQBytes = kQG * kHeads * kDI * 2;  // 128 KB: two 64 KB K halves of 512 rows x 128 B
constexpr int kEpiPerGroup = 8;                // epilogue warps per accumulator: 4 lane quarters x 2 query pairs
constexpr int kThreads = 32 * (2 + 2 * kEpiPerGroup);  // producer warp, MMA warp, 16 epilogue warps
constexpr uint32_t kTmemCols = 2 * kN;
constexpr uint32_t kWaitLimit = 1u << 22;

// shared memory, from a 1024-byte aligned base
constexpr int oQ = 0;
constexpr int oStages = oQ + kQBytes;
constexpr int oBars = oStages + kStages * kStageBytes;
constexpr int oMisc = oBars + 256;
constexpr int kSmemUsed = oMisc + 64;
constexpr int kSmem = kSmemUsed + 1024;        // + alignment slack
static_assert(kSmem <= 232448, "shared memory");
static_assert(oStages % 1024 == 0 && oBars % 8 == 0, "alignment");

constexpr uint32_t kIdesc = idesc(1, 1, kTile, kN);  // bf16 x bf16 -> fp32, K-major A and B

__device__ uint32_t g_index_many_error = 0;

// Group table (device, written by many_groups_kernel):
//   t[0] = groups, t[1] = total tiles, then per group g at t + 2 + 4 g:
//   first query, queries, request, first tile (exclusive prefix over groups).
constexpr int kTabHead = 2;
constexpr int kTabStride = 4;

struct ManyArgs {
  const float* w;            // [nq][64]
  const int32_t* n_visible;  // [nq]
  const int32_t* table;
  int batch;
  int64_t cap;
  float* scores;             // [nq][ld]
  int64_t ld;
};

// One CTA of 1024 threads.  Query i starts a group when i % 8 == 0 or its
// request differs from query i - 1's; a group ends at the next start.  A
// group needs ceil(max n_visible / 128) key tiles (n_visible clamped to
// [0, cap]; a request outside [0, batch) scores nothing: 0 tiles).
__global__ void __launch_bounds__(1024) many_groups_kernel(const int32_t* __restrict__ q_req,
                                                           const int32_t* __restrict__ n_visible, int nq, int batch,
                                                           int64_t cap, int32_t* __restrict__ table) {
  __shared__ int32_t wsum[32];
  __shared__ int32_t s_base, s_tiles;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  auto req = [&](int j) { return q_req ? q_req[j] : j; };
  if (threadIdx.x == 0) {
    s_base = 0;
    s_tiles = 0;
  }
  __syncthreads();
  for (int i0 = 0; i0 < nq; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const bool start = i < nq && (i % kQG == 0 || req(i) != req(i - 1));
    int cnt = 0, r = -1, tiles = 0;
    if (start) {
      r = req(i);
      cnt = 1;
      while (cnt < kQG && i + cnt < nq && (i + cnt) % kQG != 0 && req(i + cnt) == r) ++cnt;
      if (r >= 0 && r < batch) {
        int64_t nmax = 0;
        for (int u = 0; u < cnt; ++u)
          nmax = max(nmax, min(max(static_cast<int64_t>(n_visible[i + u]), int64_t(0)), cap));
        tiles = static_cast<int>((nmax + kTile - 1) / kTile);
      }
    }
    // ranks of the group starts and prefix sums of their tiles in this chunk
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, start);
    int tincl = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, tincl, o);
      if (lane >= o) tincl += v;
    }
    if (lane == 31) wsum[warp] = tincl;
    __syncthreads();
    int gbefore = 0, tbefore = 0, gtot = 0, ttot = 0;
    // group counts per warp come from the ballots; recompute them per warp
    __shared__ int32_t wcnt[32];
    if (lane == 0) wcnt[warp] = __popc(ball);
    __syncthreads();
    for (int v = 0; v < nw; ++v) {
      if (v < warp) {
        gbefore += wcnt[v];
        tbefore += wsum[v];
      }
      gtot += wcnt[v];
      ttot += wsum[v];
    }
    if (start) {
      const int g = s_base + gbefore + __popc(ball & ((1u << lane) - 1u));
      int32_t* e = table + kTabHead + kTabStride * g;
      e[0] = i;
      e[1] = cnt;
      e[2] = r;
      e[3] = s_tiles + tbefore + tincl - tiles;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      s_base += gtot;
      s_tiles += ttot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    table[0] = s_base;
    table[1] = s_tiles;
  }
}

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t parity, volatile int* fail) {
  if (mbar_wait(bar, parity, kWaitLimit)) return true;
  atomicOr(&g_index_many_error, 1u);
  *fail = 1;
  return false;
}

// Walks a CTA's range of (group, tile) pairs: group g, its tile lt.
struct Cursor {
  const int32_t* tab;
  int groups;
  int g, lt, tiles_g;
  __device__ void load_group() {
    const int32_t* e = tab + kTabHead + kTabStride * g;
    const int next = (g + 1 < groups) ? tab[kTabHead + kTabStride * (g + 1) + 3] : tab[1];
    tiles_g = next - e[3];
  }
  // positions the cursor at global tile u (groups with no tiles are skipped)
  __device__ void seek(int u) {
    int lo = 0, hi = groups - 1;  // last group whose first tile <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab[kTabHead + kTabStride * mid + 3] <= u) lo = mid;
      else hi = mid - 1;
    }
    g = lo;
    load_group();
    lt = u - tab[kTabHead + kTabStride * g + 3];
  }
  // advances one tile; returns true when the group changed
  __device__ bool next() {
    if (++lt < tiles_g) return false;
    do {
      ++g;
      lt = 0;
      if (g >= groups) return true;
      load_group();
    } while (tiles_g == 0);
    return true;
  }
  __device__ int first_query() const { return tab[kTabHead + kTabStride * g]; }
  __device__ int queries() const { return tab[kTabHead + kTabStride * g + 1]; }
  __device__ int request() const { return tab[kTabHead + kTabStride * g + 2]; }
};

__global__ void __launch_bounds__(kThreads, 1)
    index_many_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                         ManyArgs a) {
  const int groups = a.table[0], total = a.table[1];
  const int u0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * total / gridDim.x);
  const int u1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * total / gridDim.x);
  if (u0 >= u1) return;  // uniform over the CTA: nothing to do
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + oBars);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // [2] accumulator G holds a tile's products
  uint64_t* tempty = tfull + 2;       // [2] ... and has been read back
  uint64_t* qfull = tempty + 2;       // a group's query rows have landed
  uint64_t* qempty = qfull + 1;       // every MMA reading the previous group's rows is done
  uint64_t* mdone = qempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + oMisc);
  volatile int* fail = reinterpret_cast<volatile int*>(smem + oMisc + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tiles = u1 - u0;
  if (tid == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&qmap);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int G = 0; G < 2; ++G) {
      mbar_init(&tfull[G], 1);
      mbar_init(&tempty[G], kEpiPerGroup * 32);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    mbar_init(mdone, 1);
    *fail = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  Cursor cur;
  cur.tab = a.table;
  cur.groups = groups;
  cur.seek(u0);

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer: a group's query rows at each group change, then the tiles
      int issued = 0, seg = 0;
      bool qpending = false;
      for (int i = 0; i < n_tiles && !*fail; ++i) {
        if (i == 0 || (i > 0 && cur.next())) {
          // the previous group's MMAs must be done before its rows are overwritten
          if (seg > 0 && !wait_or_fail(qempty, (seg - 1) & 1, fail)) break;
          const int y = cur.first_query() * kHeads;
          mbar_arrive_expect_tx(qfull, kQBytes);
          for (int h = 0; h < 2; ++h)
            for (int rb = 0; rb < 2; ++rb)
              tma_load_2d(smem + oQ + h * (kQBytes / 2) + rb * (kQBytes / 4), &qmap, qfull, h * 64, y + rb * 256);
          qpending = true;
          ++seg;
        }
        const int s = i % kStages;
        if (!wait_or_fail(&empty[s], ((i / kStages) & 1) ^ 1, fail)) break;
        const int64_t row = static_cast<int64_t>(cur.request()) * a.cap + static_cast<int64_t>(cur.lt) * kTile;
        uint8_t* dst = smem + oStages + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(dst, &kmap, &full[s], 0, static_cast<int>(row));
        tma_load_2d(dst + kStageBytes / 2, &kmap, &full[s], 64, static_cast<int>(row));
        issued = i + 1;
      }
      // the copies still in flight land before the CTA winds down
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1, kWaitLimit);
      if (qpending) mbar_wait(qfull, (seg - 1) & 1, kWaitLimit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int seg = 0;
      for (int i = 0; i < n_tiles && !*fail; ++i) {
        const bool newg = (i == 0) || cur.next();
        if (newg) {
          if (!wait_or_fail(qfull, seg & 1, fail)) break;
          ++seg;
        }
        const int s = i % kStages;
        if (!wait_or_fail(&full[s], (i / kStages) & 1, fail)) break;
        bool ok = true;
        for (int G = 0; G < 2 && ok; ++G) {
          if (!wait_or_fail(&tempty[G], (i & 1) ^ 1, fail)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t abase = smem_u32(smem + oStages + s * kStageBytes);
          const uint32_t bbase = smem_u32(smem + oQ + G * (kQBytes / 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t half = kk >> 2, off = (kk & 3) * 32;
            mma_f16(tmem + G * kN, desc_k_sw128(abase + half * (kStageBytes / 2) + off),
                    desc_k_sw128(bbase + half * (kQBytes / 2) + off), kIdesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&tfull[G]);
        }
        if (!ok) break;
        mma_commit(&empty[s]);
        // the last tile of a group (or of the range): its rows may be replaced
        // once these MMAs are done
        const bool last_of_group = (cur.lt + 1 == cur.tiles_g) || (i + 1 == n_tiles);
        if (last_of_group) mma_commit(qempty);
      }
      // every MMA has completed before TMEM is read for the last time or released
      mma_commit(mdone);
      mbar_wait(mdone, 0, kWaitLimit);
    }
  } else {
    // epilogue: group G = warps 2-9 / 10-17; warp w of a group reads TMEM
    // lanes 32 (w % 4) .. + 31 for the queries 2 (w / 4), + 1 of the half
    const int G = (warp - 2) / kEpiPerGroup, sub = warp & 3, qp = ((warp - 2) % kEpiPerGroup) >> 2;
    const int row = sub * 32 + lane;
    const uint32_t lane_addr = tmem + G * kN + (static_cast<uint32_t>(sub * 32) << 16);
    for (int i = 0; i < n_tiles && !*fail; ++i) {
      if (i > 0) cur.next();
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&tfull[G], i & 1, kWaitLimit);
      __syncwarp();
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
        atomicOr(&g_index_many_error, 1u);
        *fail = 1;
        break;
      }
      tc_fence_after();
      const int q0 = cur.first_query() + G * kQH;
      const int nqh = min(kQH, cur.queries() - G * kQH);  // queries of this half (may be <= 0)
      const int64_t key = static_cast<int64_t>(cur.lt) * kTile + row;
      float sc[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int qq = 2 * qp + u;
        sc[u] = 0.f;
        if (qq < nqh) {  // warp-uniform
          uint32_t v0[32], v1[32];
          tmem_ld32(lane_addr + qq * kHeads, v0);
          tmem_ld32(lane_addr + qq * kHeads + 32, v1);
          tmem_wait_ld();
          const float4* w4 = reinterpret_cast<const float4*>(a.w + static_cast<int64_t>(q0 + qq) * kHeads);
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int h4 = 0; h4 < 8; ++h4) {
            const float4 wa = __ldg(w4 + h4), wb = __ldg(w4 + 8 + h4);
            s0 = fmaf(wa.x, fmaxf(__uint_as_float(v0[4 * h4]), 0.f), s0);
            s1 = fmaf(wa.y, fmaxf(__uint_as_float(v0[4 * h4 + 1]), 0.f), s1);
            s0 = fmaf(wa.z, fmaxf(__uint_as_float(v0[4 * h4 + 2]), 0.f), s0);
            s1 = fmaf(wa.w, fmaxf(__uint_as_float(v0[4 * h4 + 3]), 0.f), s1);
            s2 = fmaf(wb.x, fmaxf(__uint_as_float(v1[4 * h4]), 0.f), s2);
            s3 = fmaf(wb.y, fmaxf(__uint_as_float(v1[4 * h4 + 1]), 0.f), s3);
            s2 = fmaf(wb.z, fmaxf(__uint_as_float(v1[4 * h4 + 2]), 0.f), s2);
            s3 = fmaf(wb.w, fmaxf(__uint_as_float(v1[4 * h4 + 3]), 0.f), s3);
          }
          sc[u] = (s0 + s1) + (s2 + s3);
        }
      }
      // every column of the accumulator this warp reads is in registers
      tc_fence_before();
      mbar_arrive(&tempty[G]);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int qq = 2 * qp + u;
        if (qq >= nqh) break;
        const int qi = q0 + qq;
        const int64_t nv = min(max(static_cast<int64_t>(__ldg(a.n_visible + qi)), int64_t(0)), a.cap);
        if (key < nv) a.scores[static_cast<int64_t>(qi) * a.ld + key] = sc[u];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 many_encoder() {
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

// [rows][128] bf16, 128-byte swizzle, boxes of 64 columns x box_rows rows.
bool map_rows_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {kDI, rows};
  const cuuint64_t strides[1] = {kDI * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return many_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int g_sms = 0;

}  // namespace

bool index_many_tc_supported(const csa_params_t* p, int q_dtype, int k_dtype) {
  return p->h_idx == kHeads && p->d_idx == kDI && q_dtype == kBF16 && k_dtype == kBF16;
}

size_t index_many_tc_table_bytes(int nq) {
  return (static_cast<size_t>(nq) * kTabStride + kTabHead) * sizeof(int32_t);
}

// scores [nq][ld] fp32 (columns j < n_visible[i] written); table: device
// scratch of index_many_tc_table_bytes(nq) bytes.
csa_status_t launch_index_many_tc(const csa_params_t* p, int nq, const csa_tensor_t* q_idx, const float* w,
                                  const csa_tensor_t* k_idx, int batch, int64_t cap, const int32_t* q_req,
                                  const int32_t* n_visible, float* scores, int64_t ld, int32_t* table,
                                  cudaStream_t stream) {
  (void)p;
  if (nq == 0 || cap == 0) return CSA_OK;
  if (!many_encoder()) return set_error(CSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if (static_cast<int64_t>(batch) * cap >= (int64_t(1) << 31) || static_cast<int64_t>(nq) * kHeads >= (int64_t(1) << 31))
    return set_error(CSA_ERR_UNSUPPORTED, "indexer rows beyond 2^31");
  if ((cap + kTile - 1) / kTile * static_cast<int64_t>(nq) >= (int64_t(1) << 31))
    return set_error(CSA_ERR_UNSUPPORTED, "too many indexer tiles");
  CUtensorMap kmap, qmap;
  if (!map_rows_bf16(&kmap, k_idx->data, static_cast<uint64_t>(batch) * cap, kTile) ||
      !map_rows_bf16(&qmap, q_idx->data, static_cast<uint64_t>(nq) * kHeads, 256))
    return set_error(CSA_ERR_CUDA, "tensor map encoding failed");
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(index_many_tc_kernel),
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    attr = true;
  }
  prof_begin(stream);
  many_groups_kernel<<<1, 1024, 0, stream>>>(q_req, n_visible, nq, batch, cap, table);
  csa_status_t st = check_launch("many_groups_kernel", stream);
  if (st != CSA_OK) return st;
  ManyArgs a;
  a.w = w;
  a.n_visible = n_visible;
  a.table = table;
  a.batch = batch;
  a.cap = cap;
  a.scores = scores;
  a.ld = ld;
  prof_begin(stream);
  index_many_tc_kernel<<<g_sms > 0 ? g_sms : 148, kThreads, kSmem, stream>>>(kmap, qmap, a);
  return check_launch("index_many_tc_kernel", stream);
}

uint32_t index_many_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_index_many_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_index_many_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
