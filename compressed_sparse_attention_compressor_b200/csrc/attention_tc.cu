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

#include "attn_tile.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

using namespace sm100;

using namespace attn;

constexpr int kThreads = kNT;  // 8 warps; warps 4..7 read TMEM
constexpr int kTmemCols = 512;

// shared-memory layout: the attention tile (attn_tile.cuh), then this kernel's
constexpr int oBars = kTileSmem;
constexpr int oMisc = oBars + 64;
constexpr int oLut = oMisc + 64;  // MXFP4 code-byte table, 256 x bf16x2
constexpr int kSmem = oLut + 1024 + 1024;

__device__ uint32_t g_attn_tc_error = 0;

struct AttnTcArgs {
  const void* kv; const void* kv_scale; int kv_fmt; int batch; int64_t cap;
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

// FMT: storage of the compressed rows (kKvBF16 / kKvFP8 / kKvMX4); each
// format gets its own instantiation, so a launch carries only its own gather.
template <bool CLUSTER, int FMT>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  float* ml = reinterpret_cast<float*>(smem + oML);
  int32_t* ent = reinterpret_cast<int32_t*>(smem + oEnt);
  uint64_t* qbar = reinterpret_cast<uint64_t*>(smem + oBars);
  uint64_t* sbar = qbar + 1;
  uint64_t* obar = qbar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + oMisc);
  int* s_flags = reinterpret_cast<int*>(smem + oMisc + 16);  // [0] any window row, [1] failed

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qi = blockIdx.y, split = blockIdx.x;
  // barriers, the query's TMA, TMEM: nothing an earlier kernel of the
  // decode step writes (the query is the caller's input)
  auto prologue = [&]() {
    if (tid == 0) {
      prefetch_tensormap(&qmap);
      mbar_init(qbar, 1);
      mbar_init(sbar, 1);
      mbar_init(obar, 1);
      s_flags[0] = 0;
      s_flags[1] = 0;
      fence_barrier_init();
      // the query first: its load overlaps the gather of the keys
      mbar_arrive_expect_tx(qbar, kH * kD * 2);
      for (int blk = 0; blk < 8; ++blk) tma_load_2d(smem + oQ + blk * kH * 128, &qmap, qbar, blk * 64, qi * kH);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    if constexpr (FMT == kKvMX4) fill_mx4_lut(reinterpret_cast<uint32_t*>(smem + oLut));
  };
  // cluster path: the prologue runs before the wait for the previous
  // kernel (a programmatic launch overlaps it with that kernel's tail);
  // everything below reads the selection, positions and window it wrote
  if constexpr (CLUSTER) prologue();
  grid_dependency_wait();
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

  if constexpr (!CLUSTER) prologue();
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
  __syncthreads();

  if (tid < kTK && ent[tid] <= -2) s_flags[0] = 1;
  const int nsr = s1 - s0, nwr = w1 - w0;
  const uint32_t tmem = *tmem_slot;
  const uint32_t dS = tmem, dO = tmem + kH;
  Src src;
  src.kv = a.kv;
  src.kv_scale = a.kv_scale;
  src.lut = reinterpret_cast<const uint32_t*>(smem + oLut);
  src.swa_k = a.swa_k;
  src.swa_v = a.swa_v;
  src.kv_row0 = kv_row0;
  src.sw_row0 = sw_row0;
  src.tau = a.tau;
  tc_fence_before();
  __syncthreads();  // s_flags[0]
  tc_fence_after();
  attend_tile<FMT>(smem, src, CLUSTER, nsr, nwr, s_flags[0] != 0, qbar, sbar, obar, dS, dO, 1, &s_flags[1],
              &g_attn_tc_error);
  if (!CLUSTER && tid < kH) {
    pp[tid * (kD + 2)] = ml[2 * tid];
    pp[tid * (kD + 2) + 1] = ml[2 * tid + 1];
  }
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
    // this CTA's O (unnormalised) into its own shared memory as [head][dim],
    // over the key tile (both MMAs have completed): fp32, or bf16 pairs when
    // the output is bf16 (half the bytes the merge moves between the CTAs;
    // the merge accumulates in fp32, so a partial's rounding adds at most the
    // output's own rounding error)
    const bool pbf = a.out_dtype != kF32;
    float* Osm = reinterpret_cast<float*>(smem + oK);
    uint32_t* Obf = reinterpret_cast<uint32_t*>(smem + oK);  // [64][256] bf16x2
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
        if (pbf) {
          // lanes 2i and 2i + 1 hold dims 2i and 2i + 1: even lanes store the pair
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const float a0 = __uint_as_float(v0[h]), b0 = __shfl_down_sync(0xFFFFFFFFu, a0, 1);
            const float a1 = __uint_as_float(v1[h]), b1 = __shfl_down_sync(0xFFFFFFFFu, a1, 1);
            if ((lane & 1) == 0) {
              Obf[h * (kD / 2) + dim / 2] = pack_bf16(a0, b0);
              Obf[(32 + h) * (kD / 2) + dim / 2] = pack_bf16(a1, b1);
            }
          }
        } else {
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            Osm[h * kD + dim] = __uint_as_float(v0[h]);
            Osm[(32 + h) * kD + dim] = __uint_as_float(v1[h]);
          }
        }
      }
    }
    cluster.sync();
    // heads split + r * R for r = 0, 1, ...: this CTA finishes nh of them
    float* wgt = reinterpret_cast<float*>(smem + oS);  // [head][16 CTAs], then [head][2] (M, 1/L); logits are dead
    const int nh = (kH - split + R - 1) / R;
    const int dim = tid * 2;  // two consecutive dims per thread
    // bf16 partials: thread t takes eight consecutive dims of one of the
    // CTA's heads per round (task t + 256 i: head w = task / 64, dims
    // 8 (task % 64) ..), one 16-byte load from every peer; the first round's
    // loads go out before the weights are computed (their round trips overlap)
    uint4 vb[16];
    auto load_bf = [&](int task) {
      const int w = task >> 6, d8 = (task & 63) * 8;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < R && w < nh)
          vb[j] = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(Obf, j) + (split + w * R) * (kD / 2) + d8 / 2);
    };
    if (pbf) load_bf(tid);
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
    if (pbf) {
      for (int task = tid; task < nh * 64; task += kThreads) {
        if (task != tid) load_bf(task);
        const int w = task >> 6, d8 = (task & 63) * 8, h = split + w * R;
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < R) {
            const float wj = wgt[w * 16 + j];
            const uint32_t u4[4] = {vb[j].x, vb[j].y, vb[j].z, vb[j].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              o[2 * i] = fmaf(wj, __uint_as_float(u4[i] << 16), o[2 * i]);
              o[2 * i + 1] = fmaf(wj, __uint_as_float(u4[i] & 0xFFFF0000u), o[2 * i + 1]);
            }
          }
        const float inv = wgt[kH * 16 + w * 2 + 1];
        const int64_t off = (static_cast<int64_t>(qi) * kH + h) * kD + d8;
        const uint4 ov = make_uint4(pack_bf16(o[0] * inv, o[1] * inv), pack_bf16(o[2] * inv, o[3] * inv),
                                    pack_bf16(o[4] * inv, o[5] * inv), pack_bf16(o[6] * inv, o[7] * inv));
        uint16_t* dst = static_cast<uint16_t*>(a.out) + off;
        if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
          *reinterpret_cast<uint4*>(dst) = ov;
        } else {  // an output that is only 4-byte aligned
          uint32_t* d4 = reinterpret_cast<uint32_t*>(dst);
          d4[0] = ov.x; d4[1] = ov.y; d4[2] = ov.z; d4[3] = ov.w;
        }
      }
    } else {
      // fp32 partials: two heads per round, every peer's loads of both in
      // flight before the sums
      for (int w0 = 0; w0 < nh; w0 += 2) {
        float2 v[2][16];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < R && w0 + u < nh)
              v[u][j] = *reinterpret_cast<const float2*>(cluster.map_shared_rank(Osm, j) + (split + (w0 + u) * R) * kD +
                                                         dim);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int w = w0 + u;
          if (w >= nh) break;
          const int h = split + w * R;
          float o0 = 0.f, o1 = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < R) {
              const float wj = wgt[w * 16 + j];
              o0 = fmaf(wj, v[u][j].x, o0);
              o1 = fmaf(wj, v[u][j].y, o1);
            }
          const float inv = wgt[kH * 16 + w * 2 + 1];
          const int64_t off = (static_cast<int64_t>(qi) * kH + h) * kD + dim;
          *reinterpret_cast<float2*>(static_cast<float*>(a.out) + off) = make_float2(o0 * inv, o1 * inv);
        }
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
  bool attr[3][2] = {};        // per format, split / cluster kernel
  int cluster_ok[3][17] = {};  // per format and cluster size: 0 unknown, else co-resident clusters (-1: none)
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
  if (kv_dtype != kBF16 && kv_dtype != kFP8 && kv_dtype != kMXFP4) return false;
  if (has_window && swa_dtype != kBF16) return false;
  return true;
}

size_t attn_tc_workspace_bytes(int nq, int max_keys) {
  return static_cast<size_t>(nq) * attn_tc_splits(max_keys) * kH * (kD + 2) * sizeof(float);
}

csa_status_t launch_attn_merge(const float* part, int nq, int n_splits, int hq, int d, const float* sink, void* out,
                               int out_dtype, float* lse, cudaStream_t stream);

template <int FMT>
csa_status_t launch_attn_fmt(TcLauncher& L, const csa_params_t* p, int nq, int max_keys, const CUtensorMap& qmap,
                             const AttnTcArgs& a, const float* sink, const csa_tensor_t* out, float* lse,
                             cudaStream_t stream, bool pdl) {
  for (int c = 0; c < 2; ++c)
    if (!L.attr[FMT][c]) {
      void* fn = c ? reinterpret_cast<void*>(attn_tc_kernel<true, FMT>) : reinterpret_cast<void*>(attn_tc_kernel<false, FMT>);
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
      if (e == cudaSuccess && c) e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return set_error(CSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      L.attr[FMT][c] = true;
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
    if (L.cluster_ok[FMT][r] == 0) {
      int ncl = 0;
      const cudaError_t e = cudaOccupancyMaxActiveClusters(&ncl, attn_tc_kernel<true, FMT>, &cfg);
      L.cluster_ok[FMT][r] = (e == cudaSuccess && ncl >= 1) ? ncl : -1;
      cudaGetLastError();
    }
    if (L.cluster_ok[FMT][r] >= nq || (r == rmin && L.cluster_ok[FMT][r] > 0)) R = r;
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
    cudaLaunchAttribute attr2[2] = {attr[0], {}};
    if (pdl) {
      // a programmatic launch: the prologue overlaps the previous kernel's tail
      attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr2[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr2;
      cfg.numAttrs = 2;
    }
    {
      prof_begin(stream);
      const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<true, FMT>, qmap, a);
      if (e != cudaSuccess) {
        check_launch("attn_tc_cluster_kernel", stream);
        return set_error(CSA_ERR_CUDA, "attn_tc_kernel (cluster) launch: %s", cudaGetErrorString(e));
      }
      return check_launch("attn_tc_cluster_kernel", stream);
    }
  }
  if (nq > 64) return set_error(CSA_ERR_UNSUPPORTED, "attention: no cluster size fits %d queries", nq);
  prof_begin(stream);
  attn_tc_kernel<false, FMT><<<dim3(a.splits, nq), kThreads, kSmem, stream>>>(qmap, a);
  csa_status_t st = check_launch("attn_tc_kernel", stream);
  if (st != CSA_OK) return st;
  return launch_attn_merge(a.part, nq, a.splits, kH, kD, sink, out->data, out->dtype, lse, stream);
}


csa_status_t launch_attention_tc(const csa_params_t* p, int nq, const csa_tensor_t* q, const csa_tensor_t* kv,
                                 int batch, int64_t cap, const int32_t* idx, const int32_t* n_visible,
                                 const int32_t* q_req, const csa_tensor_t* swa_k, const csa_tensor_t* swa_v,
                                 const int64_t* q_pos, const int64_t* swa_lo, const float* sink,
                                 const csa_tensor_t* out, float* lse, void* workspace, int max_keys,
                                 cudaStream_t stream, bool pdl) {
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
  a.kv_fmt = kv->dtype == kFP8 ? kKvFP8 : kv->dtype == kMXFP4 ? kKvMX4 : kKvBF16;
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
  if (a.kv_fmt == kKvMX4) return launch_attn_fmt<kKvMX4>(L, p, nq, max_keys, qmap, a, sink, out, lse, stream, pdl);
  if (a.kv_fmt == kKvFP8) return launch_attn_fmt<kKvFP8>(L, p, nq, max_keys, qmap, a, sink, out, lse, stream, pdl);
  return launch_attn_fmt<kKvBF16>(L, p, nq, max_keys, qmap, a, sink, out, lse, stream, pdl);
}

uint32_t attn_tc_take_error() {
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_attn_tc_error, sizeof(v)) != cudaSuccess) return 0;
  if (v) cudaMemcpyToSymbol(g_attn_tc_error, &z, sizeof(z));
  return v;
}

}  // namespace csa
