// K1 -- the KV compressor, and the decode-step append kernel built on it.
//
// "DeepSeek-V4.1-Flash, illustrated", Equation (1) figure: the projected KV
// entries C_l and compression weights Z_l give the pooled global-KV entries;
// ratio 1 is the unpooled main-KV projection.  Atlas "Model architectures",
// "compressed KV" entry: every m KV tokens become one entry through learned
// compression weights.  Tech-report tour, "A simpler compressor": groups do
// not overlap, no absolute positional term, and the indexer key is projected
// from the main-KV entry.
//
// Per request b, block j, channel c (rows i = j*m .. j*m+m-1):
//   out[j][c] = sum_i softmax_i(Z[i][c]) * C[i][c]
// The kernel is HBM-bound: every thread owns 8 consecutive channels (one
// 16-byte bf16 vector), computes the block maximum, then the exp-weighted
// sums, in fp32.  FP8 output: the 8 lanes that own one 64-channel group
// exchange their maxima by warp shuffle, and the group's scale is
// max|x| / 448.  The optional indexer-key projection (entry . W_IK) runs
// from the fp32 pooled entries held in shared memory, one warp per entry.
#include <cooperative_groups.h>

#include "common.cuh"
#include "pool.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kCompressThreads = 256;
constexpr int kCompressNB = 8;  // blocks pooled per CTA

// One warp projects one pooled fp32 row (shared memory) through W_IK
// [d][d_idx] and stores the key row.  d_idx <= 256, a multiple of 32.
__device__ __forceinline__ void project_row(const float* pooled, int d, const void* w_ik, int w_dtype,
                                            int d_idx, const OutSpec& ko, int64_t row) {
  const int lane = threadIdx.x & 31;
  float acc[8];
  const int per = d_idx / 32;
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  for (int c = 0; c < d; ++c) {
    const float x = pooled[c];
    const char* wrow = static_cast<const char*>(w_ik) + static_cast<int64_t>(c) * d_idx * elem_bytes(w_dtype);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < per) acc[k] = fmaf(x, load1(wrow, w_dtype, lane + 32 * k, nullptr, 1), acc[k]);
  }
  if (ko.dtype == kFP8) {
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < per) amax = fmaxf(amax, fabsf(acc[k]));
    amax = warp_max(amax);
    const float s = amax > 0.f ? amax / 448.f : 1.f;
    uint8_t* dst = static_cast<uint8_t*>(ko.data) + row * ko.row_stride;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < per) dst[lane + 32 * k] = f32_to_e4m3(acc[k] / s);
    if (lane == 0) static_cast<float*>(ko.scale)[row * ko.scale_stride] = s;
  } else if (ko.dtype == kBF16) {
    uint16_t* dst = static_cast<uint16_t*>(ko.data) + row * ko.row_stride;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < per) dst[lane + 32 * k] = f32_to_bf16_bits(acc[k]);
  } else {
    float* dst = static_cast<float*>(ko.data) + row * ko.row_stride;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < per) dst[lane + 32 * k] = acc[k];
  }
}

// Largest W_IK staged in shared memory by the projection (bytes).
constexpr int kMaxWSmem = 160 * 1024;

// All threads: copy W_IK [d][d_idx] into shared memory (16-byte vectors).
__device__ __forceinline__ void stage_w(uint8_t* wsm, const void* w_ik, int bytes) {
  const uint4* src = static_cast<const uint4*>(w_ik);
  uint4* dst = reinterpret_cast<uint4*>(wsm);
  for (int i = threadIdx.x; i < bytes / 16; i += kCompressThreads) dst[i] = __ldg(src + i);
}

// All threads: kout[0..d_idx) = pooled[0..d) . W (W staged in shared memory).
// Thread t owns output pair t % (d_idx/2) over a slice of the d rows; the
// slices are summed through red[] (256 * 2 floats).  d_idx in {32, 64,
// 128, 256}.
__device__ void project_smem(const float* pooled, int d, const uint8_t* wsm, int w_dtype, int d_idx, float* red,
                             float* kout) {
  const int P = d_idx / 2, S = kCompressThreads / P;
  const int t = threadIdx.x, o2 = t % P, sl = t / P;
  const int r0 = sl * d / S, r1 = (sl + 1) * d / S;
  float a0 = 0.f, a1 = 0.f;
  if (w_dtype == kBF16) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(wsm);
#pragma unroll 8
    for (int c = r0; c < r1; ++c) {
      const uint32_t u = w[c * P + o2];
      const float x = pooled[c];
      a0 = fmaf(x, __uint_as_float(u << 16), a0);
      a1 = fmaf(x, __uint_as_float(u & 0xFFFF0000u), a1);
    }
  } else {
    const float2* w = reinterpret_cast<const float2*>(wsm);
#pragma unroll 8
    for (int c = r0; c < r1; ++c) {
      const float2 u = w[c * P + o2];
      const float x = pooled[c];
      a0 = fmaf(x, u.x, a0);
      a1 = fmaf(x, u.y, a1);
    }
  }
  red[sl * d_idx + 2 * o2] = a0;
  red[sl * d_idx + 2 * o2 + 1] = a1;
  __syncthreads();
  if (t < d_idx) {
    float v = 0.f;
    for (int q = 0; q < S; ++q) v += red[q * d_idx + t];
    kout[t] = v;
  }
  __syncthreads();
}

// One warp stores a projected key row (fp32 values in shared memory).
__device__ __forceinline__ void store_key_row(const float* kv, int d_idx, const OutSpec& ko, int64_t row) {
  const int lane = threadIdx.x & 31;
  if (ko.dtype == kFP8) {
    float amax = 0.f;
    for (int i = lane; i < d_idx; i += 32) amax = fmaxf(amax, fabsf(kv[i]));
    amax = warp_max(amax);
    const float s = amax > 0.f ? amax / 448.f : 1.f;
    uint8_t* dst = static_cast<uint8_t*>(ko.data) + row * ko.row_stride;
    for (int i = lane; i < d_idx; i += 32) dst[i] = f32_to_e4m3(kv[i] / s);
    if (lane == 0) static_cast<float*>(ko.scale)[row * ko.scale_stride] = s;
  } else if (ko.dtype == kBF16) {
    uint16_t* dst = static_cast<uint16_t*>(ko.data) + row * ko.row_stride;
    for (int i = lane; i < d_idx; i += 32) dst[i] = f32_to_bf16_bits(kv[i]);
  } else {
    float* dst = static_cast<float*>(ko.data) + row * ko.row_stride;
    for (int i = lane; i < d_idx; i += 32) dst[i] = kv[i];
  }
}

__global__ void __launch_bounds__(kCompressThreads)
compress_kernel(const void* __restrict__ C, const void* __restrict__ Z, int in_dtype, int64_t n_tokens, int d,
                int m, int64_t n_blocks, OutSpec out, int64_t out_rows, const void* __restrict__ w_ik,
                int w_dtype, int d_idx, OutSpec kout) {
  extern __shared__ float pooled[];  // [kCompressNB][d]
  const int b = blockIdx.y;
  const int64_t blk0 = static_cast<int64_t>(blockIdx.x) * kCompressNB;
  const int vecs = d / 8;
  const int tasks = kCompressNB * vecs;
  const int iters = (tasks + kCompressThreads - 1) / kCompressThreads;
  const int eb = elem_bytes(in_dtype);
  const char* Cb = static_cast<const char*>(C) + static_cast<int64_t>(b) * n_tokens * d * eb;
  const char* Zb = static_cast<const char*>(Z) + static_cast<int64_t>(b) * n_tokens * d * eb;
  for (int it = 0; it < iters; ++it) {
    const int task = it * kCompressThreads + threadIdx.x;
    const int lb = task / vecs, col = (task % vecs) * 8;
    const int64_t j = blk0 + lb;
    const bool valid = task < tasks && j < n_blocks;
    float v[8];
    if (valid) {
      const int64_t r0 = j * m;
      auto rowC = [&](int i) { return Cb + (r0 + i) * d * eb; };
      auto rowZ = [&](int i) { return Zb + (r0 + i) * d * eb; };
      pool8(rowC, rowZ, in_dtype, m, col, v);
      if (w_ik != nullptr) {
#pragma unroll
        for (int e = 0; e < 8; ++e) pooled[lb * d + col + e] = v[e];
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
    }
    store_pooled8(out, static_cast<int64_t>(b) * out_rows + j, col, v, valid);
  }
  if (w_ik == nullptr) return;
  const int wbytes = d * d_idx * elem_bytes(w_dtype);
  if (wbytes <= kMaxWSmem) {
    uint8_t* wsm = reinterpret_cast<uint8_t*>(pooled + kCompressNB * d);
    float* red = reinterpret_cast<float*>(wsm + wbytes);
    float* kvec = red + 2 * kCompressThreads;
    stage_w(wsm, w_ik, wbytes);
    __syncthreads();
    for (int lb = 0; lb < kCompressNB; ++lb) {
      const int64_t j = blk0 + lb;
      if (j >= n_blocks) break;  // uniform over the CTA
      project_smem(pooled + lb * d, d, wsm, w_dtype, d_idx, red, kvec);
      if (threadIdx.x < 32) store_key_row(kvec, d_idx, kout, static_cast<int64_t>(b) * out_rows + j);
      __syncthreads();
    }
    return;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  for (int lb = warp; lb < kCompressNB; lb += kCompressThreads / 32) {
    const int64_t j = blk0 + lb;
    if (j >= n_blocks) break;
    project_row(pooled + lb * d, d, w_ik, w_dtype, d_idx, kout, static_cast<int64_t>(b) * out_rows + j);
  }
}

// Decode-step append: one CTA per request.  Writes the token's SWA key/value
// into ring slot t % swa_cap and its C/Z row into open-block slot t % m; if
// the token closes its block, pools the block into kv row (t+1)/m - 1 and
// projects the indexer key.  Also writes the per-query n_visible and q_pos
// arrays the later kernels read.
__global__ void __launch_bounds__(kCompressThreads)
decode_append_kernel(const int64_t* __restrict__ pos, int m, int d, int act_dtype, const void* __restrict__ c_t,
                     const void* __restrict__ z_t, const void* __restrict__ k_t, const void* __restrict__ v_t,
                     void* open_c, void* open_z, void* swa_k, void* swa_v, int swa_dtype, int swa_cap,
                     OutSpec kv, int64_t cap, const void* __restrict__ w_ik, int w_dtype, int d_idx,
                     OutSpec kidx, int32_t* __restrict__ n_visible_out, int64_t* __restrict__ q_pos_out,
                     int32_t* __restrict__ q_req_out, uint4* __restrict__ zero, int64_t zero_n16) {
  extern __shared__ __align__(16) float pooled[];  // [d], then W_IK, reduction scratch
  __shared__ uint64_t wbar;
  const int b = blockIdx.x;
  const int64_t t = pos[b];
  const bool closes = (t + 1) % m == 0;
  const int wbytes = w_ik ? d * d_idx * elem_bytes(w_dtype) : 0;
  const bool w_smem = w_ik != nullptr && closes && wbytes <= kMaxWSmem;
  uint8_t* wsm = reinterpret_cast<uint8_t*>(pooled + d);
  if (w_smem && threadIdx.x == 0) {
    // W_IK by TMA bulk copies, in flight while the block is pooled
    sm100::mbar_init(&wbar, 1);
    sm100::fence_barrier_init();
    sm100::mbar_arrive_expect_tx(&wbar, wbytes);
    for (int off = 0; off < wbytes; off += 32768)
      sm100::bulk_load(wsm + off, static_cast<const uint8_t*>(w_ik) + off, min(32768, wbytes - off), &wbar);
  }
  __syncthreads();  // the barrier's initialisation is visible to every waiter
  // zero this CTA's share of the caller's control words (later kernels'
  // counters and histograms)
  if (zero != nullptr) {
    const int64_t z0 = zero_n16 * b / gridDim.x, z1 = zero_n16 * (b + 1) / gridDim.x;
    for (int64_t i = z0 + threadIdx.x; i < z1; i += kCompressThreads) zero[i] = make_uint4(0, 0, 0, 0);
  }
  const int slot_m = static_cast<int>(t % m);
  const int64_t slot_w = t % swa_cap;
  const int ea = elem_bytes(act_dtype), es = elem_bytes(swa_dtype);
  const int vecs = d / 8;
  const char* crow = static_cast<const char*>(c_t) + static_cast<int64_t>(b) * d * ea;
  const char* zrow = static_cast<const char*>(z_t) + static_cast<int64_t>(b) * d * ea;
  char* ocb = static_cast<char*>(open_c) + static_cast<int64_t>(b) * m * d * ea;
  char* ozb = static_cast<char*>(open_z) + static_cast<int64_t>(b) * m * d * ea;
  for (int vec = threadIdx.x; vec < vecs; vec += kCompressThreads) {
    const int col = vec * 8;
    float v[8];
    load8(static_cast<const char*>(k_t) + static_cast<int64_t>(b) * d * ea, act_dtype, col, nullptr, 1, v);
    store8(static_cast<char*>(swa_k) + (static_cast<int64_t>(b) * swa_cap + slot_w) * d * es, swa_dtype, col, v);
    load8(static_cast<const char*>(v_t) + static_cast<int64_t>(b) * d * ea, act_dtype, col, nullptr, 1, v);
    store8(static_cast<char*>(swa_v) + (static_cast<int64_t>(b) * swa_cap + slot_w) * d * es, swa_dtype, col, v);
    load8(crow, act_dtype, col, nullptr, 1, v);
    store8(ocb + static_cast<int64_t>(slot_m) * d * ea, act_dtype, col, v);
    load8(zrow, act_dtype, col, nullptr, 1, v);
    store8(ozb + static_cast<int64_t>(slot_m) * d * ea, act_dtype, col, v);
  }
  if (threadIdx.x == 0) {
    n_visible_out[b] = static_cast<int32_t>((t + 1) / m);
    q_pos_out[b] = t;
    q_req_out[b] = b;
  }
  if (!closes) return;  // uniform across the CTA
  const int64_t row = static_cast<int64_t>(b) * cap + (t + 1) / m - 1;
  // The current token's row is read from c_t / z_t, the others from the
  // open-block buffer (written by earlier steps).
  auto rowC = [&](int i) -> const char* { return i == slot_m ? crow : ocb + static_cast<int64_t>(i) * d * ea; };
  auto rowZ = [&](int i) -> const char* { return i == slot_m ? zrow : ozb + static_cast<int64_t>(i) * d * ea; };
  const int iters = (vecs + kCompressThreads - 1) / kCompressThreads;
  for (int it = 0; it < iters; ++it) {
    const int vec = it * kCompressThreads + threadIdx.x;
    const bool valid = vec < vecs;
    float v[8];
    if (valid) {
      pool8(rowC, rowZ, act_dtype, m, vec * 8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) pooled[vec * 8 + e] = v[e];
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
    }
    store_pooled8(kv, row, valid ? vec * 8 : 0, v, valid);
  }
  if (w_ik == nullptr) return;
  if (w_smem) {
    float* red = reinterpret_cast<float*>(wsm + wbytes);
    float* kvec = red + 2 * kCompressThreads;
    // bounded wait; on a timeout the key row is left unwritten
    if (!__syncthreads_and(sm100::mbar_wait(&wbar, 0, 1u << 22) ? 1 : 0)) return;
    project_smem(pooled, d, wsm, w_dtype, d_idx, red, kvec);
    if (threadIdx.x < 32) store_key_row(kvec, d_idx, kidx, row);
    return;
  }
  __syncthreads();
  if (threadIdx.x < 32) project_row(pooled, d, w_ik, w_dtype, d_idx, kidx, row);
}

// Decode-step append, cluster version: the CTAs of one cluster share one
// request, CTA g owning channels [64 g, 64 g + 64) (one FP8 scale group of
// the main-KV row).  Each CTA copies its slice of the token's SWA key /
// value and C / Z rows, pools its 64 channels of the closed block (rows
// spread over 32 row groups, per-channel online softmax, merged through
// shuffles and shared memory), stores them, and multiplies them into its
// 64-row slice of W_IK (one bulk copy into shared memory, issued before the
// token position is known).  The partial indexer keys are summed by CTA 0 through distributed
// shared memory, which also quantises and stores the key row.
constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads)
decode_append_cluster_kernel(const int64_t* __restrict__ pos, int m, int d, int act_dtype,
                             const void* __restrict__ c_t, const void* __restrict__ z_t,
                             const void* __restrict__ k_t, const void* __restrict__ v_t, void* open_c, void* open_z,
                             void* swa_k, void* swa_v, int swa_dtype, int swa_cap, OutSpec kv, int64_t cap,
                             const void* __restrict__ w_ik, int w_dtype, int d_idx, OutSpec kidx,
                             int32_t* __restrict__ n_visible_out, int64_t* __restrict__ q_pos_out,
                             int32_t* __restrict__ q_req_out, uint4* __restrict__ zero, int64_t zero_n16) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(128) uint8_t wsm[];  // [64][d_idx] W_IK slice
  __shared__ uint64_t wbar;
  __shared__ float pooled[64];
  __shared__ float part[kAppendThreads];  // this CTA's partial indexer key
  __shared__ float red_m[8][64], red_s[8][64], red_a[8][64];
  __shared__ float amax_w[8];
  __shared__ int part_ok;
  const int g = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = g * 64;
  // this CTA's W_IK slice (64 contiguous rows) by one bulk copy, before anything else
  const int wbytes = 64 * d_idx * elem_bytes(w_dtype);
  if (w_ik != nullptr && tid == 0) {
    sm100::mbar_init(&wbar, 1);
    sm100::fence_barrier_init();
    sm100::mbar_arrive_expect_tx(&wbar, wbytes);
    sm100::bulk_load(wsm, static_cast<const uint8_t*>(w_ik) + static_cast<int64_t>(c0) * d_idx * elem_bytes(w_dtype),
                     wbytes, &wbar);
  }
  // (the barrier's initialisation reaches the other threads through the
  // __syncthreads of the pooling below, before any of them waits on it)
  // zero this CTA's share of the later kernels' control words
  if (zero != nullptr) {
    const int64_t nb = static_cast<int64_t>(gridDim.x) * gridDim.y, me = static_cast<int64_t>(b) * gridDim.x + g;
    const int64_t z0 = zero_n16 * me / nb, z1 = zero_n16 * (me + 1) / nb;
    for (int64_t i = z0 + tid; i < z1; i += kAppendThreads) zero[i] = make_uint4(0, 0, 0, 0);
  }
  // Every load is issued before any is used: none of the addresses depends on
  // the token position (a block that closes takes its last row from the
  // token, rows 0 .. m-2 from the open-block buffer).
  const int ea = elem_bytes(act_dtype), es = elem_bytes(swa_dtype);
  const char* crow = static_cast<const char*>(c_t) + static_cast<int64_t>(b) * d * ea;
  const char* zrow = static_cast<const char*>(z_t) + static_cast<int64_t>(b) * d * ea;
  char* ocb = static_cast<char*>(open_c) + static_cast<int64_t>(b) * m * d * ea;
  char* ozb = static_cast<char*>(open_z) + static_cast<int64_t>(b) * m * d * ea;
  const int64_t t = pos[b];
  // the token's rows: 4 rows x 8 vectors of 8 channels
  float tokv[8];
  const int trow = tid >> 3, tcol = c0 + (tid & 7) * 8;
  if (tid < 32) {
    const char* src = trow == 0 ? static_cast<const char*>(k_t) : trow == 1 ? static_cast<const char*>(v_t)
                    : trow == 2 ? crow : zrow;
    if (trow < 2) src += static_cast<int64_t>(b) * d * ea;
    load8(src, act_dtype, tcol, nullptr, 1, tokv);
  }
  // pooling: thread = (row group rg, channel vector cv); rows rg, rg + 32, ...
  const int cv = tid & 7, rg = tid >> 3;
  const int col = c0 + cv * 8;
  constexpr int kRowsInRegs = 4;  // rows per thread held at once (m <= 128 in one round)
  float zr[kRowsInRegs][8], cr[kRowsInRegs][8];
#pragma unroll
  for (int k = 0; k < kRowsInRegs; ++k) {
    const int i = rg + 32 * k;
    if (i < m) {
      load8(i == m - 1 ? zrow : ozb + static_cast<int64_t>(i) * d * ea, act_dtype, col, nullptr, 1, zr[k]);
      load8(i == m - 1 ? crow : ocb + static_cast<int64_t>(i) * d * ea, act_dtype, col, nullptr, 1, cr[k]);
    }
  }
  const bool closes = (t + 1) % m == 0;
  const int slot_m = static_cast<int>(t % m);
  const int64_t slot_w = t % swa_cap;
  if (tid < 32) {
    char* dst = trow == 0 ? static_cast<char*>(swa_k) + (static_cast<int64_t>(b) * swa_cap + slot_w) * d * es
              : trow == 1 ? static_cast<char*>(swa_v) + (static_cast<int64_t>(b) * swa_cap + slot_w) * d * es
              : (trow == 2 ? ocb : ozb) + static_cast<int64_t>(slot_m) * d * ea;
    store8(dst, trow < 2 ? swa_dtype : act_dtype, tcol, tokv);
  }
  if (g == 0 && tid == 0) {
    n_visible_out[b] = static_cast<int32_t>((t + 1) / m);
    q_pos_out[b] = t;
    q_req_out[b] = b;
  }
  if (closes) {  // uniform over the cluster: every CTA serves the same request
    float mx[8], sm[8], ac[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; sm[e] = 0.f; ac[e] = 0.f; }
    for (int i0 = 0; i0 < m; i0 += 32 * kRowsInRegs) {
      if (i0 > 0) {  // blocks longer than 128 rows: the next rows
#pragma unroll
        for (int k = 0; k < kRowsInRegs; ++k) {
          const int i = i0 + rg + 32 * k;
          if (i < m) {
            load8(i == m - 1 ? zrow : ozb + static_cast<int64_t>(i) * d * ea, act_dtype, col, nullptr, 1, zr[k]);
            load8(i == m - 1 ? crow : ocb + static_cast<int64_t>(i) * d * ea, act_dtype, col, nullptr, 1, cr[k]);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kRowsInRegs; ++k) {
        if (i0 + rg + 32 * k >= m) break;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float nm = fmaxf(mx[e], zr[k][e]);
          const float f = expf(mx[e] - nm), p = expf(zr[k][e] - nm);
          sm[e] = sm[e] * f + p;
          ac[e] = ac[e] * f + p * cr[k][e];
          mx[e] = nm;
        }
      }
    }
    // merge the four row groups of this warp (lanes cv, cv + 8, cv + 16, cv + 24)
#pragma unroll
    for (int o = 8; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float om = __shfl_xor_sync(0xFFFFFFFFu, mx[e], o);
        const float os = __shfl_xor_sync(0xFFFFFFFFu, sm[e], o);
        const float oa = __shfl_xor_sync(0xFFFFFFFFu, ac[e], o);
        const float nm = fmaxf(mx[e], om);
        const float f0 = nm == -INFINITY ? 0.f : expf(mx[e] - nm), f1 = nm == -INFINITY ? 0.f : expf(om - nm);
        sm[e] = sm[e] * f0 + os * f1;
        ac[e] = ac[e] * f0 + oa * f1;
        mx[e] = nm;
      }
    if (lane < 8)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red_m[warp][cv * 8 + e] = mx[e];
        red_s[warp][cv * 8 + e] = sm[e];
        red_a[warp][cv * 8 + e] = ac[e];
      }
    __syncthreads();
    if (tid < 64) {
      float M = -INFINITY, S = 0.f, A = 0.f;
      for (int w = 0; w < 8; ++w) M = fmaxf(M, red_m[w][tid]);
      for (int w = 0; w < 8; ++w) {
        const float f = red_m[w][tid] == -INFINITY ? 0.f : expf(red_m[w][tid] - M);
        S += red_s[w][tid] * f;
        A += red_a[w][tid] * f;
      }
      pooled[tid] = A / S;
    }
    __syncthreads();
    // the main-KV row's 64 channels (FP8: this group's scale)
    const int64_t row = static_cast<int64_t>(b) * cap + (t + 1) / m - 1;
    if (warp == 0) {
      float v[8];
      const int cc = (lane & 7) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = pooled[cc + e];
      store_pooled8(kv, row, c0 + cc, v, lane < 8);
    }
    // partial indexer key of these 64 channels (bounded wait for the slice;
    // on a timeout the key row is not written)
    if (w_ik != nullptr) {
      const bool wok = sm100::mbar_wait(&wbar, 0, 1u << 22);
      float acc = 0.f;
      if (wok && tid < d_idx) {
        if (w_dtype == kBF16) {
          const uint16_t* w = reinterpret_cast<const uint16_t*>(wsm) + tid;
#pragma unroll 16
          for (int i = 0; i < 64; ++i) acc = fmaf(pooled[i], bf16_bits_to_f32(w[i * d_idx]), acc);
        } else {
          const float* w = reinterpret_cast<const float*>(wsm) + tid;
#pragma unroll 16
          for (int i = 0; i < 64; ++i) acc = fmaf(pooled[i], w[i * d_idx], acc);
        }
      }
      part[tid] = acc;
      if (tid == 0) part_ok = wok ? 1 : 0;
    }
    cluster.sync();
    int all_ok = 1;
    if (w_ik != nullptr && g == 0)
      for (int r = 0; r < static_cast<int>(cluster.num_blocks()); ++r) all_ok &= *cluster.map_shared_rank(&part_ok, r);
    if (w_ik != nullptr && g == 0 && all_ok) {
      float key = 0.f;
      if (tid < d_idx)
        for (int r = 0; r < static_cast<int>(cluster.num_blocks()); ++r) key += cluster.map_shared_rank(part, r)[tid];
      if (kidx.dtype == kFP8) {
        float a = tid < d_idx ? fabsf(key) : 0.f;
        a = warp_max(a);
        if (lane == 0) amax_w[warp] = a;
        __syncthreads();
        float amax = 0.f;
        for (int w = 0; w < 8; ++w) amax = fmaxf(amax, amax_w[w]);
        const float s = amax > 0.f ? amax / 448.f : 1.f;
        if (tid < d_idx) static_cast<uint8_t*>(kidx.data)[row * kidx.row_stride + tid] = f32_to_e4m3(key / s);
        if (tid == 0) static_cast<float*>(kidx.scale)[row * kidx.scale_stride] = s;
      } else if (tid < d_idx) {
        if (kidx.dtype == kBF16) static_cast<uint16_t*>(kidx.data)[row * kidx.row_stride + tid] = f32_to_bf16_bits(key);
        else static_cast<float*>(kidx.data)[row * kidx.row_stride + tid] = key;
      }
    }
    cluster.sync();  // CTA 0 has read every partial before any CTA exits
  } else if (w_ik != nullptr && tid == 0) {
    sm100::mbar_wait(&wbar, 0, 1u << 22);  // the W_IK copy lands before the CTA exits
  }
}

OutSpec make_out(const csa_tensor_t* t, int row_elems) { return make_out_spec(t, row_elems); }

}  // namespace

csa_status_t launch_compress(const csa_tensor_t* C, const csa_tensor_t* Z, int batch, int64_t n_tokens, int d,
                             int m, const csa_tensor_t* out, int64_t out_rows, const csa_tensor_t* w_ik,
                             int d_idx, const csa_tensor_t* kidx_out, cudaStream_t stream) {
  const int64_t n_blocks = n_tokens / m;
  if (n_blocks == 0 || batch == 0) return CSA_OK;
  dim3 grid(static_cast<unsigned>((n_blocks + kCompressNB - 1) / kCompressNB), batch);
  size_t smem = w_ik ? static_cast<size_t>(kCompressNB) * d * sizeof(float) : 0;
  if (w_ik) {
    const size_t wb = static_cast<size_t>(d) * d_idx * elem_bytes(w_ik->dtype);
    if (wb <= kMaxWSmem) smem += wb + (2 * kCompressThreads + d_idx) * sizeof(float);
  }
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  prof_begin(stream);
  compress_kernel<<<grid, kCompressThreads, smem, stream>>>(
      C->data, Z->data, C->dtype, n_tokens, d, m, n_blocks, make_out(out, d), out_rows,
      w_ik ? w_ik->data : nullptr, w_ik ? w_ik->dtype : kF32, d_idx, make_out(kidx_out, d_idx));
  return check_launch("compress_kernel", stream);
}

csa_status_t launch_decode_append(const csa_params_t* p, int batch, const csa_decode_caches_t* cc,
                                  const csa_decode_token_t* tok, const int64_t* pos, int32_t* n_visible,
                                  int64_t* q_pos, int32_t* q_req, void* zero, size_t zero_bytes,
                                  cudaStream_t stream) {
  const int groups = p->d / 64;
  if (p->d % 64 == 0 && groups >= 1 && groups <= 8 && (tok->w_ik.data == nullptr || p->d_idx <= kAppendThreads)) {
    // one cluster of d / 64 CTAs per request
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups, batch);
    cfg.blockDim = dim3(kAppendThreads);
    const int wbytes = tok->w_ik.data ? 64 * p->d_idx * elem_bytes(tok->w_ik.dtype) : 0;
    cfg.dynamicSmemBytes = wbytes;
    if (wbytes > 48 * 1024)
      cudaFuncSetAttribute(decode_append_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, wbytes);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = groups;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    prof_begin(stream);
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, decode_append_cluster_kernel, pos, p->m, p->d, tok->c.dtype, tok->c.data, tok->z.data, tok->k_swa.data,
        tok->v_swa.data, cc->open_c.data, cc->open_z.data, cc->swa_k.data, cc->swa_v.data, cc->swa_k.dtype, p->swa_cap,
        make_out(&cc->kv, p->d), cc->cap, tok->w_ik.data, tok->w_ik.dtype, p->d_idx, make_out(&cc->kidx, p->d_idx),
        n_visible, q_pos, q_req, static_cast<uint4*>(zero), static_cast<int64_t>(zero_bytes / 16));
    if (e != cudaSuccess) {
      check_launch("decode_append_cluster_kernel", stream);
      return set_error(CSA_ERR_CUDA, "decode_append_cluster_kernel launch: %s", cudaGetErrorString(e));
    }
    return check_launch("decode_append_cluster_kernel", stream);
  }
  size_t smem = static_cast<size_t>(p->d) * sizeof(float);
  if (tok->w_ik.data) {
    const size_t wb = static_cast<size_t>(p->d) * p->d_idx * elem_bytes(tok->w_ik.dtype);
    if (wb <= kMaxWSmem) smem += wb + (2 * kCompressThreads + p->d_idx) * sizeof(float);
  }
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(decode_append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  prof_begin(stream);
  decode_append_kernel<<<batch, kCompressThreads, smem, stream>>>(
      pos, p->m, p->d, tok->c.dtype, tok->c.data, tok->z.data, tok->k_swa.data, tok->v_swa.data,
      cc->open_c.data, cc->open_z.data, cc->swa_k.data, cc->swa_v.data, cc->swa_k.dtype, p->swa_cap,
      make_out(&cc->kv, p->d), cc->cap, tok->w_ik.data, tok->w_ik.dtype, p->d_idx, make_out(&cc->kidx, p->d_idx),
      n_visible, q_pos, q_req, static_cast<uint4*>(zero), static_cast<int64_t>(zero_bytes / 16));
  return check_launch("decode_append_kernel", stream);
}

}  // namespace csa
