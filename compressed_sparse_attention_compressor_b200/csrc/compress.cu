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
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kCompressThreads = 256;
constexpr int kCompressNB = 8;  // blocks pooled per CTA

struct OutSpec {
  void* data;
  float* scale;
  int dtype;
  int group;
  int64_t row_stride;    // elements between rows
  int64_t scale_stride;  // scales between rows
};

// Pools 8 channels [col, col+8) of one block.  rowC(i) / rowZ(i) give the
// i-th row of the block (i < m).  Rows are loaded four at a time, all four
// loads issued before their use: first the block maximum, then the
// exp-weighted sums.
template <class RowC, class RowZ>
__device__ __forceinline__ void pool8(RowC rowC, RowZ rowZ, int in_dtype, int m, int col, float out[8]) {
  float mx[8], den[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; den[e] = 0.f; out[e] = 0.f; }
  for (int i0 = 0; i0 < m; i0 += 4) {
    float z[4][8];
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (i0 + b < m) load8(rowZ(i0 + b), in_dtype, col, nullptr, 1, z[b]);
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (i0 + b < m)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], z[b][e]);
  }
  for (int i0 = 0; i0 < m; i0 += 4) {
    float z[4][8], c[4][8];
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (i0 + b < m) {
        load8(rowZ(i0 + b), in_dtype, col, nullptr, 1, z[b]);
        load8(rowC(i0 + b), in_dtype, col, nullptr, 1, c[b]);
      }
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (i0 + b < m)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a = expf(z[b][e] - mx[e]);
          den[e] += a;
          out[e] = fmaf(a, c[b][e], out[e]);
        }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = out[e] / den[e];
}

// Stores 8 pooled channels of one row.  For FP8 every lane of the warp must
// call this (the 8 lanes of a 64-channel group exchange maxima); `valid`
// masks the store.
__device__ __forceinline__ void store_pooled8(const OutSpec& o, int64_t row, int col, const float v[8],
                                              bool valid) {
  if (o.dtype != kFP8) {
    if (valid) store8(static_cast<char*>(o.data) + row * o.row_stride * elem_bytes(o.dtype), o.dtype, col, v);
    return;
  }
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
  // lanes 8g..8g+7 hold one 64-channel group
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
  if (!valid) return;
  const float s = amax > 0.f ? amax / 448.f : 1.f;
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e / 4] |= static_cast<uint32_t>(f32_to_e4m3(v[e] / s)) << (8 * (e % 4));
  uint8_t* dst = static_cast<uint8_t*>(o.data) + row * o.row_stride + col;
  *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  if ((col % o.group) == 0) o.scale[row * o.scale_stride + col / o.group] = s;
}

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
    if (lane == 0) ko.scale[row * ko.scale_stride] = s;
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
    if (lane == 0) ko.scale[row * ko.scale_stride] = s;
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

OutSpec make_out(const csa_tensor_t* t, int row_elems) {
  OutSpec o;
  o.data = t ? t->data : nullptr;
  o.scale = t ? t->scale : nullptr;
  o.dtype = t ? t->dtype : kF32;
  o.group = (t && t->dtype == kFP8) ? t->scale_group : 1;
  o.row_stride = row_elems;
  o.scale_stride = (t && t->dtype == kFP8) ? row_elems / t->scale_group : 0;
  return o;
}

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
