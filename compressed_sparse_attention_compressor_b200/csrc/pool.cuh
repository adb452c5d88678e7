// Block pooling and quantised row stores shared by the compressor, the
// decode-step append kernel and the indexer's in-kernel append (whose
// argument block is below).
//
// "DeepSeek-V4.1-Flash, illustrated", Equation (1) figure (compression
// weights Z over a block of projected entries C); tech-report tour, "A
// simpler compressor" (non-overlapping groups, no positional term).
#pragma once

#include "common.cuh"

namespace csa {

// Destination of pooled rows: fp32 / bf16, FP8 E4M3 codes with one fp32
// scale per `group` elements (scale = max|x| / 448, 1 for an all-zero
// group), or MXFP4 E2M1 codes with one E4M3 scale per 16 elements.
struct OutSpec {
  void* data;
  void* scale;
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

// Stores 8 pooled channels of one row.  For FP8 and MXFP4 every lane of the
// warp must call this (the 8 lanes of a 64-channel FP8 group, or the 2 lanes
// of a 16-channel MXFP4 group, exchange maxima); `valid` masks the store.
//
// MXFP4 (tech-report tour, chapter "Engram, DSpark, FP4", section "FP4 main
// KV cache"): the group's scale is the E4M3 value nearest max|x| / 6 (so
// that max|x| lands on the largest E2M1 magnitude), each element the E2M1
// value nearest x / scale, saturating at 6; an all-zero scale stores zeros.
// MX4 = false leaves the MXFP4 branch out (callers that never store MXFP4).
template <bool MX4 = true>
__device__ __forceinline__ void store_pooled8(const OutSpec& o, int64_t row, int col, const float v[8],
                                              bool valid) {
  if (MX4 && o.dtype == kMXFP4) {
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));  // lanes 2g, 2g+1: one 16-channel group
    if (!valid) return;
    const uint8_t sc = f32_to_e4m3(amax / 6.f);
    const float s = e4m3_to_f32(sc);
    uint32_t w = 0u;
    if (s > 0.f) {
#pragma unroll
      for (int e = 0; e < 8; ++e) w |= f32_to_e2m1(v[e] / s) << (4 * e);
    }
    uint8_t* dst = static_cast<uint8_t*>(o.data) + (row * o.row_stride + col) / 2;
    *reinterpret_cast<uint32_t*>(dst) = w;
    if ((col % 16) == 0) static_cast<uint8_t*>(o.scale)[row * o.scale_stride + col / 16] = sc;
    return;
  }
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
  if ((col % o.group) == 0) static_cast<float*>(o.scale)[row * o.scale_stride + col / o.group] = s;
}

inline OutSpec make_out_spec(const csa_tensor_t* t, int row_elems) {
  OutSpec o;
  o.data = t ? t->data : nullptr;
  o.scale = t ? t->scale : nullptr;
  o.dtype = t ? t->dtype : kF32;
  const bool scaled = t && (t->dtype == kFP8 || t->dtype == kMXFP4);
  o.group = scaled ? t->scale_group : 1;
  o.row_stride = row_elems;
  o.scale_stride = scaled ? row_elems / t->scale_group : 0;
  return o;
}

// The decode step's append, done inside the indexer by the CTA that owns the
// last chunk of each request: the token's SWA key / value and C / Z rows go
// to their slots; if the token closes its block, the block is pooled into a
// main-KV row and its indexer key (pooled fp32 row . W_IK) is stored, before
// that CTA streams its keys (the new key is in its last tile).
struct AppendArgs {
  const int64_t* pos;  // [batch] the new token's position t
  int m, d, act_dtype;
  const void* c_t; const void* z_t; const void* k_t; const void* v_t;  // [batch][d]
  void* open_c; void* open_z;                                         // [batch][m][d]
  void* swa_k; void* swa_v; int swa_dtype; int swa_cap;               // [batch][swa_cap][d]
  OutSpec kv;                                                          // [batch][cap][d] main-KV rows
  const void* w_ik; int w_dtype;                                      // [d][128]
  OutSpec kidx;                                                        // [batch][cap][128] indexer keys
  int32_t* n_vis_out; int64_t* q_pos_out; int32_t* q_req_out;
  int shrink;  // tiles the last chunk gives up to the other chunks
};

}  // namespace csa
