// Device-side helpers shared by the kernels of the library: storage-format
// loads/stores (fp32, bf16, FP8 E4M3 with fp32 group scales, MXFP4: E2M1
// with E4M3 scales per 16 elements: tech-report tour, "FP4 main KV cache"),
// the ordered
// 32-bit key of an fp32 score, and host-side error plumbing.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

constexpr int kF32 = CSA_F32;
constexpr int kBF16 = CSA_BF16;
constexpr int kFP8 = CSA_FP8_E4M3;
constexpr int kMXFP4 = CSA_MXFP4_E2M1;

// --------------------------------------------------------------------------
// scalar conversions
// --------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Two E4M3 codes (low byte = first element) -> two floats.  E4M3 converts
// exactly to f16 (and f16 exactly to f32).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t two_codes) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
  __half2 hh;
  hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&h));
}

// Round-to-nearest-even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// OCP E2M1: sign in bit 3, two exponent bits (bias 1), one mantissa bit;
// exponent 0 is subnormal (0 or 0.5).  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_to_f32(uint32_t code) {
  const uint32_t m = code & 7u;
  const uint32_t mag = m >= 2u ? (((m >> 1) + 126u) << 23) | ((m & 1u) << 22) : (m ? 0x3F000000u : 0u);
  return __uint_as_float(mag | ((code & 8u) << 28));
}

// Round to the nearest E2M1 value, a tie to the even code, saturating at 6:
// the decision points are the midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5
// (a midpoint itself goes to the neighbour with the even code).
__device__ __forceinline__ uint32_t f32_to_e2m1(float x) {
  const float a = fabsf(x);
  const uint32_t m = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
                   : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.f ? 6u : 7u;
  return m | ((__float_as_uint(x) >> 28) & 8u);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}

// --------------------------------------------------------------------------
// 8-element vector loads (16 B of bf16, 32 B of fp32, 8 B of fp8)
// --------------------------------------------------------------------------
// Loads elements [col, col+8) of a row into v (fp32).  For FP8, `scale`
// points at the row's fp32 group scales and `group` is the group length
// (a multiple of 8, so the 8 elements share one scale).  (MXFP4 rows: load8_kv.)
__device__ __forceinline__ void load8(const void* row, int dtype, int col, const void* scale, int group,
                                      float v[8]) {
  if (dtype == kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + col);
    float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else if (dtype == kBF16) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(row) + col));
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(row) + col));
    float s = __ldg(static_cast<const float*>(scale) + col / group);
    uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float2 lo = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] & 0xFFFF));
      float2 hi = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] >> 16));
      v[4 * i + 0] = lo.x * s; v[4 * i + 1] = lo.y * s;
      v[4 * i + 2] = hi.x * s; v[4 * i + 3] = hi.y * s;
    }
  }
}

// load8 for compressed main-KV rows, which may also be MXFP4: `row` at the
// row's first code byte, `scale` at its E4M3 scale bytes (group 16).  Kept
// apart from load8 so that the activation loads carry no MXFP4 code.
__device__ __forceinline__ void load8_kv(const void* row, int dtype, int col, const void* scale, int group,
                                         float v[8]) {
  if (dtype == kMXFP4) {
    const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(row) + col / 2));
    const float s = e4m3_to_f32(__ldg(static_cast<const uint8_t*>(scale) + col / 16));
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = e2m1_to_f32(u >> (4 * e)) * s;
  } else {
    load8(row, dtype, col, scale, group, v);
  }
}

// Stores 8 fp32 values as fp32 or bf16 (not FP8: FP8 needs a group scale).
__device__ __forceinline__ void store8(void* row, int dtype, int col, const float v[8]) {
  if (dtype == kF32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(row) + col);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = static_cast<uint32_t>(f32_to_bf16_bits(v[2 * i])) |
             (static_cast<uint32_t>(f32_to_bf16_bits(v[2 * i + 1])) << 16);
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(row) + col) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__device__ __forceinline__ float load1(const void* row, int dtype, int col, const void* scale, int group) {
  if (dtype == kF32) return __ldg(static_cast<const float*>(row) + col);
  if (dtype == kBF16) return bf16_bits_to_f32(__ldg(static_cast<const uint16_t*>(row) + col));
  return e4m3_to_f32(__ldg(static_cast<const uint8_t*>(row) + col)) *
         __ldg(static_cast<const float*>(scale) + col / group);
}

// Bytes per element (MXFP4: see row_bytes).
__host__ __device__ __forceinline__ int elem_bytes(int dtype) {
  return dtype == kF32 ? 4 : (dtype == kBF16 ? 2 : 1);
}

// Bytes of `n` elements of a row (MXFP4: two elements per byte).
__host__ __device__ __forceinline__ int64_t row_bytes(int dtype, int64_t n) {
  return dtype == kMXFP4 ? n / 2 : n * elem_bytes(dtype);
}

// --------------------------------------------------------------------------
// ordered key of an fp32 score: larger float -> larger unsigned key;
// -0 and +0 map to the same key.
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// --------------------------------------------------------------------------
// warp helpers
// --------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// --------------------------------------------------------------------------
// host-side error reporting (defined in csa_api.cu)
// --------------------------------------------------------------------------
csa_status_t set_error(csa_status_t st, const char* fmt, ...);
// Every kernel launch is bracketed by prof_begin(stream) before it and
// check_launch(name, stream) after it: check_launch reports launch errors
// and, while csa_profile_start() is active, records CUDA events around the
// launch on its stream.
void prof_begin(cudaStream_t stream);
csa_status_t check_launch(const char* what, cudaStream_t stream);

}  // namespace csa
