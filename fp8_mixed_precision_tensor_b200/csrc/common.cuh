// common.cuh -- device-side numerics shared by the libfp8 kernels.
//
// Formats ("Training and inference of large language models using 8-bit
// floating point", 제안 방법): E4M3 for weights and activations, E5M2 for
// gradients; encodings per the OCP FP8 specification.  Scale rule from the
// same section: s = 2^(floor(log2(fmt_max / amax)) - margin), evaluated here
// with integer exponent/significand arithmetic on the binary32 fields.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp8.h"

namespace fp8lib {

// Sticky device status word (FP8_STATUS_* bits), read back by fp8_get_status.
__device__ unsigned int g_status;
// The value fp8_get_status took out of g_status, for its copy to the host.
__device__ unsigned int g_status_taken;

// Read and clear the status word in one atomic operation.
__global__ void k_take_status() { g_status_taken = atomicExch(&g_status, 0u); }

constexpr float kMaxE4M3 = 448.0f;
constexpr float kMaxE5M2 = 57344.0f;
constexpr float kMaxF16 = 65504.0f;

__host__ __device__ inline float fmt_max_of(int fmt) {
  return fmt == FP8_E4M3 ? kMaxE4M3 : (fmt == FP8_E5M2 ? kMaxE5M2 : kMaxF16);
}

// Largest finite positive code (also the saturation code) of an FP8 format.
__device__ __forceinline__ uint32_t top_code(int fmt) { return fmt == FP8_E4M3 ? 0x7Eu : 0x7Bu; }

// ---------------------------------------------------------------------------
// Scale rule.  Split a finite positive binary32 into (unbiased exponent,
// 23-bit fraction of the normalised significand); subnormals are normalised.
__device__ __forceinline__ void split_binary32(float a, int &exp2, uint32_t &frac) {
  uint32_t u = __float_as_uint(a);
  int e = (u >> 23) & 0xff;
  uint32_t f = u & 0x7fffffu;
  if (e == 0) {                      // subnormal: value = f * 2^-149
    int msb = 31 - __clz(f);         // 0..22
    exp2 = msb - 149;
    frac = (f << (23 - msb)) & 0x7fffffu;
  } else {
    exp2 = e - 127;
    frac = f;
  }
}

// floor(log2(fmax / a)) = the largest e with a * 2^e <= fmax, for finite a > 0.
// With a = 1.fa * 2^ea and fmax = 1.ff * 2^ef the answer is ef - ea when
// 1.fa <= 1.ff, else one less.
__device__ __forceinline__ int floor_log2_ratio(float a, float fmax) {
  int ea, ef;
  uint32_t fa, ff;
  split_binary32(a, ea, fa);
  split_binary32(fmax, ef, ff);
  return (fa <= ff) ? (ef - ea) : (ef - ea - 1);
}

__device__ __forceinline__ float pow2f(int k) {  // k in [-126, 127]
  return __uint_as_float((uint32_t)(k + 127) << 23);
}

__device__ __forceinline__ int clamp_exp(int k) { return k < -126 ? -126 : (k > 126 ? 126 : k); }

// Exponent k of the total scale mu * s_g = 2^k for a tensor with this amax,
// where s_g = 2^clamp(floor(log2(fmax / (mu * amax))) - margin) and
// log2mu = log2(mu).  amax == 0 and a non-finite amax give s_g = 1; the
// latter returns false.
__device__ __forceinline__ bool scale_exponent(float amax, float fmax, int margin, int log2mu,
                                               int &k) {
  const bool finite = fabsf(amax) <= 3.402823466e38f;  // false for NaN and inf
  int kg = 0;
  if (finite && amax != 0.0f) kg = clamp_exp(floor_log2_ratio(amax, fmax) - log2mu - margin);
  k = clamp_exp(kg + log2mu);
  return finite;
}

// ---------------------------------------------------------------------------
// Encoding.  Finite values: round to nearest even with saturation (the
// hardware cvt with .satfinite).  Specials are fixed up explicitly so the
// result does not depend on the cvt's special-value conventions:
// +-inf -> +-max, NaN -> 0x7F (a NaN's sign is not kept).
__device__ __forceinline__ uint32_t fix_special(uint32_t code, float y, int fmt) {
  uint32_t u = __float_as_uint(y);
  uint32_t sign = (u >> 24) & 0x80u;
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7Fu;  // NaN
  if ((u & 0x7fffffffu) == 0x7f800000u) return sign | top_code(fmt);
  return code;
}

// Two floats -> two codes in the low 16 bits (a in bits 0-7, b in bits 8-15),
// with an explicit test for the special values.  The reference of enc2.
template <int FMT>
__device__ __forceinline__ uint32_t enc2_checked(float a, float b) {
  __nv_fp8x2_storage_t r = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE,
                                                    FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2);
  uint32_t c = (uint32_t)r;
  uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  if ((ua & 0x7f800000u) == 0x7f800000u || (ub & 0x7f800000u) == 0x7f800000u) {
    uint32_t ca = fix_special(c & 0xffu, a, FMT);
    uint32_t cb = fix_special((c >> 8) & 0xffu, b, FMT);
    c = ca | (cb << 8);
  }
  return c;
}

// The same two codes without a test or a branch: the saturating cvt already
// maps +-inf to +-max; a NaN code of either sign is made 0x7F with byte-wise
// SIMD compares (E4M3: the one NaN pattern S.1111.111; E5M2: S.11111.mm with
// mm != 0).  fp8_selftest_encode checks enc2 against enc2_checked on every
// binary32 value in each lane.
template <int FMT>
__device__ __forceinline__ uint32_t enc2(float a, float b) {
  const uint32_t c = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE,
                                                         FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2);
  const uint32_t mag = c & 0x7f7fu;
  const uint32_t nan = FMT == FP8_E4M3 ? __vcmpeq4(mag, 0x7f7fu) : __vcmpgtu4(mag, 0x7c7cu);
  return (c & ~nan) | (nan & 0x7f7fu);
}

// Four floats -> four codes packed little-endian in a 32-bit word.
template <int FMT>
__device__ __forceinline__ uint32_t enc4(float a, float b, float c, float d) {
  return enc2<FMT>(a, b) | (enc2<FMT>(c, d) << 16);
}

// Two floats -> two IEEE halves (round to nearest even) packed in 32 bits.
__device__ __forceinline__ uint32_t f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// ---------------------------------------------------------------------------
// Decoding of packed codes.
template <int FMT>
__device__ __forceinline__ float2 dec2(uint32_t two_codes) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_codes & 0xffffu),
                                              FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

__device__ __forceinline__ float2 h2f2(uint32_t two_halves) {
  return __half22float2(*reinterpret_cast<__half2 *>(&two_halves));
}

// A factor in both lanes of a float2, for the packed binary32 instructions
// of sm_100 (__fmul2_rn and friends: two round-to-nearest results per
// instruction, each the same as the scalar operation's).
__device__ __forceinline__ float2 both(float a) { return make_float2(a, a); }

// ---------------------------------------------------------------------------
// Magnitude of an element as the bit pattern of a binary32 (order-preserving
// for non-negative values, NaN above inf), so maxima can use integer max.
__device__ __forceinline__ uint32_t absbits_f32(float x) { return __float_as_uint(x) & 0x7fffffffu; }

__device__ __forceinline__ void atomic_max_bits(float *dst, uint32_t bits) {
  atomicMax(reinterpret_cast<unsigned int *>(dst), bits);
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) { return __reduce_max_sync(0xffffffffu, v); }

// Block-wide maximum; every thread gets the result.  `red` holds >= 32 words.
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t *red) {
  v = warp_max_u32(v);
  int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  uint32_t r = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0u;
  if (warp == 0) r = warp_max_u32(r);
  if (threadIdx.x == 0) red[0] = r;
  __syncthreads();
  return red[0];
}

// Block-wide sum of two per-thread counts added to dst[0], dst[1] (one
// atomic each per block).  `red` holds >= 64 words.
__device__ __forceinline__ void block_add_counts(uint32_t a, uint32_t b, uint32_t *red,
                                                 unsigned long long *dst) {
  a = __reduce_add_sync(0xffffffffu, a);
  b = __reduce_add_sync(0xffffffffu, b);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) {
    red[warp] = a;
    red[32 + warp] = b;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long sa = 0, sb = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) {
      sa += red[w];
      sb += red[32 + w];
    }
    if (sa) atomicAdd(dst, sa);
    if (sb) atomicAdd(dst + 1, sb);
  }
}

// log2 of a device-side mu that must be a power of two in [2^-32, 2^32];
// anything else raises FP8_STATUS_BAD_MU and counts as mu = 1.
__device__ __forceinline__ int device_log2mu(float mu) {
  const uint32_t u = __float_as_uint(mu);
  const int e = (int)(u >> 23) - 127;
  if ((u & 0x807fffffu) != 0u || e < -32 || e > 32) {
    atomicOr(&g_status, FP8_STATUS_BAD_MU);
    return 0;
  }
  return e;
}

}  // namespace fp8lib
