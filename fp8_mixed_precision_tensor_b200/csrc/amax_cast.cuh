// amax_cast.cuh -- per-tensor amax, scale and cast kernels (HBM-bound).
//
// "Training and inference of large language models using 8-bit floating
// point", 제안 방법: the scaling bias of every weight, activation and gradient
// tensor comes from its maximum absolute value; the tensor is scaled and then
// cast to FP8.  "FP8-LM: Training FP8 Large Language Models", 提案手法 O1,
// Eq. 3: gradients are auto-scaled by mu before the cast.
//
// Design: grid-stride streaming kernels over 16-byte vectors with several
// independent loads in flight per thread; amax reduces |x| as integer bit
// patterns (warp redux -> block -> one atomicMax per block); the cast reads
// its scale from device memory so amax -> scale -> cast chains with no host
// round-trip.
#pragma once

#include "common.cuh"

namespace fp8lib {

constexpr int kStreamThreads = 256;

// 16 elements of a high-precision tensor as floats.
template <int DT>
struct Vec16 {
  static constexpr int kBytes = DT == FP8_DT_F32 ? 64 : 32;
};

template <int DT>
__device__ __forceinline__ void load16(const void *base, size_t group, float (&f)[16]) {
  if constexpr (DT == FP8_DT_F32) {
    const uint4 *p = reinterpret_cast<const uint4 *>(base) + group * 4;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      uint4 v = __ldcs(p + j);
      f[4 * j + 0] = __uint_as_float(v.x);
      f[4 * j + 1] = __uint_as_float(v.y);
      f[4 * j + 2] = __uint_as_float(v.z);
      f[4 * j + 3] = __uint_as_float(v.w);
    }
  } else {
    const uint4 *p = reinterpret_cast<const uint4 *>(base) + group * 2;
#pragma unroll
    for (int j = 0; j < 2; j++) {
      uint4 v = __ldcs(p + j);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; k++) {
        if constexpr (DT == FP8_DT_BF16) {
          f[8 * j + 2 * k] = __uint_as_float(w[k] << 16);
          f[8 * j + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        } else {
          float2 t = h2f2(w[k]);
          f[8 * j + 2 * k] = t.x;
          f[8 * j + 2 * k + 1] = t.y;
        }
      }
    }
  }
}

template <int DT>
__device__ __forceinline__ float load1(const void *base, size_t i) {
  if constexpr (DT == FP8_DT_F32) return reinterpret_cast<const float *>(base)[i];
  uint32_t h = reinterpret_cast<const uint16_t *>(base)[i];
  if constexpr (DT == FP8_DT_BF16) return __uint_as_float(h << 16);
  return __half2float(__ushort_as_half((unsigned short)h));
}

// ---------------------------------------------------------------------------
// amax.  Magnitudes are compared as unsigned bit patterns: for bf16 and f32
// that is the raw |bits|; fp16 halves are widened to f32 first.
template <int DT>
__device__ __forceinline__ uint32_t group_absmax(const void *base, size_t group) {
  if constexpr (DT == FP8_DT_BF16) {
    // 16 bf16 = 2 x uint4; SIMD max over 16-bit halves of |bits|.
    const uint4 *p = reinterpret_cast<const uint4 *>(base) + group * 2;
    uint4 a = __ldcg(p), b = __ldcg(p + 1);
    uint32_t m = __vmaxu2(__vmaxu2(a.x & 0x7fff7fffu, a.y & 0x7fff7fffu),
                          __vmaxu2(a.z & 0x7fff7fffu, a.w & 0x7fff7fffu));
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(b.x & 0x7fff7fffu, b.y & 0x7fff7fffu),
                             __vmaxu2(b.z & 0x7fff7fffu, b.w & 0x7fff7fffu)));
    uint32_t hi = m >> 16, lo = m & 0xffffu;
    return (hi > lo ? hi : lo) << 16;  // bf16 -> f32 bits
  } else if constexpr (DT == FP8_DT_F32) {
    const uint4 *p = reinterpret_cast<const uint4 *>(base) + group * 4;
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      uint4 v = __ldcg(p + j);
      m = max(m, max(max(v.x & 0x7fffffffu, v.y & 0x7fffffffu), max(v.z & 0x7fffffffu, v.w & 0x7fffffffu)));
    }
    return m;
  } else {
    const uint4 *p = reinterpret_cast<const uint4 *>(base) + group * 2;
    uint4 a = __ldcg(p), b = __ldcg(p + 1);
    uint32_t m = __vmaxu2(__vmaxu2(a.x & 0x7fff7fffu, a.y & 0x7fff7fffu),
                          __vmaxu2(a.z & 0x7fff7fffu, a.w & 0x7fff7fffu));
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(b.x & 0x7fff7fffu, b.y & 0x7fff7fffu),
                             __vmaxu2(b.z & 0x7fff7fffu, b.w & 0x7fff7fffu)));
    uint32_t hi = m >> 16, lo = m & 0xffffu;
    uint32_t h = hi > lo ? hi : lo;  // largest |half| bits (NaN above inf)
    return absbits_f32(__half2float(__ushort_as_half((unsigned short)h)));
  }
}

template <int DT>
__global__ void __launch_bounds__(kStreamThreads) k_amax(const void *__restrict__ x, size_t n,
                                                         float *__restrict__ amax) {
  __shared__ uint32_t red[32];
  const size_t groups = n / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
  for (; g + 3 * stride < groups; g += 4 * stride) {
    m0 = max(m0, group_absmax<DT>(x, g));
    m1 = max(m1, group_absmax<DT>(x, g + stride));
    m2 = max(m2, group_absmax<DT>(x, g + 2 * stride));
    m3 = max(m3, group_absmax<DT>(x, g + 3 * stride));
  }
  for (; g < groups; g += stride) m0 = max(m0, group_absmax<DT>(x, g));
  uint32_t m = max(max(m0, m1), max(m2, m3));
  if (blockIdx.x == 0) {  // ragged tail (< 16 elements)
    for (size_t i = groups * 16 + threadIdx.x; i < n; i += blockDim.x)
      m = max(m, absbits_f32(load1<DT>(x, i)));
  }
  m = block_max_u32(m, red);
  if (threadIdx.x == 0) atomic_max_bits(amax, m);
}

// ---------------------------------------------------------------------------
// scale: one thread.
__global__ void k_compute_scale(const float *__restrict__ amax, float fmax, int margin, int log2mu,
                                float *__restrict__ scale, float *__restrict__ inv_scale) {
  int k;
  if (!scale_exponent(*amax, fmax, margin, log2mu, k)) atomicOr(&g_status, FP8_STATUS_NONFINITE);
  *scale = pow2f(k);
  *inv_scale = pow2f(-k);
}

// ---------------------------------------------------------------------------
// cast: 16 elements per thread-iteration, one 16-byte store of codes
// (or two of halves for the scaled-FP16 format).
template <int DT, int FMT>
__device__ __forceinline__ void cast_group(const void *x, size_t g, float s, void *q) {
  float f[16];
  load16<DT>(x, g, f);
#pragma unroll
  for (int j = 0; j < 16; j++) f[j] *= s;
  if constexpr (FMT == FP8_F16S) {
    uint4 lo = make_uint4(f16x2(f[0], f[1]), f16x2(f[2], f[3]), f16x2(f[4], f[5]), f16x2(f[6], f[7]));
    uint4 hi = make_uint4(f16x2(f[8], f[9]), f16x2(f[10], f[11]), f16x2(f[12], f[13]), f16x2(f[14], f[15]));
    uint4 *p = reinterpret_cast<uint4 *>(q) + g * 2;
    __stcs(p, lo);
    __stcs(p + 1, hi);
  } else {
    uint4 o = make_uint4(enc4<FMT>(f[0], f[1], f[2], f[3]), enc4<FMT>(f[4], f[5], f[6], f[7]),
                         enc4<FMT>(f[8], f[9], f[10], f[11]), enc4<FMT>(f[12], f[13], f[14], f[15]));
    __stcs(reinterpret_cast<uint4 *>(q) + g, o);
  }
}

// Scale source of a cast: a precomputed scale, or the amax from which every
// block derives it (fused scale + cast; block 0 also publishes scale and
// 1/scale).  With `mu` set (the payload of the FP8 gradient all-reduce) the
// scale is *mu * 2^(floor(log2(fmax / amax)) - margin), mu read from device
// memory and applied after the exponent rule, so it does not cancel.
struct CastScale {
  const float *scale;  // used when amax == nullptr
  const float *amax;
  float fmax;
  int margin, log2mu;
  float *scale_out, *inv_out;
  const float *mu;
};

__device__ __forceinline__ float cast_scale(const CastScale &cs) {
  if (cs.amax == nullptr) return *cs.scale;
  int k;
  bool finite;
  if (cs.mu != nullptr) {
    int kg;
    finite = scale_exponent(*cs.amax, cs.fmax, cs.margin, 0, kg);
    k = clamp_exp(kg + device_log2mu(*cs.mu));
  } else {
    finite = scale_exponent(*cs.amax, cs.fmax, cs.margin, cs.log2mu, k);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *cs.scale_out = pow2f(k);
    *cs.inv_out = pow2f(-k);
    if (!finite) atomicOr(&g_status, FP8_STATUS_NONFINITE);
  }
  return pow2f(k);
}

// The same cast with the under/overflow counts of its 16 elements: an
// element underflows when it is a non-zero number whose code is zero, and
// overflows when |x * s| exceeds fmax (inf included, NaN in neither).
template <int DT, int FMT>
__device__ __forceinline__ void cast_group_count(const void *x, size_t g, float s, float fmax, void *q,
                                                 uint32_t &under, uint32_t &over) {
  float f[16];
  load16<DT>(x, g, f);
  uint32_t nz = 0;
#pragma unroll
  for (int j = 0; j < 16; j++) {
    nz |= (f[j] != 0.0f && f[j] == f[j]) ? (1u << j) : 0u;
    f[j] *= s;
    over += fabsf(f[j]) > fmax ? 1u : 0u;
  }
  if constexpr (FMT == FP8_F16S) {
    uint32_t h[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
      h[j] = f16x2(f[2 * j], f[2 * j + 1]);
      under += ((nz >> (2 * j)) & 1u) && (h[j] & 0x7fffu) == 0u;
      under += ((nz >> (2 * j + 1)) & 1u) && (h[j] & 0x7fff0000u) == 0u;
    }
    uint4 *p = reinterpret_cast<uint4 *>(q) + g * 2;
    __stcs(p, make_uint4(h[0], h[1], h[2], h[3]));
    __stcs(p + 1, make_uint4(h[4], h[5], h[6], h[7]));
  } else {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
      w[j] = enc4<FMT>(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
#pragma unroll
      for (int b = 0; b < 4; b++) under += ((nz >> (4 * j + b)) & 1u) && ((w[j] >> (8 * b)) & 0x7fu) == 0u;
    }
    __stcs(reinterpret_cast<uint4 *>(q) + g, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

template <int DT, int FMT, bool COUNT>
__global__ void __launch_bounds__(kStreamThreads) k_cast(const void *__restrict__ x, size_t n,
                                                         const CastScale cs, void *__restrict__ q,
                                                         unsigned long long *__restrict__ counts) {
  const float s = cast_scale(cs);
  const size_t groups = n / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t under = 0, over = 0;
  const float fmax = FMT == FP8_E4M3 ? 448.0f : (FMT == FP8_E5M2 ? 57344.0f : 65504.0f);
  if constexpr (COUNT) {
    for (; g < groups; g += stride) cast_group_count<DT, FMT>(x, g, s, fmax, q, under, over);
  } else {
    for (; g + stride < groups; g += 2 * stride) {
      cast_group<DT, FMT>(x, g, s, q);
      cast_group<DT, FMT>(x, g + stride, s, q);
    }
    if (g < groups) cast_group<DT, FMT>(x, g, s, q);
  }
  if (blockIdx.x == 0) {
    for (size_t i = groups * 16 + threadIdx.x; i < n; i += blockDim.x) {
      const float xi = load1<DT>(x, i);
      const float y = xi * s;
      uint32_t code;
      if constexpr (FMT == FP8_F16S) {
        code = __half_as_ushort(__float2half_rn(y));
        reinterpret_cast<uint16_t *>(q)[i] = (uint16_t)code;
        code &= 0x7fffu;
      } else {
        code = enc2<FMT>(y, 0.0f) & 0xffu;
        reinterpret_cast<uint8_t *>(q)[i] = (uint8_t)code;
        code &= 0x7fu;
      }
      if constexpr (COUNT) {
        under += (xi != 0.0f && xi == xi && code == 0u) ? 1u : 0u;
        over += fabsf(y) > fmax ? 1u : 0u;
      }
    }
  }
  if constexpr (COUNT) {
    __shared__ uint32_t red[64];
    block_add_counts(under, over, red, counts);
  }
}

// ---------------------------------------------------------------------------
// amax and cast in one pass over x.  The cast uses a predicted scale -- the
// tensor's previous one, which per-tensor scales of activations and
// gradients keep from step to step unless the amax crosses a power of two --
// while the pass reduces the tensor's own amax; k_cast_redo then compares
// the scale of that amax with the prediction and, only where they differ,
// casts the tensor again with it (every block takes the same decision and
// returns at once when the prediction held).  k_compute_scale publishes the
// scale last, so no block of the redo reads a half-updated prediction.  The
// codes, amax and scales are those of k_amax followed by the fused
// scale + cast, bit for bit; the tensor is read once instead of twice when
// the prediction holds.
template <int DT, int FMT>
__device__ __forceinline__ uint32_t amax_cast_group(const void *x, size_t g, float s, void *q) {
  float f[16];
  load16<DT>(x, g, f);
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 16; j++) {
    m = max(m, absbits_f32(f[j]));
    f[j] *= s;
  }
  if constexpr (FMT == FP8_F16S) {
    uint4 lo = make_uint4(f16x2(f[0], f[1]), f16x2(f[2], f[3]), f16x2(f[4], f[5]), f16x2(f[6], f[7]));
    uint4 hi = make_uint4(f16x2(f[8], f[9]), f16x2(f[10], f[11]), f16x2(f[12], f[13]), f16x2(f[14], f[15]));
    uint4 *p = reinterpret_cast<uint4 *>(q) + g * 2;
    __stcs(p, lo);
    __stcs(p + 1, hi);
  } else {
    uint4 o = make_uint4(enc4<FMT>(f[0], f[1], f[2], f[3]), enc4<FMT>(f[4], f[5], f[6], f[7]),
                         enc4<FMT>(f[8], f[9], f[10], f[11]), enc4<FMT>(f[12], f[13], f[14], f[15]));
    __stcs(reinterpret_cast<uint4 *>(q) + g, o);
  }
  return m;
}

// One element of the ragged tail, cast as k_cast casts it.
template <int FMT>
__device__ __forceinline__ void cast_one(float y, void *q, size_t i) {
  if constexpr (FMT == FP8_F16S)
    reinterpret_cast<uint16_t *>(q)[i] = __half_as_ushort(__float2half_rn(y));
  else
    reinterpret_cast<uint8_t *>(q)[i] = (uint8_t)(enc2<FMT>(y, 0.0f) & 0xffu);
}

template <int DT, int FMT>
__global__ void __launch_bounds__(kStreamThreads) k_amax_cast(const void *__restrict__ x, size_t n,
                                                              const float *__restrict__ pred,
                                                              float *__restrict__ amax, void *__restrict__ q) {
  __shared__ uint32_t red[32];
  const float s = *pred;
  const size_t groups = n / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m0 = 0, m1 = 0;
  for (; g + stride < groups; g += 2 * stride) {
    m0 = max(m0, amax_cast_group<DT, FMT>(x, g, s, q));
    m1 = max(m1, amax_cast_group<DT, FMT>(x, g + stride, s, q));
  }
  if (g < groups) m0 = max(m0, amax_cast_group<DT, FMT>(x, g, s, q));
  uint32_t m = max(m0, m1);
  if (blockIdx.x == 0) {  // ragged tail (< 16 elements)
    for (size_t i = groups * 16 + threadIdx.x; i < n; i += blockDim.x) {
      const float xi = load1<DT>(x, i);
      m = max(m, absbits_f32(xi));
      cast_one<FMT>(xi * s, q, i);
    }
  }
  m = block_max_u32(m, red);
  if (threadIdx.x == 0) atomic_max_bits(amax, m);
}

template <int DT, int FMT>
__global__ void __launch_bounds__(kStreamThreads) k_cast_redo(const void *__restrict__ x, size_t n,
                                                              const float *__restrict__ pred,
                                                              const float *__restrict__ amax, float fmax,
                                                              int margin, int log2mu, void *__restrict__ q) {
  int k;
  scale_exponent(*amax, fmax, margin, log2mu, k);
  const float s = pow2f(k);
  if (s == *pred) return;  // the same for every block: the pass already cast with s
  const size_t groups = n / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride)
    cast_group<DT, FMT>(x, g, s, q);
  if (blockIdx.x == 0)
    for (size_t i = groups * 16 + threadIdx.x; i < n; i += blockDim.x) cast_one<FMT>(load1<DT>(x, i) * s, q, i);
}

// Self-test of enc2 against enc2_checked on the binary32 values with bit
// patterns in [lo, hi), each in the low lane (the other 0) and in the high
// lane (the other 0): counts the values whose codes differ and keeps the
// smallest such pattern.
template <int FMT>
__global__ void k_encode_selftest(uint32_t lo, unsigned long long hi, unsigned long long *bad, uint32_t *first) {
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  unsigned long long nbad = 0;
  uint32_t lowest = 0xffffffffu;
  for (unsigned long long u = lo + (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; u < hi;
       u += stride) {
    const float x = __uint_as_float((uint32_t)u);
    if (enc2<FMT>(x, 0.0f) != enc2_checked<FMT>(x, 0.0f) || enc2<FMT>(0.0f, x) != enc2_checked<FMT>(0.0f, x)) {
      nbad++;
      lowest = min(lowest, (uint32_t)u);
    }
  }
  if (nbad) {
    atomicAdd(bad, nbad);
    atomicMin(first, lowest);
  }
}

}  // namespace fp8lib
