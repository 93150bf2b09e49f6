// allreduce.cuh -- the local half of the FP8 gradient all-reduce and the
// auto-scaling rule for mu.
//
// "FP8-LM: Training FP8 Large Language Models", 提案手法 O1: gradients are
// communicated in FP8, auto-scaled by mu (Eq. 3) so that the sum over ranks
// neither overflows nor underflows; アブレーション研究: the variants are
// compared by their underflow and overflow rates.
//
// Every rank's payload was cast with one shared scale, so the codes of the
// ranks can be added as they are.  Each FP8 value is an integer multiple of
// the format's smallest subnormal (2^-16 for E5M2, 2^-9 for E4M3), so the sum
// can be formed exactly and rounded once: to binary32 with round-to-odd (24
// bits >= the 3- or 4-bit significand + 2, so the following
// round-to-nearest-even is correct), then by the saturating cvt.  Two exact
// summations: split binary32 accumulators (k_sum_codes_fast, the usual path)
// and integer unit counts (k_sum_codes, E5M2 beyond 128 ranks).
#pragma once

#include "common.cuh"

namespace fp8lib {

constexpr int kSumThreads = 256;
constexpr int kSumMaxRanks = 4096;

enum : uint32_t { SPECIAL_NAN = 1u, SPECIAL_PINF = 2u, SPECIAL_NINF = 4u };

template <int FMT>
struct SumTraits {
  // accumulator: E5M2 values reach 7 * 2^29 units, E4M3 values 15 * 2^14
  using Acc = typename std::conditional<FMT == FP8_E5M2, long long, int>::type;
  static constexpr int kMantBits = FMT == FP8_E5M2 ? 2 : 3;
  static constexpr int kUnitExp = FMT == FP8_E5M2 ? -16 : -9;
  static constexpr long long kMaxUnits = FMT == FP8_E5M2 ? 3758096384LL : 229376LL;  // fmax / unit
};

// A code as a signed count of smallest-subnormal units; specials set flags.
template <int FMT>
__device__ __forceinline__ typename SumTraits<FMT>::Acc code_units(uint32_t c, uint32_t &special) {
  using T = SumTraits<FMT>;
  using Acc = typename T::Acc;
  constexpr int MB = T::kMantBits;
  const uint32_t e = (c >> MB) & (FMT == FP8_E5M2 ? 31u : 15u);
  const uint32_t m = c & ((1u << MB) - 1u);
  if constexpr (FMT == FP8_E5M2) {
    if (e == 31u) {
      special |= m ? SPECIAL_NAN : ((c & 0x80u) ? SPECIAL_NINF : SPECIAL_PINF);
      return 0;
    }
  } else {
    if (e == 15u && m == 7u) {
      special |= SPECIAL_NAN;
      return 0;
    }
  }
  const Acc mag = e ? (Acc)((1u << MB) | m) << (e - 1u) : (Acc)m;
  return (c & 0x80u) ? -mag : mag;
}

// Exact unit count -> binary32 by round-to-odd.
__device__ __forceinline__ float units_to_float_rto(long long s) {
  float f = __ll2float_rz(s);
  if ((long long)f != s) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}
__device__ __forceinline__ float units_to_float_rto(int s) {
  float f = __int2float_rz(s);
  if ((int)f != s) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}

// Encode one exact sum; adds to the under/overflow counts.
template <int FMT>
__device__ __forceinline__ uint32_t encode_sum(typename SumTraits<FMT>::Acc s, uint32_t special,
                                               uint32_t &under, uint32_t &over) {
  using T = SumTraits<FMT>;
  if (special) {
    if ((special & SPECIAL_NAN) || (special & (SPECIAL_PINF | SPECIAL_NINF)) == (SPECIAL_PINF | SPECIAL_NINF))
      return 0x7Fu;
    over++;
    return (special & SPECIAL_NINF) ? (0x80u | top_code(FMT)) : top_code(FMT);
  }
  const float y = units_to_float_rto(s) * (FMT == FP8_E5M2 ? 0x1p-16f : 0x1p-9f);
  const uint32_t c = enc2<FMT>(y, 0.0f) & 0xffu;
  const long long a = s < 0 ? -(long long)s : (long long)s;
  over += a > T::kMaxUnits ? 1u : 0u;
  under += (s != 0 && (c & 0x7fu) == 0u) ? 1u : 0u;
  return c;
}

// out[i] = enc(sum_r dec(in[r * ld + i])) for i < n.  16 elements per thread
// step: one 16-byte load per rank row, one 16-byte store.
template <int FMT>
__global__ void __launch_bounds__(kSumThreads)
    k_sum_codes(const uint8_t *__restrict__ in, int nranks, size_t ld, size_t n, uint8_t *__restrict__ out,
                const float *__restrict__ inv_scale, float *__restrict__ g_inv,
                unsigned long long *__restrict__ counts) {
  using Acc = typename SumTraits<FMT>::Acc;
  const size_t groups = n / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  uint32_t under = 0, over = 0;
  for (size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
    Acc acc[16];
    uint32_t special[16];
#pragma unroll
    for (int j = 0; j < 16; j++) {
      acc[j] = 0;
      special[j] = 0;
    }
    for (int r = 0; r < nranks; r++) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(in + (size_t)r * ld) + g);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 16; j++) acc[j] += code_units<FMT>((w[j >> 2] >> (8 * (j & 3))) & 0xffu, special[j]);
    }
    uint32_t o[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; j++) o[j >> 2] |= encode_sum<FMT>(acc[j], special[j], under, over) << (8 * (j & 3));
    __stcs(reinterpret_cast<uint4 *>(out) + g, make_uint4(o[0], o[1], o[2], o[3]));
  }
  if (blockIdx.x == 0) {
    for (size_t i = groups * 16 + threadIdx.x; i < n; i += blockDim.x) {
      Acc acc = 0;
      uint32_t special = 0;
      for (int r = 0; r < nranks; r++) acc += code_units<FMT>(in[(size_t)r * ld + i], special);
      out[i] = (uint8_t)encode_sum<FMT>(acc, special, under, over);
    }
    if (threadIdx.x == 0 && g_inv != nullptr) *g_inv = __fmul_rn(*inv_scale, 1.0f / (float)nranks);
  }
  if (counts != nullptr) {
    __shared__ uint32_t red[64];
    block_add_counts(under, over, red, counts);
  }
}

// Faster exact sum for up to kSumFastMaxRanks ranks (E5M2; E4M3 up to
// kSumMaxRanks).  The codes are decoded by the hardware cvt (fp8x2 -> f16x2,
// exact) and each value x is split as x = t + (x - t), t = x rounded to a
// multiple of 1/2 by adding and subtracting 1.5 * 2^22 (whose binary32 ULP is
// 1/2; |x| <= 57344 keeps x + 1.5 * 2^22 in that binade).  The t are
// multiples of 1/2 below 57344 and the x - t multiples of the smallest
// subnormal (2^-16 E5M2, 2^-9 E4M3) of magnitude at most 1/4, so for up to 128
// E5M2 or 4096 E4M3 ranks neither running sum needs more than 24 significant
// bits: both are exact, and the split costs packed adds only (no compare,
// no select).  Their sum is formed in binary64 (exact), rounded to binary32
// by round-to-odd and then by the saturating cvt.  An inf or NaN code makes
// t, and so the t-sum, non-finite (the other sum then holds a NaN): a NaN
// t-sum (a NaN code, or +inf with -inf) encodes as 0x7F, an infinite one
// saturates and counts as an overflow, as in the integer path.
constexpr int kSumFastMaxRanks = 128;
constexpr float kSplitC = 0x1.8p22f;  // 1.5 * 2^22: binary32 ULP 1/2

template <int FMT>
__device__ __forceinline__ uint32_t encode_split_sum(float hi, float lo, float fmax, uint32_t &under,
                                                     uint32_t &over) {
  if (!(fabsf(hi) <= 3.402823466e38f)) {  // an inf or NaN code was summed
    if (hi != hi) return 0x7Fu;
    over++;
    return hi > 0.0f ? top_code(FMT) : (0x80u | top_code(FMT));
  }
  const double d = (double)hi + (double)lo;
  float f = __double2float_rz(d);
  if ((double)f != d) f = __uint_as_float(__float_as_uint(f) | 1u);
  const uint32_t c = enc2<FMT>(f, 0.0f) & 0xffu;
  over += fabs(d) > (double)fmax ? 1u : 0u;
  under += (d != 0.0 && (c & 0x7fu) == 0u) ? 1u : 0u;
  return c;
}

template <int FMT>
__global__ void __launch_bounds__(kSumThreads)
    k_sum_codes_fast(const uint8_t *__restrict__ in, int nranks, size_t ld, size_t n, uint8_t *__restrict__ out,
                     const float *__restrict__ inv_scale, float *__restrict__ g_inv,
                     unsigned long long *__restrict__ counts) {
  const float fmax = FMT == FP8_E5M2 ? 57344.0f : 448.0f;
  const size_t groups = n / 16;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  uint32_t under = 0, over = 0;
  const float2 c = both(kSplitC), neg_c = both(-kSplitC), minus1 = both(-1.0f);
  for (size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
    float2 hi[8], lo[8];  // pairs of elements
#pragma unroll
    for (int p = 0; p < 8; p++) hi[p] = lo[p] = both(0.0f);
    for (int r = 0; r < nranks; r++) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(in + (size_t)r * ld) + g);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int p = 0; p < 8; p++) {
        const float2 x = dec2<FMT>(w[p >> 1] >> ((p & 1) * 16));
        const float2 t = __fadd2_rn(__fadd2_rn(x, c), neg_c);  // x to a multiple of 1/2
        hi[p] = __fadd2_rn(hi[p], t);
        lo[p] = __fadd2_rn(lo[p], __ffma2_rn(t, minus1, x));   // x - t, exact
      }
    }
    uint32_t o[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const float h = (j & 1) ? hi[j >> 1].y : hi[j >> 1].x, l = (j & 1) ? lo[j >> 1].y : lo[j >> 1].x;
      o[j >> 2] |= encode_split_sum<FMT>(h, l, fmax, under, over) << (8 * (j & 3));
    }
    __stcs(reinterpret_cast<uint4 *>(out) + g, make_uint4(o[0], o[1], o[2], o[3]));
  }
  if (blockIdx.x == 0) {
    for (size_t i = groups * 16 + threadIdx.x; i < n; i += blockDim.x) {
      float hi = 0.0f, lo = 0.0f;
      for (int r = 0; r < nranks; r++) {
        const float x = dec2<FMT>(in[(size_t)r * ld + i]).x;
        const float t = __fadd_rn(__fadd_rn(x, kSplitC), -kSplitC);
        hi = __fadd_rn(hi, t);
        lo = __fadd_rn(lo, __fmaf_rn(t, -1.0f, x));
      }
      out[i] = (uint8_t)encode_split_sum<FMT>(hi, lo, fmax, under, over);
    }
    if (threadIdx.x == 0 && g_inv != nullptr) *g_inv = __fmul_rn(*inv_scale, 1.0f / (float)nranks);
  }
  if (counts != nullptr) {
    __shared__ uint32_t red[64];
    block_add_counts(under, over, red, counts);
  }
}

// The mu rule (one thread): more than theta * n overflows halve mu (not below
// mu_min) and restart the clean-step count; otherwise the count grows and
// after `interval` clean steps mu doubles (not above mu_max).  Both counts
// are then cleared for the next step.
__global__ void k_mu_update(float *__restrict__ mu, int *__restrict__ clean,
                            unsigned long long *__restrict__ counts, unsigned long long n, double theta,
                            int interval, float mu_min, float mu_max) {
  const unsigned long long overflows = counts[1];
  float m = *mu;
  if ((double)overflows > theta * (double)n) {
    m = fmaxf(m * 0.5f, mu_min);
    *clean = 0;
  } else {
    int c = *clean + 1;
    if (c >= interval) {
      m = fminf(m * 2.0f, mu_max);
      c = 0;
    }
    *clean = c;
  }
  *mu = m;
  counts[0] = 0;
  counts[1] = 0;
}

}  // namespace fp8lib
