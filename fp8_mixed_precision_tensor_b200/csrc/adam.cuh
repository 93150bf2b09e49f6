// adam.cuh -- precision-decoupled FP8 Adam ("FP8-LM: Training FP8 Large
// Language Models", 提案手法 O2): FP8 E5M2 gradient, FP8 E4M3 first moment,
// FP16 second moment and FP16 master weights, every tensor with its own
// power-of-two scale (6 bytes of state per parameter).
//
// The new scales are just-in-time: each comes from the amax of the *new*
// values (the same rule as the linear layer's casts).  A step is
//   pass 1 (stats):   decode, update in registers, reduce per chunk amax|m|,
//                     amax v (both exact), the largest step U >= max |dw|
//                     and, reading the master, an estimate A~ of the new
//                     master's amax (|A~ - A| <= 2^-16 U + 2^-21 A~), or, when
//                     the caller tracks the stored master's amax A0, U alone
//                     (not reading the master: 4 instead of 6 B); the step is
//                     estimated with the MUFU square root and reciprocal;
//   finalize 1:       new scales of m and v; the new master amax lies in
//                     [A~ - e, A~ + e] or, tracked, in [A0 - U, A0 + U], and
//                     the master's scale exponent is taken from that interval
//                     when it contains no scale threshold, otherwise the chunk
//                     is flagged;
//   pass 1b:          exact amax|w| for flagged chunks only (others skip);
//   finalize 2:       remaining scales; publish all new scales;
//   pass 2 (update):  decode, update again (bit-identical arithmetic), encode
//                     m, v, w with the new scales, optionally write the E4M3
//                     copy of the new stored master for the next forward GEMM,
//                     and reduce the stored master's amax;
//   finalize 3:       new tracked A0; every chunk's master scale checked
//                     against the exact new amax the update pass reduced.
// The phased form of the step (stats and update as separate calls, with the
// workspace MAX-reduced over ranks in between) computes the exact new amaxes
// in pass 1 instead: an interval decision there would need a second
// reduction for the flagged chunks.
// The out-of-place step (new state into separate buffers, the inputs left
// as they were) needs no stats pass: it predicts that every new scale equals
// the old one and
//   pass 6 (update):  decodes, updates and encodes with the predicted scales
//                     into the new buffers while reducing the exact amax|m|,
//                     amax v and amax|w| of the new values;
//   finalize 6:       the scales those amaxes give; a chunk whose prediction
//                     was wrong is flagged;
//   pass 7 (redo):    the update again, flagged chunks only, from the
//                     unchanged inputs with the right scales;
//   finalize 7:       tracked amax of the redone chunks.
// One pass of 6 B read and 5-6 B written per parameter when the scales hold,
// the same results as the in-place step in every case.
// Passes 8 and 9 are passes 6 and 7 reading the gradient as the wgrad left
// it, bfloat16, and casting it to E5M2 in registers with the scale of its
// amax (the codes the separate gradient cast would store), so the E5M2
// gradient is never written or read back.
// All chunks of one call share each launch: the chunk table travels in the
// kernel parameters and tiles of 4096 parameters are mapped to chunks by a
// binary search over the chunks' first-tile indices.
#pragma once

#include "common.cuh"

namespace fp8lib {

constexpr int kAdamThreads = 256;
constexpr int kAdamPerThread = 16;
constexpr int kAdamTile = kAdamThreads * kAdamPerThread;  // parameters per tile
// the chunk table travels in the kernel parameters (at most 32,764 bytes)
constexpr int kAdamMaxChunksPerLaunch = 224;
constexpr int kAdamWsFloatsPerChunk = 16;  // workspace slots per chunk (64 bytes)

// Workspace slots of one chunk (float bits; amax slots are max-reduced as
// unsigned bit patterns).
enum : int {
  WS_AMAX_M = 0, WS_AMAX_V = 1, WS_AMAX_W = 2,
  WS_OLDINV_M = 3, WS_OLDINV_V = 4, WS_OLDINV_W = 5,
  WS_NEW_M = 6, WS_NEW_V = 7, WS_NEW_W = 8,
  WS_STEP_MAX = 9,     // max |dw| of the update (tracked-master path)
  WS_FLAGS = 10,       // bit 0: needs the exact master pass; bit 1: tracked path
  WS_NEW_WQ = 11,      // scale of the E4M3 master copy
  WS_STORED_W = 12,    // max |stored FP16 master| (as f32 bits of the half)
  WS_CHECK_W = 13,     // exact amax|w| of the new f32 master (pass 2)
  WS_APPROX_W = 14,    // estimate of amax|w| of the new master (pass 1, estimated step)
};
// WS_FLAGS bits: the exact master pass must run; the chunk tracks its master
// amax; the master's scale was decided in finalize 1; the out-of-place
// step's predicted scales were wrong and the chunk is updated again.
enum : uint32_t { FLAG_EXACT = 1u, FLAG_TRACKED = 2u, FLAG_KNOWN = 4u, FLAG_REDO = 8u };

struct AdamChunkDev {
  const uint8_t *g;
  const float *g_inv;
  uint8_t *m;
  float *m_scale;
  uint16_t *v;
  float *v_scale;
  uint16_t *w;
  float *w_scale;
  float *w_amax;  // optional tracked amax of the stored master
  uint8_t *wq;    // optional E4M3 copy of the new master
  float *wq_scale, *wq_inv;
  uint8_t *m_out;    // where the update writes the new state: m, v, w
  uint16_t *v_out;   // themselves (in place) or the out-of-place step's
  uint16_t *w_out;   // new buffers
  const float *g_amax;  // passes 8, 9: amax of the bfloat16 gradient at g
  unsigned long long n;
  unsigned long long tile_begin;
};

struct AdamLaunch {
  AdamChunkDev c[kAdamMaxChunksPerLaunch];
  int nchunks;
  int margin;
  unsigned long long total_tiles;
  float beta1, beta2, eps;
  float neg_lr_bc1;  // -lr / (1 - beta1^t)
  float inv_bc2;     // 1 / (1 - beta2^t)
  int estimate;      // 1: untracked chunks take the estimated stats pass (PASS 5)
  int g_hp;          // passes 8, 9: the gradient is bfloat16, cast to E5M2 in the pass
  int g_margin, g_log2mu;  // its scale rule: margin and log2(mu)
  float *ws;         // kAdamWsFloatsPerChunk floats per chunk of this launch
};
static_assert(sizeof(AdamLaunch) <= 32764, "kernel parameters are limited to 32,764 bytes");

// Per-chunk constants of the update: the descales are folded into the Adam
// coefficients, m = (b1/s_m) m~ + ((1-b1)/(mu s_g)) g~ and
// v = (b2/s_v) v~ + ((1-b2)/(mu s_g)) g~ * (1/(mu s_g)) g~, where ~ marks a
// decoded code.  The gradient descale enters v once per factor, never
// squared: (1-b2)/(mu s_g)^2 underflows binary32 once the gradient's amax is
// below ~1e-17 (mu s_g above 2^72), while each factor stays a normal number
// and only the product, the new v itself, can be subnormal.
// Every factor is held in both lanes of a float2: parameters are updated in
// pairs with the packed binary32 instructions of sm_100 (two independent
// round-to-nearest operations per instruction, the same results as the
// scalar ones at half the issue slots).
struct AdamScalars {
  float2 cm, cgm;  // b1 / s_m,  (1 - b1) g_inv
  float2 cv, cgv;  // b2 / s_v,  (1 - b2) g_inv
  float2 g_inv;    // 1 / (mu s_g)
  float2 w_inv;    // 1 / s_w
};

__device__ __forceinline__ AdamScalars adam_scalars(const AdamLaunch &L, float g_inv, float m_inv,
                                                    float v_inv, float w_inv) {
  AdamScalars s;
  s.cm = both(__fmul_rn(L.beta1, m_inv));
  s.cgm = both(__fmul_rn(__fsub_rn(1.0f, L.beta1), g_inv));
  s.cv = both(__fmul_rn(L.beta2, v_inv));
  s.cgv = both(__fmul_rn(__fsub_rn(1.0f, L.beta2), g_inv));
  s.g_inv = both(g_inv);
  s.w_inv = both(w_inv);
  return s;
}

// MUFU approximations (flush-to-zero) of the square root and the reciprocal.
__device__ __forceinline__ float sqrt_approx(float x) {
  float r;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// The reciprocal rounded to nearest for the arguments the step gives it,
// 2^-39 <= b <= 2^66 (the range of sqrt(v_hat) + eps) and +inf: the MUFU
// approximation y and one Newton-Raphson correction y + y*e whose residual
// e = 1 - b*y is formed in a fused multiply-add (P. Markstein, "Computation
// of elementary functions on the IBM RISC System/6000 processor", IBM J.
// Res. Develop. 34(1), 1990), without a branch; +inf is selected.  Bit for
// bit CUDA's __frcp_rn on every binary32 argument of that range
// (fp8_selftest_step_reciprocal checks all of them) and cheaper in the
// update pass: 10 % at full clock, 15-20 % of the Adam step's time at the
// power-capped clock of a training step.  (The same construction for the
// square root needs a scaled residual and a final Tuckerman test to be
// correctly rounded everywhere, and was slower than __fsqrt_rn.)
__device__ __forceinline__ float rcp_rn_step(float b) {
  const float y = rcp_approx(b);
  const float e = __fmaf_rn(-b, y, 1.0f);
  const float r = __fmaf_rn(e, y, y);
  return b == __int_as_float(0x7f800000) ? 0.0f : r;
}

// The new moments and the master step dw = -lr m_hat / (sqrt(v_hat) + eps)
// of two parameters, binary32, from decoded codes.  Every operation rounds to
// nearest (the square root CUDA's correctly rounded __fsqrt_rn, subnormals
// kept; the reciprocal correctly rounded by rcp_rn_step; the quotient is m
// times that reciprocal, two roundings, 3 % faster in the update pass than a
// correctly rounded division; 2^-39 <= eps <= 2^64 keeps the reciprocal a
// normal number), so the step's
// error is a fixed number of binary32 roundings:
// |dw - dw_exact| <= 24 * 2^-24 * dw_abs, where
// dw_abs is the step with |m| replaced by b1 |m0| + (1 - b1) |g| (which also
// covers the cancellation of m's two terms), counting the hyper-parameters'
// own binary32 representation.  Explicit round-to-nearest operations keep
// every pass (and the element-wise tail, which runs the same function with
// one lane unused) on exactly the same arithmetic.
__device__ __forceinline__ void adam_moments(const AdamLaunch &L, float2 gd, float2 md, float2 vd,
                                             const AdamScalars &s, float2 &m, float2 &v, float2 &dw) {
  m = __ffma2_rn(s.cm, md, __fmul2_rn(s.cgm, gd));
  v = __ffma2_rn(s.cv, vd, __fmul2_rn(__fmul2_rn(s.cgv, gd), __fmul2_rn(s.g_inv, gd)));
  const float2 vh = __fmul2_rn(v, both(L.inv_bc2));
  const float2 den = __fadd2_rn(make_float2(__fsqrt_rn(vh.x), __fsqrt_rn(vh.y)), both(L.eps));
  dw = __fmul2_rn(both(L.neg_lr_bc1), __fmul2_rn(m, make_float2(rcp_rn_step(den.x), rcp_rn_step(den.y))));
}

// The same moments and an estimate of the step, with the MUFU square root and
// reciprocal (flush-to-zero) in place of the correctly rounded operations:
// for the stats passes, which need the exact m and v (computed the same way
// here) but only an interval for the master's new amax.  The approximations'
// relative errors (a few 2^-23, so |dw~ - dw| < 2^-18 |dw|) are covered by
// the 2^-16 U widening in the finalize stage; the flush changes nothing
// because eps >= 2^-39 makes sqrt(v_hat) + eps round to eps for every
// subnormal v_hat.  The update pass checks every scale decided this way
// against the exact new amax.
__device__ __forceinline__ void adam_moments_bound(const AdamLaunch &L, float2 gd, float2 md, float2 vd,
                                                   const AdamScalars &s, float2 &m, float2 &v, float2 &dw) {
  m = __ffma2_rn(s.cm, md, __fmul2_rn(s.cgm, gd));
  v = __ffma2_rn(s.cv, vd, __fmul2_rn(__fmul2_rn(s.cgv, gd), __fmul2_rn(s.g_inv, gd)));
  const float2 vh = __fmul2_rn(v, both(L.inv_bc2));
  const float2 den = __fadd2_rn(make_float2(sqrt_approx(vh.x), sqrt_approx(vh.y)), both(L.eps));
  dw = __fmul2_rn(both(L.neg_lr_bc1), __fmul2_rn(m, make_float2(rcp_approx(den.x), rcp_approx(den.y))));
}
constexpr float kStepBoundWiden = 1.0f + 0x1p-16f;

// w = w0 + dw as one rounding per parameter (the master's new value).
__device__ __forceinline__ float2 adam_master(float2 wd, float2 dw, const AdamScalars &s) {
  return __fadd2_rn(__fmul2_rn(wd, s.w_inv), dw);
}

// Running maxima of magnitudes as floats, NaN-propagating: a NaN anywhere
// leaves the canonical NaN 0x7FFFFFFF, whose bits order above inf, so the
// finalize stage sees it as a non-finite amax.  acc is >= +0 or that NaN.
__device__ __forceinline__ float max_abs2(float acc, float2 x) {
  float r;
  asm("{\n\t.reg .f32 t0, t1;\n\tabs.f32 t0, %2;\n\tabs.f32 t1, %3;\n\t"
      "max.NaN.f32 %0, %1, t0, t1;\n\t}"
      : "=f"(r) : "f"(acc), "f"(x.x), "f"(x.y));
  return r;
}
__device__ __forceinline__ float max_abs1(float acc, float x) {
  float r;
  asm("{\n\t.reg .f32 t0;\n\tabs.f32 t0, %2;\n\tmax.NaN.f32 %0, %1, t0;\n\t}" : "=f"(r) : "f"(acc), "f"(x));
  return r;
}

__device__ __forceinline__ int find_chunk(const AdamLaunch &L, unsigned long long tile) {
  int lo = 0, hi = L.nchunks - 1;  // last chunk whose tile_begin <= tile
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (L.c[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float ws_get(const AdamLaunch &L, int ci, int slot) {
  return L.ws[ci * kAdamWsFloatsPerChunk + slot];
}
__device__ __forceinline__ uint32_t ws_flags(const AdamLaunch &L, int ci) {
  return __float_as_uint(L.ws[ci * kAdamWsFloatsPerChunk + WS_FLAGS]);
}

// Warp-reduce three running maxima and fold them into a chunk's slots.
__device__ __forceinline__ void flush_max3(const AdamLaunch &L, int ci, int s0, float m0, int s1, float m1,
                                           int s2, float m2) {
  const uint32_t a0 = warp_max_u32(__float_as_uint(m0));
  const uint32_t a1 = warp_max_u32(__float_as_uint(m1));
  const uint32_t a2 = warp_max_u32(__float_as_uint(m2));
  if ((threadIdx.x & 31) == 0) {
    float *ws = L.ws + ci * kAdamWsFloatsPerChunk;
    atomic_max_bits(ws + s0, a0);
    atomic_max_bits(ws + s1, a1);
    atomic_max_bits(ws + s2, a2);
  }
}

// Per-chunk values of the update pass.
struct AdamNewScales {
  float2 m, v, w;  // new scales of m, v, w
  float2 q;        // s_q / s_w: stored master -> its E4M3 copy (powers of two, ~2^-7)
};

// Passes 8 and 9 run the code of passes 6 and 7 with the gradient cast in
// the pass: the pass number the rest of the code branches on, and the flag.
template <int PASS>
__host__ __device__ constexpr int base_pass() { return PASS >= 8 ? PASS - 2 : PASS; }
template <int PASS>
__host__ __device__ constexpr bool cast_grad_pass() { return PASS >= 8; }

// The gradient's E5M2 scale exponent from its amax (the rule of the fused
// scale + cast, fmt_max 57344); false for a non-finite amax (then 2^log2mu).
__device__ __forceinline__ bool grad_scale_exponent(const AdamLaunch &L, const AdamChunkDev &C, int &k) {
  return scale_exponent(*C.g_amax, 57344.0f, L.g_margin, L.g_log2mu, k);
}

// One thread's full group of 16 parameters: 16 B of g, 16 B of m, 32 B of v,
// 32 B of w.  Whether the chunk tracks its master amax and whether the E4M3
// copy is written are per chunk: the stats passes take them as template
// arguments (no per-parameter test in the element loop); the update pass,
// whose extra live values would cost a resident block per SM as separate
// instantiations, takes them at run time (TRACK = WQ = true, track_rt and
// wq_rt the chunk's flags).  The update passes (2 in place; 6 and 7 out of
// place, which also reduce the exact amaxes of the new m and v) write the
// new state through m_out, v_out, w_out.
template <int PASS_, bool TRACK, bool WQ>
__device__ __forceinline__ void adam_group(const AdamLaunch &L, const AdamChunkDev &C, size_t grp,
                                           const AdamScalars &sc, const AdamNewScales &ns, float &am, float &av,
                                           float &aw, float &au, bool track_rt = TRACK, bool wq_rt = WQ,
                                           float2 sg = make_float2(1.0f, 1.0f)) {
  constexpr int PASS = base_pass<PASS_>();
  constexpr bool kCastG = cast_grad_pass<PASS_>();
  constexpr bool kReadW = PASS != 1 || !TRACK;
  const bool track = TRACK && track_rt, wq = WQ && wq_rt;
  uint4 gq, gh1 = make_uint4(0, 0, 0, 0);  // E5M2 codes, or the first and second 8 bfloat16
  if constexpr (kCastG) {
    gq = __ldcs(reinterpret_cast<const uint4 *>(C.g) + 2 * grp);
    gh1 = __ldcs(reinterpret_cast<const uint4 *>(C.g) + 2 * grp + 1);
  } else {
    gq = __ldcs(reinterpret_cast<const uint4 *>(C.g) + grp);
  }
  const uint4 mq = __ldcs(reinterpret_cast<const uint4 *>(C.m) + grp);
  const uint4 vq0 = __ldcs(reinterpret_cast<const uint4 *>(C.v) + 2 * grp);
  const uint4 vq1 = __ldcs(reinterpret_cast<const uint4 *>(C.v) + 2 * grp + 1);
  uint4 wq0 = make_uint4(0, 0, 0, 0), wq1 = make_uint4(0, 0, 0, 0);
  if constexpr (kReadW) {
    wq0 = __ldcs(reinterpret_cast<const uint4 *>(C.w) + 2 * grp);
    wq1 = __ldcs(reinterpret_cast<const uint4 *>(C.w) + 2 * grp + 1);
  }
  const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
  const uint32_t gb[4] = {gh1.x, gh1.y, gh1.z, gh1.w};
  const uint32_t mw[4] = {mq.x, mq.y, mq.z, mq.w};
  const uint32_t vw[8] = {vq0.x, vq0.y, vq0.z, vq0.w, vq1.x, vq1.y, vq1.z, vq1.w};
  const uint32_t ww[8] = {wq0.x, wq0.y, wq0.z, wq0.w, wq1.x, wq1.y, wq1.z, wq1.w};
  uint32_t mo[4], vo[8], wo[8], qo[4];
#pragma unroll
  for (int p = 0; p < 8; p++) {  // pairs of parameters
    uint32_t g2;
    if constexpr (kCastG) {  // the gradient cast: bfloat16 pair p, times its scale, to E5M2
      const uint32_t b2 = p < 4 ? gw[p] : gb[p - 4];
      const float2 y = __fmul2_rn(make_float2(__uint_as_float(b2 << 16), __uint_as_float(b2 & 0xffff0000u)), sg);
      g2 = enc2<FP8_E5M2>(y.x, y.y);
    } else {
      g2 = (gw[p >> 1] >> ((p & 1) * 16)) & 0xffffu;
    }
    const uint32_t m2 = (mw[p >> 1] >> ((p & 1) * 16)) & 0xffffu;
    float2 m, v, d;
    if constexpr ((PASS == 1 && TRACK) || PASS == 5)  // the step is only estimated
      adam_moments_bound(L, dec2<FP8_E5M2>(g2), dec2<FP8_E4M3>(m2), h2f2(vw[p]), sc, m, v, d);
    else
      adam_moments(L, dec2<FP8_E5M2>(g2), dec2<FP8_E4M3>(m2), h2f2(vw[p]), sc, m, v, d);
    if constexpr (PASS == 5) {
      am = max_abs2(am, m);
      av = max_abs2(av, v);
      aw = max_abs2(aw, adam_master(h2f2(ww[p]), d, sc));
      au = max_abs2(au, d);
    } else if constexpr (PASS == 1) {
      am = max_abs2(am, m);
      av = max_abs2(av, v);
      aw = max_abs2(aw, TRACK ? d : adam_master(h2f2(ww[p]), d, sc));
    } else if constexpr (PASS == 3) {
      aw = max_abs2(aw, adam_master(h2f2(ww[p]), d, sc));
    } else {
      const float2 w = adam_master(h2f2(ww[p]), d, sc);
      aw = max_abs2(aw, w);  // the exact new amax: checks the decided or the predicted scale
      if constexpr (PASS != 2) {
        am = max_abs2(am, m);
        av = max_abs2(av, v);
      }
      const float2 ms = __fmul2_rn(m, ns.m), vs = __fmul2_rn(v, ns.v), ws = __fmul2_rn(w, ns.w);
      const uint32_t mc = enc2<FP8_E4M3>(ms.x, ms.y);
      if (p & 1) mo[p >> 1] |= mc << 16; else mo[p >> 1] = mc;
      vo[p] = f16x2(vs.x, vs.y);
      wo[p] = f16x2(ws.x, ws.y);
      if (track || wq) {
        const float2 st = h2f2(wo[p]);  // the stored master (scaled)
        if (track) {
          if constexpr (PASS == 2) am = max_abs2(am, st); else au = max_abs2(au, st);
        }
        if (wq) {
          // E4M3 copy of the stored master: h * (s_q / s_w), exact in f32
          const float2 qs = __fmul2_rn(st, ns.q);
          const uint32_t qc = enc2<FP8_E4M3>(qs.x, qs.y);
          if (p & 1) qo[p >> 1] |= qc << 16; else qo[p >> 1] = qc;
        }
      }
    }
  }
  if constexpr (PASS == 2 || PASS == 6 || PASS == 7) {
    __stcs(reinterpret_cast<uint4 *>(C.m_out) + grp, make_uint4(mo[0], mo[1], mo[2], mo[3]));
    __stcs(reinterpret_cast<uint4 *>(C.v_out) + 2 * grp, make_uint4(vo[0], vo[1], vo[2], vo[3]));
    __stcs(reinterpret_cast<uint4 *>(C.v_out) + 2 * grp + 1, make_uint4(vo[4], vo[5], vo[6], vo[7]));
    __stcs(reinterpret_cast<uint4 *>(C.w_out) + 2 * grp, make_uint4(wo[0], wo[1], wo[2], wo[3]));
    __stcs(reinterpret_cast<uint4 *>(C.w_out) + 2 * grp + 1, make_uint4(wo[4], wo[5], wo[6], wo[7]));
    if (wq) __stcs(reinterpret_cast<uint4 *>(C.wq) + grp, make_uint4(qo[0], qo[1], qo[2], qo[3]));
  }
}

// Per-chunk state of a pass: what a block sets up when its tile walk enters a
// new chunk, and the running maxima it folds into the chunk's workspace slots
// when it leaves.
struct AdamChunkState {
  float am = 0.f, av = 0.f, aw = 0.f, au = 0.f;  // running maxima of the current chunk
  int cur = -1;
  bool tracked = false, active = true, want_wq = false;
  AdamScalars sc{};
  AdamNewScales ns{both(1.f), both(1.f), both(1.f), both(1.f)};
  float sg = 1.0f;  // passes 8, 9: the E5M2 scale of the bfloat16 gradient
};

template <int PASS_>
__device__ __forceinline__ void adam_chunk_flush(const AdamLaunch &L, AdamChunkState &S) {
  constexpr int PASS = base_pass<PASS_>();
  constexpr bool kStats = PASS == 1 || PASS == 4;
  if constexpr (kStats)
    if (S.active) flush_max3(L, S.cur, WS_AMAX_M, S.am, WS_AMAX_V, S.av, S.tracked ? WS_STEP_MAX : WS_AMAX_W, S.aw);
  if constexpr (PASS == 5)
    if (S.active) {
      flush_max3(L, S.cur, WS_AMAX_M, S.am, WS_AMAX_V, S.av, WS_APPROX_W, S.aw);
      flush_max3(L, S.cur, WS_STEP_MAX, S.au, WS_STEP_MAX, S.au, WS_STEP_MAX, S.au);
    }
  if constexpr (PASS == 3)
    if (S.active) flush_max3(L, S.cur, WS_AMAX_W, S.aw, WS_AMAX_W, S.aw, WS_AMAX_W, S.aw);
  if constexpr (PASS == 2) flush_max3(L, S.cur, WS_STORED_W, S.am, WS_CHECK_W, S.aw, WS_CHECK_W, S.aw);
  if constexpr (PASS == 6 || PASS == 7)
    if (S.active) {
      flush_max3(L, S.cur, WS_AMAX_M, S.am, WS_AMAX_V, S.av, WS_CHECK_W, S.aw);
      if (S.tracked) flush_max3(L, S.cur, WS_STORED_W, S.au, WS_STORED_W, S.au, WS_STORED_W, S.au);
    }
  S.am = S.av = S.aw = S.au = 0.f;
}

// The gradient's descale: stored with its E5M2 codes, or (passes 8, 9) from
// the scale of its amax, as the gradient cast derives it (that scale kept
// for the cast in the pass).
template <int PASS_>
__device__ __forceinline__ float chunk_grad_inv(const AdamLaunch &L, const AdamChunkDev &C, AdamChunkState &S) {
  if constexpr (cast_grad_pass<PASS_>()) {
    int k;
    grad_scale_exponent(L, C, k);
    S.sg = pow2f(k);
    return pow2f(-k);
  } else {
    return *C.g_inv;
  }
}

template <int PASS_>
__device__ __forceinline__ void adam_chunk_enter(const AdamLaunch &L, int ci, AdamChunkState &S) {
  constexpr int PASS = base_pass<PASS_>();
  constexpr bool kStats = PASS == 1 || PASS == 4 || PASS == 5;
  const AdamChunkDev &C = L.c[ci];
  S.cur = ci;
  if constexpr (kStats) {
    S.tracked = C.w_amax != nullptr && *C.w_amax >= 0.0f;
    S.active = S.tracked == (PASS == 4);
    S.sc = adam_scalars(L, *C.g_inv, 1.0f / *C.m_scale, 1.0f / *C.v_scale, 1.0f / *C.w_scale);
  } else if constexpr (PASS == 6) {
    // the predicted new scales are the old ones (the same expressions as the
    // in-place step's, so a prediction that holds gives its exact results)
    S.tracked = C.w_amax != nullptr;
    S.active = true;
    const float sm = *C.m_scale, sv = *C.v_scale, sw = *C.w_scale;
    S.sc = adam_scalars(L, chunk_grad_inv<PASS_>(L, C, S), 1.0f / sm, 1.0f / sv, 1.0f / sw);
    S.ns.m = both(sm);
    S.ns.v = both(sv);
    S.ns.w = both(sw);
    S.want_wq = C.wq != nullptr;
    S.ns.q = both(S.want_wq ? __fmul_rn(*C.wq_scale, 1.0f / sw) : 1.0f);
  } else {
    const uint32_t fl = ws_flags(L, ci);
    // passes 2 and 7: keep the stored-master amax (and its check) for every
    // chunk that tracks it, including the step that first establishes it
    S.tracked = PASS == 3 ? (fl & FLAG_TRACKED) != 0 : C.w_amax != nullptr;
    S.active = PASS == 2 || (fl & (PASS == 7 ? FLAG_REDO : FLAG_EXACT)) != 0;
    S.sc = adam_scalars(L, chunk_grad_inv<PASS_>(L, C, S), ws_get(L, ci, WS_OLDINV_M),
                        ws_get(L, ci, WS_OLDINV_V), ws_get(L, ci, WS_OLDINV_W));
    S.ns.m = both(ws_get(L, ci, WS_NEW_M));
    S.ns.v = both(ws_get(L, ci, WS_NEW_V));
    S.ns.w = both(ws_get(L, ci, WS_NEW_W));

    S.want_wq = C.wq != nullptr;
    // the two scales are powers of two from nearly the same amax, so their
    // ratio is a normal float and (h * s_q / s_w) one exact multiplication
    S.ns.q = both(S.want_wq ? __fmul_rn(ws_get(L, ci, WS_NEW_WQ), 1.0f / S.ns.w.x) : 1.0f);
  }
}

// The ragged end of a chunk, [base, n) with n - base < 16: element by element
// from global memory (lane y of the packed arithmetic unused).
template <int PASS_>
__device__ __forceinline__ void adam_tail(const AdamLaunch &L, const AdamChunkDev &C, unsigned long long base,
                                       AdamChunkState &S) {
  constexpr int PASS = base_pass<PASS_>();
  constexpr bool kStats = PASS == 1 || PASS == 4 || PASS == 5;
  const bool read_w = PASS != 4;
  const AdamScalars &sc = S.sc;
  const AdamNewScales &ns = S.ns;
  for (unsigned long long i = base; i < C.n; i++) {
    uint32_t gc;
    if constexpr (cast_grad_pass<PASS_>())  // bfloat16 element i, times its scale, to E5M2
      gc = enc2<FP8_E5M2>(__fmul_rn(__uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(C.g)[i] << 16),
                                    S.sg), 0.0f) & 0xffu;
    else
      gc = C.g[i];
    const float2 gd = dec2<FP8_E5M2>(gc), md = dec2<FP8_E4M3>(C.m[i]);
    const float2 vd = make_float2(__half2float(__ushort_as_half(C.v[i])), 0.0f);
    const float2 wd = make_float2(read_w ? __half2float(__ushort_as_half(C.w[i])) : 0.0f, 0.0f);
    float2 m, v, d;
    if constexpr (PASS == 4 || PASS == 5)
      adam_moments_bound(L, make_float2(gd.x, 0.0f), make_float2(md.x, 0.0f), vd, sc, m, v, d);
    else
      adam_moments(L, make_float2(gd.x, 0.0f), make_float2(md.x, 0.0f), vd, sc, m, v, d);
    if constexpr (kStats) {
      S.am = max_abs1(S.am, m.x);
      S.av = max_abs1(S.av, v.x);
      S.aw = max_abs1(S.aw, S.tracked ? d.x : adam_master(wd, d, sc).x);
      if constexpr (PASS == 5) S.au = max_abs1(S.au, d.x);
    } else if constexpr (PASS == 3) {
      S.aw = max_abs1(S.aw, adam_master(wd, d, sc).x);
    } else {
      const float w = adam_master(wd, d, sc).x;
      S.aw = max_abs1(S.aw, w);
      if constexpr (PASS != 2) {
        S.am = max_abs1(S.am, m.x);
        S.av = max_abs1(S.av, v.x);
      }
      C.m_out[i] = (uint8_t)(enc2<FP8_E4M3>(__fmul_rn(m.x, ns.m.x), 0.0f) & 0xffu);
      C.v_out[i] = __half_as_ushort(__float2half_rn(__fmul_rn(v.x, ns.v.x)));
      const __half h = __float2half_rn(__fmul_rn(w, ns.w.x));
      C.w_out[i] = __half_as_ushort(h);
      const float st = __half2float(h);
      if (S.tracked) {
        if constexpr (PASS == 2) S.am = max_abs1(S.am, st); else S.au = max_abs1(S.au, st);
      }
      if (S.want_wq)
        C.wq[i] = (uint8_t)(enc2<FP8_E4M3>(__fmul_rn(st, ns.q.x), 0.0f) & 0xffu);
    }
  }
}

// One pass over all tiles of a launch.  PASS 5: stats of the chunks that do
// not track their master amax (exact amaxes of m and v, the estimate A~ and
// the step bound U).  PASS 1: the same chunks' exact new amaxes (the phased
// step).  PASS 4: stats of the chunks that track it (amaxes of m and v, U).
// PASS 3: exact master amax of flagged chunks.  PASS 2: update.  PASS 6:
// out-of-place update with the predicted scales.  PASS 7: its redo of the
// flagged chunks.  The stats
// passes are separate kernels so that the estimated arithmetic does not
// carry the register count of the exact one.
template <int PASS>
__device__ __forceinline__ void adam_pass(const AdamLaunch &L) {
  AdamChunkState S;
  for (unsigned long long tile = blockIdx.x; tile < L.total_tiles; tile += gridDim.x) {
    const int ci = find_chunk(L, tile);  // uniform across the block
    const AdamChunkDev &C = L.c[ci];
    if (ci != S.cur) {
      if (S.cur >= 0) adam_chunk_flush<PASS>(L, S);
      adam_chunk_enter<PASS>(L, ci, S);
    }
    if (!S.active) {  // passes 1b and 7: chunk not flagged; stats: the other stats pass's chunk
      // jump to this block's last tile inside the chunk; the loop step leaves it
      const unsigned long long end = C.tile_begin + (C.n + kAdamTile - 1) / kAdamTile;
      tile += ((end - tile - 1) / gridDim.x) * gridDim.x;
      continue;
    }
    const unsigned long long base =
        (tile - C.tile_begin) * kAdamTile + (unsigned long long)threadIdx.x * kAdamPerThread;
    if (base >= C.n) continue;
    if (base + kAdamPerThread <= C.n) {
      const size_t grp = base / kAdamPerThread;
      if constexpr (PASS == 4) {
        adam_group<1, true, false>(L, C, grp, S.sc, S.ns, S.am, S.av, S.aw, S.au);
      } else if constexpr (PASS == 5) {
        adam_group<5, false, false>(L, C, grp, S.sc, S.ns, S.am, S.av, S.aw, S.au);
      } else if constexpr (PASS == 1) {
        adam_group<1, false, false>(L, C, grp, S.sc, S.ns, S.am, S.av, S.aw, S.au);
      } else if constexpr (PASS == 3) {
        adam_group<3, false, false>(L, C, grp, S.sc, S.ns, S.am, S.av, S.aw, S.au);
      } else if constexpr (cast_grad_pass<PASS>()) {  // 8 or 9
        adam_group<PASS, true, true>(L, C, grp, S.sc, S.ns, S.am, S.av, S.aw, S.au, S.tracked, S.want_wq,
                                     both(S.sg));
      } else {  // an update pass: 2, 6 or 7
        adam_group<PASS, true, true>(L, C, grp, S.sc, S.ns, S.am, S.av, S.aw, S.au, S.tracked, S.want_wq);
      }
    } else {
      adam_tail<PASS>(L, C, base, S);
    }
  }
  // cur is block-uniform, so whole warps take these branches together.
  if (S.cur >= 0) adam_chunk_flush<PASS>(L, S);
}

template <int PASS>
__global__ void __launch_bounds__(kAdamThreads) k_adam(const __grid_constant__ AdamLaunch L) {
  adam_pass<PASS>(L);
}
// The in-place update pass: 64 registers and four resident blocks per SM.
// (Held to five blocks' 48 registers it spilled, 64 bytes per thread with the
// branch-free FP8 encoder; four and five blocks had measured the same when
// both were spill-free.  A variant fed through a shared-memory ring by bulk
// copies, one producer warp and eight consumer warps per block, two blocks
// per SM, was correct but 12 % slower at 64 M parameters: too few warps left
// to hide the update's arithmetic.)
template <>
__global__ void __launch_bounds__(kAdamThreads, 4) k_adam<2>(const __grid_constant__ AdamLaunch L) {
  adam_pass<2>(L);
}
// The out-of-place update and its redo: 64 registers and four resident
// blocks per SM.  (Held to five blocks' 48 registers they spilled ~100 bytes
// per thread and moved 4.2-4.4 TB/s at 2^26-2^28 parameters instead of
// 4.8-5.1.)
template <>
__global__ void __launch_bounds__(kAdamThreads, 4) k_adam<6>(const __grid_constant__ AdamLaunch L) {
  adam_pass<6>(L);
}
template <>
__global__ void __launch_bounds__(kAdamThreads, 4) k_adam<7>(const __grid_constant__ AdamLaunch L) {
  adam_pass<7>(L);
}
// The same two passes with the gradient cast in the pass.
template <>
__global__ void __launch_bounds__(kAdamThreads, 4) k_adam<8>(const __grid_constant__ AdamLaunch L) {
  adam_pass<8>(L);
}
template <>
__global__ void __launch_bounds__(kAdamThreads, 4) k_adam<9>(const __grid_constant__ AdamLaunch L) {
  adam_pass<9>(L);
}
// The estimated stats passes: six resident blocks per SM.
template <>
__global__ void __launch_bounds__(kAdamThreads, 6) k_adam<4>(const __grid_constant__ AdamLaunch L) {
  adam_pass<4>(L);
}
template <>
__global__ void __launch_bounds__(kAdamThreads, 6) k_adam<5>(const __grid_constant__ AdamLaunch L) {
  adam_pass<5>(L);
}

// Exponent of the E4M3 copy's scale from an amax of the stored master: the
// stored value of x is fp16(x s_w) / s_w (monotone in x).
__device__ __forceinline__ float stored_value(float x, float s_w) {
  return __fmul_rn(__half2float(__float2half_rn(__fmul_rn(x, s_w))), 1.0f / s_w);
}

// Scale exponents of the master (FP16) and of its E4M3 copy when the new
// master's amax is known to lie in [lo, hi] and that interval holds no scale
// threshold of either; false otherwise (also for lo <= 0 or a non-finite hi).
__device__ __forceinline__ bool interval_scales(const AdamLaunch &L, const AdamChunkDev &C, float lo, float hi,
                                                int &kw, int &kq) {
  int klo, khi;
  if (!(lo > 0.0f && scale_exponent(lo, kMaxF16, L.margin, 0, klo) &&
        scale_exponent(hi, kMaxF16, L.margin, 0, khi) && klo == khi))
    return false;
  kw = klo;
  kq = 0;
  if (C.wq_scale != nullptr) {
    const float s = pow2f(kw);
    int qlo, qhi;
    if (!(scale_exponent(stored_value(lo, s), kMaxE4M3, L.margin, 0, qlo) &&
          scale_exponent(stored_value(hi, s), kMaxE4M3, L.margin, 0, qhi) && qlo == qhi))
      return false;
    kq = qlo;
  }
  return true;
}

// STAGE 1: after the stats passes.  STAGE 2: after pass 1b.  STAGE 3: after
// pass 2.  STAGE 12: stages 1 and 2 in one launch (the phased step: every
// chunk's exact amaxes came from pass 1, so nothing is flagged).  STAGE 6:
// after the out-of-place pass 6.  STAGE 7: after its redo pass 7.
template <int STAGE>
__global__ void k_adam_finalize(const __grid_constant__ AdamLaunch L) {
  for (int ci = threadIdx.x; ci < L.nchunks; ci += blockDim.x) {
    float *ws = L.ws + ci * kAdamWsFloatsPerChunk;
    const AdamChunkDev &C = L.c[ci];
    uint32_t flags = __float_as_uint(ws[WS_FLAGS]);
    if constexpr (STAGE == 1 || STAGE == 12) {
      int km, kv;
      bool ok = scale_exponent(ws[WS_AMAX_M], kMaxE4M3, L.margin, 0, km);
      ok &= scale_exponent(ws[WS_AMAX_V], kMaxF16, L.margin, 0, kv);
      ws[WS_OLDINV_M] = 1.0f / *C.m_scale;
      ws[WS_OLDINV_V] = 1.0f / *C.v_scale;
      ws[WS_OLDINV_W] = 1.0f / *C.w_scale;
      ws[WS_NEW_M] = pow2f(km);
      ws[WS_NEW_V] = pow2f(kv);
      if (!ok) atomicOr(&g_status, FP8_STATUS_NONFINITE);
      const bool tracked = C.w_amax != nullptr && *C.w_amax >= 0.0f;
      flags = tracked ? FLAG_TRACKED : 0u;
      if (STAGE == 1 && (tracked || L.estimate)) {
        float lo, hi;
        if (tracked) {
          // amax|w_new| lies in [A0 - U, A0 + U], widened for the estimated
          // step and the one rounding of w0 + dw
          const float a0 = *C.w_amax, u = __fmul_ru(ws[WS_STEP_MAX], kStepBoundWiden);
          hi = __fmul_rn(__fadd_ru(a0, u), 1.0f + 0x1p-20f);
          lo = __fmul_rn(__fsub_rd(a0, u), 1.0f - 0x1p-20f);
        } else {
          // the estimate A~ differs from the exact amax by at most the largest
          // step error (< 2^-18 U) plus one rounding of the master (2^-23 A~)
          const float a = ws[WS_APPROX_W];
          const float e = __fadd_ru(__fmul_ru(ws[WS_STEP_MAX], 0x1p-16f), __fmul_ru(a, 0x1p-21f));
          hi = __fmul_rn(__fadd_ru(a, e), 1.0f + 0x1p-20f);
          lo = __fmul_rn(__fsub_rd(a, e), 1.0f - 0x1p-20f);
        }
        int kw, kq;
        if (interval_scales(L, C, lo, hi, kw, kq)) {
          ws[WS_NEW_W] = pow2f(kw);
          ws[WS_NEW_WQ] = pow2f(kq);
          flags |= FLAG_KNOWN;
        } else {
          flags |= FLAG_EXACT;
        }
      }
      ws[WS_FLAGS] = __uint_as_float(flags);
    }
    if constexpr (STAGE == 2 || STAGE == 12) {
      // exact master amax: from pass 1 (phased step) or pass 1b (flagged chunks)
      if (!(flags & FLAG_KNOWN)) {
        int kw, kq = 0;
        bool ok = scale_exponent(ws[WS_AMAX_W], kMaxF16, L.margin, 0, kw);
        if (C.wq_scale != nullptr)
          ok &= scale_exponent(stored_value(ws[WS_AMAX_W], pow2f(kw)), kMaxE4M3, L.margin, 0, kq);
        if (!ok) atomicOr(&g_status, FP8_STATUS_NONFINITE);
        ws[WS_NEW_W] = pow2f(kw);
        ws[WS_NEW_WQ] = pow2f(kq);
      }
      *C.m_scale = ws[WS_NEW_M];
      *C.v_scale = ws[WS_NEW_V];
      *C.w_scale = ws[WS_NEW_W];
      if (C.wq_scale != nullptr) {  // a copy was asked for (its codes may be an empty slice)
        *C.wq_scale = ws[WS_NEW_WQ];
        *C.wq_inv = 1.0f / ws[WS_NEW_WQ];
      }
    }
    if constexpr (STAGE == 6) {
      // the scales of the exact new amaxes pass 6 reduced (the rule of
      // stages 1 and 2), compared with the predicted old scales
      int km, kv, kw, kq = 0;
      bool ok = scale_exponent(ws[WS_AMAX_M], kMaxE4M3, L.margin, 0, km);
      ok &= scale_exponent(ws[WS_AMAX_V], kMaxF16, L.margin, 0, kv);
      ok &= scale_exponent(ws[WS_CHECK_W], kMaxF16, L.margin, 0, kw);
      if (C.wq_scale != nullptr)
        ok &= scale_exponent(stored_value(ws[WS_CHECK_W], pow2f(kw)), kMaxE4M3, L.margin, 0, kq);
      if (!ok) atomicOr(&g_status, FP8_STATUS_NONFINITE);
      const float sm = *C.m_scale, sv = *C.v_scale, sw = *C.w_scale;
      const float nm = pow2f(km), nv = pow2f(kv), nw = pow2f(kw), nq = pow2f(kq);
      const bool held = nm == sm && nv == sv && nw == sw && (C.wq_scale == nullptr || nq == *C.wq_scale);
      ws[WS_OLDINV_M] = 1.0f / sm;
      ws[WS_OLDINV_V] = 1.0f / sv;
      ws[WS_OLDINV_W] = 1.0f / sw;
      ws[WS_NEW_M] = nm;
      ws[WS_NEW_V] = nv;
      ws[WS_NEW_W] = nw;
      ws[WS_NEW_WQ] = nq;
      if (!held) ws[WS_STORED_W] = 0.0f;  // the redo reduces it again with the right scale
      ws[WS_FLAGS] = __uint_as_float(held ? 0u : FLAG_REDO);
      *C.m_scale = nm;
      *C.v_scale = nv;
      *C.w_scale = nw;
      if (C.wq_scale != nullptr) {
        *C.wq_scale = nq;
        *C.wq_inv = 1.0f / nq;
      }
      if (held && C.w_amax != nullptr) *C.w_amax = __fmul_rn(ws[WS_STORED_W], 1.0f / nw);
      if (L.g_hp) {  // passes 8, 9: publish the gradient's descale, as the gradient cast would
        int kg;
        if (!grad_scale_exponent(L, C, kg)) atomicOr(&g_status, FP8_STATUS_NONFINITE);
        *const_cast<float *>(C.g_inv) = pow2f(-kg);
      }
    }
    if constexpr (STAGE == 7) {
      if ((flags & FLAG_REDO) && C.w_amax != nullptr)
        *C.w_amax = __fmul_rn(ws[WS_STORED_W], 1.0f / ws[WS_NEW_W]);
    }
    if constexpr (STAGE == 3) {
      // a scale decided from an interval must be the one the exact new amax gives
      int kw;
      if ((flags & FLAG_KNOWN) && scale_exponent(ws[WS_CHECK_W], kMaxF16, L.margin, 0, kw) &&
          pow2f(kw) != ws[WS_NEW_W])
        atomicOr(&g_status, FP8_STATUS_INTERNAL);
      if (C.w_amax != nullptr) *C.w_amax = __fmul_rn(ws[WS_STORED_W], 1.0f / ws[WS_NEW_W]);
    }
  }
}

// Self-test of rcp_rn_step against CUDA's correctly rounded __frcp_rn on the
// binary32 arguments with bit patterns in [lo, hi): counts the arguments
// where the two differ (two NaNs agree) and keeps the smallest such pattern.
__global__ void k_step_reciprocal_selftest(uint32_t lo, unsigned long long hi, unsigned long long *bad,
                                           uint32_t *first) {
  const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
  unsigned long long nbad = 0;
  uint32_t lowest = 0xffffffffu;
  for (unsigned long long u = lo + (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; u < hi;
       u += stride) {
    const float x = __uint_as_float((uint32_t)u);
    const float a = rcp_rn_step(x), b = __frcp_rn(x);
    if (__float_as_uint(a) != __float_as_uint(b) && !(a != a && b != b)) {
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
