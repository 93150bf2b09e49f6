// adam.cuh -- precision-decoupled FP8 Adam ("FP8-LM: Training FP8 Large
// Language Models", 提案手法 O2): FP8 E5M2 gradient, FP8 E4M3 first moment,
// FP16 second moment and FP16 master weights, every tensor with its own
// power-of-two scale (6 bytes of state per parameter).
//
// The new scales are just-in-time: each comes from the amax of the *new*
// values (the same rule as the linear layer's casts), so a step is two
// streaming passes over all chunks plus a one-block finalize between them:
//   pass 1 (stats):  decode, update in registers, reduce amax|m|, amax v,
//                    amax|w| per chunk (nothing written but three scalars);
//   finalize:        new scales from those amaxes; old inverse scales saved;
//   pass 2 (update): decode, update again (bit-identical arithmetic),
//                    re-encode with the new scales, write m, v, w.
// All chunks of one call share each launch: the chunk table travels in the
// kernel parameters and tiles of 4096 parameters are mapped to chunks by a
// binary search over the chunks' first-tile indices.
#pragma once

#include "common.cuh"

namespace fp8lib {

constexpr int kAdamThreads = 256;
constexpr int kAdamPerThread = 16;
constexpr int kAdamTile = kAdamThreads * kAdamPerThread;  // parameters per tile
constexpr int kAdamMaxChunksPerLaunch = 256;
constexpr int kAdamWsFloatsPerChunk = 16;  // workspace slots per chunk (64 bytes)

// Workspace slots of one chunk.
enum : int {
  WS_AMAX_M = 0, WS_AMAX_V = 1, WS_AMAX_W = 2,
  WS_OLDINV_M = 3, WS_OLDINV_V = 4, WS_OLDINV_W = 5,
  WS_NEW_M = 6, WS_NEW_V = 7, WS_NEW_W = 8,
};

struct AdamChunkDev {
  const uint8_t *g;
  const float *g_inv;
  uint8_t *m;
  float *m_scale;
  uint16_t *v;
  float *v_scale;
  uint16_t *w;
  float *w_scale;
  unsigned long long n;
  unsigned long long tile_begin;
};

struct AdamLaunch {
  AdamChunkDev c[kAdamMaxChunksPerLaunch];
  int nchunks;
  int margin;
  unsigned long long total_tiles;
  float beta1, beta2, eps;
  float neg_lr_bc1;        // -lr / (1 - beta1^t)
  float inv_bc2;           // 1 / (1 - beta2^t)
  float *ws;               // kAdamWsFloatsPerChunk floats per chunk of this launch
};

// Per-chunk constants of the update: the descales are folded into the Adam
// coefficients, m = (b1/s_m) m~ + ((1-b1)/(mu s_g)) g~ and
// v = (b2/s_v) v~ + ((1-b2)/(mu s_g)^2) g~^2, where ~ marks a decoded code.
struct AdamScalars {
  float cm, cgm;   // b1 / s_m,  (1 - b1) g_inv
  float cv, cgv;   // b2 / s_v,  (1 - b2) g_inv^2
  float w_inv;     // 1 / s_w
};

__device__ __forceinline__ AdamScalars adam_scalars(const AdamLaunch &L, float g_inv, float m_inv,
                                                    float v_inv, float w_inv) {
  AdamScalars s;
  s.cm = __fmul_rn(L.beta1, m_inv);
  s.cgm = __fmul_rn(__fsub_rn(1.0f, L.beta1), g_inv);
  s.cv = __fmul_rn(L.beta2, v_inv);
  s.cgv = __fmul_rn(__fmul_rn(__fsub_rn(1.0f, L.beta2), g_inv), g_inv);
  s.w_inv = w_inv;
  return s;
}

// Approximate (MUFU) square root and reciprocal: relative error ~1e-7 on the
// step direction m_hat / (sqrt(v_hat) + eps), which moves the master weight by
// lr * O(1) -- far below an FP16 ULP of the stored master.
__device__ __forceinline__ float sqrt_approx(float x) {
  float r;
  asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// The update of one parameter, float32, from decoded codes.  Written with
// explicit round-to-nearest intrinsics so both passes evaluate exactly the
// same operations (the stats pass must see the values the update pass
// stores).  L.neg_lr_bc1 = -lr / (1 - b1^t), L.inv_bc2 = 1 / (1 - b2^t).
__device__ __forceinline__ void adam_update(const AdamLaunch &L, float gd, float md, float vd,
                                            float wd, const AdamScalars &s, float &m, float &v,
                                            float &w) {
  m = __fmaf_rn(s.cm, md, __fmul_rn(s.cgm, gd));
  v = __fmaf_rn(s.cv, vd, __fmul_rn(s.cgv, __fmul_rn(gd, gd)));
  const float denom = __fadd_rn(sqrt_approx(__fmul_rn(v, L.inv_bc2)), L.eps);
  w = __fmaf_rn(L.neg_lr_bc1, __fmul_rn(m, rcp_approx(denom)), __fmul_rn(wd, s.w_inv));
}

__device__ __forceinline__ int find_chunk(const AdamLaunch &L, unsigned long long tile) {
  int lo = 0, hi = L.nchunks - 1;  // last chunk whose tile_begin <= tile
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (L.c[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int PASS>
__global__ void __launch_bounds__(kAdamThreads) k_adam(const __grid_constant__ AdamLaunch L) {
  uint32_t am = 0, av = 0, aw = 0;  // pass 1: running maxima of the current chunk
  int cur = -1;
  AdamScalars sc{};  // of the current chunk
  float new_m = 1.f, new_v = 1.f, new_w = 1.f;

  for (unsigned long long tile = blockIdx.x; tile < L.total_tiles; tile += gridDim.x) {
    const int ci = find_chunk(L, tile);  // uniform across the block
    const AdamChunkDev &C = L.c[ci];
    if (ci != cur) {
      if constexpr (PASS == 1) {
        if (cur >= 0) {
          am = warp_max_u32(am); av = warp_max_u32(av); aw = warp_max_u32(aw);
          if ((threadIdx.x & 31) == 0) {
            float *ws = L.ws + cur * kAdamWsFloatsPerChunk;
            atomic_max_bits(ws + WS_AMAX_M, am);
            atomic_max_bits(ws + WS_AMAX_V, av);
            atomic_max_bits(ws + WS_AMAX_W, aw);
          }
          am = av = aw = 0;
        }
        sc = adam_scalars(L, *C.g_inv, 1.0f / *C.m_scale, 1.0f / *C.v_scale, 1.0f / *C.w_scale);
      } else {
        const float *ws = L.ws + ci * kAdamWsFloatsPerChunk;
        sc = adam_scalars(L, *C.g_inv, ws[WS_OLDINV_M], ws[WS_OLDINV_V], ws[WS_OLDINV_W]);
        new_m = ws[WS_NEW_M];
        new_v = ws[WS_NEW_V];
        new_w = ws[WS_NEW_W];
      }
      cur = ci;
    }
    const unsigned long long base =
        (tile - C.tile_begin) * kAdamTile + (unsigned long long)threadIdx.x * kAdamPerThread;
    if (base >= C.n) continue;
    if (base + kAdamPerThread <= C.n) {
      // Full group of 16: 16 B of g, 16 B of m, 32 B of v, 32 B of w.
      const size_t grp = base / kAdamPerThread;
      uint4 gq = __ldcs(reinterpret_cast<const uint4 *>(C.g) + grp);
      uint4 mq = __ldcs(reinterpret_cast<const uint4 *>(C.m) + grp);
      uint4 vq0 = __ldcs(reinterpret_cast<const uint4 *>(C.v) + 2 * grp);
      uint4 vq1 = __ldcs(reinterpret_cast<const uint4 *>(C.v) + 2 * grp + 1);
      uint4 wq0 = __ldcs(reinterpret_cast<const uint4 *>(C.w) + 2 * grp);
      uint4 wq1 = __ldcs(reinterpret_cast<const uint4 *>(C.w) + 2 * grp + 1);
      const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
      const uint32_t mw[4] = {mq.x, mq.y, mq.z, mq.w};
      const uint32_t vw[8] = {vq0.x, vq0.y, vq0.z, vq0.w, vq1.x, vq1.y, vq1.z, vq1.w};
      const uint32_t ww[8] = {wq0.x, wq0.y, wq0.z, wq0.w, wq1.x, wq1.y, wq1.z, wq1.w};
      uint32_t mo[4], vo[8], wo[8];
#pragma unroll
      for (int p = 0; p < 8; p++) {  // pairs of parameters
        const uint32_t g2 = (gw[p >> 1] >> ((p & 1) * 16)) & 0xffffu;
        const uint32_t m2 = (mw[p >> 1] >> ((p & 1) * 16)) & 0xffffu;
        float2 gd = dec2<FP8_E5M2>(g2), md = dec2<FP8_E4M3>(m2);
        float2 vd = h2f2(vw[p]), wd = h2f2(ww[p]);
        float m_a, v_a, w_a, m_b, v_b, w_b;
        adam_update(L, gd.x, md.x, vd.x, wd.x, sc, m_a, v_a, w_a);
        adam_update(L, gd.y, md.y, vd.y, wd.y, sc, m_b, v_b, w_b);
        if constexpr (PASS == 1) {
          am = max(am, max(absbits_f32(m_a), absbits_f32(m_b)));
          av = max(av, max(absbits_f32(v_a), absbits_f32(v_b)));
          aw = max(aw, max(absbits_f32(w_a), absbits_f32(w_b)));
        } else {
          const uint32_t mc = enc2<FP8_E4M3>(__fmul_rn(m_a, new_m), __fmul_rn(m_b, new_m));
          if (p & 1) mo[p >> 1] |= mc << 16; else mo[p >> 1] = mc;
          vo[p] = f16x2(__fmul_rn(v_a, new_v), __fmul_rn(v_b, new_v));
          wo[p] = f16x2(__fmul_rn(w_a, new_w), __fmul_rn(w_b, new_w));
        }
      }
      if constexpr (PASS == 2) {
        __stcs(reinterpret_cast<uint4 *>(C.m) + grp, make_uint4(mo[0], mo[1], mo[2], mo[3]));
        __stcs(reinterpret_cast<uint4 *>(C.v) + 2 * grp, make_uint4(vo[0], vo[1], vo[2], vo[3]));
        __stcs(reinterpret_cast<uint4 *>(C.v) + 2 * grp + 1, make_uint4(vo[4], vo[5], vo[6], vo[7]));
        __stcs(reinterpret_cast<uint4 *>(C.w) + 2 * grp, make_uint4(wo[0], wo[1], wo[2], wo[3]));
        __stcs(reinterpret_cast<uint4 *>(C.w) + 2 * grp + 1, make_uint4(wo[4], wo[5], wo[6], wo[7]));
      }
    } else {
      // Ragged end of a chunk: element by element.
      for (unsigned long long i = base; i < C.n; i++) {
        float gd = dec2<FP8_E5M2>(C.g[i]).x, md = dec2<FP8_E4M3>(C.m[i]).x;
        float vd = __half2float(__ushort_as_half(C.v[i])), wd = __half2float(__ushort_as_half(C.w[i]));
        float m, v, w;
        adam_update(L, gd, md, vd, wd, sc, m, v, w);
        if constexpr (PASS == 1) {
          am = max(am, absbits_f32(m));
          av = max(av, absbits_f32(v));
          aw = max(aw, absbits_f32(w));
        } else {
          C.m[i] = (uint8_t)(enc2<FP8_E4M3>(__fmul_rn(m, new_m), 0.0f) & 0xffu);
          C.v[i] = __half_as_ushort(__float2half_rn(__fmul_rn(v, new_v)));
          C.w[i] = __half_as_ushort(__float2half_rn(__fmul_rn(w, new_w)));
        }
      }
    }
  }
  if constexpr (PASS == 1) {
    // cur is block-uniform, so the whole warp takes this branch together.
    if (cur >= 0) {
      am = warp_max_u32(am); av = warp_max_u32(av); aw = warp_max_u32(aw);
      if ((threadIdx.x & 31) == 0) {
        float *ws = L.ws + cur * kAdamWsFloatsPerChunk;
        atomic_max_bits(ws + WS_AMAX_M, am);
        atomic_max_bits(ws + WS_AMAX_V, av);
        atomic_max_bits(ws + WS_AMAX_W, aw);
      }
    }
  }
}

// Between the passes: new scales from the new amaxes, old inverse scales
// saved for pass 2, new scales published to the caller's scale slots.
__global__ void k_adam_finalize(const __grid_constant__ AdamLaunch L) {
  for (int ci = threadIdx.x; ci < L.nchunks; ci += blockDim.x) {
    float *ws = L.ws + ci * kAdamWsFloatsPerChunk;
    const AdamChunkDev &C = L.c[ci];
    int km, kv, kw;
    bool ok = scale_exponent(ws[WS_AMAX_M], kMaxE4M3, L.margin, 0, km);
    ok &= scale_exponent(ws[WS_AMAX_V], kMaxF16, L.margin, 0, kv);
    ok &= scale_exponent(ws[WS_AMAX_W], kMaxF16, L.margin, 0, kw);
    if (!ok) atomicOr(&g_status, FP8_STATUS_NONFINITE);
    ws[WS_OLDINV_M] = 1.0f / *C.m_scale;
    ws[WS_OLDINV_V] = 1.0f / *C.v_scale;
    ws[WS_OLDINV_W] = 1.0f / *C.w_scale;
    ws[WS_NEW_M] = pow2f(km);
    ws[WS_NEW_V] = pow2f(kv);
    ws[WS_NEW_W] = pow2f(kw);
    *C.m_scale = pow2f(km);
    *C.v_scale = pow2f(kv);
    *C.w_scale = pow2f(kw);
  }
}

}  // namespace fp8lib
