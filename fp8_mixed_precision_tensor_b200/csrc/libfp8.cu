// libfp8.cu -- the C ABI of include/fp8.h: argument checks, TMA descriptor
// encoding and kernel launches.  All device code lives in the headers
// included below; this is the library's single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/fp8.h"
#include <type_traits>

#include "adam.cuh"
#include "allreduce.cuh"
#include "amax_cast.cuh"
#include "common.cuh"
#include "gemm.cuh"

using namespace fp8lib;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int adam_blocks_per_sm = 1;        // resident blocks of the update pass
  int adam_stats_blocks_per_sm = 1;  // of the exact stats pass and the exact master pass
  int adam_bound_blocks_per_sm = 1;  // of the estimated stats pass of tracking chunks
  int adam_est_blocks_per_sm = 1;    // of the estimated stats pass of the other chunks
  int adam_into_blocks_per_sm = 1;   // of the out-of-place update (and its redo)
  int adam_castg_blocks_per_sm = 1;  // of the same with the gradient cast in the pass
  int cast_blocks_per_sm = 8;        // resident blocks of the streaming cast kernels
  int pair_clusters = 0;  // co-resident 2-CTA clusters of the pair GEMM
  int wide_clusters = 0;  // co-resident 2-CTA clusters of the wide pair GEMM
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA; }

template <typename K>
int set_smem(K kernel, int bytes) {
  return cuda_rc(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
}
// The wide kernel is instantiated per output type.
template <bool A_MN, bool B_MN>
int set_wide_smem() {
  return set_smem(gemm::k_gemm3<A_MN, B_MN, FP8_DT_F32>, gemm::kWideSmemBytes) |
         set_smem(gemm::k_gemm3<A_MN, B_MN, FP8_DT_BF16>, gemm::kWideSmemBytes) |
         set_smem(gemm::k_gemm3<A_MN, B_MN, FP8_DT_F16>, gemm::kWideSmemBytes) |
         set_smem(gemm::k_gemm3<A_MN, B_MN, FP8_DT_BF16_RTO>, gemm::kWideSmemBytes);
}

// One-time per-device set-up: SM count, occupancy, kernel attributes.
int device_info(DeviceInfo **out) {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FP8_ERR_CUDA;
    int bps = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_adam<2>, kAdamThreads, 0) != cudaSuccess)
      return FP8_ERR_CUDA;
    d.adam_blocks_per_sm = bps > 0 ? bps : 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_adam<1>, kAdamThreads, 0) != cudaSuccess)
      return FP8_ERR_CUDA;
    d.adam_stats_blocks_per_sm = bps > 0 ? bps : 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_adam<4>, kAdamThreads, 0) != cudaSuccess)
      return FP8_ERR_CUDA;
    d.adam_bound_blocks_per_sm = bps > 0 ? bps : 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_adam<5>, kAdamThreads, 0) != cudaSuccess)
      return FP8_ERR_CUDA;
    d.adam_est_blocks_per_sm = bps > 0 ? bps : 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_adam<6>, kAdamThreads, 0) != cudaSuccess)
      return FP8_ERR_CUDA;
    d.adam_into_blocks_per_sm = bps > 0 ? bps : 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k_adam<8>, kAdamThreads, 0) != cudaSuccess)
      return FP8_ERR_CUDA;
    d.adam_castg_blocks_per_sm = bps > 0 ? bps : 1;
    // the cast kernels' grids are one wave of resident blocks (a grid-stride
    // loop gives each block an equal share; a partial second wave would run
    // a third of the work on a few SMs): the fewest resident blocks of the
    // instantiations the training step runs
    {
      int lo = 8;
      const void *casts[] = {(const void *)k_cast<FP8_DT_BF16, FP8_E4M3, false>,
                             (const void *)k_cast<FP8_DT_BF16, FP8_E5M2, false>,
                             (const void *)k_amax_cast<FP8_DT_BF16, FP8_E4M3>,
                             (const void *)k_amax_cast<FP8_DT_BF16, FP8_E5M2>,
                             (const void *)k_cast_redo<FP8_DT_BF16, FP8_E4M3>};
      for (const void *k : casts) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k, kStreamThreads, 0) != cudaSuccess)
          return FP8_ERR_CUDA;
        if (bps > 0 && bps < lo) lo = bps;
      }
      d.cast_blocks_per_sm = lo;
    }
    int rc = FP8_OK;
    rc |= set_smem(gemm::k_gemm<256, false, false>, gemm::Cfg<256>::SMEM_BYTES);
    rc |= set_smem(gemm::k_gemm<256, false, true>, gemm::Cfg<256>::SMEM_BYTES);
    rc |= set_smem(gemm::k_gemm<256, true, true>, gemm::Cfg<256>::SMEM_BYTES);
    rc |= set_smem(gemm::k_gemm2<false, false>, gemm::kPairSmemBytes);
    rc |= set_smem(gemm::k_gemm2<false, true>, gemm::kPairSmemBytes);
    rc |= set_smem(gemm::k_gemm2<true, true>, gemm::kPairSmemBytes);
    rc |= set_wide_smem<false, false>();
    rc |= set_wide_smem<false, true>();
    rc |= set_wide_smem<true, true>();
    if (rc) return FP8_ERR_CUDA;
    {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (d.sms / 2));
      cfg.blockDim = dim3(gemm::kThreads);
      cfg.dynamicSmemBytes = gemm::kPairSmemBytes;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, gemm::k_gemm2<false, false>, &cfg) != cudaSuccess)
        return FP8_ERR_CUDA;
      d.pair_clusters = clusters;
      cfg.blockDim = dim3(gemm::kWideThreads);
      cfg.dynamicSmemBytes = gemm::kWideSmemBytes;
      if (cudaOccupancyMaxActiveClusters(&clusters, gemm::k_gemm3<false, false, FP8_DT_BF16>, &cfg) != cudaSuccess)
        return FP8_ERR_CUDA;
      d.wide_clusters = clusters;
    }
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void *fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FP8_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return FP8_OK;
}

int launch_rc() { return cuda_rc(cudaGetLastError()); }

bool valid_dtype(int dt) { return dt == FP8_DT_F32 || dt == FP8_DT_BF16 || dt == FP8_DT_F16; }
bool valid_out_dtype(int dt) { return valid_dtype(dt) || dt == FP8_DT_BF16_RTO; }
bool valid_fmt(int f) { return f == FP8_E4M3 || f == FP8_E5M2 || f == FP8_F16S; }

unsigned grid_for(size_t work_items, int per_block, int cap) {
  size_t b = (work_items + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > (size_t)cap) b = cap;
  return (unsigned)b;
}

// 2-D row-major uint8 tensor [outer, inner] -> TMA map with a box of
// 128 bytes x box_outer rows and the 128-byte swizzle.
int make_map(CUtensorMap *m, const void *ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8_OK : FP8_ERR_CUDA;
}

// Row-major output [rows, cols] -> TMA map for 32-row boxes of 128 bytes
// (32 fp32 or 64 16-bit columns) with the 128-byte swizzle (bulk stores).
int make_out_map(CUtensorMap *m, void *out, int dtype, uint64_t rows, uint64_t cols) {
  const CUtensorMapDataType t = dtype == FP8_DT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : (dtype == FP8_DT_BF16 || dtype == FP8_DT_BF16_RTO) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const uint64_t esz = dtype == FP8_DT_F32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, t, 2, out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8_OK : FP8_ERR_CUDA;
}

// C[rows, cols] = sum_k A(r, k) B(c, k), operand majorness as template flags.
// A is [rows, K] (K-major) or [K, rows] (MN-major); B likewise with cols.
template <bool A_MN, bool B_MN>
int run_gemm(const uint8_t *A, int fmt_a, const float *inv_a, const uint8_t *B, int fmt_b,
             const float *inv_b, const void *bias, int bias_dtype, void *out, int out_dtype,
             float *out_amax, int rows, int cols, int K, cudaStream_t stream) {
  if (rows < 0 || cols < 0 || K < 0) return FP8_ERR_INVALID_ARG;
  if (!valid_out_dtype(out_dtype) || (bias && !valid_dtype(bias_dtype))) return FP8_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) {  // empty output: operands may be null
    if (out_amax) return cuda_rc(cudaMemsetAsync(out_amax, 0, sizeof(float), stream));
    return FP8_OK;
  }
  if (!A || !B || !inv_a || !inv_b || !out) return FP8_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(out)) return FP8_ERR_UNALIGNED;
  if (K == 0 || rows % 16 || cols % 16 || K % 16) return FP8_ERR_UNSUPPORTED;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  // Kernel choice: the widest tile that still gives every co-resident cluster
  // at least one tile (256x512 pair tiles, then 256x256, then one CTA 128x256).
  const int wide_tiles = ((rows + 255) / 256) * ((cols + 511) / 512);
  const int pair_tiles = ((rows + 255) / 256) * ((cols + 255) / 256);
  const int variant = (d->wide_clusters > 0 && wide_tiles >= d->wide_clusters) ? 3
                      : (d->pair_clusters > 0 && pair_tiles >= d->pair_clusters) ? 2 : 1;
  const int BN = variant == 3 ? 512 : 256;
  const uint32_t a_box = variant == 1 ? (uint32_t)gemm::BM : 128u;  // rows of A per CTA
  const uint32_t b_box = variant == 1 ? 256u : (variant == 2 ? 128u : 256u);  // B rows per CTA
  CUtensorMap ma, mb;
  if (A_MN) rc = make_map(&ma, A, (uint64_t)rows, (uint64_t)K, gemm::BK);
  else      rc = make_map(&ma, A, (uint64_t)K, (uint64_t)rows, a_box);
  if (rc) return rc;
  if (B_MN) rc = make_map(&mb, B, (uint64_t)cols, (uint64_t)K, gemm::BK);
  else      rc = make_map(&mb, B, (uint64_t)K, (uint64_t)cols, b_box);
  if (rc) return rc;
  const int tile_rows = variant == 1 ? gemm::BM : 256;
  gemm::Args a;
  a.rows = rows;
  a.cols = cols;
  a.K = K;
  a.num_m_blocks = (rows + tile_rows - 1) / tile_rows;
  a.num_n_blocks = (cols + BN - 1) / BN;
  a.num_tiles = a.num_m_blocks * a.num_n_blocks;
  a.num_k_blocks = (K + gemm::BK - 1) / gemm::BK;
  // tile order: bands of group_m row blocks, the weight-like operand swept
  // once per band; for the wide tile 16 row blocks (4096 rows) halve its
  // DRAM re-reads against 8 and measured 4 % faster in the GPT-175B step's
  // GEMMs under the power cap (32 let the band's A panels outgrow L2)
  a.group_m = variant == 3 ? 16 : (variant == 1 ? 16 : 8);
  // one MMA instruction: M = 128 (one CTA) or 256 (pair), N = 256
  a.idesc = (1u << 4)                       // accumulate in F32
            | ((uint32_t)fmt_a << 7)         // A: 0 = E4M3, 1 = E5M2
            | ((uint32_t)fmt_b << 10)        // B
            | ((uint32_t)(A_MN ? 1 : 0) << 15) | ((uint32_t)(B_MN ? 1 : 0) << 16)
            | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(tile_rows >> 4) << 24);
  a.inv_a = inv_a;
  a.inv_b = inv_b;
  a.bias = bias;
  a.bias_dtype = bias_dtype;
  a.out = out;
  a.out_dtype = out_dtype;
  a.out_amax = out_amax;
  if (out_amax && (rc = cuda_rc(cudaMemsetAsync(out_amax, 0, sizeof(float), stream)))) return rc;
  if (variant != 1) {
    const int avail = variant == 3 ? d->wide_clusters : d->pair_clusters;
    const int clusters = a.num_tiles < avail ? a.num_tiles : avail;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(variant == 3 ? gemm::kWideThreads : gemm::kThreads);
    cfg.dynamicSmemBytes = variant == 3 ? gemm::kWideSmemBytes : gemm::kPairSmemBytes;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (variant == 3) {
      CUtensorMap mo;
      if ((rc = make_out_map(&mo, out, out_dtype, (uint64_t)rows, (uint64_t)cols))) return rc;
      switch (out_dtype) {
        case FP8_DT_F32: return cuda_rc(cudaLaunchKernelEx(&cfg, gemm::k_gemm3<A_MN, B_MN, FP8_DT_F32>, ma, mb, mo, a));
        case FP8_DT_BF16: return cuda_rc(cudaLaunchKernelEx(&cfg, gemm::k_gemm3<A_MN, B_MN, FP8_DT_BF16>, ma, mb, mo, a));
        case FP8_DT_F16: return cuda_rc(cudaLaunchKernelEx(&cfg, gemm::k_gemm3<A_MN, B_MN, FP8_DT_F16>, ma, mb, mo, a));
        default: return cuda_rc(cudaLaunchKernelEx(&cfg, gemm::k_gemm3<A_MN, B_MN, FP8_DT_BF16_RTO>, ma, mb, mo, a));
      }
    }
    return cuda_rc(cudaLaunchKernelEx(&cfg, gemm::k_gemm2<A_MN, B_MN>, ma, mb, a));
  }
  unsigned grid = (unsigned)(a.num_tiles < d->sms ? a.num_tiles : d->sms);
  gemm::k_gemm<256, A_MN, B_MN><<<grid, gemm::kThreads, gemm::Cfg<256>::SMEM_BYTES, stream>>>(ma, mb, a);
  return launch_rc();
}

template <int DT>
void launch_amax(const void *x, size_t n, float *amax, cudaStream_t s, int sms) {
  unsigned grid = grid_for(n / 16, kStreamThreads * 4, sms * 8);
  k_amax<DT><<<grid, kStreamThreads, 0, s>>>(x, n, amax);
}

template <int DT, int FMT>
void launch_cast(const void *x, size_t n, const CastScale &cs, void *q, unsigned long long *counts,
                 cudaStream_t s, int max_blocks) {
  unsigned grid = grid_for(n / 16, kStreamThreads * 2, max_blocks);
  if (counts) k_cast<DT, FMT, true><<<grid, kStreamThreads, 0, s>>>(x, n, cs, q, counts);
  else k_cast<DT, FMT, false><<<grid, kStreamThreads, 0, s>>>(x, n, cs, q, nullptr);
}

template <int DT>
void launch_cast_dt(int fmt, const void *x, size_t n, const CastScale &cs, void *q, unsigned long long *counts,
                    cudaStream_t s, int max_blocks) {
  if (fmt == FP8_E4M3) launch_cast<DT, FP8_E4M3>(x, n, cs, q, counts, s, max_blocks);
  else if (fmt == FP8_E5M2) launch_cast<DT, FP8_E5M2>(x, n, cs, q, counts, s, max_blocks);
  else launch_cast<DT, FP8_F16S>(x, n, cs, q, counts, s, max_blocks);
}

int cast_common(const void *x, int dtype, size_t n, int fmt, const CastScale &cs, void *q, cudaStream_t s,
                unsigned long long *counts = nullptr) {
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  const int cap = d->sms * d->cast_blocks_per_sm;  // one wave of resident blocks
  if (dtype == FP8_DT_F32) launch_cast_dt<FP8_DT_F32>(fmt, x, n, cs, q, counts, s, cap);
  else if (dtype == FP8_DT_BF16) launch_cast_dt<FP8_DT_BF16>(fmt, x, n, cs, q, counts, s, cap);
  else launch_cast_dt<FP8_DT_F16>(fmt, x, n, cs, q, counts, s, cap);
  return launch_rc();
}

// The one-pass amax + cast: the pass with the predicted scale, the redo
// where the scale of the amax differs, then the scale published.
template <int DT, int FMT>
void launch_amax_cast(const void *x, size_t n, float *amax, int margin, int log2mu, float *scale, float *inv,
                      void *q, cudaStream_t s, int max_blocks) {
  const unsigned grid = grid_for(n / 16, kStreamThreads * 2, max_blocks);
  const float fmax = FMT == FP8_E4M3 ? 448.0f : (FMT == FP8_E5M2 ? 57344.0f : 65504.0f);
  if (n > 0) {
    k_amax_cast<DT, FMT><<<grid, kStreamThreads, 0, s>>>(x, n, scale, amax, q);
    k_cast_redo<DT, FMT><<<grid, kStreamThreads, 0, s>>>(x, n, scale, amax, fmax, margin, log2mu, q);
  }
  k_compute_scale<<<1, 1, 0, s>>>(amax, fmax, margin, log2mu, scale, inv);
}

template <int DT>
void launch_amax_cast_dt(int fmt, const void *x, size_t n, float *amax, int margin, int log2mu, float *scale,
                         float *inv, void *q, cudaStream_t s, int max_blocks) {
  if (fmt == FP8_E4M3) launch_amax_cast<DT, FP8_E4M3>(x, n, amax, margin, log2mu, scale, inv, q, s, max_blocks);
  else if (fmt == FP8_E5M2) launch_amax_cast<DT, FP8_E5M2>(x, n, amax, margin, log2mu, scale, inv, q, s, max_blocks);
  else launch_amax_cast<DT, FP8_F16S>(x, n, amax, margin, log2mu, scale, inv, q, s, max_blocks);
}

// mu must be a power of two in [2^-32, 2^32]; its log2 on success.
bool mu_log2(float mu, int *log2mu) {
  int e2;
  float frac = frexpf(mu, &e2);
  if (!(mu > 0.0f) || frac != 0.5f || e2 - 1 < -32 || e2 - 1 > 32) return false;
  *log2mu = e2 - 1;
  return true;
}

}  // namespace

extern "C" {

int fp8_amax(const void *x, int dtype, size_t n, float *amax_dev, void *stream) {
  if (!amax_dev || !valid_dtype(dtype) || (n > 0 && !x)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && !aligned16(x)) return FP8_ERR_UNALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = cuda_rc(cudaMemsetAsync(amax_dev, 0, sizeof(float), s));
  if (rc || n == 0) return rc;
  DeviceInfo *d;
  if ((rc = device_info(&d))) return rc;
  if (dtype == FP8_DT_F32) launch_amax<FP8_DT_F32>(x, n, amax_dev, s, d->sms);
  else if (dtype == FP8_DT_BF16) launch_amax<FP8_DT_BF16>(x, n, amax_dev, s, d->sms);
  else launch_amax<FP8_DT_F16>(x, n, amax_dev, s, d->sms);
  return launch_rc();
}

int fp8_compute_scale(const float *amax_dev, int fmt, int margin, float mu, float *scale_dev,
                      float *inv_scale_dev, void *stream) {
  if (!amax_dev || !scale_dev || !inv_scale_dev || !valid_fmt(fmt)) return FP8_ERR_INVALID_ARG;
  int log2mu;
  if (margin < 0 || margin > 64 || !mu_log2(mu, &log2mu)) return FP8_ERR_INVALID_ARG;
  k_compute_scale<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(amax_dev, fmt_max_of(fmt), margin,
                                                                 log2mu, scale_dev, inv_scale_dev);
  return launch_rc();
}

int fp8_cast(const void *x, int dtype, size_t n, int fmt, const float *scale_dev, void *q, void *stream) {
  if (!valid_dtype(dtype) || !valid_fmt(fmt) || !scale_dev) return FP8_ERR_INVALID_ARG;
  if (n == 0) return FP8_OK;
  if (!x || !q) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q)) return FP8_ERR_UNALIGNED;
  CastScale cs = {scale_dev, nullptr, 0.0f, 0, 0, nullptr, nullptr, nullptr};
  return cast_common(x, dtype, n, fmt, cs, q, static_cast<cudaStream_t>(stream));
}

int fp8_cast_count(const void *x, int dtype, size_t n, int fmt, const float *scale_dev, void *q,
                   unsigned long long *counts_dev, void *stream) {
  if (!valid_dtype(dtype) || !valid_fmt(fmt) || !scale_dev || !counts_dev) return FP8_ERR_INVALID_ARG;
  if (n == 0) return FP8_OK;
  if (!x || !q) return FP8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q)) return FP8_ERR_UNALIGNED;
  CastScale cs = {scale_dev, nullptr, 0.0f, 0, 0, nullptr, nullptr, nullptr};
  return cast_common(x, dtype, n, fmt, cs, q, static_cast<cudaStream_t>(stream), counts_dev);
}

int fp8_grad_cast(const void *g, int dtype, size_t n, int fmt, const float *amax_dev, int margin,
                  const float *mu_dev, float *scale_dev, float *inv_scale_dev, uint8_t *q,
                  unsigned long long *counts_dev, void *stream) {
  if (!valid_dtype(dtype) || (fmt != FP8_E4M3 && fmt != FP8_E5M2)) return FP8_ERR_INVALID_ARG;
  if (!amax_dev || !mu_dev || !scale_dev || !inv_scale_dev || margin < 0 || margin > 64)
    return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!g || !q)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!aligned16(g) || !aligned16(q))) return FP8_ERR_UNALIGNED;
  CastScale cs = {nullptr, amax_dev, fmt_max_of(fmt), margin, 0, scale_dev, inv_scale_dev, mu_dev};
  return cast_common(g, dtype, n, fmt, cs, q, static_cast<cudaStream_t>(stream), counts_dev);
}

int fp8_sum_codes(const uint8_t *in, int nranks, size_t ld, size_t n, int fmt, uint8_t *out,
                  const float *inv_scale_dev, float *g_inv_dev, unsigned long long *counts_dev,
                  void *stream) {
  if ((fmt != FP8_E4M3 && fmt != FP8_E5M2) || nranks < 1 || nranks > kSumMaxRanks || ld < n)
    return FP8_ERR_INVALID_ARG;
  if (g_inv_dev && !inv_scale_dev) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!in || !out)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!aligned16(in) || !aligned16(out) || ld % 16)) return FP8_ERR_UNALIGNED;
  if (n == 0 && !g_inv_dev) return FP8_OK;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = grid_for(n / 16, kSumThreads, d->sms * 8);
  if (fmt == FP8_E5M2 && nranks <= kSumFastMaxRanks)
    k_sum_codes_fast<FP8_E5M2><<<grid, kSumThreads, 0, s>>>(in, nranks, ld, n, out, inv_scale_dev, g_inv_dev,
                                                            counts_dev);
  else if (fmt == FP8_E5M2)
    k_sum_codes<FP8_E5M2><<<grid, kSumThreads, 0, s>>>(in, nranks, ld, n, out, inv_scale_dev, g_inv_dev, counts_dev);
  else
    k_sum_codes_fast<FP8_E4M3><<<grid, kSumThreads, 0, s>>>(in, nranks, ld, n, out, inv_scale_dev, g_inv_dev,
                                                            counts_dev);
  return launch_rc();
}

int fp8_mu_update(float *mu_dev, int *clean_dev, unsigned long long *counts_dev, unsigned long long n,
                  const fp8_mu_rule *rule, void *stream) {
  if (!mu_dev || !clean_dev || !counts_dev || !rule) return FP8_ERR_INVALID_ARG;
  int lo, hi;
  if (!(rule->theta >= 0.0f) || rule->interval < 1 || !mu_log2(rule->mu_min, &lo) ||
      !mu_log2(rule->mu_max, &hi) || lo > hi)
    return FP8_ERR_INVALID_ARG;
  k_mu_update<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(mu_dev, clean_dev, counts_dev, n,
                                                               (double)rule->theta, rule->interval,
                                                               rule->mu_min, rule->mu_max);
  return launch_rc();
}

int fp8_scale_cast(const void *x, int dtype, size_t n, int fmt, const float *amax_dev, int margin, float mu,
                   float *scale_dev, float *inv_scale_dev, void *q, void *stream) {
  int log2mu;
  if (!valid_dtype(dtype) || !valid_fmt(fmt) || !amax_dev || !scale_dev || !inv_scale_dev)
    return FP8_ERR_INVALID_ARG;
  if (margin < 0 || margin > 64 || !mu_log2(mu, &log2mu)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!x || !q)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!aligned16(x) || !aligned16(q))) return FP8_ERR_UNALIGNED;
  CastScale cs = {nullptr, amax_dev, fmt_max_of(fmt), margin, log2mu, scale_dev, inv_scale_dev, nullptr};
  return cast_common(x, dtype, n, fmt, cs, q, static_cast<cudaStream_t>(stream));
}

int fp8_amax_scale_cast(const void *x, int dtype, size_t n, int fmt, float *amax_dev, int margin, float mu,
                        float *scale_dev, float *inv_scale_dev, void *q, void *stream) {
  int log2mu;
  if (!valid_dtype(dtype) || !valid_fmt(fmt) || !amax_dev || !scale_dev || !inv_scale_dev)
    return FP8_ERR_INVALID_ARG;
  if (margin < 0 || margin > 64 || !mu_log2(mu, &log2mu)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!x || !q)) return FP8_ERR_INVALID_ARG;
  if (n > 0 && (!aligned16(x) || !aligned16(q))) return FP8_ERR_UNALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = cuda_rc(cudaMemsetAsync(amax_dev, 0, sizeof(float), s));
  if (rc) return rc;
  DeviceInfo *d;
  if ((rc = device_info(&d))) return rc;
  const int cap = d->sms * d->cast_blocks_per_sm;  // one wave of resident blocks
  if (dtype == FP8_DT_F32)
    launch_amax_cast_dt<FP8_DT_F32>(fmt, x, n, amax_dev, margin, log2mu, scale_dev, inv_scale_dev, q, s, cap);
  else if (dtype == FP8_DT_BF16)
    launch_amax_cast_dt<FP8_DT_BF16>(fmt, x, n, amax_dev, margin, log2mu, scale_dev, inv_scale_dev, q, s, cap);
  else
    launch_amax_cast_dt<FP8_DT_F16>(fmt, x, n, amax_dev, margin, log2mu, scale_dev, inv_scale_dev, q, s, cap);
  return launch_rc();
}

int fp8_linear_fwd(const uint8_t *xq, const float *x_inv, const uint8_t *wq, const float *w_inv,
                   const void *bias, int bias_dtype, void *y, int y_dtype, float *y_amax, int M,
                   int N, int K, void *stream) {
  return run_gemm<false, false>(xq, FP8_E4M3, x_inv, wq, FP8_E4M3, w_inv, bias, bias_dtype, y,
                                y_dtype, y_amax, M, N, K, static_cast<cudaStream_t>(stream));
}

int fp8_linear_dgrad(const uint8_t *dyq, const float *dy_inv, const uint8_t *wq,
                     const float *w_inv, void *dx, int dx_dtype, float *dx_amax, int M, int N,
                     int K, void *stream) {
  // dX[M,K] = dY[M,N] . W[N,K]: rows M, cols K, reduction N; W is MN-major.
  return run_gemm<false, true>(dyq, FP8_E5M2, dy_inv, wq, FP8_E4M3, w_inv, nullptr, 0, dx,
                               dx_dtype, dx_amax, M, K, N, static_cast<cudaStream_t>(stream));
}

int fp8_linear_wgrad(const uint8_t *dyq, const float *dy_inv, const uint8_t *xq,
                     const float *x_inv, void *dw, int dw_dtype, float *dw_amax, int M, int N,
                     int K, void *stream) {
  // dW[N,K] = dY[M,N]^T . X[M,K]: rows N, cols K, reduction M; both MN-major.
  return run_gemm<true, true>(dyq, FP8_E5M2, dy_inv, xq, FP8_E4M3, x_inv, nullptr, 0, dw,
                              dw_dtype, dw_amax, N, K, M, static_cast<cudaStream_t>(stream));
}

size_t fp8_adam_workspace_bytes(int nchunks) {
  if (nchunks <= 0) return 0;
  return (size_t)nchunks * kAdamWsFloatsPerChunk * sizeof(float);
}

}  // extern "C"

namespace {

// The Adam step in phases: PH_STATS runs the stats pass into the workspace,
// PH_APPLY finalizes the scales from it and runs the update, PH_ALL both.
// With PH_INTO the step is out of place (dest holds the new buffers):
// PH_STATS is then the update with the predicted scales, which leaves the
// exact new amaxes in the workspace, and PH_APPLY the scale decision and the
// redo of the chunks whose prediction was wrong.
enum { PH_STATS = 1, PH_APPLY = 2, PH_ALL = 3, PH_INTO = 4 };

bool same_buffer(const void *a, const void *b) { return a != nullptr && a == b; }

int adam_run(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp, void *workspace,
             size_t ws_bytes, void *stream, int phases, const fp8_adam_dest *dest = nullptr,
             const fp8_adam_grad_cast *gc = nullptr) {
  if (((phases & PH_INTO) != 0) != (dest != nullptr)) return FP8_ERR_INVALID_ARG;
  int g_log2mu = 0;
  if (gc) {  // the gradient cast in the pass: the whole out-of-place step only
    if (phases != (PH_INTO | PH_ALL) || !gc->amax || !mu_log2(gc->mu, &g_log2mu) || gc->margin < 0 ||
        gc->margin > 64)
      return FP8_ERR_INVALID_ARG;
    for (int i = 0; i < nchunks; i++)
      if (!gc->amax[i]) return FP8_ERR_INVALID_ARG;
  }
  if (!chunks || !hp || nchunks <= 0 || !workspace) return FP8_ERR_INVALID_ARG;
  if (ws_bytes < fp8_adam_workspace_bytes(nchunks)) return FP8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FP8_ERR_UNALIGNED;
  // eps >= 2^-39: the square root of a binary32-subnormal v_hat (< 2^-126)
  // is below 2^-63, under half an ULP of such an eps, so sqrt(v_hat) + eps
  // rounds to eps and the subnormal's lost precision never reaches the step;
  // eps = 0 would also turn a zero gradient on a zero state into 0/0.
  // eps <= 2^64: sqrt(v_hat) + eps stays below 2^66 (v_hat is a finite
  // float), so its reciprocal, by which the step multiplies, is a normal
  // number with full precision.
  if (!(hp->lr >= 0.0f && hp->lr <= 3.402823466e38f) || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) ||
      !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) || !(hp->eps >= 0x1p-39f && hp->eps <= 0x1p64f) ||
      hp->step < 1 || hp->margin < 0 || hp->margin > 64)
    return FP8_ERR_INVALID_ARG;
  for (int i = 0; i < nchunks; i++) {
    const fp8_adam_chunk &c = chunks[i];
    if (!c.g_inv || !c.m_scale || !c.v_scale || !c.w_scale) return FP8_ERR_INVALID_ARG;
    // the E4M3 copy is asked for by wq_scale; its codes may be NULL only for an empty chunk
    if ((c.wq || c.wq_scale || c.wq_inv) && (!c.wq_scale || !c.wq_inv)) return FP8_ERR_INVALID_ARG;
    if (c.wq_scale && c.n > 0 && !c.wq) return FP8_ERR_INVALID_ARG;
    if ((phases & PH_ALL) != PH_ALL && c.w_amax)
      return FP8_ERR_INVALID_ARG;  // tracking needs the whole step
    if (c.n > 0 && (!c.g || !c.m || !c.v || !c.w)) return FP8_ERR_INVALID_ARG;
    if (c.n > 0 && (!aligned16(c.g) || !aligned16(c.m) || !aligned16(c.v) || !aligned16(c.w) ||
                    (c.wq && !aligned16(c.wq))))
      return FP8_ERR_UNALIGNED;
    if (dest && c.n > 0) {
      const fp8_adam_dest &o = dest[i];
      if (!o.m || !o.v || !o.w) return FP8_ERR_INVALID_ARG;
      // the inputs must survive the first pass: no new buffer may be an old one
      if (same_buffer(o.m, c.m) || same_buffer(o.v, c.v) || same_buffer(o.w, c.w) ||
          same_buffer(o.m, c.g) || same_buffer(o.m, c.wq))
        return FP8_ERR_INVALID_ARG;
      if (!aligned16(o.m) || !aligned16(o.v) || !aligned16(o.w)) return FP8_ERR_UNALIGNED;
    }
  }
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((phases & PH_STATS) &&
      (rc = cuda_rc(cudaMemsetAsync(workspace, 0, fp8_adam_workspace_bytes(nchunks), s))))
    return rc;

  static thread_local AdamLaunch L;  // ~30 KB: kept off the stack
  L.margin = hp->margin;
  L.beta1 = hp->beta1;
  L.beta2 = hp->beta2;
  L.eps = hp->eps;
  L.neg_lr_bc1 = (float)(-(double)hp->lr / (1.0 - pow((double)hp->beta1, (double)hp->step)));
  L.inv_bc2 = (float)(1.0 / (1.0 - pow((double)hp->beta2, (double)hp->step)));
  // the whole step decides master scales from intervals (exact pass for the
  // chunks whose interval is ambiguous); the phased step reduces the exact
  // amaxes over ranks between its two calls
  L.estimate = phases == PH_ALL ? 1 : 0;
  L.g_hp = gc ? 1 : 0;
  L.g_margin = gc ? gc->margin : 0;
  L.g_log2mu = g_log2mu;
  const unsigned cap = (unsigned)(d->sms * d->adam_blocks_per_sm);
  const unsigned cap1 = (unsigned)(d->sms * d->adam_stats_blocks_per_sm);
  const unsigned cap4 = (unsigned)(d->sms * d->adam_bound_blocks_per_sm);
  const unsigned cap5 = (unsigned)(d->sms * d->adam_est_blocks_per_sm);
  const unsigned cap6 = (unsigned)(d->sms * (gc ? d->adam_castg_blocks_per_sm : d->adam_into_blocks_per_sm));
  for (int first = 0; first < nchunks; first += kAdamMaxChunksPerLaunch) {
    const int cnt = nchunks - first < kAdamMaxChunksPerLaunch ? nchunks - first : kAdamMaxChunksPerLaunch;
    unsigned long long tiles = 0;
    for (int i = 0; i < cnt; i++) {
      const fp8_adam_chunk &c = chunks[first + i];
      AdamChunkDev &e = L.c[i];
      e.g = c.g; e.g_inv = c.g_inv; e.m = c.m; e.m_scale = c.m_scale;
      e.v = c.v; e.v_scale = c.v_scale; e.w = c.w; e.w_scale = c.w_scale;
      e.w_amax = c.w_amax; e.wq = c.wq; e.wq_scale = c.wq_scale; e.wq_inv = c.wq_inv;
      if (dest) {
        e.m_out = dest[first + i].m; e.v_out = dest[first + i].v; e.w_out = dest[first + i].w;
      } else {
        e.m_out = c.m; e.v_out = c.v; e.w_out = c.w;
      }
      e.g_amax = gc ? gc->amax[first + i] : nullptr;
      e.n = c.n;
      e.tile_begin = tiles;
      tiles += (c.n + kAdamTile - 1) / kAdamTile;
    }
    L.nchunks = cnt;
    L.total_tiles = tiles;
    L.ws = reinterpret_cast<float *>(workspace) + (size_t)first * kAdamWsFloatsPerChunk;
    const unsigned grid = tiles == 0 ? 1u : (unsigned)(tiles < cap ? tiles : cap);
    const unsigned grid1 = tiles == 0 ? 1u : (unsigned)(tiles < cap1 ? tiles : cap1);
    const unsigned grid4 = tiles == 0 ? 1u : (unsigned)(tiles < cap4 ? tiles : cap4);
    const unsigned grid5 = tiles == 0 ? 1u : (unsigned)(tiles < cap5 ? tiles : cap5);
    const unsigned grid6 = tiles == 0 ? 1u : (unsigned)(tiles < cap6 ? tiles : cap6);
    bool tracked = false;
    for (int i = 0; i < cnt; i++) tracked |= L.c[i].w_amax != nullptr;
    if (phases & PH_INTO) {
      if (phases & PH_STATS) {  // update with the predicted scales
        if (gc) k_adam<8><<<grid6, kAdamThreads, 0, s>>>(L);
        else    k_adam<6><<<grid6, kAdamThreads, 0, s>>>(L);
      }
      if (phases & PH_APPLY) {
        k_adam_finalize<6><<<1, 256, 0, s>>>(L);       // the right scales; wrong predictions flagged
        if (gc) k_adam<9><<<grid6, kAdamThreads, 0, s>>>(L);   // flagged chunks again, from the inputs
        else    k_adam<7><<<grid6, kAdamThreads, 0, s>>>(L);
        k_adam_finalize<7><<<1, 256, 0, s>>>(L);
      }
    } else if (phases & PH_STATS) {
      // stats of the chunks without a known tracked amax (whether a tracking
      // chunk's amax is known yet is only visible on the device): estimated
      // (whole step) or exact (phased step); those with one: estimated
      if (L.estimate) k_adam<5><<<grid5, kAdamThreads, 0, s>>>(L);
      else            k_adam<1><<<grid1, kAdamThreads, 0, s>>>(L);
      if (tracked) k_adam<4><<<grid4, kAdamThreads, 0, s>>>(L);
    }
    if (phases == PH_ALL) {  // in place, whole step
      k_adam_finalize<1><<<1, 256, 0, s>>>(L);
      k_adam<3><<<grid1, kAdamThreads, 0, s>>>(L);  // exact master amax, flagged chunks only
      k_adam_finalize<2><<<1, 256, 0, s>>>(L);
      k_adam<2><<<grid, kAdamThreads, 0, s>>>(L);    // update
      k_adam_finalize<3><<<1, 256, 0, s>>>(L);       // check of the decided scales; tracked amax
    } else if (phases == PH_APPLY) {
      k_adam_finalize<12><<<1, 256, 0, s>>>(L);
      k_adam<2><<<grid, kAdamThreads, 0, s>>>(L);    // update
    }
    if ((rc = launch_rc())) return rc;
  }
  return FP8_OK;
}

}  // namespace

extern "C" {

int fp8_adam_step(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                  void *workspace, size_t ws_bytes, void *stream) {
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_ALL);
}

int fp8_adam_step_into(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest, int nchunks,
                       const fp8_adam_hparams *hp, void *workspace, size_t ws_bytes, void *stream) {
  if (!dest) return FP8_ERR_INVALID_ARG;
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_INTO | PH_ALL, dest);
}

int fp8_adam_step_into_castgrad(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest,
                                const fp8_adam_grad_cast *gc, int nchunks, const fp8_adam_hparams *hp,
                                void *workspace, size_t ws_bytes, void *stream) {
  if (!dest || !gc) return FP8_ERR_INVALID_ARG;
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_INTO | PH_ALL, dest, gc);
}

int fp8_adam_stats_into(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest, int nchunks,
                        const fp8_adam_hparams *hp, void *workspace, size_t ws_bytes, void *stream) {
  if (!dest) return FP8_ERR_INVALID_ARG;
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_INTO | PH_STATS, dest);
}

int fp8_adam_apply_into(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest, int nchunks,
                        const fp8_adam_hparams *hp, void *workspace, size_t ws_bytes, void *stream) {
  if (!dest) return FP8_ERR_INVALID_ARG;
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_INTO | PH_APPLY, dest);
}

int fp8_adam_stats(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                   void *workspace, size_t ws_bytes, void *stream) {
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_STATS);
}

int fp8_adam_apply(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                   void *workspace, size_t ws_bytes, void *stream) {
  return adam_run(chunks, nchunks, hp, workspace, ws_bytes, stream, PH_APPLY);
}

// Scratch of fp8_adam_step_noalloc: one 64-byte slot per chunk, in a fixed
// array so the call needs no memory from the caller.  Host code must not use
// the array's name as an address (on the host it is only a stand-in); each
// device's real address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) float
    g_adam_noalloc_scratch[FP8_ADAM_NOALLOC_MAX_CHUNKS * kAdamWsFloatsPerChunk];
static void *g_noalloc_addr[kMaxDevices];

static int noalloc_scratch(void **out) {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_adam_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FP8_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FP8_OK;
}

int fp8_adam_step_noalloc(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                          void *stream) {
  if (nchunks <= 0 || nchunks > FP8_ADAM_NOALLOC_MAX_CHUNKS) return FP8_ERR_INVALID_ARG;
  void *scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  return fp8_adam_step(chunks, nchunks, hp, scratch,
                       (size_t)FP8_ADAM_NOALLOC_MAX_CHUNKS * kAdamWsFloatsPerChunk * sizeof(float), stream);
}

int fp8_selftest_wait_timeout(unsigned limit_us, void *stream) {
  if (limit_us == 0 || limit_us > 1000000u) return FP8_ERR_INVALID_ARG;
  gemm::k_wait_selftest<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)limit_us * 1000ull);
  return launch_rc();
}

int fp8_selftest_step_reciprocal(unsigned lo_bits, unsigned long long hi_bits, unsigned long long *bad_dev,
                                 unsigned *first_dev, void *stream) {
  if (hi_bits > 0x100000000ull || lo_bits >= hi_bits || !bad_dev || !first_dev) return FP8_ERR_INVALID_ARG;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  k_step_reciprocal_selftest<<<d->sms * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(lo_bits, hi_bits,
                                                                                        bad_dev, first_dev);
  return launch_rc();
}

int fp8_selftest_encode(int fmt, unsigned lo_bits, unsigned long long hi_bits, unsigned long long *bad_dev,
                        unsigned *first_dev, void *stream) {
  if ((fmt != FP8_E4M3 && fmt != FP8_E5M2) || hi_bits > 0x100000000ull || lo_bits >= hi_bits || !bad_dev ||
      !first_dev)
    return FP8_ERR_INVALID_ARG;
  DeviceInfo *d;
  int rc = device_info(&d);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fmt == FP8_E4M3)
    k_encode_selftest<FP8_E4M3><<<d->sms * 8, 256, 0, s>>>(lo_bits, hi_bits, bad_dev, first_dev);
  else
    k_encode_selftest<FP8_E5M2><<<d->sms * 8, 256, 0, s>>>(lo_bits, hi_bits, bad_dev, first_dev);
  return launch_rc();
}

int fp8_get_status(unsigned *host_out, void *stream) {
  if (!host_out) return FP8_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned v = 0;
  k_take_status<<<1, 1, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return FP8_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FP8_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP8_ERR_CUDA;
  *host_out = v;
  return FP8_OK;
}

const char *fp8_strerror(int code) {
  switch (code) {
    case FP8_OK: return "ok";
    case FP8_ERR_INVALID_ARG: return "invalid argument";
    case FP8_ERR_UNALIGNED: return "pointer not 16-byte aligned";
    case FP8_ERR_UNSUPPORTED: return "unsupported shape (GEMM dims must be multiples of 16)";
    case FP8_ERR_CUDA: return "CUDA error";
    case FP8_ERR_TIMEOUT: return "device pipeline wait timed out";
    case FP8_ERR_NONFINITE: return "non-finite amax";
    default: return "unknown status";
  }
}

}  // extern "C"
