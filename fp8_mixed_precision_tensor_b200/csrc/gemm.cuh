// gemm.cuh -- FP8 x FP8 -> FP32 GEMM on the 5th-generation tensor cores
// (tcgen05.mma kind::f8f6f4, accumulator in TMEM, operands staged by TMA).
//
// "Training and inference of large language models using 8-bit floating
// point", 제안 방법: the linear layer multiplies FP8 operands (E4M3 weights
// and activations, E5M2 gradients) and the per-tensor scaling is undone after
// the matmul; "FP8-LM: Training FP8 Large Language Models", 新規性: FP8 in the
// linear-layer GEMMs (forward, dgrad, wgrad).
//
// One kernel serves all three products.  The output is C[rows, cols] =
// sum_k A(r, k) B(c, k), with each operand either K-major (the reduction
// index is contiguous in memory) or MN-major (the output index is
// contiguous): fwd reads X and W K-major; dgrad reads dY K-major and W
// MN-major; wgrad reads dY and X MN-major.  No operand is ever transposed in
// memory: the MN-major forms are legal tcgen05 operands for 8-bit types.
//
// Structure (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0      TMA producer: 128 x 128-byte tiles of A and BN x 128-byte
//               tiles of B into a STAGES-deep shared-memory ring (128-byte
//               swizzle), completion tracked by mbarriers.
//   warp 1      allocates TMEM (two BN-column fp32 accumulators) and issues
//               tcgen05.mma from one thread; tcgen05.commit frees ring slots
//               and hands finished accumulators to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes, descale by the
//               two inverse scales, + bias, round to the output type, store,
//               and reduce the amax of the stored values (one atomicMax per
//               warp and tile).  Double-buffered TMEM lets tile i's epilogue
//               overlap tile i+1's MMAs.
// Every mbarrier wait is bounded (wall clock, %globaltimer): on timeout the
// kernel raises FP8_STATUS_TIMEOUT, lets in-flight copies and MMAs finish,
// frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "pipeline.cuh"

namespace fp8lib {
namespace gemm {

constexpr int BM = 128;            // tile rows (TMEM lanes)
constexpr int BK = 128;            // k per stage: 128 one-byte elements = one 128B swizzle row
constexpr int UMMA_K = 32;         // k per tcgen05.mma for 8-bit inputs
constexpr int kThreads = 192;      // 6 warps

template <int BN>
struct Cfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
};

struct Args {
  int rows, cols, K;           // output [rows, cols], reduction length K
  int num_m_blocks, num_n_blocks, num_tiles, num_k_blocks;
  int group_m;                 // tile order: groups of group_m row blocks, columns inside
  uint32_t idesc;              // tcgen05 instruction descriptor
  const float *inv_a, *inv_b;  // descale factors (device scalars)
  const void *bias;            // [cols] or null
  int bias_dtype;
  void *out;                   // row-major [rows, cols]
  int out_dtype;
  float *out_amax;             // amax of the stored output (pre-zeroed) or null
};

// ---------------------------------------------------------------------------
// PTX wrappers (the mbarrier and timer helpers are in pipeline.cuh).
// Self-test of the wait above: one thread waits on a barrier that nothing
// arrives at, with a short limit, and must come back with the timeout status
// raised (the GEMMs' abort path starts from exactly this return).
__global__ void k_wait_selftest(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  abort_flag = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  mbar_wait_for(b, 0, &abort_flag, limit_ns);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Wait for a filled operand stage: one inline test first (the stage is
// usually ready), the bounded wait only on a miss.  No tcgen05 fence follows:
// the stage was written by TMA (the async proxy) and completed on this
// mbarrier, which already orders it before the MMAs that read it.  Dropping
// the per-k-block tcgen05.fence::after_thread_sync and testing inline first
// shortened the wide kernel's mainloop by ~10 % (stage waits per tile
// 6.3 -> 2.4 us at K = 4096).
__device__ __forceinline__ bool stage_ready(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
  return mbar_try_wait(bar, parity) || mbar_wait(bar, parity, abort_flag);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets row
// (lane base + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Descriptor of the k-th 32-deep slice of an operand tile.
//   K-major tile: rows of 128 bytes (the k extent), 8-row groups 1024 B apart;
//     the slice starts 32 bytes further along each row.
//   MN-major tile: 128-byte-wide columns of the MN extent (one per 128
//     outputs), each holding BK rows of k; 8-row groups of k 1024 B apart,
//     neighbouring 128-wide MN chunks BK*128 bytes apart; the slice starts
//     32 rows (4096 B) further down.
template <bool MN_MAJOR>
__device__ __forceinline__ uint64_t operand_desc(uint32_t tile_base, int kslice) {
  if constexpr (MN_MAJOR)
    return smem_desc(tile_base + kslice * (UMMA_K * 128), BK * 128, 1024);
  else
    return smem_desc(tile_base + kslice * UMMA_K, 16, 1024);
}

__device__ __forceinline__ float load_bias(const void *bias, int dt, int c) {
  if (dt == FP8_DT_F32) return reinterpret_cast<const float *>(bias)[c];
  uint32_t h = reinterpret_cast<const uint16_t *>(bias)[c];
  if (dt == FP8_DT_BF16) return __uint_as_float(h << 16);
  return __half2float(__ushort_as_half((unsigned short)h));
}

// Tile order: walk the output in bands of group_m row blocks, column-major
// inside a band, so the CTAs running at the same time share a compact block
// of A rows and B columns in L2.
__device__ __forceinline__ void tile_coords(int t, const Args &a, int &mb, int &nb) {
  const int per_band = a.group_m * a.num_n_blocks;
  const int band = t / per_band;
  const int first = band * a.group_m;
  const int rows_in_band = min(a.num_m_blocks - first, a.group_m);
  const int r = t - band * per_band;
  mb = first + r % rows_in_band;
  nb = r / rows_in_band;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory word in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on a barrier of the peer CTA.  Relaxed: every use hands over a
// resource (a TMEM accumulator whose tcgen05.ld have completed, a ring slot
// whose MMAs have completed) that the arriving thread did not write through
// generic memory, so no release ordering is needed; a release.cluster arrive
// measured about 1.2 us per hand-over on B200, a relaxed one the same as a
// local arrive.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA load whose completion is counted on a barrier that may live in the
// peer CTA of the pair (cta_group::2 form; no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                                 uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(cluster_bar)
      : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Pair MMAs that share their A operand through the tensor core's collector
// buffer: `fill` reads A from shared memory and keeps it, `lastuse` takes A
// from the buffer (its descriptor is not read again) and releases it.
__device__ __forceinline__ void tc_mma_pair_fill_a(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4.collector::a::fill [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair_lastuse_a(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                      uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once every
// tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void sleep_ns_bounded(uint32_t total_ns) {
  uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < total_ns) __nanosleep(1000);
}

// Bulk tensor store of a 128B-swizzled shared-memory box to global memory
// (bulk async-group completion; no mbarrier).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Descale (+ bias) 32 accumulator columns of one row in place; columns at or
// beyond `cols` are left as they are (zero: their B rows were zero-filled).
// The bias test stays outside the element loop: testing it per element made
// the wide kernel's epilogue about 14 % of its time at K = 4096.
__device__ __forceinline__ void descale_chunk(const Args &args, uint32_t (&r)[32], int col0, float inv_a,
                                              float inv_b) {
  if (args.bias == nullptr) {
#pragma unroll
    for (int j = 0; j < 32; j++) r[j] = __float_as_uint(__fmul_rn(__fmul_rn(__uint_as_float(r[j]), inv_a), inv_b));
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; j++) {
    float y = __fmul_rn(__fmul_rn(__uint_as_float(r[j]), inv_a), inv_b);
    if (col0 + j < args.cols) y = __fadd_rn(y, load_bias(args.bias, args.bias_dtype, col0 + j));
    r[j] = __float_as_uint(y);
  }
}

// descale_chunk with the two descales folded into one factor inv_ab =
// inv_a * inv_b (both powers of two, so the product is exact whenever it is a
// normal float, and x * inv_ab rounds no worse than two multiplications).
__device__ __forceinline__ void descale1_chunk(const Args &args, uint32_t (&r)[32], int col0, float inv_ab) {
  if (args.bias == nullptr) {
#pragma unroll
    for (int j = 0; j < 32; j++) r[j] = __float_as_uint(__fmul_rn(__uint_as_float(r[j]), inv_ab));
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; j++) {
    float y = __fmul_rn(__uint_as_float(r[j]), inv_ab);
    if (col0 + j < args.cols) y = __fadd_rn(y, load_bias(args.bias, args.bias_dtype, col0 + j));
    r[j] = __float_as_uint(y);
  }
}

// Two floats as bfloat16 rounded to odd: truncate, then set the last bit when
// any of the 16 discarded bits was set (a NaN whose payload sits in the low
// bits stays a NaN; +-0 and +-inf are exact).
__device__ __forceinline__ uint32_t bf16x2_rto(float a, float b) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  const uint32_t sticky = ((ua & 0xffffu) != 0u ? 1u : 0u) | ((ub & 0xffffu) != 0u ? 0x10000u : 0u);
  return __byte_perm(ua, ub, 0x7632) | sticky;
}

// Epilogue of one 32-column chunk: descale, bias, round, store, amax.
__device__ __forceinline__ uint32_t store_chunk(const Args &args, const uint32_t (&r)[32], int row, int col0,
                                                float inv_a, float inv_b) {
  const bool row_ok = row < args.rows;
  uint32_t amax_bits = 0;
  float y[32];
#pragma unroll
  for (int j = 0; j < 32; j++) y[j] = __fmul_rn(__fmul_rn(__uint_as_float(r[j]), inv_a), inv_b);
  if (args.bias != nullptr) {
#pragma unroll
    for (int j = 0; j < 32; j++)
      if (col0 + j < args.cols) y[j] = __fadd_rn(y[j], load_bias(args.bias, args.bias_dtype, col0 + j));
  }
  if (args.out_dtype == FP8_DT_F32) {
    float *orow = reinterpret_cast<float *>(args.out) + (size_t)row * args.cols;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      if (row_ok && col0 + j < args.cols) {
        *reinterpret_cast<float4 *>(orow + col0 + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
        amax_bits = max(amax_bits, max(max(absbits_f32(y[j]), absbits_f32(y[j + 1])),
                                       max(absbits_f32(y[j + 2]), absbits_f32(y[j + 3]))));
      }
    }
  } else {
    uint16_t *orow = reinterpret_cast<uint16_t *>(args.out) + (size_t)row * args.cols;
    const bool rto = args.out_dtype == FP8_DT_BF16_RTO;
    const bool bf = args.out_dtype == FP8_DT_BF16 || rto;
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint32_t p[4];
      uint32_t mx = 0;
#pragma unroll
      for (int t = 0; t < 4; t++) {
        uint32_t lo, hi;
        if (bf) {
          if (rto) {
            p[t] = bf16x2_rto(y[j + 2 * t], y[j + 2 * t + 1]);
          } else {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(y[j + 2 * t], y[j + 2 * t + 1]);
            p[t] = *reinterpret_cast<uint32_t *>(&h2);
          }
          lo = (p[t] & 0x7fffu) << 16;
          hi = p[t] & 0x7fff0000u;
        } else {
          p[t] = f16x2(y[j + 2 * t], y[j + 2 * t + 1]);
          float2 back = h2f2(p[t]);
          lo = absbits_f32(back.x);
          hi = absbits_f32(back.y);
        }
        mx = max(mx, max(lo, hi));
      }
      if (row_ok && col0 + j < args.cols) {
        *reinterpret_cast<uint4 *>(orow + col0 + j) = make_uint4(p[0], p[1], p[2], p[3]);
        amax_bits = max(amax_bits, mx);
      }
    }
  }
  return amax_bits;
}

// ---------------------------------------------------------------------------
template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const Args args) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-aligned for the 128B swizzle
  uint8_t *base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + C::STAGES * C::STAGE_BYTES;
  // barrier layout: full[S], empty[S], tfull[2], tempty[2], drain, then tmem slot + abort flag
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::STAGES + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + C::STAGES * C::STAGE_BYTES + 8 * (2 * C::STAGES + 5));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; s++) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);  // one arrive per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (one thread)
    // The loop runs in one thread with no warp-wide step per k-block, as the
    // MMA issuer's does: a warp-synchronous loop (lane 0 waits, the warp
    // re-converges on a shuffle) held the wide kernel's operand feed to about
    // 60 % of what this loop streams.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      // parity of the last load issued into each stage (for the abort drain)
      uint32_t issued_mask = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < args.num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + stage * C::STAGE_BYTES, sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
          if (A_MN) tma_load_2d(sa, &tmA, mb * BM, kb * BK, full_bar(stage));
          else      tma_load_2d(sa, &tmA, kb * BK, mb * BM, full_bar(stage));
          if (B_MN) {
#pragma unroll
            for (int h = 0; h < BN / 128; h++)
              tma_load_2d(sb + h * (128 * BK), &tmB, nb * BN + h * 128, kb * BK, full_bar(stage));
          } else {
            tma_load_2d(sb, &tmB, kb * BK, nb * BN, full_bar(stage));
          }
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let every issued copy land before the CTA can exit
        for (int s = 0; s < C::STAGES; s++)
          if (issued_mask & (1u << s)) mbar_wait_drain(full_bar(s), (issued_par >> s) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one thread)
    // Descriptors advance by constant adds, as in k_gemm3's issuer.
    if (lane == 0) {
      const uint64_t a_d0 = operand_desc<A_MN>(base, 0);
      const uint64_t b_d0 = operand_desc<B_MN>(base + C::A_BYTES, 0);
      constexpr uint64_t a_ks = A_MN ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
      constexpr uint64_t b_ks = B_MN ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
      constexpr uint64_t st_d = C::STAGE_BYTES >> 4;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, issued_any = false;
      for (int tile = blockIdx.x; tile < args.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!stage_ready(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          const uint64_t so = (uint64_t)stage * st_d;
#pragma unroll
          for (int ks = 0; ks < BK / UMMA_K; ks++)
            tc_mma(d_tmem, a_d0 + so + ks * a_ks, b_d0 + so + ks * b_ks, args.idesc, (kb | ks) != 0 ? 1u : 0u);
          tc_commit(empty_bar(stage));  // ring slot free once these MMAs have read it
          issued_any = true;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));  // accumulator complete
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);  // arrives once every MMA issued so far has completed
        mbar_wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const float inv_a = *args.inv_a, inv_b = *args.inv_b;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, args, mb, nb);
      // every lane waits (no divergent call); a lane whose wait ran out stops the warp
      const bool got = __all_sync(0xffffffffu, mbar_wait(tfull_bar(acc), acc_phase, abort_flag));
      if (!got) break;
      tc_fence_after();
      const int row = mb * BM + q * 32 + lane;
      uint32_t amax_bits = 0;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; cc++) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + cc * 32, r);
        amax_bits = max(amax_bits, store_chunk(args, r, row, nb * BN + cc * 32, inv_a, inv_b));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (args.out_amax != nullptr) {
        amax_bits = warp_max_u32(amax_bits);
        if (lane == 0) atomic_max_bits(args.out_amax, amax_bits);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}


// ---------------------------------------------------------------------------
// Pair kernel: a cluster of two CTAs on two SMs computes 256 x 256 output
// tiles with tcgen05.mma.cta_group::2 (M = 256, N = 256).  Each CTA loads its
// own 128 rows of A and its own 128 columns of B (32 KB per stage, 6 stages),
// so every SM streams half the B bytes of the one-CTA kernel for the same
// tensor-core work.  The even CTA (the leader) counts both CTAs' TMA bytes on
// its "full" barriers and issues the MMAs, which read A and B from both
// CTAs' shared memory and write each CTA's 128 accumulator rows into that
// CTA's TMEM.  Commits are multicast to the same barrier in both CTAs; the
// epilogue warps of both CTAs return the accumulator to the leader with a
// remote arrive.  No TMA load is multicast.  Launched as clusters of two
// CTAs (cudaLaunchAttributeClusterDimension = 2).
constexpr int kPairBN = 256;     // output columns per pair tile
constexpr int kPairHalf = 128;   // rows (and B columns) held by one CTA
constexpr int kPairStages = 6;
constexpr int kPairStageBytes = 2 * kPairHalf * BK;  // A 16 KB + B 16 KB
constexpr int kPairTmemCols = 2 * kPairBN;
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + 256 + 1024;

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const Args args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + kPairStages * kPairStageBytes;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kPairStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kPairStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kPairStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kPairStages + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + kPairStages * kPairStageBytes + 8 * (2 * kPairStages + 5));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; s++) {
      mbar_init(full_bar(s), 1);   // leader: its producer's arrive + both CTAs' bytes
      mbar_init(empty_bar(s), 1);  // one multicast commit per phase
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 8);  // leader: 4 epilogue warps x 2 CTAs
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)kPairTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs, one thread)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int tile = pair; tile < args.num_tiles && ok; tile += num_pairs) {
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        const int arow = mb * (2 * kPairHalf) + (int)rank * kPairHalf;
        const int bcol = nb * kPairBN + (int)rank * kPairHalf;
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + stage * kPairStageBytes, sb = sa + kPairHalf * BK;
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * kPairStageBytes);
          if (A_MN) tma_load_2d_pair(sa, &tmA, arow, kb * BK, fb);
          else      tma_load_2d_pair(sa, &tmA, kb * BK, arow, fb);
          if (B_MN) tma_load_2d_pair(sb, &tmB, bcol, kb * BK, fb);
          else      tma_load_2d_pair(sb, &tmB, kb * BK, bcol, fb);
          issued = true;
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && issued) sleep_ns_bounded(50000);  // let copies in flight land
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader, one thread)
    // Descriptors advance by constant adds, as in k_gemm3's issuer.
    if (leader && lane == 0) {
      const uint64_t a_d0 = operand_desc<A_MN>(base, 0);
      const uint64_t b_d0 = operand_desc<B_MN>(base + kPairHalf * BK, 0);
      constexpr uint64_t a_ks = A_MN ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
      constexpr uint64_t b_ks = B_MN ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
      constexpr uint64_t st_d = kPairStageBytes >> 4;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, issued_any = false;
      for (int tile = pair; tile < args.num_tiles && ok; tile += num_pairs) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kPairBN;
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!stage_ready(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          const uint64_t so = (uint64_t)stage * st_d;
#pragma unroll
          for (int ks = 0; ks < BK / UMMA_K; ks++)
            tc_mma_pair(d_tmem, a_d0 + so + ks * a_ks, b_d0 + so + ks * b_ks, args.idesc, (kb | ks) != 0 ? 1u : 0u);
          tc_commit_pair(empty_bar(stage));
          issued_any = true;
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && issued_any) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(drain_bar)
                     : "memory");
        mbar_wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const float inv_a = *args.inv_a, inv_b = *args.inv_b;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < args.num_tiles; tile += num_pairs) {
      int mb, nb;
      tile_coords(tile, args, mb, nb);
      // every lane waits (no divergent call); a lane whose wait ran out stops the warp
      const bool got = __all_sync(0xffffffffu, mbar_wait(tfull_bar(acc), acc_phase, abort_flag));
      if (!got) break;
      tc_fence_after();
      const int row = mb * (2 * kPairHalf) + (int)rank * kPairHalf + q * 32 + lane;
      uint32_t amax_bits = 0;
#pragma unroll 1
      for (int cc = 0; cc < kPairBN / 32; cc++) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * kPairBN + cc * 32, r);
        amax_bits = max(amax_bits, store_chunk(args, r, row, nb * kPairBN + cc * 32, inv_a, inv_b));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(tempty_bar(acc), 0));
      if (args.out_amax != nullptr) {
        amax_bits = warp_max_u32(amax_bits);
        if (lane == 0) atomic_max_bits(args.out_amax, amax_bits);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();  // the leader's MMAs no longer read this CTA's smem / TMEM
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)kPairTmemCols)
                 : "memory");
  }
}


// ---------------------------------------------------------------------------
// Wide pair kernel: a cluster of two CTAs computes 256 x 512 output tiles.
// Per k-slice the leader issues two tcgen05.mma.cta_group::2 (M = 256,
// N = 256), one into each of two accumulators that together fill all 512
// TMEM columns.  Each CTA loads its 128 rows of A (16 KB) and 256 rows of B
// (32 KB) per stage into a 3-stage ring: the same A tile feeds twice the
// tensor-core work, so each SM streams 48 KB per 2 x 128x256x128 MACs
// instead of 32 KB per one.  Column bookkeeping: CTA r holds B rows (output
// columns) [r*256, r*256+256) of the tile; the MMA reading B rows [0,128) of
// both CTAs produces tile columns {0..127, 256..383} in accumulator 0, and
// rows [128,256) produce {128..255, 384..511} in accumulator 1.  There is no
// room left in TMEM for a second tile, so the epilogue runs between tiles
// while the producer already refills the ring; it hands the accumulator back
// right after its last TMEM read and drains its staged output with pipelined
// bulk stores (two staging boxes per epilogue warp).  The MMAs' commits free
// the leader's ring slots; a relay warp frees the follower's copy of each
// slot with a remote arrive once the leader's slot is free.  Warps: 0
// producer (both CTAs), 1 TMEM allocation and MMA issue (leader), 2-9
// epilogue (both CTAs), 10 release relay (leader).
constexpr int kWideBN = 512;
constexpr int kWideStages = 3;
constexpr int kWideStageBytes = kPairHalf * BK + 2 * kPairHalf * BK;  // A 16 KB + B 32 KB
constexpr int kWideThreads = 352;                                     // 11 warps
constexpr int kWideStageOutBytes = 32 * 128;                             // per epilogue warp: 32 rows x 128 B
constexpr int kWideOutBoxes = 2;  // staging boxes per epilogue warp (stores pipelined)
constexpr int kWideSmemBytes = kWideStages * kWideStageBytes + 8 * kWideOutBoxes * kWideStageOutBytes + 256 + 1024;

// OUT: the output type (FP8_DT_*), a template argument so that the
// epilogue's element loop carries no type test.
template <bool A_MN, bool B_MN, int OUT>
__global__ void __launch_bounds__(kWideThreads, 1)
    k_gemm3(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmOut, const Args args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (base - raw);
  const uint32_t out_stage0 = base + kWideStages * kWideStageBytes;  // 8 x 2 x 4 KB, 1024-aligned
  const uint32_t bar0 = out_stage0 + 8 * kWideOutBoxes * kWideStageOutBytes;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kWideStages + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * kWideStages);
  const uint32_t tempty_bar = bar0 + 8u * (2 * kWideStages + 1);
  const uint32_t drain_bar = bar0 + 8u * (2 * kWideStages + 2);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_ptr + (bar0 - base) + 8 * (2 * kWideStages + 3));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWideStages; s++) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 16);  // leader: 8 epilogue warps x 2 CTAs
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs, one thread)
    // One thread runs the loop (no warp-wide step per k-block): the
    // warp-synchronous form streamed a stage every ~1260 SM cycles, this one
    // every ~810, ahead of the tensor core's ~1030.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int tile = pair; tile < args.num_tiles && ok; tile += num_pairs) {
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        const int arow = mb * (2 * kPairHalf) + (int)rank * kPairHalf;
        const int bcol = nb * kWideBN + (int)rank * (2 * kPairHalf);
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = base + stage * kWideStageBytes, sb = sa + kPairHalf * BK;
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * kWideStageBytes);
          if (A_MN) tma_load_2d_pair(sa, &tmA, arow, kb * BK, fb);
          else      tma_load_2d_pair(sa, &tmA, kb * BK, arow, fb);
          if (B_MN) {
            tma_load_2d_pair(sb, &tmB, bcol, kb * BK, fb);
            tma_load_2d_pair(sb + kPairHalf * BK, &tmB, bcol + kPairHalf, kb * BK, fb);
          } else {
            tma_load_2d_pair(sb, &tmB, kb * BK, bcol, fb);  // one box of 256 rows
          }
          issued = true;
          if (++stage == kWideStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && issued) sleep_ns_bounded(50000);  // let copies in flight land
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader, one thread)
    // The whole loop runs in one thread with no warp-wide step per k-block,
    // and the 64-bit operand descriptors advance by constant adds: a k-slice
    // moves the start-address field (address >> 4) by 2 (K-major, 32 B) or
    // 256 (MN-major, 32 rows of 128 B), a stage by kWideStageBytes >> 4, and
    // the field cannot carry (shared addresses stay below 2^18).
    if (leader && lane == 0) {
      const uint64_t a_d0 = operand_desc<A_MN>(base, 0);
      const uint64_t b_d0 = operand_desc<B_MN>(base + kPairHalf * BK, 0);
      const uint64_t b_d1 = operand_desc<B_MN>(base + 2 * kPairHalf * BK, 0);
      constexpr uint64_t a_ks = A_MN ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
      constexpr uint64_t b_ks = B_MN ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
      constexpr uint64_t st_d = kWideStageBytes >> 4;
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, issued_any = false;
      for (int tile = pair; tile < args.num_tiles && ok; tile += num_pairs) {
        if (!mbar_wait(tempty_bar, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!stage_ready(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          const uint64_t so = (uint64_t)stage * st_d;
#pragma unroll
          for (int ks = 0; ks < BK / UMMA_K; ks++) {
            const uint64_t ad = a_d0 + so + ks * a_ks;
            const uint32_t accum = (kb | ks) != 0 ? 1u : 0u;
            // the same A slice feeds both accumulators: read it from shared memory once
            tc_mma_pair_fill_a(tmem_base, ad, b_d0 + so + ks * b_ks, args.idesc, accum);
            tc_mma_pair_lastuse_a(tmem_base + 256, ad, b_d1 + so + ks * b_ks, args.idesc, accum);
          }
          // the leader's own ring slot; the relay warp frees the follower's
          asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           empty_bar(stage))
                       : "memory");
          issued_any = true;
          if (++stage == kWideStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar);
        acc_phase ^= 1u;
      }
      if (!ok && issued_any) {
        asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(drain_bar)
                     : "memory");
        mbar_wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else if (warp == 10) {
    // ------------------------------------------------------------ release relay (leader only)
    // Once the MMAs that read a ring slot have completed (the leader's empty
    // barrier), free the follower's copy of that slot with a relaxed remote
    // arrive: the reads are over before the arrive is issued.
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < args.num_tiles && ok; tile += num_pairs) {
        for (int kb = 0; kb < args.num_k_blocks; kb++) {
          if (!mbar_wait(empty_bar(stage), phase, abort_flag)) { ok = false; break; }
          mbar_arrive_remote(map_to_rank(empty_bar(stage), 1));
          if (++stage == kWideStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps, both CTAs)
    // Each warp drains 32 rows x 256 columns of one accumulator half in
    // 128-byte-wide column blocks: tcgen05.ld -> descale/bias/round -> its own
    // 4 KB staging box in shared memory (128B-swizzled rows) -> one bulk tensor
    // store.  The store clips rows and columns outside the output.
    const int q = warp & 3;         // TMEM lane quarter
    const int h = (warp - 2) >> 2;  // accumulator half: 0 or 1
    const float inv_a = *args.inv_a, inv_b = *args.inv_b;
    const float inv_ab = __fmul_rn(inv_a, inv_b);
    // one multiplication when the folded factor is a normal float
    const bool fold = fabsf(inv_ab) >= 1.17549435e-38f && fabsf(inv_ab) <= 3.402823466e38f;
    const uint32_t stg0 = out_stage0 + (warp - 2) * kWideOutBoxes * kWideStageOutBytes;
    uint32_t box = 0;
    constexpr bool f32out = OUT == FP8_DT_F32;
    constexpr bool rtoout = OUT == FP8_DT_BF16_RTO;
    constexpr bool bfout = OUT == FP8_DT_BF16 || rtoout;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < args.num_tiles; tile += num_pairs) {
      int mb, nb;
      tile_coords(tile, args, mb, nb);
      // every lane waits (no divergent call): measured ~0.8 % faster on the
      // GPT-7B fc1 shape than lane 0 waiting and the warp re-converging on a
      // shuffle; a lane whose wait ran out stops the warp
      const bool got = __all_sync(0xffffffffu, mbar_wait(tfull_bar, acc_phase, abort_flag));
      if (!got) break;
      tc_fence_after();
      const int row0 = mb * (2 * kPairHalf) + (int)rank * kPairHalf + q * 32;
      const bool rows_in = row0 < args.rows;
      uint32_t amax_bits = 0;
      uint32_t amax16 = 0;  // 16-bit outputs: two packed magnitude maxima
      // accumulator column c of half h holds output column
      //   nb*512 + (c < 128 ? 0 : 256) + h*128 + (c mod 128)
      constexpr int cols_per_box = f32out ? 32 : 64;
#pragma unroll 1
      for (int c = 0; c < 256; c += cols_per_box) {
        const int col0 = nb * kWideBN + (c < 128 ? 0 : 256) + h * kPairHalf + (c & 127);
        const bool last = c + cols_per_box >= 256;
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + h * 256 + c, r);
        if (fold) descale1_chunk(args, r, col0, inv_ab); else descale_chunk(args, r, col0, inv_a, inv_b);
        uint32_t w[32];  // the row's 128 bytes as 32 words
        if constexpr (f32out) {
          if (last) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(map_to_rank(tempty_bar, 0));
          }
#pragma unroll
          for (int j = 0; j < 32; j++) {
            w[j] = r[j];
            amax_bits = max(amax_bits, r[j] & 0x7fffffffu);
          }
        } else {
          uint32_t r2[32];
          tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + h * 256 + c + 32, r2);
          if (last) {  // the tile's last TMEM read: hand the accumulator back now
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(map_to_rank(tempty_bar, 0));
          }
          if (fold) descale1_chunk(args, r2, col0 + 32, inv_ab); else descale_chunk(args, r2, col0 + 32, inv_a, inv_b);
#pragma unroll
          for (int j = 0; j < 16; j++) {
            const float a0 = __uint_as_float(r[2 * j]), a1 = __uint_as_float(r[2 * j + 1]);
            const float b0 = __uint_as_float(r2[2 * j]), b1 = __uint_as_float(r2[2 * j + 1]);
            uint32_t pa, pb;
            if constexpr (rtoout) {
              pa = bf16x2_rto(a0, a1);
              pb = bf16x2_rto(b0, b1);
            } else if constexpr (bfout) {
              __nv_bfloat162 x = __floats2bfloat162_rn(a0, a1), y = __floats2bfloat162_rn(b0, b1);
              pa = *reinterpret_cast<uint32_t *>(&x);
              pb = *reinterpret_cast<uint32_t *>(&y);
            } else {
              pa = f16x2(a0, a1);
              pb = f16x2(b0, b1);
            }
            // running max of the stored 16-bit magnitudes, two per word (for
            // both types the magnitude bits order like the values, NaN on top)
            amax16 = __vmaxu2(amax16, __vmaxu2(pa & 0x7fff7fffu, pb & 0x7fff7fffu));
            w[j] = pa;
            w[16 + j] = pb;
          }
        }
        // this staging box must be free: the store that used it two boxes ago
        // has read it (every box commits one bulk group, empty when it stores
        // nothing, so "at most one group pending" means exactly that)
        const uint32_t stg = stg0 + box * kWideStageOutBytes;
        box ^= 1u;
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < 8; ch++) {  // 16-byte chunk ch of this row, 128B swizzle
          const uint32_t addr = stg + lane * 128 + ((ch ^ (lane & 7)) << 4);
          st_shared_v4(addr, w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          if (rows_in && col0 < args.cols) tma_store_2d(&tmOut, stg, col0, row0);
          bulk_commit();
        }
      }
      if constexpr (!f32out) {
        const uint32_t h16 = max(amax16 & 0xffffu, amax16 >> 16);
        amax_bits = bfout ? (h16 << 16) : absbits_f32(__half2float(__ushort_as_half((unsigned short)h16)));
      }
      if (row0 + lane >= args.rows) amax_bits = 0;  // a row past the output (holds only the bias)
      if (args.out_amax != nullptr) {
        amax_bits = warp_max_u32(amax_bits);
        if (lane == 0) atomic_max_bits(args.out_amax, amax_bits);
      }
      acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait0();  // every store has landed before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512u)
                 : "memory");
  }
}

}  // namespace gemm
}  // namespace fp8lib
