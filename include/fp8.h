/*
 * fp8.h -- C ABI of libfp8, the B200 (sm_100a) hot path of FP8 mixed-precision
 * LLM training: per-tensor dynamically scaled FP8 linear layers and the
 * precision-decoupled FP8 Adam step.
 *
 * Sources (by page title and section):
 *   [FP8-AMAX] "Training and inference of large language models using 8-bit
 *              floating point" (paper review), 제안 방법: per-tensor scaling
 *              bias from the amax of each weight, activation and gradient
 *              tensor (log2 of fmt_max / amax with a configurable margin);
 *              scale before the FP8 cast, undo the scaling after the matmul;
 *              E4M3 for weights and activations, E5M2 for gradients.
 *   [FP8-LM]   "FP8-LM: Training FP8 Large Language Models" (paper memo),
 *              提案手法: O1 gradient auto-scaling g' = mu * g (Eq. 3);
 *              O2 Adam with FP8 first moment, FP16 second moment and FP16
 *              master weights with tensor scaling.
 *
 * Conventions shared by every entry point
 *   - Ownership: the caller owns every buffer.  The library allocates and
 *     frees nothing and never synchronises the stream (fp8_get_status is the
 *     one exception and says so).  Every call only enqueues work on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream) and returns.
 *   - "dev" pointers are device memory of the current CUDA device; "host"
 *     pointers are host memory.  Scalars that chain one call into the next
 *     (amax, scale, inverse scale) stay in device memory as float.
 *   - Bulk tensors are dense and contiguous; their pointers must be 16-byte
 *     aligned (FP8_ERR_UNALIGNED otherwise).  Any element count is allowed.
 *   - Errors found on the host are returned at once and nothing is enqueued.
 *     Conditions found on the device (a non-finite amax, a pipeline wait that
 *     ran out of time) set bits of a device status word read by
 *     fp8_get_status.
 */
#ifndef FP8_B200_H
#define FP8_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ----------------------------------------------------- */
#define FP8_OK 0
#define FP8_ERR_INVALID_ARG 1 /* null pointer, bad enum, bad hyper-parameter */
#define FP8_ERR_UNALIGNED 2   /* a bulk pointer is not 16-byte aligned */
#define FP8_ERR_UNSUPPORTED 3 /* a GEMM shape the kernel cannot tile (see below) */
#define FP8_ERR_CUDA 4        /* a CUDA runtime call or kernel launch failed */
#define FP8_ERR_TIMEOUT 5     /* device status: a pipeline wait ran out of time */
#define FP8_ERR_NONFINITE 6   /* device status: an amax was NaN or inf */

/* Device status word bits (fp8_get_status). */
#define FP8_STATUS_NONFINITE 1u
#define FP8_STATUS_TIMEOUT 2u
#define FP8_STATUS_INTERNAL 4u /* a kernel's own consistency check failed */
#define FP8_STATUS_BAD_MU 8u   /* a device mu was not a power of two in [2^-32, 2^32]; 1 was used */

/* ---- element types of high-precision tensors -------------------------- */
#define FP8_DT_F32 0
#define FP8_DT_BF16 1
#define FP8_DT_F16 2
/* GEMM outputs only: bfloat16 rounded to odd (truncated, the last bit set
 * when any discarded bit was set).  An intermediate for a following FP8 cast:
 * bfloat16 keeps 8 significant bits, at least 2 more than E4M3 (4) or E5M2
 * (3) at any scaled magnitude, so rounding to nearest even from the
 * round-to-odd value gives the code the cast of the float32 result would
 * give (round-to-odd is innocuous before a rounding that keeps 2 or more
 * fewer bits), and every power-of-two scale threshold is a bfloat16 value
 * that round-to-odd never crosses, so the amax of the stored values yields
 * the scale of the float32 amax.  Read back as FP8_DT_BF16 (the gradient
 * cast reads 2 instead of 4 bytes per element). */
#define FP8_DT_BF16_RTO 3

/* ---- storage formats ---------------------------------------------------
 * FP8_E4M3: OCP E4M3, max 448, no infinities (weights, activations, Adam m1).
 * FP8_E5M2: OCP E5M2, max 57344 (gradients).
 * FP8_F16S: IEEE binary16 with a per-tensor power-of-two scale, max 65504
 *           ("FP16 with tensor scaling": Adam m2 and master weights). */
#define FP8_E4M3 0
#define FP8_E5M2 1
#define FP8_F16S 2

/*
 * fp8_amax -- amax = max_i |x_i| over n elements, written to *amax_dev as a
 * float ([FP8-AMAX] 제안 방법).  Exact: the maximum is taken over bit
 * patterns.  Any NaN element gives a NaN amax; otherwise any inf gives +inf.
 * n == 0 writes 0.
 *   x        dev, n elements of `dtype`, 16-byte aligned
 *   amax_dev dev, one float, overwritten
 */
int fp8_amax(const void *x, int dtype, size_t n, float *amax_dev, void *stream);

/*
 * fp8_compute_scale -- the per-tensor power-of-two scale of [FP8-AMAX]
 * 제안 방법 with the gradient auto-scaling factor of [FP8-LM] O1 (Eq. 3):
 *     e     = floor(log2(fmt_max / (mu * amax)))   (exact integer arithmetic)
 *     s_g   = 2^(clamp(e - margin, -126, 126))
 *     scale = mu * s_g,   inv_scale = 1 / (mu * s_g).
 * `scale` multiplies the raw tensor before the cast; `inv_scale` undoes it
 * after a GEMM (or when decoding).  amax == 0 gives s_g = 1.  A NaN or inf
 * amax gives s_g = 1 and sets FP8_STATUS_NONFINITE.
 *   amax_dev      dev, one float (typically written by fp8_amax or by a
 *                 GEMM's fused output amax)
 *   fmt           FP8_E4M3 (fmt_max 448), FP8_E5M2 (57344), FP8_F16S (65504)
 *   margin        integer >= 0; each unit halves the scale (headroom)
 *   mu            host float, a power of two in [2^-32, 2^32] (1 = off)
 *   scale_dev, inv_scale_dev  dev, one float each, overwritten
 */
int fp8_compute_scale(const float *amax_dev, int fmt, int margin, float mu, float *scale_dev,
                      float *inv_scale_dev, void *stream);

/*
 * fp8_cast -- q_i = enc_fmt(x_i * scale) ([FP8-AMAX] 제안 방법: scale, then
 * cast).  FP8 formats: round to nearest even, saturating at +-max; +-inf
 * saturates too; NaN becomes 0x7F (its sign is not kept).  FP8_F16S:
 * IEEE round to nearest even; NaN becomes 0x7FFF.  With a scale from
 * fp8_compute_scale on the tensor's own amax nothing saturates.
 *   x          dev, n elements of `dtype`, 16-byte aligned
 *   scale_dev  dev, one float (power of two times mu)
 *   q          dev, n bytes (E4M3/E5M2) or n uint16 (F16S), 16-byte aligned
 */
int fp8_cast(const void *x, int dtype, size_t n, int fmt, const float *scale_dev, void *q,
             void *stream);

/*
 * fp8_scale_cast -- fp8_compute_scale followed by fp8_cast in one launch
 * (same definitions, same results): every block derives the scale from
 * *amax_dev itself and the first block also writes scale_dev and
 * inv_scale_dev.  Arguments as in those two calls; n == 0 only writes the
 * scales.
 */
int fp8_scale_cast(const void *x, int dtype, size_t n, int fmt, const float *amax_dev, int margin,
                   float mu, float *scale_dev, float *inv_scale_dev, void *q, void *stream);

/*
 * fp8_amax_scale_cast -- fp8_amax, then fp8_scale_cast on that amax (same
 * definitions, bit for bit the same amax, scales and codes), reading x once
 * when the scale does not change: *scale_dev holds a predicted scale on entry
 * (the tensor's scale from its previous step; any float), x is cast with it
 * while its amax is reduced, and x is cast a second time, with the scale of
 * the amax, only if that scale differs from the prediction.  Per-tensor
 * scales of activations and gradients change only when the amax crosses a
 * power of two, so most steps take the single pass: 3 instead of 5 bytes of
 * HBM traffic per bf16 element.
 *   amax_dev       dev, one float (out)
 *   scale_dev      dev, one float: the prediction (in), the new scale (out)
 *   inv_scale_dev  dev, one float (out)
 * Other arguments and errors as fp8_scale_cast.
 */
int fp8_amax_scale_cast(const void *x, int dtype, size_t n, int fmt, float *amax_dev, int margin, float mu,
                        float *scale_dev, float *inv_scale_dev, void *q, void *stream);

/*
 * fp8_cast_count -- fp8_cast plus its underflow and overflow counts, the
 * measure by which [FP8-LM] アブレーション研究 compares scaling variants
 * (and [FP8-AMAX] 실험 결과, RQ3, dynamic against constant scaling): an
 * element underflows when it is a non-zero number whose code is zero, and
 * overflows when |x * scale| exceeds fmt_max (the cast saturates it; inf
 * counts, NaN counts as neither).  A constant scaling bias (FP8-CSCALE of
 * [FP8-AMAX]) is this cast with a scale of 2^bias that the caller keeps.
 *   counts_dev  dev, two uint64: [0] += underflows, [1] += overflows
 *               (accumulated; the caller zeroes them)
 * Other arguments as fp8_cast.
 */
int fp8_cast_count(const void *x, int dtype, size_t n, int fmt, const float *scale_dev, void *q,
                   unsigned long long *counts_dev, void *stream);

/*
 * FP8 gradient all-reduce ([FP8-LM] 提案手法 O1: gradients communicated in
 * FP8 with auto-scaling g' = mu * g, Eq. 3).  Every rank casts its gradient
 * with ONE shared scale taken from the amax over all ranks, so that the
 * ranks' codes can be summed as they are; mu sets the headroom the sum
 * needs.  A rank's part of one all-reduce:
 *   amax of its gradient (fp8_amax, or a GEMM's output amax)
 *   <caller> MAX all-reduce of the amax over the ranks
 *   fp8_grad_cast   payload codes with S = mu * 2^(floor(log2(fmt_max/amax)) - margin)
 *   <caller> exchange: rank j receives every rank's codes of its slice j
 *   fp8_sum_codes   exact sum of those codes, re-encoded at S (rank j's
 *                   slice of the summed gradient) and g_inv = 1 / (S * nranks)
 *   <caller> SUM all-reduce of the counts, then fp8_mu_update.
 * With mu = 1 (post-scaling: divide by the rank count after the sum) the
 * sum can saturate; with mu = 1/nranks (pre-scaling: divide before the
 * cast) small gradients underflow; fp8_mu_update moves mu between those.
 */

/*
 * fp8_grad_cast -- the payload cast: S = mu * 2^(clamp(floor(log2(fmt_max /
 * amax)) - margin)), clamped to [2^-126, 2^126]; q_i = enc_fmt(g_i * S).
 * Unlike fp8_compute_scale, mu multiplies the scale after the exponent rule
 * (it does not cancel).  amax == 0 gives the exponent 0; a NaN or inf amax
 * too, and sets FP8_STATUS_NONFINITE.
 *   g              dev, n elements of `dtype`, 16-byte aligned
 *   fmt            FP8_E5M2 (gradients) or FP8_E4M3
 *   amax_dev       dev float: the amax over all ranks
 *   mu_dev         dev float: a power of two in [2^-32, 2^32] (else 1 is used
 *                  and FP8_STATUS_BAD_MU is set)
 *   scale_dev, inv_scale_dev  dev floats, overwritten with S and 1/S
 *   q              dev, n bytes, 16-byte aligned
 *   counts_dev     dev two uint64 (as fp8_cast_count) or NULL
 * n == 0 only writes the scales.
 */
int fp8_grad_cast(const void *g, int dtype, size_t n, int fmt, const float *amax_dev, int margin,
                  const float *mu_dev, float *scale_dev, float *inv_scale_dev, uint8_t *q,
                  unsigned long long *counts_dev, void *stream);

/*
 * fp8_sum_codes -- out_i = enc_fmt(sum_r dec(in[r * ld + i])) for i < n: the
 * ranks' payload codes (all cast at one scale) summed exactly and rounded
 * once (nearest even, saturating at +-fmt_max).  A zero sum is code 0x00; a
 * NaN code, or +inf with -inf, gives 0x7F; an inf saturates.
 *   in             dev, nranks rows of ld bytes (ld >= n, a multiple of 16),
 *                  16-byte aligned; 1 <= nranks <= 4096
 *   out            dev, n bytes, 16-byte aligned
 *   inv_scale_dev  dev float 1/S (read when g_inv_dev is not NULL)
 *   g_inv_dev      dev float or NULL: receives inv_scale * (1 / nranks) (both
 *                  rounded to binary32), the descale of the mean gradient
 *   counts_dev     dev two uint64 (as fp8_cast_count, on the sums) or NULL
 */
int fp8_sum_codes(const uint8_t *in, int nranks, size_t ld, size_t n, int fmt, uint8_t *out,
                  const float *inv_scale_dev, float *g_inv_dev, unsigned long long *counts_dev,
                  void *stream);

/*
 * fp8_mu_update -- the auto-scaling rule for mu between steps ([FP8-LM] O1
 * says mu changes dynamically but gives no rule; this one is the library's
 * own, after dynamic loss scaling): if counts_dev[1] (overflows of the
 * summed gradient, over all ranks) > theta * n, mu halves (not below mu_min)
 * and *clean_dev restarts at 0; otherwise *clean_dev grows by one and at
 * `interval` mu doubles (not above mu_max) and *clean_dev restarts.  Then
 * counts_dev[0..1] are set to 0.  All state stays on the device.
 *   rule   host: theta >= 0, interval >= 1, mu_min <= mu_max powers of two
 *          in [2^-32, 2^32]
 */
typedef struct {
  float theta;
  int interval;
  float mu_min, mu_max;
} fp8_mu_rule;
int fp8_mu_update(float *mu_dev, int *clean_dev, unsigned long long *counts_dev, unsigned long long n,
                  const fp8_mu_rule *rule, void *stream);

/*
 * FP8 linear layer GEMMs ([FP8-AMAX] 제안 방법: matmul on FP8 operands, the
 * scaling undone on the output; [FP8-LM] 新規性: FP8 in the linear layers).
 * Shapes follow nn.Linear: X[M,K], W[N,K], Y[M,N]; all row-major, dense.
 * Every operand is read in place (no transposed copies): dgrad reads W and
 * wgrad reads dY and X along their rows as MN-major tensor-core operands.
 * The epilogue multiplies by the two inverse scales, adds the bias (fwd),
 * rounds to the output type and, when out_amax is not NULL, writes the amax
 * of the output *as stored* (overwritten, not accumulated).
 * Shape rule: M, N, K must each be a multiple of 16 (TMA row pitch);
 * otherwise FP8_ERR_UNSUPPORTED.  M == 0 or N == 0 is a no-op that writes an
 * amax of 0.  Output types: FP8_DT_F32, FP8_DT_BF16, FP8_DT_F16 and
 * FP8_DT_BF16_RTO (bias types: the first three).
 * A mis-tiled pipeline cannot hang: every wait is bounded, and a wait that
 * runs out sets FP8_STATUS_TIMEOUT and the kernel returns.
 */

/* Y[M,N] = (Xq . Wq^T) * x_inv * w_inv (+ bias[N]).
 *   xq  dev [M,K] E4M3,  wq dev [N,K] E4M3,  x_inv/w_inv dev floats
 *   bias dev [N] of bias_dtype or NULL;  y dev [M,N] of y_dtype */
int fp8_linear_fwd(const uint8_t *xq, const float *x_inv, const uint8_t *wq, const float *w_inv,
                   const void *bias, int bias_dtype, void *y, int y_dtype, float *y_amax, int M,
                   int N, int K, void *stream);

/* dX[M,K] = (dYq . Wq) * dy_inv * w_inv.
 *   dyq dev [M,N] E5M2,  wq dev [N,K] E4M3;  dx dev [M,K] of dx_dtype */
int fp8_linear_dgrad(const uint8_t *dyq, const float *dy_inv, const uint8_t *wq,
                     const float *w_inv, void *dx, int dx_dtype, float *dx_amax, int M, int N,
                     int K, void *stream);

/* dW[N,K] = (dYq^T . Xq) * dy_inv * x_inv.
 *   dyq dev [M,N] E5M2,  xq dev [M,K] E4M3;  dw dev [N,K] of dw_dtype */
int fp8_linear_wgrad(const uint8_t *dyq, const float *dy_inv, const uint8_t *xq,
                     const float *x_inv, void *dw, int dw_dtype, float *dw_amax, int M, int N,
                     int K, void *stream);

/*
 * Precision-decoupled FP8 Adam ([FP8-LM] 提案手法 O2): per parameter 6 bytes
 * of state -- FP8 E5M2 gradient (1 B), FP8 E4M3 first moment (1 B), FP16
 * second moment (2 B) and FP16 master weight (2 B) -- each tensor with its
 * own power-of-two scale.  One call updates every chunk (tensor) in place:
 *   g  = dec_E5M2(g) * g_inv                 (g_inv = 1 / (mu * s_g))
 *   m0 = dec_E4M3(m) / m_scale,  v0 = half(v) / v_scale,  w0 = half(w) / w_scale
 *   m  = b1 m0 + (1 - b1) g,     v  = b2 v0 + (1 - b2) g^2
 *   w  = w0 - lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * then new per-chunk scales from the amax of the new m, v, w (same rule as
 * fp8_compute_scale with `margin`, fmt_max 448 / 65504 / 65504) and the state
 * is re-encoded with them; the new scales replace m_scale, v_scale, w_scale.
 * Arithmetic is float32 with every operation rounded to nearest (square root
 * and reciprocal correctly rounded; the quotient multiplies by the
 * reciprocal); a non-finite new amax sets
 * FP8_STATUS_NONFINITE and that scale to 1.
 * Tracked master amax (optional; the first pass then moves 4 instead of 6
 * bytes per parameter): when w_amax points to the exact amax of the
 * dequantised stored master (a value >= 0), the new master amax is bounded by
 * that value -/+ the largest step |w - w0|, and the master is re-read only
 * when the interval holds a scale threshold.  Every step rewrites *w_amax; a
 * negative value means "unknown" (the step re-reads the master).  After
 * changing w or w_scale by other means, set *w_amax to -1.
 * E4M3 master copy (optional; the next forward pass's weight cast fused into
 * the update): when wq_scale is not NULL the step also writes
 * wq = E4M3(stored master * s_q), s_q from the amax of the stored master with
 * fmt_max 448 and the same margin, and s_q, 1/s_q to *wq_scale, *wq_inv
 * (wq may be NULL only when n == 0, e.g. an empty slice of a sharded step).
 * Pointers g, m, v, w, wq are dev and 16-byte aligned; the scale pointers are
 * dev floats.  Chunks must not overlap.  `chunks` is a HOST array of nchunks.
 */
typedef struct {
  const uint8_t *g;    /* dev [n] E5M2 gradient codes */
  const float *g_inv;  /* dev float: 1 / (mu * s_g) */
  uint8_t *m;          /* dev [n] E4M3 first-moment codes (in/out) */
  float *m_scale;      /* dev float (in/out) */
  uint16_t *v;         /* dev [n] FP16 second moment, scaled (in/out) */
  float *v_scale;      /* dev float (in/out) */
  uint16_t *w;         /* dev [n] FP16 master weight, scaled (in/out) */
  float *w_scale;      /* dev float (in/out) */
  size_t n;            /* parameters in this chunk (0 allowed) */
  float *w_amax;       /* dev float or NULL: tracked amax of the stored master (in/out) */
  uint8_t *wq;         /* dev [n]: E4M3 copy of the new stored master (out), or NULL */
  float *wq_scale;     /* dev float or NULL: asks for the copy (out) */
  float *wq_inv;       /* dev float, required with wq_scale (out) */
} fp8_adam_chunk;

typedef struct {
  float lr, beta1, beta2, eps; /* 0 <= lr finite, 0 <= beta < 1, 2^-39 <= eps <= 2^64
                                  (else FP8_ERR_INVALID_ARG: eps = 0 makes a zero
                                  gradient on a zero state 0/0, below 2^-39 a
                                  binary32-subnormal v_hat would reach the step, above
                                  2^64 the reciprocal of sqrt(v_hat) + eps could be
                                  subnormal) */
  int step;                    /* t >= 1 (bias correction) */
  int margin;                  /* scale margin, >= 0 */
} fp8_adam_hparams;

/* Bytes of device workspace fp8_adam_step needs for nchunks chunks. */
size_t fp8_adam_workspace_bytes(int nchunks);

/*
 * fp8_adam_step -- one step over all chunks.  workspace: dev, at least
 * fp8_adam_workspace_bytes(nchunks) bytes, 256-byte aligned, owned by the
 * caller, not touched by anything else while the step runs (it holds the
 * per-chunk amax accumulators and the old scales between the two passes).
 */
int fp8_adam_step(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                  void *workspace, size_t ws_bytes, void *stream);

/* New state buffers of one chunk for fp8_adam_step_into. */
typedef struct {
  uint8_t *m;   /* dev [n] E4M3 first-moment codes (out) */
  uint16_t *v;  /* dev [n] FP16 second moment, scaled (out) */
  uint16_t *w;  /* dev [n] FP16 master weight, scaled (out) */
} fp8_adam_dest;

/*
 * fp8_adam_step_into -- the step of fp8_adam_step with the new m, v, w
 * written to dest[i] instead of over chunks[i].m, .v, .w, which are only
 * read (a caller alternates two sets of buffers).  Every result -- codes,
 * FP16 values, scales, tracked amax, E4M3 copy -- is bit for bit the one
 * fp8_adam_step gives on the same inputs.  The step predicts that each new
 * scale equals the old one: one pass reads the old state (6 B/param) and
 * writes the new one with the predicted scales (5 B/param, +1 B for the
 * E4M3 copy) while reducing the exact new amaxes; a chunk whose prediction
 * was wrong (some new scale differs) is updated a second time from its
 * unchanged inputs with the right scales.  When the scales hold, the state
 * is read once instead of twice.
 *   dest: HOST array of nchunks; for a chunk with n > 0 its three pointers
 *   are dev, 16-byte aligned (else FP8_ERR_UNALIGNED) and must not overlap
 *   any chunk's g, m, v, w, wq or another dest (a dest pointer equal to the
 *   same chunk's m, v, w, g or wq is rejected with FP8_ERR_INVALID_ARG; other
 *   overlaps are not detected).  Scales, w_amax, wq, wq_scale, wq_inv are
 *   updated in place as by fp8_adam_step.  Workspace and errors as for
 *   fp8_adam_step; nchunks with any n.
 */
int fp8_adam_step_into(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest, int nchunks,
                       const fp8_adam_hparams *hp, void *workspace, size_t ws_bytes, void *stream);

/* The gradient cast of fp8_adam_step_into_castgrad. */
typedef struct {
  const float *const *amax;  /* HOST array of nchunks dev pointers: amax|dW| of each chunk's
                                gradient (e.g. the wgrad's fused output amax); none NULL */
  float mu;                  /* gradient auto-scaling factor, a power of two in [2^-32, 2^32] */
  int margin;                /* scale margin, 0..64 */
} fp8_adam_grad_cast;

/*
 * fp8_adam_step_into_castgrad -- the gradient cast and the out-of-place step
 * in one pass: for every chunk, chunks[i].g points to the gradient as the wgrad
 * wrote it, n bfloat16 values (FP8_DT_BF16 or FP8_DT_BF16_RTO), dev, 16-byte
 * aligned; the step casts it to E5M2 in registers with the scale
 * fp8_scale_cast(dW, FP8_E5M2, amax[i], margin, mu, ...) would derive --
 * the same codes that call would store -- and runs fp8_adam_step_into on
 * them.  The E5M2 gradient is never written: 2 B per parameter less traffic
 * than the cast followed by the step, and one kernel less per tensor.
 * chunks[i].g_inv (dev float) receives the gradient's inverse scale (what
 * the cast writes to inv_scale_dev); its scale itself is not written.  A
 * non-finite amax sets FP8_STATUS_NONFINITE (as the cast does).  All
 * results are bit for bit those of fp8_scale_cast then fp8_adam_step_into.
 * Arguments and errors otherwise as fp8_adam_step_into; FP8_ERR_INVALID_ARG
 * also for a NULL gc, a NULL amax entry, a bad mu or margin.
 */
int fp8_adam_step_into_castgrad(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest,
                                const fp8_adam_grad_cast *gc, int nchunks, const fp8_adam_hparams *hp,
                                void *workspace, size_t ws_bytes, void *stream);

/*
 * Element-sharded step ([FP8-LM] 提案手法 O3: FP8 optimizer state under a
 * ZeRO-style partition).  fp8_adam_step in two halves so that ranks which
 * each hold a contiguous slice of every tensor agree on its per-tensor
 * scales:
 *   fp8_adam_stats  clears the workspace and writes the amax of the new
 *                   m, v, w of this rank's slices (nothing else changes);
 *   <caller>        element-wise MAX of the workspace over the ranks, taken
 *                   on its 32-bit words read as int32 (every word is the bit
 *                   pattern of a float >= 0 or of +NaN, so integer order is
 *                   the amax order and a NaN wins);
 *   fp8_adam_apply  derives the new scales from the reduced workspace and
 *                   updates this rank's slices in place.
 * Chunk i must be a slice of the same tensor on every rank, with the same
 * m_scale, v_scale, w_scale values; every rank then writes the same new
 * scales, and the slices end up exactly as one fp8_adam_step over the whole
 * tensor would leave them.  Both calls take the same chunks, hparams and
 * workspace (contents kept between them); tracked master amax is not
 * available here (w_amax must be NULL, else FP8_ERR_INVALID_ARG).  A slice
 * may be empty (n = 0).  Without the reduction in between (one rank), the
 * pair equals fp8_adam_step.
 */
int fp8_adam_stats(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                   void *workspace, size_t ws_bytes, void *stream);
int fp8_adam_apply(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                   void *workspace, size_t ws_bytes, void *stream);

/*
 * The element-sharded step out of place: fp8_adam_step_into in two halves,
 * with the same MAX reduction of the workspace over the ranks in between.
 *   fp8_adam_stats_into  clears the workspace, writes this rank's new slices
 *                        into dest with the predicted (old) scales and the
 *                        exact amax of the new m, v, w into the workspace;
 *   <caller>             the element-wise int32 MAX of the workspace, as
 *                        for fp8_adam_stats;
 *   fp8_adam_apply_into  derives the new scales from the reduced amaxes
 *                        (the same on every rank), publishes them, and
 *                        writes again, from the unchanged inputs, the
 *                        slices of every tensor whose scales changed.
 * One pass over this rank's state while the scales hold (two for a tensor
 * whose scales change), the one collective of the in-place halves, and
 * every slice ends up bit for bit as fp8_adam_step over the whole tensor
 * would leave it.  Arguments and errors as for fp8_adam_stats /
 * fp8_adam_apply plus dest as for fp8_adam_step_into; both calls take the
 * same chunks, dest, hparams and workspace.
 */
int fp8_adam_stats_into(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest, int nchunks,
                        const fp8_adam_hparams *hp, void *workspace, size_t ws_bytes, void *stream);
int fp8_adam_apply_into(const fp8_adam_chunk *chunks, const fp8_adam_dest *dest, int nchunks,
                        const fp8_adam_hparams *hp, void *workspace, size_t ws_bytes, void *stream);

/*
 * fp8_adam_step_noalloc -- the same step as fp8_adam_step, for callers that
 * cannot hand the library any device memory of their own: code running under
 * a host framework whose caching allocator owns (and has already reserved)
 * the GPU's memory, plugins whose host forbids raw cudaMalloc, and loops that
 * must never hit the device-wide synchronisation cudaMalloc/cudaFree can
 * cause.  The paper has no counterpart; this is a deployment convenience.
 *
 * The per-chunk scratch lives in a fixed array compiled into the library
 * (FP8_ADAM_NOALLOC_MAX_CHUNKS x 64 bytes = 64 KiB on every GPU that loads
 * the library, held until the process exits).  The call allocates and frees
 * nothing.  nchunks above FP8_ADAM_NOALLOC_MAX_CHUNKS returns
 * FP8_ERR_INVALID_ARG before any work is enqueued.
 * The first call on a device looks up that device's copy of the array (a
 * cudaGetSymbolAddress with the device current); make that first call before
 * any stream capture.  Every call on a device shares the one array: the step
 * clears the part it needs before use, and two calls whose work overlaps on
 * the GPU (different streams, no ordering between them) race on it.
 * The looked-up address is kept per device ordinal for the life of the
 * process: do not use this entry point across a cudaDeviceReset (or any
 * other teardown of the device's primary context), after which the kept
 * address no longer belongs to the device.
 * Arguments, results and errors are otherwise those of fp8_adam_step.
 */
#define FP8_ADAM_NOALLOC_MAX_CHUNKS 1024
int fp8_adam_step_noalloc(const fp8_adam_chunk *chunks, int nchunks, const fp8_adam_hparams *hp,
                          void *stream);

/*
 * fp8_get_status -- enqueues on `stream` one atomic exchange that reads the
 * device status word (OR of FP8_STATUS_* bits raised since the last read) and
 * clears it in the same operation, so a bit raised by a kernel on another
 * stream is either in this read or left for the next one; then waits for
 * `stream` and writes the value to *host_out.  Calls on different streams
 * must not overlap (they share the one readback word).  Returns FP8_ERR_CUDA
 * if the stream reported an error.
 */
int fp8_get_status(unsigned *host_out, void *stream);

/*
 * fp8_selftest_wait_timeout -- failure-detection self-test.  Enqueues one
 * thread that runs the GEMM pipeline's bounded barrier wait on a barrier
 * that nothing ever arrives at, with a limit of limit_us microseconds
 * (1 .. 1,000,000) instead of the GEMMs' 2 s.  The wait must end by itself
 * and raise FP8_STATUS_TIMEOUT in the status word (read it with
 * fp8_get_status); the context stays usable.  Returns FP8_ERR_INVALID_ARG
 * for a limit outside the range, nothing enqueued.  The pages have no
 * counterpart; it checks the library's own hang protection.
 */
int fp8_selftest_wait_timeout(unsigned limit_us, void *stream);

/*
 * fp8_selftest_step_reciprocal -- numerics self-test of the Adam step's own
 * correctly rounded reciprocal, which the library computes without CUDA's
 * __frcp_rn.  Compares the two on every binary32 argument whose bit pattern
 * lies in [lo_bits, hi_bits) (hi_bits <= 2^32; the step's arguments are
 * 2^-39 <= b <= 2^66 and +inf, where they must agree).  Two NaNs agree.
 * Adds the number of arguments that differ to *bad_dev (dev, one uint64)
 * and lowers *first_dev (dev, one uint32) to the smallest such bit pattern;
 * the caller initialises both.  FP8_ERR_INVALID_ARG for an empty or too wide
 * range or NULL outputs.
 */
int fp8_selftest_step_reciprocal(unsigned lo_bits, unsigned long long hi_bits, unsigned long long *bad_dev,
                                 unsigned *first_dev, void *stream);

/*
 * fp8_selftest_encode -- numerics self-test of the library's FP8 encoder
 * (fmt FP8_E4M3 or FP8_E5M2): the saturating hardware conversion with a
 * branch-free canonicalisation of NaN codes, against the same conversion
 * with an explicit test of each value for inf and NaN (+-inf -> +-max, NaN
 * -> 0x7F, as fp8_cast defines), on every binary32 value whose bit pattern
 * lies in [lo_bits, hi_bits) (hi_bits <= 2^32), in either lane of the
 * two-value conversion.  Adds the number of values whose codes differ to
 * *bad_dev (dev, one uint64) and lowers *first_dev (dev, one uint32) to the
 * smallest such pattern; the caller initialises both.  FP8_ERR_INVALID_ARG
 * for another format, an empty or too wide range or NULL outputs.
 */
int fp8_selftest_encode(int fmt, unsigned lo_bits, unsigned long long hi_bits, unsigned long long *bad_dev,
                        unsigned *first_dev, void *stream);

/* Human-readable message of a status code (static string). */
const char *fp8_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* FP8_B200_H */
