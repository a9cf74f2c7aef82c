/*
 * coat.h -- C ABI of the B200 (sm_100a) COAT FP8-optimizer-state library.
 *
 * COAT ("Compressing Optimizer states and Activation for memory-efficient
 * FP8 Training") keeps the AdamW first and second moments in FP8, one scale
 * and one dynamic-range-expansion exponent k per group of elements.  Sources:
 *   [P1] web page "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍",
 *        sections "FP8优化器状态" (per-group FP8 moments; E4M3 spans
 *        0.00195..448, about 200000; typical group max/min ~1000 for m and
 *        ~10 for v) and "解决方案：动态范围扩展" (expansion f(.) with one k
 *        per group, recomputed every step; E4M3+E4M3 or E4M3+E5M2), and
 *        "解决方案：混合粒度FP8精度流" (mixed-granularity FP8 activations).
 *   [P4] web page "FP8量化训练实战指南：解决大模型训练效率瓶颈的终极方案",
 *        sections "格式选择：E4M3与E5M2的智能搭配" (1+4+3 and 1+5+2 bit
 *        layouts) and "分块级缩放：精度优化的进阶方案" (1x128 tiles for
 *        activations, 128x128 blocks for weights, one scale per tile).
 * The expansion formula is missing from the pages' text; this library fixes
 *   f(x) = sign(x) |x|^k,   k = clamp(ln(448 / 2^-9) / ln(M / mu), 1, 16),
 * with M = max|x| and mu = min nonzero |x| over the group (M == mu gives 16;
 * an all-zero group gives k = 1 and scale 1), and the same 448/2^-9 target for
 * E5M2.  Codes are y = FMT_MAX (|x|/M)^k encoded to the nearest finite FP8
 * value (ties to the even code, saturating; a zero magnitude is code 0x00).
 *
 * SCALE CONVENTION.  The per-group "scale" stored by every call is the root
 * scale s_r = M * FMT_MAX^(-1/k) (the k-th root of s = M^k / FMT_MAX, which
 * underflows FP32 for second moments); dequantisation is
 *   x = sign(q) * s_r * |fp8(q)|^(1/k)       ( = sign(q) |fp8(q) s|^(1/k) ).
 *
 * Common rules for every call below:
 *   - All data pointers are DEVICE pointers owned by the caller (except
 *     where a call says host); the library
 *     never allocates on these paths (a multi-tensor plan owns one small
 *     device table, see coat_multi_plan_create).
 *   - Work is enqueued on `stream` and runs asynchronously; a return of
 *     COAT_OK means the arguments were valid and the launch was accepted.
 *   - Arguments are validated before anything is launched; on any error no
 *     kernel runs and no output is touched.  coat_last_error() then returns a
 *     thread-local message.
 *   - Buffers passed to one call must not overlap, except where stated.
 *   - bf16 data is passed as its 16-bit patterns (uint16_t).
 */
#ifndef COAT_H_
#define COAT_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* COAT_E5M2_FULL stores E5M2 codes like COAT_E5M2, but the dynamic-range
 * expansion stretches a group to E5M2's own span (57344 / 2^-16, log2 31.8)
 * instead of E4M3's 448 / 2^-9: k = clamp(ln(57344 / 2^-16) / ln(M / mu), 1, 16).
 * With it E5M2 moments match E4M3's error after expansion, as [P1]
 * 解决方案：动态范围扩展 reports for the second moment.  For the element codec
 * (coat_fp8_encode/decode) and for dequantisation it is identical to E5M2. */
typedef enum { COAT_E4M3 = 0, COAT_E5M2 = 1, COAT_E5M2_FULL = 2 } coat_fmt;
typedef enum { COAT_F32 = 0, COAT_BF16 = 1 } coat_dtype;

typedef enum {
    COAT_OK = 0,
    COAT_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum, bad hyperparameter */
    COAT_ERR_MISALIGNED = 2,  /* a pointer or leading dimension breaks the 16-byte rule */
    COAT_ERR_UNSUPPORTED = 3, /* a valid request this library does not implement (e.g. group != 128) */
    COAT_ERR_CUDA = 4,        /* the CUDA runtime reported an error at launch or copy */
    COAT_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait; results are invalid */
    COAT_ERR_NOMEM = 6,       /* host or device allocation failed (plan creation only) */
    COAT_ERR_DEVICE_CHECK = 7 /* checked build only: a kernel's index check failed and the
                                 access was skipped; results are invalid */
} coat_status;

/* Thread-local description of the last non-OK status returned on this thread. */
const char *coat_last_error(void);

/* Library version as 10000*major + 100*minor + patch. */
int coat_version(void);

/* ---------------------------------------------------------------------------
 * FP8 element codec (the encode/decode steps of [P1]'s per-group quantiser;
 * formats of [P4] 格式选择).
 *
 * coat_fp8_encode: q[i] = nearest finite FP8 value to y[i] (FP32), round to
 *   nearest, ties to the even code, saturating to +-FMT_MAX (448 for E4M3,
 *   57344 for E5M2); NaN -> 0x7F | sign; a result of magnitude zero is 0x00.
 * coat_fp8_decode: out[i] = FP32 value of code q[i] (E5M2 0x7C is +inf;
 *   NaN codes give NaN).
 * n >= 0 elements; y / out need 4-byte alignment, q none.
 * ------------------------------------------------------------------------- */
coat_status coat_fp8_encode(const float *y, int64_t n, coat_fmt fmt, uint8_t *q,
                            cudaStream_t stream);
coat_status coat_fp8_decode(const uint8_t *q, int64_t n, coat_fmt fmt, float *out,
                            cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Per-group quantise / dequantise with dynamic range expansion ([P1]
 * 解决方案：动态范围扩展), at mixed granularity ([P1] 混合粒度FP8精度流;
 * [P4] 分块级缩放: 1x128 per-token groups, 128x128 weight blocks).
 *
 * x      : rows x cols matrix of dtype xt (COAT_F32 or COAT_BF16), row-major,
 *          leading dimension ld_x elements (ld_x >= cols).
 * groups : group_rows x group_cols blocks; supported: 1x128 and 128x128.
 *          Edge blocks that are cut by rows/cols hold only the valid elements.
 * expand : 0 -> k = 1 (plain per-group scaling), 1 -> k from the formula.
 * q      : rows x cols codes, leading dimension ld_q bytes (ld_q >= cols); only
 *          the valid elements are written.
 * scale,k: ceil(rows/group_rows) x ceil(cols/group_cols) floats, row-major.
 * out    : dequantised rows x cols of dtype ot, leading dimension ld_out.
 * Alignment: x, q, out 16-byte aligned; when rows > 1, ld_x*size(xt), ld_q and
 * ld_out*size(ot) multiples of 16 bytes; scale, k 4-byte aligned.  rows,
 * cols >= 0 (0 is a no-op).
 * ------------------------------------------------------------------------- */
coat_status coat_group_quantize(const void *x, coat_dtype xt, int64_t rows, int64_t cols,
                                int64_t ld_x, int group_rows, int group_cols, int expand,
                                coat_fmt fmt, uint8_t *q, int64_t ld_q, float *scale,
                                float *k, cudaStream_t stream);
coat_status coat_group_dequantize(const uint8_t *q, int64_t ld_q, const float *scale,
                                  const float *k, int64_t rows, int64_t cols,
                                  int group_rows, int group_cols, coat_fmt fmt, void *out,
                                  coat_dtype ot, int64_t ld_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The fused AdamW step over FP8 moments ([P1] FP8优化器状态 and
 * 动态范围扩展: per group, dequantise m and v, update, recompute k each step,
 * requantise).  For each element i (t = step >= 1):
 *   m  = dequant(m_q[i]),  v = dequant(v_q[i]),  g = bf16 grad[i]
 *   m' = b1 m + (1-b1) g;   v' = b2 v + (1-b2) g^2
 *   p  = master[i] (1 - lr wd) - (lr / (1-b1^t)) m' / (sqrt(v') / sqrt(1-b2^t) + eps)
 *   master[i] = p (FP32, in place);  weight_bf16_out[i] = RNE_bf16(p)
 * then m' and v' are requantised per group (expansion on) into m_q/m_scale/m_k
 * and v_q/v_scale/v_k, in place.  The update uses the unquantised m', v'.
 * This is torch.optim.AdamW's arithmetic (decoupled weight decay, no amsgrad).
 *
 * n        : number of elements (>= 0; 0 is a no-op).
 * group    : must be 128.
 * master   : n floats.            grad: n bf16 patterns.
 * weight_bf16_out: n bf16 patterns, or NULL to skip the bf16 copy.
 * m_q, v_q : ceil(n/128)*128 bytes; padding codes of a partial last group are
 *            ignored on input and written 0.
 * m_scale, m_k, v_scale, v_k: ceil(n/128) floats each.
 * Alignment: every pointer 16-byte aligned (COAT_ERR_MISALIGNED otherwise).
 * Hyperparameters: lr >= 0, 0 <= beta1, beta2 < 1, eps > 0, wd >= 0, all finite;
 * step >= 1.  fmt_m, fmt_v: COAT_E4M3, COAT_E5M2 or COAT_E5M2_FULL.
 * ------------------------------------------------------------------------- */
coat_status coat_adamw_step(float *master, uint16_t *weight_bf16_out, const uint16_t *grad,
                            uint8_t *m_q, float *m_scale, float *m_k, uint8_t *v_q,
                            float *v_scale, float *v_k, int64_t n, int group, float lr,
                            float beta1, float beta2, float eps, float wd, int64_t step,
                            coat_fmt fmt_m, coat_fmt fmt_v, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Group-parameter mode of every AdamW step entry point (coat_adamw_step, the
 * multi-tensor, clipped and no-allocation steps), process-wide; returns the
 * previous mode.  The COAT pages give no precision for k and the scale; the
 * definition computes them from the new moments' group maximum and nonzero
 * minimum.
 *
 * on = 0 (the default): each group's extremes are the FP32 values of m' and
 *   v' (the smallest |m'| recomputed in double, since it usually comes from
 *   cancellation between beta1 m and (1 - beta1) g), and k and the root scale
 *   are derived from them with FP32 approximations: within about 3e-7 (k) and
 *   5e-6 (scale) of the exact values.
 * on = 1: each group's extremes (max |m'|, the two smallest nonzero |m'|, max
 *   v', the smallest nonzero v') are recomputed in double from the stored codes
 *   and the gradient, and k and the root scale are computed in double and
 *   rounded to FP32 once: the correctly rounded values of the definition
 *   (except when an FP32 near-tie hides the true extreme).  Two runs that
 *   start from the same state then keep bit-identical k, scales and codes
 *   apart from rare code-rounding differences, so they stay in lockstep.  The
 *   step is 15-25% slower: the double-precision work of each group adds about
 *   20% to the instructions per parameter.
 * Codes come from the same FP32 expansion and software encoder in both modes.
 * ------------------------------------------------------------------------- */
int coat_set_exact_group_params(int on);

/* ---------------------------------------------------------------------------
 * Multi-tensor launcher over a ragged list of parameter tensors: one kernel
 * launch per step updates every tensor, each exactly as coat_adamw_step would
 * (groups never span tensors; each tensor's last group may be partial).
 *
 * coat_multi_plan_create copies `num` host descriptors (each obeying the
 * coat_adamw_step rules for its own n) into a device table owned by the plan
 * (one cudaMalloc, which also holds the gradient-norm scratch below;
 * COAT_ERR_NOMEM on failure); the copy is enqueued on `stream`.  The plan refers to the caller's buffers, which must stay valid
 * while the plan is used.  Tensors with n == 0 are allowed.  num >= 1.
 * coat_adamw_step_multi applies one step to all tensors on `stream`.
 * coat_multi_plan_destroy frees the table (after synchronising the device);
 * passing NULL is a no-op.
 * ------------------------------------------------------------------------- */
typedef struct {
    float *master;
    uint16_t *weight_bf16_out; /* may be NULL */
    const uint16_t *grad;
    uint8_t *m_q;
    float *m_scale;
    float *m_k;
    uint8_t *v_q;
    float *v_scale;
    float *v_k;
    int64_t n;
} coat_tensor_desc;

typedef struct coat_multi_plan *coat_multi_plan_t;

coat_status coat_multi_plan_create(const coat_tensor_desc *host_descs, int num, int group,
                                   coat_fmt fmt_m, coat_fmt fmt_v, cudaStream_t stream,
                                   coat_multi_plan_t *out_plan);
coat_status coat_adamw_step_multi(coat_multi_plan_t plan, float lr, float beta1, float beta2,
                                  float eps, float wd, int64_t step, cudaStream_t stream);
coat_status coat_multi_plan_destroy(coat_multi_plan_t plan);
/* Per-tensor weight decay of a plan: tensor i decays with wd * host_wd_scale[i]
 * (e.g. 0 for normalisation weights, the usual exclusion from decoupled
 * weight decay); every scale is 1 when the plan is created.  host_wd_scale
 * holds one finite value >= 0 per tensor of the plan, read during the call
 * (the call synchronises `stream` after its copy).  COAT_ERR_INVALID_ARG for a
 * NULL argument or a negative or non-finite scale. */
coat_status coat_multi_plan_set_wd_scale(coat_multi_plan_t plan, const float *host_wd_scale,
                                        cudaStream_t stream);
/* Number of elements and tensors covered by a plan. */
coat_status coat_multi_plan_info(coat_multi_plan_t plan, int64_t *total_elements,
                                 int *num_tensors);

/* ---------------------------------------------------------------------------
 * Global gradient-norm clipping and the non-finite check before the step.
 * The COAT pages do not describe this step; it is the pre-step of an ordinary
 * training loop (torch.nn.utils.clip_grad_norm_ over all parameters, and the
 * found-Inf check of a loss-scaled loop that skips the step on overflow),
 * kept on the device so that no value has to travel to the host between the
 * backward pass and the optimizer step.
 *
 * coat_multi_plan_grad_norm reads every gradient of the plan once and writes
 * one coat_grad_clip record to `d_clip` (device memory, 8-byte aligned, owned
 * by the caller) on `stream`:
 *   - sumsq: the sum of g^2 over all gradient elements, accumulated in double
 *     (squares exact; partial sums of 8 squares rounded in FP32, so sumsq is
 *     within about 3e-7 relative of the exact sum); +Inf or NaN when any
 *     element is Inf or NaN;
 *   - norm: sqrt(sumsq) rounded to FP32;
 *   - coef: min(1, max_norm / (sqrt(sumsq) + 1e-6)), evaluated in double and
 *     rounded to FP32 (1 for max_norm = +Inf);
 *   - found_inf: 1 when sumsq is not finite, else 0; reserved: 0.
 * max_norm > 0 (+Inf allowed: the norm without clipping).  The result is
 * deterministic on a given device.  The plan holds the pass's scratch (one
 * slot per CTA and a counter), so calls on one plan must be ordered on one
 * stream, as steps are.
 *
 * coat_adamw_step_multi_clipped is coat_adamw_step_multi with every gradient
 * element g replaced by coef * g, coef read from `d_clip` on the device when
 * the step runs; when found_inf is nonzero the step changes nothing (master,
 * bf16 copy, codes and metadata keep their bytes).  With coef = 1 it gives
 * the same bytes as coat_adamw_step_multi.  d_clip: as written by
 * coat_multi_plan_grad_norm, or by the caller in the same layout.
 * ------------------------------------------------------------------------- */
typedef struct {
    double sumsq;
    float norm;
    float coef;
    int32_t found_inf;
    int32_t reserved;
} coat_grad_clip; /* 24 bytes */

coat_status coat_multi_plan_grad_norm(coat_multi_plan_t plan, float max_norm,
                                      coat_grad_clip *d_clip, cudaStream_t stream);
coat_status coat_adamw_step_multi_clipped(coat_multi_plan_t plan, float lr, float beta1,
                                          float beta2, float eps, float wd, int64_t step,
                                          const coat_grad_clip *d_clip, cudaStream_t stream);
/* Clipping over data-parallel ranks, each holding part of the gradients (a
 * ZeRO-1 shard, see coat_zero1_layout): each rank runs
 * coat_multi_plan_grad_norm on its own plan (max_norm = +Inf), the callers
 * sum the records' sumsq fields over the ranks (an all-reduce of that one
 * double), and coat_grad_clip_finalize then rewrites norm, coef, found_inf and
 * reserved of the record at d_clip from its sumsq and max_norm, with the same
 * arithmetic as coat_multi_plan_grad_norm (so one rank gives that call's
 * record bit for bit).  One thread on `stream`; d_clip 8-byte aligned device
 * memory; max_norm > 0 (+Inf allowed); COAT_ERR_INVALID_ARG /
 * COAT_ERR_MISALIGNED otherwise, before anything is enqueued. */
coat_status coat_grad_clip_finalize(coat_grad_clip *d_clip, float max_norm, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * No-allocation variant of the multi-tensor step.  The COAT pages have no
 * counterpart: this is a deployment convenience of this library.
 *
 * Some callers cannot call cudaMalloc: code that runs inside a framework whose
 * caching allocator must own all device memory (a raw allocation would bypass
 * its accounting and may fail under its reservations), or code that must not
 * allocate once set up (a cudaMalloc can synchronise the device and stall a
 * latency-sensitive loop).  coat_adamw_step_multi_noalloc applies the same
 * step as coat_multi_plan_create + coat_adamw_step_multi (identical results),
 * but keeps the tensor table in a fixed array inside the library's device
 * image instead of a cudaMalloc'd plan table.  It allocates nothing: no
 * cudaMalloc/cudaFree, no allocating library routine, no heap use.
 *
 *   - host_descs: num descriptors in host memory, read before the call returns
 *     (the caller may change or free them on return).  Each obeys the
 *     coat_adamw_step rules.
 *   - num: 1 .. COAT_NOALLOC_MAX_TENSORS.  A larger num returns
 *     COAT_ERR_UNSUPPORTED (as does group != 128); other bad arguments return
 *     COAT_ERR_INVALID_ARG or COAT_ERR_MISALIGNED, before anything is enqueued.
 *     This call reports through its return code only: it does not record a
 *     message, so coat_last_error() keeps describing an earlier failure.
 *   - The fixed array holds COAT_NOALLOC_MAX_TENSORS kernel descriptors of
 *     104 bytes each (106,496 bytes); every GPU that loads the library keeps
 *     it until the process exits.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and configures the kernel.
 *   - Each call enqueues, on `stream`, small copy kernels that write the table
 *     into the array (the descriptors travel as their kernel parameters, 32
 *     per launch, so no host buffer is read after the call returns and no
 *     copy from pageable memory makes the call wait for earlier work on
 *     `stream`), then the step kernel.  All calls share the one array and it
 *     keeps the last call's contents: calls that may overlap on the GPU
 *     (different streams without ordering between them) race on it and must
 *     not be issued.
 * ------------------------------------------------------------------------- */
#define COAT_NOALLOC_MAX_TENSORS 1024
coat_status coat_adamw_step_multi_noalloc(const coat_tensor_desc *host_descs, int num, int group,
                                          float lr, float beta1, float beta2, float eps,
                                          float wd, int64_t step, coat_fmt fmt_m, coat_fmt fmt_v,
                                          cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * FP8 precision flow through a non-linear layer ([P1] FP8激活 and
 * 解决方案：混合粒度FP8精度流): the layer's input and output are FP8 tensors
 * in 1x128 per-token groups, and the backward pass reads the FP8 input as the
 * forward received it (nothing is re-quantised to save it).  The layer is
 * Llama's gated activation h = silu(gate) * up, silu(g) = g / (1 + e^-g).
 *
 * coat_fp8_act describes one rows x cols FP8 tensor in the codec's 1x128
 * layout (coat_group_quantize with group 1x128): codes q (row stride ldq
 * bytes), and per group a root scale and k (rows x ceil(cols/128), row stride
 * lds floats); a value is sign(q) scale |q|^(1/k), k = 1 without expansion.
 * gate and up may be two halves of one [rows x 2F] buffer (strides 2F and
 * 2F/128, up starting F codes / F/128 groups in, F a multiple of 128).
 *
 * coat_swiglu_fp8_forward: h = silu(gate) up computed in FP32, then quantised
 * per 1x128 group into `out` exactly as coat_group_quantize does (expand_out
 * 0: k = 1; 1: expansion).  A sigmoid below 2^-126 is 0 (FP32 with subnormals
 * flushed).  `out` must not overlap the inputs.
 * coat_swiglu_fp8_backward: grad_out (bf16, row stride ld elements) and the
 * forward's gate / up give
 *   grad_up   = grad_out silu(g),
 *   grad_gate = grad_out u sigmoid(g) (1 + g (1 - sigmoid(g))),
 * computed in FP32 and rounded to bf16 (nearest even).
 * Requirements: rows, cols >= 0 (0 is a no-op); cols a multiple of 16, and
 * at most 2^30 for the forward (COAT_ERR_UNSUPPORTED otherwise; the last group
 * may be partial); every code
 * and bf16 array 16-byte aligned with row strides that are multiples of 16
 * bytes (ldq >= cols; bf16 strides >= cols); scale / k 4-byte aligned with
 * lds >= ceil(cols/128); fmt the format of all three tensors.
 * ------------------------------------------------------------------------- */
typedef struct {
    uint8_t *q;
    float *scale;
    float *k;
    int64_t ldq;
    int64_t lds;
} coat_fp8_act;

coat_status coat_swiglu_fp8_forward(const coat_fp8_act *gate, const coat_fp8_act *up,
                                    int64_t rows, int64_t cols, coat_fmt fmt, int expand_out,
                                    const coat_fp8_act *out, cudaStream_t stream);
coat_status coat_swiglu_fp8_backward(const uint16_t *grad_out, int64_t ld_grad_out,
                                     const coat_fp8_act *gate, const coat_fp8_act *up,
                                     int64_t rows, int64_t cols, coat_fmt fmt,
                                     uint16_t *grad_gate, int64_t ld_grad_gate,
                                     uint16_t *grad_up, int64_t ld_grad_up,
                                     cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The FP8 precision flow through RMSNorm, the other non-linear layer of a
 * Llama block ([P1] FP8激活 / 混合粒度FP8精度流):
 *   y = x / sqrt(mean(x^2) + eps) * w   per row of d features,
 * x and y FP8 tensors in the 1x128 layout (coat_fp8_act), w a bf16 vector of d.
 *
 * coat_rmsnorm_fp8_forward: y computed in FP32 (the row's mean of squares
 * summed in FP32) and quantised per 1x128 group exactly as coat_group_quantize
 * does (expand_out 0 or 1).  `out` must not overlap x.
 * coat_rmsnorm_fp8_backward: from dy (bf16, row stride ld_dy) and the
 * forward's FP8 x, with xh = x rstd and g = dy w,
 *   dx = rstd (g - xh mean(g xh))         (bf16, row stride ld_dx),
 *   dw = sum over rows of dy xh            (d floats, summed per CTA in FP32
 *                                           and over CTAs in index order in
 *                                           double: deterministic on a device).
 * The backward needs `workspace` (device memory, 16-byte aligned, owned by the
 * caller) of at least coat_rmsnorm_fp8_workspace_size(d) bytes; calls that
 * share a workspace must be ordered on one stream.  rows == 0 writes dw = 0.
 * Requirements: d a multiple of 128 and at most 8192 (COAT_ERR_UNSUPPORTED
 * otherwise); eps finite and > 0; w 16-byte aligned; code and bf16 arrays as
 * for the SwiGLU calls; dw 4-byte aligned.
 * ------------------------------------------------------------------------- */
coat_status coat_rmsnorm_fp8_forward(const coat_fp8_act *x, const uint16_t *w, int64_t rows,
                                     int64_t d, float eps, coat_fmt fmt, int expand_out,
                                     const coat_fp8_act *out, cudaStream_t stream);
coat_status coat_rmsnorm_fp8_workspace_size(int64_t d, size_t *bytes);
coat_status coat_rmsnorm_fp8_backward(const uint16_t *dy, int64_t ld_dy, const coat_fp8_act *x,
                                      const uint16_t *w, int64_t rows, int64_t d, float eps,
                                      coat_fmt fmt, uint16_t *dx, int64_t ld_dx, float *dw,
                                      void *workspace, size_t workspace_bytes,
                                      cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * ZeRO-1 partition of a tensor list over data-parallel ranks.  [P1]
 * 训练加速1.43倍，显存降低1.54倍 reports per-GPU memory of a four-GPU run with
 * FP8 optimizer states (its parallelism unstated); keeping each rank's states
 * for a 1/world_size share of the parameters is this library's layout for
 * data parallelism (each group's states live on exactly one rank).
 * Host-only: this call makes no CUDA call and works on a host without a GPU.
 *
 * Flat layout, in blocks of 4 groups (B = 4 * group = 512 elements, so that
 * every piece's per-group scale and k arrays start on a 16-byte boundary, as
 * the step's descriptors require): tensor i starts at flat element
 *   flat_offset[i] = sum over j < i of ceil(n_j / B) * B,
 * so no group spans two tensors.  With T the total number of blocks and
 * shard_elems = ceil(T / world_size) * B, rank r owns flat elements
 * [r shard_elems, (r + 1) shard_elems) (the last ranks may own padding only).
 * A flat gradient or weight buffer holds flat_elems = world_size *
 * shard_elems elements, its gaps and tail padding, so that a reduce-scatter
 * or an all-gather moves shard_elems elements per rank.
 *
 * The rank's share is written as pieces, one per tensor it touches, in
 * tensor order:
 *   tensor       index into sizes;
 *   elem_begin   first element of the piece in the tensor (a multiple of B);
 *   n_elems      elements of the piece (> 0; its last group is partial when
 *                it holds a tensor's partial last group);
 *   shard_begin  first element of the piece in the rank's shard of
 *                shard_elems elements (a multiple of B); the piece's groups
 *                start at group shard_begin / group of the shard.
 * Arguments: sizes: num_tensors >= 1 host values >= 0; group 128; world_size
 * >= 1; 0 <= rank < world_size; pieces: host array of max_pieces entries
 * (at most num_tensors are needed; NULL with max_pieces = 0 asks for the
 * counts); flat_offsets: NULL or num_tensors host values, filled as above.
 * *num_pieces, *shard_elems and *flat_elems are always written on success
 * and when pieces is too small (then COAT_ERR_INVALID_ARG, and only the
 * first max_pieces entries are written).  Other errors: COAT_ERR_INVALID_ARG, COAT_ERR_UNSUPPORTED for
 * group != 128.
 * ------------------------------------------------------------------------- */
typedef struct {
    int32_t tensor;
    int32_t reserved; /* 0 */
    int64_t elem_begin;
    int64_t n_elems;
    int64_t shard_begin;
} coat_shard_piece; /* 32 bytes */

coat_status coat_zero1_layout(const int64_t *sizes, int num_tensors, int group, int world_size,
                              int rank, coat_shard_piece *pieces, int max_pieces,
                              int *num_pieces, int64_t *shard_elems, int64_t *flat_elems,
                              int64_t *flat_offsets);

/* ---------------------------------------------------------------------------
 * Device error word.  Kernels that wait on a shared-memory barrier give up
 * after a bounded time (about one second), set a flag and return;
 * coat_check_device_error synchronises `stream`, reads and clears the flag,
 * and returns COAT_ERR_TIMEOUT if it was set (COAT_OK otherwise, or
 * COAT_ERR_CUDA if the synchronisation itself failed).
 *
 * Checked build (libcoat_debug.so, compiled with COAT_DEBUG; the library's
 * stand-in for a memory checker): before each load or store whose index it
 * derives, a kernel checks the index against the extents it was given (tile
 * within its tensor, element below n, group below the group count, row and
 * column within the shape); a failed check is counted on the device and the
 * access is skipped, never trapped.  coat_check_device_error then also reads
 * and clears the counts and returns COAT_ERR_DEVICE_CHECK if any check
 * failed.  The release build (libcoat.so) compiles the checks away.
 * ------------------------------------------------------------------------- */
coat_status coat_check_device_error(cudaStream_t stream);

/* 1 in the checked build (libcoat_debug.so), 0 in the release build. */
int coat_build_checked(void);

/* Self-test of the bounded waits (the COAT pages have no counterpart; this
 * exists to test the failure path without a GPU fault).  Enqueues on `stream`
 * one warp that waits, for at most budget_cycles SM clock cycles (1000 ..
 * 2e9), on a shared-memory barrier that nothing ever arrives on; the warp gives
 * up, sets the device error word and exits.  A following
 * coat_check_device_error(stream) returns COAT_ERR_TIMEOUT and clears the
 * word; the context stays usable.  Returns COAT_ERR_INVALID_ARG for a budget
 * out of range, COAT_ERR_CUDA if the launch fails. */
coat_status coat_selftest_wait_timeout(int64_t budget_cycles, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* COAT_H_ */
