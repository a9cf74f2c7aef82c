// coat_internal.h -- host-side launch interface between the C ABI (api.cu) and
// the kernels (adamw_fp8.cu, codec.cu).  Not part of the public ABI.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace coat {

// One parameter tensor as the step kernel sees it (device pointers).
struct TensorArgs {
  float* master;
  uint16_t* wout;  // may be null
  const uint16_t* grad;
  uint8_t* mq;
  float* ms;
  float* mk;
  uint8_t* vq;
  float* vs;
  float* vk;
  int64_t n;
  int64_t tiles;       // ceil(ceil(n/128) / groups-per-tile)
  int64_t tile_begin;  // first tile of this tensor in a multi-tensor launch
  float wd_scale;      // this tensor's weight decay is wd * wd_scale (1 by default)
};

// Hyperparameters as the kernel uses them (bias corrections and the step size
// folded on the host in double): m' = beta1 m + omb1 g, v' = beta2 v + omb2 g^2,
// p <- p - p lrwd - m' / (sqrt(v') dsq + deps), which is
// p - (lr / (1-beta1^t)) m' / (sqrt(v') / sqrt(1-beta2^t) + eps).
struct StepHyper {
  float beta1, beta2, omb1, omb2;
  float dsq;        // (1 - beta1^t) / (lr sqrt(1 - beta2^t)); 0 when lr = 0
  float deps;       // eps (1 - beta1^t) / lr; +inf when lr = 0
  float lrwd;       // lr * wd
  int32_t exact;    // 1: exact group parameters (coat_set_exact_group_params)
};

// Result of the gradient-norm pass over a plan's gradients; the same layout as
// coat_grad_clip in coat.h.
struct ClipRecord {
  double sumsq;       // sum of g^2 over every gradient element (non-finite: an Inf/NaN seen)
  float norm;         // sqrt(sumsq) rounded to FP32
  float coef;         // min(1, max_norm / (sqrt(sumsq) + 1e-6)) in double, rounded to FP32
  int32_t found_inf;  // 1 when sumsq is not finite
  int32_t reserved;
};
static_assert(sizeof(ClipRecord) == 24, "ClipRecord layout");

// Failed index checks counted by each kernel file since the last read (the
// checked build; always 0 in the release build); each call clears its count.
cudaError_t index_faults_step(unsigned* count);
cudaError_t index_faults_codec(unsigned* count);
cudaError_t index_faults_flow(unsigned* count);

int sm_count(int dev);
// Grid of at most sm_count(dev) * max_blocks_per_sm CTAs for work_items items
// of per_block each (at least 1).
unsigned grid_for(int64_t work_items, int per_block, int dev, int max_blocks_per_sm);
// CTAs of a kernel launched with `threads` threads (plus dyn_smem bytes of
// dynamic shared memory) resident per SM, from the occupancy calculator,
// cached per kernel.
int resident_ctas(const void* kernel, size_t dyn_smem = 0, int threads = 256);
cudaError_t device_error_ptr(unsigned** out);
int64_t step_tile_groups();

cudaError_t launch_adamw_single(const TensorArgs& t, int fm, int fv, const StepHyper& h,
                                unsigned* err, cudaStream_t stream);
// d_descs: num descriptors in device memory, tile_begin ascending (an empty
// tensor shares the next tensor's first tile); total_tiles: sum of tiles.
// clip: null, or a record written by launch_grad_sumsq: the step uses
// coef * g as the gradient, and does nothing at all when found_inf is set.
cudaError_t launch_adamw_multi(const TensorArgs* d_descs, int num, int64_t total_tiles, int fm,
                               int fv, const StepHyper& h, const ClipRecord* clip, unsigned* err,
                               cudaStream_t stream);

// Slots of per-CTA partial sums the gradient-norm pass needs on device dev.
int grad_sumsq_slots(int dev);
// Sum of squares of every gradient element of the descriptors into *out (with
// norm, clip coefficient for max_norm and the non-finite flag).  partials:
// grad_sumsq_slots() doubles; ticket: one unsigned that is 0 before the launch
// (the launch leaves it 0).  Deterministic for a given device.
cudaError_t launch_grad_sumsq(const TensorArgs* d_descs, int num, int64_t total_tiles,
                              double* partials, unsigned* ticket, float max_norm, ClipRecord* out,
                              cudaStream_t stream);

// One warp waits (bounded by budget_cycles) on a barrier nothing arrives on.
cudaError_t launch_wait_timeout_selftest(long long budget_cycles, unsigned* err,
                                         cudaStream_t stream);

cudaError_t launch_fp8_encode(const float* y, int64_t n, int fmt, uint8_t* q, cudaStream_t s);
cudaError_t launch_fp8_decode(const uint8_t* q, int64_t n, int fmt, float* out, cudaStream_t s);
cudaError_t launch_group_quantize(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                                  int gr, int expand, int fmt, uint8_t* q, int64_t ldq,
                                  float* scale, float* k, unsigned* err, cudaStream_t s);
cudaError_t launch_group_dequantize(const uint8_t* q, int64_t ldq, const float* scale,
                                    const float* k, int64_t rows, int64_t cols, int gr, int gc,
                                    int fmt, void* out, int ot, int64_t ldo, cudaStream_t s);

// One FP8 activation tensor in 1x128 per-token groups (device pointers):
// codes rows x cols with row stride ldq bytes; root scale and k per group,
// rows x ceil(cols/128) with row stride lds floats.
struct ActArgs {
  uint8_t* q;
  float* scale;
  float* k;
  int64_t ldq;
  int64_t lds;
};

// h = silu(gate) * up, quantised per 1x128 group (cols % 16 == 0).
cudaError_t launch_swiglu_fp8_forward(const ActArgs& gate, const ActArgs& up, int64_t rows,
                                      int64_t cols, int fmt, int expand, const ActArgs& out,
                                      cudaStream_t s);
// dgate, dup (bf16) from dh (bf16) and the forward's FP8 inputs (cols % 16 == 0).
cudaError_t launch_swiglu_fp8_backward(const uint16_t* dh, int64_t lddh, const ActArgs& gate,
                                       const ActArgs& up, int64_t rows, int64_t cols, int fmt,
                                       uint16_t* dg, int64_t lddg, uint16_t* du, int64_t lddu,
                                       cudaStream_t s);

// RMSNorm y = x / sqrt(mean(x^2) + eps) * w per row (d a multiple of 128, at
// most rmsnorm_max_d()), FP8 1x128 in and out, bf16 w.
int64_t rmsnorm_max_d();
// Bytes of the backward's per-CTA dw partials for rows of d features.
size_t rmsnorm_workspace_bytes(int dev, int64_t d);
cudaError_t launch_rmsnorm_fp8_forward(const ActArgs& x, const uint16_t* w, int64_t rows, int64_t d,
                                       float eps, int fmt, int expand, const ActArgs& out,
                                       cudaStream_t s);
// dx (bf16) and dw (FP32, summed over rows in a fixed order) from dy (bf16)
// and the forward's FP8 input; partial: rmsnorm_workspace_bytes() of scratch.
cudaError_t launch_rmsnorm_fp8_backward(const uint16_t* dy, int64_t lddy, const ActArgs& x,
                                        const uint16_t* w, int64_t rows, int64_t d, float eps,
                                        int fmt, uint16_t* dx, int64_t lddx, float* dw,
                                        float* partial, cudaStream_t s);

}  // namespace coat
