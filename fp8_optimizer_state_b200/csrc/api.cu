// api.cu -- the C ABI declared in include/coat.h: argument validation (before
// any CUDA call, so a bad call launches nothing and touches nothing), error
// reporting, multi-tensor plans, and kernel launches on the caller's stream.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <limits>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "coat.h"
#include "coat_internal.h"

namespace {

thread_local std::string g_last_error;

coat_status fail(coat_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

coat_status cuda_fail(cudaError_t e, const char* where) {
  return fail(COAT_ERR_CUDA, "%s: %s (%d)", where, cudaGetErrorString(e), static_cast<int>(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool valid_fmt(int f) { return f == COAT_E4M3 || f == COAT_E5M2 || f == COAT_E5M2_FULL; }
bool valid_dtype(int d) { return d == COAT_F32 || d == COAT_BF16; }
size_t dtype_size(int d) { return d == COAT_F32 ? 4 : 2; }

}  // namespace

// ---------------------------------------------------------------------------
// device-side error word and per-device caches
// ---------------------------------------------------------------------------
__device__ unsigned g_coat_device_error;

namespace coat {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_sm_count[kMaxDevices];
unsigned* g_err_ptr[kMaxDevices];
}  // namespace

int sm_count(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    g_sm_count[dev] = v;
  }
  return g_sm_count[dev];
}

// Device address of the error word on the current device (looked up once per
// device with that device current).
cudaError_t device_error_ptr(unsigned** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_coat_device_error);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_err_ptr[dev];
  return cudaSuccess;
}

}  // namespace coat

// ---------------------------------------------------------------------------
// helpers shared by the step entry points
// ---------------------------------------------------------------------------
namespace {

coat_status check_hyper(float lr, float beta1, float beta2, float eps, float wd, int64_t step) {
  if (!std::isfinite(lr) || lr < 0.f) return fail(COAT_ERR_INVALID_ARG, "lr must be finite and >= 0");
  if (!(beta1 >= 0.f && beta1 < 1.f)) return fail(COAT_ERR_INVALID_ARG, "beta1 must be in [0, 1)");
  if (!(beta2 >= 0.f && beta2 < 1.f)) return fail(COAT_ERR_INVALID_ARG, "beta2 must be in [0, 1)");
  if (!std::isfinite(eps) || !(eps > 0.f)) return fail(COAT_ERR_INVALID_ARG, "eps must be finite and > 0");
  if (!std::isfinite(wd) || wd < 0.f) return fail(COAT_ERR_INVALID_ARG, "weight decay must be finite and >= 0");
  if (step < 1) return fail(COAT_ERR_INVALID_ARG, "step must be >= 1");
  return COAT_OK;
}

// The group-parameter mode of the step entry points (coat_set_exact_group_params).
std::atomic<int> g_exact_group_params{0};

coat::StepHyper make_hyper(float lr, float beta1, float beta2, float eps, float wd, int64_t step) {
  const double b1 = beta1, b2 = beta2;
  const double bc1 = 1.0 - std::pow(b1, static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(b2, static_cast<double>(step));
  coat::StepHyper h;
  h.beta1 = beta1;
  h.beta2 = beta2;
  h.omb1 = static_cast<float>(1.0 - b1);
  h.omb2 = static_cast<float>(1.0 - b2);
  const double dlr = lr;
  const float dsq = static_cast<float>(bc1 / (dlr * std::sqrt(bc2)));
  const float deps = static_cast<float>(static_cast<double>(eps) * bc1 / dlr);
  if (lr == 0.f || !std::isfinite(dsq) || !std::isfinite(deps)) {
    // No adaptive term (lr = 0, or lr so small that lr / (1 - beta1^t) is below
    // FP32 range): 1 / (sqrt(v') 0 + inf) = 0 makes the kernel's update zero.
    h.dsq = 0.f;
    h.deps = std::numeric_limits<float>::infinity();
  } else {
    h.dsq = dsq;
    h.deps = deps;
  }
  h.lrwd = static_cast<float>(dlr * static_cast<double>(wd));
  h.exact = g_exact_group_params.load(std::memory_order_relaxed);
  return h;
}

coat_status check_tensor(const coat_tensor_desc& d, int index) {
  if (d.n < 0) return fail(COAT_ERR_INVALID_ARG, "tensor %d: n < 0", index);
  if (d.n == 0) return COAT_OK;
  const void* req[] = {d.master, d.grad, d.m_q, d.m_scale, d.m_k, d.v_q, d.v_scale, d.v_k};
  const char* names[] = {"master", "grad", "m_q", "m_scale", "m_k", "v_q", "v_scale", "v_k"};
  for (int i = 0; i < 8; ++i) {
    if (!req[i]) return fail(COAT_ERR_INVALID_ARG, "tensor %d: %s is NULL", index, names[i]);
    if (!aligned(req[i], 16))
      return fail(COAT_ERR_MISALIGNED, "tensor %d: %s is not 16-byte aligned", index, names[i]);
  }
  if (d.weight_bf16_out && !aligned(d.weight_bf16_out, 16))
    return fail(COAT_ERR_MISALIGNED, "tensor %d: weight_bf16_out is not 16-byte aligned", index);
  return COAT_OK;
}

coat::TensorArgs to_args(const coat_tensor_desc& d, int64_t tile_begin) {
  coat::TensorArgs t;
  t.master = d.master;
  t.wout = d.weight_bf16_out;
  t.grad = d.grad;
  t.mq = d.m_q;
  t.ms = d.m_scale;
  t.mk = d.m_k;
  t.vq = d.v_q;
  t.vs = d.v_scale;
  t.vk = d.v_k;
  t.n = d.n;
  const int64_t groups = (d.n + 127) / 128;
  const int64_t tg = coat::step_tile_groups();
  t.tiles = (groups + tg - 1) / tg;
  t.tile_begin = tile_begin;
  t.wd_scale = 1.0f;
  return t;
}

}  // namespace

// ---------------------------------------------------------------------------
// public ABI
// ---------------------------------------------------------------------------
extern "C" {

const char* coat_last_error(void) { return g_last_error.c_str(); }

int coat_version(void) { return 10400; }   // 1.4: ZeRO-1 layout and clipping across ranks; 1.3: clipping pre-step, FP8 layers

coat_status coat_fp8_encode(const float* y, int64_t n, coat_fmt fmt, uint8_t* q, cudaStream_t stream) {
  if (n < 0) return fail(COAT_ERR_INVALID_ARG, "coat_fp8_encode: n < 0");
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "coat_fp8_encode: bad fmt %d", int(fmt));
  if (n == 0) return COAT_OK;
  if (!y || !q) return fail(COAT_ERR_INVALID_ARG, "coat_fp8_encode: NULL pointer");
  if (!aligned(y, 4)) return fail(COAT_ERR_MISALIGNED, "coat_fp8_encode: y not 4-byte aligned");
  cudaError_t e = coat::launch_fp8_encode(y, n, fmt, q, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, "coat_fp8_encode");
}

coat_status coat_fp8_decode(const uint8_t* q, int64_t n, coat_fmt fmt, float* out, cudaStream_t stream) {
  if (n < 0) return fail(COAT_ERR_INVALID_ARG, "coat_fp8_decode: n < 0");
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "coat_fp8_decode: bad fmt %d", int(fmt));
  if (n == 0) return COAT_OK;
  if (!q || !out) return fail(COAT_ERR_INVALID_ARG, "coat_fp8_decode: NULL pointer");
  if (!aligned(out, 4)) return fail(COAT_ERR_MISALIGNED, "coat_fp8_decode: out not 4-byte aligned");
  cudaError_t e = coat::launch_fp8_decode(q, n, fmt, out, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, "coat_fp8_decode");
}

static coat_status check_groups(const char* fn, int gr, int gc) {
  if (gr < 1 || gc < 1) return fail(COAT_ERR_INVALID_ARG, "%s: group shape must be positive", fn);
  if (!((gr == 1 && gc == 128) || (gr == 128 && gc == 128)))
    return fail(COAT_ERR_UNSUPPORTED, "%s: group %dx%d not supported (1x128 or 128x128)", fn, gr, gc);
  return COAT_OK;
}

coat_status coat_group_quantize(const void* x, coat_dtype xt, int64_t rows, int64_t cols,
                                int64_t ld_x, int group_rows, int group_cols, int expand,
                                coat_fmt fmt, uint8_t* q, int64_t ld_q, float* scale, float* k,
                                cudaStream_t stream) {
  const char* fn = "coat_group_quantize";
  if (rows < 0 || cols < 0) return fail(COAT_ERR_INVALID_ARG, "%s: negative shape", fn);
  if (!valid_dtype(xt)) return fail(COAT_ERR_INVALID_ARG, "%s: bad dtype %d", fn, int(xt));
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "%s: bad fmt %d", fn, int(fmt));
  if (expand != 0 && expand != 1) return fail(COAT_ERR_INVALID_ARG, "%s: expand must be 0 or 1", fn);
  coat_status st = check_groups(fn, group_rows, group_cols);
  if (st != COAT_OK) return st;
  if (ld_x < cols || ld_q < cols) return fail(COAT_ERR_INVALID_ARG, "%s: leading dimension < cols", fn);
  if (rows == 0 || cols == 0) return COAT_OK;
  if (!x || !q || !scale || !k) return fail(COAT_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned(x, 16) || !aligned(q, 16)) return fail(COAT_ERR_MISALIGNED, "%s: x and q must be 16-byte aligned", fn);
  if (rows > 1 && ((ld_x * int64_t(dtype_size(xt))) % 16 != 0 || ld_q % 16 != 0))
    return fail(COAT_ERR_MISALIGNED, "%s: row strides must be multiples of 16 bytes", fn);
  if (!aligned(scale, 4) || !aligned(k, 4)) return fail(COAT_ERR_MISALIGNED, "%s: scale/k not 4-byte aligned", fn);
  unsigned* err = nullptr;
  cudaError_t e = coat::device_error_ptr(&err);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  e = coat::launch_group_quantize(x, xt, rows, cols, ld_x, group_rows, expand, fmt, q, ld_q, scale,
                                  k, err, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_group_dequantize(const uint8_t* q, int64_t ld_q, const float* scale, const float* k,
                                  int64_t rows, int64_t cols, int group_rows, int group_cols,
                                  coat_fmt fmt, void* out, coat_dtype ot, int64_t ld_out,
                                  cudaStream_t stream) {
  const char* fn = "coat_group_dequantize";
  if (rows < 0 || cols < 0) return fail(COAT_ERR_INVALID_ARG, "%s: negative shape", fn);
  if (!valid_dtype(ot)) return fail(COAT_ERR_INVALID_ARG, "%s: bad dtype %d", fn, int(ot));
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "%s: bad fmt %d", fn, int(fmt));
  coat_status st = check_groups(fn, group_rows, group_cols);
  if (st != COAT_OK) return st;
  if (ld_out < cols || ld_q < cols) return fail(COAT_ERR_INVALID_ARG, "%s: leading dimension < cols", fn);
  if (rows == 0 || cols == 0) return COAT_OK;
  if (!out || !q || !scale || !k) return fail(COAT_ERR_INVALID_ARG, "%s: NULL pointer", fn);
  if (!aligned(out, 16) || !aligned(q, 16)) return fail(COAT_ERR_MISALIGNED, "%s: q and out must be 16-byte aligned", fn);
  if (rows > 1 && ((ld_out * int64_t(dtype_size(ot))) % 16 != 0 || ld_q % 16 != 0))
    return fail(COAT_ERR_MISALIGNED, "%s: row strides must be multiples of 16 bytes", fn);
  if (!aligned(scale, 4) || !aligned(k, 4)) return fail(COAT_ERR_MISALIGNED, "%s: scale/k not 4-byte aligned", fn);
  cudaError_t e = coat::launch_group_dequantize(q, ld_q, scale, k, rows, cols, group_rows,
                                                group_cols, fmt, out, ot, ld_out, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

static coat_status check_act(const char* fn, const char* name, const coat_fp8_act* a, int64_t rows,
                             int64_t cols) {
  if (!a) return fail(COAT_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
  const int64_t ng = (cols + 127) / 128;
  if (a->ldq < cols || a->lds < ng)
    return fail(COAT_ERR_INVALID_ARG, "%s: %s strides too small (ldq >= cols, lds >= groups)", fn, name);
  if (rows == 0 || cols == 0) return COAT_OK;
  if (!a->q || !a->scale || !a->k) return fail(COAT_ERR_INVALID_ARG, "%s: %s has a NULL array", fn, name);
  if (!aligned(a->q, 16) || (rows > 1 && a->ldq % 16 != 0))
    return fail(COAT_ERR_MISALIGNED, "%s: %s codes need 16-byte alignment and row stride", fn, name);
  if (!aligned(a->scale, 4) || !aligned(a->k, 4))
    return fail(COAT_ERR_MISALIGNED, "%s: %s scale/k not 4-byte aligned", fn, name);
  return COAT_OK;
}

static coat_status check_bf16(const char* fn, const char* name, const void* p, int64_t ld,
                              int64_t rows, int64_t cols) {
  if (ld < cols) return fail(COAT_ERR_INVALID_ARG, "%s: %s leading dimension < cols", fn, name);
  if (rows == 0 || cols == 0) return COAT_OK;
  if (!p) return fail(COAT_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
  if (!aligned(p, 16) || (rows > 1 && (ld * 2) % 16 != 0))
    return fail(COAT_ERR_MISALIGNED, "%s: %s needs 16-byte alignment and row stride", fn, name);
  return COAT_OK;
}

static coat::ActArgs act_args(const coat_fp8_act* a) {
  return coat::ActArgs{a->q, a->scale, a->k, a->ldq, a->lds};
}

coat_status coat_swiglu_fp8_forward(const coat_fp8_act* gate, const coat_fp8_act* up, int64_t rows,
                                    int64_t cols, coat_fmt fmt, int expand_out,
                                    const coat_fp8_act* out, cudaStream_t stream) {
  const char* fn = "coat_swiglu_fp8_forward";
  if (rows < 0 || cols < 0) return fail(COAT_ERR_INVALID_ARG, "%s: negative shape", fn);
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "%s: bad fmt %d", fn, int(fmt));
  if (expand_out != 0 && expand_out != 1)
    return fail(COAT_ERR_INVALID_ARG, "%s: expand_out must be 0 or 1", fn);
  if (cols % 16 != 0) return fail(COAT_ERR_UNSUPPORTED, "%s: cols must be a multiple of 16", fn);
  if (cols > (int64_t(1) << 30)) return fail(COAT_ERR_UNSUPPORTED, "%s: cols above 2^30", fn);
  coat_status st = check_act(fn, "gate", gate, rows, cols);
  if (st == COAT_OK) st = check_act(fn, "up", up, rows, cols);
  if (st == COAT_OK) st = check_act(fn, "out", out, rows, cols);
  if (st != COAT_OK) return st;
  if (rows == 0 || cols == 0) return COAT_OK;
  cudaError_t e = coat::launch_swiglu_fp8_forward(act_args(gate), act_args(up), rows, cols, fmt,
                                                  expand_out, act_args(out), stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_swiglu_fp8_backward(const uint16_t* grad_out, int64_t ld_grad_out,
                                     const coat_fp8_act* gate, const coat_fp8_act* up,
                                     int64_t rows, int64_t cols, coat_fmt fmt,
                                     uint16_t* grad_gate, int64_t ld_grad_gate, uint16_t* grad_up,
                                     int64_t ld_grad_up, cudaStream_t stream) {
  const char* fn = "coat_swiglu_fp8_backward";
  if (rows < 0 || cols < 0) return fail(COAT_ERR_INVALID_ARG, "%s: negative shape", fn);
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "%s: bad fmt %d", fn, int(fmt));
  if (cols % 16 != 0) return fail(COAT_ERR_UNSUPPORTED, "%s: cols must be a multiple of 16", fn);
  coat_status st = check_act(fn, "gate", gate, rows, cols);
  if (st == COAT_OK) st = check_act(fn, "up", up, rows, cols);
  if (st == COAT_OK) st = check_bf16(fn, "grad_out", grad_out, ld_grad_out, rows, cols);
  if (st == COAT_OK) st = check_bf16(fn, "grad_gate", grad_gate, ld_grad_gate, rows, cols);
  if (st == COAT_OK) st = check_bf16(fn, "grad_up", grad_up, ld_grad_up, rows, cols);
  if (st != COAT_OK) return st;
  if (rows == 0 || cols == 0) return COAT_OK;
  cudaError_t e = coat::launch_swiglu_fp8_backward(grad_out, ld_grad_out, act_args(gate),
                                                   act_args(up), rows, cols, fmt, grad_gate,
                                                   ld_grad_gate, grad_up, ld_grad_up, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

static coat_status check_rms_shape(const char* fn, int64_t rows, int64_t d, float eps,
                                   coat_fmt fmt, const uint16_t* w) {
  if (rows < 0 || d < 0) return fail(COAT_ERR_INVALID_ARG, "%s: negative shape", fn);
  if (!valid_fmt(fmt)) return fail(COAT_ERR_INVALID_ARG, "%s: bad fmt %d", fn, int(fmt));
  if (!std::isfinite(eps) || !(eps > 0.f)) return fail(COAT_ERR_INVALID_ARG, "%s: eps must be finite and > 0", fn);
  if (d % 128 != 0 || d > coat::rmsnorm_max_d())
    return fail(COAT_ERR_UNSUPPORTED, "%s: d must be a multiple of 128, at most %lld", fn,
                static_cast<long long>(coat::rmsnorm_max_d()));
  if (d > 0 && !w) return fail(COAT_ERR_INVALID_ARG, "%s: w is NULL", fn);
  if (d > 0 && !aligned(w, 16)) return fail(COAT_ERR_MISALIGNED, "%s: w is not 16-byte aligned", fn);
  return COAT_OK;
}

coat_status coat_rmsnorm_fp8_forward(const coat_fp8_act* x, const uint16_t* w, int64_t rows,
                                     int64_t d, float eps, coat_fmt fmt, int expand_out,
                                     const coat_fp8_act* out, cudaStream_t stream) {
  const char* fn = "coat_rmsnorm_fp8_forward";
  coat_status st = check_rms_shape(fn, rows, d, eps, fmt, w);
  if (st != COAT_OK) return st;
  if (expand_out != 0 && expand_out != 1)
    return fail(COAT_ERR_INVALID_ARG, "%s: expand_out must be 0 or 1", fn);
  st = check_act(fn, "x", x, rows, d);
  if (st == COAT_OK) st = check_act(fn, "out", out, rows, d);
  if (st != COAT_OK) return st;
  if (rows == 0 || d == 0) return COAT_OK;
  cudaError_t e = coat::launch_rmsnorm_fp8_forward(act_args(x), w, rows, d, eps, fmt, expand_out,
                                                   act_args(out), stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_rmsnorm_fp8_workspace_size(int64_t d, size_t* bytes) {
  const char* fn = "coat_rmsnorm_fp8_workspace_size";
  if (!bytes) return fail(COAT_ERR_INVALID_ARG, "%s: bytes is NULL", fn);
  *bytes = 0;
  if (d < 0) return fail(COAT_ERR_INVALID_ARG, "%s: negative d", fn);
  if (d % 128 != 0 || d > coat::rmsnorm_max_d())
    return fail(COAT_ERR_UNSUPPORTED, "%s: d must be a multiple of 128, at most %lld", fn,
                static_cast<long long>(coat::rmsnorm_max_d()));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  *bytes = coat::rmsnorm_workspace_bytes(dev, d);
  return COAT_OK;
}

coat_status coat_rmsnorm_fp8_backward(const uint16_t* dy, int64_t ld_dy, const coat_fp8_act* x,
                                      const uint16_t* w, int64_t rows, int64_t d, float eps,
                                      coat_fmt fmt, uint16_t* dx, int64_t ld_dx, float* dw,
                                      void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
  const char* fn = "coat_rmsnorm_fp8_backward";
  coat_status st = check_rms_shape(fn, rows, d, eps, fmt, w);
  if (st != COAT_OK) return st;
  st = check_act(fn, "x", x, rows, d);
  if (st == COAT_OK) st = check_bf16(fn, "dy", dy, ld_dy, rows, d);
  if (st == COAT_OK) st = check_bf16(fn, "dx", dx, ld_dx, rows, d);
  if (st != COAT_OK) return st;
  if (d == 0) return COAT_OK;
  if (!dw) return fail(COAT_ERR_INVALID_ARG, "%s: dw is NULL", fn);
  if (!aligned(dw, 4)) return fail(COAT_ERR_MISALIGNED, "%s: dw is not 4-byte aligned", fn);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  const size_t need = coat::rmsnorm_workspace_bytes(dev, d);
  if (rows > 0) {
    if (!workspace || workspace_bytes < need)
      return fail(COAT_ERR_INVALID_ARG, "%s: workspace needs %zu bytes", fn, need);
    if (!aligned(workspace, 16)) return fail(COAT_ERR_MISALIGNED, "%s: workspace is not 16-byte aligned", fn);
  }
  e = coat::launch_rmsnorm_fp8_backward(dy, ld_dy, act_args(x), w, rows, d, eps, fmt, dx, ld_dx,
                                        dw, static_cast<float*>(workspace), stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_adamw_step(float* master, uint16_t* weight_bf16_out, const uint16_t* grad,
                            uint8_t* m_q, float* m_scale, float* m_k, uint8_t* v_q, float* v_scale,
                            float* v_k, int64_t n, int group, float lr, float beta1, float beta2,
                            float eps, float wd, int64_t step, coat_fmt fmt_m, coat_fmt fmt_v,
                            cudaStream_t stream) {
  if (n < 0) return fail(COAT_ERR_INVALID_ARG, "coat_adamw_step: n < 0");
  if (group < 1) return fail(COAT_ERR_INVALID_ARG, "coat_adamw_step: group must be positive");
  if (group != 128) return fail(COAT_ERR_UNSUPPORTED, "coat_adamw_step: group %d not supported (128)", group);
  if (!valid_fmt(fmt_m) || !valid_fmt(fmt_v)) return fail(COAT_ERR_INVALID_ARG, "coat_adamw_step: bad fmt");
  coat_status st = check_hyper(lr, beta1, beta2, eps, wd, step);
  if (st != COAT_OK) return st;
  const coat_tensor_desc d = {master, weight_bf16_out, grad, m_q, m_scale, m_k, v_q, v_scale, v_k, n};
  st = check_tensor(d, 0);
  if (st != COAT_OK) return st;
  if (n == 0) return COAT_OK;
  unsigned* err = nullptr;
  cudaError_t e = coat::device_error_ptr(&err);
  if (e != cudaSuccess) return cuda_fail(e, "coat_adamw_step");
  e = coat::launch_adamw_single(to_args(d, 0), fmt_m, fmt_v,
                                make_hyper(lr, beta1, beta2, eps, wd, step), err, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, "coat_adamw_step");
}

}  // extern "C"

namespace {

// Norm, coefficient and found-Inf of a clip record from its sum of squares:
// the arithmetic of the gradient-norm pass's last CTA (double sqrt and
// division, both correctly rounded, then FP32), so that a record finalised
// here equals one the pass writes for the same sum.
__global__ void clip_finalize_kernel(coat::ClipRecord* rec, float max_norm) {
  const double total = rec->sumsq;
  const double c = static_cast<double>(max_norm) / (sqrt(total) + 1e-6);
  rec->norm = static_cast<float>(sqrt(total));
  rec->coef = static_cast<float>(c < 1.0 ? c : 1.0);
  rec->found_inf = isfinite(total) ? 0 : 1;
  rec->reserved = 0;
}

}  // namespace

struct coat_multi_plan {
  coat::TensorArgs* d_descs = nullptr;  // device copy of the descriptors (tile_begin ascending)
  double* d_partials = nullptr;         // gradient-norm pass: one slot per CTA
  unsigned* d_ticket = nullptr;         // gradient-norm pass: CTAs finished (0 between calls)
  int64_t total_tiles = 0;
  int64_t total_elements = 0;
  int num = 0;
  int fmt_m = 0, fmt_v = 0;
  int device = 0;
};

extern "C" {

coat_status coat_multi_plan_create(const coat_tensor_desc* host_descs, int num, int group,
                                   coat_fmt fmt_m, coat_fmt fmt_v, cudaStream_t stream,
                                   coat_multi_plan_t* out_plan) {
  const char* fn = "coat_multi_plan_create";
  if (!out_plan) return fail(COAT_ERR_INVALID_ARG, "%s: out_plan is NULL", fn);
  *out_plan = nullptr;
  if (!host_descs || num < 1) return fail(COAT_ERR_INVALID_ARG, "%s: need num >= 1 descriptors", fn);
  if (group < 1) return fail(COAT_ERR_INVALID_ARG, "%s: group must be positive", fn);
  if (group != 128) return fail(COAT_ERR_UNSUPPORTED, "%s: group %d not supported (128)", fn, group);
  if (!valid_fmt(fmt_m) || !valid_fmt(fmt_v)) return fail(COAT_ERR_INVALID_ARG, "%s: bad fmt", fn);
  std::vector<coat::TensorArgs> descs(static_cast<size_t>(num));
  int64_t tiles = 0, elems = 0;
  for (int i = 0; i < num; ++i) {
    coat_status st = check_tensor(host_descs[i], i);
    if (st != COAT_OK) return st;
    descs[i] = to_args(host_descs[i], tiles);
    tiles += descs[i].tiles;
    elems += host_descs[i].n;
  }

  coat_multi_plan* p = new (std::nothrow) coat_multi_plan;
  if (!p) return fail(COAT_ERR_NOMEM, "%s: host allocation failed", fn);
  // one allocation: descriptor table | gradient-norm slots | ticket
  const size_t desc_bytes = sizeof(coat::TensorArgs) * num;
  const size_t off_partials = (desc_bytes + 255) / 256 * 256;
  void* mem = nullptr;
  cudaError_t e = cudaGetDevice(&p->device);
  const size_t slot_bytes =
      e == cudaSuccess ? sizeof(double) * static_cast<size_t>(coat::grad_sumsq_slots(p->device)) : 0;
  const size_t off_ticket = off_partials + (slot_bytes + 255) / 256 * 256;
  if (e == cudaSuccess) e = cudaMalloc(&mem, off_ticket + 256);
  if (e != cudaSuccess) {
    delete p;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? fail(COAT_ERR_NOMEM, "%s: device allocation failed", fn)
                                          : cuda_fail(e, fn);
  }
  p->d_descs = static_cast<coat::TensorArgs*>(mem);
  p->d_partials = reinterpret_cast<double*>(static_cast<char*>(mem) + off_partials);
  p->d_ticket = reinterpret_cast<unsigned*>(static_cast<char*>(mem) + off_ticket);
  e = cudaMemcpyAsync(p->d_descs, descs.data(), desc_bytes, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(p->d_ticket, 0, sizeof(unsigned), stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // the host vector dies on return
  if (e != cudaSuccess) {
    cudaFree(mem);
    delete p;
    return cuda_fail(e, fn);
  }
  p->total_tiles = tiles;
  p->total_elements = elems;
  p->num = num;
  p->fmt_m = fmt_m;
  p->fmt_v = fmt_v;
  *out_plan = p;
  return COAT_OK;
}

coat_status coat_adamw_step_multi(coat_multi_plan_t plan, float lr, float beta1, float beta2,
                                  float eps, float wd, int64_t step, cudaStream_t stream) {
  if (!plan) return fail(COAT_ERR_INVALID_ARG, "coat_adamw_step_multi: plan is NULL");
  coat_status st = check_hyper(lr, beta1, beta2, eps, wd, step);
  if (st != COAT_OK) return st;
  if (plan->total_tiles == 0) return COAT_OK;
  unsigned* err = nullptr;
  cudaError_t e = coat::device_error_ptr(&err);
  if (e != cudaSuccess) return cuda_fail(e, "coat_adamw_step_multi");
  e = coat::launch_adamw_multi(plan->d_descs, plan->num, plan->total_tiles, plan->fmt_m,
                               plan->fmt_v, make_hyper(lr, beta1, beta2, eps, wd, step), nullptr,
                               err, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, "coat_adamw_step_multi");
}

static_assert(sizeof(coat_grad_clip) == sizeof(coat::ClipRecord) &&
                  offsetof(coat_grad_clip, sumsq) == offsetof(coat::ClipRecord, sumsq) &&
                  offsetof(coat_grad_clip, norm) == offsetof(coat::ClipRecord, norm) &&
                  offsetof(coat_grad_clip, coef) == offsetof(coat::ClipRecord, coef) &&
                  offsetof(coat_grad_clip, found_inf) == offsetof(coat::ClipRecord, found_inf),
              "coat_grad_clip and ClipRecord must share one layout");

coat_status coat_multi_plan_grad_norm(coat_multi_plan_t plan, float max_norm,
                                      coat_grad_clip* d_clip, cudaStream_t stream) {
  const char* fn = "coat_multi_plan_grad_norm";
  if (!plan) return fail(COAT_ERR_INVALID_ARG, "%s: plan is NULL", fn);
  if (!d_clip) return fail(COAT_ERR_INVALID_ARG, "%s: d_clip is NULL", fn);
  if (!aligned(d_clip, 8)) return fail(COAT_ERR_MISALIGNED, "%s: d_clip is not 8-byte aligned", fn);
  if (!(max_norm > 0.f)) return fail(COAT_ERR_INVALID_ARG, "%s: max_norm must be > 0", fn);
  cudaError_t e = coat::launch_grad_sumsq(plan->d_descs, plan->num, plan->total_tiles,
                                          plan->d_partials, plan->d_ticket, max_norm,
                                          reinterpret_cast<coat::ClipRecord*>(d_clip), stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_grad_clip_finalize(coat_grad_clip* d_clip, float max_norm,
                                    cudaStream_t stream) {
  const char* fn = "coat_grad_clip_finalize";
  if (!d_clip) return fail(COAT_ERR_INVALID_ARG, "%s: d_clip is NULL", fn);
  if (!aligned(d_clip, 8)) return fail(COAT_ERR_MISALIGNED, "%s: d_clip is not 8-byte aligned", fn);
  if (!(max_norm > 0.f)) return fail(COAT_ERR_INVALID_ARG, "%s: max_norm must be > 0", fn);
  clip_finalize_kernel<<<1, 1, 0, stream>>>(reinterpret_cast<coat::ClipRecord*>(d_clip), max_norm);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_adamw_step_multi_clipped(coat_multi_plan_t plan, float lr, float beta1,
                                          float beta2, float eps, float wd, int64_t step,
                                          const coat_grad_clip* d_clip, cudaStream_t stream) {
  const char* fn = "coat_adamw_step_multi_clipped";
  if (!plan) return fail(COAT_ERR_INVALID_ARG, "%s: plan is NULL", fn);
  if (!d_clip) return fail(COAT_ERR_INVALID_ARG, "%s: d_clip is NULL", fn);
  if (!aligned(d_clip, 8)) return fail(COAT_ERR_MISALIGNED, "%s: d_clip is not 8-byte aligned", fn);
  coat_status st = check_hyper(lr, beta1, beta2, eps, wd, step);
  if (st != COAT_OK) return st;
  if (plan->total_tiles == 0) return COAT_OK;
  unsigned* err = nullptr;
  cudaError_t e = coat::device_error_ptr(&err);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  e = coat::launch_adamw_multi(plan->d_descs, plan->num, plan->total_tiles, plan->fmt_m,
                               plan->fmt_v, make_hyper(lr, beta1, beta2, eps, wd, step),
                               reinterpret_cast<const coat::ClipRecord*>(d_clip), err, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_multi_plan_set_wd_scale(coat_multi_plan_t plan, const float* host_wd_scale,
                                        cudaStream_t stream) {
  const char* fn = "coat_multi_plan_set_wd_scale";
  if (!plan) return fail(COAT_ERR_INVALID_ARG, "%s: plan is NULL", fn);
  if (!host_wd_scale) return fail(COAT_ERR_INVALID_ARG, "%s: host_wd_scale is NULL", fn);
  for (int i = 0; i < plan->num; ++i)
    if (!std::isfinite(host_wd_scale[i]) || host_wd_scale[i] < 0.f)
      return fail(COAT_ERR_INVALID_ARG, "%s: wd_scale[%d] must be finite and >= 0", fn, i);
  // one strided copy into the wd_scale field of every device descriptor
  cudaError_t e = cudaMemcpy2DAsync(&plan->d_descs[0].wd_scale, sizeof(coat::TensorArgs),
                                    host_wd_scale, sizeof(float), sizeof(float), plan->num,
                                    cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);   // the host array may go on return
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_multi_plan_destroy(coat_multi_plan_t plan) {
  if (!plan) return COAT_OK;
  cudaError_t e = cudaFree(plan->d_descs);
  delete plan;
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, "coat_multi_plan_destroy");
}

coat_status coat_multi_plan_info(coat_multi_plan_t plan, int64_t* total_elements, int* num_tensors) {
  if (!plan) return fail(COAT_ERR_INVALID_ARG, "coat_multi_plan_info: plan is NULL");
  if (total_elements) *total_elements = plan->total_elements;
  if (num_tensors) *num_tensors = plan->num;
  return COAT_OK;
}

coat_status coat_zero1_layout(const int64_t* sizes, int num_tensors, int group, int world_size,
                              int rank, coat_shard_piece* pieces, int max_pieces,
                              int* num_pieces, int64_t* shard_elems, int64_t* flat_elems,
                              int64_t* flat_offsets) {
  const char* fn = "coat_zero1_layout";
  if (!sizes || !num_pieces || !shard_elems || !flat_elems)
    return fail(COAT_ERR_INVALID_ARG, "%s: NULL argument", fn);
  if (num_tensors < 1) return fail(COAT_ERR_INVALID_ARG, "%s: num_tensors must be >= 1", fn);
  if (group != 128) return fail(COAT_ERR_UNSUPPORTED, "%s: group %d not supported (128)", fn, group);
  if (world_size < 1 || rank < 0 || rank >= world_size)
    return fail(COAT_ERR_INVALID_ARG, "%s: need world_size >= 1 and 0 <= rank < world_size", fn);
  if (max_pieces < 0 || (max_pieces > 0 && !pieces))
    return fail(COAT_ERR_INVALID_ARG, "%s: pieces is NULL or max_pieces < 0", fn);
  // Blocks of 4 groups: a piece's first group then has its four per-group
  // floats on a 16-byte boundary, as the step's descriptors require.
  const int64_t blk = 4 * static_cast<int64_t>(group);
  constexpr int64_t kMaxBlocks = std::numeric_limits<int64_t>::max() / 512 / 2;
  int64_t total_blocks = 0;
  for (int i = 0; i < num_tensors; ++i) {
    if (sizes[i] < 0) return fail(COAT_ERR_INVALID_ARG, "%s: sizes[%d] < 0", fn, i);
    if (sizes[i] > kMaxBlocks * blk) return fail(COAT_ERR_INVALID_ARG, "%s: too many elements", fn);
    total_blocks += (sizes[i] + blk - 1) / blk;
    if (total_blocks > kMaxBlocks) return fail(COAT_ERR_INVALID_ARG, "%s: too many elements", fn);
  }
  const int64_t shard = (total_blocks + world_size - 1) / world_size * blk;
  const int64_t lo_e = shard * rank, hi_e = shard * (rank + 1);
  // Pieces: the intersection of [lo_e, hi_e) with each tensor's flat range.
  int count = 0;
  int64_t off = 0;
  for (int i = 0; i < num_tensors; ++i) {
    if (flat_offsets) flat_offsets[i] = off;
    const int64_t lo = std::max(off, lo_e), hi = std::min(off + sizes[i], hi_e);
    if (lo < hi) {
      if (count < max_pieces) {
        coat_shard_piece& pc = pieces[count];
        pc.tensor = i;
        pc.reserved = 0;
        pc.elem_begin = lo - off;
        pc.n_elems = hi - lo;
        pc.shard_begin = lo - lo_e;
      }
      ++count;
    }
    off += (sizes[i] + blk - 1) / blk * blk;
  }
  *num_pieces = count;
  *shard_elems = shard;
  *flat_elems = shard * world_size;
  if (count > max_pieces)
    return fail(COAT_ERR_INVALID_ARG, "%s: %d pieces needed, max_pieces is %d", fn, count,
                max_pieces);
  return COAT_OK;
}

coat_status coat_selftest_wait_timeout(int64_t budget_cycles, cudaStream_t stream) {
  const char* fn = "coat_selftest_wait_timeout";
  constexpr int64_t kMaxBudget = 2000000000;   // the kernels' own bound, about one second
  if (budget_cycles < 1000 || budget_cycles > kMaxBudget)
    return fail(COAT_ERR_INVALID_ARG, "%s: budget_cycles must be in [1000, %lld]", fn,
                static_cast<long long>(kMaxBudget));
  unsigned* err = nullptr;
  cudaError_t e = coat::device_error_ptr(&err);
  if (e == cudaSuccess) e = coat::launch_wait_timeout_selftest(budget_cycles, err, stream);
  return e == cudaSuccess ? COAT_OK : cuda_fail(e, fn);
}

coat_status coat_check_device_error(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "coat_check_device_error");
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_coat_device_error, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "coat_check_device_error");
  // failed index checks of the checked build (each read clears its count)
  unsigned fs = 0, fc = 0, ff = 0;
  if (e == cudaSuccess) e = coat::index_faults_step(&fs);
  if (e == cudaSuccess) e = coat::index_faults_codec(&fc);
  if (e == cudaSuccess) e = coat::index_faults_flow(&ff);
  if (e != cudaSuccess) return cuda_fail(e, "coat_check_device_error");
  if (v != 0) {
    const unsigned zero = 0;
    cudaMemcpyToSymbol(g_coat_device_error, &zero, sizeof(zero));
    return fail(COAT_ERR_TIMEOUT, "a kernel gave up a bounded wait (device error bits 0x%x)", v);
  }
  if (fs + fc + ff != 0)
    return fail(COAT_ERR_DEVICE_CHECK,
                "checked build: %u device index checks failed (step %u, codec %u, layers %u)",
                fs + fc + ff, fs, fc, ff);
  return COAT_OK;
}

int coat_set_exact_group_params(int on) {
  return g_exact_group_params.exchange(on ? 1 : 0);
}

int coat_build_checked(void) {
#ifdef COAT_DEBUG
  return 1;
#else
  return 0;
#endif
}

}  // extern "C"

// ---------------------------------------------------------------------------
// coat_adamw_step_multi_noalloc: the multi-tensor step for callers that cannot
// allocate device memory.  Its descriptor table lives in a fixed file-scope
// device array instead of a plan's cudaMalloc'd table.
// ---------------------------------------------------------------------------
namespace {

struct NoAllocScratch {
  coat::TensorArgs descs[COAT_NOALLOC_MAX_TENSORS];
};
// The size include/coat.h states for the array (104 bytes per descriptor).
static_assert(sizeof(coat::TensorArgs) == 104, "descriptor size stated in coat.h");
static_assert(sizeof(NoAllocScratch) == 106496, "array size stated in coat.h");

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoAllocScratch)];

// Descriptors travel to the array as kernel parameters, a chunk per launch:
// the launch copies its parameters when it is enqueued, so no host buffer has
// to outlive the call and no pageable-memory copy (which may wait for earlier
// work on the stream) is involved.  32 descriptors keep the parameters below
// the classic 4 KB limit.
constexpr int kNoAllocChunk = 32;
struct NoAllocChunk {
  coat::TensorArgs d[kNoAllocChunk];
};
static_assert(sizeof(NoAllocChunk) + 16 <= 4096, "kernel parameter space");

__global__ void noalloc_stage_kernel(const NoAllocChunk chunk, int count, coat::TensorArgs* dst) {
  const int i = threadIdx.x;
  if (i < count) dst[i] = chunk.d[i];
}

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64];

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
cudaError_t noalloc_scratch_ptr(NoAllocScratch** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<NoAllocScratch*>(g_noalloc_ptr[dev]);
  return cudaSuccess;
}

bool noalloc_desc_ok(const coat_tensor_desc& d, coat_status* st) {
  if (d.n < 0) { *st = COAT_ERR_INVALID_ARG; return false; }
  if (d.n == 0) return true;
  const void* req[] = {d.master, d.grad, d.m_q, d.m_scale, d.m_k, d.v_q, d.v_scale, d.v_k};
  for (const void* p : req) {
    if (!p) { *st = COAT_ERR_INVALID_ARG; return false; }
    if (!aligned(p, 16)) { *st = COAT_ERR_MISALIGNED; return false; }
  }
  if (d.weight_bf16_out && !aligned(d.weight_bf16_out, 16)) { *st = COAT_ERR_MISALIGNED; return false; }
  return true;
}

}  // namespace

extern "C" coat_status coat_adamw_step_multi_noalloc(const coat_tensor_desc* host_descs, int num,
                                                     int group, float lr, float beta1,
                                                     float beta2, float eps, float wd,
                                                     int64_t step, coat_fmt fmt_m, coat_fmt fmt_v,
                                                     cudaStream_t stream) {
  if (!host_descs || num < 1) return COAT_ERR_INVALID_ARG;
  if (group < 1 || !valid_fmt(fmt_m) || !valid_fmt(fmt_v)) return COAT_ERR_INVALID_ARG;
  if (group != 128 || num > COAT_NOALLOC_MAX_TENSORS) return COAT_ERR_UNSUPPORTED;
  if (!std::isfinite(lr) || lr < 0.f || !(beta1 >= 0.f && beta1 < 1.f) ||
      !(beta2 >= 0.f && beta2 < 1.f) || !std::isfinite(eps) || !(eps > 0.f) ||
      !std::isfinite(wd) || wd < 0.f || step < 1)
    return COAT_ERR_INVALID_ARG;
  coat_status st = COAT_OK;
  for (int i = 0; i < num; ++i)
    if (!noalloc_desc_ok(host_descs[i], &st)) return st;

  NoAllocScratch* scratch = nullptr;
  unsigned* err = nullptr;
  if (noalloc_scratch_ptr(&scratch) != cudaSuccess || coat::device_error_ptr(&err) != cudaSuccess)
    return COAT_ERR_CUDA;

  // The table, chunk by chunk, each entry built exactly as a plan builds it.
  NoAllocChunk chunk = {};
  int64_t tiles = 0;
  for (int c0 = 0; c0 < num; c0 += kNoAllocChunk) {
    const int cn = num - c0 < kNoAllocChunk ? num - c0 : kNoAllocChunk;
    for (int j = 0; j < cn; ++j) {
      chunk.d[j] = to_args(host_descs[c0 + j], tiles);
      tiles += chunk.d[j].tiles;
    }
    noalloc_stage_kernel<<<1, kNoAllocChunk, 0, stream>>>(chunk, cn, scratch->descs + c0);
    if (cudaGetLastError() != cudaSuccess) return COAT_ERR_CUDA;
  }
  if (tiles == 0) return COAT_OK;
  const cudaError_t e =
      coat::launch_adamw_multi(scratch->descs, num, tiles, fmt_m, fmt_v,
                               make_hyper(lr, beta1, beta2, eps, wd, step), nullptr, err, stream);
  return e == cudaSuccess ? COAT_OK : COAT_ERR_CUDA;
}
