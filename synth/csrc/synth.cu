// Device side of the seeded input generator (see synth/__init__.py for the
// recipe).  Every step is an integer operation or one correctly rounded IEEE
// operation written as an explicit intrinsic, so the numbers match the NumPy
// host generator bit for bit.  Holds none of the optimizer's arithmetic.
//
// Philox4x32-10 follows its published definition (Salmon et al., SC'11).
#include <cstdint>
#include <cuda_runtime.h>

namespace {

enum : uint32_t { MASTER = 1, GRAD = 2, MSTATE = 3, VSTATE = 4, GSCALE = 5, ACT = 6,
                  ACT_OUTLIER = 7, WEIGHT = 8, MCODE = 9, VCODE = 10, GSTATE = 11 };

constexpr double kIH4Scale = 1.7320508075688772 / 4294967296.0;  // sqrt(3)/2^32
constexpr int64_t kIH4Centre = (int64_t(1) << 33) - 2;
constexpr uint32_t kOutlierThreshold = 4294967u;
constexpr int64_t kGroup = 128;

struct Words { uint32_t w0, w1, w2, w3; };

__device__ __forceinline__ Words philox10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                          uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return {c0, c1, c2, c3};
}

__device__ __forceinline__ Words draw(uint32_t seed, uint32_t stream, int64_t idx,
                                      uint32_t tensor, uint32_t step) {
  return philox10(static_cast<uint32_t>(idx & 0xFFFFFFFF), static_cast<uint32_t>(idx >> 32),
                  tensor, step, seed, stream);
}

__device__ __forceinline__ double ih4(const Words& u) {
  const int64_t s = int64_t(u.w0) + int64_t(u.w1) + int64_t(u.w2) + int64_t(u.w3) - kIH4Centre;
  return __dmul_rn(static_cast<double>(s), kIH4Scale);
}

__device__ __forceinline__ float loguniform(uint32_t u, float lo, float hi) {
  const uint32_t lb = __float_as_uint(lo), hb = __float_as_uint(hi);
  const uint32_t off = static_cast<uint32_t>((uint64_t(u) * uint64_t(hb - lb)) >> 32);
  return __uint_as_float(lb + off);
}

__device__ __forceinline__ uint16_t bf16_rne(float f) {
  const uint32_t u = __float_as_uint(f);
  return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

__device__ __forceinline__ float group_scale_of_group(uint32_t seed, uint32_t tensor, int64_t g) {
  const Words u = draw(seed, GSCALE, g, tensor, 0);
  return loguniform(u.w0, 1e-5f, 1e-2f);
}

__device__ __forceinline__ float group_scale(uint32_t seed, uint32_t tensor, int64_t i) {
  return group_scale_of_group(seed, tensor, i / kGroup);
}

__device__ __forceinline__ float unit24(uint32_t u) {
  return __fmul_rn(static_cast<float>(u >> 8), 5.9604644775390625e-08f);  // 2^-24
}

template <class F>
__global__ void fill_kernel(int64_t count, F f) {
  for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < count;
       t += int64_t(gridDim.x) * blockDim.x)
    f(t);
}

template <class F>
int launch(int64_t count, cudaStream_t s, F f) {
  if (count <= 0) return 0;
  const int threads = 256;
  int64_t blocks = (count + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  fill_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(count, f);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

extern "C" {

int synth_master(float* out, int64_t count, uint32_t seed, uint32_t tensor, int64_t start,
                 cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const double z = ih4(draw(seed, MASTER, start + t, tensor, 0));
    out[t] = __double2float_rn(__dmul_rn(0.02, z));
  });
}

int synth_grad(uint16_t* out, int64_t count, uint32_t seed, uint32_t tensor, uint32_t step,
               int64_t start, cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const int64_t i = start + t;
    const double z = ih4(draw(seed, GRAD, i, tensor, step));
    const float sg = group_scale(seed, tensor, i);
    out[t] = bf16_rne(__double2float_rn(__dmul_rn(static_cast<double>(sg), z)));
  });
}

int synth_m_warm(float* out, int64_t count, uint32_t seed, uint32_t tensor, int64_t start,
                 cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const int64_t i = start + t;
    const Words u = draw(seed, MSTATE, i, tensor, 0);
    const float sg = group_scale(seed, tensor, i);
    const float mag = loguniform(u.w0, __fmul_rn(sg, 1e-3f), sg);
    out[t] = (u.w1 >> 31) ? -mag : mag;
  });
}

int synth_v_warm(float* out, int64_t count, uint32_t seed, uint32_t tensor, int64_t start,
                 cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const int64_t i = start + t;
    const Words u = draw(seed, VSTATE, i, tensor, 0);
    const float sg = group_scale(seed, tensor, i);
    const float sg2 = __fmul_rn(sg, sg);
    out[t] = loguniform(u.w0, __fmul_rn(sg2, 0.1f), sg2);
  });
}

int synth_activations(uint16_t* out, int64_t count, uint32_t seed, uint32_t tensor,
                      int64_t start, cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const int64_t i = start + t;
    double z = ih4(draw(seed, ACT, i, tensor, 0));
    if (draw(seed, ACT_OUTLIER, i, tensor, 0).w0 < kOutlierThreshold) z = __dmul_rn(z, 100.0);
    out[t] = bf16_rne(__double2float_rn(z));
  });
}

int synth_weight(uint16_t* out, int64_t count, uint32_t seed, uint32_t tensor, int64_t start,
                 cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const double z = ih4(draw(seed, WEIGHT, start + t, tensor, 0));
    out[t] = bf16_rne(__double2float_rn(__dmul_rn(0.02, z)));
  });
}

int synth_state_codes(uint8_t* out, int64_t count, uint32_t seed, uint32_t tensor, uint32_t step,
                      int64_t start, int fmt, int is_signed, cudaStream_t s) {
  // E4M3 0x01-0x7E; E5M2 0x34-0x7B (the literal span); E5M2 full span 0x01-0x7B
  const uint32_t lo = fmt == 1 ? 0x34u : 0x01u, hi = fmt == 0 ? 0x7Eu : 0x7Bu;
  return launch(count, s, [=] __device__(int64_t t) {
    const Words u = draw(seed, is_signed ? MCODE : VCODE, start + t, tensor, step);
    uint32_t c = lo + u.w0 % (hi - lo + 1u);
    if (is_signed && (u.w1 >> 31)) c |= 0x80u;
    out[t] = static_cast<uint8_t>(c);
  });
}

int synth_state_groups(float* k_m, float* s_m, float* k_v, float* s_v, int64_t count, uint32_t seed,
                       uint32_t tensor, uint32_t step, int64_t gstart, cudaStream_t s) {
  return launch(count, s, [=] __device__(int64_t t) {
    const int64_t g = gstart + t;
    const Words u = draw(seed, GSTATE, g, tensor, step);
    const float sg = group_scale_of_group(seed, tensor, g);
    k_m[t] = __fadd_rn(__fmul_rn(0.7f, unit24(u.w0)), 1.5f);
    s_m[t] = __fmul_rn(sg, __fadd_rn(__fmul_rn(0.04f, unit24(u.w1)), 0.02f));
    k_v[t] = __fadd_rn(__fmul_rn(4.0f, unit24(u.w2)), 4.0f);
    s_v[t] = __fmul_rn(__fmul_rn(sg, sg), __fadd_rn(__fmul_rn(0.2f, unit24(u.w3)), 0.1f));
  });
}

}  // extern "C"
