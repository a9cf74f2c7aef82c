// codec.cu -- FP8 element codec and the per-group quantiser / dequantiser with
// dynamic range expansion, at the two granularities of the mixed-granularity
// activation path: 1x128 groups along a row (per token) and 128x128 blocks
// (weights).  Sources: [P1] "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍",
// sections "解决方案：动态范围扩展" and "解决方案：混合粒度FP8精度流"; [P4]
// "FP8量化训练实战指南", section "分块级缩放：精度优化的进阶方案" (1x128 tiles for
// activations and gradients, 128x128 blocks for weights, one scale per tile).
//
// All kernels are HBM-bound streaming kernels: 16-byte (or 8/4-byte)
// coalesced loads and stores, no shared-memory staging except the 256-entry
// log2 decode table, grids sized in multiples of the SM count.
#include <cstdint>
#include <cuda_runtime.h>

#include "coat_device.cuh"
#include "coat_internal.h"

namespace coat {
namespace {

// ---------------------------------------------------------------------------
// element codec
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void fp8_encode_kernel(const float* __restrict__ y, int64_t n, uint8_t* __restrict__ q) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float v = y[i];
    q[i] = static_cast<uint8_t>(enc_signed<FMT>(v, fabsf(v)));
  }
}

template <int FMT>
__global__ void fp8_decode_kernel(const uint8_t* __restrict__ q, int64_t n, float* __restrict__ out) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x)
    out[i] = dec_value<FMT>(q[i]);
}

// ---------------------------------------------------------------------------
// loading 4 contiguous elements of a row as float
// ---------------------------------------------------------------------------
template <int DT>
__device__ __forceinline__ void load4(const void* base, int64_t idx, int valid, float v[4]) {
  if (DT == 0) {
    const float* p = static_cast<const float*>(base) + idx;
    if (valid >= 4) {
      const float4 t = *reinterpret_cast<const float4*>(p);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = i < valid ? p[i] : 0.f;
    }
  } else {
    const uint16_t* p = static_cast<const uint16_t*>(base) + idx;
    if (valid >= 4) {
      const uint2 t = *reinterpret_cast<const uint2*>(p);
      v[0] = bf16lo(t.x); v[1] = bf16hi(t.x); v[2] = bf16lo(t.y); v[3] = bf16hi(t.y);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = i < valid ? __uint_as_float(uint32_t(p[i]) << 16) : 0.f;
    }
  }
}

__device__ __forceinline__ void store_codes4(uint8_t* q, uint32_t c[4], int valid) {
  if (valid >= 4) {
    *reinterpret_cast<uint32_t*>(q) = pack4(c[0], c[1], c[2], c[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < valid) q[i] = static_cast<uint8_t>(c[i]);
  }
}

__device__ __forceinline__ int clamp_valid(int64_t left) {
  return left <= 0 ? 0 : (left >= 4 ? 4 : static_cast<int>(left));
}

// ---------------------------------------------------------------------------
// 1 x 128 groups: 8 lanes per group, 16 elements per lane (4 chunks of 4),
// 4 groups per warp; group max / min-nonzero by 3 xor-shuffles.
// ---------------------------------------------------------------------------
template <int FMT, int DT>
__global__ void __launch_bounds__(256) quant_row_kernel(const void* __restrict__ x, int64_t rows,
                                                        int64_t cols, int64_t ldx, int expand,
                                                        uint8_t* __restrict__ q, int64_t ldq,
                                                        float* __restrict__ scale,
                                                        float* __restrict__ kk) {
  const int lane = threadIdx.x & 31, slot = lane >> 3, l = lane & 7;
  const int64_t nbc = (cols + kGroup - 1) / kGroup;
  const int64_t ngroups = rows * nbc;
  const int64_t warp0 = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = warp0; w * 4 < ngroups; w += nwarps) {
    const int64_t gidx = w * 4 + slot;
    const bool active = gidx < ngroups;
    const int64_t r = active ? gidx / nbc : 0, gc = active ? gidx % nbc : 0;
    float v[16];
    float M = 0.f;
    uint32_t mink = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c0 = gc * kGroup + 32 * j + 4 * l;
      const int valid = active ? clamp_valid(cols - c0) : 0;
      load4<DT>(x, r * ldx + c0, valid, &v[4 * j]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        M = fmaxf(M, fabsf(v[4 * j + i]));
        mink = min(mink, (__float_as_uint(v[4 * j + i]) & 0x7FFFFFFFu) - 1u);
      }
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, off));
      mink = min(mink, __shfl_xor_sync(0xFFFFFFFFu, mink, off));
    }
    float k, sr, invM;
    group_params<FMT>(M, __uint_as_float(mink + 1u), expand != 0, k, sr, invM);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c0 = gc * kGroup + 32 * j + 4 * l;
      const int valid = active ? clamp_valid(cols - c0) : 0;
      uint32_t c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        c[i] = enc_signed<FMT>(v[4 * j + i], codec_value<FMT>(v[4 * j + i], M, invM, k));
      if (valid > 0) store_codes4(q + r * ldq + c0, c, valid);
    }
    if (active && l == 0) {
      scale[gidx] = sr;
      kk[gidx] = k;
    }
  }
}

// ---------------------------------------------------------------------------
// 128 x 128 blocks: one 256-thread CTA per block; warp w takes rows
// 16w..16w+15 of the block, lane takes 4 columns; two-level reduction
// (shuffles, then shared memory across the 8 warps).
// ---------------------------------------------------------------------------
template <int FMT, int DT>
__global__ void __launch_bounds__(256) quant_block_kernel(const void* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ldx, int expand,
                                                          uint8_t* __restrict__ q, int64_t ldq,
                                                          float* __restrict__ scale,
                                                          float* __restrict__ kk) {
  __shared__ float sM[8];
  __shared__ uint32_t sK[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nbc = (cols + 127) / 128, nbr = (rows + 127) / 128;
  for (int64_t b = blockIdx.x; b < nbr * nbc; b += gridDim.x) {
    const int64_t br = b / nbc, bc = b % nbc;
    const int64_t c0 = bc * 128 + 4 * lane;
    const int cvalid = clamp_valid(cols - c0);
    float v[64];
    float M = 0.f;
    uint32_t mink = 0xFFFFFFFFu;
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
      const int64_t r = br * 128 + warp * 16 + rr;
      const int valid = r < rows ? cvalid : 0;
      load4<DT>(x, r * ldx + c0, valid, &v[4 * rr]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        M = fmaxf(M, fabsf(v[4 * rr + i]));
        mink = min(mink, (__float_as_uint(v[4 * rr + i]) & 0x7FFFFFFFu) - 1u);
      }
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, off));
      mink = min(mink, __shfl_xor_sync(0xFFFFFFFFu, mink, off));
    }
    __syncthreads();  // previous block's readers are done with sM / sK
    if (lane == 0) {
      sM[warp] = M;
      sK[warp] = mink;
    }
    __syncthreads();
    M = sM[0];
    mink = sK[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      M = fmaxf(M, sM[w]);
      mink = min(mink, sK[w]);
    }
    float k, sr, invM;
    group_params<FMT>(M, __uint_as_float(mink + 1u), expand != 0, k, sr, invM);
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
      const int64_t r = br * 128 + warp * 16 + rr;
      const int valid = r < rows ? cvalid : 0;
      uint32_t c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        c[i] = enc_signed<FMT>(v[4 * rr + i], codec_value<FMT>(v[4 * rr + i], M, invM, k));
      if (valid > 0) store_codes4(q + r * ldq + c0, c, valid);
    }
    if (threadIdx.x == 0) {
      scale[b] = sr;
      kk[b] = k;
    }
  }
}

// ---------------------------------------------------------------------------
// dequantise: one thread per 4 contiguous codes of a row (one group each).
// ---------------------------------------------------------------------------
template <int FMT, int OT>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ q, int64_t ldq,
                                                      const float* __restrict__ scale,
                                                      const float* __restrict__ kk, int64_t rows,
                                                      int64_t cols, int gr, int gc,
                                                      void* __restrict__ out, int64_t ldo) {
  __shared__ float tab[256];
  fill_log2_table<FMT>(tab);
  __syncthreads();
  const int64_t cpr = (cols + 3) / 4;  // chunks per row
  const int64_t nbc = (cols + gc - 1) / gc;
  for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < rows * cpr;
       t += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = t / cpr, c0 = (t % cpr) * 4;
    const int valid = clamp_valid(cols - c0);
    const int64_t g = (r / gr) * nbc + c0 / gc;
    const float invk = rcp_approx(kk[g]), s = scale[g];
    uint32_t w = 0;
    const uint8_t* qp = q + r * ldq + c0;
    if (valid >= 4) {
      w = *reinterpret_cast<const uint32_t*>(qp);
    } else {
      for (int i = 0; i < valid; ++i) w |= uint32_t(qp[i]) << (8 * i);
    }
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t c = (w >> (8 * i)) & 0xFFu;
      const float a = ex2_approx(tab[c] * invk) * s;
      x[i] = __uint_as_float(__float_as_uint(a) ^ ((c & 0x80u) << 24));
    }
    if (OT == 0) {
      float* o = static_cast<float*>(out) + r * ldo + c0;
      if (valid >= 4)
        *reinterpret_cast<float4*>(o) = make_float4(x[0], x[1], x[2], x[3]);
      else
        for (int i = 0; i < valid; ++i) o[i] = x[i];
    } else {
      uint16_t* o = static_cast<uint16_t*>(out) + r * ldo + c0;
      if (valid >= 4)
        *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
      else
        for (int i = 0; i < valid; ++i) o[i] = static_cast<uint16_t>(pack_bf16x2(x[i], 0.f));
    }
  }
}

unsigned grid_for(int64_t work_items, int per_block, int dev, int max_blocks_per_sm) {
  int64_t b = (work_items + per_block - 1) / per_block;
  const int64_t cap = int64_t(sm_count(dev)) * max_blocks_per_sm;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return static_cast<unsigned>(b);
}

}  // namespace

cudaError_t launch_fp8_encode(const float* y, int64_t n, int fmt, uint8_t* q, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned g = grid_for(n, 256, dev, 16);
  if (fmt == kE4M3) fp8_encode_kernel<kE4M3><<<g, 256, 0, s>>>(y, n, q);
  else fp8_encode_kernel<kE5M2><<<g, 256, 0, s>>>(y, n, q);
  return cudaGetLastError();
}

cudaError_t launch_fp8_decode(const uint8_t* q, int64_t n, int fmt, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned g = grid_for(n, 256, dev, 16);
  if (fmt == kE4M3) fp8_decode_kernel<kE4M3><<<g, 256, 0, s>>>(q, n, out);
  else fp8_decode_kernel<kE5M2><<<g, 256, 0, s>>>(q, n, out);
  return cudaGetLastError();
}

template <int FMT, int DT>
static void quant_dispatch(const void* x, int64_t rows, int64_t cols, int64_t ldx, int gr,
                           int expand, uint8_t* q, int64_t ldq, float* scale, float* k,
                           int dev, cudaStream_t s) {
  if (gr == 1) {
    const int64_t groups = rows * ((cols + 127) / 128);
    const unsigned g = grid_for((groups + 3) / 4, 8, dev, 8);   // 8 warps per block
    quant_row_kernel<FMT, DT><<<g, 256, 0, s>>>(x, rows, cols, ldx, expand, q, ldq, scale, k);
  } else {
    const int64_t blocks = ((rows + 127) / 128) * ((cols + 127) / 128);
    const unsigned g = grid_for(blocks, 1, dev, 4);
    quant_block_kernel<FMT, DT><<<g, 256, 0, s>>>(x, rows, cols, ldx, expand, q, ldq, scale, k);
  }
}

cudaError_t launch_group_quantize(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                                  int gr, int expand, int fmt, uint8_t* q, int64_t ldq,
                                  float* scale, float* k, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  if (fmt == kE4M3) {
    if (xt == 0) quant_dispatch<kE4M3, 0>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, dev, s);
    else quant_dispatch<kE4M3, 1>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, dev, s);
  } else {
    if (xt == 0) quant_dispatch<kE5M2, 0>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, dev, s);
    else quant_dispatch<kE5M2, 1>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, dev, s);
  }
  return cudaGetLastError();
}

cudaError_t launch_group_dequantize(const uint8_t* q, int64_t ldq, const float* scale,
                                    const float* k, int64_t rows, int64_t cols, int gr, int gc,
                                    int fmt, void* out, int ot, int64_t ldo, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned g = grid_for(rows * ((cols + 3) / 4), 256, dev, 8);
  if (fmt == kE4M3) {
    if (ot == 0) dequant_kernel<kE4M3, 0><<<g, 256, 0, s>>>(q, ldq, scale, k, rows, cols, gr, gc, out, ldo);
    else dequant_kernel<kE4M3, 1><<<g, 256, 0, s>>>(q, ldq, scale, k, rows, cols, gr, gc, out, ldo);
  } else {
    if (ot == 0) dequant_kernel<kE5M2, 0><<<g, 256, 0, s>>>(q, ldq, scale, k, rows, cols, gr, gc, out, ldo);
    else dequant_kernel<kE5M2, 1><<<g, 256, 0, s>>>(q, ldq, scale, k, rows, cols, gr, gc, out, ldo);
  }
  return cudaGetLastError();
}

}  // namespace coat
