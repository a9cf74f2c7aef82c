// codec.cu -- FP8 element codec and the per-group quantiser / dequantiser with
// dynamic range expansion, at the two granularities of the mixed-granularity
// activation path: 1x128 groups along a row (per token) and 128x128 blocks
// (weights).  Sources: [P1] "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍",
// sections "解决方案：动态范围扩展" and "解决方案：混合粒度FP8精度流"; [P4]
// "FP8量化训练实战指南", section "分块级缩放：精度优化的进阶方案" (1x128 tiles for
// activations and gradients, 128x128 blocks for weights, one scale per tile).
//
// All kernels are HBM-bound streaming kernels: 16-byte coalesced loads and
// stores, persistent grids sized to the resident CTAs of every SM, and the
// next work item loaded into registers while the current one is computed; no
// shared-memory staging except the 256-entry log2 decode table.
#include <cstdint>
#include <mutex>
#include <unordered_map>
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
// 16 contiguous elements of a row, as loaded (bf16 pairs or fp32), so that the
// next work item can be fetched into registers while the current one is
// computed.  Row starts are 16-byte aligned (checked by the API), so a chunk
// that starts at a multiple of 16 columns is 16-byte aligned too.
// ---------------------------------------------------------------------------
template <int DT> struct Raw16;
template <> struct Raw16<0> { float4 a, b, c, d; };   // fp32
template <> struct Raw16<1> { uint4 a, b; };          // bf16 pairs

template <int DT>
__device__ __forceinline__ void load16(const void* row, int64_t c, int valid, Raw16<DT>& r) {
  if constexpr (DT == 0) {
    const float* p = static_cast<const float*>(row) + c;
    if (valid >= 16) {
      r.a = __ldg(reinterpret_cast<const float4*>(p));
      r.b = __ldg(reinterpret_cast<const float4*>(p) + 1);
      r.c = __ldg(reinterpret_cast<const float4*>(p) + 2);
      r.d = __ldg(reinterpret_cast<const float4*>(p) + 3);
    } else {
      float t[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) t[i] = i < valid ? p[i] : 0.f;
      r.a = make_float4(t[0], t[1], t[2], t[3]);
      r.b = make_float4(t[4], t[5], t[6], t[7]);
      r.c = make_float4(t[8], t[9], t[10], t[11]);
      r.d = make_float4(t[12], t[13], t[14], t[15]);
    }
  } else {
    const uint16_t* p = static_cast<const uint16_t*>(row) + c;
    if (valid >= 16) {
      r.a = __ldg(reinterpret_cast<const uint4*>(p));
      r.b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    } else {
      uint32_t t[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) t[i] = i < valid ? uint32_t(p[i]) : 0u;
      r.a = make_uint4(t[0] | (t[1] << 16), t[2] | (t[3] << 16), t[4] | (t[5] << 16),
                       t[6] | (t[7] << 16));
      r.b = make_uint4(t[8] | (t[9] << 16), t[10] | (t[11] << 16), t[12] | (t[13] << 16),
                       t[14] | (t[15] << 16));
    }
  }
}

template <int DT>
__device__ __forceinline__ void unpack16(const Raw16<DT>& r, float v[16]) {
  if constexpr (DT == 0) {
    const float4 q[4] = {r.a, r.b, r.c, r.d};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[4 * j] = q[j].x; v[4 * j + 1] = q[j].y; v[4 * j + 2] = q[j].z; v[4 * j + 3] = q[j].w;
    }
  } else {
    const uint32_t w[8] = {r.a.x, r.a.y, r.a.z, r.a.w, r.b.x, r.b.y, r.b.z, r.b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[2 * j] = bf16lo(w[j]);
      v[2 * j + 1] = bf16hi(w[j]);
    }
  }
}


// ---------------------------------------------------------------------------
// 1 x 128 groups: 8 lanes per group, 16 contiguous elements per lane, 4 groups
// (one quad) per warp and work item.  The rows x quads items are taken in
// row-major order, a contiguous range per warp, with the lane's column
// advanced by 512 and a row carry; the next item's elements are loaded before
// the current one is computed.  EXPAND (a template parameter): without
// expansion the group statistics are one NaN-propagating max per element (one
// test then finds NaN and Inf); with it, max and min-nonzero on the bit
// patterns.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

template <int DT>
struct RowItem {
  Raw16<DT> raw;
  int64_t r, c;   // row and the lane's first column
  int valid;      // elements of the lane's 16 that exist
};

// Codes of 8 bf16 values (the words of u) of a group without an Inf or a NaN,
// with k = 1: the same codes as encode_words<FMT, 8, true> with use_div, with
// the arithmetic on element pairs.  The magnitudes are the words with their
// sign bits cleared; the correctly rounded quotients FMT_MAX |x| / M
// (div_exact) and the encoder's fused adds run as packed FP32 pairs, and the
// signs come from the words' top bits.
template <int FMT>
__device__ __forceinline__ void encode8_bf16_div(const uint4& u, const GroupDiv& d,
                                                 uint32_t (&cw)[2]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  const float2 num2 = make_float2(d.num, d.num), y2 = make_float2(d.y, d.y);
  const float2 nb2 = make_float2(-d.b, -d.b);
  uint32_t mag[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t aw = w[j] & 0x7FFF7FFFu;
    const float2 a = mul2(make_float2(__uint_as_float(aw * 65536u), bf16hi(aw)), num2);
    const float2 q0 = mul2(a, y2);
    const float2 y = fma2(fma2(q0, nb2, a), y2, q0);
    const uint2 c = enc_mag_bounded2<FMT, FMT>(y.x, y.y);
    mag[2 * j] = c.x;
    mag[2 * j + 1] = c.y;
  }
  // packing and signs as multiply-adds where the bits do not overlap (the
  // codes are 7 bits; the sign bits land on zero bits), which the FMA pipe
  // executes beside the integer pipe that the encoder keeps busy
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint32_t mags =
        mag[4 * t] + 256u * (mag[4 * t + 1] + 256u * (mag[4 * t + 2] + 256u * mag[4 * t + 3]));
    const uint32_t top = __byte_perm(w[2 * t], w[2 * t + 1], 0x7531u);
    cw[t] = mags + (top & (mags + 0x7F7F7F7Fu) & 0x80808080u);
  }
}

// Codes of 8 bf16 values (the words of u) of an expanded group without an Inf
// or a NaN: the same codes as encode_words<FMT, 8, true> with expansion, with
// y = 2^(k log2(|x| invM) + log2 FMT_MAX) evaluated by the same operations on
// element pairs.
template <int FMT>
__device__ __forceinline__ void encode8_bf16_expand(const uint4& u, float invM, float k,
                                                    uint32_t (&cw)[2]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  const float2 invM2 = make_float2(invM, invM), k2 = make_float2(k, k);
  const float2 L2 = make_float2(F8<FMT>::LOG2MAX_HI, F8<FMT>::LOG2MAX_HI);
  uint32_t mag[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t aw = w[j] & 0x7FFF7FFFu;
    const float2 a = mul2(make_float2(__uint_as_float(aw * 65536u), bf16hi(aw)), invM2);
    const float2 t = fma2(k2, make_float2(lg2_approx(a.x), lg2_approx(a.y)), L2);
    const uint2 c = enc_mag_bounded2<FMT, FMT>(ex2_approx(t.x), ex2_approx(t.y));
    mag[2 * j] = c.x;
    mag[2 * j + 1] = c.y;
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint32_t mags =
        mag[4 * t] + 256u * (mag[4 * t + 1] + 256u * (mag[4 * t + 2] + 256u * mag[4 * t + 3]));
    const uint32_t top = __byte_perm(w[2 * t], w[2 * t + 1], 0x7531u);
    cw[t] = mags + (top & (mags + 0x7F7F7F7Fu) & 0x80808080u);
  }
}

// bf16 input without expansion, when none of the warp's four groups holds an
// Inf, a NaN or a maximum above 2^100 (returns false otherwise, and the caller
// takes the general path): the general path's codes and scales.  The group
// maximum is an unsigned 16-bit max over the words with their sign bits
// cleared, whose halves order like the magnitudes they encode (an Inf or a NaN
// pattern is above every finite one).
template <int FMT>
__device__ __forceinline__ bool quant_bf16_plain(const RowItem<1>& it, int64_t rows, int64_t cols,
                                                 int l, int64_t nbc, uint8_t* __restrict__ q,
                                                 int64_t ldq, float* __restrict__ scale,
                                                 float* __restrict__ kk) {
  const uint4 u[2] = {it.raw.a, it.raw.b};
  uint32_t mx2 = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h)
    mx2 = __vmaxu2(mx2, __vmaxu2(__vmaxu2(u[h].x & 0x7FFF7FFFu, u[h].y & 0x7FFF7FFFu),
                                 __vmaxu2(u[h].z & 0x7FFF7FFFu, u[h].w & 0x7FFF7FFFu)));
  uint32_t mxb = max(mx2 & 0xFFFFu, mx2 >> 16);
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) mxb = max(mxb, __shfl_xor_sync(0xFFFFFFFFu, mxb, off));
  // an Inf, a NaN or a maximum above 2^100 (0x7180): the general path
  if (__any_sync(0xFFFFFFFFu, mxb > 0x7180u)) return false;
  const float M = __uint_as_float(mxb << 16);
  const GroupDiv d = codec_div_short<FMT>(M);
  uint32_t lo[2], hi[2];
  encode8_bf16_div<FMT>(u[0], d, lo);
  encode8_bf16_div<FMT>(u[1], d, hi);
  const uint32_t cw[4] = {lo[0], lo[1], hi[0], hi[1]};
  if (it.valid > 0 && COAT_INDEX_OK(it.r < rows && it.c + it.valid <= cols))
    store16(q + it.r * ldq + it.c, cw, it.valid);
  if (l == 0 && it.valid > 0) {
    const int64_t g = it.r * nbc + (it.c >> 7);
    if (COAT_INDEX_OK(g < rows * nbc)) {
      scale[g] = M > 0.0f ? div_fmax<FMT>(M) : 1.0f;
      kk[g] = 1.0f;
    }
  }
  return true;
}

// One work item of the 16-element layout (4 groups of one row, 8 lanes of 16
// elements each, loaded): group statistics, k and root scale, codes; stores
// the codes and each group's scale and k.  Called by all 32 lanes of a warp.
template <int FMT, int DT, bool EXPAND>
__device__ __forceinline__ void quant_row_item(const RowItem<DT>& cur, int64_t rows, int64_t cols,
                                               int l, int64_t nbc, uint8_t* __restrict__ q,
                                               int64_t ldq, float* __restrict__ scale,
                                               float* __restrict__ kk) {
  if constexpr (DT == 1 && !EXPAND) {
    if (quant_bf16_plain<FMT>(cur, rows, cols, l, nbc, q, ldq, scale, kk)) return;
  }
  float v[16];
  unpack16<DT>(cur.raw, v);
  float M, mu = 0.0f;
  bool special;
  if (EXPAND) {
    uint32_t maxb = 0u, mink = 0xFFFFFFFFu;
    stats_bits(v, maxb, mink);
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      maxb = max(maxb, __shfl_xor_sync(0xFFFFFFFFu, maxb, off));
      mink = min(mink, __shfl_xor_sync(0xFFFFFFFFu, mink, off));
    }
    // an Inf or a NaN in the group, or a finite maximum outside [2^-100, 2^100]
    // (twice the bits)
    special = maxb > 0xE3000000u || (maxb != 0u && maxb < 0x1B000000u);
    M = __uint_as_float(maxb >> 1);
    mu = __uint_as_float((mink + 2u) >> 1);
  } else {
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) mx = fmax_nan(mx, fabsf(v[i]));
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    // NaN, Inf, or a maximum above 2^100 (small maxima need nothing here)
    special = !(mx <= 0x1p100f);
    M = mx;
  }
  float M0 = M, sig = 1.0f;
  if (__any_sync(0xFFFFFFFFu, special)) {
    float Mn = max_abs_nonnan(v);
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) Mn = fmaxf(Mn, __shfl_xor_sync(0xFFFFFFFFu, Mn, off));
    if (special) M = Mn;
    M0 = M;
    // a maximum outside [2^-100, 2^100]: the group's values scaled into range
    sig = range_sigma(M);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] *= sig;
    M *= sig;
    mu *= sig;
  }
  float k, sr, invM = 0.0f;
  if (EXPAND) {
    group_params<FMT>(M, mu, true, k, sr, invM);
    if (sig != 1.0f) sr *= sig < 1.0f ? 0x1p100f : 0x1p-100f;
  } else {
    // k = 1: the root scale is M / FMT_MAX, correctly rounded (1 for an all-zero group)
    k = 1.0f;
    sr = M0 > 0.0f ? div_fmax<FMT>(M0) : 1.0f;
  }
  const bool use_div = !EXPAND || k == 1.0f;
  GroupDiv d{};
  if (use_div) d = codec_div<FMT>(M);
  uint32_t cw[4];
  if (!special)
    encode_words<FMT, 16, true>(v, use_div, d, invM, k, cw);
  else
    encode_words<FMT, 16, false>(v, use_div, d, invM, k, cw);
  if (cur.valid > 0 && COAT_INDEX_OK(cur.r < rows && cur.c + cur.valid <= cols))
    store16(q + cur.r * ldq + cur.c, cw, cur.valid);
  // lane 0 of a group holds its first column, so it exists exactly when the group does
  if (l == 0 && cur.valid > 0) {
    const int64_t g = cur.r * nbc + (cur.c >> 7);
    if (COAT_INDEX_OK(g < rows * nbc)) {
      scale[g] = sr;
      kk[g] = k;
    }
  }
}

template <int FMT, int DT, bool EXPAND>
__global__ void __launch_bounds__(256) quant_row_kernel(const void* __restrict__ x, int64_t rows,
                                                        int64_t cols, int64_t ldx,
                                                        uint8_t* __restrict__ q, int64_t ldq,
                                                        float* __restrict__ scale,
                                                        float* __restrict__ kk) {
  const int lane = threadIdx.x & 31, slot = lane >> 3, l = lane & 7;
  const int64_t nbc = (cols + kGroup - 1) / kGroup;   // groups per row
  const int64_t nq = (nbc + 3) / 4;                    // quads per row
  const int64_t nitems = rows * nq;
  const int64_t wid = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t i0 = wid * nitems / nw, i1 = (wid + 1) * nitems / nw;
  if (i0 >= i1) return;
  const size_t esz = DT == 0 ? 4 : 2;
  const int64_t rowspan = nq * 4 * kGroup;
  int64_t cr = i0 / nq;                                  // the next item to load
  int64_t cc = (i0 - cr * nq) * 4 * kGroup + slot * kGroup + 16 * l;
  auto load = [&](RowItem<DT>& it) {
    it.r = cr;
    it.c = cc;
    it.valid = COAT_INDEX_OK(cr < rows) ? clamp_valid(cols - cc, 16) : 0;
    load16<DT>(static_cast<const char*>(x) + cr * ldx * esz, cc, it.valid, it.raw);
    cc += 4 * kGroup;
    if (cc >= rowspan) { cc -= rowspan; ++cr; }
  };
  RowItem<DT> cur;
  load(cur);
  for (int64_t item = i0; item < i1; ++item) {
    RowItem<DT> nxt;
    if (item + 1 < i1) load(nxt);
    quant_row_item<FMT, DT, EXPAND>(cur, rows, cols, l, nbc, q, ldq, scale, kk);
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// bf16 input, the activation codec's case: 4 lanes per group and 32
// contiguous elements per lane (8 groups, 1024 columns, per warp and work
// item), so that each lane's share of the per-group work (the extremes'
// shuffles, k, the divisor, the root scale) and of the per-item addressing
// covers twice as many elements as in the 16-element layout.  The extremes
// come from the sign-cleared words, two elements per instruction: their 16-bit
// halves order like the magnitudes (an Inf or a NaN pattern is above every
// finite one), and subtracting one from each half first makes zeros the
// largest for the minimum.  A work item whose groups hold an Inf or a NaN, or
// a maximum outside the range range_sigma() describes, is redone by the
// general code (quant_row_item) as the two 512-column items of the 16-element
// layout, read again from global memory.
// ---------------------------------------------------------------------------
struct Row32Item {
  uint4 u[4];     // 32 bf16 values, as loaded
  int64_t r, c;   // row and the lane's first column
  int valid;      // elements of the lane's 32 that exist
};

template <int FMT, bool EXPAND>
__global__ void __launch_bounds__(256) quant_row32_bf16_kernel(const void* __restrict__ x,
                                                               int64_t rows, int64_t cols,
                                                               int64_t ldx,
                                                               uint8_t* __restrict__ q,
                                                               int64_t ldq,
                                                               float* __restrict__ scale,
                                                               float* __restrict__ kk) {
  const int lane = threadIdx.x & 31, sub = lane >> 2, l4 = lane & 3;
  const int64_t nbc = (cols + kGroup - 1) / kGroup;   // groups per row
  const int64_t no = (nbc + 7) / 8;                    // 8-group items per row
  const int64_t nitems = rows * no;
  const int64_t wid = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t i0 = wid * nitems / nw, i1 = (wid + 1) * nitems / nw;
  if (i0 >= i1) return;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const int64_t rowspan = no * 8 * kGroup;
  int64_t cr = i0 / no;                                  // the next item to load
  int64_t cc = (i0 - cr * no) * 8 * kGroup + sub * kGroup + 32 * l4;
  auto load = [&](Row32Item& it) {
    it.r = cr;
    it.c = cc;
    it.valid = COAT_INDEX_OK(cr < rows) ? clamp_valid(cols - cc, 32) : 0;
    const uint16_t* p = xb + cr * ldx + cc;
    if (it.valid >= 32) {
#pragma unroll
      for (int h = 0; h < 4; ++h) it.u[h] = __ldg(reinterpret_cast<const uint4*>(p) + h);
    } else {
      uint32_t t[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) t[i] = i < it.valid ? uint32_t(p[i]) : 0u;
#pragma unroll
      for (int h = 0; h < 4; ++h)
        it.u[h] = make_uint4(t[8 * h] | (t[8 * h + 1] << 16), t[8 * h + 2] | (t[8 * h + 3] << 16),
                             t[8 * h + 4] | (t[8 * h + 5] << 16), t[8 * h + 6] | (t[8 * h + 7] << 16));
    }
    cc += 8 * kGroup;
    if (cc >= rowspan) { cc -= rowspan; ++cr; }
  };
  Row32Item cur;
  load(cur);
  for (int64_t item = i0; item < i1; ++item) {
    Row32Item nxt;
    if (item + 1 < i1) load(nxt);

    // group maximum over the sign-cleared words (16-bit halves order like the
    // magnitudes; an Inf or a NaN pattern is above every finite one)
    uint32_t mx2 = 0u;
#pragma unroll
    for (int h = 0; h < 4; ++h)
      mx2 = __vmaxu2(mx2, __vmaxu2(__vmaxu2(cur.u[h].x & 0x7FFF7FFFu, cur.u[h].y & 0x7FFF7FFFu),
                                   __vmaxu2(cur.u[h].z & 0x7FFF7FFFu, cur.u[h].w & 0x7FFF7FFFu)));
    uint32_t mxb = max(mx2 & 0xFFFFu, mx2 >> 16);
    mxb = max(mxb, __shfl_xor_sync(0xFFFFFFFFu, mxb, 1));
    mxb = max(mxb, __shfl_xor_sync(0xFFFFFFFFu, mxb, 2));
    uint32_t mnb = 0xFFFFu;   // (min nonzero magnitude bits) - 1; 0xFFFF: all zero
    if (EXPAND) {
      uint32_t mn2 = 0xFFFFFFFFu;
#pragma unroll
      for (int h = 0; h < 4; ++h)
        mn2 = __vminu2(mn2, __vminu2(__vminu2(__vsub2(cur.u[h].x & 0x7FFF7FFFu, 0x00010001u),
                                              __vsub2(cur.u[h].y & 0x7FFF7FFFu, 0x00010001u)),
                                     __vminu2(__vsub2(cur.u[h].z & 0x7FFF7FFFu, 0x00010001u),
                                              __vsub2(cur.u[h].w & 0x7FFF7FFFu, 0x00010001u))));
      mnb = min(mn2 & 0xFFFFu, mn2 >> 16);
      mnb = min(mnb, __shfl_xor_sync(0xFFFFFFFFu, mnb, 1));
      mnb = min(mnb, __shfl_xor_sync(0xFFFFFFFFu, mnb, 2));
    }
    // an Inf, a NaN, a maximum above 2^100 (bits 0x7180) or a nonzero one
    // below 2^-100 (0x0D80): the general path (so that below, the root scale
    // M / FMT_MAX takes div_fmax's correction step without its range test)
    const bool slow = mxb > 0x7180u || (mxb != 0u && mxb < 0x0D80u);
    if (!__any_sync(0xFFFFFFFFu, slow)) {
      const float M = __uint_as_float(mxb << 16);
      float k = 1.0f, sr, invM = 0.0f;
      if (EXPAND) {
        group_params<FMT>(M, __uint_as_float(((mnb + 1u) & 0xFFFFu) << 16), true, k, sr, invM);
      } else {
        const float q0 = M * F8<FMT>::RCPMAX;
        sr = M > 0.0f ? __fmaf_rn(__fmaf_rn(-q0, F8<FMT>::MAXV, M), F8<FMT>::RCPMAX, q0) : 1.0f;
      }
      uint32_t cw[8];
      if (!EXPAND || k == 1.0f) {
        const GroupDiv d = codec_div_short<FMT>(M);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t two[2];
          encode8_bf16_div<FMT>(cur.u[h], d, two);
          cw[2 * h] = two[0];
          cw[2 * h + 1] = two[1];
        }
      } else {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t two[2];
          encode8_bf16_expand<FMT>(cur.u[h], invM, k, two);
          cw[2 * h] = two[0];
          cw[2 * h + 1] = two[1];
        }
      }
      if (cur.valid > 0 && COAT_INDEX_OK(cur.r < rows && cur.c + cur.valid <= cols)) {
        uint8_t* qp = q + cur.r * ldq + cur.c;
        if (cur.valid >= 32) {
          reinterpret_cast<uint4*>(qp)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          reinterpret_cast<uint4*>(qp)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < cur.valid) qp[i] = static_cast<uint8_t>(cw[i >> 2] >> (8 * (i & 3)));
        }
      }
      // lane 0 of a group holds its first column, so it exists exactly when the group does
      if (l4 == 0 && cur.valid > 0) {
        const int64_t g = cur.r * nbc + (cur.c >> 7);
        if (COAT_INDEX_OK(g < rows * nbc)) {
          scale[g] = sr;
          kk[g] = k;
        }
      }
    } else {
      // the two 512-column halves of the item in the 16-element layout
      const int slot = lane >> 3, l = lane & 7;
      const int64_t c0 = cur.c - sub * kGroup - 32 * l4;   // the item's first column
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        RowItem<1> it;
        it.r = cur.r;
        it.c = c0 + h * 4 * kGroup + slot * kGroup + 16 * l;
        it.valid = COAT_INDEX_OK(cur.r < rows) ? clamp_valid(cols - it.c, 16) : 0;
        load16<1>(xb + cur.r * ldx, it.c, it.valid, it.raw);
        quant_row_item<FMT, 1, EXPAND>(it, rows, cols, l, nbc, q, ldq, scale, kk);
      }
    }
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// 128 x 128 blocks: one 256-thread CTA per block at a time; warp w takes rows
// 16w..16w+15, each load instruction covers two rows (half-warp per row, 8
// contiguous columns per lane); max / min by shuffles, then across the 8
// warps through shared memory.  bf16 input: the next block is loaded into a
// second register buffer before the current one is computed.
// ---------------------------------------------------------------------------
template <int DT> struct Block8;   // the 64 elements a thread holds, as loaded
template <> struct Block8<0> { float4 a[8], b[8]; };
template <> struct Block8<1> { uint4 a[8]; };

template <int DT>
__device__ __forceinline__ void load_block(const void* x, int64_t rows, int64_t cols, int64_t ldx,
                                           int64_t br, int64_t bc, int warp, int lane,
                                           Block8<DT>& B) {
  const int64_t c = bc * 128 + 8 * (lane & 15);
  const int cv = clamp_valid(cols - c, 8);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = br * 128 + warp * 16 + 2 * i + (lane >> 4);
    const int valid = r < rows ? cv : 0;
    if constexpr (DT == 0) {
      const float* p = static_cast<const float*>(x) + r * ldx + c;
      float4 u = make_float4(0.f, 0.f, 0.f, 0.f), w = u;
      if (valid >= 8) {
        u = __ldg(reinterpret_cast<const float4*>(p));
        w = __ldg(reinterpret_cast<const float4*>(p) + 1);
      } else if (valid > 0) {
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = e < valid ? p[e] : 0.f;
        u = make_float4(t[0], t[1], t[2], t[3]);
        w = make_float4(t[4], t[5], t[6], t[7]);
      }
      B.a[i] = u;
      B.b[i] = w;
    } else {
      const uint16_t* p = static_cast<const uint16_t*>(x) + r * ldx + c;
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (valid >= 8) {
        u = __ldg(reinterpret_cast<const uint4*>(p));
      } else if (valid > 0) {
        uint32_t t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = e < valid ? uint32_t(p[e]) : 0u;
        u = make_uint4(t[0] | (t[1] << 16), t[2] | (t[3] << 16), t[4] | (t[5] << 16),
                       t[6] | (t[7] << 16));
      }
      B.a[i] = u;
    }
  }
}

template <int DT>
__device__ __forceinline__ void block_row(const Block8<DT>& B, int i, float v[8]) {
  if constexpr (DT == 0) {
    v[0] = B.a[i].x; v[1] = B.a[i].y; v[2] = B.a[i].z; v[3] = B.a[i].w;
    v[4] = B.b[i].x; v[5] = B.b[i].y; v[6] = B.b[i].z; v[7] = B.b[i].w;
  } else {
    const uint4 u = B.a[i];
    v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
    v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
  }
}

template <int FMT, int DT, bool EXPAND>
__global__ void __launch_bounds__(256) quant_block_kernel(const void* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ldx,
                                                          uint8_t* __restrict__ q, int64_t ldq,
                                                          float* __restrict__ scale,
                                                          float* __restrict__ kk) {
  __shared__ uint32_t sM[2][8];
  __shared__ uint32_t sK[2][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nbc = (cols + 127) / 128, nbr = (rows + 127) / 128;
  const int64_t nb = nbr * nbc;
  int64_t b = blockIdx.x;
  if (b >= nb) return;
  const int64_t dbr = gridDim.x / nbc, dbc = gridDim.x % nbc;
  int64_t br = b / nbc, bc = b % nbc;
  Block8<DT> cur;
  load_block<DT>(x, rows, cols, ldx, br, bc, warp, lane, cur);
  int par = 0;
  while (b < nb) {
    const int64_t bn = b + gridDim.x;
    int64_t brn = br + dbr, bcn = bc + dbc;
    if (bcn >= nbc) { bcn -= nbc; ++brn; }
    Block8<DT> nxt;
    if (DT == 1 && bn < nb) load_block<DT>(x, rows, cols, ldx, brn, bcn, warp, lane, nxt);

    // with expansion: max and min-nonzero on twice the bit patterns; without:
    // the bit pattern of a NaN-propagating max |x| (non-negative floats and
    // the NaN it returns order like their bit patterns)
    uint32_t maxb = 0u, mink = 0xFFFFFFFFu;
    if constexpr (EXPAND) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float v[8];
        block_row<DT>(cur, i, v);
        stats_bits(v, maxb, mink);
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        maxb = max(maxb, __shfl_xor_sync(0xFFFFFFFFu, maxb, off));
        mink = min(mink, __shfl_xor_sync(0xFFFFFFFFu, mink, off));
      }
    } else if constexpr (DT == 1) {
      // bf16: |x| bit patterns compared two at a time (16-bit lanes); NaN
      // patterns are above Inf's, so the test below still finds both
      uint32_t m2 = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 u = cur.a[i];
        m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu),
                                   __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu)));
      }
      uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      maxb = m >= 0x7F80u ? 0x7FFFFFFFu : (m << 16);
    } else {
      float mx = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float v[8];
        block_row<DT>(cur, i, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx = fmax_nan(mx, fabsf(v[e]));
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      maxb = __float_as_uint(mx);
    }
    // double-buffered partials: one barrier per block
    if (lane == 0) {
      sM[par][warp] = maxb;
      sK[par][warp] = mink;
    }
    __syncthreads();
    maxb = sM[par][0];
    mink = sK[par][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      maxb = max(maxb, sM[par][w]);
      mink = min(mink, sK[par][w]);
    }
    // special (CTA-uniform): an Inf or a NaN in the block, or a finite maximum
    // outside [2^-100, 2^100] (bits 0x71800000 and 0x0D800000, doubled with
    // expansion; without expansion small maxima need nothing), whose values
    // are scaled into range (range_sigma)
    const bool special = EXPAND ? maxb > 0xE3000000u || (maxb != 0u && maxb < 0x1B000000u)
                                : maxb > 0x71800000u;
    float M = __uint_as_float(EXPAND ? maxb >> 1 : maxb);
    float mu = EXPAND ? __uint_as_float((mink + 2u) >> 1) : 0.0f;
    float M0 = M, sig = 1.0f;
    if (special) {
      // max |x| ignoring NaN, through the other half of the partials buffer
      float Mn = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float v[8];
        block_row<DT>(cur, i, v);
        Mn = fmaxf(Mn, max_abs_nonnan(v));
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) Mn = fmaxf(Mn, __shfl_xor_sync(0xFFFFFFFFu, Mn, off));
      if (lane == 0) sM[par ^ 1][warp] = __float_as_uint(Mn);
      __syncthreads();
      M = __uint_as_float(sM[par ^ 1][0]);
#pragma unroll
      for (int w = 1; w < 8; ++w) M = fmaxf(M, __uint_as_float(sM[par ^ 1][w]));
      __syncthreads();   // the partials buffer is free again before the next block writes it
      M0 = M;
      sig = range_sigma(M);
      M *= sig;
      mu *= sig;
    }
    par ^= 1;
    float k, sr, invM = 0.0f;
    if (EXPAND) {
      group_params<FMT>(M, mu, true, k, sr, invM);
      if (special && sig != 1.0f) sr *= sig < 1.0f ? 0x1p100f : 0x1p-100f;
    } else {
      // k = 1: the root scale is M / FMT_MAX, correctly rounded (1 for an all-zero block)
      k = 1.0f;
      sr = M0 > 0.0f ? div_fmax<FMT>(M0) : 1.0f;
    }
    const bool use_div = !EXPAND || k == 1.0f;
    GroupDiv d{};
    if (use_div) d = DT == 1 && !special ? codec_div_short<FMT>(M) : codec_div<FMT>(M);
    const int64_t c = bc * 128 + 8 * (lane & 15);
    const int cv = clamp_valid(cols - c, 8);
    // the 8 codes of this lane's row i of the block
    auto put = [&](int i, const uint32_t (&cw)[2]) {
      const int64_t r = br * 128 + warp * 16 + 2 * i + (lane >> 4);
      const int valid = r < rows && COAT_INDEX_OK(cv == 0 || c + cv <= cols) ? cv : 0;
      uint8_t* qp = q + r * ldq + c;
      if (valid >= 8) {
        *reinterpret_cast<uint2*>(qp) = make_uint2(cw[0], cw[1]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (e < valid) qp[e] = static_cast<uint8_t>(cw[e >> 2] >> (8 * (e & 3)));
      }
    };
    if constexpr (DT == 1) {
      // bf16: one unrolled loop per fast path (the CTA-uniform branch is taken
      // once per block), so that the loop's code stays small
      if (!special && use_div) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t cw[2];
          encode8_bf16_div<FMT>(cur.a[i], d, cw);
          put(i, cw);
        }
      } else if (!special) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t cw[2];
          encode8_bf16_expand<FMT>(cur.a[i], invM, k, cw);
          put(i, cw);
        }
      } else {
        // a block with special values or an out-of-range maximum: the general
        // encoder, one row at a time, each row read again from global memory
        // (a rolled loop cannot index the registers that hold the block)
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {
          const int64_t r = br * 128 + warp * 16 + 2 * i + (lane >> 4);
          const int valid = r < rows ? cv : 0;
          const uint16_t* xp = static_cast<const uint16_t*>(x) + r * ldx + c;
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = e < valid ? bf16lo(uint32_t(xp[e])) * sig : 0.0f;
          uint32_t cw[2];
          encode_words<FMT, 8, false>(v, use_div, d, invM, k, cw);
          put(i, cw);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float v[8];
        block_row<DT>(cur, i, v);
        uint32_t cw[2];
        if (special) {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] *= sig;
          encode_words<FMT, 8, false>(v, use_div, d, invM, k, cw);
        } else {
          encode_words<FMT, 8, true>(v, use_div, d, invM, k, cw);
        }
        put(i, cw);
      }
    }
    if (threadIdx.x == 0 && COAT_INDEX_OK(b < nb)) {
      scale[b] = sr;
      kk[b] = k;
    }
    b = bn;
    br = brn;
    bc = bcn;
    if (DT == 1) {
      cur = nxt;
    } else if (b < nb) {
      load_block<DT>(x, rows, cols, ldx, br, bc, warp, lane, cur);
    }
  }
}

// ---------------------------------------------------------------------------
// dequantise: one thread per 16 contiguous codes of a row (all in one group,
// since groups are 128 columns wide and start at multiples of 128); chunks
// are walked row-major with a fixed stride per thread, and the next chunk's
// codes and group metadata are loaded before the current chunk is computed.
// GR: rows per group (1 or 128).
// ---------------------------------------------------------------------------
// 16 values of one group from their codes: x = sign(q) s 2^(log2|q| / k), with
// tabl = this lane's copy of the log2 table (entry c at tabl[32 c]).
__device__ __forceinline__ void dequant16(const uint4& w, const float* tabl, float invk, float s,
                                          float (&xv)[16]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t wd = ws[i >> 2];
    const uint32_t c = __byte_perm(wd, 0u, 0x4440u + (i & 3));
    const float a = ex2_approx(tabl[c << 5] * invk) * s;
    xv[i] = __uint_as_float(__float_as_uint(a) ^ ((wd << (24 - 8 * (i & 3))) & 0x80000000u));
  }
}

template <int OT>
__device__ __forceinline__ void store_out16(void* o, const float (&xv)[16]) {
  if (OT == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      reinterpret_cast<float4*>(o)[j] = make_float4(xv[4 * j], xv[4 * j + 1], xv[4 * j + 2], xv[4 * j + 3]);
  } else {
    uint32_t p[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(xv[2 * j], xv[2 * j + 1]);
    reinterpret_cast<uint4*>(o)[0] = make_uint4(p[0], p[1], p[2], p[3]);
    reinterpret_cast<uint4*>(o)[1] = make_uint4(p[4], p[5], p[6], p[7]);
  }
}

// log2 table replicated once per lane (entry c of lane j at 32 c + j), so that
// the per-element lookups of a warp never share a bank; called by the whole CTA.
template <int FMT>
__device__ __forceinline__ const float* lane_log2_table(float* tab1, float* tab) {
  fill_log2_table<FMT>(tab1);
  __syncthreads();
  for (int e = threadIdx.x; e < 256 * 32; e += blockDim.x) tab[e] = tab1[e >> 5];
  __syncthreads();
  return tab + (threadIdx.x & 31);
}

// 16 values of one group with k = 1: the codes converted exactly (FP8 -> f16 ->
// f32 in hardware) times the scale, one rounding.
template <int FMT>
__device__ __forceinline__ void dequant16_k1(const uint4& w, float s, float (&xv)[16]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 a = f16x2_to_float2(fp8x2_to_f16x2<FMT>(ws[j]));
    const float2 b = f16x2_to_float2(fp8x2_to_f16x2<FMT>(ws[j] >> 16));
    xv[4 * j] = a.x * s;
    xv[4 * j + 1] = a.y * s;
    xv[4 * j + 2] = b.x * s;
    xv[4 * j + 3] = b.y * s;
  }
}

// Rows whose width is a multiple of 16: every chunk is whole, and the code,
// output and metadata positions advance with the stride by pointer increments.
// A thread loads kBatch chunks (its next kBatch positions of the stride walk)
// before it computes any of them, so that each thread keeps kBatch 16-byte
// loads in flight.
constexpr int kBatch = 4;

template <int FMT, int OT, int GR>
__global__ void __launch_bounds__(256) dequant_full_kernel(const uint8_t* __restrict__ q,
                                                           int64_t ldq,
                                                           const float* __restrict__ scale,
                                                           const float* __restrict__ kk,
                                                           int64_t rows, int64_t cols,
                                                           void* __restrict__ out, int64_t ldo) {
  __shared__ float tab1[256];
  __shared__ float tab[256 * 32];
  const float* tabl = lane_log2_table<FMT>(tab1, tab);
  constexpr int64_t kOsz = OT == 0 ? 4 : 2;
  const int64_t cpr = cols / 16;  // chunks per row
  const int64_t nbc = (cols + 127) / 128;
  const int64_t t0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const int64_t nt = int64_t(gridDim.x) * blockDim.x;
  const int64_t dr = nt / cpr, dc = nt % cpr;
  int64_t r = t0 / cpr, cc = t0 % cpr;
  // byte steps of the code and output pointers: without / with a row carry
  const int64_t qs = dr * ldq + 16 * dc, qsc = qs + ldq - 16 * cpr;
  const int64_t os = (dr * ldo + 16 * dc) * kOsz, osc = os + (ldo - 16 * cpr) * kOsz;
  const uint8_t* qp = q + r * ldq + 16 * cc;
  char* op = static_cast<char*>(out) + (r * ldo + 16 * cc) * kOsz;
  while (r < rows) {
    uint4 w[kBatch];
    float s[kBatch], kv[kBatch];
    char* o[kBatch];
    bool ok[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      ok[j] = r < rows && COAT_INDEX_OK(16 * cc + 16 <= cols);
      if (ok[j]) {
        w[j] = __ldg(reinterpret_cast<const uint4*>(qp));
        const int64_t g = (GR == 1 ? r : r / GR) * nbc + (cc >> 3);
        s[j] = __ldg(scale + g);
        kv[j] = __ldg(kk + g);
        o[j] = op;
        int64_t cn = cc + dc;
        const bool carry = cn >= cpr;
        if (carry) cn -= cpr;
        r += dr + (carry ? 1 : 0);
        cc = cn;
        qp += carry ? qsc : qs;
        op += carry ? osc : os;
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (!ok[j]) break;
      float xv[16];
      if (kv[j] == 1.0f)
        dequant16_k1<FMT>(w[j], s[j], xv);
      else
        dequant16(w[j], tabl, rcp_approx(kv[j]), s[j], xv);
      store_out16<OT>(o[j], xv);
    }
  }
}

template <int FMT, int OT, int GR>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* __restrict__ q, int64_t ldq,
                                                      const float* __restrict__ scale,
                                                      const float* __restrict__ kk, int64_t rows,
                                                      int64_t cols, void* __restrict__ out,
                                                      int64_t ldo) {
  __shared__ float tab1[256];
  __shared__ float tab[256 * 32];
  const float* tabl = lane_log2_table<FMT>(tab1, tab);
  const int64_t cpr = (cols + 15) / 16;  // chunks per row
  const int64_t nbc = (cols + 127) / 128;
  const int64_t t0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const int64_t nt = int64_t(gridDim.x) * blockDim.x;
  const int64_t dr = nt / cpr, dc = nt % cpr;
  int64_t r = t0 / cpr, cc = t0 % cpr;
  auto fetch = [&](int64_t rr, int64_t ch, uint4& w, float& s, float& kv, int& valid) {
    const int64_t c0 = ch * 16;
    valid = COAT_INDEX_OK(rr < rows && c0 < cols) ? clamp_valid(cols - c0, 16) : 0;
    const uint8_t* qp = q + rr * ldq + c0;
    if (valid >= 16) {
      w = __ldg(reinterpret_cast<const uint4*>(qp));
    } else {
      uint32_t t[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < valid) t[i >> 2] |= uint32_t(qp[i]) << (8 * (i & 3));
      w = make_uint4(t[0], t[1], t[2], t[3]);
    }
    const int64_t g = (GR == 1 ? rr : rr / GR) * nbc + (ch >> 3);
    s = valid > 0 ? __ldg(scale + g) : 0.f;
    kv = valid > 0 ? __ldg(kk + g) : 1.f;
  };
  uint4 w;
  float s, kv;
  int valid;
  if (r < rows) fetch(r, cc, w, s, kv, valid);
  while (r < rows) {
    int64_t rn = r + dr, cn = cc + dc;
    if (cn >= cpr) { cn -= cpr; ++rn; }
    uint4 wn;
    float sn, kn;
    int validn;
    if (rn < rows) fetch(rn, cn, wn, sn, kn, validn);

    float xv[16];
    if (kv == 1.0f)
      dequant16_k1<FMT>(w, s, xv);
    else
      dequant16(w, tabl, rcp_approx(kv), s, xv);
    const int64_t c0 = cc * 16;
    if (OT == 0) {
      float* o = static_cast<float*>(out) + r * ldo + c0;
      if (valid >= 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          reinterpret_cast<float4*>(o)[j] = make_float4(xv[4 * j], xv[4 * j + 1], xv[4 * j + 2], xv[4 * j + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < valid) o[i] = xv[i];
      }
    } else {
      uint16_t* o = static_cast<uint16_t*>(out) + r * ldo + c0;
      if (valid >= 16) {
        uint32_t p[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(xv[2 * j], xv[2 * j + 1]);
        reinterpret_cast<uint4*>(o)[0] = make_uint4(p[0], p[1], p[2], p[3]);
        reinterpret_cast<uint4*>(o)[1] = make_uint4(p[4], p[5], p[6], p[7]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < valid) o[i] = static_cast<uint16_t>(pack_bf16x2(xv[i], 0.f));
      }
    }
    r = rn;
    cc = cn;
    w = wn;
    s = sn;
    kv = kn;
    valid = validn;
  }
}

}  // namespace

COAT_INDEX_FAULT_READER(index_faults_codec)

unsigned grid_for(int64_t work_items, int per_block, int dev, int max_blocks_per_sm) {
  int64_t b = (work_items + per_block - 1) / per_block;
  const int64_t cap = int64_t(sm_count(dev)) * max_blocks_per_sm;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return static_cast<unsigned>(b);
}

// CTAs of `kernel` (256 threads, plus dyn_smem bytes of dynamic shared memory) resident per SM,
// from the occupancy calculator, cached per kernel (all B200s give the same).
namespace {
std::mutex g_occ_mu;
std::unordered_map<const void*, int> g_occ;
}  // namespace

int resident_ctas(const void* kernel, size_t dyn_smem, int threads) {
  std::lock_guard<std::mutex> lk(g_occ_mu);
  auto it = g_occ.find(kernel);
  if (it != g_occ.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, dyn_smem) != cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    n = 1;
  }
  g_occ.emplace(kernel, n);
  return n;
}


cudaError_t launch_fp8_encode(const float* y, int64_t n, int fmt, uint8_t* q, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned g = grid_for(n, 256, dev, 16);
  if (fmt == kE4M3) fp8_encode_kernel<kE4M3><<<g, 256, 0, s>>>(y, n, q);
  else fp8_encode_kernel<kE5M2><<<g, 256, 0, s>>>(y, n, q);   // E5M2 and E5M2 full span
  return cudaGetLastError();
}

cudaError_t launch_fp8_decode(const uint8_t* q, int64_t n, int fmt, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned g = grid_for(n, 256, dev, 16);
  if (fmt == kE4M3) fp8_decode_kernel<kE4M3><<<g, 256, 0, s>>>(q, n, out);
  else fp8_decode_kernel<kE5M2><<<g, 256, 0, s>>>(q, n, out);   // E5M2 and E5M2 full span
  return cudaGetLastError();
}

template <int FMT, int DT>
static cudaError_t quant_dispatch(const void* x, int64_t rows, int64_t cols, int64_t ldx, int gr,
                                  int expand, uint8_t* q, int64_t ldq, float* scale, float* k,
                                  unsigned* err, int dev, cudaStream_t s) {
  if (gr == 1) {
    // bf16: 32 elements per lane; FP32: 16 (the general layout)
    if constexpr (DT == 1) {
      const int64_t octs = rows * (((cols + 127) / 128 + 7) / 8);
      auto kern = expand ? quant_row32_bf16_kernel<FMT, true> : quant_row32_bf16_kernel<FMT, false>;
      const unsigned g = grid_for(octs, 8, dev, resident_ctas(reinterpret_cast<const void*>(kern)));
      kern<<<g, 256, 0, s>>>(x, rows, cols, ldx, q, ldq, scale, k);
    } else {
      const int64_t quads = rows * (((cols + 127) / 128 + 3) / 4);
      auto kern = expand ? quant_row_kernel<FMT, DT, true> : quant_row_kernel<FMT, DT, false>;
      const unsigned g =
          grid_for(quads, 8, dev, resident_ctas(reinterpret_cast<const void*>(kern)));
      kern<<<g, 256, 0, s>>>(x, rows, cols, ldx, q, ldq, scale, k);
    }
  } else {
    const int64_t blocks = ((rows + 127) / 128) * ((cols + 127) / 128);
    auto kern = expand ? quant_block_kernel<FMT, DT, true> : quant_block_kernel<FMT, DT, false>;
    const unsigned g = grid_for(blocks, 1, dev, resident_ctas(reinterpret_cast<const void*>(kern)));
    kern<<<g, 256, 0, s>>>(x, rows, cols, ldx, q, ldq, scale, k);
  }
  return cudaSuccess;
}

cudaError_t launch_group_quantize(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                                  int gr, int expand, int fmt, uint8_t* q, int64_t ldq,
                                  float* scale, float* k, unsigned* err, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t e;
  if (fmt == kE4M3) {
    e = xt == 0 ? quant_dispatch<kE4M3, 0>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, err, dev, s)
                : quant_dispatch<kE4M3, 1>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, err, dev, s);
  } else if (fmt == kE5M2) {
    e = xt == 0 ? quant_dispatch<kE5M2, 0>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, err, dev, s)
                : quant_dispatch<kE5M2, 1>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, err, dev, s);
  } else {
    e = xt == 0
            ? quant_dispatch<kE5M2Full, 0>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, err, dev, s)
            : quant_dispatch<kE5M2Full, 1>(x, rows, cols, ldx, gr, expand, q, ldq, scale, k, err, dev, s);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT, int OT>
static void dequant_dispatch(const uint8_t* q, int64_t ldq, const float* scale, const float* k,
                             int64_t rows, int64_t cols, int gr, void* out, int64_t ldo, int dev,
                             cudaStream_t s) {
  auto kern = cols % 16 == 0
                  ? (gr == 1 ? dequant_full_kernel<FMT, OT, 1> : dequant_full_kernel<FMT, OT, 128>)
                  : (gr == 1 ? dequant_kernel<FMT, OT, 1> : dequant_kernel<FMT, OT, 128>);
  const unsigned g = grid_for(rows * ((cols + 15) / 16), 256, dev,
                              resident_ctas(reinterpret_cast<const void*>(kern)));
  kern<<<g, 256, 0, s>>>(q, ldq, scale, k, rows, cols, out, ldo);
}

cudaError_t launch_group_dequantize(const uint8_t* q, int64_t ldq, const float* scale,
                                    const float* k, int64_t rows, int64_t cols, int gr, int gc,
                                    int fmt, void* out, int ot, int64_t ldo, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  if (gc != 128 || (gr != 1 && gr != 128)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  if (fmt == kE4M3) {
    if (ot == 0) dequant_dispatch<kE4M3, 0>(q, ldq, scale, k, rows, cols, gr, out, ldo, dev, s);
    else dequant_dispatch<kE4M3, 1>(q, ldq, scale, k, rows, cols, gr, out, ldo, dev, s);
  } else {   // E5M2 and E5M2 full span: the same codes
    if (ot == 0) dequant_dispatch<kE5M2, 0>(q, ldq, scale, k, rows, cols, gr, out, ldo, dev, s);
    else dequant_dispatch<kE5M2, 1>(q, ldq, scale, k, rows, cols, gr, out, ldo, dev, s);
  }
  return cudaGetLastError();
}

}  // namespace coat
