// fp8_flow.cu -- the FP8 precision flow through a non-linear layer on sm_100a.
//
// What it computes ([P1] "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍",
// sections "FP8激活" and "解决方案：混合粒度FP8精度流"): a non-linear layer whose
// input and output are FP8 tensors, so that the FP8 input itself is what the
// backward pass keeps.  The layer is Llama's gated activation
// h = silu(gate) * up, silu(g) = g / (1 + e^-g), on FP8 gate / up tensors in
// 1x128 per-token groups (the codec's layout: codes, a root scale and k per
// group); the output is quantised per 1x128 group like the codec's quantiser
// (expansion on or off).  The backward pass reads the same FP8 gate / up and
// a bf16 output gradient dh and writes bf16 input gradients:
//   dup = dh silu(g),  dgate = dh u sigmoid(g) (1 + g (1 - sigmoid(g))).
//
// Both kernels stream HBM (no tensor cores: nothing here is a contraction):
//  * forward (3.19 algorithmic bytes per element: two codes in, one code out,
//    24 B of group metadata per 128 elements): 8 lanes per 128-column group,
//    16 contiguous columns per lane, 4 groups per warp and work item, the
//    next item's codes and metadata loaded before the current one is
//    computed; group statistics by 3 xor-shuffles; the quantiser arithmetic
//    is the codec's (the expansion, the software RNE encoder, the NaN/Inf
//    slow path), with k = 1 groups scaled by one multiply;
//  * backward (8.13 B per element: dh in, two codes in, two bf16 out, group
//    metadata): one thread per 16 contiguous columns, no cross-lane work.
// Dequantisation of a k = 1 group (no expansion, the usual activation case)
// converts code pairs exactly to f16 with the hardware FP8 conversion (and
// the forward folds both scales into one product per group); other groups
// use a 256-entry log2 table and ex2.
// The sigmoid is 1 / (1 + 2^(-g log2 e)) with the approximate ex2 and
// reciprocal (relative error a few 2^-23); results below FP32's normal range
// flush to 0.
#include <cstdint>
#include <cuda_runtime.h>

#include "coat_device.cuh"
#include "coat_internal.h"

namespace coat {
namespace {

// The 16 values x = sign(q) s |q|^(1/k) of one lane's codes (all in one group).
template <int FMT>
__device__ __forceinline__ void decode16(const uint4& w, float s, float k, const float* tab,
                                         float (&x)[16]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  if (k == 1.0f) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 a = f16x2_to_float2(fp8x2_to_f16x2<FMT>(ws[j]));
      const float2 b = f16x2_to_float2(fp8x2_to_f16x2<FMT>(ws[j] >> 16));
      x[4 * j] = a.x * s;
      x[4 * j + 1] = a.y * s;
      x[4 * j + 2] = b.x * s;
      x[4 * j + 3] = b.y * s;
    }
  } else {
    const float invk = rcp_approx(k);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t wd = ws[i >> 2];
      const uint32_t c = __byte_perm(wd, 0u, 0x4440u + (i & 3));
      const float a = ex2_approx(tab[c] * invk) * s;
      x[i] = __uint_as_float(__float_as_uint(a) ^ ((wd << (24 - 8 * (i & 3))) & 0x80000000u));
    }
  }
}

// max(a, b) that returns NaN when either is NaN.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// sigmoid(g) = 1 / (1 + e^-g); 0 once the result is below 2^-126 (the
// reciprocal flushes), 1 for large g.
__device__ __forceinline__ float sigmoid(float g) {
  return rcp_approx(1.0f + ex2_approx(g * -1.4426950408889634f));
}

// |q|^(1/k) with the code's sign for the 16 codes of one lane (the group's
// scale is applied by the caller).  plain: every group of the warp has k = 1,
// so the values are the FP8 values themselves, converted exactly.
template <int FMT>
__device__ __forceinline__ void decode16_raw(const uint4& w, float k, bool plain,
                                             const float* tab, float (&f)[16]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  if (plain) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 a = f16x2_to_float2(fp8x2_to_f16x2<FMT>(ws[j]));
      const float2 b = f16x2_to_float2(fp8x2_to_f16x2<FMT>(ws[j] >> 16));
      f[4 * j] = a.x;
      f[4 * j + 1] = a.y;
      f[4 * j + 2] = b.x;
      f[4 * j + 3] = b.y;
    }
  } else if (k == 1.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      f[i] = dec_value<FMT>(__byte_perm(ws[i >> 2], 0u, 0x4440u + (i & 3)));
  } else {
    const float invk = rcp_approx(k);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t wd = ws[i >> 2];
      const uint32_t c = __byte_perm(wd, 0u, 0x4440u + (i & 3));
      const float a = ex2_approx(tab[c] * invk);
      f[i] = __uint_as_float(__float_as_uint(a) ^ ((wd << (24 - 8 * (i & 3))) & 0x80000000u));
    }
  }
}

// One lane's forward work item: 16 gate and 16 up codes, their groups'
// metadata, and the item's row and the lane's first column.
struct FwdItem {
  uint4 gw, uw;
  float gs, gk, us, uk;
  int64_t r;
  int32_t c;
  bool valid;   // the lane's 16 columns exist
};

// h = silu(g) u with g = f_g s_g, u = f_u s_u, as ((f_g f_u) sigmoid(g)) (s_g s_u):
// f_g f_u is exact for k = 1 inputs (two FP8 significands), so h takes two
// roundings besides the sigmoid's.  The output codes: k = 1 groups encode
// FMT_MAX |h| / M as |h| (FMT_MAX / M) (a few ulps from the correctly rounded
// quotient, which only decides codes at exact ties of the real-number result;
// at most FMT_MAX (1 + 2^-21), inside the bounded encoder's range) with root
// scale M / FMT_MAX; expanded groups use the codec's expansion.  EXPAND:
// output expansion on.
// Work: the rows x ceil(groups/4) items (4 groups of a row, 8 lanes each) in
// row-major order, a contiguous range per warp (columns advanced by 512 with
// a row carry); the next item is loaded before the current one is computed.
template <int FMT, bool EXPAND>
__global__ void __launch_bounds__(256) swiglu_fwd_kernel(const ActArgs gate, const ActArgs up,
                                                         int64_t rows, int64_t cols,
                                                         const ActArgs out) {
  __shared__ float tab[256];
  fill_log2_table<FMT>(tab);
  __syncthreads();
  const int lane = threadIdx.x & 31, slot = lane >> 3, l = lane & 7;
  const int64_t nbc = (cols + kGroup - 1) / kGroup;   // groups per row
  const int64_t nq = (nbc + 3) / 4;                    // quads per row
  const int64_t nitems = rows * nq;
  const int64_t wid = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nw = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t i0 = wid * nitems / nw, i1 = (wid + 1) * nitems / nw;
  if (i0 >= i1) return;
  const int lc = slot * kGroup + 16 * l;   // the lane's column within an item
  int64_t cr = i0 / nq;                     // row and lane column of the next item to load
  int32_t cc = static_cast<int32_t>((i0 - cr * nq) * 4 * kGroup) + lc;
  const int32_t rowspan = static_cast<int32_t>(nq * 4 * kGroup);
  auto load = [&](FwdItem& it) {
    it.r = cr;
    it.c = cc;
    it.valid = cc < cols;
    const int32_t g = cc >> 7;
    if (it.valid) {
      it.gw = __ldg(reinterpret_cast<const uint4*>(gate.q + cr * gate.ldq + cc));
      it.uw = __ldg(reinterpret_cast<const uint4*>(up.q + cr * up.ldq + cc));
      it.gs = __ldg(gate.scale + cr * gate.lds + g);
      it.gk = __ldg(gate.k + cr * gate.lds + g);
      it.us = __ldg(up.scale + cr * up.lds + g);
      it.uk = __ldg(up.k + cr * up.lds + g);
    } else {
      it.gw = it.uw = make_uint4(0u, 0u, 0u, 0u);
      it.gs = it.gk = it.us = it.uk = 1.0f;
    }
    cc += 4 * kGroup;
    if (cc >= rowspan) { cc -= rowspan; ++cr; }
  };
  FwdItem cur;
  load(cur);
  for (int64_t item = i0; item < i1; ++item) {
    FwdItem nxt;
    if (item + 1 < i1) load(nxt);

    const bool plain = __all_sync(0xFFFFFFFFu, cur.gk == 1.0f && cur.uk == 1.0f);
    float fg[16], fu[16], h[16];
    decode16_raw<FMT>(cur.gw, cur.gk, plain, tab, fg);
    decode16_raw<FMT>(cur.uw, cur.uk, plain, tab, fu);
    const float ct = cur.gs * -1.4426950408889634f;   // -log2(e) s_g
    const float S = cur.gs * cur.us;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float sg = rcp_approx(1.0f + ex2_approx(fg[i] * ct));
      h[i] = ((fg[i] * fu[i]) * sg) * S;
    }

    // group max |h| (NaN-propagating, so that one test finds NaN and Inf) and,
    // with expansion, min nonzero |h| on twice the bit patterns (zero becomes
    // the largest key)
    float mx = 0.0f;
    uint32_t mink = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      mx = fmax_nan(mx, fabsf(h[i]));
      if (EXPAND) mink = min(mink, __float_as_uint(h[i]) * 2u - 2u);
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      mx = fmax_nan(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      if (EXPAND) mink = min(mink, __shfl_xor_sync(0xFFFFFFFFu, mink, off));
    }
    // slow path: an Inf or a NaN in the group, a scale product that overflowed,
    // or a maximum so small that 1/M would leave FP32 (below 2^-64)
    const bool special = !(mx <= 3.40282347e38f) || !(S <= 3.40282347e38f) ||
                         (mx > 0.0f && mx < 5.421010862427522e-20f);
    uint32_t cw[4];
    float k, sr;
    if (!__any_sync(0xFFFFFFFFu, special)) {
      const float M = mx;
      float invM;
      if (EXPAND) {
        group_params<FMT>(M, __uint_as_float((mink + 2u) >> 1), true, k, sr, invM);
      } else {
        k = 1.0f;
        sr = M > 0.0f ? __fdiv_rn(M, F8<FMT>::MAXV) : 1.0f;   // M / FMT_MAX, correctly rounded
        invM = M > 0.0f ? rcp_approx(M) : 0.0f;   // an all-zero group encodes to zeros
      }
      uint32_t mag[16];
      if (k == 1.0f) {
        const float c = F8<FMT>::MAXV * invM;
#pragma unroll
        for (int i = 0; i < 16; ++i) mag[i] = enc_mag_bounded<FMT>(fabsf(h[i]) * c);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) mag[i] = enc_mag_bounded<FMT>(expand_value<FMT>(h[i], invM, k));
      }
#pragma unroll
      for (int w = 0; w < 4; ++w)
        cw[w] = merge_signs4(pack4(mag[4 * w], mag[4 * w + 1], mag[4 * w + 2], mag[4 * w + 3]),
                             h[4 * w], h[4 * w + 1], h[4 * w + 2], h[4 * w + 3]);
    } else {
      // the codec's slow path: the maximum ignores NaN, IEEE division for k = 1
      float Mn = max_abs_nonnan(h);
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) Mn = fmaxf(Mn, __shfl_xor_sync(0xFFFFFFFFu, Mn, off));
      uint32_t mk2 = 0xFFFFFFFFu;
#pragma unroll
      for (int i = 0; i < 16; ++i) mk2 = min(mk2, __float_as_uint(h[i]) * 2u - 2u);
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) mk2 = min(mk2, __shfl_xor_sync(0xFFFFFFFFu, mk2, off));
      const float M = special ? Mn : mx;
      float invM;
      group_params<FMT>(M, __uint_as_float((mk2 + 2u) >> 1), EXPAND, k, sr, invM);
      const bool use_div = k == 1.0f;
      GroupDiv d{};
      if (use_div) d = codec_div<FMT>(M);
      if (special)
        encode_words<FMT, 16, false>(h, use_div, d, invM, k, cw);
      else
        encode_words<FMT, 16, true>(h, use_div, d, invM, k, cw);
    }
    if (cur.valid) {
      *reinterpret_cast<uint4*>(out.q + cur.r * out.ldq + cur.c) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      if (l == 0) {
        out.scale[cur.r * out.lds + (cur.c >> 7)] = sr;
        out.k[cur.r * out.lds + (cur.c >> 7)] = k;
      }
    }
    cur = nxt;
  }
}

// One thread's backward work item: 16 columns of dh, gate and up.
struct BwdItem {
  uint4 d0, d1;   // dh, bf16 pairs
  uint4 gw, uw;
  float gs, gk, us, uk;
};

template <int FMT>
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const uint16_t* __restrict__ dh,
                                                         int64_t lddh, const ActArgs gate,
                                                         const ActArgs up, int64_t rows,
                                                         int64_t cols, uint16_t* __restrict__ dg,
                                                         int64_t lddg, uint16_t* __restrict__ du,
                                                         int64_t lddu) {
  __shared__ float tab[256];
  fill_log2_table<FMT>(tab);
  __syncthreads();
  const int64_t cpr = cols / 16;   // chunks per row
  const int64_t t0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  const int64_t nt = int64_t(gridDim.x) * blockDim.x;
  const int64_t dr = nt / cpr, dc = nt % cpr;
  int64_t r = t0 / cpr, cc = t0 % cpr;
  auto fetch = [&](int64_t rr, int64_t ch, BwdItem& it) {
    const int64_t c = ch * 16, g = ch >> 3;
    const uint4* dp = reinterpret_cast<const uint4*>(dh + rr * lddh + c);
    it.d0 = __ldcs(dp);
    it.d1 = __ldcs(dp + 1);
    it.gw = __ldcs(reinterpret_cast<const uint4*>(gate.q + rr * gate.ldq + c));
    it.uw = __ldcs(reinterpret_cast<const uint4*>(up.q + rr * up.ldq + c));
    it.gs = __ldg(gate.scale + rr * gate.lds + g);
    it.gk = __ldg(gate.k + rr * gate.lds + g);
    it.us = __ldg(up.scale + rr * up.lds + g);
    it.uk = __ldg(up.k + rr * up.lds + g);
  };
  BwdItem cur;
  if (r < rows) fetch(r, cc, cur);
  while (r < rows) {
    int64_t rn = r + dr, cn = cc + dc;
    if (cn >= cpr) { cn -= cpr; ++rn; }
    BwdItem nxt;
    if (rn < rows) fetch(rn, cn, nxt);

    float g[16], u[16];
    decode16<FMT>(cur.gw, cur.gs, cur.gk, tab, g);
    decode16<FMT>(cur.uw, cur.us, cur.uk, tab, u);
    const uint32_t dw[8] = {cur.d0.x, cur.d0.y, cur.d0.z, cur.d0.w,
                            cur.d1.x, cur.d1.y, cur.d1.z, cur.d1.w};
    uint32_t og[8], ou[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float a[2], b[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * j + e;
        const float d = e ? bf16hi(dw[j]) : bf16lo(dw[j]);
        const float sg = sigmoid(g[i]);
        const float t = d * sg;
        b[e] = t * g[i];                                          // dh silu(g)
        a[e] = (t * u[i]) * __fmaf_rn(g[i], 1.0f - sg, 1.0f);     // dh u s (1 + g (1 - s))
      }
      og[j] = pack_bf16x2(a[0], a[1]);
      ou[j] = pack_bf16x2(b[0], b[1]);
    }
    const int64_t c = cc * 16;
    uint4* gp = reinterpret_cast<uint4*>(dg + r * lddg + c);
    uint4* up_ = reinterpret_cast<uint4*>(du + r * lddu + c);
    gp[0] = make_uint4(og[0], og[1], og[2], og[3]);
    gp[1] = make_uint4(og[4], og[5], og[6], og[7]);
    up_[0] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
    up_[1] = make_uint4(ou[4], ou[5], ou[6], ou[7]);
    r = rn;
    cc = cn;
    cur = nxt;
  }
}

template <int FMT>
void fwd_launch(const ActArgs& gate, const ActArgs& up, int64_t rows, int64_t cols, int expand,
                const ActArgs& out, int dev, cudaStream_t s) {
  auto kern = expand ? swiglu_fwd_kernel<FMT, true> : swiglu_fwd_kernel<FMT, false>;
  const int64_t quads = rows * (((cols + 127) / 128 + 3) / 4);
  const unsigned g = grid_for(quads, 8, dev, resident_ctas(reinterpret_cast<const void*>(kern)));
  kern<<<g, 256, 0, s>>>(gate, up, rows, cols, out);
}

template <int FMT>
void bwd_launch(const uint16_t* dh, int64_t lddh, const ActArgs& gate, const ActArgs& up,
                int64_t rows, int64_t cols, uint16_t* dg, int64_t lddg, uint16_t* du,
                int64_t lddu, int dev, cudaStream_t s) {
  auto kern = swiglu_bwd_kernel<FMT>;
  const unsigned g = grid_for(rows * (cols / 16), 256, dev,
                              resident_ctas(reinterpret_cast<const void*>(kern)));
  kern<<<g, 256, 0, s>>>(dh, lddh, gate, up, rows, cols, dg, lddg, du, lddu);
}

}  // namespace

cudaError_t launch_swiglu_fp8_forward(const ActArgs& gate, const ActArgs& up, int64_t rows,
                                      int64_t cols, int fmt, int expand, const ActArgs& out,
                                      cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  if (cols % 16 != 0) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (fmt == kE4M3) fwd_launch<kE4M3>(gate, up, rows, cols, expand, out, dev, s);
  else if (fmt == kE5M2) fwd_launch<kE5M2>(gate, up, rows, cols, expand, out, dev, s);
  else fwd_launch<kE5M2Full>(gate, up, rows, cols, expand, out, dev, s);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_fp8_backward(const uint16_t* dh, int64_t lddh, const ActArgs& gate,
                                       const ActArgs& up, int64_t rows, int64_t cols, int fmt,
                                       uint16_t* dg, int64_t lddg, uint16_t* du, int64_t lddu,
                                       cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  if (cols % 16 != 0) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // decoding is the same for both E5M2 variants (the span only matters when quantising)
  if (fmt == kE4M3) bwd_launch<kE4M3>(dh, lddh, gate, up, rows, cols, dg, lddg, du, lddu, dev, s);
  else bwd_launch<kE5M2>(dh, lddh, gate, up, rows, cols, dg, lddg, du, lddu, dev, s);
  return cudaGetLastError();
}

}  // namespace coat
