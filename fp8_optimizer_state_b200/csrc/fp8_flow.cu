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

// FP8 codes of 16 signed values y with |y| <= FMT_MAX (1 + 2^-16), four per
// word, by the hardware conversion (cvt.rn.satfinite, two values per
// instruction: round to nearest even, saturating to +-FMT_MAX).  On that range
// it gives the software encoder's codes (tests compare the two on every FP32
// value up to FMT_MAX (1 + 2^-16)), except that it keeps the sign of a value
// that rounds to zero: such codes are set back to 0x00, the library's only
// zero code.
template <int FMT>
__device__ __forceinline__ void encode_hw16(const float (&y)[16], uint32_t (&cw)[4]) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint16_t lo, hi;
    if (FMT == kE4M3) {
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(y[4 * w + 1]), "f"(y[4 * w]));
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(y[4 * w + 3]), "f"(y[4 * w + 2]));
    } else {
      asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(y[4 * w + 1]), "f"(y[4 * w]));
      asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(y[4 * w + 3]), "f"(y[4 * w + 2]));
    }
    const uint32_t v = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    const uint32_t mags = v & 0x7F7F7F7Fu;
    // (mag + 0x7F) has bit 7 set iff mag != 0; adding to four bytes <= 0x7F never carries
    cw[w] = mags | (v & (mags + 0x7F7F7F7Fu) & 0x80808080u);
  }
}

// y with the sign of s (y >= 0).
__device__ __forceinline__ float with_sign_of(float y, float s) {
  return __uint_as_float(__float_as_uint(y) | (__float_as_uint(s) & 0x80000000u));
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

// Quantise the 16 values a lane holds of an 8-lane 1x128 group, as the 1x128
// codec does (called by all 32 lanes of a warp: 4 groups).  Group max |h| by a
// NaN-propagating max (one test then finds NaN and Inf) and, with expansion,
// min nonzero |h| on twice the bit patterns (zero becomes the largest key).
// k = 1 groups encode FMT_MAX |h| / M as |h| (FMT_MAX / M) (a few ulps from the
// correctly rounded quotient, which decides a code only at an exact tie of
// the real-number result; at most FMT_MAX (1 + 2^-21), inside the bounded
// encoder's range) with root scale M / FMT_MAX correctly rounded; expanded
// groups use the codec's expansion.  The slow path (the codec's NaN rules and
// IEEE division) takes groups with a NaN or an Inf, a maximum below 2^-64 or
// above 2^100 (their values are scaled into range there, see range_sigma), or
// force_slow (the same for the 8 lanes of a group).
template <int FMT, bool EXPAND>
__device__ __forceinline__ void quantize_lane16(const float (&h)[16], bool force_slow,
                                                uint32_t (&cw)[4], float& k, float& sr) {
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
  const bool special = !(mx <= 0x1p100f) || force_slow ||
                       (mx > 0.0f && mx < 5.421010862427522e-20f);
  if (!__any_sync(0xFFFFFFFFu, special)) {
    const float M = mx;
    float invM;
    if (EXPAND) {
      group_params<FMT>(M, __uint_as_float((mink + 2u) >> 1), true, k, sr, invM);
    } else {
      k = 1.0f;
      sr = M > 0.0f ? div_fmax<FMT>(M) : 1.0f;   // M / FMT_MAX, correctly rounded
      invM = M > 0.0f ? rcp_approx(M) : 0.0f;   // an all-zero group encodes to zeros
    }
    float y[16];
    if (k == 1.0f) {
      const float c = F8<FMT>::MAXV * invM;
      const float2 c2 = make_float2(c, c);
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float2 q = mul2(make_float2(h[i], h[i + 1]), c2);
        y[i] = q.x;
        y[i + 1] = q.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) y[i] = with_sign_of(expand_value<FMT>(h[i], invM, k), h[i]);
    }
    encode_hw16<FMT>(y, cw);
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
    const float M0 = special ? Mn : mx;
    // a maximum outside [2^-100, 2^100]: the values scaled into range
    const float sig = range_sigma(M0), M = M0 * sig;
    float hs[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) hs[i] = h[i] * sig;
    float invM;
    group_params<FMT>(M, __uint_as_float((mk2 + 2u) >> 1) * sig, EXPAND, k, sr, invM);
    if (sig != 1.0f) sr *= sig < 1.0f ? 0x1p100f : 0x1p-100f;
    if (!EXPAND) sr = M0 > 0.0f ? __fdiv_rn(M0, F8<FMT>::MAXV) : 1.0f;
    const bool use_div = k == 1.0f;
    GroupDiv d{};
    if (use_div) d = codec_div<FMT>(M);
    if (special)
      encode_words<FMT, 16, false>(hs, use_div, d, invM, k, cw);
    else
      encode_words<FMT, 16, true>(hs, use_div, d, invM, k, cw);
  }
}

// Quantise y = p C (C > 0, one value per group) from a lane's 16 values p of
// an 8-lane 1x128 group.  Without expansion the codes are decided on the
// ratio |p_i| / max|p| = |y_i| / max|y| (C cancels, so y itself is never
// rounded); the root scale is max|y| / FMT_MAX.  EXACT: the ratio as one
// correctly rounded division (for exact p an exact tie of the real-number
// result stays a tie and is broken to even, as the oracle does); otherwise
// one multiply by FMT_MAX / max|p| (a few ulps; for p that are not exact
// anyway).  With expansion, and for groups with a NaN/Inf, a maximum |p|
// below 2^-64 or above 2^100 or an unusable C, the values y go through
// quantize_lane16.
template <int FMT, bool EXPAND, bool EXACT>
__device__ __forceinline__ void quantize_scaled16(const float (&p)[16], float C, uint32_t (&cw)[4],
                                                  float& k, float& sr, bool short_sig = false) {
  if (EXPAND) {
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = p[i] * C;
    quantize_lane16<FMT, true>(y, false, cw, k, sr);
    return;
  }
  float mp = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) mp = fmax_nan(mp, fabsf(p[i]));
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) mp = fmax_nan(mp, __shfl_xor_sync(0xFFFFFFFFu, mp, off));
  const float My = mp * C;
  const bool special = !(mp <= 0x1p100f) || !(My <= 3.40282347e38f) || !(C > 0.0f) ||
                       (mp > 0.0f && mp < 5.421010862427522e-20f);
  if (__any_sync(0xFFFFFFFFu, special)) {
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = p[i] * C;
    quantize_lane16<FMT, false>(y, special, cw, k, sr);
    return;
  }
  k = 1.0f;
  sr = My > 0.0f ? div_fmax<FMT>(My) : 1.0f;
  float y[16];
  if (EXACT) {
    // div_exact on the signed values, two at a time: every step rounds to
    // nearest, which is symmetric in the sign, so each result is
    // sign(p) RN(FMT_MAX |p| / max|p|)
    GroupDiv dv;
    if (short_sig)
      dv = codec_div_short<FMT>(mp);   // exact for the short significands of k = 1 products
    else
      dv = codec_div<FMT>(mp);
    const float2 num2 = make_float2(dv.num, dv.num), y2 = make_float2(dv.y, dv.y);
    const float2 nb2 = make_float2(-dv.b, -dv.b);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 a = mul2(make_float2(p[i], p[i + 1]), num2);
      const float2 q0 = mul2(a, y2);
      const float2 q = fma2(fma2(q0, nb2, a), y2, q0);
      y[i] = q.x;
      y[i + 1] = q.y;
    }
  } else {
    const float c = mp > 0.0f ? F8<FMT>::MAXV * rcp_approx(mp) : 0.0f;
    const float2 c2 = make_float2(c, c);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 q = mul2(make_float2(p[i], p[i + 1]), c2);
      y[i] = q.x;
      y[i + 1] = q.y;
    }
  }
  encode_hw16<FMT>(y, cw);
}

// One lane's forward work item: 16 gate and 16 up codes, their groups'
// metadata, and the item's row and the lane's first column.
struct FwdItem {
  uint4 gw, uw;
  float gs, gk, us, uk;
  int64_t oq;   // the lane's first output code: r ldq_out + c
  int64_t om;   // its group's output scale and k: r lds_out + c / 128
  bool valid;   // the lane's 16 columns exist
};

// h = silu(g) u with g = f_g s_g, u = f_u s_u, as ((f_g f_u) sigmoid(g)) (s_g s_u):
// f_g f_u is exact for k = 1 inputs (two FP8 significands); h / (s_g s_u) takes
// one rounding besides the sigmoid's and is quantised with the group's scale
// product by quantize_scaled16 (the product cancels from the codes).
// EXPAND: output expansion on.
// Work: the rows x ceil(groups/4) items (4 groups of a row, 8 lanes each) in
// row-major order, a contiguous range per warp (columns advanced by 512 with
// a row carry); the next item is loaded before the current one is computed.
template <int FMT, bool EXPAND>
__global__ void __launch_bounds__(256, 3) swiglu_fwd_kernel(const ActArgs gate, const ActArgs up,
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
  // row offsets of the next item's row in each array, advanced by one row
  // stride at a row carry (no per-item 64-bit multiplies)
  int64_t rg = cr * gate.ldq, ru = cr * up.ldq, rmg = cr * gate.lds, rmu = cr * up.lds;
  int64_t ro = cr * out.ldq, rmo = cr * out.lds;
  auto load = [&](FwdItem& it) {
    it.oq = ro + cc;
    it.valid = cc < cols && COAT_INDEX_OK(cr < rows && cc + 16 <= cols);
    const int32_t g = cc >> 7;
    it.om = rmo + g;
    if (it.valid) {
      it.gw = __ldg(reinterpret_cast<const uint4*>(gate.q + rg + cc));
      it.uw = __ldg(reinterpret_cast<const uint4*>(up.q + ru + cc));
      it.gs = __ldg(gate.scale + rmg + g);
      it.gk = __ldg(gate.k + rmg + g);
      it.us = __ldg(up.scale + rmu + g);
      it.uk = __ldg(up.k + rmu + g);
    } else {
      it.gw = it.uw = make_uint4(0u, 0u, 0u, 0u);
      it.gs = it.gk = it.us = it.uk = 1.0f;
    }
    cc += 4 * kGroup;
    if (cc >= rowspan) {
      cc -= rowspan;
      ++cr;
      rg += gate.ldq;
      ru += up.ldq;
      rmg += gate.lds;
      rmu += up.lds;
      ro += out.ldq;
      rmo += out.lds;
    }
  };
  auto body = [&](const FwdItem& cur) {
    const bool plain = __all_sync(0xFFFFFFFFu, cur.gk == 1.0f && cur.uk == 1.0f);
    float fg[16], fu[16], h[16];
    decode16_raw<FMT>(cur.gw, cur.gk, plain, tab, fg);
    decode16_raw<FMT>(cur.uw, cur.uk, plain, tab, fu);
    const float ct = cur.gs * -1.4426950408889634f;   // -log2(e) s_g
    const float S = cur.gs * cur.us;
    const float2 ct2 = make_float2(ct, ct), one2 = make_float2(1.0f, 1.0f);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      // sigmoid(g) = 1 / (1 + 2^(-log2(e) g)) and h / (s_g s_u) = (f_g f_u) sigmoid(g),
      // two elements per operation
      const float2 f = make_float2(fg[i], fg[i + 1]);
      const float2 e = mul2(f, ct2);
      const float2 den = add2(make_float2(ex2_approx(e.x), ex2_approx(e.y)), one2);
      const float2 hh = mul2(mul2(f, make_float2(fu[i], fu[i + 1])),
                             make_float2(rcp_approx(den.x), rcp_approx(den.y)));
      h[i] = hh.x;
      h[i + 1] = hh.y;
    }

    uint32_t cw[4];
    float k, sr;
    quantize_scaled16<FMT, EXPAND, false>(h, S, cw, k, sr);
    if (cur.valid) {
      *reinterpret_cast<uint4*>(out.q + cur.oq) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      if (l == 0) {
        out.scale[cur.om] = sr;
        out.k[cur.om] = k;
      }
    }
  };
  FwdItem cur;
  load(cur);
  for (int64_t item = i0; item < i1; ++item) {
    FwdItem nxt;
    if (item + 1 < i1) load(nxt);
    body(cur);
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
    if (!COAT_INDEX_OK(rr < rows && c + 16 <= cols)) {
      it = BwdItem{};
      return;
    }
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
    if (COAT_INDEX_OK(c + 16 <= cols)) {
      uint4* gp = reinterpret_cast<uint4*>(dg + r * lddg + c);
      uint4* up_ = reinterpret_cast<uint4*>(du + r * lddu + c);
      gp[0] = make_uint4(og[0], og[1], og[2], og[3]);
      gp[1] = make_uint4(og[4], og[5], og[6], og[7]);
      up_[0] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
      up_[1] = make_uint4(ou[4], ou[5], ou[6], ou[7]);
    }
    r = rn;
    cc = cn;
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// RMSNorm, the other non-linear layer of a Llama block:
// y = x / sqrt(mean(x^2) + eps) * w per row of d features (d a multiple of
// 128, at most 256 * 16 * 2), FP8 1x128 input and output, bf16 w.  One CTA of
// NT threads (128 or 256) per row at a time (a persistent loop over rows);
// thread t holds the 16-column chunks t, t + NT, ... (CPT of them), so that 8
// consecutive threads hold one 128-column group and w stays in registers
// across rows.  Row sums go through warp shuffles and shared memory.  The
// backward uses 256-thread CTAs.
// ---------------------------------------------------------------------------
constexpr int kNormThreads = 256;

// Sum of v over the NT threads of the CTA, returned to every thread (red: NT/32
// floats per value, reused only after the barrier that ends this call's reads).
template <int NV, int NT>
__device__ __forceinline__ void cta_sum_all(float (&v)[NV], float (*red)[NT / 32]) {
#pragma unroll
  for (int n = 0; n < NV; ++n)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v[n] += __shfl_xor_sync(0xFFFFFFFFu, v[n], off);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int n = 0; n < NV; ++n) red[n][warp] = v[n];
  __syncthreads();
#pragma unroll
  for (int n = 0; n < NV; ++n) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) t += red[n][w];
    v[n] = t;
  }
  __syncthreads();
}

// 16 bf16 values to floats.
__device__ __forceinline__ void bf16x16(const uint4& a, const uint4& b, float (&f)[16]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    f[2 * j] = bf16lo(w[j]);
    f[2 * j + 1] = bf16hi(w[j]);
  }
}

template <int FMT, bool EXPAND, int CPT, int NT>
__global__ void __launch_bounds__(NT, CPT == 2 ? 16 / (NT / 32) : 1) rmsnorm_fwd_kernel(const ActArgs x,
                                                                   const uint16_t* __restrict__ w,
                                                                   int64_t rows, int64_t d,
                                                                   float eps, const ActArgs out) {
  constexpr int NW = NT / 32;
  __shared__ float tab[256];
  __shared__ float red[1][NW];
  __shared__ double redd[NW];    // the row's warp partials in double, when its FP32 sum overflows
  fill_log2_table<FMT>(tab);
  __syncthreads();
  const float inv_d = 1.0f / static_cast<float>(d);
  const int warp = threadIdx.x >> 5;
  float wv[CPT][16];
  bool ok[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int64_t c = (threadIdx.x + int64_t(j) * NT) * 16;
    ok[j] = c < d;
    if (ok[j]) {
      const uint4* wp = reinterpret_cast<const uint4*>(w + c);
      bf16x16(__ldg(wp), __ldg(wp + 1), wv[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) wv[j][i] = 0.0f;
    }
  }
  // the next row's codes and metadata are loaded before this row's work
  struct In { uint4 q; float s, k; };
  auto load = [&](int64_t r, In (&in)[CPT]) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int64_t c = (threadIdx.x + int64_t(j) * NT) * 16;
      in[j].q = make_uint4(0u, 0u, 0u, 0u);
      in[j].s = in[j].k = 1.0f;
      if (ok[j]) {
        in[j].q = __ldcs(reinterpret_cast<const uint4*>(x.q + r * x.ldq + c));
        in[j].s = __ldg(x.scale + r * x.lds + (c >> 7));
        in[j].k = __ldg(x.k + r * x.lds + (c >> 7));
      }
    }
  };
  auto body = [&](int64_t r, const In (&cur)[CPT]) {
    // p = f w (f the FP8 value, or |q|^(1/k) with its sign; x = f s): exact
    // for k = 1 (an FP8 value times a bf16 value); the row's sum of x^2 as
    // the sum over chunks of (sum of f^2) s^2
    float pv[CPT][16], sfv[CPT];
    bool plain[CPT];
    float ss[1] = {0.0f};
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      plain[j] = __all_sync(0xFFFFFFFFu, cur[j].k == 1.0f);
      float f[16];
      decode16_raw<FMT>(cur[j].q, cur[j].k, plain[j], tab, f);
      float2 sf = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float2 f2 = make_float2(f[i], f[i + 1]);
        sf = fma2(f2, f2, sf);
        const float2 p2 = mul2(f2, make_float2(wv[j][i], wv[j][i + 1]));
        pv[j][i] = p2.x;
        pv[j][i + 1] = p2.y;
      }
      sfv[j] = sf.x + sf.y;
      ss[0] = __fmaf_rn(sfv[j], cur[j].s * cur[j].s, ss[0]);
    }
    cta_sum_all<1, NT>(ss, red);
    float C[CPT];
    if (ss[0] <= 3.40282347e38f) {
      // rstd only scales the root scales (the codes depend on p / max|p| alone)
      const float rstd = rsqrt_approx(__fmaf_rn(ss[0], inv_d, eps));
#pragma unroll
      for (int j = 0; j < CPT; ++j) C[j] = cur[j].s * rstd;
    } else {
      // The FP32 sum is Inf or NaN (CTA-uniform).  Finite inputs whose x^2
      // sum leaves FP32 are summed again in double, where no such sum
      // overflows; the scale products s rstd are formed in double and rounded
      // once.  A NaN or an Inf input keeps a non-finite sum.
      double sd = 0.0;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const double sj = static_cast<double>(cur[j].s);
        sd = fma(static_cast<double>(sfv[j]), sj * sj, sd);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sd += __shfl_xor_sync(0xFFFFFFFFu, sd, off);
      if ((threadIdx.x & 31) == 0) redd[warp] = sd;
      __syncthreads();
      double td = 0.0;
#pragma unroll
      for (int v = 0; v < NW; ++v) td += redd[v];
      const double rstd = 1.0 / sqrt(td / static_cast<double>(d) + static_cast<double>(eps));
#pragma unroll
      for (int j = 0; j < CPT; ++j) C[j] = static_cast<float>(static_cast<double>(cur[j].s) * rstd);
    }
    auto store = [&](int j, const uint32_t (&cw)[4], float sr, float k) {
      const int64_t c = (threadIdx.x + int64_t(j) * NT) * 16;
      if (ok[j] && COAT_INDEX_OK(c + 16 <= d)) {
        *reinterpret_cast<uint4*>(out.q + r * out.ldq + c) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        if ((threadIdx.x & 7) == 0) {
          out.scale[r * out.lds + (c >> 7)] = sr;
          out.k[r * out.lds + (c >> 7)] = k;
        }
      }
    };
    // Without expansion, when no group of the warp's chunks needs the general
    // path, the chunks are quantised in one block without branches, so that
    // their dependency chains interleave: the group maxima and their shuffles,
    // one vote over every range condition, the divisions by a Newton
    // reciprocal (exact for the short significands of k = 1 products, within
    // an ulp for expanded inputs, whose products are approximate anyway) and
    // the root scales by the correction step without its range test.  Every
    // other case takes quantize_scaled16 chunk by chunk.
    bool fast = false;
    float mp[CPT], My[CPT];
    if constexpr (!EXPAND) {
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmax_nan(m, fabsf(pv[j][i]));
        mp[j] = m;
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1)
#pragma unroll
        for (int j = 0; j < CPT; ++j) mp[j] = fmax_nan(mp[j], __shfl_xor_sync(0xFFFFFFFFu, mp[j], off));
      bool sp = false;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        My[j] = mp[j] * C[j];
        sp = sp || !(mp[j] <= 0x1p100f) || (mp[j] > 0.0f && mp[j] < 5.421010862427522e-20f) ||
             !(My[j] <= 3.40282347e38f) || !(C[j] > 0.0f) ||
             (My[j] > 0.0f && My[j] < 7.888609052210118e-31f);
      }
      fast = !__any_sync(0xFFFFFFFFu, sp);
    }
    if (fast) {
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const GroupDiv dv = codec_div_short<FMT>(mp[j]);
        const float2 num2 = make_float2(dv.num, dv.num), y2 = make_float2(dv.y, dv.y);
        const float2 nb2 = make_float2(-dv.b, -dv.b);
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          // sign(p) RN(FMT_MAX |p| / max|p|): every step rounds to nearest,
          // which is symmetric in the sign
          const float2 a = mul2(make_float2(pv[j][i], pv[j][i + 1]), num2);
          const float2 q0 = mul2(a, y2);
          const float2 q = fma2(fma2(q0, nb2, a), y2, q0);
          y[i] = q.x;
          y[i + 1] = q.y;
        }
        uint32_t cw[4];
        encode_hw16<FMT>(y, cw);
        // M / FMT_MAX correctly rounded (div_fmax's step; My is in its range)
        const float q0 = My[j] * F8<FMT>::RCPMAX;
        const float sr = My[j] > 0.0f
                             ? __fmaf_rn(__fmaf_rn(-q0, F8<FMT>::MAXV, My[j]), F8<FMT>::RCPMAX, q0)
                             : 1.0f;
        store(j, cw, sr, 1.0f);
      }
    } else {
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        uint32_t cw[4];
        float k, sr;
        quantize_scaled16<FMT, EXPAND, true>(pv[j], C[j], cw, k, sr, plain[j]);
        store(j, cw, sr, k);
      }
    }
  };
  In cur[CPT];
  if (blockIdx.x < rows) load(blockIdx.x, cur);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    In nxt[CPT];
    if (r + gridDim.x < rows) load(r + gridDim.x, nxt);
    body(r, cur);
#pragma unroll
    for (int j = 0; j < CPT; ++j) cur[j] = nxt[j];
  }
}

// Backward: with xh = x rstd and g = dy w,
//   dx = rstd (g - xh mean(g xh)) = rstd g - (rstd^2 mean) x,
// and each CTA sums dy xh over its rows into its own row of `partial`
// (partial[blockIdx.x][0..d)); rmsnorm_dw_kernel adds the rows in index order.
template <int FMT, int CPT>
__global__ void __launch_bounds__(kNormThreads) rmsnorm_bwd_kernel(
    const uint16_t* __restrict__ dy, int64_t lddy, const ActArgs x,
    const uint16_t* __restrict__ w, int64_t rows, int64_t d, float eps,
    uint16_t* __restrict__ dx, int64_t lddx, float* __restrict__ partial) {
  __shared__ float tab[256];
  __shared__ float red[2][kNormThreads / 32];
  fill_log2_table<FMT>(tab);
  __syncthreads();
  const float inv_d = 1.0f / static_cast<float>(d);
  float wv[CPT][16], acc[CPT][16];
  bool ok[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int64_t c = (threadIdx.x + int64_t(j) * kNormThreads) * 16;
    ok[j] = c < d;
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[j][i] = 0.0f;
    if (ok[j]) {
      const uint4* wp = reinterpret_cast<const uint4*>(w + c);
      bf16x16(__ldg(wp), __ldg(wp + 1), wv[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) wv[j][i] = 0.0f;
    }
  }
  // the next row's codes, scales and dy are loaded before this row's reduction
  struct In { uint4 q, d0, d1; float s, k; };
  auto load = [&](int64_t r, In (&in)[CPT]) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int64_t c = (threadIdx.x + int64_t(j) * kNormThreads) * 16;
      in[j].q = in[j].d0 = in[j].d1 = make_uint4(0u, 0u, 0u, 0u);
      in[j].s = in[j].k = 1.0f;
      if (ok[j]) {
        in[j].q = __ldcs(reinterpret_cast<const uint4*>(x.q + r * x.ldq + c));
        in[j].s = __ldg(x.scale + r * x.lds + (c >> 7));
        in[j].k = __ldg(x.k + r * x.lds + (c >> 7));
        const uint4* dp = reinterpret_cast<const uint4*>(dy + r * lddy + c);
        in[j].d0 = __ldcs(dp);
        in[j].d1 = __ldcs(dp + 1);
      }
    }
  };
  In cur[CPT];
  if (blockIdx.x < rows) load(blockIdx.x, cur);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    In nxt[CPT];
    if (r + gridDim.x < rows) load(r + gridDim.x, nxt);
    // pass 1: the row sums, element pairs in two interleaved partial sums each;
    // the decoded values are not kept across the barrier
    float sums[2];   // sum x^2, sum g x
    {
      float2 sxx = make_float2(0.0f, 0.0f), sgx = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const bool plain = __all_sync(0xFFFFFFFFu, cur[j].k == 1.0f);
        float f[16], dv[16];
        decode16_raw<FMT>(cur[j].q, cur[j].k, plain, tab, f);
        bf16x16(cur[j].d0, cur[j].d1, dv);
        const float2 s2 = make_float2(cur[j].s, cur[j].s);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float2 xv = mul2(make_float2(f[i], f[i + 1]), s2);
          const float2 g = mul2(make_float2(dv[i], dv[i + 1]), make_float2(wv[j][i], wv[j][i + 1]));
          sxx = fma2(xv, xv, sxx);
          sgx = fma2(g, xv, sgx);
        }
      }
      sums[0] = sxx.x + sxx.y;
      sums[1] = sgx.x + sgx.y;
    }
    cta_sum_all<2, kNormThreads>(sums, red);
    const float rstd = rsqrt_approx(__fmaf_rn(sums[0], inv_d, eps));
    // rstd^2 mean(g xh) = rstd^3 sum(g x) / d
    const float cx = rstd * rstd * rstd * sums[1] * inv_d;
    const float2 rstd2 = make_float2(rstd, rstd), ncx2 = make_float2(-cx, -cx);
    // pass 2: dx and the dw sums, decoding again, element pairs
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const bool plain = __all_sync(0xFFFFFFFFu, cur[j].k == 1.0f);
      float f[16], dv[16];
      decode16_raw<FMT>(cur[j].q, cur[j].k, plain, tab, f);
      bf16x16(cur[j].d0, cur[j].d1, dv);
      const float2 s2 = make_float2(cur[j].s, cur[j].s);
      uint32_t o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = 2 * e;
        const float2 dv2 = make_float2(dv[i], dv[i + 1]);
        const float2 xv = mul2(make_float2(f[i], f[i + 1]), s2);
        const float2 g = mul2(dv2, make_float2(wv[j][i], wv[j][i + 1]));
        // dx = rstd g - cx x; dw += dy x rstd
        const float2 a = fma2(rstd2, g, mul2(ncx2, xv));
        const float2 ac = fma2(dv2, mul2(xv, rstd2), make_float2(acc[j][i], acc[j][i + 1]));
        acc[j][i] = ac.x;
        acc[j][i + 1] = ac.y;
        o[e] = pack_bf16x2(a.x, a.y);
      }
      const int64_t c = (threadIdx.x + int64_t(j) * kNormThreads) * 16;
      if (ok[j] && COAT_INDEX_OK(c + 16 <= d)) {
        uint4* op = reinterpret_cast<uint4*>(dx + r * lddx + c);
        op[0] = make_uint4(o[0], o[1], o[2], o[3]);
        op[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
#pragma unroll
    for (int j = 0; j < CPT; ++j) cur[j] = nxt[j];
  }
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int64_t c = (threadIdx.x + int64_t(j) * kNormThreads) * 16;
    if (!ok[j] || !COAT_INDEX_OK(c + 16 <= d)) continue;
    float4* pp = reinterpret_cast<float4*>(partial + blockIdx.x * d + c);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      pp[v] = make_float4(acc[j][4 * v], acc[j][4 * v + 1], acc[j][4 * v + 2], acc[j][4 * v + 3]);
  }
}

// dw[c] = sum over the nparts rows of partial[., c] in double, in a fixed
// order: a 1024-thread CTA takes 32 columns; warp w adds rows w, w + 32, ...
// (coalesced 128-byte reads, four loads in flight), then warp 0 adds the 32
// warp sums.
constexpr int kDwCols = 32;
constexpr int kDwThreads = 1024;
__global__ void __launch_bounds__(kDwThreads) rmsnorm_dw_kernel(const float* __restrict__ partial,
                                                                int nparts, int64_t d,
                                                                float* __restrict__ dw) {
  constexpr int kWarps = kDwThreads / 32;
  __shared__ double red[kWarps][kDwCols];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c = blockIdx.x * int64_t(kDwCols) + lane;
  double t = 0.0;
  if (c < d) {
    int p = warp;
    for (; p + 3 * kWarps < nparts; p += 4 * kWarps) {
      const float a0 = __ldg(partial + int64_t(p) * d + c);
      const float a1 = __ldg(partial + int64_t(p + kWarps) * d + c);
      const float a2 = __ldg(partial + int64_t(p + 2 * kWarps) * d + c);
      const float a3 = __ldg(partial + int64_t(p + 3 * kWarps) * d + c);
      t += static_cast<double>(a0);
      t += static_cast<double>(a1);
      t += static_cast<double>(a2);
      t += static_cast<double>(a3);
    }
    for (; p < nparts; p += kWarps) t += static_cast<double>(__ldg(partial + int64_t(p) * d + c));
  }
  red[warp][lane] = t;
  __syncthreads();
  if (warp == 0 && c < d) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][lane];
    dw[c] = static_cast<float>(s);
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

constexpr int kNormMaxCtasPerSm = 8;

template <int FMT, bool EXPAND, int CPT, int NT>
cudaError_t rms_fwd_launch(const ActArgs& x, const uint16_t* w, int64_t rows, int64_t d, float eps,
                           const ActArgs& out, int dev, cudaStream_t s) {
  auto kern = rmsnorm_fwd_kernel<FMT, EXPAND, CPT, NT>;
  const int per_sm = resident_ctas(reinterpret_cast<const void*>(kern), 0, NT);
  const unsigned g = grid_for(rows, 1, dev, per_sm < kNormMaxCtasPerSm ? per_sm : kNormMaxCtasPerSm);
  kern<<<g, NT, 0, s>>>(x, w, rows, d, eps, out);
  return cudaGetLastError();
}

// The forward's shape for rows of d features: 128-thread CTAs holding one or
// two 16-column chunks per thread up to d = 4096 (so that a thread's per-row
// work -- its part of the row sum, the group maxima and divisors -- covers as
// many elements as the registers allow, and an SM keeps four rows in flight),
// 256 threads with two chunks above.
template <int FMT, bool EXPAND>
cudaError_t rms_fwd_dispatch(const ActArgs& x, const uint16_t* w, int64_t rows, int64_t d,
                             float eps, const ActArgs& out, int dev, cudaStream_t s) {
  if (d <= 128 * 16) return rms_fwd_launch<FMT, EXPAND, 1, 128>(x, w, rows, d, eps, out, dev, s);
  if (d <= 128 * 32) return rms_fwd_launch<FMT, EXPAND, 2, 128>(x, w, rows, d, eps, out, dev, s);
  return rms_fwd_launch<FMT, EXPAND, 2, kNormThreads>(x, w, rows, d, eps, out, dev, s);
}

template <int FMT, int CPT>
cudaError_t rms_bwd_launch(const uint16_t* dy, int64_t lddy, const ActArgs& x, const uint16_t* w,
                           int64_t rows, int64_t d, float eps, uint16_t* dx, int64_t lddx,
                           float* dw, float* partial, int dev, cudaStream_t s) {
  auto kern = rmsnorm_bwd_kernel<FMT, CPT>;
  const int per_sm = resident_ctas(reinterpret_cast<const void*>(kern));
  const unsigned g = grid_for(rows, 1, dev, per_sm < kNormMaxCtasPerSm ? per_sm : kNormMaxCtasPerSm);
  kern<<<g, kNormThreads, 0, s>>>(dy, lddy, x, w, rows, d, eps, dx, lddx, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  rmsnorm_dw_kernel<<<static_cast<unsigned>((d + kDwCols - 1) / kDwCols), kDwThreads, 0, s>>>(
      partial, static_cast<int>(g), d, dw);
  return cudaGetLastError();
}

}  // namespace

COAT_INDEX_FAULT_READER(index_faults_flow)

size_t rmsnorm_workspace_bytes(int dev, int64_t d) {
  return sizeof(float) * size_t(sm_count(dev)) * kNormMaxCtasPerSm * size_t(d);
}

int64_t rmsnorm_max_d() { return int64_t(kNormThreads) * 16 * 2; }

cudaError_t launch_rmsnorm_fp8_forward(const ActArgs& x, const uint16_t* w, int64_t rows, int64_t d,
                                       float eps, int fmt, int expand, const ActArgs& out,
                                       cudaStream_t s) {
  if (rows == 0 || d == 0) return cudaSuccess;
  if (d % kGroup != 0 || d > rmsnorm_max_d()) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
#define COAT_RMS_FWD(F)                                                                        \
  return expand ? rms_fwd_dispatch<F, true>(x, w, rows, d, eps, out, dev, s)                   \
                : rms_fwd_dispatch<F, false>(x, w, rows, d, eps, out, dev, s);
  if (fmt == kE4M3) { COAT_RMS_FWD(kE4M3) }
  if (fmt == kE5M2) { COAT_RMS_FWD(kE5M2) }
  COAT_RMS_FWD(kE5M2Full)
#undef COAT_RMS_FWD
}

cudaError_t launch_rmsnorm_fp8_backward(const uint16_t* dy, int64_t lddy, const ActArgs& x,
                                        const uint16_t* w, int64_t rows, int64_t d, float eps,
                                        int fmt, uint16_t* dx, int64_t lddx, float* dw,
                                        float* partial, cudaStream_t s) {
  if (d == 0) return cudaSuccess;
  if (d % kGroup != 0 || d > rmsnorm_max_d()) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (rows == 0) return cudaMemsetAsync(dw, 0, sizeof(float) * size_t(d), s);
  const bool two = d > int64_t(kNormThreads) * 16;
  // decoding is the same for both E5M2 variants
  if (fmt == kE4M3)
    return two ? rms_bwd_launch<kE4M3, 2>(dy, lddy, x, w, rows, d, eps, dx, lddx, dw, partial, dev, s)
               : rms_bwd_launch<kE4M3, 1>(dy, lddy, x, w, rows, d, eps, dx, lddx, dw, partial, dev, s);
  return two ? rms_bwd_launch<kE5M2, 2>(dy, lddy, x, w, rows, d, eps, dx, lddx, dw, partial, dev, s)
             : rms_bwd_launch<kE5M2, 1>(dy, lddy, x, w, rows, d, eps, dx, lddx, dw, partial, dev, s);
}

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
