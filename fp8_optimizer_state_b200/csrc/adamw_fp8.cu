// adamw_fp8.cu -- the fused COAT AdamW step over FP8 moments on sm_100a.
//
// What it computes ([P1] "FP8训练新范式：减少40%显存占用，训练速度提高1.4倍",
// sections "FP8优化器状态" and "解决方案：动态范围扩展"; AdamW as in
// torch.optim.AdamW): per group of 128 elements, dequantise the FP8 moments
// (x = sign(q) s_r |q|^(1/k)), update them with the bf16 gradient, apply the
// decoupled-weight-decay AdamW update to the FP32 master weight, write its
// bf16 copy, recompute each moment's expansion exponent k and root scale from
// the new group max/min, and requantise.
//
// Design (HBM-bound: 16.25 algorithmic bytes per parameter, no tensor cores):
//  * one persistent CTA per SM, 16 warps (4 per SM sub-partition, so a thread
//    may use 128 registers); tiles of 60 groups (7680 elements); CTA b takes
//    tiles b, b + grid, b + 2 grid, ...;
//  * one producer thread streams whole tiles (master, grad, both code arrays,
//    the four metadata arrays: 62,400 B) into a 3-stage shared-memory ring
//    with 1-D cp.async.bulk copies completing on an mbarrier (30 KB per copy
//    of the master array), so that bytes in flight do not depend on
//    registers; every byte is read once, so the copies carry an L2
//    evict-first policy and the results are written with streaming stores.
//    It walks the tensor list forward with its tiles, keeps the current
//    tensor's descriptor in registers and writes the tile's array pointers
//    into the stage header;
//  * 15 consumer warps; each warp owns 4 groups of a tile, 8 lanes per group,
//    16 elements per lane in 4 chunks of 4 contiguous elements (chunk order
//    rotated per group to keep shared-memory reads conflict-free); group
//    max / min-nonzero by 3 xor-shuffles inside the 8 lanes;
//  * a consumer copies its slice of the stage into registers and releases the
//    stage before computing; results go straight to HBM with coalesced
//    16/8/4-byte stores (every warp store instruction writes whole sectors);
//  * fully valid tiles run a specialised body with no bounds logic; a
//    tensor's last tile, when not fully valid, takes a direct path: the
//    consumers load from global memory with bounds checks, padding elements
//    count as zero and their codes are written 0;
//  * every mbarrier wait is bounded (about a second); on timeout the kernel
//    sets a device error bit and returns (the producer first waits, bounded,
//    for the copies it still has in flight).
#include <cstdint>
#include <cuda_runtime.h>

#include "coat_device.cuh"
#include "coat_internal.h"

namespace coat {
namespace {

constexpr int kConsumerWarps = 15;
constexpr int kGroupsPerWarp = 4;
constexpr int kTileGroups = kConsumerWarps * kGroupsPerWarp;  // 60
constexpr int kTileElems = kTileGroups * kGroup;               // 7680
constexpr int kStages = 3;
constexpr int kThreads = (kConsumerWarps + 1) * 32;             // 512
constexpr int kCtasPerSm = 1;

// Stage layout (bytes): the element arrays start on 128-byte boundaries, the
// metadata arrays (240 B each) on 16-byte boundaries; stages are padded to a
// multiple of 128 bytes.
constexpr uint32_t kOffMaster = 0;
constexpr uint32_t kOffGrad = kOffMaster + kTileElems * 4;   // 30720
constexpr uint32_t kOffMq = kOffGrad + kTileElems * 2;       // 46080
constexpr uint32_t kOffVq = kOffMq + kTileElems;             // 53760
constexpr uint32_t kOffMs = kOffVq + kTileElems;             // 61440
constexpr uint32_t kOffMk = kOffMs + kTileGroups * 4;
constexpr uint32_t kOffVs = kOffMk + kTileGroups * 4;
constexpr uint32_t kOffVk = kOffVs + kTileGroups * 4;
constexpr uint32_t kTxBytes = kOffVk + kTileGroups * 4;      // 62400 copied per tile
constexpr uint32_t kStageBytes = ((kTxBytes + 127) / 128) * 128;
static_assert(kTileElems % 16 == 0 && (kTileGroups * 4) % 16 == 0, "bulk copies need 16-byte sizes");

// What the lanes need of a tile: its tensor's arrays offset to the tile's
// first element (and first group, for the per-group arrays), so that a lane
// addresses everything with its own tile-invariant 32-bit offsets.
struct __align__(16) TileHeader {
  float* master;
  uint16_t* wout;  // null: no bf16 copy
  uint8_t* mq;
  uint8_t* vq;
  float* ms;
  float* mk;
  float* vs;
  float* vk;
  const uint16_t* grad;
  int32_t nvalid;   // elements of the tile that exist (kTileElems: full tile, staged)
  int32_t ngroups;  // groups of the tile that exist
  float lrwd;       // lr * wd of the tile's tensor (lr * wd * wd_scale)
};

constexpr int64_t kNoTile = 0x7FFFFFFFFFFFFFFFLL;

// The producer's current tensor: its descriptor and where the next one starts.
struct Feed {
  TensorArgs d;
  int64_t next_begin;  // first tile of the next tensor (kNoTile: none)
  int32_t ti;          // index of the current tensor
};

// log2(F) and 1/F for F = 1 + (j + 1/2)/128, the centre of the j-th of 128
// equal bins of [1, 2) (log2_table below).
struct LogEntry {
  double log2f, inv;
};

struct Smem {
  double tabd_m[256];   // log2|value(code)| of the m format, double (group extremes)
  double tabd_v[256];   // log2|value(code)| of the v format, double
  LogEntry lgt[128];
  double exp2_16[16];   // 2^(j/16), double
  float tab_m[256];     // log2|value(code)| of the m format
  float tab_v[256];     // log2|value(code)| of the v format
  uint64_t full_bar[kStages];
  uint64_t empty_bar[kStages];
  TileHeader hdr[kStages];
  // each consumer lane's m codes, v codes and gradients of the current tile
  // (64 bytes: 16 + 16 + 32), read back by the lanes that recompute a group's
  // extreme elements
  uint4 scratch[kConsumerWarps * 32 * 4];
};
constexpr size_t kSmemHead = ((sizeof(Smem) + 127) / 128) * 128;
constexpr size_t kSmemBytes = kSmemHead + size_t(kStages) * kStageBytes;
static_assert(kSmemBytes * kCtasPerSm <= 227 * 1024, "shared memory per SM");

// Tile -> tensor.  Tensor i owns tiles [tile_begin_i, tile_begin_i + tiles_i),
// in ascending order; an empty tensor shares the next tensor's first tile.
// Single-tensor launches pass one descriptor by value.
struct SingleTensor {
  TensorArgs t;
  __device__ __forceinline__ int64_t tiles() const { return t.tiles; }
  __device__ __forceinline__ int32_t find(int64_t) const { return 0; }
  __device__ __forceinline__ TensorArgs get(int32_t) const { return t; }
  __device__ __forceinline__ int64_t begin_of(int32_t) const { return kNoTile; }  // no successor
  __device__ __forceinline__ int32_t advance(int32_t ti, int64_t) const { return ti; }
};
// Multi-tensor launches read a device table of descriptors; the producer finds
// the tensor of its first tile by binary search (the last tensor whose first
// tile is <= the tile, which skips empty tensors) and then walks forward.
struct MultiTensor {
  const TensorArgs* descs;
  int32_t num;
  int64_t total_tiles;
  __device__ __forceinline__ int64_t tiles() const { return total_tiles; }
  __device__ __forceinline__ int32_t find(int64_t tile) const {
    int32_t lo = 0, hi = num - 1;
    while (lo < hi) {
      const int32_t mid = (lo + hi + 1) >> 1;
      if (descs[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  __device__ __forceinline__ TensorArgs get(int32_t i) const { return descs[i]; }
  __device__ __forceinline__ int64_t begin_of(int32_t i) const {
    return i < num ? descs[i].tile_begin : kNoTile;
  }
  // The tensor of `tile` (the last one whose first tile is <= tile), searching
  // forward from tensor ti, which starts at or before it.  Eight first-tile
  // indices are read per round with independent loads, so a jump across many
  // small tensors costs one memory latency per eight of them.
  __device__ __forceinline__ int32_t advance(int32_t ti, int64_t tile) const {
    for (;;) {
      int64_t b[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) b[k] = begin_of(ti + 1 + k);
      int c = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) c += b[k] <= tile ? 1 : 0;
      ti += c;
      if (c < 8) return ti;
    }
  }
};

// The 16 elements a lane owns, as loaded.
struct LaneIn {
  float4 p[4];
  uint2 g[4];
  uint32_t mq[4], vq[4];
  float ms, mk, vs, vk;
};

__device__ __forceinline__ int chunk_of(int j, int slot) { return (j + slot) & 3; }

__device__ __forceinline__ void load_from_stage(const uint8_t* st, const int (&off)[4], int lg,
                                                LaneIn& in) {
  const float* sm = reinterpret_cast<const float*>(st + kOffMaster);
  const uint16_t* sg = reinterpret_cast<const uint16_t*>(st + kOffGrad);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = off[j];
    in.p[j] = *reinterpret_cast<const float4*>(sm + e);
    in.g[j] = *reinterpret_cast<const uint2*>(sg + e);
    in.mq[j] = *reinterpret_cast<const uint32_t*>(st + kOffMq + e);
    in.vq[j] = *reinterpret_cast<const uint32_t*>(st + kOffVq + e);
  }
  in.ms = reinterpret_cast<const float*>(st + kOffMs)[lg];
  in.mk = reinterpret_cast<const float*>(st + kOffMk)[lg];
  in.vs = reinterpret_cast<const float*>(st + kOffVs)[lg];
  in.vk = reinterpret_cast<const float*>(st + kOffVk)[lg];
}

// Direct loads for a tile that is not entirely valid.  Elements at or beyond
// the tile's valid count read as zero; codes of a group that exists are always
// readable (the code arrays hold whole groups).  off[j]: the lane's element
// offsets within the tile; lg: its group within the tile.
__device__ __forceinline__ void load_direct(const TileHeader& hd, const int (&off)[4], int lg,
                                            bool active, LaneIn& in) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = off[j];
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
    uint2 g = make_uint2(0u, 0u);
    uint32_t mq = 0u, vq = 0u;
    if (active) {
      if (e + 4 <= hd.nvalid) {
        p = *reinterpret_cast<const float4*>(hd.master + e);
        g = *reinterpret_cast<const uint2*>(hd.grad + e);
      } else {
        float pv[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t gv[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (e + i < hd.nvalid) {
            pv[i] = hd.master[e + i];
            gv[i] = hd.grad[e + i];
          }
        p = make_float4(pv[0], pv[1], pv[2], pv[3]);
        g = make_uint2(gv[0] | (gv[1] << 16), gv[2] | (gv[3] << 16));
      }
      if (COAT_INDEX_OK(e + 4 <= hd.ngroups * kGroup)) {
        mq = *reinterpret_cast<const uint32_t*>(hd.mq + e);
        vq = *reinterpret_cast<const uint32_t*>(hd.vq + e);
      }
    }
    in.p[j] = p;
    in.g[j] = g;
    in.mq[j] = mq;
    in.vq[j] = vq;
  }
  in.ms = active ? hd.ms[lg] : 1.f;
  in.mk = active ? hd.mk[lg] : 1.f;
  in.vs = active ? hd.vs[lg] : 1.f;
  in.vk = active ? hd.vk[lg] : 1.f;
}

__device__ __forceinline__ float f4get(const float4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// 2^t in double for |t| < 1000, table-driven (P. T. P. Tang, "Table-driven
// implementation of the exponential function", ACM TOMS 15(2), 1989):
// t = (16n' + j)/16 + r with |r| <= 1/32, 2^t = 2^n' * 2^(j/16) * e^(r ln 2),
// the last factor by its Taylor series to the z^7 term (|z| <= ln2/32, so the
// truncation is below 2e-18 relative).
__device__ __forceinline__ double exp2_table(double t, const double* exp2_16) {
  const double s = t * 16.0;
  const double n = rint(s);
  const double z = (s - n) * 0.043321698784996581;  // (s - n)/16 * ln 2
  const int ni = static_cast<int>(n);
  double p = fma(z, 1.0 / 5040.0, 1.0 / 720.0);
  p = fma(p, z, 1.0 / 120.0);
  p = fma(p, z, 1.0 / 24.0);
  p = fma(p, z, 1.0 / 6.0);
  p = fma(p, z, 0.5);
  p = fma(p, z, 1.0);
  p = fma(p, z, 1.0);
  const double scale = __longlong_as_double(static_cast<long long>((ni >> 4) + 1023) << 52);
  return exp2_16[ni & 15] * p * scale;
}

// log2(x) in double for a finite normal x > 0, table-driven: x = 2^e f with f in
// [1, 2), F the centre of f's bin of width 1/128 (f - F is exact), r = (f - F)/F
// with |r| < 2^-8, log2 x = e + log2 F + ln(1 + r) log2(e), ln(1 + r) by its
// series to the r^6 term (truncation below 1e-17).
__device__ __forceinline__ double log2_table(double x, const LogEntry* lgt) {
  const long long b = __double_as_longlong(x);
  const int e = static_cast<int>(b >> 52) - 1023;
  const int j = static_cast<int>((b >> 45) & 127);
  const double f = __longlong_as_double((b & 0x000FFFFFFFFFFFFFLL) | 0x3FF0000000000000LL);
  const double F = 1.0 + (static_cast<double>(j) + 0.5) * (1.0 / 128.0);
  const LogEntry E = lgt[j];
  const double r = (f - F) * E.inv;
  double q = fma(r, -1.0 / 6.0, 0.2);
  q = fma(q, r, -0.25);
  q = fma(q, r, 1.0 / 3.0);
  q = fma(q, r, -0.5);
  q = fma(q, r, 1.0);
  return fma(q * r, 1.4426950408889634, static_cast<double>(e) + E.log2f);
}

// 1/x in double for x in [2^-120, 2^120]: the FP32 reciprocal refined by two
// Newton steps (within about an ulp of 1/x; no division).
__device__ __forceinline__ double rcp_d(double x) {
  double r = static_cast<double>(rcp_approx(__double2float_rn(x)));
  r = r * fma(-x, r, 2.0);
  return r * fma(-x, r, 2.0);
}

// The fast group parameters' minimum: the element of a group with the
// smallest nonzero |m'| usually comes from cancellation between beta1 m and
// (1 - beta1) g, so its FP32 value carries the FP32 dequantisation error
// amplified by |beta1 m| / |m'| (often 100x-1000x), and k depends on it
// through ln(max/min).  The kernel keeps the two smallest candidates (their
// positions packed into the low bits of the comparison keys) and recomputes
// them in double precision: dequantisation (zero for a zero code), then
// m' = beta1 m + (1 - beta1) gs g, gs the gradient-clipping coefficient.
__device__ __forceinline__ float recompute_m_double(const LaneIn& in, int idx, double invk,
                                                    const StepHyper& h, float gs,
                                                    const double* tabd_m,
                                                    const double* exp2_16) {
  const int j = idx >> 2, i = idx & 3;
  const uint32_t mw = j == 0 ? in.mq[0] : j == 1 ? in.mq[1] : j == 2 ? in.mq[2] : in.mq[3];
  const uint2 gw2 = j == 0 ? in.g[0] : j == 1 ? in.g[1] : j == 2 ? in.g[2] : in.g[3];
  const uint32_t c = (mw >> (8 * i)) & 0xFFu;
  const uint32_t gw = (i < 2) ? gw2.x : gw2.y;
  const float g = (i & 1) ? bf16hi(gw) : bf16lo(gw);
  double x = (c & 0x7Fu) ? exp2_table(tabd_m[c] * invk, exp2_16) * static_cast<double>(in.ms) : 0.0;
  if (c & 0x80u) x = -x;
  const double b1 = static_cast<double>(h.beta1);
  const double m1 = fma(b1, x, (1.0 - b1) * (static_cast<double>(gs) * static_cast<double>(g)));
  return __double2float_rn(fabs(m1));
}
__device__ __forceinline__ uint32_t min_key(float x, int idx) {
  return ((__float_as_uint(x) * 2u - 2u) & 0xFFFFFFE0u) | static_cast<uint32_t>(idx);
}

// Comparison keys ordered like |x|, with the element index i (0..15) in the
// low bits: for m' twice the FP32 bits (the sign drops out) with the low 5 bits
// replaced by i, for v' (never negative) the FP32 bits with the low 4 bits
// replaced by i.  A zero gives the key i, below every nonzero key.
__device__ __forceinline__ uint32_t key_m(float x, int i) {
  return ((__float_as_uint(x) << 1) & 0xFFFFFFE0u) | static_cast<uint32_t>(i);
}
__device__ __forceinline__ uint32_t key_v(float x, int i) {
  return (__float_as_uint(x) & 0xFFFFFFF0u) | static_cast<uint32_t>(i);
}

// The per-lane body: everything after the loads.  FULL: every element of the
// tile is valid (no bounds logic).  The gradient enters scaled by gs (the
// clipping coefficient, 1 without clipping), folded into the moment weights:
// omb1 = (1 - beta1) gs and omb2 = (1 - beta2) gs^2.
template <int FM, int FV, bool EXACT, bool FULL>
__device__ __forceinline__ void process(const LaneIn& in, const TileHeader& t, const int (&off)[4],
                                        int lg, bool active, int slot, int l, const StepHyper& h,
                                        float omb1, float omb2, float gs, const Smem& S,
                                        uint4* scratch_lane, const uint8_t* scratch_warp) {
  // this lane's codes and gradients, for the lanes that recompute the group's
  // extreme elements (the previous tile's reads ended at the last shuffle)
  if constexpr (EXACT) {
    __syncwarp();
    scratch_lane[0] = make_uint4(in.mq[0], in.mq[1], in.mq[2], in.mq[3]);
    scratch_lane[1] = make_uint4(in.vq[0], in.vq[1], in.vq[2], in.vq[3]);
    scratch_lane[2] = make_uint4(in.g[0].x, in.g[0].y, in.g[1].x, in.g[1].y);
    scratch_lane[3] = make_uint4(in.g[2].x, in.g[2].y, in.g[3].x, in.g[3].y);
  }

  // dequantisation constants of this group (stored k and root scale), as
  // (m, v) pairs for the packed FP32 operations
  const float2 invk = make_float2(rcp_approx(in.mk), rcp_approx(in.vk));
  const float2 sb = mul2(make_float2(in.ms, in.vs), make_float2(h.beta1, h.beta2));
  const float2 dsq2 = make_float2(h.dsq, h.dsq), deps2 = make_float2(h.deps, h.deps);
  const float2 lrwd2 = make_float2(t.lrwd, t.lrwd), omb2x2 = make_float2(omb2, omb2);

  float m1[16], v1[16];
  // EXACT: keys (key_m, key_v) of the group's extremes: max |m'|, the two
  // smallest nonzero |m'|, max v', smallest nonzero v' (for the minima the keys
  // are shifted down by one index block, so that zeros wrap to the top).
  // Otherwise: max |m'|, max v' and min nonzero v' in FP32, and the keys
  // (min_key) of the two smallest nonzero |m'|.
  uint32_t maxmk = 0u, maxvk = 0u, minvk = 0xFFFFFFFFu;
  float maxm = 0.f, maxv = 0.f;
  uint32_t minv = 0xFFFFFFFFu;
  uint32_t minm1 = 0xFFFFFFFFu, minm2 = 0xFFFFFFFFu;

#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = off[j];
    float pn[4];
    // element pairs (2u, 2u + 1): the two bf16 gradients of one word
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t gw = u ? in.g[j].y : in.g[j].x;
      const float2 g2 = make_float2(bf16lo(gw), bf16hi(gw));
      const float2 og = mul2(g2, omb2x2);   // (1 - beta2) g, both elements
      float2 mv[2];                         // (m', v') of each element
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int i = 2 * u + w;
        const float g = w ? g2.y : g2.x;
        const uint32_t cm = __byte_perm(in.mq[j], 0u, 0x4440u + i);
        const uint32_t cv = __byte_perm(in.vq[j], 0u, 0x4440u + i);
        // beta1 * m and beta2 * v, dequantised: s_r * beta * 2^(log2|q| / k)
        const float2 tl = mul2(make_float2(S.tab_m[cm], S.tab_v[cv]), invk);
        float2 b = mul2(make_float2(ex2_approx(tl.x), ex2_approx(tl.y)), sb);
        b.x = __uint_as_float(__float_as_uint(b.x) ^ ((in.mq[j] << (24 - 8 * i)) & 0x80000000u));
        // m' = beta1 m + (1 - beta1) g, v' = beta2 v + (1 - beta2) g^2
        mv[w] = fma2(make_float2(omb1, w ? og.y : og.x), make_float2(g, g), b);
      }
      // p - (p lr wd + m' / (sqrt(v') dsq + deps)) for both elements
      const float2 den = fma2(make_float2(sqrt_approx(mv[0].y), sqrt_approx(mv[1].y)), dsq2, deps2);
      const float2 upd = mul2(make_float2(mv[0].x, mv[1].x),
                              make_float2(rcp_approx(den.x), rcp_approx(den.y)));
      const float2 p = make_float2(f4get(in.p[j], 2 * u), f4get(in.p[j], 2 * u + 1));
      const float2 pnew = sub2(p, fma2(p, lrwd2, upd));
      pn[2 * u] = pnew.x;
      pn[2 * u + 1] = pnew.y;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int i = 2 * u + w;
        float mn = mv[w].x, vn = mv[w].y;
        if (!FULL) {
          const bool valid = active && (e + i < t.nvalid);
          mn = valid ? mn : 0.f;
          vn = valid ? vn : 0.f;
        }
        m1[4 * j + i] = mn;
        v1[4 * j + i] = vn;
        if constexpr (!EXACT) {
          maxm = fmaxf(maxm, fabsf(mn));
          maxv = fmaxf(maxv, vn);
          minv = min(minv, __float_as_uint(vn) - 1u);
        }
      }
    }
    if constexpr (EXACT) {
      // keys of the elements, in pairs (0,1), (2,3); the two smallest m keys
      // merge the sorted pair into the running pair
  #pragma unroll
      for (int i = 0; i < 4; i += 2) {
        const uint32_t ka = key_m(m1[4 * j + i], 4 * j + i);
        const uint32_t kb = key_m(m1[4 * j + i + 1], 4 * j + i + 1);
        maxmk = max(maxmk, max(ka, kb));
        const uint32_t a = ka - 32u, b = kb - 32u;
        const uint32_t lo = min(a, b), hi = max(a, b);
        minm2 = min(max(minm1, lo), min(minm2, hi));
        minm1 = min(minm1, lo);
        const uint32_t va = key_v(v1[4 * j + i], 4 * j + i);
        const uint32_t vb = key_v(v1[4 * j + i + 1], 4 * j + i + 1);
        maxvk = max(maxvk, max(va, vb));
        minvk = min(minvk, min(va - 16u, vb - 16u));
      }
    } else {
      // two smallest m keys: merge the sorted pairs of elements (0,1), (2,3)
#pragma unroll
      for (int i = 0; i < 4; i += 2) {
        const uint32_t ka = min_key(m1[4 * j + i], 4 * j + i);
        const uint32_t kb = min_key(m1[4 * j + i + 1], 4 * j + i + 1);
        const uint32_t lo = min(ka, kb), hi = max(ka, kb);
        minm2 = min(max(minm1, lo), min(minm2, hi));
        minm1 = min(minm1, lo);
      }
    }
    if (FULL ? COAT_INDEX_OK(e + 4 <= t.nvalid) : (active && e + 4 <= t.nvalid)) {
      __stcs(reinterpret_cast<float4*>(t.master + e), make_float4(pn[0], pn[1], pn[2], pn[3]));
      if (t.wout)
        __stcs(reinterpret_cast<uint2*>(t.wout + e),
               make_uint2(pack_bf16x2(pn[0], pn[1]), pack_bf16x2(pn[2], pn[3])));
    } else if (active) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (e + i < t.nvalid) {
          t.master[e + i] = pn[i];
          if (t.wout) t.wout[e + i] = static_cast<uint16_t>(pack_bf16x2(pn[i], 0.f));
        }
    }
  }

  const bool vrole = l >= 4;   // lanes 4-7 of a group work on v, lanes 0-3 on m
  float kx, srx, invMx;
  if constexpr (EXACT) {
    // Group extremes over the 8 lanes.  The keys take the lane in bits 5-7 (m)
    // or 4-6 (v), so that each carries its element's position (ordering to
    // 2^-16 relative); merging two sorted pairs keeps the two smallest.
    const uint32_t lm = static_cast<uint32_t>(l) << 5, lv = static_cast<uint32_t>(l) << 4;
    maxmk = (maxmk & ~0xE0u) | lm;
    minm1 = (minm1 & ~0xE0u) | lm;
    minm2 = (minm2 & ~0xE0u) | lm;
    maxvk = (maxvk & ~0x70u) | lv;
    minvk = (minvk & ~0x70u) | lv;
  #pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      maxmk = max(maxmk, __shfl_xor_sync(0xFFFFFFFFu, maxmk, off));
      maxvk = max(maxvk, __shfl_xor_sync(0xFFFFFFFFu, maxvk, off));
      minvk = min(minvk, __shfl_xor_sync(0xFFFFFFFFu, minvk, off));
      const uint32_t o1 = __shfl_xor_sync(0xFFFFFFFFu, minm1, off);
      const uint32_t o2 = __shfl_xor_sync(0xFFFFFFFFu, minm2, off);
      minm2 = min(max(minm1, o1), min(minm2, o2));
      minm1 = min(minm1, o1);
    }

    // The group's k and root scale are computed in double from the extremes
    // recomputed in double, as the definition has them, so that the FP32 k and
    // s_r stored are the correctly rounded values of the exact ones (FP32 values
    // of the extremes carry the dequantisation error, and the smallest |m'|
    // usually comes from cancellation between beta1 m and (1 - beta1) g, which
    // amplifies it by |beta1 m| / |m'|).  Each extreme is recomputed by one lane
    // of the group, from the owner's codes and gradient in the scratch copy:
    // lane 0 max |m'|, lanes 1 and 2 the two smallest |m'| (FP32 may misorder a
    // near-tie), lane 4 max v', lane 5 the smallest v'; lanes 3, 6, 7 repeat a
    // maximum.
    const int role = l & 3;
    const bool is_min = role == 1 || (!vrole && role == 2);
    const uint32_t key = vrole ? (role == 1 ? minvk : maxvk)
                               : (role == 1 ? minm1 : role == 2 ? minm2 : maxmk);
    const bool found = is_min ? key < 0xFFFFFF00u : key >= 0x100u;
    const int owner = static_cast<int>(vrole ? (key >> 4) & 7u : (key >> 5) & 7u);
    const int idx = static_cast<int>(key & 15u);
    const uint8_t* src = scratch_warp + (slot * 8 + owner) * 64;
    const uint32_t code = src[(vrole ? 16 : 0) + idx];
    const uint32_t gbits = *reinterpret_cast<const uint16_t*>(src + 32 + 2 * idx);
    // val: |m'| or v' of the extreme in double; lval: its log2 (-inf for a zero
    // maximum, +inf for a missing minimum)
    double val, lval;
    {
      const double invkd = rcp_d(static_cast<double>(vrole ? in.vk : in.mk));
      const double srd = static_cast<double>(vrole ? in.vs : in.ms);
      const double beta = static_cast<double>(vrole ? h.beta2 : h.beta1);
      const double* tabd = vrole ? S.tabd_v : S.tabd_m;
      // x = sign(q) s_r |q|^(1/k) (zero for a zero code)
      double x = (code & 0x7Fu) ? exp2_table(tabd[code] * invkd, S.exp2_16) * srd : 0.0;
      if (!vrole && (code & 0x80u)) x = -x;
      // m' = beta1 m + (1 - beta1) g, v' = beta2 v + ((1 - beta2) g) g, g the
      // clipped gradient, each product and the sum rounded separately
      const double gi = static_cast<double>(gs) * static_cast<double>(__uint_as_float(gbits << 16));
      double term = __dmul_rn(1.0 - beta, gi);
      if (vrole) term = __dmul_rn(term, gi);
      const double r = fabs(__dadd_rn(__dmul_rn(beta, x), term));
      const double inf = __longlong_as_double(0x7FF0000000000000LL);
      val = found ? r : 0.0;
      lval = found && r > 0.0 ? log2_table(r, S.lgt) : (is_min ? inf : -inf);
    }
    const int base = slot << 3;
    const double M = __shfl_sync(0xFFFFFFFFu, val, base + (vrole ? 4 : 0));
    const double lM = __shfl_sync(0xFFFFFFFFu, lval, base + (vrole ? 4 : 0));
    const double lmu = fmin(__shfl_sync(0xFFFFFFFFu, lval, base + (vrole ? 5 : 1)),
                            __shfl_sync(0xFFFFFFFFu, lval, base + (vrole ? 5 : 2)));
    // lanes 0-3 derive the m parameters, lanes 4-7 the v ones:
    // k = clamp(log2(R) / log2(M / mu), 1, 16) (16 when M == mu; 1, s_r = 1
    // for an all-zero group), then s_r = M FMT_MAX^(-1/k) = 2^(log2 M -
    // log2(FMT_MAX) / k) with the FP32 k.
    const bool nonzero = M > 0.0;
    const bool spread = nonzero && lmu < lM;
    double kd = spread ? fmin(fmax((vrole ? F8<FV>::LOG2_TARGET_D : F8<FM>::LOG2_TARGET_D) *
                                       rcp_d(lM - lmu), 1.0), 16.0)
                       : 16.0;
    if (!nonzero) kd = 1.0;
    kx = __double2float_rn(kd);
    const double ex = lM - (vrole ? F8<FV>::LOG2MAX_D : F8<FM>::LOG2MAX_D) *
                               rcp_d(static_cast<double>(kx));
    srx = nonzero ? __double2float_rn(exp2_table(ex, S.exp2_16)) : 1.0f;
    invMx = nonzero ? rcp_approx(__double2float_rn(M)) : 0.0f;
  } else {
    minm1 = (minm1 & ~0xE0u) | (static_cast<uint32_t>(l) << 5);
    minm2 = (minm2 & ~0xE0u) | (static_cast<uint32_t>(l) << 5);
  #pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      maxm = fmaxf(maxm, __shfl_xor_sync(0xFFFFFFFFu, maxm, off));
      maxv = fmaxf(maxv, __shfl_xor_sync(0xFFFFFFFFu, maxv, off));
      minv = min(minv, __shfl_xor_sync(0xFFFFFFFFu, minv, off));
      const uint32_t o1 = __shfl_xor_sync(0xFFFFFFFFu, minm1, off);
      const uint32_t o2 = __shfl_xor_sync(0xFFFFFFFFu, minm2, off);
      minm2 = min(max(minm1, o1), min(minm2, o2));
      minm1 = min(minm1, o1);
    }
    const double kd0 = static_cast<double>(in.mk), r0 = static_cast<double>(rcp_approx(in.mk));
    const double invk_md = r0 * fma(-kd0, r0, 2.0);
    // min |m'| exact as FP32: the lane owning the smallest candidate recomputes
    // it; the runner-up is recomputed too when its FP32 key is within about
    // 2^-7 relative of the smallest (a near-tie that the FP32 values may
    // misorder).  Every lane recomputes the element at the smallest key's index
    // (only the owner's registers hold it; the others' values are discarded),
    // so the common case runs converged.
    const bool any_m = minm1 < 0xFFFFFF00u;
    const bool tie = minm2 < 0xFFFFFF00u && (minm2 >> 8) - (minm1 >> 8) < (1u << 9);
    float mum = recompute_m_double(in, static_cast<int>(minm1 & 15u), invk_md, h, gs, S.tabd_m,
                                   S.exp2_16);
    mum = __shfl_sync(0xFFFFFFFFu, mum, (slot << 3) | static_cast<int>((minm1 >> 5) & 7u));
    if (__any_sync(0xFFFFFFFFu, tie)) {
      float m2 = __int_as_float(0x7F800000);
      if (tie && static_cast<int>((minm2 >> 5) & 7u) == l)
        m2 = recompute_m_double(in, static_cast<int>(minm2 & 15u), invk_md, h, gs, S.tabd_m,
                                S.exp2_16);
  #pragma unroll
      for (int off = 1; off < 8; off <<= 1) m2 = fminf(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, off));
      mum = fminf(mum, m2);
    }
    if (!any_m) mum = 0.f;
    const float muv = __uint_as_float(minv + 1u);
    // lanes 0-3 of the group derive the m parameters, lanes 4-7 the v ones
    group_params_rt(vrole ? maxv : maxm, vrole ? muv : mum, true,
                    vrole ? F8<FV>::LOG2MAX_HI : F8<FM>::LOG2MAX_HI,
                    vrole ? F8<FV>::LOG2MAX_LO : F8<FM>::LOG2MAX_LO,
                    vrole ? F8<FV>::LOG2_TARGET : F8<FM>::LOG2_TARGET, kx, srx, invMx);
  }
  const int lane_m = slot << 3, lane_v = lane_m + 4;
  const float km = __shfl_sync(0xFFFFFFFFu, kx, lane_m);
  const float invMm = __shfl_sync(0xFFFFFFFFu, invMx, lane_m);
  const float kv = __shfl_sync(0xFFFFFFFFu, kx, lane_v);
  const float invMv = __shfl_sync(0xFFFFFFFFu, invMx, lane_v);
  const float2 invM2 = make_float2(invMm, invMv), k2 = make_float2(km, kv);
  const float2 log2max2 = make_float2(F8<FM>::LOG2MAX_HI, F8<FV>::LOG2MAX_HI);

  // expand + encode, store codes (whole group, padding included) and metadata
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = off[j];
    uint32_t cmw[4], cvw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // y = FMT_MAX (|x| / M)^k = 2^(k log2(|x| / M) + log2 FMT_MAX) for m' and v'
      const float2 a = mul2(make_float2(m1[4 * j + i], v1[4 * j + i]), invM2);
      const float2 ty = fma2(k2, make_float2(lg2_approx(fabsf(a.x)), lg2_approx(fabsf(a.y))), log2max2);
      const uint2 c = enc_mag_bounded2<FM, FV>(ex2_approx(ty.x), ex2_approx(ty.y));
      cmw[i] = c.x;
      cvw[i] = c.y;
    }
    if ((FULL || active) && COAT_INDEX_OK(e + 4 <= t.ngroups * kGroup)) {
      __stcs(reinterpret_cast<unsigned int*>(t.mq + e),
             merge_signs4(pack4(cmw[0], cmw[1], cmw[2], cmw[3]), m1[4 * j], m1[4 * j + 1],
                          m1[4 * j + 2], m1[4 * j + 3]));
      __stcs(reinterpret_cast<unsigned int*>(t.vq + e), pack4(cvw[0], cvw[1], cvw[2], cvw[3]));
    }
  }
  if ((FULL || active) && (l & 3) == 0 && COAT_INDEX_OK(lg < t.ngroups)) {
    (vrole ? t.vs : t.ms)[lg] = srx;
    (vrole ? t.vk : t.mk)[lg] = kx;
  }
}

// ---------------------------------------------------------------------------
// The producer thread stages the CTA's tiles.
// ---------------------------------------------------------------------------
template <class Map>
__device__ __forceinline__ void feed_start(const Map& map, Feed& f, int64_t tile) {
  const int32_t ti = map.find(tile);
  f.ti = ti;
  f.d = map.get(ti);
  f.next_begin = map.begin_of(ti + 1);
}

// Make f describe the tensor of `tile` (tiles only move forward).
template <class Map>
__device__ __forceinline__ void feed_locate(const Map& map, Feed& f, int64_t tile) {
  if (tile >= f.next_begin) {
    const int32_t ti = map.advance(f.ti, tile);
    f.ti = ti;
    f.d = map.get(ti);
    f.next_begin = map.begin_of(ti + 1);
  }
}

// Stage `tile` (located in f) into `st` (header into `hd`), completing on
// `bar`: a fully valid tile is copied (kTxBytes of transaction), any other tile
// only arrives and is read from global memory by the lanes.
__device__ __forceinline__ void feed_issue(const Feed& f, int64_t tile, uint8_t* st,
                                           TileHeader& hd, uint64_t* bar, float lrwd,
                                           uint64_t policy) {
  const TensorArgs& ct = f.d;
  const int64_t g0 = (tile - ct.tile_begin) * kTileGroups;
  const int64_t groups = (ct.n + kGroup - 1) / kGroup;
  const int64_t ng = (groups - g0) < kTileGroups ? (groups - g0) : int64_t(kTileGroups);
  const int64_t e0 = g0 * kGroup;
  const bool full = (e0 + kTileElems <= ct.n);
  if (!COAT_INDEX_OK(tile >= ct.tile_begin && tile < ct.tile_begin + ct.tiles && e0 < ct.n)) {
    hd.nvalid = 0;   // a tile outside its tensor: the lanes find no group and touch nothing
    hd.ngroups = 0;
    mbar_arrive(bar);
    return;
  }
  hd.master = ct.master + e0;
  hd.wout = ct.wout ? ct.wout + e0 : nullptr;
  hd.mq = ct.mq + e0;
  hd.vq = ct.vq + e0;
  hd.ms = ct.ms + g0;
  hd.mk = ct.mk + g0;
  hd.vs = ct.vs + g0;
  hd.vk = ct.vk + g0;
  hd.grad = ct.grad + e0;
  hd.nvalid = full ? kTileElems : static_cast<int32_t>(ct.n - e0);
  hd.ngroups = static_cast<int32_t>(ng);
  hd.lrwd = lrwd * ct.wd_scale;
  if (full) {
    mbar_arrive_expect_tx(bar, kTxBytes);
    bulk_g2s_hint(st + kOffMaster, ct.master + e0, kTileElems * 4, bar, policy);
    bulk_g2s_hint(st + kOffGrad, ct.grad + e0, kTileElems * 2, bar, policy);
    bulk_g2s_hint(st + kOffMq, ct.mq + e0, kTileElems, bar, policy);
    bulk_g2s_hint(st + kOffVq, ct.vq + e0, kTileElems, bar, policy);
    bulk_g2s_hint(st + kOffMs, ct.ms + g0, kTileGroups * 4, bar, policy);
    bulk_g2s_hint(st + kOffMk, ct.mk + g0, kTileGroups * 4, bar, policy);
    bulk_g2s_hint(st + kOffVs, ct.vs + g0, kTileGroups * 4, bar, policy);
    bulk_g2s_hint(st + kOffVk, ct.vk + g0, kTileGroups * 4, bar, policy);
  } else {
    mbar_arrive(bar);
  }
}

template <int FM, int FV, bool EXACT, class Map>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    adamw_fp8_kernel(const Map map, const StepHyper h, const ClipRecord* clip, unsigned* err) {
  // Gradient clipping: a record with found_inf set skips the step (nothing is
  // read or written); otherwise the gradient is scaled by its coefficient.
  float gs = 1.f;
  if (clip != nullptr) {
    if (clip->found_inf) return;
    gs = clip->coef;
  }
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  uint8_t* stages = smem_raw + kSmemHead;

  fill_log2_table<FM>(S.tab_m);
  fill_log2_table<FV>(S.tab_v);
  for (int c = threadIdx.x; c < 256; c += blockDim.x) {
    S.tabd_m[c] = log2(static_cast<double>(fabsf(dec_value<FM>(c))));
    if (EXACT) S.tabd_v[c] = log2(static_cast<double>(fabsf(dec_value<FV>(c))));
  }
  if (EXACT) {
    for (int j = threadIdx.x; j < 128; j += blockDim.x) {
      const double F = 1.0 + (static_cast<double>(j) + 0.5) * (1.0 / 128.0);
      S.lgt[j].log2f = log2(F);
      S.lgt[j].inv = 1.0 / F;
    }
  }
  if (threadIdx.x < 16) S.exp2_16[threadIdx.x] = exp2(static_cast<double>(threadIdx.x) / 16.0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full_bar[s], 1);
      mbar_init(&S.empty_bar[s], kConsumerWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ... (at any moment the
  // CTAs stream neighbouring regions of every array)
  const int64_t ntiles = map.tiles();
  const int64_t t0 = blockIdx.x, dt = gridDim.x;

  if (warp == kConsumerWarps) {
    // ---------------- producer ----------------
    if (lane != 0 || t0 >= ntiles) return;
    Feed f;
    feed_start(map, f, t0);
    const uint64_t policy = l2_evict_first_policy();
    int64_t it = 0;
    for (int64_t tile = t0; tile < ntiles; tile += dt, ++it) {
      const int s = static_cast<int>(it % kStages);
      const uint32_t use = static_cast<uint32_t>(it / kStages);
      feed_locate(map, f, tile);   // before the wait: its loads overlap it
      if (use > 0 && !mbar_wait(&S.empty_bar[s], (use - 1) & 1u, kWaitBudgetCycles)) {
        atomicOr(err, kErrTimeoutProducer);
        // Drain copies still in flight into stages the consumers never freed.
        for (int d = 0; d < kStages; ++d) {
          const int64_t itd = it - 1 - d;
          if (itd < 0) break;
          const int sd = static_cast<int>(itd % kStages);
          if (!mbar_wait(&S.full_bar[sd], static_cast<uint32_t>(itd / kStages) & 1u,
                         kWaitBudgetCycles))
            atomicOr(err, kErrCopyDrain);
        }
        return;
      }
      feed_issue(f, tile, stages + size_t(s) * kStageBytes, S.hdr[s], &S.full_bar[s], h.lrwd,
                 policy);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int slot = lane >> 3, l = lane & 7;
  const int lg = warp * kGroupsPerWarp + slot;  // group within the tile
  uint4* scratch_lane = S.scratch + (warp * 32 + lane) * 4;
  const uint8_t* scratch_warp = reinterpret_cast<const uint8_t*>(S.scratch + warp * 32 * 4);
  const float omb1 = h.omb1 * gs, omb2 = h.omb2 * gs * gs;
  // the lane's elements: 4 chunks of 4, chunk j at 32 chunk_of(j, slot) + 4 l
  // within its group
  int off[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) off[j] = lg * kGroup + 32 * chunk_of(j, slot) + 4 * l;
  int64_t it = 0;
  for (int64_t tile = t0; tile < ntiles; tile += dt, ++it) {
    const int s = static_cast<int>(it % kStages);
    const uint32_t use = static_cast<uint32_t>(it / kStages);
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&S.full_bar[s], use & 1u, kWaitBudgetCycles))) {
      if (lane == 0) atomicOr(err, kErrTimeoutConsumer);
      return;
    }
    // the header is copied to registers before the stage is released
    const TileHeader t = S.hdr[s];
    const bool full = t.nvalid == kTileElems;
    const bool active = lg < t.ngroups;
    LaneIn in;
    if (full)
      load_from_stage(stages + size_t(s) * kStageBytes, off, lg, in);
    else
      load_direct(t, off, lg, active, in);
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty_bar[s]);
    if (full)
      process<FM, FV, EXACT, true>(in, t, off, lg, true, slot, l, h, omb1, omb2, gs, S, scratch_lane,
                            scratch_warp);
    else
      process<FM, FV, EXACT, false>(in, t, off, lg, active, slot, l, h, omb1, omb2, gs, S, scratch_lane,
                             scratch_warp);
  }
}

template <int FM, int FV, bool EXACT, class Map>
cudaError_t launch_step(const Map& map, int64_t ntiles, const StepHyper& h,
                        const ClipRecord* clip, unsigned* err, cudaStream_t stream) {
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  auto kern = adamw_fp8_kernel<FM, FV, EXACT, Map>;
  if (dev < 64 && !configured[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int64_t want = int64_t(sm_count(dev)) * kCtasPerSm;
  const int64_t grid = ntiles < want ? ntiles : want;
  if (grid <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(map, h, clip, err);
  return cudaGetLastError();
}

template <class Map>
cudaError_t dispatch(int fm, int fv, const Map& map, int64_t ntiles, const StepHyper& h,
                     const ClipRecord* clip, unsigned* err, cudaStream_t stream) {
  switch (fm * 3 + fv) {
#define COAT_STEP_CASE(A, B)                                                  \
  case A * 3 + B:                                                             \
    return h.exact ? launch_step<A, B, true>(map, ntiles, h, clip, err, stream) \
                   : launch_step<A, B, false>(map, ntiles, h, clip, err, stream);
    COAT_STEP_CASE(kE4M3, kE4M3)
    COAT_STEP_CASE(kE4M3, kE5M2)
    COAT_STEP_CASE(kE4M3, kE5M2Full)
    COAT_STEP_CASE(kE5M2, kE4M3)
    COAT_STEP_CASE(kE5M2, kE5M2)
    COAT_STEP_CASE(kE5M2, kE5M2Full)
    COAT_STEP_CASE(kE5M2Full, kE4M3)
    COAT_STEP_CASE(kE5M2Full, kE5M2)
    COAT_STEP_CASE(kE5M2Full, kE5M2Full)
#undef COAT_STEP_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int64_t step_tile_groups() { return kTileGroups; }

COAT_INDEX_FAULT_READER(index_faults_step)

cudaError_t launch_adamw_single(const TensorArgs& t, int fm, int fv, const StepHyper& h,
                                unsigned* err, cudaStream_t stream) {
  SingleTensor map{t};
  return dispatch(fm, fv, map, t.tiles, h, nullptr, err, stream);
}

cudaError_t launch_adamw_multi(const TensorArgs* d_descs, int num, int64_t total_tiles, int fm,
                               int fv, const StepHyper& h, const ClipRecord* clip, unsigned* err,
                               cudaStream_t stream) {
  MultiTensor map{d_descs, num, total_tiles};
  return dispatch(fm, fv, map, total_tiles, h, clip, err, stream);
}

// ---------------------------------------------------------------------------
// Gradient-norm pass before a clipped step (global-norm clipping as
// torch.nn.utils.clip_grad_norm_ defines it, with the non-finite check of a
// loss-scaled training loop): sum of g^2 over every gradient of the plan.
//
// HBM-bound (2 bytes per element read, nothing else): kNormCtasPerSm CTAs per
// SM, each over a contiguous range of the step's tiles, so that every CTA
// streams whole runs of each tensor's gradient with 16-byte loads.  A thread
// squares the 8 bf16 values of a load in FP32 -- each square is exact there,
// the 8-term sum rounds a few times at 2^-24 relative -- and adds the sum to a
// double accumulator; if that FP32 sum overflowed (an element of magnitude
// 2^64 or more) or met an Inf/NaN, the 8 values are redone in double, where no
// sum of bf16 squares can overflow, so the total is non-finite exactly when an
// element is.  CTA sums go to per-CTA slots; the last CTA to finish (ticket
// counter) adds the slots in index order, so the result depends only on the
// grid, which is fixed per device.
// ---------------------------------------------------------------------------
namespace {

constexpr int kNormThreads = 256;
constexpr int kNormCtasPerSm = 4;
constexpr int kNormUnroll = 4;

__device__ __forceinline__ double sumsq8(const uint4 w) {
  const uint32_t a[4] = {w.x, w.y, w.z, w.w};
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float lo = __uint_as_float(a[k] << 16), hi = __uint_as_float(a[k] & 0xFFFF0000u);
    s0 = __fmaf_rn(lo, lo, s0);
    s1 = __fmaf_rn(hi, hi, s1);
  }
  const float s = s0 + s1;
  if (s <= 3.40282347e38f) return static_cast<double>(s);
  double d = 0.0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const double lo = __uint_as_float(a[k] << 16), hi = __uint_as_float(a[k] & 0xFFFF0000u);
    d = fma(lo, lo, d);
    d = fma(hi, hi, d);
  }
  return d;
}

// Sum of g^2 over cnt elements from g (16-byte aligned) by the CTA's threads.
__device__ __forceinline__ double sumsq_run(const uint16_t* g, int64_t cnt) {
  const uint4* v = reinterpret_cast<const uint4*>(g);
  const int64_t nv = cnt >> 3;
  constexpr int T = kNormThreads;
  double acc = 0.0;
  int64_t i = threadIdx.x;
  for (; i + (kNormUnroll - 1) * T < nv; i += kNormUnroll * T) {
    uint4 w[kNormUnroll];
#pragma unroll
    for (int u = 0; u < kNormUnroll; ++u) w[u] = __ldcs(v + i + u * T);
#pragma unroll
    for (int u = 0; u < kNormUnroll; ++u) acc += sumsq8(w[u]);
  }
  for (; i < nv; i += T) acc += sumsq8(__ldcs(v + i));
  const int64_t rem = cnt & 7;
  if (threadIdx.x < rem) {
    const double x = __uint_as_float(static_cast<uint32_t>(g[nv * 8 + threadIdx.x]) << 16);
    acc = fma(x, x, acc);
  }
  return acc;
}

// Sum over the CTA in a fixed order; the result is valid in thread 0.
__device__ __forceinline__ double cta_sum(double x, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  const int warp = threadIdx.x >> 5;
  __syncthreads();  // red may still be read from an earlier call
  if ((threadIdx.x & 31) == 0) red[warp] = x;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < kNormThreads / 32; ++w) t += red[w];
  return t;
}

__global__ void __launch_bounds__(kNormThreads, kNormCtasPerSm)
    grad_sumsq_kernel(const MultiTensor map, double* partials, unsigned* ticket, float max_norm,
                      ClipRecord* out) {
  __shared__ double red[kNormThreads / 32];
  __shared__ bool last;
  const int64_t ntiles = map.tiles();
  const int64_t t0 = int64_t(blockIdx.x) * ntiles / gridDim.x;
  const int64_t t1 = int64_t(blockIdx.x + 1) * ntiles / gridDim.x;
  double acc = 0.0;
  if (t0 < t1) {
    // walk the tensors that own tiles [t0, t1): each contributes one run of
    // its gradient (tile boundaries are 7680 elements apart, so every run
    // starts 16-byte aligned)
    int32_t ti = map.find(t0);
    int64_t tile = t0;
    while (tile < t1 && ti < map.num) {
      const TensorArgs& d = map.descs[ti];
      const int64_t tb = d.tile_begin, te = tb + d.tiles;
      if (tile < te) {
        const int64_t tend = te < t1 ? te : t1;
        const int64_t ea = (tile - tb) * kTileElems;
        const int64_t eb_tiles = (tend - tb) * kTileElems;
        const int64_t eb = eb_tiles < d.n ? eb_tiles : d.n;
        if (COAT_INDEX_OK(ea >= 0 && ea <= eb && eb <= d.n)) acc += sumsq_run(d.grad + ea, eb - ea);
        tile = tend;
      }
      ++ti;
    }
  }
  const double cta = cta_sum(acc, red);
  if (threadIdx.x == 0) {
    partials[blockIdx.x] = cta;
    __threadfence();
    last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  // the last CTA: every other CTA's slot is written and visible
  __threadfence();
  double a = 0.0;
  for (int i = threadIdx.x; i < static_cast<int>(gridDim.x); i += kNormThreads)
    a += __ldcg(partials + i);
  const double total = cta_sum(a, red);
  if (threadIdx.x == 0) {
    const double c = static_cast<double>(max_norm) / (sqrt(total) + 1e-6);
    ClipRecord r;
    r.sumsq = total;
    r.norm = static_cast<float>(sqrt(total));
    r.coef = static_cast<float>(c < 1.0 ? c : 1.0);
    r.found_inf = isfinite(total) ? 0 : 1;
    r.reserved = 0;
    *out = r;
    *ticket = 0u;  // ready for the next launch on this plan
  }
}

}  // namespace

int grad_sumsq_slots(int dev) { return sm_count(dev) * kNormCtasPerSm; }

cudaError_t launch_grad_sumsq(const TensorArgs* d_descs, int num, int64_t total_tiles,
                              double* partials, unsigned* ticket, float max_norm, ClipRecord* out,
                              cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int64_t slots = grad_sumsq_slots(dev);
  int64_t grid = total_tiles < slots ? total_tiles : slots;
  if (grid < 1) grid = 1;  // an empty plan still writes its record
  MultiTensor map{d_descs, num, total_tiles};
  grad_sumsq_kernel<<<static_cast<unsigned>(grid), kNormThreads, 0, stream>>>(map, partials, ticket,
                                                                             max_norm, out);
  return cudaGetLastError();
}

namespace {
// One warp waits, with the given bound, on an mbarrier that nothing arrives on.
__global__ void wait_timeout_selftest_kernel(long long budget, unsigned* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (!__all_sync(0xFFFFFFFFu, mbar_wait(&bar, 0u, budget)) && threadIdx.x == 0)
    atomicOr(err, kErrTimeoutConsumer);
}
}  // namespace

cudaError_t launch_wait_timeout_selftest(long long budget_cycles, unsigned* err,
                                         cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(budget_cycles, err);
  return cudaGetLastError();
}

}  // namespace coat
