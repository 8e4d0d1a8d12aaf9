// Router: FP32 gate GEMM on CUDA cores, then softmax and bias-adjusted top-k
// per token (dots.llm1 Technical Report, Method: the gate projection runs in
// FP32 for stable routing; selection uses the auxiliary-loss-free bias).
//
// router_gemm_kernel  split-K fp32 GEMM: partial[s, t, e] = sum over the s-th
//                     k-chunk of x[t, i] * w_gate[e, i]  (x bf16 -> fp32 exactly)
// router_topk_kernel  one warp per token: z = sum_s partial[s] (s ascending),
//                     p = softmax(z), key = p + bias, k rounds of warp arg-max
//                     (equal keys: lower expert id), w = p_sel / sum p_sel
#include <cuda_bf16.h>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BT = kRouterBT;  // tokens per tile
constexpr int BE = 128;        // experts per tile (all of them; E <= 128)
constexpr int BK = kRouterBK;  // k-chunk in shared memory
constexpr int kFold = 4;      // staged chunks summed in fp32 before each fp64 add
constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// 256 threads as a 16 x 16 grid; thread (ty, tx) owns tokens
// {ty*4 .. ty*4+3, 64+ty*4 .. 64+ty*4+3} and experts {tx*4 .., 64+tx*4 ..}.
// Accumulation is two-level: the products are fp32 FMAs and the kFold*BK
// products of kFold staged chunks are summed from zero in fp32; the running
// sum across those groups is carried in fp64 (one conversion and add per
// kFold*BK FMAs, so the slow float->double conversions stay a small share of
// the issue slots).  A single fp32 running sum over k = 5120 terms loses
// ~1e-5 relative in the softmax probabilities when one term is large (e.g. a
// logit offset); with 64-term fp32 groups the error stays near 2e-6.
__global__ void __launch_bounds__(kThreads, 1)
router_gemm_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wg,
                   float* __restrict__ part, int T, int d, int E, int kchunk) {
  __shared__ __align__(16) float xs[2][BK][BT];
  __shared__ __align__(16) float ws[2][BK][BE];

  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * BT;
  const int split = blockIdx.y;
  const int k_begin = split * kchunk;
  const int k_end = min(d, k_begin + kchunk);
  const int nk = (k_end - k_begin) / BK;

  // loader roles: one 16-byte bf16 vector of x and two float4 of w_gate per chunk
  const int lrow = tid & 127;
  const int lq = tid >> 7;  // 0 or 1
  const bool x_ok = (t0 + lrow) < T;
  const bool w_ok = lrow < E;
  const uint16_t* xrow = x + (size_t)(x_ok ? t0 + lrow : 0) * d;
  const float* wrow = wg + (size_t)(w_ok ? lrow : 0) * d;

  uint4 xv = make_uint4(0, 0, 0, 0);
  float4 wv0 = make_float4(0.f, 0.f, 0.f, 0.f), wv1 = wv0;
  auto gload = [&](int kc) {
    const int k = k_begin + kc * BK;
    if (x_ok) xv = *reinterpret_cast<const uint4*>(xrow + k + lq * 8);
    if (w_ok) {
      wv0 = *reinterpret_cast<const float4*>(wrow + k + lq * 4);
      wv1 = *reinterpret_cast<const float4*>(wrow + k + 8 + lq * 4);
    }
  };
  auto sstore = [&](int buf) {
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[buf][lq * 8 + 2 * i][lrow] = bf16_bits_to_float(xw[i] & 0xFFFFu);
      xs[buf][lq * 8 + 2 * i + 1][lrow] = bf16_bits_to_float(xw[i] >> 16);
    }
    ws[buf][lq * 4 + 0][lrow] = wv0.x;
    ws[buf][lq * 4 + 1][lrow] = wv0.y;
    ws[buf][lq * 4 + 2][lrow] = wv0.z;
    ws[buf][lq * 4 + 3][lrow] = wv0.w;
    ws[buf][8 + lq * 4 + 0][lrow] = wv1.x;
    ws[buf][8 + lq * 4 + 1][lrow] = wv1.y;
    ws[buf][8 + lq * 4 + 2][lrow] = wv1.z;
    ws[buf][8 + lq * 4 + 3][lrow] = wv1.w;
  };

  const int ty = tid >> 4, tx = tid & 15;
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;

  if (nk > 0) {
    gload(0);
    sstore(0);
  }
  __syncthreads();
  float part_acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) part_acc[i][j] = 0.f;
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    if (kc + 1 < nk) gload(kc + 1);
    // unrolled by 4, not fully: measured 15-25 % faster (the fully unrolled
    // chunk at 255 registers issues worse); the arithmetic order is the same
#pragma unroll 4
    for (int kk = 0; kk < BK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ws[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ws[buf][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) part_acc[i][j] = fmaf(a[i], b[j], part_acc[i][j]);
    }
    if ((kc % kFold) == kFold - 1 || kc + 1 == nk) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc[i][j] += (double)part_acc[i][j];
          part_acc[i][j] = 0.f;
        }
    }
    if (kc + 1 < nk) sstore(buf ^ 1);
    __syncthreads();
  }

  float* out = part + (size_t)split * T * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (t >= T) continue;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int e0 = half * 64 + tx * 4;
      float* dst = out + (size_t)t * E + e0;
      if (e0 + 3 < E && (E & 3) == 0) {
        *reinterpret_cast<float4*>(dst) =
            make_float4((float)acc[i][half * 4 + 0], (float)acc[i][half * 4 + 1],
                        (float)acc[i][half * 4 + 2], (float)acc[i][half * 4 + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (e0 + j < E) dst[j] = (float)acc[i][half * 4 + j];
      }
    }
  }
}

// Decode-sized batches (one token tile, K slices of 64): the CTA's whole
// slice of x and w_gate is loaded at once -- one memory round trip instead of
// four -- and each output is summed in fp32 from zero over its 64 products in
// ascending k, the same group the streaming kernel forms, so the partials are
// bit-identical to that kernel's.
constexpr int kOneShotK = 64;
constexpr size_t kOneShotSmem = (size_t)kOneShotK * (BT + BE) * sizeof(float);

__global__ void __launch_bounds__(kThreads, 1)
router_gemm_oneshot_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wg,
                           float* __restrict__ part, int T, int d, int E) {
  extern __shared__ __align__(16) float osm[];
  float* xs = osm;                   // [kOneShotK][BT]
  float* ws = osm + kOneShotK * BT;  // [kOneShotK][BE]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * BT;
  const int split = blockIdx.y;
  const int k0 = split * kOneShotK;
  const int row = tid & 127, h = tid >> 7;
  const bool x_ok = (t0 + row) < T;
  const bool w_ok = row < E;
  const uint16_t* xrow = x + (size_t)(x_ok ? t0 + row : 0) * d + k0;
  const float* wrow = wg + (size_t)(w_ok ? row : 0) * d + k0;
  // every load first: 8 bf16 of x per uint4 (q = h + 2i of 8), 4 floats of
  // w_gate per float4 (q = h + 2i of 16)
  uint4 xv[4];
  float4 wv[8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    xv[i] = x_ok ? *reinterpret_cast<const uint4*>(xrow + (h + 2 * i) * 8) : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    wv[i] = w_ok ? *reinterpret_cast<const float4*>(wrow + (h + 2 * i) * 4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int kb = (h + 2 * i) * 8;
    const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xs[(kb + 2 * j) * BT + row] = bf16_bits_to_float(xw[j] & 0xFFFFu);
      xs[(kb + 2 * j + 1) * BT + row] = bf16_bits_to_float(xw[j] >> 16);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int kb = (h + 2 * i) * 4;
    ws[(kb + 0) * BE + row] = wv[i].x;
    ws[(kb + 1) * BE + row] = wv[i].y;
    ws[(kb + 2) * BE + row] = wv[i].z;
    ws[(kb + 3) * BE + row] = wv[i].w;
  }
  __syncthreads();

  const int ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int kk = 0; kk < kOneShotK; ++kk) {
    const float4 a0 = *reinterpret_cast<const float4*>(&xs[kk * BT + ty * 4]);
    const float4 a1 = *reinterpret_cast<const float4*>(&xs[kk * BT + 64 + ty * 4]);
    const float4 b0 = *reinterpret_cast<const float4*>(&ws[kk * BE + tx * 4]);
    const float4 b1 = *reinterpret_cast<const float4*>(&ws[kk * BE + 64 + tx * 4]);
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }

  float* out = part + (size_t)split * T * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (t >= T) continue;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int e0 = half * 64 + tx * 4;
      float* dst = out + (size_t)t * E + e0;
      if (e0 + 3 < E && (E & 3) == 0) {
        *reinterpret_cast<float4*>(dst) = make_float4(acc[i][half * 4 + 0], acc[i][half * 4 + 1],
                                                      acc[i][half * 4 + 2], acc[i][half * 4 + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (e0 + j < E) dst[j] = acc[i][half * 4 + j];
      }
    }
  }
}

struct Cand {
  float key;
  int e;
  float p;
};

__device__ __forceinline__ bool better(const Cand& a, const Cand& b) {
  return a.key > b.key || (a.key == b.key && a.e < b.e);
}

constexpr int kTopkWarps = 8;

// WPT warps per token: warp q sums the contiguous run of split partials
// [q * per, (q + 1) * per) in fp64 in ascending order (the loads of 16 splits
// issued together so their latencies overlap), the runs are added in q order
// through shared memory, and the token's first warp does softmax and top-k.
// Many splits (decode) use 8 warps per token so each warp needs one round of
// loads; a few splits (prefill) use one.
template <int WPT>
__global__ void __launch_bounds__(kTopkWarps * 32)
router_topk_kernel(const float* __restrict__ part, int splits, const float* __restrict__ bias,
                   float* __restrict__ probs, int32_t* __restrict__ topk_idx,
                   float* __restrict__ topk_w, int T, int E, int k) {
  constexpr int kTok = kTopkWarps / WPT;  // tokens per CTA
  __shared__ double red[WPT > 1 ? kTopkWarps : 1][WPT > 1 ? 128 : 1];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int q = warp % WPT;
  const int t = blockIdx.x * kTok + warp / WPT;
  const bool live = t < T;

  bool valid[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) valid[i] = lane + 32 * i < E;
  const int per = (splits + WPT - 1) / WPT;
  const int sp_begin = q * per;
  const int sp_end = min(splits, sp_begin + per);
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  constexpr int kU = 16;
  for (int sp0 = sp_begin; live && sp0 < sp_end; sp0 += kU) {
    float v[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int sp = min(sp0 + u, sp_end - 1);  // clamped: every load is in bounds
#pragma unroll
      for (int i = 0; i < 4; ++i)
        v[u][i] = __ldg(part + ((size_t)sp * T + t) * E + min(lane + 32 * i, E - 1));
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (sp0 + u < sp_end) acc[i] += (double)v[u][i];
  }
  if constexpr (WPT > 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane + 32 * i] = acc[i];
    __syncthreads();
    if (q != 0) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[i] = red[warp][lane + 32 * i];
#pragma unroll
      for (int r = 1; r < WPT; ++r) acc[i] += red[warp + r][lane + 32 * i];
    }
  }
  if (!live) return;
  float z[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) z[i] = valid[i] ? (float)acc[i] : -INFINITY;
  float m = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float ex[4];
  float lsum = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ex[i] = valid[i] ? expf(z[i] - m) : 0.f;
    lsum += ex[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);

  Cand c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = lane + 32 * i;
    const float p = ex[i] / lsum;
    if (valid[i] && probs != nullptr) probs[(size_t)t * E + e] = p;
    float key = p + (bias != nullptr && valid[i] ? bias[e] : 0.f);
    if (!valid[i] || key != key) key = -INFINITY;  // NaN keys rank last
    c[i].key = key;
    c[i].e = valid[i] ? e : 0x7fffffff;
    c[i].p = p;
  }

  unsigned taken = 0;
  int my_idx = 0;
  float my_p = 0.f;
  for (int r = 0; r < k; ++r) {
    Cand best = {-INFINITY, 0x7fffffff, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (!(taken & (1u << i)) && better(c[i], best)) best = c[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Cand other;
      other.key = __shfl_xor_sync(0xffffffffu, best.key, o);
      other.e = __shfl_xor_sync(0xffffffffu, best.e, o);
      other.p = __shfl_xor_sync(0xffffffffu, best.p, o);
      if (better(other, best)) best = other;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (c[i].e == best.e) taken |= 1u << i;
    if (lane == r) {
      my_idx = best.e;
      my_p = best.p;
    }
  }
  float psum = 0.f;
  for (int r = 0; r < k; ++r) psum += __shfl_sync(0xffffffffu, my_p, r);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = my_idx;
    topk_w[(size_t)t * k + lane] = my_p / psum;
  }
}

struct SplitPlan {
  int splits;
  int kchunk;
};

// Split of K: one CTA per SM runs at a time, so pick the split count whose
// CTA count wastes the least of the last wave (waves / splits smallest),
// preferring fewer splits on near-ties, within a cap on the partial-logit
// buffer (16 MiB, or one split per tile if even that exceeds it).
SplitPlan plan_splits(const Shape& s, int num_sms) {
  const int tiles = (int)ceil_div(s.T, BT);
  int max_splits = s.d / (BK * 4) > 0 ? s.d / (BK * 4) : 1;
  const int64_t per_split = (int64_t)s.T * s.E * (int64_t)sizeof(float);
  const int64_t cap_bytes = int64_t(16) << 20;
  if (per_split > 0 && max_splits > cap_bytes / per_split)
    max_splits = (int)(cap_bytes / per_split) > 0 ? (int)(cap_bytes / per_split) : 1;
  int best = 1;
  double best_cost = 1e30;
  for (int sp = 1; sp <= max_splits && tiles > 0; ++sp) {
    const int kchunk = (int)round_up(ceil_div(s.d, sp), BK);
    const int real = (int)ceil_div(s.d, kchunk);
    const double waves = (double)ceil_div((int64_t)tiles * real, num_sms);
    const double cost = waves * kchunk;  // time ~ waves x work per CTA
    if (cost < best_cost * 0.98) {
      best_cost = cost;
      best = real;
    }
  }
  const int kchunk = (int)round_up(ceil_div(s.d, best), BK);
  return {(int)ceil_div(s.d, kchunk), kchunk};
}

}  // namespace

int router_splits(const Shape& s, int num_sms) { return plan_splits(s, num_sms).splits; }

size_t router_partials_bytes(const Shape& s, int num_sms) {
  return (size_t)plan_splits(s, num_sms).splits * (size_t)s.T * (size_t)s.E * sizeof(float);
}

cudaError_t launch_router(const Shape& s, const uint16_t* x, const float* w_gate,
                          const float* bias, float* probs, int32_t* topk_idx, float* topk_w,
                          float* partials, int num_sms, cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  const SplitPlan sp = plan_splits(s, num_sms);
  dim3 grid((unsigned)ceil_div(s.T, BT), (unsigned)sp.splits);
  cudaError_t err;
  if (grid.x == 1 && sp.kchunk == kOneShotK && (int64_t)sp.splits * kOneShotK == s.d) {
    err = cudaFuncSetAttribute(router_gemm_oneshot_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOneShotSmem);
    if (err != cudaSuccess) return err;
    router_gemm_oneshot_kernel<<<grid, kThreads, kOneShotSmem, st>>>(x, w_gate, partials, s.T,
                                                                     s.d, s.E);
  } else {
    router_gemm_kernel<<<grid, kThreads, 0, st>>>(x, w_gate, partials, s.T, s.d, s.E, sp.kchunk);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  auto topk = [&](auto kern, int wpt) {
    kern<<<(unsigned)ceil_div(s.T, kTopkWarps / wpt), kTopkWarps * 32, 0, st>>>(
        partials, sp.splits, bias, probs, topk_idx, topk_w, s.T, s.E, s.k);
  };
  if (sp.splits > 64)
    topk(router_topk_kernel<8>, 8);
  else if (sp.splits > 32)
    topk(router_topk_kernel<4>, 4);
  else if (sp.splits > 16)
    topk(router_topk_kernel<2>, 2);
  else
    topk(router_topk_kernel<1>, 1);
  return cudaGetLastError();
}

}  // namespace moe
