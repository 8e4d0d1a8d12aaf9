// Backward of the MoE layer outside the expert GEMMs (selection held fixed;
// the bias only enters the selection key and gets no gradient):
//
//   combine_bwd_kernel     dy_perm[row(t,j)] = w[t,j] * dy[t];  dw[t,j] = <dy[t], y_perm[row(t,j)]>
//   zero_padding_rows      dy_perm padding rows = 0 (the wgrad sums run over them)
//   router_bwd_kernel      renormalisation and softmax backward, one warp per token:
//                          dp_j = (dw_j - sum_i w_i dw_i) / sum_sel p;
//                          dz_e = p_e (dp_e - sum_e' p_e' dp_e')  (dp = 0 off the chosen experts)
//   sgemm_kernel           fp32 GEMMs on CUDA cores for the gate: dz Wg (-> dx) and
//                          dz^T x (-> dWg, split-K partials summed in order)
//   unpermute_bwd_kernel   dx[t] = dx_shared[t] + dz Wg [t] + sum_j dx_perm[row(t,j)]
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "checks.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);  // one paired cvt, lo in the low half
  return *reinterpret_cast<const uint32_t*>(&h2);
}

constexpr int kCbThreads = 128;

// One CTA per token.  Each thread takes its 16-byte vectors of dy[t] in turn
// and, for each, issues the loads of all k routed rows before using them (the
// k rows are independent streams, so their HBM latencies overlap).  The dot
// products are reduced in a fixed order (per thread over its vectors, then
// warp butterfly, then warps in order), so dw is deterministic.
constexpr int kCbMaxK = 8;

__global__ void __launch_bounds__(kCbThreads)
combine_bwd_kernel(const uint16_t* __restrict__ dy, const float* __restrict__ y_perm,
                   const int32_t* __restrict__ row_of, const float* __restrict__ topk_w,
                   uint16_t* __restrict__ dy_perm, float* __restrict__ dw, int d, int k,
                   int64_t cap) {
  const int t = blockIdx.x;
  __shared__ float red[kCbMaxK][kCbThreads / 32];
  __shared__ const float* yrow[kCbMaxK];
  __shared__ uint16_t* orow[kCbMaxK];
  __shared__ float wsel[kCbMaxK];
  if ((int)threadIdx.x < k) {
    const int j = threadIdx.x;
    const int r = row_of[(size_t)t * k + j];
    const bool ok = MOE_CHECK(r >= -1 && r < cap) && r >= 0 && r < cap;  // -1: pair skipped
    yrow[j] = ok ? y_perm + (size_t)r * d : nullptr;
    orow[j] = ok ? dy_perm + (size_t)r * d : nullptr;
    wsel[j] = topk_w[(size_t)t * k + j];
  }
  __syncthreads();
  const int nv = d / 8;
  float part[kCbMaxK];
#pragma unroll
  for (int j = 0; j < kCbMaxK; ++j) part[j] = 0.f;
#pragma unroll 1
  for (int v = threadIdx.x; v < nv; v += kCbThreads) {
    const uint4 gv = reinterpret_cast<const uint4*>(dy + (size_t)t * d)[v];
    float4 ya[kCbMaxK], yb[kCbMaxK];
#pragma unroll
    for (int j = 0; j < kCbMaxK; ++j) {
      if (j < k && yrow[j] != nullptr) {
        const float4* yr = reinterpret_cast<const float4*>(yrow[j]);
        ya[j] = __ldg(yr + 2 * v);
        yb[j] = __ldg(yr + 2 * v + 1);
      }
    }
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int j = 0; j < kCbMaxK; ++j) {
      if (j < k && yrow[j] != nullptr) {
        const float yv[8] = {ya[j].x, ya[j].y, ya[j].z, ya[j].w,
                             yb[j].x, yb[j].y, yb[j].z, yb[j].w};
        const float w = wsel[j];
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          part[j] = fmaf(bf16lo(gw[q]), yv[2 * q], part[j]);
          part[j] = fmaf(bf16hi(gw[q]), yv[2 * q + 1], part[j]);
          o[q] = pack_bf16(w * bf16lo(gw[q]), w * bf16hi(gw[q]));
        }
        reinterpret_cast<uint4*>(orow[j])[v] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kCbMaxK; ++j) {
    if (j < k) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
      if ((threadIdx.x & 31) == 0) red[j][threadIdx.x >> 5] = part[j];
    }
  }
  __syncthreads();
  if ((int)threadIdx.x < k) {
    float s = 0.f;
    for (int i = 0; i < kCbThreads / 32; ++i) s += red[threadIdx.x][i];
    dw[(size_t)t * k + threadIdx.x] = s;
  }
}

constexpr int kPadWarps = 8;

__global__ void __launch_bounds__(kPadWarps * 32)
zero_padding_rows_kernel(uint16_t* __restrict__ rows, int d, const int32_t* __restrict__ offsets,
                         int E, const int32_t* __restrict__ token_of_row, int64_t cap) {
  const int64_t r = (int64_t)blockIdx.x * kPadWarps + (threadIdx.x >> 5);
  if (r >= cap || r >= offsets[E] || token_of_row[r] >= 0) return;
  uint4* dst = reinterpret_cast<uint4*>(rows + (size_t)r * d);
  for (int v = threadIdx.x & 31; v < d / 8; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
}

constexpr int kRbWarps = 8;

__global__ void __launch_bounds__(kRbWarps * 32)
router_bwd_kernel(const float* __restrict__ probs, const int32_t* __restrict__ topk_idx,
                  const float* __restrict__ topk_w, const float* __restrict__ dw,
                  float* __restrict__ dz, int T, int E, int k) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRbWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  // chosen experts, their probabilities and weight gradients (lane j < k)
  int e_j = 0;
  float p_j = 0.f, w_j = 0.f, dw_j = 0.f;
  if (lane < k) {
    e_j = topk_idx[(size_t)t * k + lane];
    e_j = min(max(e_j, 0), E - 1);
    p_j = probs[(size_t)t * E + e_j];
    w_j = topk_w[(size_t)t * k + lane];
    dw_j = dw[(size_t)t * k + lane];
  }
  float psum = 0.f, wdw = 0.f;
  for (int j = 0; j < k; ++j) {  // fixed order
    psum += __shfl_sync(0xffffffffu, p_j, j);
    wdw += __shfl_sync(0xffffffffu, w_j * dw_j, j);
  }
  const float dp_j = lane < k ? (dw_j - wdw) / psum : 0.f;
  float pdp = 0.f;
  for (int j = 0; j < k; ++j) pdp += __shfl_sync(0xffffffffu, p_j * dp_j, j);
  for (int i = 0; i < 4; ++i) {
    const int e = lane + 32 * i;
    if (e >= E) break;
    float dpe = 0.f;
    for (int j = 0; j < k; ++j) {
      const int ej = __shfl_sync(0xffffffffu, e_j, j);
      const float dpj = __shfl_sync(0xffffffffu, dp_j, j);
      if (ej == e) dpe = dpj;
    }
    const float pe = probs[(size_t)t * E + e];
    dz[(size_t)t * E + e] = pe * (dpe - pdp);
  }
}

// fp32 GEMM on CUDA cores: C[m, n] = sum_k A(m, k) B(k, n) over one K split.
//   A(m, k) = a[m * lda + k]  (A_MMAJOR = false)  or  a[k * lda + m]  (true)
//   B(k, n) = b[k * ldb + n]  (TB = float, or bf16 bits)
// 128 x 128 tile, 16-deep k chunks double-buffered in smem with the next
// chunk prefetched into registers; 16 x 16 threads of 8 x 8 outputs, one fp32
// running sum each (these gradients are held to bf16-level tolerances; an
// fp32 sum of K = 8192 terms is good to ~1e-5 relative).  blockIdx.z is the split of K; each split writes
// its own partial C slab.  Requires lda % 4 == 0 and ldb % 8 == 0.
constexpr int SB = 128, SK = 16, kSgThreads = 256;

template <bool A_MMAJOR, typename TB>
__global__ void __launch_bounds__(kSgThreads, 2)
sgemm_kernel(const float* __restrict__ a, int lda, const TB* __restrict__ b, int ldb,
             float* __restrict__ c, int ldc, int64_t c_split_stride, int M, int N, int K,
             int kchunk) {
  __shared__ __align__(16) float As[2][SK][SB];
  __shared__ __align__(16) float Bs[2][SK][SB];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * SB, n0 = blockIdx.x * SB;
  const int k_begin = blockIdx.z * kchunk;
  const int k_end = min(K, k_begin + kchunk);
  const int nk = (k_end - k_begin + SK - 1) / SK;
  const int ty = tid >> 4, tx = tid & 15;

  float4 ra[2];
  float4 rb[2];
  auto load_a = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (A_MMAJOR) {  // 16 k-rows x 32 float4 along m
        const int kk = (tid >> 5) + 8 * i, m4 = (tid & 31) * 4;
        const int gk = k0 + kk, gm = m0 + m4;
        if (gk < k_end) {
          const float* src = a + (size_t)gk * lda + gm;
          if (gm + 3 < M) {
            v = *reinterpret_cast<const float4*>(src);
          } else {
            if (gm < M) v.x = src[0];
            if (gm + 1 < M) v.y = src[1];
            if (gm + 2 < M) v.z = src[2];
          }
        }
      } else {  // 128 m-rows x 4 float4 along k
        const int idx = tid + kSgThreads * i;
        const int mm = idx >> 2, kq = idx & 3;
        const int gm = m0 + mm, gk = k0 + kq * 4;
        if (gm < M) {
          const float* src = a + (size_t)gm * lda + gk;
          if (gk + 3 < k_end) {
            v = *reinterpret_cast<const float4*>(src);
          } else {
            if (gk < k_end) v.x = src[0];
            if (gk + 1 < k_end) v.y = src[1];
            if (gk + 2 < k_end) v.z = src[2];
          }
        }
      }
      ra[i] = v;
    }
  };
  auto store_a = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (A_MMAJOR) {
        const int kk = (tid >> 5) + 8 * i, m4 = (tid & 31) * 4;
        *reinterpret_cast<float4*>(&As[buf][kk][m4]) = ra[i];
      } else {
        const int idx = tid + kSgThreads * i;
        const int mm = idx >> 2, kq = idx & 3;
        As[buf][kq * 4 + 0][mm] = ra[i].x;
        As[buf][kq * 4 + 1][mm] = ra[i].y;
        As[buf][kq * 4 + 2][mm] = ra[i].z;
        As[buf][kq * 4 + 3][mm] = ra[i].w;
      }
    }
  };
  auto load_b = [&](int k0) {
    if constexpr (sizeof(TB) == 2) {  // 16 k-rows x 16 vectors of 8 bf16
      const int kk = tid >> 4, n8 = (tid & 15) * 8;
      const int gk = k0 + kk, gn = n0 + n8;
      uint4 w = make_uint4(0, 0, 0, 0);
      if (gk < k_end && gn < N) w = *reinterpret_cast<const uint4*>(b + (size_t)gk * ldb + gn);
      rb[0] = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                          __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
      rb[1] = make_float4(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u),
                          __uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u));
    } else {  // 16 k-rows x 32 float4
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int kk = (tid >> 5) + 8 * i, n4 = (tid & 31) * 4;
        const int gk = k0 + kk, gn = n0 + n4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (gk < k_end && gn < N) v = *reinterpret_cast<const float4*>(b + (size_t)gk * ldb + gn);
        rb[i] = v;
      }
    }
  };
  auto store_b = [&](int buf) {
    if constexpr (sizeof(TB) == 2) {
      const int kk = tid >> 4, n8 = (tid & 15) * 8;
      *reinterpret_cast<float4*>(&Bs[buf][kk][n8]) = rb[0];
      *reinterpret_cast<float4*>(&Bs[buf][kk][n8 + 4]) = rb[1];
    } else {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int kk = (tid >> 5) + 8 * i, n4 = (tid & 31) * 4;
        *reinterpret_cast<float4*>(&Bs[buf][kk][n4]) = rb[i];
      }
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  if (nk > 0) {
    load_a(k_begin);
    load_b(k_begin);
    store_a(0);
    store_b(0);
  }
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    if (kc + 1 < nk) {
      load_a(k_begin + (kc + 1) * SK);
      load_b(k_begin + (kc + 1) * SK);
    }
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (kc + 1 < nk) {
      store_a(buf ^ 1);
      store_b(buf ^ 1);
    }
    __syncthreads();
  }
  float* cs = c + (size_t)blockIdx.z * c_split_stride;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int gn = n0 + half * 64 + tx * 4;
      float* dst = cs + (size_t)gm * ldc + gn;
      if (gn + 3 < N) {
        *reinterpret_cast<float4*>(dst) = make_float4(acc[i][half * 4], acc[i][half * 4 + 1],
                                                      acc[i][half * 4 + 2], acc[i][half * 4 + 3]);
      } else {
        for (int j = 0; j < 4; ++j)
          if (gn + j < N) dst[j] = acc[i][half * 4 + j];
      }
    }
  }
}

__global__ void sum_splits_kernel(const float* __restrict__ part, int splits, int64_t n,
                                  float* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  double s = 0.0;
  for (int sp = 0; sp < splits; ++sp) s += (double)part[(size_t)sp * n + i];
  out[i] = (float)s;
}

// dx [T, d]: the fp32 sum, rounded once to bf16, or kept in fp32 (F32).
template <bool F32>
__global__ void __launch_bounds__(kCbThreads)
unpermute_bwd_kernel(const float* __restrict__ dx_shared, const float* __restrict__ dx_router,
                     const float* __restrict__ dx_perm, const int32_t* __restrict__ row_of,
                     void* __restrict__ dx, int d, int k, int64_t cap) {
  const int t = blockIdx.x;
  __shared__ int rows[8];
  if (threadIdx.x < k) {
    const int r = row_of[(size_t)t * k + threadIdx.x];
    rows[threadIdx.x] = (MOE_CHECK(r >= -1 && r < cap) && r >= 0 && r < cap) ? r : -1;
  }
  __syncthreads();
  for (int v = threadIdx.x; v < d / 8; v += kCbThreads) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (dx_shared != nullptr) {
      const float4* s = reinterpret_cast<const float4*>(dx_shared + (size_t)t * d) + 2 * v;
      const float4 p0 = s[0], p1 = s[1];
      acc[0] = p0.x; acc[1] = p0.y; acc[2] = p0.z; acc[3] = p0.w;
      acc[4] = p1.x; acc[5] = p1.y; acc[6] = p1.z; acc[7] = p1.w;
    }
    {
      const float4* s = reinterpret_cast<const float4*>(dx_router + (size_t)t * d) + 2 * v;
      const float4 p0 = s[0], p1 = s[1];
      acc[0] += p0.x; acc[1] += p0.y; acc[2] += p0.z; acc[3] += p0.w;
      acc[4] += p1.x; acc[5] += p1.y; acc[6] += p1.z; acc[7] += p1.w;
    }
    for (int j = 0; j < k; ++j) {
      if (rows[j] < 0) continue;
      const float4* src = reinterpret_cast<const float4*>(dx_perm + (size_t)rows[j] * d) + 2 * v;
      const float4 p0 = src[0], p1 = src[1];
      acc[0] += p0.x; acc[1] += p0.y; acc[2] += p0.z; acc[3] += p0.w;
      acc[4] += p1.x; acc[5] += p1.y; acc[6] += p1.z; acc[7] += p1.w;
    }
    if (F32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(dx) + (size_t)t * d) + 2 * v;
      o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) o[q] = pack_bf16(acc[2 * q], acc[2 * q + 1]);
      reinterpret_cast<uint4*>(static_cast<uint16_t*>(dx) + (size_t)t * d)[v] =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace

int dwg_splits(const Shape& s) {
  const int tiles = (int)ceil_div(s.d, SB) * (int)ceil_div(s.E, SB);
  int sp = tiles > 0 ? 296 / tiles : 1;
  sp = sp < 1 ? 1 : sp;
  const int max_sp = s.T / 256 > 0 ? s.T / 256 : 1;
  return sp > max_sp ? max_sp : sp;
}

cudaError_t launch_backward_misc_pre(const Shape& s, const BackwardMiscArgs& a, cudaStream_t st) {
  if (s.T > 0) {
    combine_bwd_kernel<<<s.T, kCbThreads, 0, st>>>(a.dy, a.y_perm, a.row_of, a.topk_w, a.dy_perm,
                                                   a.dw, s.d, s.k, s.cap);
    router_bwd_kernel<<<(unsigned)ceil_div(s.T, kRbWarps), kRbWarps * 32, 0, st>>>(
        a.probs, a.topk_idx, a.topk_w, a.dw, a.dz, s.T, s.E, s.k);
  }
  if (s.cap > 0)
    zero_padding_rows_kernel<<<(unsigned)ceil_div(s.cap, kPadWarps), kPadWarps * 32, 0, st>>>(
        a.dy_perm, s.d, a.offsets, s.E, a.token_of_row, s.cap);
  return cudaGetLastError();
}

cudaError_t launch_backward_misc_post(const Shape& s, const BackwardMiscArgs& a,
                                      cudaStream_t st) {
  if (s.T == 0) {
    return cudaMemsetAsync(a.dw_gate, 0, (size_t)s.E * s.d * sizeof(float), st);
  }
  // dz Wg -> dx_router [T, d]   (A = dz [T, E] K-major, B = Wg [E, d])
  {
    dim3 grid((unsigned)ceil_div(s.d, SB), (unsigned)ceil_div(s.T, SB), 1);
    sgemm_kernel<false, float><<<grid, kSgThreads, 0, st>>>(a.dz, s.E, a.w_gate, s.d, a.dx_router,
                                                            s.d, 0, s.T, s.d, s.E, s.E);
  }
  // dz^T x -> dWg [E, d]   (A(e, t) = dz[t, e], B = x [T, d] bf16), split-K over tokens
  {
    const int sp = dwg_splits(s);
    const int kchunk = (int)round_up(ceil_div(s.T, sp), SK);
    const int splits = (int)ceil_div(s.T, kchunk);
    dim3 grid((unsigned)ceil_div(s.d, SB), (unsigned)ceil_div(s.E, SB), (unsigned)splits);
    sgemm_kernel<true, uint16_t><<<grid, kSgThreads, 0, st>>>(
        a.dz, s.E, a.x, s.d, a.dwg_partials, s.d, (int64_t)s.E * s.d, s.E, s.d, s.T, kchunk);
    const int64_t n = (int64_t)s.E * s.d;
    sum_splits_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, st>>>(a.dwg_partials, splits, n,
                                                                   a.dw_gate);
  }
  if (a.dx_f32)
    unpermute_bwd_kernel<true><<<s.T, kCbThreads, 0, st>>>(a.dx_shared, a.dx_router, a.dx_perm,
                                                           a.row_of, a.dx, s.d, s.k, s.cap);
  else
    unpermute_bwd_kernel<false><<<s.T, kCbThreads, 0, st>>>(a.dx_shared, a.dx_router, a.dx_perm,
                                                            a.row_of, a.dx, s.d, s.k, s.cap);
  return cudaGetLastError();
}

}  // namespace moe

MOE_CHECKS_UNIT(backward)
