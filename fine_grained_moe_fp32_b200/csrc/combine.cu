// Combine: weighted un-permute of the routed expert outputs plus the shared
// experts (dots.llm1 Technical Report, Method: shared experts are always on;
// the routed experts enter with their gate weights).  With expert parallelism
// the routed rows are read from the receive buffers of the ranks that own the
// experts (the return half of the all-to-all, fused into the sum).
//
//   y[t] = y_shared[t] + sum_{j < k} w[t, j] * y_perm[row_of[t*k + j]]
//
// The routed outputs y_perm are fp32 (the down GEMM's accumulators, not
// rounded), so the only rounding of y is the final one.  fp32 accumulation,
// slot j in ascending order.  CTA (t, b) covers 8-element groups
// b*128 .. b*128+127 of token t, one per thread (two 16-byte loads per
// routed row), with the k routed rows' loads all issued before the sum.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "checks.cuh"

namespace moe {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxK = 8;

__device__ __forceinline__ void add_f32x8(float (&acc)[8], float4 a, float4 b, float w) {
  acc[0] = fmaf(w, a.x, acc[0]);
  acc[1] = fmaf(w, a.y, acc[1]);
  acc[2] = fmaf(w, a.z, acc[2]);
  acc[3] = fmaf(w, a.w, acc[3]);
  acc[4] = fmaf(w, b.x, acc[4]);
  acc[5] = fmaf(w, b.y, acc[5]);
  acc[6] = fmaf(w, b.z, acc[6]);
  acc[7] = fmaf(w, b.w, acc[7]);
}

// Where slot j of token t lives: its row of this rank's segment buffer.
struct LocalRows {
  const float* y_perm;
  const int32_t* row_of;
  int64_t cap;
  __device__ const float* row(size_t p, int d) const {
    const int r = row_of[p];
    if (!MOE_CHECK(r >= -1 && r < cap)) return nullptr;  // -1: a pair that was skipped
    return (r >= 0 && r < cap) ? y_perm + (size_t)r * d : nullptr;
  }
};

// Expert parallel: the row the dispatch wrote into the owner's receive
// buffer, read back from there (peer loads when the owner is another GPU).
struct OwnerRows {
  const float* const* y_recv;
  const int32_t* topk_idx;
  const int32_t* remote_row;
  int E, El;
  int64_t cap;
  __device__ const float* row(size_t p, int d) const {
    const int e = topk_idx[p], r = remote_row[p];
    if (!MOE_CHECK(r >= -1 && r < cap)) return nullptr;  // -1: a pair that was not sent
    if (e < 0 || e >= E || r < 0 || r >= cap) return nullptr;
    const float* b = y_recv[e / El];
    return (reinterpret_cast<uintptr_t>(b) & 15) ? nullptr : b + (size_t)r * d;
  }
};

template <typename Rows>
__global__ void __launch_bounds__(kThreads)
combine_kernel(Rows src, const float* __restrict__ topk_w, const float* __restrict__ y_shared,
               uint16_t* __restrict__ y, int d, int k) {
  const int t = blockIdx.x;
  __shared__ const float* rows[kMaxK];
  __shared__ float ws[kMaxK];
  if (threadIdx.x < k) {
    rows[threadIdx.x] = src.row((size_t)t * k + threadIdx.x, d);
    ws[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  const int nv = d / 8;
  const int v = blockIdx.y * kThreads + threadIdx.x;
  if (v < nv) {
    float acc[8];
    if (y_shared != nullptr) {
      const float4* s = reinterpret_cast<const float4*>(y_shared + (size_t)t * d) + 2 * v;
      const float4 a = s[0], b = s[1];
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    }
    float4 va[kMaxK], vb[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && rows[j] != nullptr) {
        const float4* r = reinterpret_cast<const float4*>(rows[j]) + 2 * v;
        va[j] = __ldg(r);
        vb[j] = __ldg(r + 1);
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && rows[j] != nullptr) add_f32x8(acc, va[j], vb[j], ws[j]);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      o[i] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    reinterpret_cast<uint4*>(y + (size_t)t * d)[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const float* y_perm, const int32_t* row_of,
                           const float* topk_w, const float* y_shared, uint16_t* y,
                           cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  const dim3 grid((unsigned)s.T, (unsigned)ceil_div(s.d / 8, kThreads));
  combine_kernel<<<grid, kThreads, 0, st>>>(LocalRows{y_perm, row_of, s.cap}, topk_w, y_shared, y,
                                            s.d, s.k);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const Shape& s, int world, const float* const* y_recv,
                              const int32_t* topk_idx, const int32_t* remote_row, int64_t cap,
                              const float* topk_w, const float* y_shared, uint16_t* y,
                              cudaStream_t st) {
  if (s.T == 0) return cudaSuccess;
  const dim3 grid((unsigned)s.T, (unsigned)ceil_div(s.d / 8, kThreads));
  const OwnerRows src{y_recv, topk_idx, remote_row, s.E, s.E / world, cap};
  combine_kernel<<<grid, kThreads, 0, st>>>(src, topk_w, y_shared, y, s.d, s.k);
  return cudaGetLastError();
}

}  // namespace moe

MOE_CHECKS_UNIT(combine)
