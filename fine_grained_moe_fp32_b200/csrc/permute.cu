// Permutation of the (token, slot) pairs into per-expert segments padded to
// `align` rows (dots.llm1 Technical Report, Method, systems paragraph: expert
// segments are padded to MMA tile multiples).  A stable counting sort:
//
//   permute_count_kernel    per chunk of 256 tokens: expert histogram
//   permute_scan_kernel     one CTA: per-expert exclusive scan over chunks,
//                           counts, padded segment offsets, -1 on padding rows
//   permute_scatter_kernel  per chunk: rank of each pair among the chunk's
//                           earlier tokens of the same expert (warp ballot
//                           masks + per-warp prefix), row_of / token_of_row
//   permute_copy_kernel     one CTA per token: x[t] read once, stored into
//                           the rows of its k pairs; one CTA per expert zeroes
//                           its segment's padding rows (16-byte vectors)
//
// A batch of at most one chunk (decode) runs count, scan and scatter as one
// CTA (permute_index_one_chunk_kernel): the same ranks and rows, two launches
// fewer.
#include "moe_internal.h"
#include "checks.cuh"

namespace moe {
namespace {

constexpr int kChunk = kChunkTokens;  // tokens per chunk = threads per CTA
constexpr int kMaxE = 128;
constexpr int kWarps = kChunk / 32;

__device__ __forceinline__ void set_status(unsigned int* status, unsigned int code) {
  if (status != nullptr) atomicCAS(status, 0u, code);
}

__global__ void __launch_bounds__(kChunk)
permute_count_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                     int32_t* __restrict__ chunk_counts, unsigned int* status) {
  __shared__ int hist[kMaxE];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t = c * kChunk + threadIdx.x;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= idx[(size_t)t * k + jj] == e;
      if (e >= 0 && e < E && !dup)
        atomicAdd(&hist[e], 1);
      else
        set_status(status, DEV_BAD_EXPERT_ID);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(size_t)c * E + e] = hist[e];
}

__global__ void __launch_bounds__(kMaxE)
permute_scan_kernel(const int32_t* __restrict__ chunk_counts, int nchunks, int E, int align,
                    int64_t cap, int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts,
                    int32_t* __restrict__ offsets, int32_t* __restrict__ token_of_row) {
  __shared__ int scan[kMaxE];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      chunk_base[(size_t)c * E + e] = total;
      total += chunk_counts[(size_t)c * E + e];
    }
    counts[e] = total;
  }
  const int padded = e < E ? (int)round_up(total, align) : 0;
  scan[e] = padded;
  __syncthreads();
  // inclusive Hillis-Steele scan over the (at most 128) experts
  for (int o = 1; o < kMaxE; o <<= 1) {
    const int v = e >= o ? scan[e - o] : 0;
    __syncthreads();
    scan[e] += v;
    __syncthreads();
  }
  const int end = scan[e];
  const int start = end - padded;
  if (e < E) {
    offsets[e] = start;
    if (e == E - 1) offsets[E] = end;
    for (int r = start + total; r < end; ++r)
      if (MOE_CHECK(r < cap)) token_of_row[r] = -1;
  }
  const int used = scan[E - 1];
  for (int64_t r = used + e; r < cap; r += blockDim.x) token_of_row[r] = -1;
}

__global__ void __launch_bounds__(kChunk)
permute_scatter_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                       const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets,
                       int32_t* __restrict__ row_of, int32_t* __restrict__ token_of_row,
                       int64_t cap) {
  __shared__ unsigned int masks[kWarps][kMaxE];
  __shared__ int pre[kWarps][kMaxE];
  __shared__ int base[kMaxE];
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += blockDim.x) (&masks[0][0])[i] = 0u;
  __syncthreads();
  const int t = c * kChunk + threadIdx.x;
  const bool tok_ok = t < T;
  if (tok_ok) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= idx[(size_t)t * k + jj] == e;
      if (e >= 0 && e < E && !dup) atomicOr(&masks[warp][e], 1u << lane);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      pre[w][e] = run;
      run += __popc(masks[w][e]);
    }
    base[e] = offsets[e] + chunk_base[(size_t)c * E + e];
  }
  __syncthreads();
  if (tok_ok) {
    const unsigned int lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= idx[(size_t)t * k + jj] == e;
      int row = -1;
      if (e >= 0 && e < E && !dup) {
        row = base[e] + pre[warp][e] + __popc(masks[warp][e] & lt);
        if (MOE_CHECK(row >= 0 && row < cap))
          token_of_row[row] = t;
        else
          row = -1;
      }
      row_of[(size_t)t * k + j] = row;
    }
  }
}

// count + scan + scatter for T <= kChunk tokens in one CTA of kChunk threads
// (token t = thread t): the per-warp ballot masks give both each expert's
// count and each pair's rank among earlier tokens.
__global__ void __launch_bounds__(kChunk)
permute_index_one_chunk_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int align,
                               int64_t cap, int32_t* __restrict__ counts,
                               int32_t* __restrict__ offsets, int32_t* __restrict__ row_of,
                               int32_t* __restrict__ token_of_row, unsigned int* status) {
  __shared__ unsigned int masks[kWarps][kMaxE];
  __shared__ int pre[kWarps][kMaxE];
  __shared__ int scan[kMaxE];
  __shared__ int base[kMaxE];
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  for (int i = t; i < kWarps * kMaxE; i += blockDim.x) (&masks[0][0])[i] = 0u;
  __syncthreads();
  const bool tok_ok = t < T;
  if (tok_ok) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= idx[(size_t)t * k + jj] == e;
      if (e >= 0 && e < E && !dup)
        atomicOr(&masks[warp][e], 1u << lane);
      else
        set_status(status, DEV_BAD_EXPERT_ID);
    }
  }
  __syncthreads();
  int total = 0, padded = 0;
  if (t < kMaxE) {
    if (t < E) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        pre[w][t] = total;
        total += __popc(masks[w][t]);
      }
      counts[t] = total;
      padded = (int)round_up(total, align);
    }
    scan[t] = padded;
  }
  __syncthreads();
  // inclusive Hillis-Steele scan over the (at most 128) experts
  for (int o = 1; o < kMaxE; o <<= 1) {
    const int v = (t < kMaxE && t >= o) ? scan[t - o] : 0;
    __syncthreads();
    if (t < kMaxE) scan[t] += v;
    __syncthreads();
  }
  if (t < E) {
    const int end = scan[t];
    const int start = end - padded;
    offsets[t] = start;
    if (t == E - 1) offsets[E] = end;
    base[t] = start;
    for (int r = start + total; r < end; ++r)
      if (MOE_CHECK(r < cap)) token_of_row[r] = -1;
  }
  const int used = scan[E - 1];
  for (int64_t r = used + t; r < cap; r += blockDim.x) token_of_row[r] = -1;
  __syncthreads();
  if (tok_ok) {
    const unsigned int lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      bool dup = false;
      for (int jj = 0; jj < j; ++jj) dup |= idx[(size_t)t * k + jj] == e;
      int row = -1;
      if (e >= 0 && e < E && !dup) {
        row = base[e] + pre[warp][e] + __popc(masks[warp][e] & lt);
        if (MOE_CHECK(row >= 0 && row < cap))
          token_of_row[row] = t;
        else
          row = -1;
      }
      row_of[(size_t)t * k + j] = row;
    }
  }
}

constexpr int kCopyThreads = 128;
constexpr int kMaxK = 8;

// x_perm, token-major: CTA t < T reads token t's row once and stores it into
// the rows of its k pairs (row_of); CTA T + e zeroes the padding rows of
// segment e (the rows between its count and the next segment).  Each x row is
// read once instead of once per pair, which matters when x does not fit in L2.
__global__ void __launch_bounds__(kCopyThreads)
permute_copy_kernel(const uint16_t* __restrict__ x, int T, int d, int k, int E,
                    const int32_t* __restrict__ row_of, const int32_t* __restrict__ counts,
                    const int32_t* __restrict__ offsets, int64_t cap,
                    uint16_t* __restrict__ x_perm) {
  const int nv = d / 8;
  if ((int)blockIdx.x >= T) {
    const int e = (int)blockIdx.x - T;
    const int64_t r0 = (int64_t)offsets[e] + counts[e], r1 = offsets[e + 1];
    if (!MOE_CHECK(r0 >= 0 && r1 <= cap)) return;
    uint4* base = reinterpret_cast<uint4*>(x_perm);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t i = r0 * nv + threadIdx.x; i < r1 * nv; i += kCopyThreads) base[i] = z;
    return;
  }
  const int t = blockIdx.x;
  __shared__ uint4* dst[kMaxK];
  if ((int)threadIdx.x < k) {
    const int r = row_of[(size_t)t * k + threadIdx.x];
    const bool ok = MOE_CHECK(r >= -1 && r < cap) && r >= 0 && r < cap;  // -1: pair skipped
    dst[threadIdx.x] = ok ? reinterpret_cast<uint4*>(x_perm + (size_t)r * d) : nullptr;
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  for (int v = threadIdx.x; v < nv; v += kCopyThreads) {
    const uint4 val = __ldg(src + v);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && dst[j] != nullptr) dst[j][v] = val;
  }
}

}  // namespace

size_t permute_scratch_bytes(const Shape& s) {
  const size_t nchunks = (size_t)ceil_div(s.T, kChunk);
  return 2 * nchunks * (size_t)s.E * sizeof(int32_t);
}

cudaError_t launch_permute(const Shape& s, const int32_t* topk_idx, const uint16_t* x,
                           int32_t* counts, int32_t* offsets, int32_t* row_of,
                           int32_t* token_of_row, uint16_t* x_perm, void* scratch,
                           unsigned int* status, cudaStream_t st) {
  const int nchunks = (int)ceil_div(s.T, kChunk);
  int32_t* chunk_counts = static_cast<int32_t*>(scratch);
  int32_t* chunk_base = chunk_counts + (size_t)nchunks * s.E;
  if (nchunks == 1) {
    permute_index_one_chunk_kernel<<<1, kChunk, 0, st>>>(topk_idx, s.T, s.k, s.E, s.align, s.cap,
                                                         counts, offsets, row_of, token_of_row,
                                                         status);
  } else {
    if (nchunks > 0) {
      permute_count_kernel<<<nchunks, kChunk, 0, st>>>(topk_idx, s.T, s.k, s.E, chunk_counts,
                                                       status);
    }
    permute_scan_kernel<<<1, kMaxE, 0, st>>>(chunk_counts, nchunks, s.E, s.align, s.cap,
                                             chunk_base, counts, offsets, token_of_row);
    if (nchunks > 0) {
      permute_scatter_kernel<<<nchunks, kChunk, 0, st>>>(topk_idx, s.T, s.k, s.E, chunk_base,
                                                         offsets, row_of, token_of_row, s.cap);
    }
  }
  if (s.cap > 0 && x_perm != nullptr && s.T + s.E > 0) {
    permute_copy_kernel<<<(unsigned)(s.T + s.E), kCopyThreads, 0, st>>>(
        x, s.T, s.d, s.k, s.E, row_of, counts, offsets, s.cap, x_perm);
  }
  return cudaGetLastError();
}

}  // namespace moe

MOE_CHECKS_UNIT(permute)
