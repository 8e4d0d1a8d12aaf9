// Expert parallelism: the all-to-all dispatch of the MoE layer over W ranks
// that each own E/W experts (dots.llm1 Technical Report, Method / Key claims,
// systems paragraph: the MoE all-to-all between ranks, overlapped with the
// grouped GEMMs; "How dots.llm1's 14B MoE Architecture Matches 72B LLM
// Performance", Computational Infrastructure Innovations).
//
// Receive layout on rank r, owner of experts r*El .. r*El + El-1 (El = E/W):
// one segment per local expert, padded to `align` rows, holding the (token,
// slot) pairs of every source rank in rank order, each source's pairs in its
// own segment order (ascending token id).  Every rank derives the same layout
// from all ranks' per-expert counts, so the exchange needs no reply: a source
// writes each of its pairs' token rows straight into the owner's receive
// buffer (stores to peer memory over NVLink when that buffer is another
// GPU's) and the combine reads the expert outputs back from there.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPlanThreads = 128;  // one thread per expert (E <= 128)
constexpr int kCopyThreads = 128;
constexpr int kMaxK = 8;

__device__ __forceinline__ void flag(unsigned int* status, unsigned int code) {
  if (status != nullptr) atomicCAS(status, 0u, code);
}

// Thread e: the pairs of expert e from all ranks, its padded segment, and
// where this rank's pairs of e start in the owner's receive buffer.  A count
// table that is negative, disagrees with this rank's own counts, or overflows
// an owner's receive buffer is flagged and turns the whole exchange into a
// no-op (every dst_row -1, this rank receives nothing).
__global__ void __launch_bounds__(kPlanThreads)
ep_plan_kernel(const int32_t* const* __restrict__ counts_of, const int32_t* __restrict__ own,
               int world, int rank, int E, int align, int64_t recv_cap,
               int32_t* __restrict__ dst_row, int32_t* __restrict__ recv_offsets,
               int32_t* __restrict__ recv_counts, unsigned int* status) {
  __shared__ int64_t padded[kPlanThreads];
  const int e = threadIdx.x, El = E / world;
  int64_t tot = 0, before = 0;
  bool bad = false;
  if (e < E) {
    for (int s = 0; s < world; ++s) {
      const int32_t c = counts_of[s][e];
      bad |= c < 0;
      if (s < rank) before += c;
      tot += c;
    }
    bad |= counts_of[rank][e] != own[e];
  }
  padded[e] = e < E ? round_up(tot, align) : 0;
  __syncthreads();
  int64_t base = 0, end = 0;
  if (e < E) {
    const int first = (e / El) * El;
    for (int i = first; i < first + El; ++i) {
      if (i < e) base += padded[i];
      end += padded[i];
    }
    bad |= end > recv_cap;
  }
  bad = __syncthreads_or(bad) != 0;
  if (e < E) {
    dst_row[e] = bad ? -1 : (int32_t)(base + before);
    if (e / El == rank) {
      const int le = e - rank * El;
      recv_offsets[le] = bad ? 0 : (int32_t)base;
      recv_counts[le] = bad ? 0 : (int32_t)tot;
      if (le == El - 1) recv_offsets[El] = bad ? 0 : (int32_t)(base + padded[e]);
    }
  }
  if (bad && e == 0) flag(status, DEV_BAD_EP_LAYOUT);
}

// CTA t < T: token t's row, read once, stored into the receive row of each of
// its k pairs (remote_row records that row for the combine).  CTA T + le:
// zero the padding rows of this rank's own segment le.  The row of pair p in
// the owner's buffer is dst_row[e] plus the pair's place inside this rank's
// segment of e (row_of[p] - offsets[e]).
__global__ void __launch_bounds__(kCopyThreads)
ep_dispatch_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ topk_idx,
                   const int32_t* __restrict__ row_of, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ dst_row, uint16_t* const* __restrict__ x_recv,
                   const int32_t* __restrict__ recv_offsets,
                   const int32_t* __restrict__ recv_counts, int T, int d, int k, int E, int El,
                   int rank, int64_t recv_cap, int32_t* __restrict__ remote_row,
                   unsigned int* status) {
  const int nv = d / 8;
  if ((int)blockIdx.x >= T) {
    const int le = (int)blockIdx.x - T;
    const int64_t r0 = (int64_t)recv_offsets[le] + recv_counts[le], r1 = recv_offsets[le + 1];
    uint4* base = reinterpret_cast<uint4*>(x_recv[rank]);
    if (r1 > recv_cap || (reinterpret_cast<uintptr_t>(base) & 15)) {
      if (threadIdx.x == 0) flag(status, DEV_BAD_EP_LAYOUT);
      return;
    }
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t i = r0 * nv + threadIdx.x; i < r1 * nv; i += kCopyThreads) base[i] = z;
    return;
  }
  const int t = blockIdx.x;
  __shared__ uint4* dst[kMaxK];
  if ((int)threadIdx.x < k) {
    const int p = t * k + threadIdx.x;
    const int e = topk_idx[p];
    uint4* q = nullptr;
    int32_t rr = -1;
    if (e >= 0 && e < E && dst_row[e] >= 0) {
      const int64_t row = (int64_t)dst_row[e] + (row_of[p] - offsets[e]);
      uint16_t* buf = x_recv[e / El];
      if (row >= 0 && row < recv_cap && !(reinterpret_cast<uintptr_t>(buf) & 15)) {
        rr = (int32_t)row;
        q = reinterpret_cast<uint4*>(buf + row * d);
      } else {
        flag(status, DEV_BAD_EP_LAYOUT);
      }
    } else if (e < 0 || e >= E) {
      flag(status, DEV_BAD_EXPERT_ID);
    }
    dst[threadIdx.x] = q;
    remote_row[p] = rr;
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  for (int v = threadIdx.x; v < nv; v += kCopyThreads) {
    const uint4 val = __ldg(src + v);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && dst[j] != nullptr) dst[j][v] = val;
  }
  // the rows reach the owners' memory before this rank signals its peers
  __threadfence_system();
}

}  // namespace

int64_t ep_recv_capacity(const Shape& s, int world) {
  return (int64_t)world * s.T * s.k + (int64_t)(s.E / world) * (s.align - 1);
}

cudaError_t launch_ep_dispatch(const Shape& s, int world, int rank, const uint16_t* x,
                               const int32_t* topk_idx, const int32_t* row_of,
                               const int32_t* offsets, const int32_t* counts,
                               const int32_t* const* counts_of, uint16_t* const* x_recv,
                               int32_t* dst_row, int32_t* recv_offsets, int32_t* recv_counts,
                               int32_t* remote_row, unsigned int* status, cudaStream_t st) {
  const int El = s.E / world;
  const int64_t cap = ep_recv_capacity(s, world);
  ep_plan_kernel<<<1, kPlanThreads, 0, st>>>(counts_of, counts, world, rank, s.E, s.align, cap,
                                             dst_row, recv_offsets, recv_counts, status);
  ep_dispatch_kernel<<<(unsigned)(s.T + El), kCopyThreads, 0, st>>>(
      x, topk_idx, row_of, offsets, dst_row, x_recv, recv_offsets, recv_counts, s.T, s.d, s.k,
      s.E, El, rank, cap, remote_row, status);
  return cudaGetLastError();
}

}  // namespace moe
