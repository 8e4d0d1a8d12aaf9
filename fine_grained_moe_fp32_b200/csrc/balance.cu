// Load balancing on the training side (dots.llm1 Technical Report, Method:
// the router is balanced by the DeepSeek auxiliary-loss-free per-expert bias,
// stepped after each batch from the experts' loads, together with a
// sequence-wise balance loss against extreme imbalance inside a sequence).
// The report gives no formulas; the DeepSeek forms are used:
//
//   f[s,e] = E / (k L) * #{(t, j) : t in sequence s, idx[t,j] = e}
//   P[s,e] = (1 / L) * sum_{t in s} p[t,e]
//   loss   = alpha / n_seq * sum_s sum_e f[s,e] P[s,e]
//   b_e   <- b_e - gamma * sign(count_e - T k / E)
//
// Every sum is fp64 in a fixed order, so the results are deterministic.
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;  // one thread per expert (E <= 128)
constexpr int kChunk = 64;     // tokens per partial-sum CTA
constexpr int kLossThreads = 256;
constexpr int kBatch = 16;     // independent loads in flight per thread

__device__ __forceinline__ void flag(unsigned int* status, unsigned int code) {
  if (status != nullptr) atomicCAS(status, 0u, code);
}

// CTA s * chunks + c: tokens [s L + c kChunk, min(s L + (c+1) kChunk, (s+1) L))
// of sequence s (a 1-D grid: n_seq may exceed the 65535 limit of grid y).
// Thread e sums p[t, e] over those tokens (one coalesced row of E floats per
// token across the CTA) and the CTA counts the pairs per expert with
// shared-memory integer atomics (exact, order-free).
__global__ void __launch_bounds__(kThreads)
balance_partial_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx, int E,
                       int k, int seq_len, int chunks, double* __restrict__ part_p,
                       int32_t* __restrict__ part_c, unsigned int* status) {
  __shared__ int hist[kThreads];
  const int s = (int)(blockIdx.x / chunks), c = (int)(blockIdx.x % chunks), e = threadIdx.x;
  const int64_t t0 = (int64_t)s * seq_len + (int64_t)c * kChunk;
  const int64_t t1 = min((int64_t)(s + 1) * seq_len, t0 + kChunk);
  hist[e] = 0;
  __syncthreads();
  const int n = (int)(t1 - t0) * k;
  const int32_t* id = idx + t0 * k;
  for (int i = e; i < n; i += kThreads) {
    const int v = id[i];
    if (v >= 0 && v < E)
      atomicAdd(&hist[v], 1);
    else
      flag(status, DEV_BAD_EXPERT_ID);
  }
  // ascending token order; the loads of kBatch tokens are issued together
  double acc = 0.0;
  if (e < E) {
    const float* col = probs + t0 * E + e;
    const int nt = (int)(t1 - t0);
    int t = 0;
    for (; t + kBatch <= nt; t += kBatch) {
      float v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) v[u] = __ldg(col + (size_t)(t + u) * E);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) acc += (double)v[u];
    }
    for (; t < nt; ++t) acc += (double)__ldg(col + (size_t)t * E);
  }
  __syncthreads();
  if (e < E) {
    const size_t o = ((size_t)s * chunks + c) * E + e;
    part_p[o] = acc;
    part_c[o] = hist[e];
  }
}

// CTA s: f and P of sequence s from its chunks (ascending chunk order), and
// the sequence's sum_e f P (ascending-stride tree in shared memory).
__global__ void __launch_bounds__(kThreads)
balance_seq_kernel(const double* __restrict__ part_p, const int32_t* __restrict__ part_c, int E,
                   int k, int seq_len, int chunks, float* __restrict__ f, float* __restrict__ P,
                   double* __restrict__ seq_fp) {
  __shared__ double red[kThreads];
  const int s = blockIdx.x, e = threadIdx.x;
  double fp = 0.0;
  if (e < E) {
    double ps = 0.0;
    int64_t cnt = 0;
    const size_t base = (size_t)s * chunks * E + e;
    int c = 0;
    for (; c + kBatch <= chunks; c += kBatch) {   // ascending chunk order, batched loads
      double vp[kBatch];
      int vc[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        vp[u] = part_p[base + (size_t)(c + u) * E];
        vc[u] = part_c[base + (size_t)(c + u) * E];
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        ps += vp[u];
        cnt += vc[u];
      }
    }
    for (; c < chunks; ++c) {
      ps += part_p[base + (size_t)c * E];
      cnt += part_c[base + (size_t)c * E];
    }
    // E*cnt and k*L are exact integers, so fv is one correctly rounded quotient
    const double fv = (double)((int64_t)E * cnt) / (double)((int64_t)k * seq_len);
    const double pv = ps / (double)seq_len;
    f[(size_t)s * E + e] = (float)fv;
    P[(size_t)s * E + e] = (float)pv;
    fp = fv * pv;
  }
  red[e] = fp;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (e < w) red[e] += red[e + w];
    __syncthreads();
  }
  if (e == 0) seq_fp[s] = red[0];
}

// One CTA: loss = alpha * (sum_s seq_fp[s]) / n_seq, summed per thread over a
// fixed stride, then by a fixed tree.
__global__ void __launch_bounds__(kLossThreads)
balance_loss_kernel(const double* __restrict__ seq_fp, int n_seq, float alpha,
                    float* __restrict__ loss) {
  __shared__ double red[kLossThreads];
  const int i = threadIdx.x;
  double a = 0.0;
  for (int s = i; s < n_seq; s += kLossThreads) a += seq_fp[s];
  red[i] = a;
  __syncthreads();
  for (int w = kLossThreads / 2; w > 0; w >>= 1) {
    if (i < w) red[i] += red[i + w];
    __syncthreads();
  }
  if (i == 0) *loss = n_seq > 0 ? (float)((double)alpha * red[0] / (double)n_seq) : 0.f;
}

// b_e - gamma if E*count_e > T*k (above the mean load), b_e + gamma if below,
// b_e unchanged (bit for bit) at the mean.  bias_out may alias bias_in: each
// thread reads its element before writing it.
__global__ void __launch_bounds__(kThreads)
bias_update_kernel(const int32_t* __restrict__ counts, const float* bias_in, float* bias_out,
                   int E, int64_t Tk, float gamma) {
  const int e = threadIdx.x;
  if (e >= E) return;
  const int64_t excess = (int64_t)E * counts[e] - Tk;
  const float b = bias_in[e];
  bias_out[e] = excess > 0 ? b - gamma : (excess < 0 ? b + gamma : b);
}

struct BalancePlan {
  int n_seq, chunks;
  size_t off_c, off_seq, total;
};

size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

BalancePlan plan(const Shape& s, int seq_len) {
  BalancePlan p{};
  p.n_seq = s.T / seq_len;
  p.chunks = (int)ceil_div(seq_len, kChunk);
  const size_t n = (size_t)p.n_seq * p.chunks * s.E;
  p.off_c = al256(n * sizeof(double));
  p.off_seq = p.off_c + al256(n * sizeof(int32_t));
  p.total = p.off_seq + al256((size_t)p.n_seq * sizeof(double));
  return p;
}

}  // namespace

size_t balance_workspace_bytes(const Shape& s, int seq_len) {
  return plan(s, seq_len).total + kGuardBytes;
}

cudaError_t launch_balance_stats(const Shape& s, int seq_len, const float* probs,
                                 const int32_t* topk_idx, float alpha, float* f, float* P,
                                 float* loss, void* workspace, unsigned int* status,
                                 cudaStream_t st) {
  const BalancePlan p = plan(s, seq_len);
  if (p.n_seq == 0) {
    balance_loss_kernel<<<1, kLossThreads, 0, st>>>(nullptr, 0, alpha, loss);
    return cudaGetLastError();
  }
  char* ws = static_cast<char*>(workspace);
  double* part_p = reinterpret_cast<double*>(ws);
  int32_t* part_c = reinterpret_cast<int32_t*>(ws + p.off_c);
  double* seq_fp = reinterpret_cast<double*>(ws + p.off_seq);
  const unsigned int blocks = (unsigned int)((int64_t)p.n_seq * p.chunks);
  balance_partial_kernel<<<blocks, kThreads, 0, st>>>(
      probs, topk_idx, s.E, s.k, seq_len, p.chunks, part_p, part_c, status);
  balance_seq_kernel<<<p.n_seq, kThreads, 0, st>>>(part_p, part_c, s.E, s.k, seq_len, p.chunks,
                                                   f, P, seq_fp);
  balance_loss_kernel<<<1, kLossThreads, 0, st>>>(seq_fp, p.n_seq, alpha, loss);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(const Shape& s, const int32_t* counts, float gamma,
                               const float* bias_in, float* bias_out, cudaStream_t st) {
  bias_update_kernel<<<1, kThreads, 0, st>>>(counts, bias_in, bias_out, s.E,
                                             (int64_t)s.T * s.k, gamma);
  return cudaGetLastError();
}

}  // namespace moe
