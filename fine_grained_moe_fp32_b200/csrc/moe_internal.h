// Host-side declarations shared by the translation units of the library.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

// Device-side error codes written into the per-device status word (the first
// non-zero code wins; the host maps them to the public MOE_ERR_* values).
enum DevStatus : unsigned int {
  DEV_OK = 0,
  DEV_BAD_EXPERT_ID = 1,
  DEV_TIMEOUT = 2,
  DEV_BAD_EP_LAYOUT = 3,  // expert-parallel counts inconsistent or over capacity
  DEV_BOUNDS = 4,         // a MOE_CHECKS bounds check failed (the access was skipped)
};

// Bytes of the guard zone after every workspace region (and at the end of
// every workspace) in the MOE_CHECKS build: the library never writes them,
// so a caller that fills the workspace with a pattern can detect overruns.
#ifdef MOE_CHECKS
constexpr size_t kGuardBytes = 256;
#else
constexpr size_t kGuardBytes = 0;
#endif

// MOE_CHECKS build: point every translation unit's copy of the status
// pointer at the device status word (checks.cuh); a no-op otherwise.
cudaError_t checks_init_all(unsigned int* status);
#ifdef MOE_CHECKS
cudaError_t checks_init_grouped_gemm(unsigned int* status);
cudaError_t checks_init_grouped_gemm_pair(unsigned int* status);
cudaError_t checks_init_grouped_gemm_bwd(unsigned int* status);
cudaError_t checks_init_grouped_gemm_bwd_pair(unsigned int* status);
cudaError_t checks_init_permute(unsigned int* status);
cudaError_t checks_init_combine(unsigned int* status);
cudaError_t checks_init_backward(unsigned int* status);
#endif

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

struct Shape {
  int T, d, E, k, I, S, align;
  int64_t cap;  // T*k + E*(align-1)
};

// ---- router (router.cu)
constexpr int kRouterBT = 128;  // tokens per CTA tile
constexpr int kRouterBK = 16;   // k-chunk staged in shared memory
int router_splits(const Shape& s, int num_sms);
size_t router_partials_bytes(const Shape& s, int num_sms);
cudaError_t launch_router(const Shape& s, const uint16_t* x, const float* w_gate,
                          const float* bias, float* probs, int32_t* topk_idx, float* topk_w,
                          float* partials, int num_sms, cudaStream_t st);

// ---- permutation (permute.cu)
constexpr int kChunkTokens = 256;  // tokens per CTA in the count / scatter kernels
size_t permute_scratch_bytes(const Shape& s);
cudaError_t launch_permute(const Shape& s, const int32_t* topk_idx, const uint16_t* x,
                           int32_t* counts, int32_t* offsets, int32_t* row_of,
                           int32_t* token_of_row, uint16_t* x_perm, void* scratch,
                           unsigned int* status, cudaStream_t st);

// ---- grouped GEMMs (grouped_gemm.cu)
struct GroupedGemmArgs {
  // routed experts
  const uint16_t* x_perm;  // [cap, d]
  const int32_t* offsets;  // [E+1]
  const uint16_t *w1, *w3, *w2;
  uint16_t* h_perm;  // [cap, I]
  void* y_perm;      // [cap, d] fp32, or bf16 when !y_perm_f32 (the dense FFN's y)
  bool y_perm_f32 = true;
  // which groups a launch covers: both, the routed experts only, or the
  // shared experts only (the shared ones do not depend on the routing, so
  // they can run while the router and the permutation do)
  enum Part : int { kAll = 0, kRoutedOnly = 1, kSharedOnly = 2 };
  int part = kAll;
  // dense FFN at small T: the down GEMM split over K into down_splits fp32
  // partials [down_splits, cap, d] (down_partials), summed into the bf16 y
  int down_splits = 1;
  float* down_partials = nullptr;
  // dense FFN at small T: the gate/up GEMM split over K into up_splits fp32
  // partials [up_splits, 2 (g, u), cap, I] (up_partials), summed in order
  // before the SwiGLU (it is not linear); may share down_partials' memory
  int up_splits = 1;
  float* up_partials = nullptr;
  // shared experts (S > 0 and all non-null to enable)
  const uint16_t* x;  // [T, d]
  const uint16_t *ws1, *ws3, *ws2;
  uint16_t* h_shared;  // [T, S*I]
  float* y_shared;     // [T, d]
  // training: pre-activations of the gate/up GEMM, fp32 (null = not stored)
  float* g_perm = nullptr;    // [cap, I]
  float* u_perm = nullptr;    // [cap, I]
  float* g_shared = nullptr;  // [T, S*I]
  float* u_shared = nullptr;  // [T, S*I]
};
// `between` (may be null) is recorded on `st` after the gate/up GEMM is launched.
cudaError_t launch_grouped_gemms(const Shape& s, const GroupedGemmArgs& a, int num_sms,
                                 unsigned int* status, uint64_t wait_limit_ns, cudaStream_t st,
                                 cudaEvent_t between = nullptr);

// true when launch_grouped_gemms runs the paired-CTA kernels (prefill-sized
// segments) for this shape
bool uses_pair_gemms(const Shape& s);

// ---- paired-CTA grouped GEMMs for prefill-sized segments (grouped_gemm_pair.cu)
bool pair_gemms_supported(const Shape& s);
// K splits of the dense FFN's down GEMM (one group, no shared experts) when
// its tiles alone cannot fill the SM pairs; 1 otherwise
int down_k_splits(const Shape& s, int num_sms);
int up_k_splits(const Shape& s, int num_sms);
cudaError_t launch_grouped_gemms_pair(const Shape& s, const GroupedGemmArgs& a, int num_sms,
                                      unsigned int* status, uint64_t wait_limit_ns,
                                      cudaStream_t st, cudaEvent_t between);

// ---- backward grouped GEMMs (grouped_gemm_bwd.cu)
struct BackwardGemmArgs {
  const int32_t* offsets;
  const uint16_t *w1, *w3, *w2, *ws1, *ws3, *ws2;
  const uint16_t *x, *x_perm;                             // forward inputs
  const uint16_t *h_perm, *h_shared;                      // forward activations
  const float *g_perm, *u_perm, *g_shared, *u_shared;     // saved pre-activations (fp32)
  const uint16_t *dy, *dy_perm;  // upstream gradient: per token, and w * dy per segment row
  uint16_t* dgu_perm;    // [cap, 2I]  [dG | dU]
  uint16_t* dgu_shared;  // [T, 2*S*I]
  float* dx_perm;        // [cap, d]
  float* dx_shared;      // [T, d]
  void *dw1, *dw3, *dw2, *dws1, *dws3, *dws2;  // bf16, or fp32 when dw_f32
  bool dw_f32 = false;
};
// `events` (may be null): 4 events recorded after the dH/SwiGLU dgrad, the dW2
// wgrad, the dX dgrad and the dW1/dW3 wgrads.
bool pair_backward_supported(const Shape& s);
cudaError_t launch_backward_gemms_pair(const Shape& s, const BackwardGemmArgs& a, int num_sms,
                                       unsigned int* status, uint64_t wait_ns, cudaStream_t st,
                                       const cudaEvent_t* events);
cudaError_t launch_backward_gemms(const Shape& s, const BackwardGemmArgs& a, int num_sms,
                                  unsigned int* status, uint64_t wait_ns, cudaStream_t st,
                                  const cudaEvent_t* events = nullptr);

// ---- backward outside the expert GEMMs (backward.cu)
struct BackwardMiscArgs {
  const uint16_t *x, *dy;
  const float* y_perm;  // [cap, d] routed expert outputs
  const float *w_gate, *probs, *topk_w;
  const int32_t *topk_idx, *row_of, *offsets, *token_of_row;
  uint16_t* dy_perm;    // [cap, d]
  float* dw;            // [T, k]
  float* dz;            // [T, E]
  const float* dx_perm;    // [cap, d]
  const float* dx_shared;  // [T, d] or null
  float* dx_router;     // [T, d]
  float* dwg_partials;  // [splits, E, d]
  float* dw_gate;       // [E, d]
  void* dx;             // [T, d] bf16, or fp32 when dx_f32
  bool dx_f32 = false;
};
int dwg_splits(const Shape& s);
cudaError_t launch_backward_misc_pre(const Shape& s, const BackwardMiscArgs& a, cudaStream_t st);
cudaError_t launch_backward_misc_post(const Shape& s, const BackwardMiscArgs& a, cudaStream_t st);

// ---- load balancing, training side (balance.cu)
size_t balance_workspace_bytes(const Shape& s, int seq_len);
cudaError_t launch_balance_stats(const Shape& s, int seq_len, const float* probs,
                                 const int32_t* topk_idx, float alpha, float* f, float* P,
                                 float* loss, void* workspace, unsigned int* status,
                                 cudaStream_t st);
cudaError_t launch_bias_update(const Shape& s, const int32_t* counts, float gamma,
                               const float* bias_in, float* bias_out, cudaStream_t st);

// ---- combine (combine.cu); routed expert outputs in fp32
cudaError_t launch_combine(const Shape& s, const float* y_perm, const int32_t* row_of,
                           const float* topk_w, const float* y_shared, uint16_t* y,
                           cudaStream_t st);
// expert parallel: rows pulled from the owners' receive buffers
// y_recv[idx / (E/world)] at remote_row (rows < cap; -1 = skipped)
cudaError_t launch_ep_combine(const Shape& s, int world, const float* const* y_recv,
                              const int32_t* topk_idx, const int32_t* remote_row, int64_t cap,
                              const float* topk_w, const float* y_shared, uint16_t* y,
                              cudaStream_t st);

// ---- expert parallelism (expert_parallel.cu)
// rows of a rank's receive buffer: world*T*k + (E/world)*(align-1)
int64_t ep_recv_capacity(const Shape& s, int world);
cudaError_t launch_ep_dispatch(const Shape& s, int world, int rank, const uint16_t* x,
                               const int32_t* topk_idx, const int32_t* row_of,
                               const int32_t* offsets, const int32_t* counts,
                               const int32_t* const* counts_of, uint16_t* const* x_recv,
                               int32_t* dst_row, int32_t* recv_offsets, int32_t* recv_counts,
                               int32_t* remote_row, unsigned int* status, cudaStream_t st);

}  // namespace moe
