// C ABI of the library: argument checks, workspace layout and the launch
// sequence of every entry point declared in include/moe_b200.h.
#include <cstdint>
#include <cstring>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>
#include <mutex>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace moe {
namespace {

// First device-side error since the last moe_get_last_device_status().
__device__ unsigned int g_device_status = 0;

constexpr int kMaxDevices = 64;
constexpr int kPlanSMs = 148;  // split-K planning of the router is device independent
constexpr uint64_t kDefaultWaitNs = 1000000000ull;
uint64_t g_wait_limit_ns = kDefaultWaitNs;
constexpr int kFwdEvents = 6, kAllEvents = 13;
cudaEvent_t g_phase_events[kAllEvents] = {};
bool g_phase_on = false;       // forward events set
bool g_bwd_phase_on = false;   // backward events set too

// A null entry of the event list is a point the caller does not time.
cudaError_t phase(int i, cudaStream_t st) {
  return g_phase_on && g_phase_events[i] != nullptr ? cudaEventRecord(g_phase_events[i], st)
                                                     : cudaSuccess;
}

cudaError_t bwd_phase(int i, cudaStream_t st) {
  cudaEvent_t e = g_phase_events[kFwdEvents + i];
  return g_bwd_phase_on && e != nullptr ? cudaEventRecord(e, st) : cudaSuccess;
}

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  unsigned int* status = nullptr;
  // inference forward: the shared experts' GEMMs run on `side` beside the
  // router and the permutation on the caller's stream (fork, join)
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
std::mutex g_fork_mu;  // one fork/join sequence at a time (the events are per device)

}  // namespace

cudaError_t checks_init_all(unsigned int* status) {
#ifdef MOE_CHECKS
  cudaError_t e;
  if ((e = checks_init_grouped_gemm(status)) != cudaSuccess ||
      (e = checks_init_grouped_gemm_pair(status)) != cudaSuccess ||
      (e = checks_init_grouped_gemm_bwd(status)) != cudaSuccess ||
      (e = checks_init_grouped_gemm_bwd_pair(status)) != cudaSuccess ||
      (e = checks_init_permute(status)) != cudaSuccess ||
      (e = checks_init_combine(status)) != cudaSuccess ||
      (e = checks_init_backward(status)) != cudaSuccess)
    return e;
#else
  (void)status;
#endif
  return cudaSuccess;
}

namespace {

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return nullptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    d.status = static_cast<unsigned int*>(p);
    if (checks_init_all(d.status) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithFlags(&d.side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&d.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&d.join, cudaEventDisableTiming) != cudaSuccess) {
      // leave nothing half made: the next call starts over
      if (d.join != nullptr) cudaEventDestroy(d.join);
      if (d.fork != nullptr) cudaEventDestroy(d.fork);
      if (d.side != nullptr) cudaStreamDestroy(d.side);
      d.side = nullptr;
      d.fork = d.join = nullptr;
      return nullptr;
    }
    d.ready = true;
  }
  return &d;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Host-side NVTX range around one phase of a call (visible in Nsight
// timelines; a no-op unless a tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Consecutive phase ranges inside a call: next() closes the open one.
struct NvtxPhases {
  bool open = false;
  void next(const char* name) {
    if (open) nvtxRangePop();
    nvtxRangePushA(name);
    open = true;
  }
  ~NvtxPhases() {
    if (open) nvtxRangePop();
  }
};

int check_dims(const moe_dims* dims, Shape* s) {
  if (dims == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_dims& m = *dims;
  if (m.T < 0 || m.d <= 0 || m.E <= 0 || m.k <= 0 || m.I <= 0 || m.n_shared < 0 || m.align <= 0)
    return MOE_ERR_INVALID_ARG;
  if (m.E > 128 || m.k > m.E || m.k > 8 || m.d % 128 != 0 || m.I % 64 != 0 || m.align % 16 != 0 ||
      m.n_shared > 4)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const int64_t cap = (int64_t)m.T * m.k + (int64_t)m.E * (m.align - 1);
  if (cap >= (int64_t)INT32_MAX / 2 || (int64_t)m.T * m.k >= INT32_MAX / 2)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  *s = Shape{m.T, m.d, m.E, m.k, m.I, m.n_shared, m.align, cap};
  return MOE_OK;
}

size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

// Bytes a workspace region takes: its size rounded up to 256, plus the
// MOE_CHECKS build's guard zone (kGuardBytes, 0 otherwise).
size_t region(size_t b) { return al256(b) + kGuardBytes; }

moe_ws_layout make_layout(const Shape& s) {
  moe_ws_layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += region(bytes);
    return at;
  };
  L.route_partials = take(router_partials_bytes(s, kPlanSMs));
  L.probs = take((size_t)s.T * s.E * 4);
  L.topk_idx = take((size_t)s.T * s.k * 4);
  L.topk_w = take((size_t)s.T * s.k * 4);
  L.counts = take((size_t)s.E * 4);
  L.offsets = take((size_t)(s.E + 1) * 4);
  L.row_of = take((size_t)s.T * s.k * 4);
  L.token_of_row = take((size_t)s.cap * 4);
  L.permute_scratch = take(permute_scratch_bytes(s));
  L.x_perm = take((size_t)s.cap * s.d * 2);
  L.h_perm = take((size_t)s.cap * s.I * 2);
  L.y_perm = take((size_t)s.cap * s.d * 4);
  L.h_shared = take((size_t)s.T * s.S * s.I * 2);
  L.y_shared = take((size_t)s.T * s.d * 4);
  L.total = off;
  return L;
}

moe_train_layout make_train_layout(const Shape& s) {
  moe_train_layout L{};
  L.fwd = make_layout(s);
  size_t off = L.fwd.total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += region(bytes);
    return at;
  };
  const size_t SI = (size_t)s.S * s.I;
  L.g_perm = take((size_t)s.cap * s.I * 4);
  L.u_perm = take((size_t)s.cap * s.I * 4);
  L.g_shared = take((size_t)s.T * SI * 4);
  L.u_shared = take((size_t)s.T * SI * 4);
  L.dy_perm = take((size_t)s.cap * s.d * 2);
  L.dw = take((size_t)s.T * s.k * 4);
  L.dz = take((size_t)s.T * s.E * 4);
  L.dgu_perm = take((size_t)s.cap * 2 * s.I * 2);
  L.dgu_shared = take((size_t)s.T * 2 * SI * 2);
  L.dx_perm = take((size_t)s.cap * s.d * 4);
  L.dx_shared = take((size_t)s.T * s.d * 4);
  L.dx_router = take((size_t)s.T * s.d * 4);
  L.dwg_partials = take((size_t)dwg_splits(s) * s.E * s.d * 4);
  L.total = off;
  return L;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int64_t moe_capacity(const moe_dims* dims) {
  Shape s;
  if (check_dims(dims, &s) != MOE_OK) return 0;
  return s.cap;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "a bounded device wait ran out";
    case MOE_ERR_BOUNDS: return "a device-side bounds check failed (checks build)";
    default: return "unknown status";
  }
}

size_t moe_route_workspace_size(const moe_dims* dims) {
  Shape s;
  if (check_dims(dims, &s) != MOE_OK) return 0;
  return region(router_partials_bytes(s, kPlanSMs));
}

int moe_route(const moe_dims* dims, const moe_bf16* x, const float* w_gate, const float* bias,
              float* probs, int32_t* topk_idx, float* topk_w, void* workspace,
              size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (s.T == 0) return MOE_OK;
  if (x == nullptr || w_gate == nullptr || topk_idx == nullptr || topk_w == nullptr ||
      !aligned(x, 16) || !aligned(w_gate, 16))
    return MOE_ERR_INVALID_ARG;
  const size_t need = router_partials_bytes(s, kPlanSMs);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  if (device_info() == nullptr) return MOE_ERR_CUDA;
  return cuda_status(launch_router(s, x, w_gate, bias, probs, topk_idx, topk_w,
                                   static_cast<float*>(workspace), kPlanSMs,
                                   static_cast<cudaStream_t>(stream)));
}

size_t moe_permute_workspace_size(const moe_dims* dims) {
  Shape s;
  if (check_dims(dims, &s) != MOE_OK) return 0;
  return region(permute_scratch_bytes(s));
}

int moe_permute(const moe_dims* dims, const int32_t* topk_idx, const moe_bf16* x, int32_t* counts,
                int32_t* offsets, int32_t* row_of, int32_t* token_of_row, moe_bf16* x_perm,
                void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (counts == nullptr || offsets == nullptr || token_of_row == nullptr || x_perm == nullptr ||
      (s.T > 0 && (topk_idx == nullptr || x == nullptr || row_of == nullptr)) ||
      !aligned(x, 16) || !aligned(x_perm, 16))
    return MOE_ERR_INVALID_ARG;
  const size_t need = permute_scratch_bytes(s);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)))
    return MOE_ERR_WORKSPACE;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  return cuda_status(launch_permute(s, topk_idx, x, counts, offsets, row_of, token_of_row, x_perm,
                                    workspace, di->status, static_cast<cudaStream_t>(stream)));
}

int moe_grouped_swiglu(const moe_dims* dims, const moe_bf16* x_perm, const int32_t* offsets,
                       const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                       moe_bf16* h_perm, float* y_perm, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (x_perm == nullptr || offsets == nullptr || w1 == nullptr || w3 == nullptr || w2 == nullptr ||
      h_perm == nullptr || y_perm == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x_perm, 16) || !aligned(w1, 16) || !aligned(w3, 16) || !aligned(w2, 16) ||
      !aligned(h_perm, 16) || !aligned(y_perm, 16))
    return MOE_ERR_INVALID_ARG;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  GroupedGemmArgs a{};
  a.x_perm = x_perm;
  a.offsets = offsets;
  a.w1 = w1;
  a.w3 = w3;
  a.w2 = w2;
  a.h_perm = h_perm;
  a.y_perm = y_perm;
  return cuda_status(launch_grouped_gemms(s, a, di->num_sms, di->status, g_wait_limit_ns,
                                          static_cast<cudaStream_t>(stream)));
}

int moe_combine(const moe_dims* dims, const float* y_perm, const int32_t* row_of,
                const float* topk_w, const float* y_shared, moe_bf16* y, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (s.T == 0) return MOE_OK;
  if (y_perm == nullptr || row_of == nullptr || topk_w == nullptr || y == nullptr ||
      !aligned(y_perm, 16) || !aligned(y, 16) || (y_shared != nullptr && !aligned(y_shared, 16)))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_combine(s, y_perm, row_of, topk_w, y_shared, y,
                                    static_cast<cudaStream_t>(stream)));
}

size_t moe_workspace_size(const moe_dims* dims) {
  Shape s;
  if (check_dims(dims, &s) != MOE_OK) return 0;
  return make_layout(s).total;
}

int moe_forward_layout(const moe_dims* dims, moe_ws_layout* layout) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  *layout = make_layout(s);
  return MOE_OK;
}

}  // extern "C"

namespace moe {
namespace {

// The fused forward; with `train` it also stores the gate/up pre-activations.
int forward_impl(const moe_dims* dims, const moe_bf16* x, const float* w_gate, const float* bias,
                 const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2, const moe_bf16* ws1,
                 const moe_bf16* ws3, const moe_bf16* ws2, moe_bf16* y, void* workspace,
                 size_t workspace_bytes, void* stream, bool train) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (w_gate == nullptr || w1 == nullptr || w3 == nullptr || w2 == nullptr ||
      (s.T > 0 && (x == nullptr || y == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (s.S > 0 && (ws1 == nullptr || ws3 == nullptr || ws2 == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_gate, 16) || !aligned(w1, 16) || !aligned(w3, 16) ||
      !aligned(w2, 16) || !aligned(y, 16) || !aligned(ws1, 16) || !aligned(ws3, 16) ||
      !aligned(ws2, 16))
    return MOE_ERR_INVALID_ARG;
  const moe_train_layout TL = make_train_layout(s);
  const moe_ws_layout& L = TL.fwd;
  const size_t need = train ? TL.total : L.total;
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = workspace;

  float* probs = at<float>(ws, L.probs);
  int32_t* idx = at<int32_t>(ws, L.topk_idx);
  float* wts = at<float>(ws, L.topk_w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  int32_t* tor = at<int32_t>(ws, L.token_of_row);
  uint16_t* x_perm = at<uint16_t>(ws, L.x_perm);
  uint16_t* h_perm = at<uint16_t>(ws, L.h_perm);
  float* y_perm = at<float>(ws, L.y_perm);
  uint16_t* h_sh = at<uint16_t>(ws, L.h_shared);
  float* y_sh = at<float>(ws, L.y_shared);

  GroupedGemmArgs a{};
  a.x_perm = x_perm;
  a.offsets = offsets;
  a.w1 = w1;
  a.w3 = w3;
  a.w2 = w2;
  a.h_perm = h_perm;
  a.y_perm = y_perm;
  if (s.S > 0) {
    a.x = x;
    a.ws1 = ws1;
    a.ws3 = ws3;
    a.ws2 = ws2;
    a.h_shared = h_sh;
    a.y_shared = y_sh;
  }
  if (train) {
    a.g_perm = at<float>(ws, TL.g_perm);
    a.u_perm = at<float>(ws, TL.u_perm);
    a.g_shared = at<float>(ws, TL.g_shared);
    a.u_shared = at<float>(ws, TL.u_shared);
  }
  // The shared experts' GEMMs do not depend on the routing, so the inference
  // forward runs them on the library's side stream and the caller's stream
  // waits for them (one event) before the combine.
  //  * Prefill-sized batches: launched after the router, before the
  //    permutation, on every SM: their CTAs are resident first and the
  //    permutation's HBM-bound row copy runs beside those compute-bound
  //    GEMMs.  Same-box A/B against one stream: 2.6 % faster at T = 4096,
  //    1.3 % at 16384; the training forward (which also stores g and u) was
  //    1.2 % slower, so it keeps one stream.
  //  * Decode-sized batches: launched before the router on two thirds of the
  //    SMs, so the shared weights stream while the latency-bound router and
  //    permutation run on the rest.  With T = 128 the shared gate/up GEMM has
  //    88 tiles: on half of the SMs it took two waves and held SMs into the
  //    routed gate/up GEMM (same-box A/B, per step: 74 CTAs 0.923-0.930 ms,
  //    100 CTAs 0.915-0.919, 112 CTAs 0.919-0.921, 148 CTAs 0.921-0.923).
  const bool pair = uses_pair_gemms(s);
  const bool split = !train && s.S > 0 && s.T > 0;
  std::unique_lock<std::mutex> fork_lock(g_fork_mu, std::defer_lock);
  NvtxRange call(train ? "moe_forward_train" : "moe_forward");
  NvtxPhases ph;
  cudaError_t e = cudaSuccess;
  bool forked = false;
  auto fork_shared = [&](int ctas) {
    ph.next("shared_experts (side stream)");
    fork_lock.lock();
    GroupedGemmArgs sh = a;
    sh.part = GroupedGemmArgs::kSharedOnly;
    if ((e = cudaEventRecord(di->fork, st)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(di->side, di->fork, 0)) != cudaSuccess)
      return false;
    forked = true;
    e = launch_grouped_gemms(s, sh, ctas, di->status, g_wait_limit_ns, di->side);
    // recorded whatever the launch did, so the caller's stream can always be
    // ordered after the side stream's work
    const cudaError_t ej = cudaEventRecord(di->join, di->side);
    if (e == cudaSuccess) e = ej;
    if (e != cudaSuccess) return false;
    a.part = GroupedGemmArgs::kRoutedOnly;
    return true;
  };
  // an error after the fork still orders the caller's stream after the side
  // stream's kernels, which write the caller's workspace
  auto fail = [&]() {
    if (forked) cudaStreamWaitEvent(st, di->join, 0);
    return MOE_ERR_CUDA;
  };
  if ((e = phase(0, st)) != cudaSuccess) return MOE_ERR_CUDA;
  if (split && !pair && !fork_shared(di->num_sms * 2 / 3)) return fail();
  ph.next("router");
  e = launch_router(s, x, w_gate, bias, probs, idx, wts, at<float>(ws, L.route_partials),
                    kPlanSMs, st);
  if (e == cudaSuccess) e = phase(1, st);
  if (e != cudaSuccess) return fail();
  if (split && pair && !fork_shared(di->num_sms)) return fail();
  ph.next("permute");
  e = launch_permute(s, idx, x, counts, offsets, row_of, tor, x_perm,
                     at<void>(ws, L.permute_scratch), di->status, st);
  if (e == cudaSuccess) e = phase(2, st);
  if (e != cudaSuccess) return fail();
  ph.next("grouped_gemms");
  e = launch_grouped_gemms(s, a, di->num_sms, di->status, g_wait_limit_ns, st,
                           g_phase_on ? g_phase_events[3] : nullptr);
  if (e == cudaSuccess) e = phase(4, st);
  if (e != cudaSuccess) return fail();
  if (forked && (e = cudaStreamWaitEvent(st, di->join, 0)) != cudaSuccess) return MOE_ERR_CUDA;
  ph.next("combine");
  e = launch_combine(s, y_perm, row_of, wts, s.S > 0 ? y_sh : nullptr, y, st);
  if (e == cudaSuccess) e = phase(5, st);
  return cuda_status(e);
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_forward(const moe_dims* dims, const moe_bf16* x, const float* w_gate, const float* bias,
                const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2, const moe_bf16* ws1,
                const moe_bf16* ws3, const moe_bf16* ws2, moe_bf16* y, void* workspace,
                size_t workspace_bytes, void* stream) {
  return forward_impl(dims, x, w_gate, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace,
                      workspace_bytes, stream, false);
}

size_t moe_train_workspace_size(const moe_dims* dims) {
  Shape s;
  if (check_dims(dims, &s) != MOE_OK) return 0;
  return make_train_layout(s).total;
}

int moe_train_layout_of(const moe_dims* dims, moe_train_layout* layout) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  *layout = make_train_layout(s);
  return MOE_OK;
}

int moe_forward_train(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                      const float* bias, const moe_bf16* w1, const moe_bf16* w3,
                      const moe_bf16* w2, const moe_bf16* ws1, const moe_bf16* ws3,
                      const moe_bf16* ws2, moe_bf16* y, void* workspace, size_t workspace_bytes,
                      void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (s.I % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  return forward_impl(dims, x, w_gate, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace,
                      workspace_bytes, stream, true);
}

}  // extern "C"

namespace moe {
namespace {

// The backward; `f32` selects fp32 dx and weight gradients (else bf16).
int backward_impl(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                  const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                  const moe_bf16* ws1, const moe_bf16* ws3, const moe_bf16* ws2,
                  const moe_bf16* dy, void* workspace, size_t workspace_bytes, void* dx,
                  float* dw_gate, void* dw1, void* dw3, void* dw2, void* dws1, void* dws3,
                  void* dws2, void* stream, bool f32) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (s.I % 128 != 0 || s.E % 4 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (w_gate == nullptr || w1 == nullptr || w3 == nullptr || w2 == nullptr ||
      dw_gate == nullptr || dw1 == nullptr || dw3 == nullptr || dw2 == nullptr ||
      (s.T > 0 && (x == nullptr || dy == nullptr || dx == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (s.S > 0 && (ws1 == nullptr || ws3 == nullptr || ws2 == nullptr || dws1 == nullptr ||
                  dws3 == nullptr || dws2 == nullptr))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_gate, w1, w3, w2, ws1, ws3, ws2, dy, dx, dw_gate,
                        dw1, dw3, dw2, dws1, dws3, dws2};
  for (const void* q : ptrs)
    if (!aligned(q, 16)) return MOE_ERR_INVALID_ARG;
  const moe_train_layout TL = make_train_layout(s);
  if (workspace == nullptr || workspace_bytes < TL.total || !aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  const moe_ws_layout& L = TL.fwd;

  BackwardMiscArgs m{};
  m.x = x;
  m.dy = dy;
  m.y_perm = at<float>(ws, L.y_perm);
  m.w_gate = w_gate;
  m.probs = at<float>(ws, L.probs);
  m.topk_w = at<float>(ws, L.topk_w);
  m.topk_idx = at<int32_t>(ws, L.topk_idx);
  m.row_of = at<int32_t>(ws, L.row_of);
  m.offsets = at<int32_t>(ws, L.offsets);
  m.token_of_row = at<int32_t>(ws, L.token_of_row);
  m.dy_perm = at<uint16_t>(ws, TL.dy_perm);
  m.dw = at<float>(ws, TL.dw);
  m.dz = at<float>(ws, TL.dz);
  m.dx_perm = at<float>(ws, TL.dx_perm);
  m.dx_shared = s.S > 0 ? at<float>(ws, TL.dx_shared) : nullptr;
  m.dx_router = at<float>(ws, TL.dx_router);
  m.dwg_partials = at<float>(ws, TL.dwg_partials);
  m.dw_gate = dw_gate;
  m.dx = dx;
  m.dx_f32 = f32;
  NvtxRange call("moe_backward");
  NvtxPhases ph;
  ph.next("combine_router_bwd");
  cudaError_t e = bwd_phase(0, st);
  if (e == cudaSuccess) e = launch_backward_misc_pre(s, m, st);
  if (e == cudaSuccess) e = bwd_phase(1, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;

  BackwardGemmArgs g{};
  g.offsets = m.offsets;
  g.w1 = w1;
  g.w3 = w3;
  g.w2 = w2;
  g.ws1 = ws1;
  g.ws3 = ws3;
  g.ws2 = ws2;
  g.x = x;
  g.x_perm = at<uint16_t>(ws, L.x_perm);
  g.h_perm = at<uint16_t>(ws, L.h_perm);
  g.h_shared = at<uint16_t>(ws, L.h_shared);
  g.g_perm = at<float>(ws, TL.g_perm);
  g.u_perm = at<float>(ws, TL.u_perm);
  g.g_shared = at<float>(ws, TL.g_shared);
  g.u_shared = at<float>(ws, TL.u_shared);
  g.dy = dy;
  g.dy_perm = m.dy_perm;
  g.dgu_perm = at<uint16_t>(ws, TL.dgu_perm);
  g.dgu_shared = at<uint16_t>(ws, TL.dgu_shared);
  g.dx_perm = at<float>(ws, TL.dx_perm);
  g.dx_shared = at<float>(ws, TL.dx_shared);
  g.dw1 = dw1;
  g.dw3 = dw3;
  g.dw2 = dw2;
  g.dws1 = dws1;
  g.dws3 = dws3;
  g.dws2 = dws2;
  g.dw_f32 = f32;
  ph.next("grouped_gemms_bwd");
  e = launch_backward_gemms(s, g, di->num_sms, di->status, g_wait_limit_ns, st,
                            g_bwd_phase_on ? &g_phase_events[kFwdEvents + 2] : nullptr);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  ph.next("gate_gemms_unpermute");
  e = launch_backward_misc_post(s, m, st);
  if (e == cudaSuccess) e = bwd_phase(6, st);
  return cuda_status(e);
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_backward(const moe_dims* dims, const moe_bf16* x, const float* w_gate, const moe_bf16* w1,
                 const moe_bf16* w3, const moe_bf16* w2, const moe_bf16* ws1, const moe_bf16* ws3,
                 const moe_bf16* ws2, const moe_bf16* dy, void* workspace, size_t workspace_bytes,
                 moe_bf16* dx, float* dw_gate, moe_bf16* dw1, moe_bf16* dw3, moe_bf16* dw2,
                 moe_bf16* dws1, moe_bf16* dws3, moe_bf16* dws2, void* stream) {
  return backward_impl(dims, x, w_gate, w1, w3, w2, ws1, ws3, ws2, dy, workspace,
                       workspace_bytes, dx, dw_gate, dw1, dw3, dw2, dws1, dws3, dws2, stream,
                       false);
}

int moe_backward_f32(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                     const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                     const moe_bf16* ws1, const moe_bf16* ws3, const moe_bf16* ws2,
                     const moe_bf16* dy, void* workspace, size_t workspace_bytes, float* dx,
                     float* dw_gate, float* dw1, float* dw3, float* dw2, float* dws1,
                     float* dws3, float* dws2, void* stream) {
  return backward_impl(dims, x, w_gate, w1, w3, w2, ws1, ws3, ws2, dy, workspace,
                       workspace_bytes, dx, dw_gate, dw1, dw3, dw2, dws1, dws3, dws2, stream,
                       true);
}

}  // extern "C"

namespace moe {
namespace {

// The dense FFN runs the grouped GEMMs as one group holding every token.
__global__ void dense_offsets_kernel(int32_t* offsets, int T) {
  offsets[0] = 0;
  offsets[1] = T;
}

int dense_shape(const moe_dims* dims, Shape* s) {
  if (dims == nullptr || dims->T < 0 || dims->d <= 0 || dims->I <= 0) return MOE_ERR_INVALID_ARG;
  if (dims->d % 128 != 0 || dims->I % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)dims->T * dims->I >= INT32_MAX / 2 || (int64_t)dims->T * dims->d >= INT32_MAX / 2)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  // capacity = T: the token operand is x itself, and its tensor map must not
  // claim rows past the caller's T (tiles read zeros beyond it)
  *s = Shape{dims->T, dims->d, 1, 1, dims->I, 0, 16, (int64_t)dims->T};
  return MOE_OK;
}

size_t dense_h_offset() { return al256(2 * sizeof(int32_t)); }

// fp32 K-split partials of the down GEMM after h (none when it is not split)
size_t dense_partials_offset(const Shape& s) {
  return dense_h_offset() + region((size_t)s.T * s.I * 2);
}
// (the gate/up GEMM's K-split partials use the same memory first)
size_t dense_partials_bytes(const Shape& s) {
  const int sd = down_k_splits(s, kPlanSMs), su = up_k_splits(s, kPlanSMs);
  const size_t down = sd > 1 ? (size_t)sd * s.T * s.d * 4 : 0;
  const size_t up = su > 1 ? (size_t)su * 2 * s.T * s.I * 4 : 0;
  return down > 0 || up > 0 ? region(std::max(down, up)) : 0;
}

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_dense_workspace_size(const moe_dims* dims) {
  Shape s;
  if (dense_shape(dims, &s) != MOE_OK) return 0;
  return dense_partials_offset(s) + dense_partials_bytes(s);
}

int moe_dense_swiglu(const moe_dims* dims, const moe_bf16* x, const moe_bf16* w1,
                     const moe_bf16* w3, const moe_bf16* w2, moe_bf16* y, void* workspace,
                     size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = dense_shape(dims, &s);
  if (rc != MOE_OK) return rc;
  if (s.T == 0) return MOE_OK;
  if (x == nullptr || w1 == nullptr || w3 == nullptr || w2 == nullptr || y == nullptr ||
      !aligned(x, 16) || !aligned(w1, 16) || !aligned(w3, 16) || !aligned(w2, 16) ||
      !aligned(y, 16))
    return MOE_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned(workspace, 256) ||
      workspace_bytes < moe_dense_workspace_size(dims))
    return MOE_ERR_WORKSPACE;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* offsets = at<int32_t>(workspace, 0);
  dense_offsets_kernel<<<1, 1, 0, st>>>(offsets, s.T);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  GroupedGemmArgs a{};
  a.x_perm = x;
  a.offsets = offsets;
  a.w1 = w1;
  a.w3 = w3;
  a.w2 = w2;
  a.h_perm = at<uint16_t>(workspace, dense_h_offset());
  a.y_perm = y;
  a.y_perm_f32 = false;  // the dense FFN's output is the caller's bf16 y
  a.down_splits = down_k_splits(s, kPlanSMs);
  if (a.down_splits > 1) a.down_partials = at<float>(workspace, dense_partials_offset(s));
  a.up_splits = up_k_splits(s, kPlanSMs);
  if (a.up_splits > 1) a.up_partials = at<float>(workspace, dense_partials_offset(s));
  return cuda_status(
      launch_grouped_gemms(s, a, di->num_sms, di->status, g_wait_limit_ns, st, nullptr));
}

size_t moe_balance_workspace_size(const moe_dims* dims, int seq_len) {
  Shape s;
  if (check_dims(dims, &s) != MOE_OK || seq_len <= 0 || s.T % seq_len != 0) return 0;
  return balance_workspace_bytes(s, seq_len);
}

int moe_balance_stats(const moe_dims* dims, int seq_len, const float* probs,
                      const int32_t* topk_idx, float alpha, float* f, float* P, float* loss,
                      void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (seq_len <= 0 || s.T % seq_len != 0 || loss == nullptr) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (probs == nullptr || topk_idx == nullptr || f == nullptr || P == nullptr ||
                  workspace == nullptr || !aligned(workspace, 256)))
    return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && workspace_bytes < balance_workspace_bytes(s, seq_len)) return MOE_ERR_WORKSPACE;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  return cuda_status(launch_balance_stats(s, seq_len, probs, topk_idx, alpha, f, P, loss,
                                          workspace, di->status,
                                          static_cast<cudaStream_t>(stream)));
}

int moe_bias_update(const moe_dims* dims, const int32_t* counts, float gamma,
                    const float* bias_in, float* bias_out, void* stream) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != MOE_OK) return rc;
  if (counts == nullptr || bias_in == nullptr || bias_out == nullptr) return MOE_ERR_INVALID_ARG;
  return cuda_status(
      launch_bias_update(s, counts, gamma, bias_in, bias_out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace moe {
namespace {

// Expert parallelism: the rank's own shape plus the receive capacity.
int check_ep(const moe_dims* dims, int world, Shape* s, int64_t* rcap) {
  int rc = check_dims(dims, s);
  if (rc != MOE_OK) return rc;
  if (world <= 0 || world > s->E || s->E % world != 0) return MOE_ERR_INVALID_ARG;
  *rcap = ep_recv_capacity(*s, world);
  if (*rcap >= (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_ep_layout make_ep_layout(const Shape& s, int world, int64_t rcap) {
  moe_ep_layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += region(bytes);
    return at;
  };
  const int El = s.E / world;
  L.route_partials = take(router_partials_bytes(s, kPlanSMs));
  L.probs = take((size_t)s.T * s.E * 4);
  L.topk_idx = take((size_t)s.T * s.k * 4);
  L.topk_w = take((size_t)s.T * s.k * 4);
  L.counts = take((size_t)s.E * 4);
  L.offsets = take((size_t)(s.E + 1) * 4);
  L.row_of = take((size_t)s.T * s.k * 4);
  L.token_of_row = take((size_t)s.cap * 4);
  L.permute_scratch = take(permute_scratch_bytes(s));
  L.dst_row = take((size_t)s.E * 4);
  L.recv_offsets = take((size_t)(El + 1) * 4);
  L.recv_counts = take((size_t)El * 4);
  L.remote_row = take((size_t)s.T * s.k * 4);
  L.h_recv = take((size_t)rcap * s.I * 2);
  L.h_shared = take((size_t)s.T * s.S * s.I * 2);
  L.y_shared = take((size_t)s.T * s.d * 4);
  L.total = off;
  return L;
}

// Shared prologue of the EP entries: shape and workspace checks.
int ep_prologue(const moe_dims* dims, int world, void* workspace, size_t workspace_bytes,
                Shape* s, int64_t* rcap, moe_ep_layout* L) {
  int rc = check_ep(dims, world, s, rcap);
  if (rc != MOE_OK) return rc;
  *L = make_ep_layout(*s, world, *rcap);
  if (workspace == nullptr || workspace_bytes < L->total || !aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" {

int64_t moe_ep_recv_capacity(const moe_dims* dims, int world) {
  Shape s;
  int64_t rcap = 0;
  return check_ep(dims, world, &s, &rcap) == MOE_OK ? rcap : 0;
}

size_t moe_ep_workspace_size(const moe_dims* dims, int world) {
  Shape s;
  int64_t rcap = 0;
  if (check_ep(dims, world, &s, &rcap) != MOE_OK) return 0;
  return make_ep_layout(s, world, rcap).total;
}

int moe_ep_layout_of(const moe_dims* dims, int world, moe_ep_layout* layout) {
  Shape s;
  int64_t rcap = 0;
  int rc = check_ep(dims, world, &s, &rcap);
  if (rc != MOE_OK) return rc;
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  *layout = make_ep_layout(s, world, rcap);
  return MOE_OK;
}

int moe_ep_route(const moe_dims* dims, int world, const moe_bf16* x, const float* w_gate,
                 const float* bias, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int64_t rcap;
  moe_ep_layout L;
  int rc = ep_prologue(dims, world, workspace, workspace_bytes, &s, &rcap, &L);
  if (rc != MOE_OK) return rc;
  if (w_gate == nullptr || (s.T > 0 && x == nullptr) || !aligned(x, 16) || !aligned(w_gate, 16))
    return MOE_ERR_INVALID_ARG;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  cudaError_t e = launch_router(s, x, w_gate, bias, at<float>(ws, L.probs),
                                at<int32_t>(ws, L.topk_idx), at<float>(ws, L.topk_w),
                                at<float>(ws, L.route_partials), kPlanSMs, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_permute(s, at<int32_t>(ws, L.topk_idx), x, at<int32_t>(ws, L.counts),
                                    at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.row_of),
                                    at<int32_t>(ws, L.token_of_row), nullptr,
                                    at<void>(ws, L.permute_scratch), di->status, st));
}

int moe_ep_dispatch(const moe_dims* dims, int world, int rank, const moe_bf16* x,
                    const int32_t* const* counts_of, moe_bf16* const* x_recv, void* workspace,
                    size_t workspace_bytes, void* stream) {
  Shape s;
  int64_t rcap;
  moe_ep_layout L;
  int rc = ep_prologue(dims, world, workspace, workspace_bytes, &s, &rcap, &L);
  if (rc != MOE_OK) return rc;
  if (rank < 0 || rank >= world || counts_of == nullptr || x_recv == nullptr ||
      (s.T > 0 && x == nullptr) || !aligned(x, 16))
    return MOE_ERR_INVALID_ARG;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  void* ws = workspace;
  return cuda_status(launch_ep_dispatch(
      s, world, rank, x, at<int32_t>(ws, L.topk_idx), at<int32_t>(ws, L.row_of),
      at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.counts), counts_of, x_recv,
      at<int32_t>(ws, L.dst_row), at<int32_t>(ws, L.recv_offsets), at<int32_t>(ws, L.recv_counts),
      at<int32_t>(ws, L.remote_row), di->status, static_cast<cudaStream_t>(stream)));
}

int moe_ep_experts(const moe_dims* dims, int world, const moe_bf16* x, const moe_bf16* x_recv,
                   const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                   const moe_bf16* ws1, const moe_bf16* ws3, const moe_bf16* ws2,
                   float* y_recv, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int64_t rcap;
  moe_ep_layout L;
  int rc = ep_prologue(dims, world, workspace, workspace_bytes, &s, &rcap, &L);
  if (rc != MOE_OK) return rc;
  if (x_recv == nullptr || y_recv == nullptr || w1 == nullptr || w3 == nullptr ||
      w2 == nullptr || (s.T > 0 && s.S > 0 && x == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (s.S > 0 && (ws1 == nullptr || ws3 == nullptr || ws2 == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_recv, 16) || !aligned(y_recv, 16) || !aligned(w1, 16) ||
      !aligned(w3, 16) || !aligned(w2, 16) || !aligned(ws1, 16) || !aligned(ws3, 16) ||
      !aligned(ws2, 16))
    return MOE_ERR_INVALID_ARG;
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  // the local experts' grouped GEMMs: El groups over the receive buffer
  const Shape se{s.T, s.d, s.E / world, s.k, s.I, s.S, s.align, rcap};
  void* ws = workspace;
  GroupedGemmArgs a{};
  a.x_perm = x_recv;
  a.offsets = at<int32_t>(ws, L.recv_offsets);
  a.w1 = w1;
  a.w3 = w3;
  a.w2 = w2;
  a.h_perm = at<uint16_t>(ws, L.h_recv);
  a.y_perm = y_recv;
  if (s.S > 0) {
    a.x = x;
    a.ws1 = ws1;
    a.ws3 = ws3;
    a.ws2 = ws2;
    a.h_shared = at<uint16_t>(ws, L.h_shared);
    a.y_shared = at<float>(ws, L.y_shared);
  }
  return cuda_status(launch_grouped_gemms(se, a, di->num_sms, di->status, g_wait_limit_ns,
                                          static_cast<cudaStream_t>(stream)));
}

int moe_ep_combine(const moe_dims* dims, int world, const float* const* y_recv, moe_bf16* y,
                   void* workspace, size_t workspace_bytes, void* stream) {
  Shape s;
  int64_t rcap;
  moe_ep_layout L;
  int rc = ep_prologue(dims, world, workspace, workspace_bytes, &s, &rcap, &L);
  if (rc != MOE_OK) return rc;
  if (s.T == 0) return MOE_OK;
  if (y_recv == nullptr || y == nullptr || !aligned(y, 16)) return MOE_ERR_INVALID_ARG;
  if (device_info() == nullptr) return MOE_ERR_CUDA;
  void* ws = workspace;
  return cuda_status(launch_ep_combine(s, world, y_recv, at<int32_t>(ws, L.topk_idx),
                                       at<int32_t>(ws, L.remote_row), rcap,
                                       at<float>(ws, L.topk_w),
                                       s.S > 0 ? at<float>(ws, L.y_shared) : nullptr, y,
                                       static_cast<cudaStream_t>(stream)));
}

int moe_ipc_export(const void* ptr, void* handle, uint64_t* offset) {
  if (ptr == nullptr || handle == nullptr || offset == nullptr) return MOE_ERR_INVALID_ARG;
  static PFN_cuMemGetAddressRange_v3020 range = nullptr;
  if (range == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return MOE_ERR_CUDA;
    range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  }
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
    return MOE_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return MOE_ERR_CUDA;
  static_assert(sizeof(h) == 64, "IPC handle size");
  std::memcpy(handle, &h, sizeof(h));
  *offset = reinterpret_cast<uint64_t>(ptr) - static_cast<uint64_t>(base);
  return MOE_OK;
}

int moe_ipc_open(const void* handle, uint64_t offset, void** ptr) {
  if (handle == nullptr || ptr == nullptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
    return MOE_ERR_CUDA;
  *ptr = static_cast<char*>(base) + offset;
  return MOE_OK;
}

int moe_ipc_close(void* ptr, uint64_t offset) {
  if (ptr == nullptr) return MOE_ERR_INVALID_ARG;
  return cudaIpcCloseMemHandle(static_cast<char*>(ptr) - offset) == cudaSuccess ? MOE_OK
                                                                                 : MOE_ERR_CUDA;
}

int moe_get_last_device_status(void* stream) {
  const DeviceInfo* di = device_info();
  if (di == nullptr) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, di->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpy(di->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return MOE_ERR_CUDA;
  switch (v) {
    case DEV_OK: return MOE_OK;
    case DEV_BAD_EXPERT_ID: return MOE_ERR_INVALID_ARG;
    case DEV_BAD_EP_LAYOUT: return MOE_ERR_INVALID_ARG;
    case DEV_TIMEOUT: return MOE_ERR_TIMEOUT;
    case DEV_BOUNDS: return MOE_ERR_BOUNDS;
    default: return MOE_ERR_CUDA;
  }
}

int moe_set_phase_events(void* const* events, int n) {
  if (events == nullptr || n == 0) {
    g_phase_on = g_bwd_phase_on = false;
    return MOE_OK;
  }
  if (n != kFwdEvents && n != kAllEvents) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) g_phase_events[i] = static_cast<cudaEvent_t>(events[i]);
  g_phase_on = true;
  g_bwd_phase_on = n == kAllEvents;
  return MOE_OK;
}

int moe_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns == 0 ? kDefaultWaitNs : ns;
  return MOE_OK;
}

}  // extern "C"
