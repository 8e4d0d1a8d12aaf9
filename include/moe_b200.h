/*
 * moe_b200.h -- C ABI of the dots.llm1 fine-grained MoE FFN layer for NVIDIA
 * B200 (sm_100a).
 *
 * The layer (dots.llm1 Technical Report, Method; "Model Architecture Features"
 * on the kdjingpai.com page): an FP32 gate scores E = 128 routed experts, the
 * auxiliary-loss-free per-expert bias picks the top k = 6, two shared experts
 * are always on, every expert is a SwiGLU feed-forward network, and the
 * outputs are summed with the renormalised gate weights.  The grouped GEMM
 * pads every expert's token segment to a multiple of the MMA tile (Technical
 * Report, Key claims / Method, systems paragraph).
 *
 * Conventions shared by every call
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates device memory; scratch ("workspace") is caller-provided
 *    and its size is queried first.
 *  - Layouts are row-major.  Weights follow the [out, in] convention:
 *      w1, w3 [E, I, d]  gate / up projections of routed expert e
 *      w2     [E, d, I]  down projection of routed expert e
 *      ws1, ws3 [S, I, d], ws2 [S, d, I]  the S shared experts (same I)
 *  - bf16 tensors are passed as moe_bf16 (the raw 16-bit pattern).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and does no host synchronisation.  Argument errors are
 *    detected on the host before anything is launched and are returned as a
 *    negative status.  Errors that only the device can see (an expert id out
 *    of range, a bounded wait that ran out) are recorded in a per-device
 *    status word that moe_get_last_device_status() returns.
 *  - Routing convention (readings where the pages are silent): softmax over
 *    the E fp32 logits; the bias is added to the probabilities for the
 *    selection only; the chosen probabilities are renormalised to sum to 1;
 *    equal keys rank the lower expert id first; shared experts have weight 1;
 *    SwiGLU h = silu(w1 x) * (w3 x), silu(g) = g / (1 + exp(-g)).
 *  - Shape limits: 1 <= E <= 128, 1 <= k <= min(E, 8), d % 128 == 0,
 *    I % 64 == 0, align % 16 == 0, 0 <= n_shared <= 4, T >= 0.
 *    Violations return MOE_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;

/* Status codes. */
enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,       /* null pointer, negative size, bad idx */
  MOE_ERR_UNSUPPORTED_SHAPE = -2, /* shape outside the limits above       */
  MOE_ERR_WORKSPACE = -3,         /* workspace missing, small or unaligned */
  MOE_ERR_CUDA = -4,              /* a CUDA runtime call failed            */
  MOE_ERR_TIMEOUT = -5,           /* a bounded device-side wait ran out    */
  MOE_ERR_BOUNDS = -6             /* a device bounds check failed (only the
                                     MOE_CHECKS build checks; see below)  */
};

/* Layer dimensions.
 *   T tokens, d hidden size, E routed experts, k experts chosen per token,
 *   I intermediate size of every expert (routed and shared), n_shared shared
 *   experts, align = segment padding granularity in rows (multiple of 16). */
typedef struct moe_dims {
  int T, d, E, k, I, n_shared, align;
} moe_dims;

/* Rows of the permuted buffers: T*k + E*(align-1), the most any routing can
 * need once every segment is rounded up to `align`.  Returns 0 on bad dims. */
int64_t moe_capacity(const moe_dims* dims);

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int status);

/* ------------------------------------------------------------------------
 * moe_route -- the FP32 gate and bias-adjusted top-k selection.
 * Technical Report, Method: gate projection in FP32, auxiliary-loss-free
 * bias, top-6 of 128.
 *
 *   x        [T, d]  bf16 tokens
 *   w_gate   [E, d]  fp32 gate weights
 *   bias     [E]     fp32 selection bias (may be NULL: zero bias)
 *   probs    [T, E]  fp32 out: softmax of the logits (may be NULL)
 *   topk_idx [T, k]  int32 out: chosen experts by descending p + bias
 *   topk_w   [T, k]  fp32 out: renormalised probabilities of the chosen experts
 *   workspace        device scratch of moe_route_workspace_size() bytes,
 *                    256-byte aligned (partial gate logits of the split-K
 *                    fp32 GEMM)
 * The logits are accumulated in fp32 in a fixed order, so results are
 * deterministic for given dims.  Returns MOE_OK or a negative status.
 * ---------------------------------------------------------------------- */
size_t moe_route_workspace_size(const moe_dims* dims);
int moe_route(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
              const float* bias, float* probs, int32_t* topk_idx,
              float* topk_w, void* workspace, size_t workspace_bytes,
              void* stream);

/* ------------------------------------------------------------------------
 * moe_route_noalloc -- moe_route without a caller workspace.
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory when they route -- an inference engine's
 * plugin/enqueue hook that is handed a stream and its buffers but no
 * allocator, or a serving loop that forbids allocation after warm-up because
 * cudaMalloc can synchronise the device and fragments a pool owned by someone
 * else.  It allocates nothing: the split-K partial logits live in a fixed
 * 16 MiB array inside the library, which every GPU that loads the library
 * holds until the process exits.
 *
 * Arguments and results are those of moe_route (same kernels, bit-identical
 * output).  The split-K planner keeps the partials within 16 MiB whenever one
 * split fits, so a shape is rejected (MOE_ERR_WORKSPACE, nothing launched)
 * exactly when one split alone needs more: T * E * 4 bytes > 16 MiB, i.e.
 * T * E > 4194304 (T > 32768 at E = 128).
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  The address is cached for the life of the process: after a
 * cudaDeviceReset the cached address (and the library's device status word
 * address, cached the same way) is stale, so do not call the library again
 * in that process after a reset.  All calls share the array: it needs no
 * clearing (every partial read is written first in the same call), but calls
 * that overlap on the GPU (other streams, other host threads on the same
 * device) race on it.
 * ---------------------------------------------------------------------- */
int moe_route_noalloc(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                      const float* bias, float* probs, int32_t* topk_idx,
                      float* topk_w, void* stream);

/* ------------------------------------------------------------------------
 * moe_permute -- counting sort of the (token, slot) pairs into per-expert
 * segments padded to `align` rows, and the row gather of x.
 * Technical Report, Method (systems paragraph): expert segments are padded to
 * tile multiples so every MMA tile holds rows of one expert only.
 *
 *   topk_idx     [T, k]     int32 expert ids (each in [0, E))
 *   x            [T, d]     bf16 tokens
 *   counts       [E]        int32 out: pairs routed to each expert
 *   offsets      [E+1]      int32 out: first row of each segment; segment e
 *                           spans counts[e] rounded up to `align` rows
 *   row_of       [T*k]      int32 out: row of pair (t, j) at index t*k + j;
 *                           rows of a segment follow ascending token id
 *   token_of_row [cap]      int32 out: token of each row; -1 for padding
 *                           rows and for rows >= offsets[E]
 *   x_perm       [cap, d]   bf16 out: x_perm[r] = x[token_of_row[r]], padding
 *                           rows inside segments are zero; rows at or after
 *                           offsets[E] are not written
 *   workspace               moe_permute_workspace_size() bytes (per-chunk
 *                           expert histograms)
 * cap = moe_capacity(dims).  Ids out of range are skipped and flagged as
 * MOE_ERR_INVALID_ARG in the device status word.
 * ---------------------------------------------------------------------- */
size_t moe_permute_workspace_size(const moe_dims* dims);
int moe_permute(const moe_dims* dims, const int32_t* topk_idx,
                const moe_bf16* x, int32_t* counts, int32_t* offsets,
                int32_t* row_of, int32_t* token_of_row, moe_bf16* x_perm,
                void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_grouped_swiglu -- the grouped SwiGLU expert GEMMs over the segments.
 * Technical Report, Key claims / Method (grouped GEMM over tile-padded expert
 * segments); SwiGLU experts per the Model Architecture Features paragraph.
 * tcgen05 tensor-core MMAs (bf16 in, fp32 accumulate in tensor memory), fed by
 * TMA; SwiGLU is fused into the epilogue of the gate/up GEMM.
 *
 *   x_perm  [cap, d]   bf16 segment rows (moe_permute output)
 *   offsets [E+1]      int32 segment starts (moe_permute output)
 *   w1, w3  [E, I, d]  bf16;  w2 [E, d, I] bf16
 *   h_perm  [cap, I]   bf16 out: silu(x w1^T) * (x w3^T) for every segment row
 *   y_perm  [cap, d]   fp32 out: h w2^T for every segment row (the fp32
 *                      accumulators, not rounded: a bf16 copy would round a
 *                      dominant expert's output twice on its way into y)
 * Rows outside [0, offsets[E]) are neither read nor written.  Padding rows are
 * computed like the others (zero rows give zero outputs).  No workspace.
 * ---------------------------------------------------------------------- */
int moe_grouped_swiglu(const moe_dims* dims, const moe_bf16* x_perm,
                       const int32_t* offsets, const moe_bf16* w1,
                       const moe_bf16* w3, const moe_bf16* w2,
                       moe_bf16* h_perm, float* y_perm, void* stream);

/* ------------------------------------------------------------------------
 * moe_combine -- weighted un-permute and shared-expert add.
 * Technical Report, Method: output = shared experts (weight 1) + the k routed
 * experts weighted by the gate.
 *
 *   y_perm   [cap, d]  fp32 routed expert outputs per segment row
 *   row_of   [T*k]     int32 row of each (token, slot) pair
 *   topk_w   [T, k]    fp32 weights
 *   y_shared [T, d]    fp32 sum of the shared experts' outputs (may be NULL)
 *   y        [T, d]    bf16 out: y[t] = y_shared[t] + sum_j w[t,j] y_perm[row_of[t*k+j]]
 * The sum runs in fp32, slot j in ascending order, and is rounded once.
 * ---------------------------------------------------------------------- */
int moe_combine(const moe_dims* dims, const float* y_perm,
                const int32_t* row_of, const float* topk_w,
                const float* y_shared, moe_bf16* y, void* stream);

/* ------------------------------------------------------------------------
 * moe_forward -- the whole layer in one call: route, permute, grouped SwiGLU
 * GEMMs for the routed experts and the shared experts, combine.
 *
 *   x [T, d] bf16; w_gate [E, d] fp32; bias [E] fp32 (NULL = zero)
 *   w1, w3 [E, I, d], w2 [E, d, I] bf16 routed experts
 *   ws1, ws3 [S, I, d], ws2 [S, d, I] bf16 shared experts (NULL iff S == 0)
 *   y [T, d] bf16 out
 *   workspace  moe_workspace_size() bytes, 256-byte aligned.  After the call
 *              it holds every intermediate at the offsets moe_forward_layout()
 *              reports (probs, idx, weights, counts, offsets, row_of,
 *              token_of_row, x_perm, h_perm, y_perm, h_shared, y_shared).
 * ---------------------------------------------------------------------- */
typedef struct moe_ws_layout {
  size_t route_partials;  /* fp32 [splits, T, E] split-K partial logits    */
  size_t probs;           /* fp32 [T, E]                                   */
  size_t topk_idx;        /* int32 [T, k]                                  */
  size_t topk_w;          /* fp32 [T, k]                                   */
  size_t counts;          /* int32 [E]                                     */
  size_t offsets;         /* int32 [E+1]                                   */
  size_t row_of;          /* int32 [T*k]                                   */
  size_t token_of_row;    /* int32 [cap]                                   */
  size_t permute_scratch; /* moe_permute_workspace_size() bytes            */
  size_t x_perm;          /* bf16 [cap, d]                                 */
  size_t h_perm;          /* bf16 [cap, I]                                 */
  size_t y_perm;          /* fp32 [cap, d]                                 */
  size_t h_shared;        /* bf16 [T, S*I]; column s*I + i = shared expert s */
  size_t y_shared;        /* fp32 [T, d]   sum of the shared experts        */
  size_t total;           /* = moe_workspace_size()                        */
} moe_ws_layout;

size_t moe_workspace_size(const moe_dims* dims);
int moe_forward_layout(const moe_dims* dims, moe_ws_layout* layout);
int moe_forward(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                const float* bias, const moe_bf16* w1, const moe_bf16* w3,
                const moe_bf16* w2, const moe_bf16* ws1, const moe_bf16* ws3,
                const moe_bf16* ws2, moe_bf16* y, void* workspace,
                size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Training: moe_forward_train and moe_backward.
 * Technical Report, Results: the grouped GEMM is measured in the forward and
 * in the backward pass.
 *
 * moe_forward_train is moe_forward that also keeps the gate/up
 * pre-activations (g = w1 x, u = w3 x) for the backward, in fp32: they feed
 * only the SwiGLU backward's arithmetic, not a tensor-core operand, and bf16
 * copies of them would cost the shared experts' weight gradients about 1 %
 * of their rms in accuracy.  Its workspace
 * (moe_train_workspace_size() bytes, 256-byte aligned) starts with the
 * forward layout (same offsets as moe_forward_layout) and adds the regions
 * of moe_train_layout.
 *
 * moe_backward takes that workspace after moe_forward_train on the same x and
 * weights, and the upstream gradient dy [T, d] bf16, and writes
 *   dx [T, d] bf16, dw_gate [E, d] fp32, dw1, dw3 [E, I, d], dw2 [E, d, I],
 *   dws1, dws3 [S, I, d], dws2 [S, d, I] (bf16; every element is written,
 *   experts that received no token get zero).
 * moe_backward_f32 is the same computation with dx and every expert weight
 * gradient written in fp32: the tensor-core accumulators and the fp32 sum of
 * dx are stored unrounded (moe_backward's outputs are exactly their bf16
 * roundings, to nearest even).  Use it where the gradients are accumulated or
 * applied in fp32; it writes twice the bytes.
 * The routing choice of the forward is held fixed; the bias only enters the
 * selection key and gets no gradient.  Gradients flow through the combine
 * weights, the renormalisation and the softmax into w_gate and x.  Extra
 * limits: I % 128 == 0 (moe_forward_train too) and E % 4 == 0.
 * ---------------------------------------------------------------------- */
typedef struct moe_train_layout {
  moe_ws_layout fwd;    /* the forward intermediates (moe_forward_layout)  */
  size_t g_perm;        /* fp32 [cap, I]  gate pre-activations             */
  size_t u_perm;        /* fp32 [cap, I]  up pre-activations               */
  size_t g_shared;      /* fp32 [T, S*I]                                   */
  size_t u_shared;      /* fp32 [T, S*I]                                   */
  size_t dy_perm;       /* bf16 [cap, d]  w * dy per segment row            */
  size_t dw;            /* fp32 [T, k]    gradient of the combine weights   */
  size_t dz;            /* fp32 [T, E]    gradient of the gate logits       */
  size_t dgu_perm;      /* bf16 [cap, 2I] [dG | dU]                         */
  size_t dgu_shared;    /* bf16 [T, 2*S*I]                                  */
  size_t dx_perm;       /* fp32 [cap, d]                                    */
  size_t dx_shared;     /* fp32 [T, d]                                      */
  size_t dx_router;     /* fp32 [T, d]    dz w_gate                         */
  size_t dwg_partials;  /* fp32 [splits, E, d]                              */
  size_t total;         /* = moe_train_workspace_size()                     */
} moe_train_layout;

size_t moe_train_workspace_size(const moe_dims* dims);
int moe_train_layout_of(const moe_dims* dims, moe_train_layout* layout);
int moe_forward_train(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                      const float* bias, const moe_bf16* w1, const moe_bf16* w3,
                      const moe_bf16* w2, const moe_bf16* ws1, const moe_bf16* ws3,
                      const moe_bf16* ws2, moe_bf16* y, void* workspace,
                      size_t workspace_bytes, void* stream);
int moe_backward(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                 const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                 const moe_bf16* ws1, const moe_bf16* ws3, const moe_bf16* ws2,
                 const moe_bf16* dy, void* workspace, size_t workspace_bytes,
                 moe_bf16* dx, float* dw_gate, moe_bf16* dw1, moe_bf16* dw3,
                 moe_bf16* dw2, moe_bf16* dws1, moe_bf16* dws3, moe_bf16* dws2,
                 void* stream);
int moe_backward_f32(const moe_dims* dims, const moe_bf16* x, const float* w_gate,
                     const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                     const moe_bf16* ws1, const moe_bf16* ws3, const moe_bf16* ws2,
                     const moe_bf16* dy, void* workspace, size_t workspace_bytes, float* dx,
                     float* dw_gate, float* dw1, float* dw3, float* dw2, float* dws1,
                     float* dws3, float* dws2, void* stream);

/* ------------------------------------------------------------------------
 * moe_dense_swiglu -- the dense SwiGLU FFN of the model's first layer
 * (Technical Report, Method: layer 1 is a dense SwiGLU FFN, layers 2-62 are
 * MoE).  Runs on the same grouped GEMM kernels as the experts, as one group
 * holding every token:
 *
 *   y = (silu(x w1^T) * (x w3^T)) w2^T
 *
 *   dims       T, d and I (the FFN's intermediate size) are used; E, k,
 *              n_shared and align are ignored.  d % 128 == 0, I % 64 == 0.
 *   x  [T, d]  bf16;  w1, w3 [I, d], w2 [d, I] bf16
 *   y  [T, d]  bf16 out (h rounded to bf16, fp32 accumulation, one rounding)
 *   workspace  moe_dense_workspace_size() bytes, 256-byte aligned: h [T, I],
 *              and at small T (too few tiles for the SMs) the fp32 partial
 *              sums of a GEMM split over K, added in a fixed order before the
 *              SwiGLU (gate/up) or the one rounding of y (down).
 * Returns INVALID_ARG (null or misaligned pointer), UNSUPPORTED_SHAPE,
 * WORKSPACE, CUDA.  T == 0 is a no-op.
 * ---------------------------------------------------------------------- */
size_t moe_dense_workspace_size(const moe_dims* dims);
int moe_dense_swiglu(const moe_dims* dims, const moe_bf16* x, const moe_bf16* w1,
                     const moe_bf16* w3, const moe_bf16* w2, moe_bf16* y,
                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Load balancing, training side.  Technical Report, Method: the router is
 * balanced by the DeepSeek auxiliary-loss-free per-expert bias, stepped after
 * each batch from the experts' loads, plus a sequence-wise balance loss
 * against extreme imbalance inside one sequence.  The report names both and
 * gives no formula; the published DeepSeek forms are taken (stated below).
 *
 * moe_balance_workspace_size -- bytes of workspace moe_balance_stats needs for
 * dims->T tokens in sequences of seq_len tokens (0 on invalid arguments).
 *
 * moe_balance_stats -- per-sequence load statistics and the balance loss.
 *   seq_len   tokens per sequence; T must be a whole number of sequences
 *   probs     [T, E] fp32 softmax probabilities (moe_route / moe_forward)
 *   topk_idx  [T, k] int32 chosen experts
 *   alpha     balance-loss coefficient
 *   f, P      [T/seq_len, E] fp32 out, for sequence s and expert e:
 *               f[s,e] = E / (k seq_len) * #pairs of s routed to e
 *               P[s,e] = mean over the tokens t of s of probs[t,e]
 *   loss      [1] fp32 out: alpha * mean over s of sum_e f[s,e] P[s,e]
 *             (0 when T == 0)
 *   workspace moe_balance_workspace_size() bytes, 256-byte aligned
 * Sums run in fp64 in a fixed order (deterministic); f is one rounding of the
 * exact quotient.  An id outside [0, E) is skipped and recorded as
 * MOE_ERR_INVALID_ARG in the device status word.  Returns INVALID_ARG (null
 * pointer, seq_len <= 0, T not a multiple of seq_len), WORKSPACE, CUDA.
 *
 * moe_bias_update -- one auxiliary-loss-free bias step from a batch's loads:
 *   counts    [E] int32 pairs per expert (the counts moe_permute and
 *             moe_forward write); dims->T is the number of tokens they cover.
 *             With data-parallel replicas the caller sums counts and T over
 *             the replicas first, so that every replica takes the same step.
 *   bias_out[e] = bias_in[e] - gamma  if E*counts[e] > T*k  (above the mean)
 *                 bias_in[e] + gamma  if E*counts[e] < T*k  (below the mean)
 *                 bias_in[e]          otherwise (bit for bit)
 *   bias_out may alias bias_in.  The comparison is exact integer arithmetic;
 *   the step is one fp32 rounding.  Returns INVALID_ARG (null pointer), CUDA.
 * ---------------------------------------------------------------------- */
size_t moe_balance_workspace_size(const moe_dims* dims, int seq_len);
int moe_balance_stats(const moe_dims* dims, int seq_len, const float* probs,
                      const int32_t* topk_idx, float alpha, float* f, float* P,
                      float* loss, void* workspace, size_t workspace_bytes,
                      void* stream);
int moe_bias_update(const moe_dims* dims, const int32_t* counts, float gamma,
                    const float* bias_in, float* bias_out, void* stream);

/* ------------------------------------------------------------------------
 * Expert parallelism.  Technical Report, Method / Key claims (systems
 * paragraph): the MoE all-to-all between ranks, overlapped with the grouped
 * GEMMs; "How dots.llm1's 14B MoE Architecture Matches 72B LLM Performance",
 * Computational Infrastructure Innovations: all-to-all expert communication.
 * The pages name the exchange, not its layout; the layout used:
 *
 *   world W ranks, every rank routes its own T tokens (same dims on every
 *   rank); rank r owns the routed experts r*El .. r*El + El-1, El = E/W, and
 *   holds only their weights; the shared experts are replicated and run on
 *   each rank's own tokens.  Rank r's receive buffer holds one segment per
 *   local expert, padded to `align` rows, with the (token, slot) pairs of
 *   every source rank in rank order, each source's pairs by ascending token.
 *   Every rank derives this layout from all ranks' counts, so a source writes
 *   its token rows straight into the owners' receive buffers and the combine
 *   reads the expert outputs back from them.
 *
 * A step on rank r, with barriers between ranks where marked:
 *   moe_ep_route       router + permutation index of the own tokens
 *   -- barrier (every rank's counts written) --
 *   moe_ep_dispatch    layout from every rank's counts; each pair's token row
 *                      stored into its owner's receive buffer; padding rows of
 *                      the own receive buffer zeroed
 *   -- barrier (every receive buffer complete) --
 *   moe_ep_experts     grouped SwiGLU GEMMs of the El local experts over the
 *                      receive buffer, and the shared experts on own tokens
 *   -- barrier (every owner's outputs complete) --
 *   moe_ep_combine     y[t] = shared + sum_j w[t,j] * (row of pair (t, j) in
 *                      its owner's output buffer), fp32, j ascending, as
 *                      moe_combine
 * The barriers are the caller's (e.g. a one-element NCCL all-reduce on the
 * same stream); the library waits on nothing.  Cross-rank arguments are
 * DEVICE arrays of W device pointers, element s for rank s: peer pointers
 * (CUDA IPC or a symmetric allocation) on a multi-GPU node, or plain buffers
 * of this GPU when several ranks are emulated by one process.
 *
 * moe_ep_recv_capacity  rows of a receive buffer: W*T*k + El*(align-1)
 *                       (0 on invalid arguments)
 * moe_ep_workspace_size bytes of one rank's workspace; moe_ep_layout_of
 *                       reports where its regions are:
 */
typedef struct moe_ep_layout {
  size_t route_partials;  /* fp32 router split-K partials                   */
  size_t probs;           /* fp32 [T, E]                                   */
  size_t topk_idx;        /* int32 [T, k]                                  */
  size_t topk_w;          /* fp32 [T, k]                                   */
  size_t counts;          /* int32 [E]   own pairs per expert (peers read)  */
  size_t offsets;         /* int32 [E+1] own segment layout                */
  size_t row_of;          /* int32 [T*k]                                   */
  size_t token_of_row;    /* int32 [T*k + E*(align-1)]                     */
  size_t permute_scratch; /* permutation scratch                           */
  size_t dst_row;         /* int32 [E]   first receive row of the own pairs
                                         of expert e on its owner (-1 after
                                         a rejected count table)           */
  size_t recv_offsets;    /* int32 [El+1] segment starts in the own buffer  */
  size_t recv_counts;     /* int32 [El]  pairs received per local expert    */
  size_t remote_row;      /* int32 [T*k] receive row of pair (t, j), -1 if
                                         not sent                          */
  size_t h_recv;          /* bf16 [recv_cap, I] local experts' SwiGLU out   */
  size_t h_shared;        /* bf16 [T, S*I]                                 */
  size_t y_shared;        /* fp32 [T, d]                                   */
  size_t total;           /* = moe_ep_workspace_size()                     */
} moe_ep_layout;

int64_t moe_ep_recv_capacity(const moe_dims* dims, int world);
size_t moe_ep_workspace_size(const moe_dims* dims, int world);
int moe_ep_layout_of(const moe_dims* dims, int world, moe_ep_layout* layout);

/* moe_ep_route -- x [T, d] bf16, w_gate [E, d] fp32, bias [E] fp32 (NULL =
 * zero): moe_route and the index half of moe_permute (no row gather) into
 * the workspace.  Results equal theirs bit for bit. */
int moe_ep_route(const moe_dims* dims, int world, const moe_bf16* x,
                 const float* w_gate, const float* bias, void* workspace,
                 size_t workspace_bytes, void* stream);

/* moe_ep_dispatch --
 *   counts_of  device array [W] of int32 [E] pointers: every rank's counts
 *              (element s = rank s's workspace counts, or a gathered copy);
 *              element `rank` must equal this rank's own counts
 *   x_recv     device array [W] of bf16 [recv_cap, d] receive buffers,
 *              16-byte aligned
 * A count table that is negative, disagrees with the own counts or overflows
 * a receive buffer is recorded as MOE_ERR_INVALID_ARG in the device status
 * word and nothing is sent or received. */
int moe_ep_dispatch(const moe_dims* dims, int world, int rank, const moe_bf16* x,
                    const int32_t* const* counts_of, moe_bf16* const* x_recv,
                    void* workspace, size_t workspace_bytes, void* stream);

/* moe_ep_experts --
 *   x        [T, d] bf16 own tokens (shared experts)
 *   x_recv   [recv_cap, d] this rank's receive buffer
 *   w1, w3   [El, I, d], w2 [El, d, I] bf16: this rank's experts only
 *   ws1, ws3 [S, I, d], ws2 [S, d, I] shared experts (NULL iff S == 0)
 *   y_recv   [recv_cap, d] fp32 out: expert outputs per receive row
 * Rows at or after the last segment are neither read nor written. */
int moe_ep_experts(const moe_dims* dims, int world, const moe_bf16* x,
                   const moe_bf16* x_recv, const moe_bf16* w1, const moe_bf16* w3,
                   const moe_bf16* w2, const moe_bf16* ws1, const moe_bf16* ws3,
                   const moe_bf16* ws2, float* y_recv, void* workspace,
                   size_t workspace_bytes, void* stream);

/* moe_ep_combine --
 *   y_recv  device array [W] of the ranks' fp32 expert-output buffers
 *   y       [T, d] bf16 out
 * Same arithmetic as moe_combine; a pair that was not sent contributes 0. */
int moe_ep_combine(const moe_dims* dims, int world, const float* const* y_recv,
                   moe_bf16* y, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * CUDA IPC of the expert-parallel buffers (receive buffers, counts) between
 * the processes of one node, one process per GPU.
 *
 * moe_ipc_export -- ptr: a device address inside an allocation of this
 *   process made by cudaMalloc (PyTorch's default allocator); writes the
 *   allocation's 64-byte IPC handle to `handle` and ptr's offset inside the
 *   allocation to `offset`.
 * moe_ipc_open -- maps another process's allocation on the current device
 *   (peer access enabled lazily) and returns the address of handle + offset
 *   in *ptr.  A process cannot open its own handles (CUDA rejects them).
 * moe_ipc_close -- unmaps what moe_ipc_open returned (same offset).
 * Return MOE_OK, MOE_ERR_INVALID_ARG (null pointer) or MOE_ERR_CUDA.
 * ---------------------------------------------------------------------- */
int moe_ipc_export(const void* ptr, void* handle, uint64_t* offset);
int moe_ipc_open(const void* handle, uint64_t offset, void** ptr);
int moe_ipc_close(void* ptr, uint64_t offset);

/* ------------------------------------------------------------------------
 * Device status and bounded waits.
 *
 * moe_get_last_device_status: synchronises `stream`, returns the first error
 * the kernels recorded on the current device since the last call (MOE_OK if
 * none) and clears it.  MOE_ERR_TIMEOUT means a pipeline wait inside a kernel
 * gave up; the kernel then drained its own copies, freed its tensor memory and
 * returned, so the context stays usable.
 *
 * moe_set_wait_limit_ns: limit of every pipeline wait inside the GEMM kernels
 * (default 1e9 ns; 0 restores the default).  A test hook: a tiny limit makes
 * the waits run out on purpose.  Process-wide, not thread-safe.
 * ---------------------------------------------------------------------- */
int moe_get_last_device_status(void* stream);
int moe_set_wait_limit_ns(uint64_t ns);

/* ------------------------------------------------------------------------
 * moe_set_phase_events -- measurement hook.  With n == 6 CUDA events
 * (cudaEvent_t handles owned by the caller), every later moe_forward /
 * moe_forward_train records events[0] before its first kernel and
 * events[1..5] after the router, the permutation, the gate/up GEMM, the down
 * GEMM and the combine, on its stream.  With n == 13, moe_backward also
 * records events[6] before its first kernel and events[7..12] after the
 * combine/router backward, the dH + SwiGLU-backward dgrad, the dW2 wgrad, the
 * dX dgrad, the dW1/dW3 wgrads and the gate GEMMs + un-permute.  An entry may
 * be NULL: that point is not recorded (timing one phase needs only its two
 * bounding events, which keeps the hook's own cost out of the others).
 * n == 0 (or events == NULL) turns the hook off.  Process-wide; the events
 * must outlive every call issued while they are set.
 * ---------------------------------------------------------------------- */
int moe_set_phase_events(void* const* events, int n);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
