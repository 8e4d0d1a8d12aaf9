// Backward grouped GEMMs on the tcgen05 tensor cores (sm_100a).
//
// dots.llm1 Technical Report, Results: the grouped GEMM is also measured in
// the backward pass.  With y = combine(experts(x)) and the selection fixed,
// the expert part of the backward is three grouped GEMM kinds over the same
// tile-padded segments as the forward:
//
//   kDgradDown  dH = dY W2 per segment (swap-AB: M = I features, N = tokens,
//               K = d), with the SwiGLU backward fused in the epilogue:
//               dG = dH * U * silu'(G), dU = dH * silu(G) from the stored
//               pre-activations; writes dGU = [dG | dU] (bf16)
//   kDgradUp    dX = dG W1 + dU W3 (M = d features, N = tokens, K = 2I: the
//               W1 rows then the W3 rows)
//   kWgrad      dW = A^T B with K = the segment's tokens: dW2 = dY^T H,
//               dW1 = dG^T X, dW3 = dU^T X (M, N = weight rows / columns)
//
// The weights enter the dgrads transposed and the activations enter the
// wgrads transposed, so those operands are MN-major in shared memory (TMA
// boxes of 64 MN-elements x 64 K-rows, 128-byte swizzle; the descriptor's
// leading byte offset steps between 64-wide MN blocks).  Token operands of the
// dgrads stay K-major as in the forward.  The pipeline is the forward's:
// persistent CTAs, TMA ring, double-buffered TMEM accumulators, warp roles,
// bounded waits.  The shared experts are extra groups over all T tokens.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "moe_internal.h"
#include "checks.cuh"
#include "ptx_sm100.cuh"

namespace moe {
namespace {

enum BwdMode : int { kDgradDown = 0, kDgradUp = 1, kWgrad = 2 };

constexpr int kBK = 64;
constexpr int kBoxB = 32;           // token rows per TMA box of a K-major token operand
constexpr int kABytes = 128 * 128;  // A stage: 128 MN x 64 K bf16
constexpr int kNT = 256;            // N per tile (tokens for dgrad, weight columns for wgrad)
constexpr int kBBytes = kNT * 128;  // B stage
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kStages = 4;
constexpr int kMaxGroups = 136;     // 128 routed + up to 8 shared groups
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 2 * kNT;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

struct BwdParams {
  int E;            // routed groups
  int n_sgroups;    // shared groups (dgrad: 0 or 1; wgrad: S or 0)
  int T;
  int I, d, S;
  const int32_t* offsets;
  int mt_routed, mt_shared;            // M tiles (of 128) per group
  int nt_routed, nt_shared;            // wgrad: N tiles (of kNT) per group
  int ntot_routed, ntot_shared;        // wgrad: N extent of the output
  int kit_routed, kit_shared;          // dgrad: K chunks of 64
  int ksplit_routed, ksplit_shared;    // dgrad-up: first chunk read from the second A map
  int a_col0_routed, a_col0_shared, a_step_shared;  // wgrad: A column offsets
  // wgrad: M tiles at or past m_split belong to a second output (out2_*),
  // their A columns start at a_col1_* (0 = one output)
  int m_split;
  int a_col1_routed, a_col1_shared;
  void *out2_routed, *out2_shared;
  int b_col0_routed, b_col0_shared, b_step_shared;  // wgrad: B column offsets
  void* out_routed;
  int ld_routed;
  void* out_shared;
  int ld_shared;
  int shared_f32;
  int out_f32;                             // wgrad: fp32 weight gradients (else bf16)
  int64_t gstride_routed, gstride_shared;  // wgrad: elements between groups' outputs
  const float *g_routed, *u_routed, *g_shared, *u_shared;  // dgrad-down: fp32 pre-activations
  int ld_gu_routed, ld_gu_shared;
  int ucol_routed, ucol_shared;  // dgrad-down: column of dU in the output
  unsigned int* status;
  uint64_t wait_limit_ns;
  int64_t rows_routed, rows_shared;  // dgrads: token rows of the routed / shared buffers
};

struct Tile {
  int g;        // group
  int mt;       // M tile
  int row0;     // first token row of the group (dgrad: of the tile)
  int nrows;    // dgrad: token rows of the tile; wgrad: K rows of the group
  int n;        // MMA N (dgrad: rows rounded to 16; wgrad: columns of the tile)
  int ncol0;    // wgrad: first output column of the tile
  int kchunks;  // K chunks of 64
  int last_k16; // MMAs of K = 16 in the last chunk
};

struct Ctl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int ngroups;
  int total_tiles;
  int prefix[kMaxGroups + 1];
  int row0[kMaxGroups];
  int rows[kMaxGroups];
};

__device__ __forceinline__ bool aborted(const Ctl& c) {
  return *reinterpret_cast<const volatile int*>(&c.abort_flag) != 0;
}

__device__ __forceinline__ void record_timeout(Ctl& c, const BwdParams& p) {
  *reinterpret_cast<volatile int*>(&c.abort_flag) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0u, (unsigned)DEV_TIMEOUT);
}

// MN-major operand stored by TMA boxes of 64 MN x 64 K (128-byte rows, one
// row per K index, 128-byte swizzle): 8-row atoms of 1024 bytes along K
// (stride byte offset), 64-wide MN blocks 8192 bytes apart (leading byte
// offset).  K advances by 16 rows = 2048 bytes per MMA.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(8192 >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: D fp32, A/B bf16, M = 128, A MN-major,
// B MN-major when b_mn.
__device__ __forceinline__ uint32_t idesc_bwd(uint32_t n, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((n >> 3) << 17) | ((128u >> 4) << 24);
}

template <int MODE>
__device__ __forceinline__ Tile decode(const Ctl& c, const BwdParams& p, int tile) {
  int lo = 0, hi = c.ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.g = lo;
  const bool routed = lo < p.E;
  const int local = tile - c.prefix[lo];
  if (MODE == kWgrad) {
    const int nt = routed ? p.nt_routed : p.nt_shared;
    const int ntot = routed ? p.ntot_routed : p.ntot_shared;
    t.mt = local / nt;
    const int ntile = local - t.mt * nt;
    t.ncol0 = ntile * kNT;
    t.n = min(kNT, ntot - t.ncol0);
    t.row0 = c.row0[lo];
    t.nrows = c.rows[lo];
    t.kchunks = (t.nrows + kBK - 1) / kBK;
    const int rem = t.nrows - (t.kchunks - 1) * kBK;
    t.last_k16 = t.kchunks > 0 ? (rem + 15) / 16 : 0;
  } else {
    const int mtn = routed ? p.mt_routed : p.mt_shared;
    const int tt = local / mtn;
    t.mt = local - tt * mtn;
    t.row0 = c.row0[lo] + tt * kNT;
    t.nrows = min(kNT, c.rows[lo] - tt * kNT);
    t.n = (t.nrows + 15) & ~15;
    t.ncol0 = 0;
    t.kchunks = routed ? p.kit_routed : p.kit_shared;
    t.last_k16 = 4;
  }
  return t;
}

__device__ __forceinline__ float sigmoid_f(float g) { return 1.0f / (1.0f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_bwd_kernel(const __grid_constant__ CUtensorMap tmA_r,
                        const __grid_constant__ CUtensorMap tmA2_r,
                        const __grid_constant__ CUtensorMap tmB_r,
                        const __grid_constant__ CUtensorMap tmA_s,
                        const __grid_constant__ CUtensorMap tmA2_s,
                        const __grid_constant__ CUtensorMap tmB_s, const BwdParams p) {
  __shared__ Ctl ctl;
  extern __shared__ uint8_t dsmem_raw[];
  const uint32_t raw = smem_u32(dsmem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  // epilogue staging tile of the SwiGLU backward: g then u, [32][128] bf16 each
  uint16_t* epi_g = reinterpret_cast<uint16_t*>(dsmem_raw + (sbase - raw) + kStages * kStageBytes);
  uint16_t* epi_u = epi_g + 32 * 128;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0) {
    const int G = p.E + p.n_sgroups;
    int local[5];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const int g = lane * 5 + i;
      int tiles = 0;
      if (g < G) {
        int r0, nr;
        const bool routed = g < p.E;
        if (routed) {
          r0 = p.offsets[g];
          nr = p.offsets[g + 1] - r0;
        } else {
          r0 = 0;
          nr = p.T;
        }
        if (nr < 0) nr = 0;
        ctl.row0[g] = r0;
        ctl.rows[g] = nr;
        if (MODE == kWgrad)
          tiles = routed ? p.mt_routed * p.nt_routed : p.mt_shared * p.nt_shared;
        else
          tiles = (int)ceil_div(nr, kNT) * (routed ? p.mt_routed : p.mt_shared);
      }
      local[i] = tiles;
      sum += tiles;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const int g = lane * 5 + i;
      if (g < G) ctl.prefix[g] = run;
      run += local[i];
    }
    if (lane == 31) {
      ctl.prefix[G] = incl;
      ctl.total_tiles = incl;
      ctl.ngroups = G;
    }
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(smem_u32(&ctl.full[s]), 1);
        mbar_init(smem_u32(&ctl.empty[s]), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&ctl.tfull[b]), 1);
        mbar_init(smem_u32(&ctl.tempty[b]), kEpiThreads);
      }
      mbar_init(smem_u32(&ctl.drain), 1);
      ctl.abort_flag = 0;
      fence_mbar_init();
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl.tmem_base;
  const int total = ctl.total_tiles;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      const uint64_t pol_a = policy_evict_normal();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0, fill_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const Tile t = decode<MODE>(ctl, p, tile);
        const bool routed = t.g < p.E;
        const int s_idx = t.g - p.E;  // shared group index
        for (int kc = 0; kc < t.kchunks; ++kc) {
          if (aborted(ctl)) { ok = false; break; }
          if (!mbar_wait_bounded(smem_u32(&ctl.empty[stage]), phase ^ 1u, p.wait_limit_ns)) {
            record_timeout(ctl, p);
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&ctl.full[stage]);
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint32_t sB = sA + kABytes;
          const int kk = kc * kBK;
          if (MODE == kDgradDown || MODE == kDgradUp) {
            const int nbox = (t.n + kBoxB - 1) / kBoxB;
            mbar_arrive_expect_tx(fb, kABytes + nbox * kBoxB * 128);
            if (MODE == kDgradDown) {
              // A = W2^T: rows o (K) of W2 [.., d, I], columns f (M)
              if (routed) {
                for (int h = 0; h < 2; ++h)
                  tma_load_3d(sA + h * 8192, &tmA_r, fb, t.mt * 128 + h * 64, t.g * p.d + kk, 0,
                              pol_a);
              } else {
                const int fg = t.mt * 128;
                const int sp = fg / p.I;
                for (int h = 0; h < 2; ++h)
                  tma_load_3d(sA + h * 8192, &tmA_s, fb, fg - sp * p.I + h * 64, kk, sp, pol_a);
              }
            } else {
              // A = [W1 ; W3]^T: rows f (K) of W1 / W3 [.., I, d], columns o (M)
              const int ks = routed ? p.ksplit_routed : p.ksplit_shared;
              const bool second = kc >= ks;
              const CUtensorMap* tA = routed ? (second ? &tmA2_r : &tmA_r)
                                             : (second ? &tmA2_s : &tmA_s);
              const int frow = (second ? kk - ks * kBK : kk) + (routed ? t.g * p.I : 0);
              for (int h = 0; h < 2; ++h)
                tma_load_3d(sA + h * 8192, tA, fb, t.mt * 128 + h * 64, frow, 0, pol_a);
            }
            const CUtensorMap* tB = routed ? &tmB_r : &tmB_s;
            for (int b = 0; b < nbox; ++b)
              tma_load_3d(sB + b * kBoxB * 128, tB, fb, kk, t.row0 + b * kBoxB, 0, pol_b);
          } else {
            // wgrad: A (M columns) and B (N columns) of token-major sources, K = tokens
            const int nblk = t.n / 64;
            mbar_arrive_expect_tx(fb, kABytes + nblk * 8192);
            const bool second = p.m_split > 0 && t.mt >= p.m_split;
            const int mt = second ? t.mt - p.m_split : t.mt;
            const int acol = second
                ? (routed ? p.a_col1_routed : p.a_col1_shared + s_idx * p.a_step_shared)
                : (routed ? p.a_col0_routed : p.a_col0_shared + s_idx * p.a_step_shared);
            const int bcol = routed ? p.b_col0_routed : p.b_col0_shared + s_idx * p.b_step_shared;
            const CUtensorMap* tA = routed ? &tmA_r : &tmA_s;
            const CUtensorMap* tB = routed ? &tmB_r : &tmB_s;
            for (int h = 0; h < 2; ++h)
              tma_load_3d(sA + h * 8192, tA, fb, acol + mt * 128 + h * 64, t.row0 + kk, 0, pol_b);
            for (int j = 0; j < nblk; ++j)
              tma_load_3d(sB + j * 8192, tB, fb, bcol + t.ncol0 + j * 64, t.row0 + kk, 0, pol_b);
          }
          filled |= 1u << stage;
          fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < kStages; ++s) {
        if (((filled >> s) & 1u) &&
            !mbar_wait_bounded(smem_u32(&ctl.full[s]), (fill_parity >> s) & 1u, kDrainLimitNs))
          record_timeout(ctl, p);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const Tile t = decode<MODE>(ctl, p, tile);
        const uint32_t idesc = idesc_bwd((uint32_t)t.n, MODE == kWgrad);
        if (aborted(ctl) ||
            !mbar_wait_bounded(smem_u32(&ctl.tempty[acc]), acc_phase ^ 1u, p.wait_limit_ns)) {
          if (!aborted(ctl)) record_timeout(ctl, p);
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * kNT);
        for (int kc = 0; kc < t.kchunks; ++kc) {
          if (aborted(ctl) ||
              !mbar_wait_bounded(smem_u32(&ctl.full[stage]), phase, p.wait_limit_ns)) {
            if (!aborted(ctl)) record_timeout(ctl, p);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint32_t sB = sA + kABytes;
          const int nk16 = (kc == t.kchunks - 1) ? t.last_k16 : 4;
          for (int k4 = 0; k4 < nk16; ++k4) {
            const uint64_t ad = sdesc_mnmajor_sw128(sA + k4 * 2048);
            const uint64_t bd = MODE == kWgrad ? sdesc_mnmajor_sw128(sB + k4 * 2048)
                                               : sdesc_kmajor_sw128(sB + k4 * 32);
            mma_bf16_ss(dt, ad, bd, idesc, (kc | k4) != 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&ctl.empty[stage]));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(smem_u32(&ctl.tfull[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      mma_commit(smem_u32(&ctl.drain));
      if (!mbar_wait_bounded(smem_u32(&ctl.drain), 0, kDrainLimitNs)) record_timeout(ctl, p);
    }
  } else {
    // ================= epilogue (warps 2..5) =================
    const int q = warp & 3;
    const int mrow = q * 32 + lane;  // accumulator row = TMEM lane
    int acc = 0;
    uint32_t acc_phase = 0;
    const int et = threadIdx.x - 64;  // 0..127 over the epilogue warps
    // SwiGLU backward: this thread's feature (its TMEM lane) of the fp32 g / u
    // rows of one 32-token chunk.  For each token the warp's 32 lanes read 32
    // consecutive features (128 coalesced bytes); the loads are issued before
    // the accumulator is read so their latency overlaps it.
    float gv[32], uv[32];
    auto load_gu = [&](const Tile& t, int c0) {
      const bool routed = t.g < p.E;
      const float* gsrc = routed ? p.g_routed : p.g_shared;
      const float* usrc = routed ? p.u_routed : p.u_shared;
      const int ldgu = routed ? p.ld_gu_routed : p.ld_gu_shared;
      int nj = min(32, t.nrows - c0);
      if (!MOE_CHECK((int64_t)t.row0 + c0 + nj <= (routed ? p.rows_routed : p.rows_shared)))
        nj = 0;
      const size_t at0 = (size_t)(t.row0 + c0) * ldgu + t.mt * 128 + mrow;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        gv[j] = j < nj ? gsrc[at0 + (size_t)j * ldgu] : 0.f;
        uv[j] = j < nj ? usrc[at0 + (size_t)j * ldgu] : 0.f;
      }
    };
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const Tile t = decode<MODE>(ctl, p, tile);
      bool bad = aborted(ctl);
      if (!bad && !mbar_wait_bounded(smem_u32(&ctl.tfull[acc]), acc_phase, p.wait_limit_ns)) {
        record_timeout(ctl, p);
        bad = true;
      }
      if (bar_red_or(2, kEpiThreads, bad)) break;
      tc_fence_after();
      const bool routed = t.g < p.E;
      const uint32_t tbase = tmem_base + (uint32_t)(acc * kNT) + ((uint32_t)(q * 32) << 16);
      const int ncols = MODE == kWgrad ? t.n : t.nrows;
      for (int c0 = 0; c0 < ncols; c0 += 32) {
        if (MODE == kDgradDown) load_gu(t, c0);
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
        tmem_ld_wait();
        int nj = min(32, ncols - c0);
        if (MODE != kWgrad &&
            !MOE_CHECK((int64_t)t.row0 + c0 + nj <= (routed ? p.rows_routed : p.rows_shared)))
          nj = 0;  // token rows outside the buffer: recorded, stores skipped
        if (MODE == kWgrad) {
          // dW[group][mt*128 + mrow][ncol0 + c0 + j], 16-byte stores of bf16
          // (8 values) or fp32 (4 values)
          const bool second = p.m_split > 0 && t.mt >= p.m_split;
          const int mt = second ? t.mt - p.m_split : t.mt;
          void* out = second ? (routed ? p.out2_routed : p.out2_shared)
                             : (routed ? p.out_routed : p.out_shared);
          const int ldo = routed ? p.ntot_routed : p.ntot_shared;
          const int64_t gbase = routed ? (int64_t)t.g * p.gstride_routed
                                       : (int64_t)(t.g - p.E) * p.gstride_shared;
          const int64_t at = gbase + (int64_t)(mt * 128 + mrow) * ldo + t.ncol0 + c0;
          const bool zero = t.kchunks == 0;  // no tokens: the gradient is zero
          if (p.out_f32) {
            float* dst = static_cast<float*>(out) + at;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              if (j4 * 4 < nj) {
                const uint4 w = zero ? make_uint4(0, 0, 0, 0)
                                     : make_uint4(v[j4 * 4], v[j4 * 4 + 1], v[j4 * 4 + 2],
                                                  v[j4 * 4 + 3]);
                *reinterpret_cast<uint4*>(dst + j4 * 4) = w;
              }
            }
          } else {
            uint16_t* dst = static_cast<uint16_t*>(out) + at;
#pragma unroll
            for (int j8 = 0; j8 < 4; ++j8) {
              if (j8 * 8 < nj) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float lo = zero ? 0.f : __uint_as_float(v[j8 * 8 + 2 * i]);
                  const float hi = zero ? 0.f : __uint_as_float(v[j8 * 8 + 2 * i + 1]);
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);  // one paired cvt
                  w[i] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(dst + j8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        } else if (MODE == kDgradDown) {
          // SwiGLU backward: each thread works on its own feature (TMEM lane)
          // from the fp32 g and u in registers; dG / dU are staged in smem as
          // a 32-token x 128-feature bf16 tile and go out as coalesced
          // 16-byte rows.
          const int f0 = t.mt * 128;
          uint16_t* out = static_cast<uint16_t*>(routed ? p.out_routed : p.out_shared);
          const int ldo = routed ? p.ld_routed : p.ld_shared;
          const int ucol = routed ? p.ucol_routed : p.ucol_shared;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j < nj) {
              const float dh = __uint_as_float(v[j]);
              const float g = gv[j];
              const float u = uv[j];
              const float sg = sigmoid_f(g);
              const float dg = dh * u * (sg * (1.0f + g * (1.0f - sg)));
              const float du = dh * (g * sg);
              epi_g[j * 128 + mrow] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
              epi_u[j * 128 + mrow] = __bfloat16_as_ushort(__float2bfloat16_rn(du));
            }
          }
          named_bar_sync(1, kEpiThreads);
          for (int i = et; i < 32 * 16; i += kEpiThreads) {
            const int r = i >> 4, cv = i & 15;
            if (r < nj) {
              const size_t row = (size_t)(t.row0 + c0 + r) * ldo + f0 + cv * 8;
              *reinterpret_cast<uint4*>(out + row) =
                  *reinterpret_cast<const uint4*>(epi_g + r * 128 + cv * 8);
              *reinterpret_cast<uint4*>(out + row + ucol) =
                  *reinterpret_cast<const uint4*>(epi_u + r * 128 + cv * 8);
            }
          }
          named_bar_sync(1, kEpiThreads);  // the tile is reused by the next chunk
        } else {
          // dX for feature o and token rows (fp32: the k routed rows of a
          // token are summed later, so they are not rounded to bf16 here)
          const int col = t.mt * 128 + mrow;
          float* out = static_cast<float*>(routed ? p.out_routed : p.out_shared);
          const int ldo = routed ? p.ld_routed : p.ld_shared;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nj) out[(size_t)(t.row0 + c0 + j) * ldo + col] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&ctl.tempty[acc]));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 tensor (inner, rows, planes), box (64, box_rows, 1), 128-byte swizzle.
bool make_map3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
               uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {inner, rows == 0 ? 1 : rows, planes};
  cuuint64_t strides[2] = {inner * 2, inner * (rows == 0 ? 1 : rows) * 2};
  cuuint32_t box[3] = {64u, box_rows, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_bwd(const CUtensorMap* m, const BwdParams& p, int num_sms, cudaStream_t st) {
  constexpr size_t smem = (size_t)kStages * kStageBytes + 2 * 32 * 128 * 2 + 1024;
  static_assert(smem + sizeof(Ctl) <= 232448, "shared memory budget");
  auto kern = grouped_gemm_bwd_kernel<MODE>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<num_sms, kThreads, smem, st>>>(m[0], m[1], m[2], m[3], m[4], m[5], p);
  return cudaGetLastError();
}

BwdParams base_params(const Shape& s, const int32_t* offsets, unsigned int* status,
                      uint64_t wait_ns) {
  BwdParams p{};
  p.E = s.E;
  p.T = s.T;
  p.I = s.I;
  p.d = s.d;
  p.S = s.S;
  p.offsets = offsets;
  p.status = status;
  p.wait_limit_ns = wait_ns;
  p.rows_routed = s.cap;
  p.rows_shared = s.T;
  return p;
}

}  // namespace

cudaError_t launch_backward_gemms(const Shape& s, const BackwardGemmArgs& a, int num_sms,
                                  unsigned int* status, uint64_t wait_ns, cudaStream_t st,
                                  const cudaEvent_t* events) {
  // prefill-sized segments run on CTA pairs (grouped_gemm_bwd_pair.cu)
  const bool small = (int64_t)s.T * s.k <= (int64_t)24 * s.E;
  if (!small && pair_backward_supported(s))
    return launch_backward_gemms_pair(s, a, num_sms, status, wait_ns, st, events);
  auto mark = [&](int i) {
    return events != nullptr && events[i] != nullptr ? cudaEventRecord(events[i], st)
                                                     : cudaSuccess;
  };
  const bool shared = s.S > 0 && s.T > 0;
  const int SI = s.S * s.I;
  CUtensorMap m[6];
  cudaError_t err;
  if (s.S > 0 && s.T == 0) {  // no tokens: the shared experts' gradients are zero
    const size_t bytes = (size_t)s.S * s.I * s.d * (a.dw_f32 ? 4 : 2);
    if ((err = cudaMemsetAsync(a.dws1, 0, bytes, st)) != cudaSuccess ||
        (err = cudaMemsetAsync(a.dws3, 0, bytes, st)) != cudaSuccess ||
        (err = cudaMemsetAsync(a.dws2, 0, bytes, st)) != cudaSuccess)
      return err;
  }

  // ---- dH = dY W2 with the SwiGLU backward -> dGU = [dG | dU]
  {
    bool ok = make_map3(&m[0], a.w2, s.I, (uint64_t)s.E * s.d, 1, 64) &&
              make_map3(&m[2], a.dy_perm, s.d, s.cap, 1, kBoxB);
    m[1] = m[0];
    if (shared)
      ok = ok && make_map3(&m[3], a.ws2, s.I, s.d, s.S, 64) &&
           make_map3(&m[5], a.dy, s.d, s.T, 1, kBoxB);
    else
      m[3] = m[0], m[5] = m[2];
    m[4] = m[3];
    if (!ok) return cudaErrorInvalidValue;
    BwdParams p = base_params(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? 1 : 0;
    p.mt_routed = s.I / 128;
    p.mt_shared = SI / 128;
    p.kit_routed = s.d / kBK;
    p.kit_shared = s.d / kBK;
    p.out_routed = a.dgu_perm;
    p.ld_routed = 2 * s.I;
    p.out_shared = a.dgu_shared;
    p.ld_shared = 2 * SI;
    p.g_routed = a.g_perm;
    p.u_routed = a.u_perm;
    p.g_shared = a.g_shared;
    p.u_shared = a.u_shared;
    p.ld_gu_routed = s.I;
    p.ld_gu_shared = SI;
    p.ucol_routed = s.I;
    p.ucol_shared = SI;
    if ((err = launch_bwd<kDgradDown>(m, p, num_sms, st)) != cudaSuccess) return err;
    if ((err = mark(0)) != cudaSuccess) return err;
  }
  // ---- dW2 = dY^T H (routed) and dWs2[s] = dy^T H_shared[:, s]
  {
    bool ok = make_map3(&m[0], a.dy_perm, s.d, s.cap, 1, 64) &&
              make_map3(&m[2], a.h_perm, s.I, s.cap, 1, 64);
    m[1] = m[0];
    if (shared)
      ok = ok && make_map3(&m[3], a.dy, s.d, s.T, 1, 64) &&
           make_map3(&m[5], a.h_shared, SI, s.T, 1, 64);
    else
      m[3] = m[0], m[5] = m[2];
    m[4] = m[3];
    if (!ok) return cudaErrorInvalidValue;
    BwdParams p = base_params(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? s.S : 0;
    p.mt_routed = p.mt_shared = s.d / 128;
    p.ntot_routed = p.ntot_shared = s.I;
    p.nt_routed = p.nt_shared = (int)ceil_div(s.I, kNT);
    p.a_col0_routed = 0;
    p.a_col0_shared = 0;
    p.a_step_shared = 0;
    p.b_col0_routed = 0;
    p.b_col0_shared = 0;
    p.b_step_shared = s.I;
    p.out_routed = a.dw2;
    p.out_shared = a.dws2;
    p.out_f32 = a.dw_f32 ? 1 : 0;
    p.gstride_routed = p.gstride_shared = (int64_t)s.d * s.I;
    if ((err = launch_bwd<kWgrad>(m, p, num_sms, st)) != cudaSuccess) return err;
    if ((err = mark(1)) != cudaSuccess) return err;
  }
  // ---- dX = dG W1 + dU W3 (token rows), shared into fp32
  {
    bool ok = make_map3(&m[0], a.w1, s.d, (uint64_t)s.E * s.I, 1, 64) &&
              make_map3(&m[1], a.w3, s.d, (uint64_t)s.E * s.I, 1, 64) &&
              make_map3(&m[2], a.dgu_perm, 2 * (uint64_t)s.I, s.cap, 1, kBoxB);
    if (shared)
      ok = ok && make_map3(&m[3], a.ws1, s.d, SI, 1, 64) &&
           make_map3(&m[4], a.ws3, s.d, SI, 1, 64) &&
           make_map3(&m[5], a.dgu_shared, 2 * (uint64_t)SI, s.T, 1, kBoxB);
    else
      m[3] = m[0], m[4] = m[1], m[5] = m[2];
    if (!ok) return cudaErrorInvalidValue;
    BwdParams p = base_params(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? 1 : 0;
    p.mt_routed = p.mt_shared = s.d / 128;
    p.kit_routed = 2 * s.I / kBK;
    p.kit_shared = 2 * SI / kBK;
    p.ksplit_routed = s.I / kBK;
    p.ksplit_shared = SI / kBK;
    p.out_routed = a.dx_perm;
    p.ld_routed = s.d;
    p.out_shared = a.dx_shared;
    p.ld_shared = s.d;
    p.shared_f32 = 1;
    if ((err = launch_bwd<kDgradUp>(m, p, num_sms, st)) != cudaSuccess) return err;
    if ((err = mark(2)) != cudaSuccess) return err;
  }
  // ---- dW1 = dG^T X and dW3 = dU^T X in one launch (routed: x_perm;
  // shared: x): M tiles [0, I/128) write dW1, [I/128, 2I/128) write dW3, and
  // both halves stream the same token panels
  {
    bool ok = make_map3(&m[0], a.dgu_perm, 2 * (uint64_t)s.I, s.cap, 1, 64) &&
              make_map3(&m[2], a.x_perm, s.d, s.cap, 1, 64);
    m[1] = m[0];
    if (shared)
      ok = ok && make_map3(&m[3], a.dgu_shared, 2 * (uint64_t)SI, s.T, 1, 64) &&
           make_map3(&m[5], a.x, s.d, s.T, 1, 64);
    else
      m[3] = m[0], m[5] = m[2];
    m[4] = m[3];
    if (!ok) return cudaErrorInvalidValue;
    BwdParams p = base_params(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? s.S : 0;
    p.mt_routed = p.mt_shared = 2 * s.I / 128;
    p.m_split = s.I / 128;
    p.ntot_routed = p.ntot_shared = s.d;
    p.nt_routed = p.nt_shared = (int)ceil_div(s.d, kNT);
    p.a_col0_routed = 0;
    p.a_col1_routed = s.I;
    p.a_col0_shared = 0;
    p.a_col1_shared = SI;
    p.a_step_shared = s.I;
    p.b_col0_routed = 0;
    p.b_col0_shared = 0;
    p.b_step_shared = 0;
    p.out_routed = a.dw1;
    p.out2_routed = a.dw3;
    p.out_shared = a.dws1;
    p.out2_shared = a.dws3;
    p.out_f32 = a.dw_f32 ? 1 : 0;
    p.gstride_routed = p.gstride_shared = (int64_t)s.I * s.d;
    if ((err = launch_bwd<kWgrad>(m, p, num_sms, st)) != cudaSuccess) return err;
  }
  return mark(3);
}

}  // namespace moe

MOE_CHECKS_UNIT(grouped_gemm_bwd)
