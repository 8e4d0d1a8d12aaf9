// Paired-CTA backward grouped GEMMs (tcgen05 cta_group::2, sm_100a).
//
// The three backward GEMM kinds of grouped_gemm_bwd.cu on clusters of two
// CTAs, built like the forward's paired kernel:
//
//   kPDgradDown  dH = dY W2 per segment (M = I features, N = tokens, K = d),
//                SwiGLU backward in the epilogue -> dGU = [dG | dU]
//   kPDgradUp    dX = dG W1 + dU W3 (M = d features, N = tokens, K = 2I)
//   kPWgrad      dW = A^T B with K = the segment's tokens (M, N = weight
//                rows / columns): dW2 = dY^T H, [dW1 ; dW3] = [dG | dU]^T X
//
//  * M = 256 per MMA: each CTA loads its own 128 rows of A and half of B's N
//    columns; the even CTA ("leader") issues tcgen05.mma.cta_group::2, which
//    reads A and B from both CTAs and leaves each CTA's 128 accumulator rows
//    in its own TMEM.  Against one CTA per 128 x 256 tile this halves the B
//    bytes each SM loads (dgrads) or cuts the A + B bytes by a third (wgrads).
//  * A is always MN-major in shared memory (weights enter the dgrads
//    transposed, activations enter the wgrads transposed): TMA boxes of 64
//    MN x 64 K rows with the 128-byte swizzle, 64-wide MN blocks 8 KB apart.
//    B is K-major (tokens) in the dgrads and MN-major in the wgrads.
//  * 128-deep K stages (two 64-deep sub-blocks) in one ring filled by two
//    producer warps per CTA (A and B), both arming the leader's full barrier;
//    the leader's commits free a stage in both CTAs at once; both epilogues
//    arrive on the leader's tmem-empty barrier.  No TMA load uses cluster
//    multicast.
//  * M tiles that reach past a group's extent (I = 1408 is 5.5 tiles of 256)
//    read zero-filled A rows from TMA and their CTA skips the epilogue.
//  * Bounded waits and drains as in the other kernels; a cluster barrier at
//    the end keeps either CTA's shared memory alive until its peer is done.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "moe_internal.h"
#include "checks.cuh"
#include "ptx_sm100.cuh"

namespace moe {
namespace {

enum PBwdMode : int { kPDgradDown = 0, kPDgradUp = 1, kPWgrad = 2 };

constexpr int kBK = 128;            // dgrads: K per stage, two 64-deep sub-blocks
constexpr int kSubK = 64;
constexpr int kMnBlk = 8192;        // one MN-major box: 64 MN x 64 K rows of bf16
constexpr int kASub = 2 * kMnBlk;   // this CTA's 128 A rows for one K sub-block

constexpr int kBoxB = 128;          // token rows per K-major B box (this CTA's half)
constexpr int kBSub = 128 * 128;    // one K sub-block of this CTA's B (either layout)
constexpr int kMaxStages = 6;
// weight gradients: stage depth and count (the same 192 KB in flight as 6
// stages of 64 measured 3-5 % slower than 3 stages of 128)
constexpr int kWgradKSubs = 2, kWgradStages = 3;
constexpr int kNT = 256;            // N per pair tile
// Warp 0 A producer, 1 MMA, 2 .. 1 + epi_warps(MODE) epilogue, the next one
// B producer.  The weight gradients and the dH dgrad run 8 epilogue warps
// (two per TMEM lane quarter): the weight gradients' tiles are short (K = one
// segment's few hundred tokens) and the dH epilogue carries the SwiGLU
// backward, so with 4 warps their epilogues would pace the MMAs.  The
// weight-gradient warps take alternate 64-column blocks, the dH warps form two
// groups of 4 that take alternate 32-token chunks.
constexpr int epi_warps(int mode) { return mode == 1 ? 4 : 8; }
constexpr int block_threads(int mode) { return 32 * (3 + epi_warps(mode)); }
constexpr int kEpiStaging = 32768;  // epilogue staging bytes, shared by the epilogue warps
constexpr uint32_t kTmemCols = 2 * kNT;
constexpr int kMaxGroups = 136;     // 128 routed + up to 8 shared groups
constexpr uint64_t kDrainLimitNs = 1000000000ull;

struct PBParams {
  int E;          // routed groups
  int n_sgroups;  // shared groups (dgrads: 0 or 1; wgrad: S or 0)
  int T, I, d;
  const int32_t* offsets;
  int mt_routed, mt_shared;      // M tiles (of 256) per group
  int mext_routed, mext_shared;  // M extent per group (rows past it are skipped)
  int nt_routed, nt_shared;      // wgrad: N tiles per group
  int ntot_routed, ntot_shared;  // wgrad: N extent of the output
  int kit_routed, kit_shared;    // dgrads: K chunks of kBK
  int ksplit_routed, ksplit_shared;  // dgrad-up: first chunk read from the second A map
  // wgrad A columns: an M row r < a_split (or any r when a_split == 0) reads
  // column a_c0 + r, a row past it column a_c1 + r - a_split; shared groups
  // add s * a_step_shared.  Rows past a_split go to the second output.
  int a_split;
  int a_c0_routed, a_c1_routed, a_c0_shared, a_c1_shared, a_step_shared;
  int b_c0_routed, b_c0_shared, b_step_shared;  // wgrad B columns
  void *out_routed, *out_shared;  // dgrads (the weight gradients go through TMA store maps)
  int ld_routed, ld_shared;
  int out_f32;                    // wgrad: the store maps are fp32 (else bf16)
  const float *g_routed, *u_routed, *g_shared, *u_shared;  // dgrad-down fp32 pre-activations
  int ld_gu_routed, ld_gu_shared;
  int ucol_routed, ucol_shared;  // dgrad-down: column of dU in the output
  unsigned int* status;
  uint64_t wait_limit_ns;
  int64_t rows_routed, rows_shared;  // dgrads: token rows of the routed / shared buffers
};

struct PBTile {
  int g;         // group
  int mt;        // M tile (of 256)
  int row0;      // dgrads: first token row of the tile; wgrad: of the group
  int nrows;     // dgrads: token rows of the tile; wgrad: K rows of the group
  int n;         // MMA N (dgrads: rows rounded to 16; wgrad: columns of the tile)
  int ncol0;     // wgrad: first output column of the tile
  int kchunks;   // K chunks of kBK
  int last_k16;  // MMAs of K = 16 in the last chunk
};

struct PBCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
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

__device__ __forceinline__ bool pb_aborted(const PBCtl& c) {
  return *reinterpret_cast<const volatile int*>(&c.abort_flag) != 0;
}

__device__ __forceinline__ void pb_timeout(PBCtl& c, const PBParams& p) {
  *reinterpret_cast<volatile int*>(&c.abort_flag) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0u, (unsigned)DEV_TIMEOUT);
}

// MN-major operand in 64 MN x 64 K boxes (128-byte rows, one per K index,
// 128-byte swizzle): 8-row atoms 1024 bytes apart along K, 64-wide MN blocks
// 8192 bytes apart.  K advances 16 rows = 2048 bytes per MMA.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(kMnBlk >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16, D fp32, A/B bf16, M = 256 (pair), A MN-major, B MN-major when b_mn.
__device__ __forceinline__ uint32_t idesc_pbwd(uint32_t n, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((n >> 3) << 17) | ((256u >> 4) << 24);
}

template <int MODE, int BK>
__device__ __forceinline__ PBTile pb_decode(const PBCtl& c, const PBParams& p, int tile) {
  int lo = 0, hi = c.ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  PBTile t;
  t.g = lo;
  const bool routed = lo < p.E;
  const int local = tile - c.prefix[lo];
  if (MODE == kPWgrad) {
    const int nt = routed ? p.nt_routed : p.nt_shared;
    const int ntot = routed ? p.ntot_routed : p.ntot_shared;
    t.mt = local / nt;
    const int ntile = local - t.mt * nt;
    t.ncol0 = ntile * kNT;
    t.n = min(kNT, ntot - t.ncol0);
    t.row0 = c.row0[lo];
    t.nrows = c.rows[lo];
    t.kchunks = (t.nrows + BK - 1) / BK;
    const int rem = t.nrows - (t.kchunks - 1) * BK;
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
    t.last_k16 = BK / 16;
  }
  return t;
}

__device__ __forceinline__ float pb_sigmoid(float g) { return 1.0f / (1.0f + __expf(-g)); }

// KSUBS 64-deep K sub-blocks per stage, STAGES stages in the ring.
template <int MODE, int KSUBS, int STAGES>
__global__ void __launch_bounds__(block_threads(MODE), 1)
grouped_gemm_bwd_pair_kernel(const __grid_constant__ CUtensorMap tmA_r,
                             const __grid_constant__ CUtensorMap tmA2_r,
                             const __grid_constant__ CUtensorMap tmB_r,
                             const __grid_constant__ CUtensorMap tmA_s,
                             const __grid_constant__ CUtensorMap tmA2_s,
                             const __grid_constant__ CUtensorMap tmB_s,
                             const __grid_constant__ CUtensorMap tmO_r,
                             const __grid_constant__ CUtensorMap tmO2_r,
                             const __grid_constant__ CUtensorMap tmO_s,
                             const __grid_constant__ CUtensorMap tmO2_s, const PBParams p) {
  static_assert(epi_warps(kPDgradUp) == 4 && epi_warps(kPWgrad) == 8 &&
                    epi_warps(kPDgradDown) == 8,
                "epi_warps keys on the mode values");
  constexpr int kEpiWarps = epi_warps(MODE);
  constexpr int kEpiThreads = 32 * kEpiWarps;
  constexpr int kBWarp = 2 + kEpiWarps;  // B producer
  // weight-gradient store buffers per epilogue warp (4 KB each: 32 rows x 64 columns)
  constexpr int kBufs = kEpiStaging / 4096 / kEpiWarps;
  static_assert(kBufs >= 1, "staging");
  constexpr int BK = KSUBS * kSubK;
  constexpr int kABytes = KSUBS * kASub;
  constexpr int kStageBytes = kABytes + KSUBS * kBSub;
  static_assert(STAGES <= kMaxStages, "barrier arrays");
  __shared__ PBCtl ctl;
  extern __shared__ uint8_t dsmem_raw[];
  const uint32_t raw = smem_u32(dsmem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  // epilogue staging, 32 KB: per dH epilogue group the SwiGLU backward's dG
  // then dU tiles ([32][128] bf16 each), or per weight-gradient epilogue warp
  // one 4 KB store buffer (32 rows x 64 columns of bf16 or 32 x 32 of fp32,
  // 128-byte swizzle)
  uint8_t* epi = dsmem_raw + (sbase - raw) + STAGES * kStageBytes;
  uint16_t* epi_g = reinterpret_cast<uint16_t*>(epi);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

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
        if (MODE == kPWgrad)
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
      for (int s = 0; s < STAGES; ++s) {
        mbar_init(smem_u32(&ctl.full[s]), 2);  // armed by both of the leader's producers
        mbar_init(smem_u32(&ctl.empty[s]), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&ctl.tfull[b]), 1);
        mbar_init(smem_u32(&ctl.tempty[b]), 2 * kEpiWarps);  // one lane per epilogue warp, both CTAs
      }
      mbar_init(smem_u32(&ctl.drain), 1);
      ctl.abort_flag = 0;
      fence_mbar_init();
      prefetch_tmap(&tmA_r);
      prefetch_tmap(&tmB_r);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(smem_u32(&ctl.tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();  // barriers of both CTAs exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = ctl.tmem_base;
  const int total = ctl.total_tiles;
  const int pair = (int)cluster_id_x();
  const int npairs = (int)nclusters_x();

  if (warp == 0 || warp == kBWarp) {
    // ========== TMA producers (both CTAs): warp 0 operand A, warp 6 operand B ==========
    if (lane == 0) {
      const bool wA = warp == 0;
      // the weights of the dgrads stream from HBM once; activations are re-read
      const uint64_t pol =
          (wA && MODE != kPWgrad) ? policy_evict_normal() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // leader: stages whose full phase it armed
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const PBTile t = pb_decode<MODE, BK>(ctl, p, tile);
        const bool routed = t.g < p.E;
        const int s_idx = t.g - p.E;
        const int r0 = t.mt * 256 + (int)rank * 128;  // this CTA's first M row
        const int half = t.n >> 1;                    // this CTA's share of N
        uint32_t tx_pair;
        if (wA) {
          tx_pair = 2u * kABytes;
        } else if (MODE == kPWgrad) {
          tx_pair = 2u * KSUBS * (uint32_t)((half / 64) * kMnBlk);
        } else {
          tx_pair = 2u * KSUBS * (uint32_t)(kBoxB * 128);
        }
        // A coordinates that do not change along K
        int a_x = 0, a_plane = 0;
        const CUtensorMap* tA = routed ? &tmA_r : &tmA_s;
        if (MODE == kPDgradDown) {
          if (routed) {
            a_x = r0;
          } else {
            a_plane = r0 / p.I;  // the shared experts' W2 are the planes of a 3-D map
            a_x = r0 - a_plane * p.I;
          }
        } else if (MODE == kPDgradUp) {
          a_x = r0;
        } else {
          const bool second = p.a_split > 0 && r0 >= p.a_split;
          a_x = second ? (routed ? p.a_c1_routed : p.a_c1_shared + s_idx * p.a_step_shared) +
                             r0 - p.a_split
                       : (routed ? p.a_c0_routed : p.a_c0_shared + s_idx * p.a_step_shared) + r0;
        }
        const int b_col = MODE == kPWgrad
                              ? (routed ? p.b_c0_routed : p.b_c0_shared + s_idx * p.b_step_shared) +
                                    t.ncol0 + (int)rank * half
                              : 0;
        const int b_row = t.row0 + (int)rank * half;  // dgrads: this CTA's token rows
        const CUtensorMap* tB = routed ? &tmB_r : &tmB_s;
        for (int kc = 0; kc < t.kchunks; ++kc) {
          if (pb_aborted(ctl)) { ok = false; break; }
          if (!mbar_wait_bounded(smem_u32(&ctl.empty[stage]), phase ^ 1u, p.wait_limit_ns)) {
            pb_timeout(ctl, p);
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&ctl.full[stage]);
          const uint32_t fb = mapa_shared(fb_local, 0);  // the leader's barrier
          if (leader) {
            mbar_arrive_expect_tx(fb_local, tx_pair);
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint32_t sB = sA + kABytes;
          for (int j = 0; j < KSUBS; ++j) {  // the 64-deep K sub-blocks
            const int kj = kc * BK + j * kSubK;
            if (wA) {
              if (MODE == kPDgradDown) {
                // A = W2^T: K rows d of W2 [.., d, I], M columns = features
                const int krow = routed ? t.g * p.d + kj : kj;
                for (int h = 0; h < 2; ++h)
                  tma_load_3d_pair(sA + j * kASub + h * kMnBlk, tA, fb, a_x + h * 64, krow, a_plane,
                                   pol);
              } else if (MODE == kPDgradUp) {
                // A = [W1 ; W3]^T: K rows f of W1 / W3 [.., I, d], M columns = d
                const int ks = routed ? p.ksplit_routed : p.ksplit_shared;
                const bool second = kc >= ks;
                const CUtensorMap* tAk =
                    routed ? (second ? &tmA2_r : &tmA_r) : (second ? &tmA2_s : &tmA_s);
                const int krow = (second ? kj - ks * BK : kj) + (routed ? t.g * p.I : 0);
                for (int h = 0; h < 2; ++h)
                  tma_load_3d_pair(sA + j * kASub + h * kMnBlk, tAk, fb, a_x + h * 64, krow, 0,
                                   pol);
              } else {
                // A = activations^T: K rows = the group's tokens
                for (int h = 0; h < 2; ++h)
                  tma_load_3d_pair(sA + j * kASub + h * kMnBlk, tA, fb, a_x + h * 64, t.row0 + kj,
                                   0, pol);
              }
            } else {
              if (MODE == kPWgrad) {
                for (int h = 0; h < half / 64; ++h)
                  tma_load_3d_pair(sB + j * kBSub + h * kMnBlk, tB, fb, b_col + h * 64,
                                   t.row0 + kj, 0, pol);
              } else {
                tma_load_3d_pair(sB + j * kBSub, tB, fb, kj, b_row, 0, pol);
              }
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (leader) {
        // every phase this CTA armed completes only once both CTAs' bytes land
        for (int s = 0; s < STAGES; ++s) {
          if (((armed >> s) & 1u) &&
              !mbar_wait_bounded(smem_u32(&ctl.full[s]), (armed_parity >> s) & 1u, kDrainLimitNs))
            pb_timeout(ctl, p);
        }
      } else if (!ok) {
        // a peer that gave up cannot see its last copies land (they signal the
        // leader); give them time before the cluster barrier lets both exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer (leader only) =================
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const PBTile t = pb_decode<MODE, BK>(ctl, p, tile);
        const uint32_t idesc = idesc_pbwd((uint32_t)t.n, MODE == kPWgrad);
        if (pb_aborted(ctl) ||
            !mbar_wait_bounded(smem_u32(&ctl.tempty[acc]), acc_phase ^ 1u, p.wait_limit_ns)) {
          if (!pb_aborted(ctl)) pb_timeout(ctl, p);
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * kNT);
        for (int kc = 0; kc < t.kchunks; ++kc) {
          if (pb_aborted(ctl) ||
              !mbar_wait_bounded(smem_u32(&ctl.full[stage]), phase, p.wait_limit_ns)) {
            if (!pb_aborted(ctl)) pb_timeout(ctl, p);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint32_t sB = sA + kABytes;
          const int nk16 = (kc == t.kchunks - 1) ? t.last_k16 : BK / 16;
          for (int k8 = 0; k8 < nk16; ++k8) {
            const uint32_t offa = (k8 >> 2) * kASub + (k8 & 3) * 2048;
            const uint64_t ad = sdesc_mn_sw128(sA + offa);
            const uint64_t bd = MODE == kPWgrad
                                    ? sdesc_mn_sw128(sB + (k8 >> 2) * kBSub + (k8 & 3) * 2048)
                                    : sdesc_kmajor_sw128(sB + (k8 >> 2) * kBSub + (k8 & 3) * 32);
            mma_bf16_ss_pair(dt, ad, bd, idesc, (kc | k8) != 0 ? 1u : 0u);
          }
          mma_commit_pair(smem_u32(&ctl.empty[stage]), 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(smem_u32(&ctl.tfull[acc]), 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      mma_commit_pair(smem_u32(&ctl.drain), 0x1);
      if (!mbar_wait_bounded(smem_u32(&ctl.drain), 0, kDrainLimitNs)) pb_timeout(ctl, p);
    }
  } else {
    // ============ epilogue (warps 2 .. kBWarp - 1, both CTAs) ============
    const int q = warp & 3;          // TMEM lane quarter a warp may read
    const int mrow = q * 32 + lane;  // accumulator row = TMEM lane
    const int et = threadIdx.x - 64; // 0 .. kEpiThreads - 1 over the epilogue warps
    const int ew = warp - 2;         // epilogue warp index
    // dH dgrad: two groups of 4 warps, each over all 128 TMEM lanes, take
    // alternate 32-token chunks with their own staging and named barrier
    constexpr bool kGroups = MODE == kPDgradDown && kEpiWarps == 8;
    constexpr int kGrpThreads = 128;
    constexpr int kChunkStep = kGroups ? 64 : 32;
    const int grp = kGroups ? (ew >> 2) : 0;
    const int eg = et & (kGrpThreads - 1);  // thread index inside the group
    uint16_t* const gbuf = epi_g + grp * (2 * 32 * 128);
    uint16_t* const ubuf = gbuf + 32 * 128;
    const int gbar = 1 + 2 * grp;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&ctl.tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&ctl.tempty[1]), 0);
    // SwiGLU backward: this thread's feature (its TMEM lane) of the fp32 g / u
    // rows of one 32-token chunk.  For each token the warp's 32 lanes read 32
    // consecutive features (128 coalesced bytes); the loads are issued before
    // the accumulator is read so their latency overlaps it.
    float gv[32], uv[32];
    auto load_gu = [&](const PBTile& t, int f0, int c0) {
      const bool routed = t.g < p.E;
      const float* gsrc = routed ? p.g_routed : p.g_shared;
      const float* usrc = routed ? p.u_routed : p.u_shared;
      const int ldgu = routed ? p.ld_gu_routed : p.ld_gu_shared;
      int nj = min(32, t.nrows - c0);
      if (!MOE_CHECK((int64_t)t.row0 + c0 + nj <= (routed ? p.rows_routed : p.rows_shared)))
        nj = 0;
      const size_t at0 = (size_t)(t.row0 + c0) * ldgu + f0 + mrow;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        gv[j] = j < nj ? gsrc[at0 + (size_t)j * ldgu] : 0.f;
        uv[j] = j < nj ? usrc[at0 + (size_t)j * ldgu] : 0.f;
      }
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t nstore = 0;  // weight-gradient chunks this CTA has handed to TMA
    // hand the accumulator back to the MMA warp: every lane's TMEM reads have
    // completed (tcgen05.wait::ld), then one lane per warp arrives on the
    // leader's barrier (one arrival instead of 32 remote ones)
    auto release = [&](int a) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(smem_u32(&ctl.tempty[a]));
        else
          mbar_arrive_remote(a ? tempty_leader1 : tempty_leader0);
      }
    };
    for (int tile = pair; tile < total; tile += npairs) {
      const PBTile t = pb_decode<MODE, BK>(ctl, p, tile);
      const bool routed = t.g < p.E;
      const int r0 = t.mt * 256 + (int)rank * 128;
      // rows past the group's M extent hold zero-filled products: skipped
      const bool live = r0 < (routed ? p.mext_routed : p.mext_shared);
      bool bad = pb_aborted(ctl);
      if (!bad && !mbar_wait_bounded(smem_u32(&ctl.tfull[acc]), acc_phase, p.wait_limit_ns)) {
        pb_timeout(ctl, p);
        bad = true;
      }
      if (bar_red_or(2, kEpiThreads, bad)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (uint32_t)(acc * kNT) + ((uint32_t)(q * 32) << 16);
      const int ncols = MODE == kPWgrad ? t.n : t.nrows;
      bool freed = false;
      if (MODE == kPWgrad && live) {
        // dW[group][row0 + mrow][ncol0 + c0 .. + 64] in bf16.  Each warp owns
        // 32 rows: it stages its 32 x 64 block (128-byte rows, 128-byte
        // swizzle) and hands it to a TMA store (whole rows, coalesced) with
        // warp-level syncs only; its two buffers alternate, and the TMEM loads
        // of the next 64 columns are in flight while these are staged.
        const bool second = p.a_split > 0 && r0 >= p.a_split;
        const CUtensorMap* tO =
            second ? (routed ? &tmO2_r : &tmO2_s) : (routed ? &tmO_r : &tmO_s);
        const int orow = (second ? r0 - p.a_split : r0) + q * 32;
        const int plane = routed ? t.g : t.g - p.E;
        const bool zero = t.kchunks == 0;  // no tokens: the gradient is zero
        auto pack = [&](const uint32_t (&v)[32], uint32_t (&w)[16]) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float lo = zero ? 0.f : __uint_as_float(v[2 * i]);
            const float hi = zero ? 0.f : __uint_as_float(v[2 * i + 1]);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);  // one paired cvt
            w[i] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        };
        // tile widths are multiples of 64: columns go 64 at a time (va, vb);
        // the warps sharing a lane quarter take alternate 64-column blocks
        constexpr int kStep = 64 * (kEpiWarps / 4);
        const int cfirst = 64 * (ew >> 2);
        uint32_t va[32], vb[32];
        if (p.out_f32) {
          // fp32: each 32-column half is one 32 x 32 box (128-byte rows),
          // staged in this warp's buffer after the previous store has read it
          auto put = [&](const uint32_t (&v)[32], int col) {
            uint8_t* buf = epi + ew * (kBufs * 4096) + (nstore % kBufs) * 4096u;
            if (lane == 0) bulk_wait_group_read<kBufs - 1>();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {  // 128-byte swizzle: 16-byte chunk c ^ (row % 8)
              const int phys = c ^ (lane & 7);
              *reinterpret_cast<uint4*>(buf + lane * 128 + phys * 16) =
                  zero ? make_uint4(0, 0, 0, 0)
                       : make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(tO, smem_u32(buf), t.ncol0 + col, orow, plane);
              bulk_commit_group();
            }
            ++nstore;
          };
          for (int c0 = cfirst; c0 < ncols; c0 += kStep) {
            tmem_ld_32x32b_x32(tbase + (uint32_t)c0, va);
            tmem_ld_32x32b_x32(tbase + (uint32_t)(c0 + 32), vb);
            tmem_ld_wait();
            if (c0 + kStep >= ncols) {  // this warp's last columns are in registers
              release(acc);
              freed = true;
            }
            put(va, c0);
            put(vb, c0 + 32);
          }
        } else {
        if (cfirst < ncols) {
          tmem_ld_32x32b_x32(tbase + (uint32_t)cfirst, va);
          tmem_ld_32x32b_x32(tbase + (uint32_t)(cfirst + 32), vb);
          tmem_ld_wait();
        }
        if (cfirst + kStep >= ncols) {  // every column is in registers: the MMAs may go on
          release(acc);
          freed = true;
        }
        for (int c0 = cfirst; c0 < ncols; c0 += kStep) {
          uint32_t wa[16], wb[16];
          pack(va, wa);
          pack(vb, wb);
          const bool more = c0 + kStep < ncols;
          if (more) {
            tmem_ld_32x32b_x32(tbase + (uint32_t)(c0 + kStep), va);
            tmem_ld_32x32b_x32(tbase + (uint32_t)(c0 + kStep + 32), vb);
          }
          uint8_t* buf = epi + ew * (kBufs * 4096) + (nstore % kBufs) * 4096u;
          // the store that last used buf has read it
          if (lane == 0) bulk_wait_group_read<kBufs - 1>();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {  // 128-byte swizzle: 16-byte chunk c ^ (row % 8)
            const int phys = c ^ (lane & 7);
            const uint32_t* w = c < 4 ? &wa[4 * c] : &wb[4 * (c - 4)];
            *reinterpret_cast<uint4*>(buf + lane * 128 + phys * 16) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(tO, smem_u32(buf), t.ncol0 + c0, orow, plane);
            bulk_commit_group();
          }
          ++nstore;
          if (more) {
            tmem_ld_wait();
            if (c0 + 2 * kStep >= ncols) {  // those were this warp's last columns
              release(acc);
              freed = true;
            }
          }
        }
        }
      }
      for (int c0 = grp * 32; MODE != kPWgrad && live && c0 < ncols; c0 += kChunkStep) {
        if (MODE == kPDgradDown) load_gu(t, r0, c0);
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
        tmem_ld_wait();
        int nj = min(32, ncols - c0);
        if (!MOE_CHECK((int64_t)t.row0 + c0 + nj <= (routed ? p.rows_routed : p.rows_shared)))
          nj = 0;  // token rows outside the buffer: recorded, stores skipped
        if (MODE == kPDgradDown) {
          // SwiGLU backward on a 32-token x 128-feature tile staged in smem
          uint16_t* out = static_cast<uint16_t*>(routed ? p.out_routed : p.out_shared);
          const int ldo = routed ? p.ld_routed : p.ld_shared;
          const int ucol = routed ? p.ucol_routed : p.ucol_shared;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j < nj) {
              const float dh = __uint_as_float(v[j]);
              const float g = gv[j];
              const float u = uv[j];
              const float sg = pb_sigmoid(g);
              const float dg = dh * u * (sg * (1.0f + g * (1.0f - sg)));
              const float du = dh * (g * sg);
              gbuf[j * 128 + mrow] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
              ubuf[j * 128 + mrow] = __bfloat16_as_ushort(__float2bfloat16_rn(du));
            }
          }
          named_bar_sync(gbar, kGrpThreads);
          for (int i = eg; i < 32 * 16; i += kGrpThreads) {
            const int r = i >> 4, cv = i & 15;
            if (r < nj) {
              const size_t row = (size_t)(t.row0 + c0 + r) * ldo + r0 + cv * 8;
              *reinterpret_cast<uint4*>(out + row) =
                  *reinterpret_cast<const uint4*>(gbuf + r * 128 + cv * 8);
              *reinterpret_cast<uint4*>(out + row + ucol) =
                  *reinterpret_cast<const uint4*>(ubuf + r * 128 + cv * 8);
            }
          }
          named_bar_sync(gbar, kGrpThreads);  // the tile is reused by the next chunk
        } else {
          // dX for feature r0 + mrow and the tile's token rows, fp32
          const int col = r0 + mrow;
          float* out = static_cast<float*>(routed ? p.out_routed : p.out_shared);
          const int ldo = routed ? p.ld_routed : p.ld_shared;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nj) out[(size_t)(t.row0 + c0 + j) * ldo + col] = __uint_as_float(v[j]);
        }
      }
      if (!freed) release(acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (MODE == kPWgrad && lane == 0) bulk_wait_group<0>();  // every store has landed
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();  // neither CTA leaves while its peer may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
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

// Output (inner, rows, planes) written by TMA stores of 128-byte x 32-row
// boxes with the 128-byte swizzle (the staging layout of the weight-gradient
// epilogue): 64 columns of bf16, or 32 columns of fp32 when f32.
bool make_store_map3(CUtensorMap* m, void* base, uint64_t inner, uint64_t rows, uint64_t planes,
                     bool f32) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {inner, rows, planes};
  cuuint64_t strides[2] = {inner * es, inner * rows * es};
  cuuint32_t box[3] = {f32 ? 32u : 64u, 32u, 1u};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base,
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// m[0..5]: operand maps; m[6..9]: output maps of the weight gradients.
template <int MODE, int KSUBS, int STAGES>
cudaError_t launch_pb(const CUtensorMap* m, const PBParams& p, int num_sms, cudaStream_t st) {
  constexpr size_t smem = (size_t)STAGES * KSUBS * (kASub + kBSub) + 32768 + 1024;
  static_assert(smem + sizeof(PBCtl) <= 232448, "shared memory budget");
  auto kern = grouped_gemm_bwd_pair_kernel<MODE, KSUBS, STAGES>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(block_threads(MODE), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_clusters = 0;
  cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
      max_clusters <= 0)
    max_clusters = num_sms / 2;
  if (max_clusters > num_sms / 2) max_clusters = num_sms / 2;
  cfg.gridDim = dim3((unsigned)(2 * max_clusters), 1, 1);
  err = cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], m[8],
                           m[9], p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

PBParams pb_base(const Shape& s, const int32_t* offsets, unsigned int* status, uint64_t wait_ns) {
  PBParams p{};
  p.E = s.E;
  p.T = s.T;
  p.I = s.I;
  p.d = s.d;
  p.offsets = offsets;
  p.status = status;
  p.wait_limit_ns = wait_ns;
  p.rows_routed = s.cap;
  p.rows_shared = s.T;
  return p;
}

}  // namespace

bool pair_backward_supported(const Shape& s) {
  return s.I % 128 == 0 && s.d % 128 == 0 && s.E + s.S <= kMaxGroups && s.T > 0;
}

cudaError_t launch_backward_gemms_pair(const Shape& s, const BackwardGemmArgs& a, int num_sms,
                                       unsigned int* status, uint64_t wait_ns, cudaStream_t st,
                                       const cudaEvent_t* events) {
  auto mark = [&](int i) {
    return events != nullptr && events[i] != nullptr ? cudaEventRecord(events[i], st)
                                                     : cudaSuccess;
  };
  const bool shared = s.S > 0;
  const int SI = s.S * s.I;
  CUtensorMap m[10];
  cudaError_t err;

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
    m[6] = m[7] = m[8] = m[9] = m[0];  // no output maps
    PBParams p = pb_base(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? 1 : 0;
    p.mt_routed = (int)ceil_div(s.I, 256);
    p.mt_shared = (int)ceil_div(SI, 256);
    p.mext_routed = s.I;
    p.mext_shared = SI;
    p.kit_routed = p.kit_shared = s.d / kBK;
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
    if ((err = launch_pb<kPDgradDown, 2, 3>(m, p, num_sms, st)) != cudaSuccess) return err;
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
    ok = ok && make_store_map3(&m[6], a.dw2, s.I, s.d, s.E, a.dw_f32);
    if (shared) ok = ok && make_store_map3(&m[8], a.dws2, s.I, s.d, s.S, a.dw_f32);
    else m[8] = m[6];
    m[7] = m[6];
    m[9] = m[8];
    if (!ok) return cudaErrorInvalidValue;
    PBParams p = pb_base(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? s.S : 0;
    p.mt_routed = p.mt_shared = (int)ceil_div(s.d, 256);
    p.mext_routed = p.mext_shared = s.d;
    p.ntot_routed = p.ntot_shared = s.I;
    p.nt_routed = p.nt_shared = (int)ceil_div(s.I, kNT);
    p.b_step_shared = s.I;
    p.out_f32 = a.dw_f32 ? 1 : 0;
    if ((err = launch_pb<kPWgrad, kWgradKSubs, kWgradStages>(m, p, num_sms, st)) != cudaSuccess) return err;
    if ((err = mark(1)) != cudaSuccess) return err;
  }
  // ---- dX = dG W1 + dU W3 (token rows), fp32
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
    m[6] = m[7] = m[8] = m[9] = m[0];  // no output maps
    PBParams p = pb_base(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? 1 : 0;
    p.mt_routed = p.mt_shared = (int)ceil_div(s.d, 256);
    p.mext_routed = p.mext_shared = s.d;
    p.kit_routed = 2 * s.I / kBK;
    p.kit_shared = 2 * SI / kBK;
    p.ksplit_routed = s.I / kBK;
    p.ksplit_shared = SI / kBK;
    p.out_routed = a.dx_perm;
    p.ld_routed = s.d;
    p.out_shared = a.dx_shared;
    p.ld_shared = s.d;
    if ((err = launch_pb<kPDgradUp, 2, 3>(m, p, num_sms, st)) != cudaSuccess) return err;
    if ((err = mark(2)) != cudaSuccess) return err;
  }
  // ---- [dW1 ; dW3] = [dG | dU]^T X in one launch (routed: x_perm; shared: x)
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
    ok = ok && make_store_map3(&m[6], a.dw1, s.d, s.I, s.E, a.dw_f32) &&
         make_store_map3(&m[7], a.dw3, s.d, s.I, s.E, a.dw_f32);
    if (shared)
      ok = ok && make_store_map3(&m[8], a.dws1, s.d, s.I, s.S, a.dw_f32) &&
           make_store_map3(&m[9], a.dws3, s.d, s.I, s.S, a.dw_f32);
    else
      m[8] = m[6], m[9] = m[7];
    if (!ok) return cudaErrorInvalidValue;
    PBParams p = pb_base(s, a.offsets, status, wait_ns);
    p.n_sgroups = shared ? s.S : 0;
    p.mt_routed = p.mt_shared = (int)ceil_div(2 * s.I, 256);
    p.mext_routed = p.mext_shared = 2 * s.I;
    p.a_split = s.I;
    p.a_c0_routed = 0;
    p.a_c1_routed = s.I;
    p.a_c0_shared = 0;
    p.a_c1_shared = SI;
    p.a_step_shared = s.I;
    p.ntot_routed = p.ntot_shared = s.d;
    p.nt_routed = p.nt_shared = (int)ceil_div(s.d, kNT);
    p.out_f32 = a.dw_f32 ? 1 : 0;
    if ((err = launch_pb<kPWgrad, kWgradKSubs, kWgradStages>(m, p, num_sms, st)) != cudaSuccess) return err;
  }
  return mark(3);
}

}  // namespace moe

MOE_CHECKS_UNIT(grouped_gemm_bwd_pair)
