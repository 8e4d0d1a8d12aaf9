// Paired-CTA grouped expert GEMMs for prefill-sized segments (tcgen05
// cta_group::2, sm_100a).
//
// Same computation as grouped_gemm.cu (swap-AB: weights are M, a segment's
// tokens are N; gate/up stacked in the A tile so SwiGLU runs in the epilogue;
// shared experts as one more group), with the MMA spread over a cluster of
// two CTAs on neighbouring SMs:
//
//  * M = 256 per MMA: each CTA loads its own 128 weight rows (gate/up GEMM:
//    64 W1 + 64 W3 rows; down GEMM: 128 W2 rows) and HALF of the tile's
//    token rows; the even CTA ("leader") issues tcgen05.mma.cta_group::2,
//    which reads A and B from both CTAs' shared memory and leaves each CTA's
//    128 output rows in its own TMEM.  Per SM this halves the token bytes
//    loaded per flop.  The weights (from HBM) and the token rows (from L2)
//    have separate producer warps that fill one ring of three 64 KB stages.
//  * Both CTAs' TMA loads complete on the leader's "full" barrier (the
//    leader arms it with the pair's byte count); the leader's MMA commits
//    arrive on the "empty" / "tmem full" barriers of both CTAs at once; both
//    epilogues arrive on the leader's "tmem empty" barrier.  No TMA load uses
//    cluster multicast.
//  * Bounded waits and drains as in the 1-CTA kernel; the cluster barrier at
//    the end keeps either CTA's shared memory alive until its peer is done.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "moe_internal.h"
#include "checks.cuh"
#include "ptx_sm100.cuh"

namespace moe {
namespace {

enum PairMode : int { kPairSwiGLU = 0, kPairDown = 1 };

constexpr int kBK = 128;                    // K per stage: two 64-wide swizzle sub-tiles
constexpr int kSubK = 64;
constexpr int kBoxB = 128;                  // one TMA box covers this CTA's token rows
constexpr int kASub = 128 * 128;            // one K sub-tile of this CTA's 128 A rows
constexpr int kABytes = 2 * kASub;
constexpr int kNT = 256;                    // tokens per pair tile
constexpr int kBSub = (kNT / 2) * 128;     // one K sub-tile of this CTA's half of the tokens
constexpr int kBBytes = 2 * kBSub;
// One ring of 64 KB stages (weights 32 KB, tokens 32 KB) filled by two
// producer threads -- weights and tokens -- that both arm the stage's full
// barrier; one commit frees a stage after its 8 MMAs.
constexpr int kStages = 3;
constexpr int kThreads = 224;               // warp 6 = token producer
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = 2 * kNT;
constexpr int kMaxGroups = 129;
constexpr uint64_t kDrainLimitNs = 1000000000ull;

struct PairParams {
  int E, has_shared, T;
  int ft_routed, ft_shared;   // feature tiles per group (gate/up: 128 features; down: 256)
  int kit_routed, kit_shared;
  int k_plane;
  int a_rows_group;
  const int32_t* offsets;
  void* out_routed;
  int ld_routed;
  void* out_shared;
  int ld_shared;
  int shared_f32;
  int routed_f32;  // down GEMM: routed rows stored in fp32 (else bf16)
  float *g_routed, *u_routed, *g_shared, *u_shared;  // training: fp32 pre-activations
  unsigned int* status;
  uint64_t wait_limit_ns;
  int64_t rows_routed, rows_shared;  // token rows of the routed / shared buffers
  // down GEMM split over K (ksplit > 1): tile (.., ks) sums K chunks
  // [ks*kit_split, ..) and stores fp32 partials to out_split[ks][row][col]
  int ksplit, kit_split;
  float* out_split;
};

struct PTile {
  int g, ft, row0, nrows, nmma, kit;
  int ks, k0;  // split of K (down GEMM with ksplit > 1) and its first K chunk
};

struct PCtl {
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

__device__ __forceinline__ PTile pdecode(const PCtl& c, const PairParams& p, int tile) {
  int lo = 0, hi = c.ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (c.prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  PTile t;
  t.g = lo;
  const bool routed = lo < p.E;
  const int nft = routed ? p.ft_routed : p.ft_shared;
  const int nks = p.ksplit > 1 ? p.ksplit : 1;
  const int local = tile - c.prefix[lo];
  t.ks = local % nks;
  const int rest = local / nks;
  const int tt = rest / nft;
  t.ft = rest - tt * nft;
  t.row0 = c.row0[lo] + tt * kNT;
  t.nrows = min(kNT, c.rows[lo] - tt * kNT);
  t.nmma = (t.nrows + 15) & ~15;
  const int kit = routed ? p.kit_routed : p.kit_shared;
  t.k0 = nks > 1 ? t.ks * p.kit_split : 0;
  t.kit = nks > 1 ? min(p.kit_split, kit - t.k0) : kit;
  return t;
}

__device__ __forceinline__ bool paborted(const PCtl& c) {
  return *reinterpret_cast<const volatile int*>(&c.abort_flag) != 0;
}

__device__ __forceinline__ void precord_timeout(PCtl& c, const PairParams& p) {
  *reinterpret_cast<volatile int*>(&c.abort_flag) = 1;
  if (p.status != nullptr) atomicCAS(p.status, 0u, (unsigned)DEV_TIMEOUT);
}

__device__ __forceinline__ float psilu(float g) { return g / (1.0f + __expf(-g)); }

// kind::f16, D fp32, A/B bf16 K-major, M = 256 (pair), N given.
__device__ __forceinline__ uint32_t idesc_pair(uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((256u >> 4) << 24);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA_r,
                         const __grid_constant__ CUtensorMap tmA2_r,
                         const __grid_constant__ CUtensorMap tmB_r,
                         const __grid_constant__ CUtensorMap tmA_s,
                         const __grid_constant__ CUtensorMap tmA2_s,
                         const __grid_constant__ CUtensorMap tmB_s, const PairParams p) {
  __shared__ PCtl ctl;
  extern __shared__ uint8_t dsmem_raw[];
  const uint32_t raw = smem_u32(dsmem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  // SwiGLU epilogue staging: one 32-token chunk of u, then of g ([32][64] fp32 each)
  float* up_buf =
      reinterpret_cast<float*>(dsmem_raw + (sbase - raw) + kStages * (kABytes + kBBytes));
  float* gate_buf = up_buf + 32 * 64;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (warp == 0) {
    const int G = p.E + (p.has_shared ? 1 : 0);
    int local[5];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const int g = lane * 5 + i;
      int tiles = 0;
      if (g < G) {
        int r0, nr, nft;
        if (g < p.E) {
          r0 = p.offsets[g];
          nr = p.offsets[g + 1] - r0;
          nft = p.ft_routed;
        } else {
          r0 = 0;
          nr = p.T;
          nft = p.ft_shared;
        }
        if (nr < 0) nr = 0;
        ctl.row0[g] = r0;
        ctl.rows[g] = nr;
        tiles = (int)ceil_div(nr, kNT) * nft * (p.ksplit > 1 ? p.ksplit : 1);
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
        mbar_init(smem_u32(&ctl.full[s]), 2);  // armed by both producers
        mbar_init(smem_u32(&ctl.empty[s]), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&ctl.tfull[b]), 1);
        mbar_init(smem_u32(&ctl.tempty[b]), 2 * (kEpiThreads / 32));  // a lane per epilogue warp
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

  if (warp == 0 || warp == 6) {
    // ========== TMA producers (both CTAs): warp 0 weights, warp 6 tokens ==========
    if (lane == 0) {
      const bool wA = warp == 0;
      const int nst = kStages;
      uint64_t* fullb = ctl.full;
      uint64_t* emptyb = ctl.empty;
      const uint64_t pol = wA ? policy_evict_normal() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // leader: stages whose full phase it armed
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const PTile t = pdecode(ctl, p, tile);
        const bool routed = t.g < p.E;
        const CUtensorMap* tA = routed ? &tmA_r : &tmA_s;
        const CUtensorMap* tA2 = routed ? &tmA2_r : &tmA2_s;
        const CUtensorMap* tB = routed ? &tmB_r : &tmB_s;
        const int half = t.nmma >> 1;
        const int nbox = (half + kBoxB - 1) / kBoxB;
        const uint32_t tx_pair = wA ? 2u * kABytes : 2u * 2u * (uint32_t)(nbox * kBoxB * 128);
        const int arow = MODE == kPairSwiGLU
                             ? (routed ? t.g * p.a_rows_group : 0) + t.ft * 128 + (int)rank * 64
                             : (routed ? t.g * p.a_rows_group : 0) + t.ft * 256 + (int)rank * 128;
        const int brow = t.row0 + (int)rank * half;
        for (int kc = 0; kc < t.kit; ++kc) {
          if (paborted(ctl)) { ok = false; break; }
          if (!mbar_wait_bounded(smem_u32(&emptyb[stage]), phase ^ 1u, p.wait_limit_ns)) {
            precord_timeout(ctl, p);
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&fullb[stage]);
          const uint32_t fb = mapa_shared(fb_local, 0);  // the leader's barrier
          if (leader) {
            mbar_arrive_expect_tx(fb_local, tx_pair);
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          }
          const int kk = (t.k0 + kc) * kBK;
          const uint32_t sA = sbase + stage * (kABytes + kBBytes);
          const uint32_t sB = sA + kABytes;
          for (int j = 0; j < 2; ++j) {  // the two 64-wide K sub-tiles
            const int kj = kk + j * kSubK;
            if (wA) {
              if (MODE == kPairSwiGLU) {
                tma_load_3d_pair(sA + j * kASub, tA, fb, kj, arow, 0, pol);
                tma_load_3d_pair(sA + j * kASub + kASub / 2, tA2, fb, kj, arow, 0, pol);
              } else {
                const int plane = kj / p.k_plane;
                tma_load_3d_pair(sA + j * kASub, tA, fb, kj - plane * p.k_plane, arow, plane, pol);
              }
            } else {
              for (int b = 0; b < nbox; ++b)
                tma_load_3d_pair(sB + j * kBSub + b * kBoxB * 128, tB, fb, kj, brow + b * kBoxB, 0,
                                 pol);
            }
          }
          if (++stage == nst) { stage = 0; phase ^= 1u; }
        }
      }
      if (leader) {
        // every phase this CTA armed completes only once both CTAs' bytes land
        for (int s = 0; s < nst; ++s) {
          if (((armed >> s) & 1u) &&
              !mbar_wait_bounded(smem_u32(&fullb[s]), (armed_parity >> s) & 1u, kDrainLimitNs))
            precord_timeout(ctl, p);
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
        const PTile t = pdecode(ctl, p, tile);
        const uint32_t idesc = idesc_pair((uint32_t)t.nmma);
        if (paborted(ctl) ||
            !mbar_wait_bounded(smem_u32(&ctl.tempty[acc]), acc_phase ^ 1u, p.wait_limit_ns)) {
          if (!paborted(ctl)) precord_timeout(ctl, p);
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem_base + (uint32_t)(acc * kNT);
        for (int kc = 0; kc < t.kit; ++kc) {
          if (paborted(ctl) ||
              !mbar_wait_bounded(smem_u32(&ctl.full[stage]), phase, p.wait_limit_ns)) {
            if (!paborted(ctl)) precord_timeout(ctl, p);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * (kABytes + kBBytes);
          const uint32_t sB = sA + kABytes;
#pragma unroll
          for (int k8 = 0; k8 < kBK / 16; ++k8) {
            const uint32_t off = (k8 >> 2) * kASub + (k8 & 3) * 32;
            const uint32_t offb = (k8 >> 2) * kBSub + (k8 & 3) * 32;
            const uint64_t ad = sdesc_kmajor_sw128(sA + off);
            const uint64_t bd = sdesc_kmajor_sw128(sB + offb);
            mma_bf16_ss_pair(dt, ad, bd, idesc, (kc | k8) != 0 ? 1u : 0u);
          }
          mma_commit_pair(smem_u32(&ctl.empty[stage]), 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(smem_u32(&ctl.tfull[acc]), 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      mma_commit_pair(smem_u32(&ctl.drain), 0x1);
      if (!mbar_wait_bounded(smem_u32(&ctl.drain), 0, kDrainLimitNs)) precord_timeout(ctl, p);
    }
  } else {
    // ================= epilogue (warps 2..5, both CTAs) =================
    // (warps 0, 1 and 6 are handled above)
    const int q = warp & 3;
    const int frow = q * 32 + lane;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&ctl.tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&ctl.tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const PTile t = pdecode(ctl, p, tile);
      bool bad = paborted(ctl);
      if (!bad && !mbar_wait_bounded(smem_u32(&ctl.tfull[acc]), acc_phase, p.wait_limit_ns)) {
        precord_timeout(ctl, p);
        bad = true;
      }
      if (bar_red_or(2, kEpiThreads, bad)) break;
      tc_fence_after();
      const bool routed = t.g < p.E;
      const uint32_t tbase = tmem_base + (uint32_t)(acc * kNT) + ((uint32_t)(q * 32) << 16);
      for (int c0 = 0; c0 < t.nrows; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)c0, v);
        tmem_ld_wait();
        int nj = min(32, t.nrows - c0);
        if (!MOE_CHECK((int64_t)t.row0 + c0 + nj <= (routed ? p.rows_routed : p.rows_shared)))
          nj = 0;  // rows outside the buffer: recorded, stores skipped
        if (MODE == kPairDown) {
          const int col = t.ft * 256 + (int)rank * 128 + frow;
          if (routed && p.ksplit > 1) {  // one K split's fp32 partial
            float* out = p.out_split + (size_t)t.ks * p.rows_routed * p.ld_routed;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nj) out[(size_t)(t.row0 + c0 + j) * p.ld_routed + col] = __uint_as_float(v[j]);
          } else if (routed && p.routed_f32) {
            float* out = static_cast<float*>(p.out_routed);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nj) out[(size_t)(t.row0 + c0 + j) * p.ld_routed + col] = __uint_as_float(v[j]);
          } else if (routed) {
            uint16_t* out = static_cast<uint16_t*>(p.out_routed);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nj)
                out[(size_t)(t.row0 + c0 + j) * p.ld_routed + col] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
          } else if (p.shared_f32) {
            float* out = static_cast<float*>(p.out_shared);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nj) out[(size_t)(t.row0 + c0 + j) * p.ld_shared + col] = __uint_as_float(v[j]);
          } else {
            uint16_t* out = static_cast<uint16_t*>(p.out_shared);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nj)
                out[(size_t)(t.row0 + c0 + j) * p.ld_shared + col] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
          }
        } else if (routed && p.ksplit > 1) {
          // one K split's fp32 pre-activations: g from the gate lanes (q < 2),
          // u from the up lanes, as planes 0 and 1 of the split's partial
          const int col = t.ft * 128 + (int)rank * 64 + (frow & 63);
          float* out = p.out_split +
                       ((size_t)t.ks * 2 + (q < 2 ? 0 : 1)) * p.rows_routed * p.ld_routed;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nj) out[(size_t)(t.row0 + c0 + j) * p.ld_routed + col] = __uint_as_float(v[j]);
        } else {
          // the gate lanes (q < 2) stage g, the up lanes (q >= 2) stage u;
          // then each pair of warps finishes half of the chunk's tokens for
          // the same 64 features, so all four warps share the SwiGLU and the
          // stores of h (and, training, of g and u)
          const int f = frow & 63;  // feature of this lane's accumulator row
          float* mine = q < 2 ? gate_buf : up_buf;
#pragma unroll
          for (int j = 0; j < 32; ++j) mine[j * 64 + f] = __uint_as_float(v[j]);
          named_bar_sync(1, kEpiThreads);
          uint16_t* out = static_cast<uint16_t*>(routed ? p.out_routed : p.out_shared);
          const int ld = routed ? p.ld_routed : p.ld_shared;
          const int col = t.ft * 128 + (int)rank * 64 + f;
          const int jb = q < 2 ? 0 : 16;  // this warp's half of the tokens
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = jb + jj;
            if (j < nj) {
              const float h = psilu(gate_buf[j * 64 + f]) * up_buf[j * 64 + f];
              out[(size_t)(t.row0 + c0 + j) * ld + col] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(h));
            }
          }
          float* gs = routed ? p.g_routed : p.g_shared;
          float* us = routed ? p.u_routed : p.u_shared;
          if (gs != nullptr) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = jb + jj;
              if (j < nj) {
                const size_t at = (size_t)(t.row0 + c0 + j) * ld + col;
                gs[at] = gate_buf[j * 64 + f];
                us[at] = up_buf[j * 64 + f];
              }
            }
          }
          named_bar_sync(1, kEpiThreads);
        }
      }
      // every lane's TMEM reads are done: one lane per warp hands the
      // accumulator back (one arrival instead of 32 remote ones)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(smem_u32(&ctl.tempty[acc]));
        else
          mbar_arrive_remote(acc ? tempty_leader1 : tempty_leader0);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
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
cudaError_t launch_pair(const CUtensorMap* m, const PairParams& p, int num_sms, cudaStream_t st) {
  constexpr size_t smem = (size_t)kStages * (kABytes + kBBytes) + 2 * 32 * 64 * 4 + 1024;
  static_assert(smem + sizeof(PCtl) <= 232448, "shared memory budget");
  auto kern = grouped_gemm_pair_kernel<MODE>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one resident cluster per SM pair: as many as the device can hold at once
  int max_clusters = 0;
  cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess ||
      max_clusters <= 0)
    max_clusters = num_sms / 2;
  if (max_clusters > num_sms / 2) max_clusters = num_sms / 2;
  cfg.gridDim = dim3((unsigned)(2 * max_clusters), 1, 1);
  err = cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], m[5], p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

bool pair_gemms_supported(const Shape& s) { return s.I % 128 == 0 && s.d % 256 == 0; }

namespace {

// y[i] = bf16(sum over the K splits of part[s][i]), s ascending, fp32 sum.
__global__ void split_sum_kernel(const float* __restrict__ part, int splits, int64_t n4,
                                 uint16_t* __restrict__ y) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 acc = reinterpret_cast<const float4*>(part)[i];
  for (int sp = 1; sp < splits; ++sp) {
    const float4 v = reinterpret_cast<const float4*>(part + (size_t)sp * n4 * 4)[i];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  reinterpret_cast<uint2*>(y)[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                              *reinterpret_cast<const uint32_t*>(&hi));
}

// h[i] = bf16(silu(g) * u) with g and u the fp32 sums over the K splits of
// part[s][0][i] and part[s][1][i], s ascending (plane = n4 float4s).
__global__ void split_swiglu_kernel(const float* __restrict__ part, int splits, int64_t n4,
                                    uint16_t* __restrict__ h) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4* p4 = reinterpret_cast<const float4*>(part);
  float4 g = p4[i], u = p4[n4 + i];
  for (int sp = 1; sp < splits; ++sp) {
    const float4 a = p4[(size_t)sp * 2 * n4 + i], b = p4[(size_t)sp * 2 * n4 + n4 + i];
    g.x += a.x; g.y += a.y; g.z += a.z; g.w += a.w;
    u.x += b.x; u.y += b.y; u.z += b.z; u.w += b.w;
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(psilu(g.x) * u.x, psilu(g.y) * u.y);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(psilu(g.z) * u.z, psilu(g.w) * u.w);
  reinterpret_cast<uint2*>(h)[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                              *reinterpret_cast<const uint32_t*>(&hi));
}

// K splits for a GEMM of `base` pair tiles of `kit` K chunks each: the fewest
// splits among those with the least (waves x K chunks per tile).  Only a GEMM
// of at most two waves of pair tiles is split, and only when that cuts the
// cost by 15 % or more: the fp32 partials take a round trip through HBM.
int plan_k_splits(int base, int kit, int num_sms) {
  const int pairs = num_sms / 2;
  if (pairs <= 0 || base > 2 * pairs || kit < 4) return 1;
  int best = 1;
  const int64_t unsplit = ceil_div(base, pairs) * kit;
  int64_t best_cost = unsplit;
  for (int sp = 2; sp <= 8 && sp <= kit / 2; ++sp) {
    if (ceil_div(kit, sp) * (sp - 1) >= kit) continue;  // every split gets K chunks
    const int64_t cost = ceil_div((int64_t)base * sp, pairs) * ceil_div(kit, sp);
    if (cost < best_cost) {
      best_cost = cost;
      best = sp;
    }
  }
  return best_cost * 100 <= unsplit * 85 ? best : 1;
}

}  // namespace

int down_k_splits(const Shape& s, int num_sms) {
  if (!uses_pair_gemms(s) || s.S > 0 || s.E != 1) return 1;
  return plan_k_splits((int)ceil_div(s.T, kNT) * (s.d / 256), s.I / kBK, num_sms);
}

int up_k_splits(const Shape& s, int num_sms) {
  if (!uses_pair_gemms(s) || s.S > 0 || s.E != 1) return 1;
  return plan_k_splits((int)ceil_div(s.T, kNT) * (s.I / 128), s.d / kBK, num_sms);
}

cudaError_t launch_grouped_gemms_pair(const Shape& s, const GroupedGemmArgs& a, int num_sms,
                                      unsigned int* status, uint64_t wait_limit_ns,
                                      cudaStream_t st, cudaEvent_t between) {
  const bool shared = a.part != GroupedGemmArgs::kRoutedOnly && s.S > 0 && a.x != nullptr &&
                      a.ws1 != nullptr && a.ws3 != nullptr && a.ws2 != nullptr &&
                      a.h_shared != nullptr && a.y_shared != nullptr && s.T > 0;
  // routed groups in the schedule (none for a shared-only launch; the routed
  // maps stay valid, they are just not used)
  const int E_run = a.part == GroupedGemmArgs::kSharedOnly ? 0 : s.E;
  const int SI = s.S * s.I;
  CUtensorMap m[6];
  cudaError_t err;
  // ---- gate/up GEMM + SwiGLU: a pair tile = 128 features x up to 256 tokens
  {
    bool ok = make_map3(&m[0], a.w1, s.d, (uint64_t)s.E * s.I, 1, 64) &&
              make_map3(&m[1], a.w3, s.d, (uint64_t)s.E * s.I, 1, 64) &&
              make_map3(&m[2], a.x_perm, s.d, s.cap, 1, kBoxB);
    if (shared)
      ok = ok && make_map3(&m[3], a.ws1, s.d, SI, 1, 64) &&
           make_map3(&m[4], a.ws3, s.d, SI, 1, 64) && make_map3(&m[5], a.x, s.d, s.T, 1, kBoxB);
    else
      m[3] = m[0], m[4] = m[1], m[5] = m[2];
    if (!ok) return cudaErrorInvalidValue;
    PairParams p{};
    p.E = E_run;
    p.has_shared = shared ? 1 : 0;
    p.T = s.T;
    p.ft_routed = s.I / 128;
    p.ft_shared = SI / 128;
    p.kit_routed = p.kit_shared = s.d / kBK;
    p.k_plane = s.d;
    p.a_rows_group = s.I;
    p.offsets = a.offsets;
    p.out_routed = a.h_perm;
    p.ld_routed = s.I;
    p.out_shared = a.h_shared;
    p.ld_shared = SI;
    p.g_routed = a.g_perm;
    p.u_routed = a.u_perm;
    p.g_shared = shared ? a.g_shared : nullptr;
    p.u_shared = shared ? a.u_shared : nullptr;
    p.status = status;
    p.rows_routed = s.cap;
    p.rows_shared = s.T;
    p.wait_limit_ns = wait_limit_ns;
    const bool split = a.up_splits > 1 && a.up_partials != nullptr && !shared &&
                       a.g_perm == nullptr;
    if (split) {
      p.ksplit = a.up_splits;
      p.kit_split = (int)ceil_div(p.kit_routed, a.up_splits);
      p.out_split = a.up_partials;
    }
    if ((err = launch_pair<kPairSwiGLU>(m, p, num_sms, st)) != cudaSuccess) return err;
    if (split) {
      const int64_t n4 = (int64_t)s.cap * s.I / 4;
      split_swiglu_kernel<<<(unsigned)ceil_div(n4, 256), 256, 0, st>>>(
          a.up_partials, (int)ceil_div(p.kit_routed, p.kit_split), n4, a.h_perm);
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (between != nullptr && (err = cudaEventRecord(between, st)) != cudaSuccess) return err;
  }
  // ---- down GEMM: a pair tile = 256 output features x up to 256 tokens
  {
    bool ok = make_map3(&m[0], a.w2, s.I, (uint64_t)s.E * s.d, 1, 128) &&
              make_map3(&m[2], a.h_perm, s.I, s.cap, 1, kBoxB);
    m[1] = m[0];
    if (shared)
      ok = ok && make_map3(&m[3], a.ws2, s.I, s.d, s.S, 128) &&
           make_map3(&m[5], a.h_shared, SI, s.T, 1, kBoxB);
    else
      m[3] = m[0], m[5] = m[2];
    m[4] = m[3];
    if (!ok) return cudaErrorInvalidValue;
    PairParams p{};
    p.E = E_run;
    p.has_shared = shared ? 1 : 0;
    p.T = s.T;
    p.ft_routed = p.ft_shared = s.d / 256;
    p.kit_routed = s.I / kBK;
    p.kit_shared = SI / kBK;
    p.k_plane = s.I;
    p.a_rows_group = s.d;
    p.offsets = a.offsets;
    p.out_routed = a.y_perm;
    p.routed_f32 = a.y_perm_f32 ? 1 : 0;
    p.ld_routed = s.d;
    p.out_shared = a.y_shared;
    p.ld_shared = s.d;
    p.shared_f32 = 1;
    p.status = status;
    p.rows_routed = s.cap;
    p.rows_shared = s.T;
    p.wait_limit_ns = wait_limit_ns;
    const bool split = a.down_splits > 1 && a.down_partials != nullptr && !shared &&
                       !a.y_perm_f32;
    if (split) {
      p.ksplit = a.down_splits;
      p.kit_split = (int)ceil_div(p.kit_routed, a.down_splits);
      p.out_split = a.down_partials;
    }
    if ((err = launch_pair<kPairDown>(m, p, num_sms, st)) != cudaSuccess) return err;
    if (split) {
      const int64_t n4 = (int64_t)s.cap * s.d / 4;
      split_sum_kernel<<<(unsigned)ceil_div(n4, 256), 256, 0, st>>>(
          a.down_partials, (int)ceil_div(p.kit_routed, p.kit_split), n4,
          static_cast<uint16_t*>(a.y_perm));
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
  }
  return cudaSuccess;
}

}  // namespace moe

MOE_CHECKS_UNIT(grouped_gemm_pair)
