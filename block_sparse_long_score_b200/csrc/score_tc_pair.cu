// score_tc_pair.cu -- strided antidiagonal scoring on the 5th-generation tensor
// cores ("XAttention: Block Sparse Attention with Antidiagonal Scoring",
// §2.1 Importance Prediction and Algorithm 1).
//
// The reshaped product x = Q_r K_r^T is a plain GEMM per (batch, query head):
// M = N = R = L/S reshaped rows, K-dim = S*d. Reshaped query row rho is
// [Q[rho S + S-1], ..., Q[rho S]] and reshaped key row c is
// [K[c S], ..., K[c S + S-1]], so k-chunk i (d features) of the GEMM pairs query
// token rho S + S-1-i with key token c S + i. Neither operand is copied: Q and
// K are read through 4-D TMA views [head][rho][s][feature], and chunk i takes
// s = S-1-i on the query side and s = i on the key side. The query sub-row of
// each chunk comes from a permutation argument, so the same kernel also runs
// the diagonal (s = i) and random-permutation patterns of the sparsity-pattern
// ablation (Knowl 9 of the chapterpal page, §3.4 Ablation Study).
//
// A pair of CTAs on two SMs (a cluster of two) computes one 256 (rho) x 256
// (c) tile with M = 256 MMAs of both tensor cores (tcgen05 cta_group::2):
// each CTA loads its own 128 query rows and half (128) of the key rows, so a
// pipeline stage is 32 KB per CTA instead of the 48 KB a lone CTA needs for a
// 128 x 256 tile. The kernel is bound by how many bytes the TMA ring keeps in
// flight, and this is what lets seven stages fit. Each CTA's TMEM holds the
// accumulator of its 128 rows over all 256 columns, twice (512 columns), so
// the epilogue of one tile overlaps the MMAs of the next.
// The epilogue never stores x: for each row it reduces every key block's r
// reshaped columns to one partial log2-sum-exp, which the reduce kernel turns
// into block probabilities. Causal tiles entirely above the reshaped diagonal
// are skipped.
//
// Warp roles (384 threads a CTA, 1 CTA per SM, persistent over tiles):
//   warp 0      TMA producer of this CTA's halves; rank 0 also posts the
//               stage's expected bytes (both CTAs' loads complete on rank 0's
//               barrier)
//   warp 1      TMEM allocator (both CTAs); MMA issuer (rank 0 only, one
//               elected lane), whose commits reach both CTAs' barriers
//   warps 4..11 epilogue, one TMEM lane (= one reshaped row) per thread;
//               warps 4..7 reduce columns 0..127 of a tile, warps 8..11 columns
//               128..255 (a key block never straddles the halves: r divides 128);
//               both CTAs free an accumulator on rank 0's barrier
#include "score_epi.cuh"

namespace xattn {
namespace {

using namespace scoring;

constexpr int kBM = 128;            // reshaped query rows per CTA (256 per pair)
constexpr int kPairM = 2 * kBM;     // reshaped query rows per tile
constexpr int kBNHalf = kBN / 2;    // key rows each CTA loads
constexpr int kStages = 7;
constexpr int kABytes = kBM * kBK * 2;       // 16 KB
constexpr int kBBytes = kBNHalf * kBK * 2;   // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 8;       // two epilogue warpgroups, one per 128-column half
constexpr int kThreads = 128 + kEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(kPairM, kBN, 0, 0);
constexpr uint16_t kPairMask = 0x3;  // both CTAs of the cluster


struct Smem {
  uint64_t full[kStages];    // rank 0: both CTAs' halves of the stage landed
  uint64_t empty[kStages];   // both: the pair MMAs of the stage are done
  uint64_t acc_full[2];      // both: the tile's MMAs are done
  uint64_t acc_empty[2];     // rank 0: both CTAs' epilogues read the accumulator
  uint64_t mma_done;         // rank 0: every MMA the CTA issued has completed
  uint32_t tmem_base;
  int abort;
};

// Number of causal tiles in tile rows [0, m): tile row i (256 reshaped rows)
// needs key tiles nt with nt*256 <= i*256 + 255, i.e. min(NT, i + 1) tiles, so
// rows below NT hold m(m+1)/2 and every later row NT.
__host__ __device__ __forceinline__ long long tiles_before(int m, int NT) {
  const long long mu = m < NT ? m : NT;
  return mu * (mu + 1) / 2 + static_cast<long long>(NT) * (m > NT ? m - NT : 0);
}

__device__ __forceinline__ void decode_tile(long long t, const Params& p, int& bh, int& mt,
                                            int& nt) {
  bh = static_cast<int>(t / p.tiles_per_head);
  int rem = static_cast<int>(t % p.tiles_per_head);
  if (!p.causal) {
    mt = rem / p.NT;
    nt = rem % p.NT;
    return;
  }
  // Causal: bisection on the closed-form count of tiles in rows [0, m).
  int lo = 0, hi = p.MT;  // invariant: tiles_before(lo) <= rem < tiles_before(hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tiles_before(mid, p.NT) <= rem) lo = mid; else hi = mid;
  }
  mt = lo;
  nt = rem - static_cast<int>(tiles_before(lo, p.NT));
}

__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stage_mem = base;
  Smem* sm = reinterpret_cast<Smem*>(base + kStages * kStageBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();            // 0 or 1 within the pair
  const long long pair = blockIdx.x >> 1;
  const long long npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm->acc_full[b], 1);
      mbar_init(&sm->acc_empty[b], 2 * kEpiWarps * 32);
    }
    mbar_init(&sm->mma_done, 1);
    sm->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers and TMEM exist before either touches the other's
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;

  if (warp == 0) {
    // -------------------------------------------------------- TMA producer
    // Both CTAs load their halves; the bytes complete on rank 0's full
    // barrier, where rank 0 posts the expected total of the pair.
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    for (long long t = pair; t < p.total_tiles && !*abort; t += npairs) {
      int bh, mt, nt;
      decode_tile(t, p, bh, mt, nt);
      const int kvbh = (bh / p.hq) * p.hkv + (bh % p.hq) / p.group;
      const int m0 = mt * kPairM + static_cast<int>(rank) * kBM;
      const int n0 = nt * kBN + static_cast<int>(rank) * kBNHalf;
      for (int i = 0; i < p.S && !*abort; ++i) {
        for (int f = 0; f < 2; ++f) {
          if (!warp_wait(&sm->empty[stage], phase ^ 1, abort)) break;
          if (elect_one()) {
            uint8_t* sa = stage_mem + stage * kStageBytes;
            const uint32_t full0 = mapa_shared(&sm->full[stage], 0);
            if (rank == 0) mbar_arrive_expect_tx(&sm->full[stage], 2 * kStageBytes);
            tma_load_4d_pair(sa, &tmQ, full0, f * kBK, p.perm.q[i], m0, bh);
            tma_load_4d_pair(sa + kABytes, &tmK, full0, f * kBK, i, n0, kvbh);
          }
          __syncwarp();
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
    if (*abort) {
      // This CTA's copies complete on rank 0's barrier, which it cannot wait
      // on: give any copy still in flight time to land before the final
      // cluster barrier (copies take microseconds).
      const unsigned long long t0 = globaltimer();
      while (issued > 0 && globaltimer() - t0 < 200000ull) {
      }
    }
  } else if (warp == 1 && rank == 0) {
    // -------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (long long t = pair; t < p.total_tiles; t += npairs, ++it) {
      const int buf = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      // both CTAs' epilogues arrive here (the peer's from its own SM)
      if (!warp_wait_cluster(&sm->acc_empty[buf], aph ^ 1, abort)) break;
      tc_fence_after();
      const uint32_t dacc = tmem + buf * kBN;
      const int ksteps = 2 * p.S;
      bool ok = true;
      for (int ks = 0; ks < ksteps; ++ks) {
        if (!warp_wait(&sm->full[stage], phase, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t sa = smem_u32(stage_mem + stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t da = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t db = smem_desc_sw128(sb + kk * 32, 16, 1024);
            umma_ss_pair(dacc, da, db, kIdesc, (ks | kk) != 0);
          }
          umma_commit_pair_mc(&sm->empty[stage], kPairMask);
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (elect_one()) umma_commit_pair_mc(&sm->acc_full[buf], kPairMask);
      __syncwarp();
    }
    // every MMA this thread issued (they write both CTAs' TMEM) completes
    // before the pair tears down
    if (elect_one()) umma_commit_pair_mc(&sm->mma_done, 0x1);
    __syncwarp();
    const uint32_t addr = smem_u32(&sm->mma_done);
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(addr, 0) && globaltimer() - t0 < kWaitLimitNs) {
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------- epilogue
    // warps 4..7 take columns 0..127 of the tile, warps 8..11 columns 128..255
    const int half = (warp - 4) / 4;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int it = 0;
    for (long long t = pair; t < p.total_tiles; t += npairs, ++it) {
      const int buf = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!warp_wait(&sm->acc_full[buf], aph, abort)) break;
      tc_fence_after();
      int bh, mt, nt;
      decode_tile(t, p, bh, mt, nt);
      const int m0 = mt * kPairM + static_cast<int>(rank) * kBM, n0 = nt * kBN;
      const int rho = m0 + row;
      const bool row_ok = rho < p.R;
      const int b = rho / p.r;
      const int jmax = p.causal ? b : p.NB - 1;
      float* prow = p.part + static_cast<size_t>(bh) * p.part_head +
                    part_row_offset(row_ok ? rho : 0, p.r, p.NB, p.causal != 0);
      const bool need_mask = (n0 + kBN > p.R) || (p.causal && n0 + kBN - 1 > m0);
      const uint32_t tacc = tmem + lane_addr + buf * kBN;
      switch (p.r) {
        case 1: epilogue_tile<1>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        case 2: epilogue_tile<2>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        case 4: epilogue_tile<4>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        case 8: epilogue_tile<8>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        case 16: epilogue_tile<16>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        case 32: epilogue_tile<32>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        case 64: epilogue_tile<64>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
        default: epilogue_tile<128>(tacc, rho, n0, p, prow, jmax, row_ok, need_mask, half); break;
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(&sm->acc_empty[buf], 0));
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees TMEM) while the other may still signal its
  // barriers or while pair MMAs may still write its TMEM
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
  if (threadIdx.x == 0 && sm->abort) atomicExch(p.status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_score_tc_pair(const Dims& D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                            const PermArg& perm, float* part, int* status, int num_sms,
                            cudaStream_t st) {
  Params p{};
  p.perm = perm;
  p.R = D.R;
  p.S = D.S;
  p.r = D.r;
  p.NB = D.NB;
  p.causal = D.causal;
  p.hq = D.hq;
  p.hkv = D.hkv;
  p.group = D.group;
  p.MT = (D.R + kPairM - 1) / kPairM;
  p.NT = (D.R + kBN - 1) / kBN;
  if (D.causal) {
    long long n = 0;
    for (int m = 0; m < p.MT; ++m) n += (m + 1 < p.NT) ? (m + 1) : p.NT;
    if (n != tiles_before(p.MT, p.NT)) return cudaErrorInvalidValue;  // closed form check
    p.tiles_per_head = static_cast<int>(n);
  } else {
    p.tiles_per_head = p.MT * p.NT;
  }
  p.total_tiles = static_cast<long long>(p.tiles_per_head) * D.batch * D.hq;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(double(D.d) * D.S));
  p.part = part;
  p.part_head = part_head_elems(D.NB, D.r, D.R, D.causal != 0);
  p.status = status;

  const size_t smem = 1024 + kStages * kStageBytes + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;

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
  // persistent pairs: as many as can be resident at once (a cluster needs
  // two free SMs of one GPC), never more than there are tiles
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1), 1, 1);
  int resident = 0;
  e = cudaOccupancyMaxActiveClusters(&resident, score_tc_kernel, &cfg);
  if (e != cudaSuccess) return e;
  long long pairs = resident;
  if (pairs > p.total_tiles) pairs = p.total_tiles;
  if (pairs < 1) pairs = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, score_tc_kernel, tmQ, tmK, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace xattn
