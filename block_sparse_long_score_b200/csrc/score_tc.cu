// score_tc.cu -- strided antidiagonal scoring on the 5th-generation tensor
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
// This kernel serves the short strides (S < 8: at most 8 k-steps of 64
// features a tile, where the epilogue, not the tensor core, bounds a tile);
// score_tc_pair.cu runs the longer ones on CTA pairs.
//
// Tiles are 128 (rho) x 256 (c), accumulated in TMEM (fp32), two accumulators
// (512 columns) so the epilogue of one tile overlaps the MMAs of the next.
// The epilogue never stores x: for each row it reduces every key block's r
// reshaped columns to one partial log2-sum-exp, which the reduce kernel turns
// into block probabilities. Causal tiles entirely above the reshaped diagonal
// are skipped.
//
// Warp roles (384 threads, 1 CTA per SM, persistent over tiles):
//   warp 0      TMA producer (one elected lane issues the copies)
//   warp 1      TMEM allocator + MMA issuer (one elected lane issues the MMAs)
//   warps 4..11 epilogue, one TMEM lane (= one reshaped row) per thread;
//               warps 4..7 reduce columns 0..127 of a tile, warps 8..11 columns
//               128..255 (a key block never straddles the halves: r divides 128)
#include "score_epi.cuh"

namespace xattn {
namespace {

using namespace scoring;

constexpr int kBM = 128;            // reshaped query rows per tile
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 8;       // two epilogue warpgroups, one per 128-column half
constexpr int kThreads = 128 + kEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, 0, 0);


struct Smem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

// Number of causal tiles in tile rows [0, m): sum over rows of min(NT, row/2 + 1).
// Rows below 2*NT are uncapped: sum_{i<m} (floor(i/2) + 1) = m + q(q-1) (m = 2q)
// or m + q^2 (m = 2q + 1).
__host__ __device__ __forceinline__ long long tiles_before(int m, int NT) {
  const long long mu = m < 2 * NT ? m : 2 * NT;
  const long long q = mu >> 1;
  const long long uncapped = mu + ((mu & 1) ? q * q : q * (q - 1));
  return uncapped + static_cast<long long>(NT) * (m > 2 * NT ? m - 2 * NT : 0);
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
  // Causal: tile row m needs key tiles nt with nt*256 <= m*128 + 127, i.e.
  // nt <= m / 2, so it holds min(NT, m/2 + 1) tiles. Bisection on the
  // closed-form count of tiles in rows [0, m).
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm->acc_full[b], 1);
      mbar_init(&sm->acc_empty[b], kEpiWarps * 32);
    }
    sm->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;

  // The producer and MMA roles run on whole warps (bookkeeping stays warp-
  // uniform); one elected lane issues each TMA copy, MMA and commit.
  if (warp == 0) {
    {
      // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (long long t = blockIdx.x; t < p.total_tiles && !*abort; t += gridDim.x) {
        int bh, mt, nt;
        decode_tile(t, p, bh, mt, nt);
        const int kvbh = (bh / p.hq) * p.hkv + (bh % p.hq) / p.group;
        const int m0 = mt * kBM, n0 = nt * kBN;
        for (int i = 0; i < p.S; ++i) {
          for (int f = 0; f < 2; ++f) {
            if (!warp_wait(&sm->empty[stage], phase ^ 1, abort)) goto producer_done;
            if (elect_one()) {
              uint8_t* sa = stage_mem + stage * kStageBytes;
              mbar_arrive_expect_tx(&sm->full[stage], kStageBytes);
              tma_load_4d(sa, &tmQ, &sm->full[stage], f * kBK, p.perm.q[i], m0, bh);
              tma_load_4d(sa + kABytes, &tmK, &sm->full[stage], f * kBK, i, n0, kvbh);
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
    producer_done:
      // Make sure no copy is still landing in shared memory before exit.
      if (*abort) {
        const long long n = issued < kStages ? issued : kStages;
        for (long long k = 1; k <= n; ++k) {
          const long long q = issued - k;
          const int s = static_cast<int>(q % kStages);
          const uint32_t ph = static_cast<uint32_t>((q / kStages) & 1);
          const uint32_t addr = smem_u32(&sm->full[s]);
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(addr, ph) && globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (long long t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!warp_wait(&sm->acc_empty[buf], aph ^ 1, abort)) break;
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
              umma_ss(dacc, da, db, kIdesc, (ks | kk) != 0);
            }
            umma_commit(&sm->empty[stage]);
          }
          __syncwarp();
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) umma_commit(&sm->acc_full[buf]);
        __syncwarp();
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------- epilogue
    // warps 4..7 take columns 0..127 of the tile, warps 8..11 columns 128..255
    const int half = (warp - 4) / 4;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int it = 0;
    for (long long t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!warp_wait(&sm->acc_full[buf], aph, abort)) break;
      tc_fence_after();
      int bh, mt, nt;
      decode_tile(t, p, bh, mt, nt);
      const int m0 = mt * kBM, n0 = nt * kBN;
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
      mbar_arrive(&sm->acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && sm->abort) atomicExch(p.status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_score_tc(const Dims& D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
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
  p.MT = (D.R + kBM - 1) / kBM;
  p.NT = (D.R + kBN - 1) / kBN;
  if (D.causal) {
    long long n = 0;
    for (int m = 0; m < p.MT; ++m) n += (m / 2 + 1 < p.NT) ? (m / 2 + 1) : p.NT;
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
  long long grid = p.total_tiles < num_sms ? p.total_tiles : num_sms;
  if (grid < 1) grid = 1;
  score_tc_kernel<<<static_cast<int>(grid), kThreads, smem, st>>>(tmQ, tmK, p);
  return cudaGetLastError();
}

}  // namespace xattn
