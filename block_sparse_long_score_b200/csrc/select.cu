// select.cu -- find_blocks threshold selection ("XAttention: Block Sparse
// Attention with Antidiagonal Scoring", §2.2 Threshold Block Selection: the
// smallest set of blocks whose probability mass reaches tau).
//
// Sorting a row (up to 4096 blocks) is not needed. With the blocks ranked by
// (probability descending, index ascending), the chosen set is everything
// strictly above a cut value v*, plus the lowest-index ties at v*. v* is the
// value of the ranked element where the running sum first reaches tau.
//
// One warp per row:
//   1. Stage the row's fp32 bit patterns in shared memory (monotone in value
//      for p >= 0) and sum the row in fp64.
//   2. Radix-select v* in four passes over the 31 value bits (8/8/8/7 bits).
//      Each pass builds a 256-bucket histogram (count and fp64 sum) of the
//      elements that share the prefix found so far, scans the buckets from the
//      top, and keeps the bucket where the running sum crosses tau.
//   3. Take the ties at v* in index order until the sum reaches tau.
//   4. Emit mask words with warp ballots, and the ascending index list with a
//      ballot prefix count.
// All sums are fp64, so the choice matches a sequential fp64 walk of the
// ranked row (up to rounding in the last bits).
#include "common.cuh"

namespace xattn {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_excl_scan_d(double v, int lane) {
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  return incl - v;
}

__global__ void __launch_bounds__(kThreads)
    select_kernel(const float* __restrict__ probs, const TauArg tau, int NB, int hq, int causal,
                  long long rows, int nb_stage, uint32_t* __restrict__ mask,
                  int32_t* __restrict__ counts, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (row >= rows) return;

  // per-warp shared memory: sums[256] (f64), cnt[256] (u32), keys[nb_stage] (u32)
  uint8_t* wbase = smem + static_cast<size_t>(warp) * (256 * 8 + 256 * 4 + nb_stage * 4);
  double* hsum = reinterpret_cast<double*>(wbase);
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(wbase + 256 * 8);
  uint32_t* keys = hcnt + 256;

  const long long bh = row / NB;
  const int b = static_cast<int>(row % NB);
  const int h = static_cast<int>(bh % hq);
  const int n = causal ? b + 1 : NB;
  const float t = tau.v[h];
  const float* prow = probs + row * NB;

  double tot = 0.0;
  for (int j = lane; j < n; j += 32) {
    const uint32_t k = __float_as_uint(prow[j]) & 0x7FFFFFFFu;
    keys[j] = k;
    tot += static_cast<double>(__uint_as_float(k));
  }
  tot = warp_sum_d(tot);
  __syncwarp();

  const bool take_all = (t >= 1.0f) || (tot < static_cast<double>(t));
  uint32_t vstar = 0;
  int need_ties = 0;
  if (!take_all) {
    uint32_t prefix = 0, pmask = 0;
    double above = 0.0;  // sum of elements ranked strictly above the current prefix group
    uint32_t last_cnt = 0;
    const int shifts[4] = {23, 15, 7, 0};
    const uint32_t dmasks[4] = {0xFFu, 0xFFu, 0xFFu, 0x7Fu};
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int sh = shifts[pass];
      const uint32_t dm = dmasks[pass];
      for (int q = lane; q < 256; q += 32) {
        hsum[q] = 0.0;
        hcnt[q] = 0u;
      }
      __syncwarp();
      for (int j = lane; j < n; j += 32) {
        const uint32_t k = keys[j];
        if ((k & pmask) == prefix) {
          const uint32_t dgt = (k >> sh) & dm;
          atomicAdd(&hcnt[dgt], 1u);
          atomicAdd(&hsum[dgt], static_cast<double>(__uint_as_float(k)));
        }
      }
      __syncwarp();
      // lane l owns buckets 255-8l down to 248-8l (descending rank order)
      double ls = 0.0;
#pragma unroll
      for (int q = 0; q < 8; ++q) ls += hsum[255 - 8 * lane - q];
      const double excl = warp_excl_scan_d(ls, lane);
      const bool hit = above + excl + ls >= static_cast<double>(t);
      const unsigned bal = __ballot_sync(0xffffffffu, hit);
      // With exact sums some lane always hits; fall back to the lowest
      // non-empty bucket if rounding says otherwise.
      int dsel = -1;
      double acc_sel = 0.0;
      const int owner = bal ? (__ffs(bal) - 1) : 31;
      if (lane == owner) {
        double acc = above + excl;
        int last_nonempty = -1;
        double acc_last = acc;
        for (int q = 0; q < 8; ++q) {
          const int dg = 255 - 8 * lane - q;
          if (hcnt[dg] == 0u) continue;
          if (acc + hsum[dg] >= static_cast<double>(t)) {
            dsel = dg;
            acc_sel = acc;
            break;
          }
          last_nonempty = dg;
          acc_last = acc;
          acc += hsum[dg];
        }
        if (dsel < 0) {
          dsel = last_nonempty;
          acc_sel = acc_last;
        }
      }
      dsel = __shfl_sync(0xffffffffu, dsel, owner);
      acc_sel = __shfl_sync(0xffffffffu, acc_sel, owner);
      if (dsel < 0) {  // nothing left in this group (only reachable through rounding)
        break;
      }
      above = acc_sel;
      prefix |= static_cast<uint32_t>(dsel) << sh;
      pmask |= dm << sh;
      last_cnt = hcnt[dsel];
      __syncwarp();
    }
    vstar = prefix;
    // ties at v*: take them in index order while the sum is below tau
    const double v = static_cast<double>(__uint_as_float(vstar));
    double acc = above;
    uint32_t m = 0;
    while (m < last_cnt && acc < static_cast<double>(t)) {
      acc += v;
      ++m;
    }
    need_ties = static_cast<int>(m);
  }

  const int W = (NB + 31) / 32;
  uint32_t* mrow = mask + row * W;
  int32_t* irow = idx + row * NB;
  int running = 0, ties_seen = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int j0 = 0; j0 < W * 32; j0 += 32) {
    const int j = j0 + lane;
    const bool in = j < n;
    bool sel;
    if (take_all) {
      sel = in;
    } else {
      const uint32_t k = in ? keys[j] : 0u;
      const bool gt = in && k > vstar;
      const bool eq = in && k == vstar;
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      const int rank = ties_seen + __popc(eqb & lt);
      sel = gt || (eq && rank < need_ties);
      ties_seen += __popc(eqb);
    }
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) mrow[j0 / 32] = sb;
    if (sel) irow[running + __popc(sb & lt)] = j;
    running += __popc(sb);
  }
  if (lane == 0) counts[row] = running;
}

}  // namespace

cudaError_t launch_select(const Dims& D, const float* probs, const TauArg& tau, uint32_t* mask,
                          int32_t* counts, int32_t* idx, cudaStream_t st) {
  const long long rows = static_cast<long long>(D.batch) * D.hq * D.NB;
  const int nb_stage = (D.NB + 3) & ~3;
  const size_t smem = static_cast<size_t>(kWarps) * (256 * 8 + 256 * 4 + nb_stage * 4);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long grid = (rows + kWarps - 1) / kWarps;
  select_kernel<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(
      probs, tau, D.NB, D.hq, D.causal, rows, nb_stage, mask, counts, idx);
  return cudaGetLastError();
}

}  // namespace xattn
