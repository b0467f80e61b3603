// select.cu -- find_blocks threshold selection ("XAttention: Block Sparse
// Attention with Antidiagonal Scoring", §2.2 Threshold Block Selection: the
// smallest set of blocks whose probability mass reaches tau), and the
// fixed-budget Top-K / Top-Ratio selection of the pages' ablation.
//
// One warp per row. The row's fp32 bit patterns (monotone in value for
// p >= 0) are staged in shared memory and summed in fp64; the cut search
// (octave histograms refined on the mantissa bits) is in select_core.cuh,
// shared with the fused score->select kernel. All sums are fp64, so the choice
// matches a sequential fp64 walk of the ranked row up to rounding in the last
// bits.
#include "select_core.cuh"

namespace xattn {
namespace {

using sel::WarpSmem;
using sel::emit_row;
using sel::kBuckets;
using sel::warp_sum_d;

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

// ---------------------------------------------------------------------------
// Fixed-budget selection: the Top-K and Top-Ratio strategies of the
// selection-strategy ablation (Knowl 9 of the chapterpal page, §3.4 Ablation
// Study). A row keeps its k best allowed blocks in the find_blocks ranking
// (probability descending, index ascending): k = min(k_h, n) for Top-K, and
// k = round-half-up(ratio_h * n), at least 1, for Top-Ratio (n = allowed
// blocks). ratio_h * n + 1/2 is exact in fp64 (fp32 ratio, n < 2^13), so the
// count is exact.
//
// The cut is the k-th ranked key: a radix select on counts over the 31 key
// bits, 5 bits a level from the top (7 levels, the last one bit wide). Each
// level histograms the current group into a [32 buckets][32 lanes] table,
// picks the bucket where the running count from the top reaches the blocks
// still needed, and narrows the group to it. If the whole bucket is needed the
// cut is its lowest key; otherwise, once all bits are fixed, the remaining
// blocks are the first ties of v* in index order.
constexpr int kBudgetWarps = 8;
constexpr int kBudgetTable = kBuckets * 32 * 4;  // bytes of the count table per warp

__global__ void __launch_bounds__(kBudgetWarps * 32)
    select_budget_kernel(const float* __restrict__ probs, const BudgetArg budget, int NB, int hq,
                         int causal, long long rows, int nb_stage, uint32_t* __restrict__ mask,
                         int32_t* __restrict__ counts, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kBudgetWarps + warp;
  if (row >= rows) return;

  uint8_t* wbase = smem + static_cast<size_t>(warp) * (kBudgetTable + nb_stage * 4);
  uint32_t(*hcnt)[32] = reinterpret_cast<uint32_t(*)[32]>(wbase);
  uint32_t* keys = reinterpret_cast<uint32_t*>(wbase + kBudgetTable);

  const long long bh = row / NB;
  const int b = static_cast<int>(row % NB);
  const int h = static_cast<int>(bh % hq);
  const int n = causal ? b + 1 : NB;
  const float* prow = probs + row * NB;

  for (int j0 = 0; j0 < n; j0 += 8 * 32) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 32 + lane;
      v[u] = j < n ? __float_as_uint(__ldg(prow + j)) & 0x7FFFFFFFu : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 32 + lane;
      if (j < n) keys[j] = v[u];
    }
  }
  __syncwarp();

  int k;
  if (budget.use_ratio) {
    const double x = __dadd_rn(__dmul_rn(static_cast<double>(budget.ratio[h]),
                                         static_cast<double>(n)),
                               0.5);
    k = static_cast<int>(floor(x));
  } else {
    k = budget.k[h];
  }
  k = max(1, min(n, k));
  const bool take_all = k >= n;
  uint32_t vstar = 0xFFFFFFFFu;
  int icut = -1;
  if (!take_all) {
    uint32_t prefix = 0, pmask = 0;
    uint32_t need = static_cast<uint32_t>(k);  // blocks still to take inside the group
    bool done = false;
    for (int level = 0; level < 7 && !done; ++level) {
      const int hi = 30 - 5 * level;
      const int width = hi >= 4 ? 5 : hi + 1;
      const int lo = hi - width + 1;
      const uint32_t dmask = (1u << width) - 1u;
#pragma unroll
      for (int q = 0; q < kBuckets; ++q) hcnt[q][lane] = 0u;
      for (int j = lane; j < n; j += 32) {
        const uint32_t key = keys[j];
        if ((key & pmask) == prefix) hcnt[dmask - ((key >> lo) & dmask)][lane] += 1u;
      }
      __syncwarp();
      uint32_t bc = 0;  // lane q totals bucket q (bucket 0 = largest digit)
#pragma unroll 8
      for (int l = 0; l < 32; ++l) bc += hcnt[lane][(l + lane) & 31];
      __syncwarp();
      uint32_t incl = bc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      // The group holds at least `need` keys, so some non-empty bucket reaches it.
      const unsigned bal = __ballot_sync(0xffffffffu, bc > 0 && incl >= need);
      const int D = __ffs(bal) - 1;
      const uint32_t ex = __shfl_sync(0xffffffffu, incl - bc, D);
      const uint32_t cnt = __shfl_sync(0xffffffffu, bc, D);
      need -= ex;
      prefix |= (dmask - static_cast<uint32_t>(D)) << lo;
      pmask |= dmask << lo;
      if (cnt == need) {  // the whole bucket is taken: cut at its lowest key
        vstar = prefix;
        icut = 0x7FFFFFFF;
        done = true;
      }
    }
    if (!done) {  // v* is exact; take the first `need` of its ties by index
      vstar = prefix;
      icut = n;
      uint32_t seen = 0;
      for (int j0 = 0; j0 < n; j0 += 32) {
        const int j = j0 + lane;
        const unsigned m = __ballot_sync(0xffffffffu, j < n && keys[j] == vstar);
        const uint32_t c = static_cast<uint32_t>(__popc(m));
        if (seen + c >= need) {
          unsigned mm = m;
          for (uint32_t q = 1; q < need - seen; ++q) mm &= mm - 1;
          icut = j0 + __ffs(mm) - 1;
          break;
        }
        seen += c;
      }
    }
  }
  emit_row(keys, n, NB, take_all, vstar, icut, row, lane, mask, counts, idx);
}

__global__ void __launch_bounds__(kThreads)
    select_kernel(const float* __restrict__ probs, const TauArg tau, int NB, int hq, int causal,
                  long long rows, int nb_stage, uint32_t* __restrict__ mask,
                  int32_t* __restrict__ counts, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;
  if (row >= rows) return;

  uint8_t* wbase = smem + static_cast<size_t>(warp) * (sizeof(WarpSmem) + nb_stage * 4);
  WarpSmem& W = *reinterpret_cast<WarpSmem*>(wbase);
  uint32_t* keys = reinterpret_cast<uint32_t*>(wbase + sizeof(WarpSmem));

  const long long bh = row / NB;
  const int b = static_cast<int>(row % NB);
  const int h = static_cast<int>(bh % hq);
  const int n = causal ? b + 1 : NB;
  const double t = static_cast<double>(tau.v[h]);
  const float* prow = probs + row * NB;

  double tot = 0.0;
  uint32_t kmax = 0;
  // 8 independent loads in flight per lane before any is used
  for (int j0 = 0; j0 < n; j0 += 8 * 32) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 32 + lane;
      v[u] = j < n ? __float_as_uint(__ldg(prow + j)) & 0x7FFFFFFFu : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 32 + lane;
      if (j < n) {
        keys[j] = v[u];
        tot += static_cast<double>(__uint_as_float(v[u]));
        kmax = max(kmax, v[u]);
      }
    }
  }
  tot = warp_sum_d(tot);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  __syncwarp();

  bool take_all;
  uint32_t vstar;
  int icut;
  sel::find_cut(keys, n, t, tot, kmax, W, lane, take_all, vstar, icut);
  emit_row(keys, n, NB, take_all, vstar, icut, row, lane, mask, counts, idx);
}

}  // namespace

cudaError_t launch_select_budget(const Dims& D, const float* probs, const BudgetArg& budget,
                                 uint32_t* mask, int32_t* counts, int32_t* idx,
                                 cudaStream_t st) {
  const long long rows = static_cast<long long>(D.batch) * D.hq * D.NB;
  const int nb_stage = (D.NB + 3) & ~3;
  const size_t smem = static_cast<size_t>(kBudgetWarps) * (kBudgetTable + nb_stage * 4);
  cudaError_t e = cudaFuncSetAttribute(select_budget_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long grid = (rows + kBudgetWarps - 1) / kBudgetWarps;
  select_budget_kernel<<<static_cast<unsigned>(grid), kBudgetWarps * 32, smem, st>>>(
      probs, budget, D.NB, D.hq, D.causal, rows, nb_stage, mask, counts, idx);
  return cudaGetLastError();
}

cudaError_t launch_select(const Dims& D, const float* probs, const TauArg& tau, uint32_t* mask,
                          int32_t* counts, int32_t* idx, cudaStream_t st) {
  const long long rows = static_cast<long long>(D.batch) * D.hq * D.NB;
  const int nb_stage = (D.NB + 3) & ~3;
  const size_t smem = static_cast<size_t>(kWarps) * (sizeof(WarpSmem) + nb_stage * 4);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long grid = (rows + kWarps - 1) / kWarps;
  select_kernel<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(
      probs, tau, D.NB, D.hq, D.causal, rows, nb_stage, mask, counts, idx);
  return cudaGetLastError();
}

}  // namespace xattn
