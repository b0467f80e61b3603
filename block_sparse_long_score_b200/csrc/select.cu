// select.cu -- find_blocks threshold selection ("XAttention: Block Sparse
// Attention with Antidiagonal Scoring", §2.2 Threshold Block Selection: the
// smallest set of blocks whose probability mass reaches tau), and the
// fixed-budget Top-K / Top-Ratio selection of the pages' ablation.
//
// find_blocks runs as two kernels, one warp per row in each. The first is the
// threshold filter of select_filter.cuh: it gathers the few blocks at or
// above a threshold that already holds tau of the mass, sorts them and adds
// their probabilities in fp64 in ranked order, exactly as the definition does;
// it decides almost every row of a long-context layer. The rows it cannot
// decide go to the second, which stages the row's fp32 bit patterns (monotone
// in value for p >= 0) in shared memory and runs the histogram search of
// select_core.cuh (shared with the fused score->select kernel). Its sums are
// fp64 too, so its choice matches the sequential fp64 walk up to rounding in
// the last bits.
#include "select_core.cuh"
#include "select_filter.cuh"

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

// ---------------------------------------------------------------------------
// find_blocks in two kernels.
//
// select_filter_kernel (one warp per row): the threshold filter of
// select_filter.cuh. A row of at most 1024 blocks is read once into registers
// (32 loads a lane in flight); a longer one is streamed from memory for each
// pass (the re-reads hit L1/L2). Rows the filter cannot decide -- more than
// filt::kCand blocks at or above the threshold that reaches tau, as in flat
// rows -- are marked (count -1) for select_fallback_kernel, the histogram
// search of select_core.cuh, which runs on the marked rows only.
constexpr int kFiltWarps = 8;

__global__ void __launch_bounds__(kFiltWarps * 32, 3)
    select_filter_kernel(const RowSource src, const TauArg tau, int NB, int hq,
                         int causal, long long rows, uint32_t* __restrict__ mask,
                         int32_t* __restrict__ counts, int32_t* __restrict__ idx) {
  __shared__ filt::WarpBuf bufs[kFiltWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kFiltWarps + warp;
  if (row >= rows) return;

  const long long bh = row / NB;
  const int b = static_cast<int>(row % NB);
  const int h = static_cast<int>(bh % hq);
  const int n = causal ? b + 1 : NB;
  const double t = tau_of(tau, h);
  const float* prow =
      src.layout == 0
          ? src.p + row * NB
          : src.p + static_cast<size_t>(bh) * src.part_head +
                part_row_offset(b * src.r, src.r, NB, causal != 0);

  unsigned long long cut = 0;
  int ncand = 0;
  filt::Outcome oc;
  if (n <= 32 * filt::kRegU) {
    filt::RegRow rr;
#pragma unroll
    for (int u = 0; u < filt::kRegU; ++u) {
      const int j = u * 32 + lane;
      rr.k[u] = j < n ? __float_as_uint(__ldg(prow + j)) & 0x7FFFFFFFu : 0u;
    }
    oc = filt::filter_cut(rr, n, t, lane, bufs[warp], &cut, &ncand);
  } else {
    auto ld = [prow](int j) { return __float_as_uint(__ldg(prow + j)) & 0x7FFFFFFFu; };
    const filt::MemRow<decltype(ld)> mr{ld};
    oc = filt::filter_cut(mr, n, t, lane, bufs[warp], &cut, &ncand);
  }
  if (oc == filt::kUndecided) {
    if (lane == 0) counts[row] = -1;
    return;
  }
  filt::emit(oc, cut, ncand, n, NB, row, lane, bufs[warp], mask, counts, idx);
}

// The histogram search of one row (select_core.cuh), with its keys staged in
// the warp's shared memory.
__device__ __forceinline__ void select_row_hist(const RowSource& src, const TauArg& tau,
                                                int NB, int hq, int causal, long long row,
                                                WarpSmem& W, uint32_t* keys, int lane,
                                                uint32_t* __restrict__ mask,
                                                int32_t* __restrict__ counts,
                                                int32_t* __restrict__ idx) {
  const long long bh = row / NB;
  const int b = static_cast<int>(row % NB);
  const int h = static_cast<int>(bh % hq);
  const int n = causal ? b + 1 : NB;
  const double t = tau_of(tau, h);  // valid: the filter only leaves rows of valid tau
  const float* prow =
      src.layout == 0
          ? src.p + row * NB
          : src.p + static_cast<size_t>(bh) * src.part_head +
                part_row_offset(b * src.r, src.r, NB, causal != 0);

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
  __syncwarp();  // the keys are overwritten by the warp's next row
}

// Persistent: warp g of G owns rows g, g + G, g + 2G, ... and runs the
// histogram search on those the fast kernel marked.
constexpr int kFbWarps = 1;

__global__ void __launch_bounds__(kFbWarps * 32)
    select_fallback_kernel(const RowSource src, const TauArg tau, int NB, int hq,
                           int causal, long long rows, int nb_stage, uint32_t* __restrict__ mask,
                           int32_t* __restrict__ counts, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint8_t* wbase = smem + static_cast<size_t>(warp) * (sizeof(WarpSmem) + nb_stage * 4);
  WarpSmem& W = *reinterpret_cast<WarpSmem*>(wbase);
  uint32_t* keys = reinterpret_cast<uint32_t*>(wbase + sizeof(WarpSmem));

  const long long G = static_cast<long long>(gridDim.x) * kFbWarps;
  const long long g = static_cast<long long>(blockIdx.x) * kFbWarps + warp;
  for (long long r0 = g; r0 < rows; r0 += 32 * G) {
    const long long r = r0 + lane * G;
    unsigned todo = __ballot_sync(0xffffffffu, r < rows && counts[r] < 0);
    while (todo) {
      const int q = __ffs(todo) - 1;
      todo &= todo - 1;
      select_row_hist(src, tau, NB, hq, causal, r0 + q * G, W, keys, lane, mask, counts, idx);
    }
  }
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

cudaError_t launch_select_rows(const Dims& D, const RowSource& src, const TauArg& tau,
                               uint32_t* mask, int32_t* counts, int32_t* idx, int num_sms,
                               cudaStream_t st) {
  const long long rows = static_cast<long long>(D.batch) * D.hq * D.NB;
  const long long filt_grid = (rows + kFiltWarps - 1) / kFiltWarps;
  select_filter_kernel<<<static_cast<unsigned>(filt_grid), kFiltWarps * 32, 0, st>>>(
      src, tau, D.NB, D.hq, D.causal, rows, mask, counts, idx);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_select_fallback(D, src, tau, mask, counts, idx, num_sms, st);
}

cudaError_t launch_select(const Dims& D, const float* probs, const TauArg& tau, uint32_t* mask,
                          int32_t* counts, int32_t* idx, int num_sms, cudaStream_t st) {
  const RowSource src{probs, 0, 0, 0};
  return launch_select_rows(D, src, tau, mask, counts, idx, num_sms, st);
}

cudaError_t launch_select_fallback(const Dims& D, const RowSource& src, const TauArg& tau,
                                   uint32_t* mask, int32_t* counts, int32_t* idx, int num_sms,
                                   cudaStream_t st) {
  const long long rows = static_cast<long long>(D.batch) * D.hq * D.NB;
  const int nb_stage = (D.NB + 3) & ~3;
  const size_t smem = static_cast<size_t>(kFbWarps) * (sizeof(WarpSmem) + nb_stage * 4);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_fallback_kernel,
                                                                kFbWarps * 32, smem);
  if (e != cudaSuccess) return e;
  const long long full = static_cast<long long>(num_sms) * (per_sm > 0 ? per_sm : 1);
  const long long need = (rows + kFbWarps - 1) / kFbWarps;
  const long long grid = need < full ? need : full;
  select_fallback_kernel<<<static_cast<unsigned>(grid), kFbWarps * 32, smem, st>>>(
      src, tau, D.NB, D.hq, D.causal, rows, nb_stage, mask, counts, idx);
  return cudaGetLastError();
}

}  // namespace xattn
