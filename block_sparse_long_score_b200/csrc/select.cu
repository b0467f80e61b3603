// select.cu -- find_blocks threshold selection ("XAttention: Block Sparse
// Attention with Antidiagonal Scoring", §2.2 Threshold Block Selection: the
// smallest set of blocks whose probability mass reaches tau).
//
// Sorting a row (up to 4096 blocks) is not needed. With the blocks ranked by
// (probability descending, index ascending), the chosen set is every block
// that ranks at or before a cut block (v*, i*): value > v*, or value == v* and
// index <= i*. The cut is the ranked block where the running sum first reaches
// tau.
//
// One warp per row; the row's fp32 bit patterns (monotone in value for p >= 0)
// are staged in shared memory and the row is summed in fp64.
//   level 0  histogram of octaves below the row maximum (32 buckets: exponent
//            E_max - b). Each lane accumulates into its own column of a
//            [32 buckets][32 lanes] table (fp64 sums, counts): no atomics and
//            no bank conflicts. The buckets are scanned from the top in fp64 to
//            find the one where the running sum crosses tau.
//   level k  while that bucket holds more than 32 blocks, split it again on
//            the next 5 mantissa bits (same table, same scan).
//   cut      the <= 32 blocks of the final bucket are sorted across the warp by
//            (value desc, index asc) and scanned in fp64 from the sum of all
//            higher buckets: the first position that reaches tau is the cut.
//            (If all 31 bits are fixed and more than 32 equal values remain,
//            ties are taken in index order.)
// Emit: mask words by warp ballot, the ascending index list by ballot prefix
// counts. All sums are fp64, so the choice matches a sequential fp64 walk of
// the ranked row up to rounding in the last bits.
#include "common.cuh"

namespace xattn {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kBuckets = 32;

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

struct WarpSmem {
  double hsum[kBuckets][32];   // [bucket][lane]
  uint32_t hcnt[kBuckets][32];
};

// Bucket of key k at a refinement level, or -1 if k is not in the current
// prefix group. Level 0: octave below the row maximum (0 = the top octave,
// 31 = everything 31+ octaves down). Level L >= 1: mantissa bits
// [22 - 5(L-1), 18 - 5(L-1)] (the last level has 3 bits), mapped so that
// bucket 0 holds the largest values.
__device__ __forceinline__ int bucket_of(uint32_t k, int level, uint32_t emax, uint32_t pmask,
                                         uint32_t prefix) {
  if (level == 0) {
    const uint32_t e = k >> 23;
    const uint32_t d = emax - e;
    return static_cast<int>(d > 31u ? 31u : d);
  }
  if ((k & pmask) != prefix) return -1;
  const int hi = 22 - 5 * (level - 1);
  const int width = hi >= 4 ? 5 : hi + 1;
  const uint32_t dig = (k >> (hi - width + 1)) & ((1u << width) - 1u);
  return static_cast<int>(((1u << width) - 1u) - dig);
}

// Writes one row's outputs. Block j < n is selected iff take_all, or its key
// ranks at or before the cut (v*, i*): key > v*, or key == v* and j <= i*.
// v* = 0xFFFFFFFF (above every key) selects nothing.
__device__ __forceinline__ void emit_row(const uint32_t* keys, int n, int NB, bool take_all,
                                         uint32_t vstar, int icut, long long row, int lane,
                                         uint32_t* __restrict__ mask, int32_t* __restrict__ counts,
                                         int32_t* __restrict__ idx) {
  const int Wn = (NB + 31) / 32;
  uint32_t* mrow = mask + row * Wn;
  int32_t* irow = idx + row * NB;
  int running = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int j0 = 0; j0 < Wn * 32; j0 += 32) {
    const int j = j0 + lane;
    bool sel = false;
    if (j < n) {
      if (take_all) {
        sel = true;
      } else {
        const uint32_t k = keys[j];
        sel = k > vstar || (k == vstar && j <= icut);
        if (vstar == 0xFFFFFFFFu) sel = false;
      }
    }
    const unsigned sb = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) mrow[j0 / 32] = sb;
    if (sel) irow[running + __popc(sb & lt)] = j;
    running += __popc(sb);
  }
  if (lane == 0) counts[row] = running;
}

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

  const bool take_all = (t >= 1.0) || (tot < t);
  uint32_t vstar = 0xFFFFFFFFu;  // cut value (fp32 bits); none selected above it
  int icut = -1;                 // cut index among blocks equal to vstar
  if (!take_all) {
    const uint32_t emax = kmax >> 23;
    uint32_t pmask = 0, prefix = 0;
    double above = 0.0;   // sum of the blocks ranked strictly above the current group
    uint32_t cnt = 0;
    int level = 0;
    bool fallback_tail = false;
    for (;;) {
      // ---- histogram of the current group over 32 buckets
#pragma unroll
      for (int q = 0; q < kBuckets; ++q) {
        W.hsum[q][lane] = 0.0;
        W.hcnt[q][lane] = 0u;
      }
      for (int j = lane; j < n; j += 32) {
        const uint32_t k = keys[j];
        const int q = bucket_of(k, level, emax, pmask, prefix);
        if (q >= 0) {
          W.hsum[q][lane] += static_cast<double>(__uint_as_float(k));
          W.hcnt[q][lane] += 1u;
        }
      }
      __syncwarp();
      // lane q totals bucket q
      double bs = 0.0;
      uint32_t bc = 0;
#pragma unroll 8
      for (int l = 0; l < 32; ++l) {
        bs += W.hsum[lane][(l + lane) & 31];
        bc += W.hcnt[lane][(l + lane) & 31];
      }
      __syncwarp();
      const double excl = warp_excl_scan_d(bs, lane);
      const bool hit = bc > 0 && above + excl + bs >= t;
      unsigned bal = __ballot_sync(0xffffffffu, hit);
      if (bal == 0) {  // rounding: take the lowest non-empty bucket
        bal = __ballot_sync(0xffffffffu, bc > 0);
        bal = bal ? (1u << (31 - __clz(bal))) : 1u;
      }
      const int D = __ffs(bal) - 1;
      above += __shfl_sync(0xffffffffu, excl, D);
      cnt = __shfl_sync(0xffffffffu, bc, D);
      // fix this level's digits into the prefix
      if (level == 0) {
        if (D == 31) {  // the cut lies 31+ octaves below the maximum
          fallback_tail = true;
          break;
        }
        pmask = 0x7F800000u;
        prefix = (emax - static_cast<uint32_t>(D)) << 23;
      } else {
        const int hi = 22 - 5 * (level - 1);
        const int width = hi >= 4 ? 5 : hi + 1;
        const uint32_t dig = ((1u << width) - 1u) - static_cast<uint32_t>(D);
        const int lo = hi - width + 1;
        pmask |= ((1u << width) - 1u) << lo;
        prefix |= dig << lo;
      }
      if (cnt <= 32u || level == 5) break;
      ++level;
    }

    if (fallback_tail) {
      // Blocks 31+ octaves below the maximum decide the cut (tau within about
      // n * 2^-31 of the row sum). Walk the ranked tail exactly: repeatedly
      // take the largest remaining tail block.
      uint32_t lim = (emax >= 31u) ? ((emax - 31u) << 23) | 0x7FFFFFu : 0u;  // tail: k <= lim
      uint32_t cur_hi = lim;
      int cur_idx_floor = -1;
      for (;;) {
        // largest (key, then lowest index) among tail blocks ranked after the last taken
        uint32_t bk = 0;
        int bi = 0x7FFFFFFF;
        for (int j = lane; j < n; j += 32) {
          const uint32_t k = keys[j];
          const bool after = k < cur_hi || (k == cur_hi && j > cur_idx_floor);
          if (k <= lim && after && (k > bk || (k == bk && j < bi))) {
            bk = k;
            bi = j;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const uint32_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ok > bk || (ok == bk && oi < bi)) {
            bk = ok;
            bi = oi;
          }
        }
        if (bi == 0x7FFFFFFF) {  // tail exhausted: take everything
          vstar = 0u;
          icut = 0x7FFFFFFF;
          break;
        }
        above += static_cast<double>(__uint_as_float(bk));
        cur_hi = bk;
        cur_idx_floor = bi;
        if (above >= t) {
          vstar = bk;
          icut = bi;
          break;
        }
      }
    } else if (cnt <= 32u) {
      // gather the group's blocks, one per lane (the histogram table is free now)
      uint32_t* ckey = &W.hcnt[0][0];
      uint32_t* cidx = &W.hcnt[1][0];
      int got = 0;
      for (int j0 = 0; j0 < n && got < static_cast<int>(cnt); j0 += 32) {
        const int j = j0 + lane;
        const bool in = j < n && (keys[j] & pmask) == prefix;
        const unsigned m = __ballot_sync(0xffffffffu, in);
        const int pos = got + __popc(m & ((1u << lane) - 1u));
        if (in && pos < 32) {
          ckey[pos] = keys[j];
          cidx[pos] = static_cast<uint32_t>(j);
        }
        got += __popc(m);
      }
      __syncwarp();
      const uint32_t ck = lane < static_cast<int>(cnt) ? ckey[lane] : 0u;
      const int ci = lane < static_cast<int>(cnt) ? static_cast<int>(cidx[lane]) : 0x7FFFFFFF;
      __syncwarp();
      // bitonic sort, descending by (key, -index)
      unsigned long long sk =
          (static_cast<unsigned long long>(ck) << 32) | static_cast<uint32_t>(~ci);
      if (ci == 0x7FFFFFFF) sk = 0ull;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, sk, stride);
          const bool up = (lane & size) == 0;       // this run sorts descending
          const bool lower = (lane & stride) == 0;  // keep the larger in the lower lane
          const bool take_max = (up == lower);
          sk = take_max ? (o > sk ? o : sk) : (o < sk ? o : sk);
        }
      }
      const uint32_t sk_key = static_cast<uint32_t>(sk >> 32);
      const int sk_idx = static_cast<int>(~static_cast<uint32_t>(sk));
      const double v = sk != 0ull ? static_cast<double>(__uint_as_float(sk_key)) : 0.0;
      double incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const bool reach = sk != 0ull && above + incl >= t;
      unsigned rb = __ballot_sync(0xffffffffu, reach);
      if (rb == 0) {  // rounding: take the whole group
        rb = __ballot_sync(0xffffffffu, sk != 0ull);
        rb = rb ? (1u << (31 - __clz(rb))) : 1u;
      }
      const int cl = __ffs(rb) - 1;
      vstar = __shfl_sync(0xffffffffu, sk_key, cl);
      icut = __shfl_sync(0xffffffffu, sk_idx, cl);
    } else {
      // more than 32 blocks share one exact value: take them in index order
      vstar = prefix;
      const double v = static_cast<double>(__uint_as_float(vstar));
      double acc = above;
      uint32_t need = 0;
      while (need < cnt && acc < t) {
        acc += v;
        ++need;
      }
      int seen = 0;
      icut = n;
      for (int j0 = 0; j0 < n; j0 += 32) {
        const int j = j0 + lane;
        const bool eq = j < n && keys[j] == vstar;
        const unsigned m = __ballot_sync(0xffffffffu, eq);
        const int c = __popc(m);
        if (seen + c >= static_cast<int>(need)) {
          // the (need - seen)-th set bit of m
          unsigned mm = m;
          for (int q = 1; q < static_cast<int>(need) - seen; ++q) mm &= mm - 1;
          icut = j0 + __ffs(mm) - 1;
          break;
        }
        seen += c;
      }
    }
  }

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
