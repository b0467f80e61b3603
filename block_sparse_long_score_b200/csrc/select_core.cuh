// select_core.cuh -- the per-row cut search of find_blocks ("XAttention:
// Block Sparse Attention with Antidiagonal Scoring", §2.2 Threshold Block
// Selection), shared by the selection kernel and the fused score->select
// kernel.
//
// A row's allowed blocks are staged in shared memory as fp32 bit patterns
// (monotone in value for p >= 0). Ranked by (value desc, index asc), the chosen
// set is every block at or before a cut block (v*, i*): value > v*, or
// value == v* and index <= i*. The cut is the ranked block where the running
// sum first reaches tau. It is found with octave histograms below the row
// maximum (32 buckets; each lane accumulates into its own column of a
// [32 buckets][32 lanes] table of fp64 sums and counts: no atomics, no bank
// conflicts, a fixed summation order), scanned from the top in fp64 to find
// the bucket where the running sum crosses tau. That bucket is split on the
// next 5 mantissa bits until it holds at most 32 blocks, which are sorted
// across the warp by (value desc, index asc) and scanned. Equal values past
// the last bit are taken in index order; a cut more than 31 octaves below the
// maximum is walked exactly.
// Mask words come from warp ballots and the index lists from ballot prefix
// counts.
#pragma once

#include "common.cuh"

namespace xattn {
namespace sel {

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

// Histogram search for the cut of a row whose sum reaches t (see the header).
__device__ __forceinline__ void threshold_cut_hist(const uint32_t* keys, int n, double t,
                                                   uint32_t kmax, WarpSmem& W, int lane,
                                                   uint32_t& vstar, int& icut) {
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

// The find_blocks cut of a staged row: tot is the row's fp64 sum and kmax its
// largest key (both warp-uniform). take_all: tau >= 1 or the sum never reaches
// tau -- every allowed block is selected.
__device__ __forceinline__ void find_cut(const uint32_t* keys, int n, double t, double tot,
                                         uint32_t kmax, WarpSmem& W, int lane, bool& take_all,
                                         uint32_t& vstar, int& icut) {
  take_all = (t >= 1.0) || (tot < t);
  vstar = 0xFFFFFFFFu;  // cut value (fp32 bits); none selected above it
  icut = -1;            // cut index among blocks equal to vstar
  if (take_all) return;
  threshold_cut_hist(keys, n, t, kmax, W, lane, vstar, icut);
}

}  // namespace sel
}  // namespace xattn
