// select_filter.cuh -- the find_blocks cut of one row by a threshold filter
// ("XAttention: Block Sparse Attention with Antidiagonal Scoring", §2.2
// Threshold Block Selection: the smallest set of blocks, taken in the order
// probability descending / index ascending, whose probabilities sum to at
// least tau), for one warp per row. Shared by the selection kernel (row read
// from P in global memory) and the fused score->select kernel (row staged in
// shared memory).
//
// Every block below a value theta ranks after every block at or above it. So
// if the blocks at or above theta hold at least tau of the mass, the cut is
// one of them, and the ranked walk over just those candidates -- sorted by
// (value desc, index asc) and added one after another in fp64 -- is exactly
// the definition's walk up to the cut. The warp finds the row maximum m, then
// tries theta = m * 2^-6, 2^-12, 2^-18 until the candidates' fp32 sum reaches
// tau (within rounding), gathers the candidates in index order (at most
// kCand = 256 of them) into shared memory, sorts them across the warp with a
// bitonic network (one to eight keys a lane) and walks them. A walk that
// covers every non-zero block without reaching tau takes the whole row. Rows
// that need more than kCand candidates (flat rows) are left to the histogram
// search (select_core.cuh).
//
// The work per element is a handful of instructions (maximum, threshold sum,
// ballot compaction); the sort, the walk and the emit depend on the number of
// candidates only. The emit writes the mask row from a shared-memory staging
// of its words and the index list from the candidates, which are already in
// index order.
#pragma once

#include "common.cuh"

namespace xattn {
namespace filt {

constexpr int kCand = 256;      // candidates a warp sorts (up to eight per lane)
constexpr int kMaxWords = XATTN_MAX_BLOCKS / 32;
constexpr int kRegU = 32;       // row elements a lane holds in registers (n <= 1024)

// Per-warp shared memory of the filter.
struct WarpBuf {
  unsigned long long cand[kCand];  // candidates' rank keys, in index order
  uint32_t words[kMaxWords];       // mask row staging
};

// Rank key of block j with fp32 bits k (sign cleared): larger ranks first;
// ~j puts the lower index first among equal values. No key is 0.
__device__ __forceinline__ unsigned long long rank_key(uint32_t k, int j) {
  return (static_cast<unsigned long long>(k) << 32) | static_cast<uint32_t>(~j);
}
__device__ __forceinline__ float key_value(unsigned long long key) {
  return __uint_as_float(static_cast<uint32_t>(key >> 32));
}
__device__ __forceinline__ int key_index(unsigned long long key) {
  return static_cast<int>(~static_cast<uint32_t>(key));
}

// Row held in registers: element j = 32u + lane of an n <= 32 * kRegU row
// (0 past n).
struct RegRow {
  uint32_t k[kRegU];
  template <class F>
  __device__ __forceinline__ void each(int n, int lane, F f) const {
#pragma unroll
    for (int u = 0; u < kRegU; ++u) {
      if (u * 32 >= n) break;  // warp-uniform
      f(k[u], u * 32 + lane);
    }
  }
};

// Row read on demand from memory through `Load` (global P or a staged row),
// 8 elements a lane in flight; any n.
template <class Load>
struct MemRow {
  Load load;
  template <class F>
  __device__ __forceinline__ void each(int n, int lane, F f) const {
    for (int j0 = 0; j0 < n; j0 += 8 * 32) {
      uint32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * 32 + lane;
        v[u] = j < n ? load(j) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) f(v[u], j0 + u * 32 + lane);
    }
  }
};

// Bitonic sort, descending, of 32 * KPL keys held KPL a lane: k[q] is
// position lane + 32 q. Partners 32 or more positions apart sit in the same
// lane; closer ones are exchanged with warp shuffles.
template <int KPL>
__device__ __forceinline__ void sort_desc(unsigned long long (&k)[KPL], int lane) {
  constexpr int N = 32 * KPL;
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32) {
        const int qs = stride / 32;
#pragma unroll
        for (int q = 0; q < KPL; ++q) {
          if ((q & qs) != 0) continue;
          // positions p (this entry) and p + stride (entry q | qs)
          const bool up = ((lane + 32 * q) & size) == 0;  // descending run
          const unsigned long long x = k[q], y = k[q | qs];
          const unsigned long long hi = x > y ? x : y, lo = x > y ? y : x;
          k[q] = up ? hi : lo;
          k[q | qs] = up ? lo : hi;
        }
      } else {
        const bool lower = (lane & stride) == 0;
#pragma unroll
        for (int q = 0; q < KPL; ++q) {
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, k[q], stride);
          const bool up = ((lane + 32 * q) & size) == 0;
          k[q] = (up == lower) ? (o > k[q] ? o : k[q]) : (o < k[q] ? o : k[q]);
        }
      }
    }
  }
}

// Loads the c candidates (in index order) KPL a lane, sorts them descending
// and finds where the ranked fp64 sum reaches t. True (and the cut key) if it
// does.
//
// The definition adds one probability after another in fp64. With exact_sums
// the candidates all lie within 19 binades below the row maximum (theta is at
// least m * 2^-18), so each is a multiple of the smallest one's ulp and any
// sum of at most 256 of them needs at most 18 + 24 + 8 = 50 significant bits:
// every partial sum is exact in fp64, whatever the order of the additions. A
// warp prefix scan then gives the very sums of the one-by-one walk, and the
// cut is the first position where the scan reaches t. Otherwise (theta is the
// smallest non-zero pattern) the walk adds one candidate after another.
template <int KPL>
__device__ __forceinline__ bool sort_walk(const WarpBuf& W, int c, double t, bool exact_sums,
                                          int lane, unsigned long long* cut) {
  unsigned long long k[KPL];
#pragma unroll
  for (int q = 0; q < KPL; ++q) k[q] = lane + 32 * q < c ? W.cand[lane + 32 * q] : 0ull;
  sort_desc<KPL>(k, lane);
  if (exact_sums) {
    double carry = 0.0;  // sum of the positions before this group of 32
#pragma unroll
    for (int q = 0; q < KPL; ++q) {
      if (32 * q >= c) break;  // warp-uniform
      double incl = static_cast<double>(key_value(k[q]));  // 0 past c (key 0)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, lane + 32 * q < c && carry + incl >= t);
      if (hit) {
        *cut = __shfl_sync(0xffffffffu, k[q], __ffs(hit) - 1);
        return true;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    return false;
  }
  double acc = 0.0;
#pragma unroll
  for (int q = 0; q < KPL; ++q) {
    if (32 * q >= c) break;  // warp-uniform
    const int m = min(32, c - 32 * q);
    for (int ii = 0; ii < m; ++ii) {
      const unsigned long long key = __shfl_sync(0xffffffffu, k[q], ii);
      acc += static_cast<double>(key_value(key));
      if (acc >= t) {
        *cut = key;
        return true;
      }
    }
  }
  return false;
}

// Outcome of the filter for one row.
enum Outcome { kUndecided = 0, kCut = 1, kTakeAll = 2, kNone = 3 };

// find_blocks cut of a row of n allowed blocks with threshold t (warp-uniform
// arguments). On kCut, the blocks whose rank key is >= *cut are chosen, and
// W.cand holds the *ncand candidates in index order (a superset of them).
// kTakeAll: every allowed block (t >= 1, or the row never reaches t).
// kNone: nothing (t < 0 marks an invalid threshold). kUndecided: the row
// needs the histogram search.
template <class Row>
__device__ __forceinline__ Outcome filter_cut(const Row& row, int n, double t, int lane,
                                              WarpBuf& W, unsigned long long* cut, int* ncand) {
  if (t < 0.0) return kNone;
  if (t >= 1.0) return kTakeAll;
  uint32_t mx = 0;
  row.each(n, lane, [&](uint32_t k, int) { mx = max(mx, k); });
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (mx == 0u) return kTakeAll;  // an all-zero row never reaches t > 0
  const int emx = static_cast<int>(mx >> 23);
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll 1
  for (int shift = 6; shift <= 18; shift += 6) {
    // theta: a power of two at most m * 2^-shift; 1 (the smallest non-zero
    // pattern) once that would underflow, so that every non-zero block is a
    // candidate
    const uint32_t th = emx > shift ? static_cast<uint32_t>(emx - shift) << 23 : 1u;
    const bool all_nonzero = th == 1u;
    float s = 0.f;
    int c = 0;
    row.each(n, lane, [&](uint32_t k, int) {
      const bool p = k >= th;
      s += p ? __uint_as_float(k) : 0.f;
      c += p ? 1 : 0;
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    c = __reduce_add_sync(0xffffffffu, c);
    // fp32 sum of at most n terms <= 1: rounding stays far below 1e-5
    if (!all_nonzero && static_cast<double>(s) < t - 1e-5) continue;
    if (c > kCand) return kUndecided;
    // gather the candidates in index order
    int base = 0;
    row.each(n, lane, [&](uint32_t k, int j) {
      const bool p = k >= th;
      const unsigned b = __ballot_sync(0xffffffffu, p);
      if (p) W.cand[base + __popc(b & lt)] = rank_key(k, j);
      base += __popc(b);
    });
    __syncwarp();
    // the definition's walk: ranked order, one fp64 addition after another
    const bool ex = !all_nonzero;
    const bool reached = c <= 32   ? sort_walk<1>(W, c, t, ex, lane, cut)
                         : c <= 64  ? sort_walk<2>(W, c, t, ex, lane, cut)
                         : c <= 128 ? sort_walk<4>(W, c, t, ex, lane, cut)
                                    : sort_walk<8>(W, c, t, ex, lane, cut);
    if (reached) {
      *ncand = c;
      return kCut;
    }
    if (all_nonzero) return kTakeAll;  // the whole row sums to less than t
    __syncwarp();  // the next attempt overwrites the candidates
  }
  return kUndecided;
}

// Writes one row's outputs for a decided outcome: the mask row (all NB
// columns), the ascending index list and the count.
__device__ __forceinline__ void emit(Outcome oc, unsigned long long cut, int ncand, int n, int NB,
                                     long long row, int lane, WarpBuf& W,
                                     uint32_t* __restrict__ mask, int32_t* __restrict__ counts,
                                     int32_t* __restrict__ idx) {
  const int Wn = (NB + 31) / 32;
  uint32_t* mrow = mask + row * Wn;
  int32_t* irow = idx + row * NB;
  if (oc == kTakeAll) {
    for (int w = lane; w < Wn; w += 32) {
      const int left = n - 32 * w;
      mrow[w] = left >= 32 ? 0xFFFFFFFFu : (left <= 0 ? 0u : (1u << left) - 1u);
    }
    for (int j = lane; j < n; j += 32) irow[j] = j;
    if (lane == 0) counts[row] = n;
    return;
  }
  for (int w = lane; w < Wn; w += 32) W.words[w] = 0u;
  __syncwarp();
  int running = 0;
  const unsigned lt = (1u << lane) - 1u;
  if (oc == kCut) {
    for (int i0 = 0; i0 < ncand; i0 += 32) {
      const int i = i0 + lane;
      const unsigned long long key = i < ncand ? W.cand[i] : 0ull;
      const bool sel = i < ncand && key >= cut;
      const unsigned b = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int j = key_index(key);
        irow[running + __popc(b & lt)] = j;
        atomicOr(&W.words[j >> 5], 1u << (j & 31));
      }
      running += __popc(b);
    }
  }
  __syncwarp();
  for (int w = lane; w < Wn; w += 32) mrow[w] = W.words[w];
  if (lane == 0) counts[row] = running;
  __syncwarp();  // the staging is reused by the warp's next row
}

}  // namespace filt
}  // namespace xattn
