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
// kCand of them) into shared memory, sorts them across the warp with a bitonic
// network and walks them. A walk that covers every non-zero block without
// reaching tau takes the whole row. Rows that need more than kCand candidates
// (flat rows) are left to the histogram search (select_core.cuh).
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

constexpr int kCand = 64;       // candidates a warp sorts (two per lane)
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

// Bitonic sort, descending, of one key a lane (32 keys).
__device__ __forceinline__ unsigned long long sort32_desc(unsigned long long x, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, x, stride);
      const bool take_max = ((lane & size) == 0) == ((lane & stride) == 0);
      x = take_max ? (o > x ? o : x) : (o < x ? o : x);
    }
  }
  return x;
}

// Bitonic sort, descending, of 64 keys held two a lane: a at position lane,
// b at position lane + 32.
__device__ __forceinline__ void sort64_desc(unsigned long long& a, unsigned long long& b,
                                            int lane) {
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {  // partners sit in the same lane (only for size 64: descending)
        const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
        a = hi;
        b = lo;
      } else {
        const unsigned long long oa = __shfl_xor_sync(0xffffffffu, a, stride);
        const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b, stride);
        const bool lower = (lane & stride) == 0;
        const bool up_a = (lane & size) == 0;          // position lane
        const bool up_b = ((lane + 32) & size) == 0;   // position lane + 32
        a = (up_a == lower) ? (oa > a ? oa : a) : (oa < a ? oa : a);
        b = (up_b == lower) ? (ob > b ? ob : b) : (ob < b ? ob : b);
      }
    }
  }
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
    unsigned long long a = lane < c ? W.cand[lane] : 0ull;
    unsigned long long b = lane + 32 < c ? W.cand[lane + 32] : 0ull;
    if (c <= 32) {
      a = sort32_desc(a, lane);
    } else {
      sort64_desc(a, b, lane);
    }
    // the definition's walk: ranked order, one fp64 addition after another
    double acc = 0.0;
    for (int i = 0; i < c; ++i) {
      const unsigned long long key = __shfl_sync(0xffffffffu, i < 32 ? a : b, i & 31);
      acc += static_cast<double>(key_value(key));
      if (acc >= t) {
        *cut = key;
        *ncand = c;
        return kCut;
      }
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
