// sched.cu -- the order in which the persistent attention CTAs take the
// sparse-attention work units.
//
// A work unit is one (batch*head, query block) pair; its cost is proportional
// to its number of selected key blocks. Causal lists grow with the query-block
// index, so the units are ordered by block count, descending (a counting sort
// over counts 0..NB in one CTA). The CTAs take entries round-robin, and every
// other round of the order is reversed (serpentine), so the long lists are
// spread first and evenly. When the lists are long on average, the order is
// grouped by KV head first, so that all CTAs work on one head's K/V at a
// time (it stays in L2); the kernel decides from the count histogram.
//
// Each order entry packs everything the attention kernel needs to start a
// unit into one 64-bit word, so that it costs one (prefetchable) load:
//   bits  0..31  unit index (bh * NB + query block)
//   bits 32..47  effective block count: causal lists drop trailing blocks above
//                the diagonal (lists are ascending)
//   bit  48      the last listed block needs a column mask: it is the diagonal
//                block (causal), or the short last block of a sequence whose
//                length B does not divide (non-causal)
#include "common.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 1024;

// Effective block count and mask flag (bit 48) of units u, u + kThreads, ...
// (8 of them): causal lists drop trailing blocks above the diagonal.
__device__ __forceinline__ void unit_info8(const int32_t* __restrict__ counts,
                                           const int32_t* __restrict__ idx, int u, int units,
                                           int NB, int causal, int ragged, int (&n)[8],
                                           bool (&diag)[8]) {
  int c[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int uu = u + q * kThreads;
    const int v = uu < units ? counts[uu] : 0;
    c[q] = v < 0 ? 0 : (v > NB ? NB : v);
  }
  if (causal) {
    int last[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int uu = u + q * kThreads;
      last[q] = (uu < units && c[q] > 0) ? idx[static_cast<size_t>(uu) * NB + c[q] - 1] : -1;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int uu = u + q * kThreads;
      const int qb = uu % NB;
      if (uu < units && last[q] > qb) {  // rare: trailing blocks above the diagonal
        const int32_t* list = idx + static_cast<size_t>(uu) * NB;
        while (c[q] > 0 && list[c[q] - 1] > qb) --c[q];
        last[q] = c[q] > 0 ? list[c[q] - 1] : -1;
      }
      diag[q] = uu < units && c[q] > 0 && last[q] == qb;
    }
  } else if (ragged) {
    // non-causal with a short last block: lists are ascending, so block NB-1
    // can only be a list's last entry
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int uu = u + q * kThreads;
      diag[q] = uu < units && c[q] > 0 && idx[static_cast<size_t>(uu) * NB + c[q] - 1] == NB - 1;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) diag[q] = false;
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) n[q] = c[q];
}

// Lists at least this long on average (selected blocks per unit) make the
// K/V reuse inside a KV-head group worth grouping the order by group; with
// shorter lists the global longest-first order balances the CTAs better.
constexpr int kGroupMinAvgBlocks = 48;

__global__ void __launch_bounds__(kThreads)
    sched_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ idx, int units,
                 int NB, int causal, int ragged, int groups, int units_per_group, int ctas,
                 unsigned long long* __restrict__ order) {
  // plain[NB - count] counts units by length; grouped[g * (NB + 1) + NB - count]
  // by KV-head group and length (only when there is more than one group)
  extern __shared__ int bins[];
  int* plain = bins;
  int* grouped = bins + (NB + 1);
  const int ngrouped = groups > 1 ? groups * (NB + 1) : 0;
  for (int i = threadIdx.x; i < NB + 1 + ngrouped; i += kThreads) bins[i] = 0;
  __syncthreads();
  // 8 units per thread per batch: their load chains overlap
  for (int u0 = 0; u0 < units; u0 += 8 * kThreads) {
    int n[8];
    bool diag[8];
    unit_info8(counts, idx, u0 + threadIdx.x, units, NB, causal, ragged, n, diag);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int u = u0 + threadIdx.x + q * kThreads;
      if (u >= units) continue;
      atomicAdd(&plain[NB - n[q]], 1);
      if (ngrouped) atomicAdd(&grouped[(u / units_per_group) * (NB + 1) + NB - n[q]], 1);
    }
  }
  __syncthreads();
  // total selected blocks, from the length histogram
  __shared__ long long blk_tot[kThreads / 32];
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  long long blocks = 0;
  for (int i = threadIdx.x; i < NB + 1; i += kThreads)
    blocks += static_cast<long long>(plain[i]) * (NB - i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) blocks += __shfl_xor_sync(0xffffffffu, blocks, o);
  if (lane == 0) blk_tot[warp] = blocks;
  __syncthreads();
  long long total = 0;
  for (int w = 0; w < kThreads / 32; ++w) total += blk_tot[w];
  const bool by_group =
      ngrouped > 0 && total >= static_cast<long long>(kGroupMinAvgBlocks) * units;
  int* hist = by_group ? grouped : plain;
  const int nbins = by_group ? ngrouped : NB + 1;
  // exclusive scan of the chosen bins: each thread sums a contiguous chunk
  __shared__ int warp_tot[kThreads / 32];
  const int per = (nbins + kThreads - 1) / kThreads;
  const int lo = threadIdx.x * per;
  const int hi = min(lo + per, nbins);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += hist[i];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_tot[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of the warp totals
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - local;
  for (int i = lo; i < hi; ++i) {
    const int c = hist[i];
    hist[i] = run;
    run += c;
  }
  __syncthreads();
  for (int u0 = 0; u0 < units; u0 += 8 * kThreads) {
    int n[8];
    bool diag[8];
    unit_info8(counts, idx, u0 + threadIdx.x, units, NB, causal, ragged, n, diag);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int u = u0 + threadIdx.x + q * kThreads;
      if (u >= units) continue;
      const int bin = by_group ? (u / units_per_group) * (NB + 1) + NB - n[q] : NB - n[q];
      int pos = atomicAdd(&hist[bin], 1);
      // the attention CTAs deal the order out in rounds of `ctas` units (CTA
      // i takes entries i, i + ctas, ...); every other round runs backwards,
      // so the CTA that gets a round's longest unit gets the next round's
      // shortest
      const int round = pos / ctas;
      if (round & 1) {
        const int m = min(ctas, units - round * ctas);
        pos = round * ctas + (m - 1 - (pos - round * ctas));
      }
      order[pos] = static_cast<unsigned long long>(static_cast<uint32_t>(u)) |
                   (static_cast<unsigned long long>(n[q]) << 32) |
                   (static_cast<unsigned long long>(diag[q] ? 1 : 0) << 48);
    }
  }
}

}  // namespace

cudaError_t launch_sched(const Dims& D, const int32_t* counts, const int32_t* idx,
                         unsigned long long* order, int num_sms, cudaStream_t st) {
  const int units = D.batch * D.hq * D.NB;
  // With long lists, units are grouped by KV head (the hq/hkv query heads
  // that share one K/V), longest list first inside a group: the persistent
  // CTAs take units round-robin, so they all work on one group's K/V at a
  // time, which stays in L2, instead of every KV head at once. The kernel
  // makes the choice from the counts (kGroupMinAvgBlocks).
  int groups = D.batch * D.hkv;
  const int per_group = D.group * D.NB;  // units of one KV head (unit = bh * NB + qb)
  if (static_cast<size_t>(groups + 1) * (D.NB + 1) * sizeof(int) > 160 * 1024)
    groups = 1;  // too many bins for shared memory: the plain order only
  const size_t smem =
      static_cast<size_t>(groups > 1 ? groups + 1 : 1) * (D.NB + 1) * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(sched_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // the attention kernel runs min(SMs, units) persistent CTAs
  const int ctas = num_sms < units ? num_sms : (units > 0 ? units : 1);
  sched_kernel<<<1, kThreads, smem, st>>>(counts, idx, units, D.NB, D.causal,
                                          D.tail != D.B ? 1 : 0, groups, per_group, ctas,
                                          order);
  return cudaGetLastError();
}

}  // namespace xattn
