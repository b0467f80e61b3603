// sched.cu -- longest-list-first order of the sparse-attention work units.
//
// A work unit is one (batch*head, query block) pair; its cost is proportional
// to its number of selected key blocks. Causal lists grow with the query-block
// index, so the units are ordered by count, descending (a counting sort over
// counts 0..NB in one CTA). The persistent attention CTAs then take units
// round-robin from this order, which spreads the long lists first.
#include "common.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
    sched_kernel(const int32_t* __restrict__ counts, int units, int NB,
                 uint32_t* __restrict__ order) {
  extern __shared__ int hist[];  // NB + 1 bins, bin = NB - count
  const int nbins = NB + 1;
  for (int i = threadIdx.x; i < nbins; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int u = threadIdx.x; u < units; u += kThreads) {
    int c = counts[u];
    c = c < 0 ? 0 : (c > NB ? NB : c);
    atomicAdd(&hist[NB - c], 1);
  }
  __syncthreads();
  // exclusive scan of the bins: each thread sums a contiguous chunk
  __shared__ int warp_tot[kThreads / 32];
  const int per = (nbins + kThreads - 1) / kThreads;
  const int lo = threadIdx.x * per;
  const int hi = min(lo + per, nbins);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += hist[i];
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
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
  for (int u = threadIdx.x; u < units; u += kThreads) {
    int c = counts[u];
    c = c < 0 ? 0 : (c > NB ? NB : c);
    const int pos = atomicAdd(&hist[NB - c], 1);
    order[pos] = static_cast<uint32_t>(u);
  }
}

}  // namespace

cudaError_t launch_sched(const Dims& D, const int32_t* counts, uint32_t* order,
                         cudaStream_t st) {
  const int units = D.batch * D.hq * D.NB;
  const size_t smem = static_cast<size_t>(D.NB + 1) * sizeof(int);
  sched_kernel<<<1, kThreads, smem, st>>>(counts, units, D.NB, order);
  return cudaGetLastError();
}

}  // namespace xattn
