// reduce_core.cuh -- block probabilities of one query block from the scoring
// partials ("XAttention: Block Sparse Attention with Antidiagonal Scoring",
// §2.2: softmax of the antidiagonal sums, then the sum over each block),
// shared by the reduce kernel and the fused score->select kernel so that both
// produce the same P bit for bit.
//
// Input: for every reshaped query row rho and allowed key block j, the partial
// L[rho, j] = log2 sum_{c in block j} 2^(x[rho, c] log2 e). For query block b
// with r_b reshaped rows (r, or fewer for a short last block):
//   LSE[rho]  = log2 sum_j 2^L[rho, j]                (row normaliser)
//   P[b, j]   = (1/r_b) sum_{rho in block b} 2^(L[rho, j] - LSE[rho])
// and P[b, j] = 0 for the causally masked j > b.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace red {

// Number of reshaped rows of query block b: r, or fewer for a short last block.
__device__ __forceinline__ int block_rows(int b, int r, int R) {
  const int left = R - b * r;
  return left < r ? left : r;
}

// Fills row_off[t] and lse[t] (t < rb, the block's reshaped rows) for query
// block b; every thread of the CTA takes part, and the function ends with
// __syncthreads.
__device__ __forceinline__ void block_row_lse(const float* __restrict__ base, int b, int NB, int r,
                                              int rb, int nj, bool causal, float* lse,
                                              size_t* row_off) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwarps = blockDim.x / 32;
  for (int t = threadIdx.x; t < rb; t += blockDim.x)
    row_off[t] = part_row_offset(b * r + t, r, NB, causal);
  __syncthreads();
  // row log-sum-exp: online (max, sum) over 8 loads in flight per lane
  for (int t = warp; t < rb; t += nwarps) {
    const float* row = base + row_off[t];
    float m = -INFINITY, s = 0.f;
    for (int j0 = 0; j0 < nj; j0 += 8 * 32) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * 32 + lane;
        v[u] = j < nj ? __ldg(row + j) : -INFINITY;
      }
      float cm = m;
#pragma unroll
      for (int u = 0; u < 8; ++u) cm = fmaxf(cm, v[u]);
      if (cm != -INFINITY) {
        float cs = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) cs += ex2(v[u] - cm);
        s = s * ex2(m - cm) + cs;
        m = cm;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      const float mm = fmaxf(m, m2);
      if (mm != -INFINITY) {
        s = s * ex2(m - mm) + s2 * ex2(m2 - mm);
        m = mm;
      }
    }
    if (lane == 0) lse[t] = m + lg2(s);
  }
  __syncthreads();
}

// P[b, j] for an allowed block j < nj over the block's r (= r_b) rows; r loads
// in flight per thread.
__device__ __forceinline__ float block_prob(const float* __restrict__ base, const size_t* row_off,
                                            const float* lse, int r, int j, float inv_r) {
  float acc = 0.f;
  int t = 0;
  for (; t + 8 <= r; t += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(base + row_off[t + u] + j);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += ex2(v[u] - lse[t + u]);
  }
  for (; t < r; ++t) acc += ex2(__ldg(base + row_off[t] + j) - lse[t]);
  return acc * inv_r;
}

}  // namespace red
}  // namespace xattn
