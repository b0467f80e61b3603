// score_reduce.cu -- block probabilities from the scoring partials
// ("XAttention: Block Sparse Attention with Antidiagonal Scoring", §2.2:
// softmax of the antidiagonal sums, then the sum over each block).
//
// Input: for every reshaped query row rho and allowed key block j, the partial
// L[rho, j] = log2 sum_{c in block j} 2^(x[rho, c] log2 e). Per query block b:
//   LSE[rho]  = log2 sum_j 2^L[rho, j]                (row normaliser)
//   P[b, j]   = (1/r) sum_{rho in block b} 2^(L[rho, j] - LSE[rho])
// and P[b, j] = 0 for the causally masked j > b. Memory-bound: each partial is
// read twice (the second read hits L1/L2), P is written once, coalesced.
#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    score_reduce_kernel(const float* __restrict__ part, float* __restrict__ probs, int NB, int r,
                        int R, int causal) {
  extern __shared__ float lse[];  // r entries
  const int b = blockIdx.x;
  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwarps = kThreads / 32;
  const int nj = causal ? b + 1 : NB;
  const float* base = part + static_cast<size_t>(bh) * part_head_elems(NB, r, R, causal != 0);

  for (int t = warp; t < r; t += nwarps) {
    const float* row = base + part_row_offset(b * r + t, r, NB, causal != 0);
    float m = -INFINITY;
    for (int j = lane; j < nj; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
    for (int j = lane; j < nj; j += 32) s += ex2(row[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) lse[t] = m + lg2(s);
  }
  __syncthreads();

  float* out = probs + (static_cast<size_t>(bh) * NB + b) * NB;
  const float inv_r = 1.0f / static_cast<float>(r);
  for (int j = threadIdx.x; j < NB; j += kThreads) {
    float acc = 0.f;
    if (j < nj) {
      for (int t = 0; t < r; ++t) {
        const float* row = base + part_row_offset(b * r + t, r, NB, causal != 0);
        acc += ex2(row[j] - lse[t]);
      }
    }
    out[j] = acc * inv_r;
  }
}

}  // namespace

cudaError_t launch_score_reduce(const Dims& D, const float* part, float* probs,
                                cudaStream_t st) {
  dim3 grid(D.NB, D.batch * D.hq);
  score_reduce_kernel<<<grid, kThreads, D.r * sizeof(float), st>>>(part, probs, D.NB, D.r, D.R,
                                                                   D.causal);
  return cudaGetLastError();
}

}  // namespace xattn
