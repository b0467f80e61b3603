// score_reduce.cu -- block probabilities from the scoring partials
// ("XAttention: Block Sparse Attention with Antidiagonal Scoring", §2.2:
// softmax of the antidiagonal sums, then the sum over each block).
//
// Input: for every reshaped query row rho and allowed key block j, the partial
// L[rho, j] = log2 sum_{c in block j} 2^(x[rho, c] log2 e). Per query block b:
//   LSE[rho]  = log2 sum_j 2^L[rho, j]                (row normaliser)
//   P[b, j]   = (1/r_b) sum_{rho in block b} 2^(L[rho, j] - LSE[rho])
// (r_b = r reshaped rows, or fewer for a short last block)
// and P[b, j] = 0 for the causally masked j > b. Memory-bound: each partial is
// read twice (the second read hits L1/L2), P is written once, coalesced.
#include "reduce_core.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    score_reduce_kernel(const float* __restrict__ part, float* __restrict__ probs, int NB, int r,
                        int R, int causal) {
  extern __shared__ float smem[];
  float* lse = smem;                                                   // r entries
  size_t* row_off = reinterpret_cast<size_t*>(smem + ((r + 1) & ~1));  // r entries
  const int b = blockIdx.x;
  const int bh = blockIdx.y;
  const int nj = causal ? b + 1 : NB;
  const float* base = part + static_cast<size_t>(bh) * part_head_elems(NB, r, R, causal != 0);
  const int rb = red::block_rows(b, r, R);
  red::block_row_lse(base, b, NB, r, rb, nj, causal != 0, lse, row_off);
  float* out = probs + (static_cast<size_t>(bh) * NB + b) * NB;
  const float inv_r = 1.0f / static_cast<float>(rb);
  for (int j = threadIdx.x; j < NB; j += kThreads)
    out[j] = j < nj ? red::block_prob(base, row_off, lse, rb, j, inv_r) : 0.f;
}

}  // namespace

// Shapes the staged kernel of score_bulk.cu does not take (r above 32, i.e.
// strides 1 and 2 at B = 128, or a workspace that is not 16-byte aligned): the
// two-pass reduce of
// reduce_core.cuh straight from global memory.
cudaError_t launch_score_reduce_wide(const Dims& D, const float* part, float* probs,
                                     cudaStream_t st) {
  dim3 grid(D.NB, D.batch * D.hq);
  const size_t smem = ((D.r + 1) & ~1) * sizeof(float) + D.r * sizeof(size_t);
  score_reduce_kernel<<<grid, kThreads, smem, st>>>(part, probs, D.NB, D.r, D.R, D.causal);
  return cudaGetLastError();
}

}  // namespace xattn
