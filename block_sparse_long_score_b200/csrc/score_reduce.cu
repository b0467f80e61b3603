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
  extern __shared__ float smem[];
  float* lse = smem;                                   // r entries
  size_t* row_off = reinterpret_cast<size_t*>(smem + ((r + 1) & ~1));  // r entries
  const int b = blockIdx.x;
  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwarps = kThreads / 32;
  const int nj = causal ? b + 1 : NB;
  const float* base = part + static_cast<size_t>(bh) * part_head_elems(NB, r, R, causal != 0);

  for (int t = threadIdx.x; t < r; t += kThreads)
    row_off[t] = part_row_offset(b * r + t, r, NB, causal != 0);
  __syncthreads();
  // row log-sum-exp: online (max, sum) over 8 loads in flight per lane
  for (int t = warp; t < r; t += nwarps) {
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

  // P[b, j] = (1/r) sum_t 2^(part[t][j] - lse[t]); r loads in flight per thread
  float* out = probs + (static_cast<size_t>(bh) * NB + b) * NB;
  const float inv_r = 1.0f / static_cast<float>(r);
  for (int j = threadIdx.x; j < NB; j += kThreads) {
    float acc = 0.f;
    if (j < nj) {
      int t = 0;
      for (; t + 8 <= r; t += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = __ldg(base + row_off[t + u] + j);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc += ex2(v[u] - lse[t + u]);
      }
      for (; t < r; ++t)
        acc += ex2(__ldg(base + row_off[t] + j) - lse[t]);
    }
    out[j] = acc * inv_r;
  }
}

}  // namespace

cudaError_t launch_score_reduce(const Dims& D, const float* part, float* probs,
                                cudaStream_t st) {
  dim3 grid(D.NB, D.batch * D.hq);
  const size_t smem = ((D.r + 1) & ~1) * sizeof(float) + D.r * sizeof(size_t);
  score_reduce_kernel<<<grid, kThreads, smem, st>>>(part, probs, D.NB, D.r, D.R, D.causal);
  return cudaGetLastError();
}

}  // namespace xattn
