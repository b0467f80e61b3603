// score_simt.cu -- fp32 antidiagonal scoring on CUDA cores, for small fp32
// problems ("XAttention: Block Sparse Attention with Antidiagonal Scoring",
// §2.1 and Algorithm 1). It writes the same partial log2-sum-exp layout as the
// tensor-core kernel, so the same reduce kernel produces P.
//
// One CTA per (reshaped query row rho, batch*head). The reshaped query row
// [Q[rho S + S-1], ..., Q[rho S]] (in general [Q[rho S + q[0]], ...,
// Q[rho S + q[S-1]]] for a pattern permutation q) is staged in shared memory. Each warp takes
// one key block at a time; its lanes take that block's reshaped columns c,
// whose reshaped key rows K[c S .. c S + S-1] are contiguous in memory.
#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float mm = fmaxf(m, m2);
  s = s * ex2(m - mm) + s2 * ex2(m2 - mm);
  m = mm;
}

__global__ void __launch_bounds__(kThreads)
    score_simt_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                      float* __restrict__ part, Dims D, float sl2, PermArg perm) {
  extern __shared__ float qr[];  // S * d
  const int rho = blockIdx.x;
  const int bh = blockIdx.y;
  const int kvbh = (bh / D.hq) * D.hkv + (bh % D.hq) / D.group;
  const int SD = D.S * D.d;
  const float* Qh = Q + static_cast<size_t>(bh) * D.L * D.d;
  const float* Kh = K + static_cast<size_t>(kvbh) * D.L * D.d;

  for (int e = threadIdx.x; e < SD; e += kThreads) {
    const int i = e / D.d, f = e % D.d;
    qr[e] = Qh[static_cast<size_t>(rho * D.S + perm.q[i]) * D.d + f];
  }
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = rho / D.r;
  const int jmax = D.causal ? b : D.NB - 1;
  float* prow = part + static_cast<size_t>(bh) * part_head_elems(D.NB, D.r, D.R, D.causal != 0) +
                part_row_offset(rho, D.r, D.NB, D.causal != 0);
  for (int j = warp; j <= jmax; j += kThreads / 32) {
    float m = -INFINITY, s = 0.f;
    for (int cc = lane; cc < D.r; cc += 32) {
      const int c = j * D.r + cc;
      if (c >= D.R || (D.causal && c > rho)) continue;  // short last block / causal
      const float* kr = Kh + static_cast<size_t>(c) * SD;
      float x = 0.f;
      for (int e = 0; e < SD; ++e) x = fmaf(qr[e], kr[e], x);
      lse_merge(m, s, x * sl2, 1.0f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      lse_merge(m, s, m2, s2);
    }
    if (lane == 0) prow[j] = m + lg2(s);
  }
}

}  // namespace

cudaError_t launch_score_simt(const Dims& D, const float* Q, const float* K,
                              const PermArg& perm, float* part, cudaStream_t st) {
  const float sl2 = static_cast<float>(1.4426950408889634 / sqrt(double(D.d) * D.S));
  const size_t smem = static_cast<size_t>(D.S) * D.d * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(score_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(D.R, D.batch * D.hq);
  score_simt_kernel<<<grid, kThreads, smem, st>>>(Q, K, part, D, sl2, perm);
  return cudaGetLastError();
}

}  // namespace xattn
