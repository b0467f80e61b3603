// attn_simt.cu -- fp32 block-sparse attention on CUDA cores, for small fp32
// problems ("XAttention: Block Sparse Attention with Antidiagonal Scoring",
// §1 step 3).
//
// One warp per query row. For each listed key block, the lanes take 32 keys at
// a time: each lane computes one score q . k / sqrt(d), the warp updates the
// online softmax, and each lane accumulates d/32 output features.
#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace {

constexpr int kWarps = 8;

template <int DW>  // d / 32 features per lane
__global__ void __launch_bounds__(kWarps * 32)
    attn_simt_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                     const float* __restrict__ V, const int32_t* __restrict__ counts,
                     const int32_t* __restrict__ idx, float* __restrict__ O,
                     float* __restrict__ lse, Dims D, float sl2) {
  __shared__ float qs[kWarps][DW * 32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long grow = static_cast<long long>(blockIdx.x) * kWarps + warp;
  const long long nrows = static_cast<long long>(D.batch) * D.hq * D.L;
  if (grow >= nrows) return;
  const int d = DW * 32;
  const int bh = static_cast<int>(grow / D.L);
  const int q = static_cast<int>(grow % D.L);
  const int qb = q / D.B;
  const int kvbh = (bh / D.hq) * D.hkv + (bh % D.hq) / D.group;
  const size_t unit = static_cast<size_t>(bh) * D.NB + qb;
  const int n = min(max(counts[unit], 0), D.NB);
  const int32_t* list = idx + unit * D.NB;
  const float* Kh = K + static_cast<size_t>(kvbh) * D.L * d;
  const float* Vh = V + static_cast<size_t>(kvbh) * D.L * d;

#pragma unroll
  for (int t = 0; t < DW; ++t) qs[warp][lane + 32 * t] = Q[static_cast<size_t>(grow) * d + lane + 32 * t];
  __syncwarp();

  float o[DW];
#pragma unroll
  for (int t = 0; t < DW; ++t) o[t] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int jj = 0; jj < n; ++jj) {
    const int kb = list[jj];
    if (D.causal && kb > qb) break;  // ascending list: the rest is above the diagonal
    if (kb < 0 || kb >= D.NB) continue;
    const int kend = min((kb + 1) * D.B, D.L);  // a short last block ends at L
    for (int k0 = kb * D.B; k0 < kend; k0 += 32) {
      const int key = k0 + lane;
      const bool valid = key < kend && !(D.causal && key > q);
      float sc = -INFINITY;
      if (valid) {
        const float* kr = Kh + static_cast<size_t>(key) * d;
        float acc = 0.f;
        for (int f = 0; f < d; ++f) acc = fmaf(qs[warp][f], kr[f], acc);
        sc = acc * sl2;
      }
      float mx = sc;
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      if (mx == -INFINITY) continue;
      const float m_new = fmaxf(m, mx);
      const float alpha = ex2(m - m_new);
      const float pv = valid ? ex2(sc - m_new) : 0.f;
      float ps = pv;
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      l = l * alpha + ps;
#pragma unroll
      for (int t = 0; t < DW; ++t) o[t] *= alpha;
      for (int kk = 0; kk < 32; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, pv, kk);
        if (pk == 0.f) continue;
        const float* vr = Vh + static_cast<size_t>(k0 + kk) * d;
#pragma unroll
        for (int t = 0; t < DW; ++t) o[t] = fmaf(pk, vr[lane + 32 * t], o[t]);
      }
      m = m_new;
    }
  }
  const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
  for (int t = 0; t < DW; ++t) O[static_cast<size_t>(grow) * d + lane + 32 * t] = o[t] * inv;
  if (lse && lane == 0) lse[grow] = l > 0.f ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace

cudaError_t launch_attn_simt(const Dims& D, const float* Q, const float* K, const float* V,
                             const int32_t* counts, const int32_t* idx, float* O, float* lse,
                             cudaStream_t st) {
  const float sl2 = static_cast<float>(1.4426950408889634 / sqrt(double(D.d)));
  const long long nrows = static_cast<long long>(D.batch) * D.hq * D.L;
  const unsigned grid = static_cast<unsigned>((nrows + kWarps - 1) / kWarps);
  switch (D.d) {
    case 32:
      attn_simt_kernel<1><<<grid, kWarps * 32, 0, st>>>(Q, K, V, counts, idx, O, lse, D, sl2);
      break;
    case 64:
      attn_simt_kernel<2><<<grid, kWarps * 32, 0, st>>>(Q, K, V, counts, idx, O, lse, D, sl2);
      break;
    default:
      attn_simt_kernel<4><<<grid, kWarps * 32, 0, st>>>(Q, K, V, counts, idx, O, lse, D, sl2);
      break;
  }
  return cudaGetLastError();
}

}  // namespace xattn
