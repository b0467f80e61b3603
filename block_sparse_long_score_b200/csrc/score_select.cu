// score_select.cu -- block probabilities and find_blocks in one kernel
// ("XAttention: Block Sparse Attention with Antidiagonal Scoring", §2.2: the
// block sums of the antidiagonal softmax, then the threshold selection).
//
// One CTA per (batch*head, query block) row. All its warps reduce the scoring
// partials to the row of P (the same arithmetic as the reduce kernel, so P is
// bit-identical to xattn_score's) and stage it in shared memory; P goes to
// HBM only if the caller asks for it. Warp 0 then finds the find_blocks cut of
// the staged row (the selection kernel's threshold filter, and its histogram
// search for a row the filter leaves) and writes the mask, the count and the
// ascending index list; the other warps are done. Compared
// with xattn_score followed by xattn_select this saves P's write and re-read
// and one launch.
#include "reduce_core.cuh"
#include "select_core.cuh"
#include "select_filter.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 128;

__global__ void __launch_bounds__(kThreads)
    score_select_kernel(const float* __restrict__ part, float* __restrict__ probs,
                        const TauArg tau, int NB, int r, int R, int causal, int hq,
                        int nb_stage, uint32_t* __restrict__ mask, int32_t* __restrict__ counts,
                        int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem[];
  sel::WarpSmem& W = *reinterpret_cast<sel::WarpSmem*>(smem);
  filt::WarpBuf& FB = *reinterpret_cast<filt::WarpBuf*>(smem + sizeof(sel::WarpSmem));
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + sizeof(sel::WarpSmem) +
                                               sizeof(filt::WarpBuf));  // nb_stage
  size_t* row_off = reinterpret_cast<size_t*>(keys + nb_stage);                 // r
  float* lse = reinterpret_cast<float*>(row_off + r);                           // r
  const int b = blockIdx.x;
  const int bh = blockIdx.y;
  const int nj = causal ? b + 1 : NB;
  const float* base = part + static_cast<size_t>(bh) * part_head_elems(NB, r, R, causal != 0);
  const int rb = red::block_rows(b, r, R);
  red::block_row_lse(base, b, NB, r, rb, nj, causal != 0, lse, row_off);

  const long long row = static_cast<long long>(bh) * NB + b;
  float* out = probs ? probs + row * NB : nullptr;
  const float inv_r = 1.0f / static_cast<float>(rb);
  for (int j = threadIdx.x; j < NB; j += kThreads) {
    const float pj = j < nj ? red::block_prob(base, row_off, lse, rb, j, inv_r) : 0.f;
    if (out) out[j] = pj;
    if (j < nj) keys[j] = __float_as_uint(pj) & 0x7FFFFFFFu;
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;

  // ---- warp 0: find_blocks on the staged row: the threshold filter of the
  // selection kernel first, the histogram search for a row it leaves
  const int lane = threadIdx.x;
  const double t = tau_of(tau, bh % hq);
  {
    auto ld = [keys](int j) { return keys[j]; };
    const filt::MemRow<decltype(ld)> mr{ld};
    unsigned long long cut = 0;
    int ncand = 0;
    const filt::Outcome oc = filt::filter_cut(mr, nj, t, lane, FB, &cut, &ncand);
    if (oc != filt::kUndecided) {
      filt::emit(oc, cut, ncand, nj, NB, row, lane, FB, mask, counts, idx);
      return;
    }
  }
  // (sums in the selection kernel's order: each lane adds its blocks
  // j = lane, lane + 32, ... in turn)
  double tot = 0.0;
  uint32_t kmax = 0;
  for (int j = lane; j < nj; j += 32) {
    const uint32_t k = keys[j];
    tot += static_cast<double>(__uint_as_float(k));
    kmax = max(kmax, k);
  }
  tot = sel::warp_sum_d(tot);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  bool take_all = false;
  uint32_t vstar = 0xFFFFFFFFu;  // selects nothing (an invalid device tau)
  int icut = -1;
  if (t >= 0.0) sel::find_cut(keys, nj, t, tot, kmax, W, lane, take_all, vstar, icut);
  sel::emit_row(keys, nj, NB, take_all, vstar, icut, row, lane, mask, counts, idx);
}

}  // namespace

// Shapes the staged kernel of score_bulk.cu does not take (r above 32, i.e.
// strides 1 and 2 at B = 128, or a workspace that is not 16-byte aligned).
cudaError_t launch_score_select_wide(const Dims& D, const float* part, float* probs,
                                     const TauArg& tau, uint32_t* mask, int32_t* counts,
                                     int32_t* idx, cudaStream_t st) {
  const int nb_stage = (D.NB + 3) & ~3;
  const size_t smem = sizeof(sel::WarpSmem) + sizeof(filt::WarpBuf) +
                      static_cast<size_t>(nb_stage) * 4 +
                      static_cast<size_t>(D.r) * (sizeof(size_t) + sizeof(float));
  cudaError_t e = cudaFuncSetAttribute(score_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(D.NB, D.batch * D.hq);
  score_select_kernel<<<grid, kThreads, smem, st>>>(part, probs, tau, D.NB, D.r, D.R, D.causal,
                                                    D.hq, nb_stage, mask, counts, idx);
  return cudaGetLastError();
}

}  // namespace xattn
