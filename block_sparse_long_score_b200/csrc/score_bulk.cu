// score_bulk.cu -- block probabilities from the scoring partials, and
// find_blocks on them, with each query block's partials staged in shared
// memory by one bulk copy ("XAttention: Block Sparse Attention with
// Antidiagonal Scoring", §2.2: the block sums of the antidiagonal softmax,
// then the threshold selection).
//
// Input: for every reshaped query row rho and allowed key block j, the partial
// L[rho, j] = log2 sum_{c in block j} 2^(x[rho, c] log2 e). For query block b
// with r_b reshaped rows t (r, or fewer for a short last block):
//   M_t = max_j L[t, j],  e[t, j] = 2^(L[t, j] - M_t),  S_t = sum_j e[t, j]
//   P[b, j] = (1/r_b) sum_t e[t, j] / S_t
// and P[b, j] = 0 for the causally masked j > b.
//
// The partials of a query block are one contiguous r_b x n_j array (row t at
// t * n_j). One thread copies it into shared memory with a single bulk copy
// (the TMA engine moves it; no registers wait on it), so every resident CTA
// keeps a whole block in flight. The CTA then works from shared memory: a
// warp per row takes M_t, writes e in place (one exp2 per partial) and sums
// S_t; then every thread forms P for its columns. A block too large for the
// stage, or whose array is not 16-byte aligned, is read from global memory
// with the two-pass arithmetic of reduce_core.cuh instead.
//
// For xattn_score_select the kernel also writes each block's row of P (its
// n_j allowed entries) over the first partials of the block, which the CTA has
// consumed; the selection kernels then read the rows from there, with no
// separate P buffer. xattn_score and xattn_score_select both run this kernel,
// with the same choice of path for every block, so their P, and the lists
// find_blocks takes from it, are bit-identical.
#include "ptx.cuh"
#include "reduce_core.cuh"

namespace xattn {

cudaError_t launch_score_reduce_wide(const Dims& D, const float* part, float* probs,
                                     cudaStream_t st);
cudaError_t launch_score_select_wide(const Dims& D, const float* part, float* probs,
                                     const TauArg& tau, uint32_t* mask, int32_t* counts,
                                     int32_t* idx, cudaStream_t st);

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kMinR = 1, kMaxR = 32;        // r this kernel takes
constexpr int kStageCap = 32 * 1024 / 4;    // floats of the staging buffer at most

__global__ void __launch_bounds__(kThreads)
    score_bulk_kernel(const float* __restrict__ part, float* __restrict__ probs, int NB, int r,
                      int R, int causal, int stage_floats, int p_to_part,
                      int* __restrict__ status) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* stage = reinterpret_cast<float*>(smem);  // stage_floats
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ float row_inv[kMaxR];
  __shared__ float lse[kMaxR];
  __shared__ size_t row_off[kMaxR];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x;
  const int bh = blockIdx.y;
  const int nj = causal ? b + 1 : NB;
  const int rb = red::block_rows(b, r, R);
  const float* head = part + static_cast<size_t>(bh) * part_head_elems(NB, r, R, causal != 0);
  float* base = const_cast<float*>(head) + part_row_offset(b * r, r, NB, causal != 0);
  const long long row = static_cast<long long>(bh) * NB + b;
  float* prow = probs ? probs + row * NB : nullptr;
  float* srow = p_to_part ? base : nullptr;  // the row of P over the consumed partials
  const float inv_rb = 1.0f / static_cast<float>(rb);

  const size_t bytes = static_cast<size_t>(rb) * nj * sizeof(float);
  const bool staged = bytes <= static_cast<size_t>(stage_floats) * sizeof(float) &&
                      (bytes & 15u) == 0 && (reinterpret_cast<uintptr_t>(base) & 15u) == 0;
  if (staged) {
    if (tid == 0) {
      mbar_init(&bar, 1);
      abort_flag = 0;
      fence_barrier_init();
    }
    __syncthreads();
    if (tid == 0) {
      mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(bytes));
      bulk_load(stage, base, static_cast<uint32_t>(bytes), &bar);
    }
    volatile int* abort = &abort_flag;
    if (!warp_wait(&bar, 0, abort)) {
      // the copy did not land within the time limit: record it, and give the
      // copy (bounded) time to finish before the CTA's shared memory is freed
      if (tid == 0) atomicExch(status, kStatusTimeout);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(&bar), 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
      return;
    }
    // a warp per row: M_t, e in place, S_t
    for (int t = warp; t < rb; t += kWarps) {
      float* rowp = stage + static_cast<size_t>(t) * nj;
      float m = -INFINITY;
      for (int j = lane; j < nj; j += 32) m = fmaxf(m, rowp[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float s = 0.f;
      for (int j = lane; j < nj; j += 32) {
        const float e = ex2(rowp[j] - m);
        rowp[j] = e;
        s += e;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) row_inv[t] = 1.0f / s;
    }
    __syncthreads();
    for (int j = tid; j < nj; j += kThreads) {
      float p = 0.f;
      for (int t = 0; t < rb; ++t) p = fmaf(stage[static_cast<size_t>(t) * nj + j], row_inv[t], p);
      p *= inv_rb;
      if (prow) prow[j] = p;
      if (srow) srow[j] = p;
    }
  } else {
    // the block does not fit the stage (or its array is misaligned): the
    // two-pass reduce straight from global memory. Column j of the block is
    // read only by the thread that writes the row of P there.
    red::block_row_lse(head, b, NB, r, rb, nj, causal != 0, lse, row_off);
    for (int j = tid; j < nj; j += kThreads) {
      const float p = red::block_prob(head, row_off, lse, rb, j, inv_rb);
      if (prow) prow[j] = p;
      if (srow) srow[j] = p;
    }
  }
  if (prow)
    for (int j = nj + tid; j < NB; j += kThreads) prow[j] = 0.f;  // causally masked blocks
}

// Floats of the staging buffer: the largest block's partials, up to the cap.
int stage_floats_for(const Dims& D) {
  const long long most = static_cast<long long>(D.r) * D.NB;
  const long long f = most < kStageCap ? most : kStageCap;
  return static_cast<int>((f + 3) & ~3ll);
}

bool takes(const Dims& D, const float* part) {
  return D.r >= kMinR && D.r <= kMaxR && (reinterpret_cast<uintptr_t>(part) & 15u) == 0;
}

cudaError_t launch_bulk(const Dims& D, const float* part, float* probs, bool p_to_part,
                        int* status, cudaStream_t st) {
  const int sf = stage_floats_for(D);
  const size_t smem = static_cast<size_t>(sf) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(score_bulk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(D.NB, D.batch * D.hq);
  score_bulk_kernel<<<grid, kThreads, smem, st>>>(part, probs, D.NB, D.r, D.R, D.causal, sf,
                                                  p_to_part ? 1 : 0, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_reduce(const Dims& D, const float* part, float* probs, int* status,
                                cudaStream_t st) {
  if (!takes(D, part)) return launch_score_reduce_wide(D, part, probs, st);
  return launch_bulk(D, part, probs, false, status, st);
}

cudaError_t launch_score_select(const Dims& D, const float* part, float* probs,
                                const TauArg& tau, uint32_t* mask, int32_t* counts, int32_t* idx,
                                int* status, int num_sms, cudaStream_t st) {
  if (!takes(D, part))
    return launch_score_select_wide(D, part, probs, tau, mask, counts, idx, st);
  cudaError_t e = launch_bulk(D, part, probs, true, status, st);
  if (e != cudaSuccess) return e;
  // find_blocks on the rows of P written over the consumed partials
  const RowSource src{part, 1, part_head_elems(D.NB, D.r, D.R, D.causal != 0), D.r};
  return launch_select_rows(D, src, tau, mask, counts, idx, num_sms, st);
}

}  // namespace xattn
