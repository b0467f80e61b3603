// common.cuh -- shapes, workspace layout and launcher declarations shared by
// the kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/xattn.h"

namespace xattn {

// Device status codes written into the per-device status word.
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadTau = 2;  // a device-resident tau was outside (0, 1] (or NaN)

struct Dims {
  int batch, hq, hkv, L, d, B, S, causal, dtype;
  int NB, r, R, group;  // ceil(L/B), B/S, L/S, hq/hkv
  int tail;             // tokens of the last block: L - (NB-1)*B (B when B divides L)
};

// Partial log-sum-exp workspace of the scoring step.
//
// For every (batch, query head) there is one fp32 entry per (reshaped query
// row rho, allowed key block j): log2 of the sum over the reshaped columns c
// of block j of 2^(x[rho, c] * log2(e)), with x the scaled reshaped logits.
// Causal rows of query block b = rho / r keep only j <= b, packed
// row after row. Non-causal rows keep all NB entries.
__host__ __device__ inline size_t part_head_elems(int NB, int r, int R, bool causal) {
  return causal ? static_cast<size_t>(r) * NB * (NB + 1) / 2
                : static_cast<size_t>(R) * NB;
}

__host__ __device__ inline size_t part_row_offset(int rho, int r, int NB, bool causal) {
  if (!causal) return static_cast<size_t>(rho) * NB;
  const size_t b = static_cast<size_t>(rho / r);
  const size_t t = static_cast<size_t>(rho % r);
  return static_cast<size_t>(r) * b * (b + 1) / 2 + t * (b + 1);
}

// Sampling pattern of the scoring step: feature chunk i of a reshaped row
// pairs query sub-row q[i] with key sub-row i of every S x S tile. The
// antidiagonal is q[i] = S-1-i. Entries past S are unused.
struct PermArg {
  uint8_t q[256];
};

// Fixed-budget selection (Top-K / Top-Ratio): per query head either a block
// count k, or a ratio of the row's allowed blocks.
struct BudgetArg {
  int32_t k[XATTN_MAX_HEADS];
  float ratio[XATTN_MAX_HEADS];
  int use_ratio;
};

// ------------------------------------------------------------ launchers
// Each returns cudaSuccess or the launch error. All are asynchronous.

// bf16 tensor-core scoring GEMM: partials for every (bh, rho, allowed j).
// One CTA per 128 x 256 tile; the key map's box is 256 reshaped rows.
cudaError_t launch_score_tc(const Dims& D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                            const PermArg& perm, float* part, int* status, int num_sms,
                            cudaStream_t st);
// The same partials from CTA pairs, one 256 x 256 tile per pair (M = 256
// MMAs across two SMs); the key map's box is 128 reshaped rows.
cudaError_t launch_score_tc_pair(const Dims& D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                 const PermArg& perm, float* part, int* status, int num_sms,
                                 cudaStream_t st);
// Strides from which the pair kernel is used (a tile then has 2S >= 16
// k-steps; with fewer, the epilogue bounds a tile and one CTA per tile is
// faster).
constexpr int kScorePairMinS = 8;

// fp32 CUDA-core scoring, same partial layout.
cudaError_t launch_score_simt(const Dims& D, const float* Q, const float* K,
                              const PermArg& perm, float* part, cudaStream_t st);

// partials -> block probabilities P [bh, NB, NB].
cudaError_t launch_score_reduce(const Dims& D, const float* part, float* probs, int* status,
                                cudaStream_t st);

// Per-head thresholds: read from the device array `dev` when it is set (the
// C ABI's xattn_select / xattn_score_select), else taken from `v` (calls that
// receive tau in host memory and pass it by value). A device value outside
// (0, 1] is reported through `status` (kStatusBadTau) and its head's rows
// select nothing.
struct TauArg {
  float v[XATTN_MAX_HEADS];
  const float* dev;
  int* status;
};

// tau of query head h, or a negative value when a device-resident tau is
// invalid (the caller then selects nothing and the status word records it).
__device__ __forceinline__ double tau_of(const TauArg& tau, int h) {
  if (tau.dev == nullptr) return static_cast<double>(tau.v[h]);
  const float t = __ldg(tau.dev + h);
  if (t > 0.0f && t <= 1.0f) return static_cast<double>(t);  // false for NaN
  atomicExch(tau.status, kStatusBadTau);
  return -1.0;
}

// find_blocks on every row of P (a register-only walk of the ranking, then
// the histogram search on the rows it leaves; num_sms sizes that second grid).
cudaError_t launch_select(const Dims& D, const float* probs, const TauArg& tau, uint32_t* mask,
                          int32_t* counts, int32_t* idx, int num_sms, cudaStream_t st);

// partials -> P (optional) and find_blocks, fused (same outputs as
// launch_score_reduce followed by launch_select); num_sms sizes the grid of
// the histogram search for rows the threshold filter leaves. `status` receives
// time-outs of the kernel's bounded waits.
cudaError_t launch_score_select(const Dims& D, const float* part, float* probs,
                                const TauArg& tau, uint32_t* mask, int32_t* counts, int32_t* idx,
                                int* status, int num_sms, cudaStream_t st);

// Where the histogram search finds the P row of a marked row: in P itself
// ([rows][NB], layout 0), or written over the first partials of the row's
// query block (layout 1: part + bh * part_head + part_row_offset(b * r)).
struct RowSource {
  const float* p;
  int layout;
  size_t part_head;
  int r;
};

// find_blocks on every row of P read from `src` (the threshold filter, then
// the histogram search on the rows it leaves).
cudaError_t launch_select_rows(const Dims& D, const RowSource& src, const TauArg& tau,
                               uint32_t* mask, int32_t* counts, int32_t* idx, int num_sms,
                               cudaStream_t st);

// The histogram search of find_blocks on the rows marked with count -1.
cudaError_t launch_select_fallback(const Dims& D, const RowSource& src, const TauArg& tau,
                                   uint32_t* mask, int32_t* counts, int32_t* idx, int num_sms,
                                   cudaStream_t st);

// One CTA whose bounded wait runs out (failure-detection self-test).
cudaError_t launch_selftest_timeout(int* status, cudaStream_t st);

// Top-K / Top-Ratio on every row of P (same outputs as launch_select).
cudaError_t launch_select_budget(const Dims& D, const float* probs, const BudgetArg& budget,
                                 uint32_t* mask, int32_t* counts, int32_t* idx,
                                 cudaStream_t st);

// Longest-list-first order of the work units (bh, b) into `order`: one packed
// 64-bit entry per unit (unit index, effective block count, diagonal flag).
cudaError_t launch_sched(const Dims& D, const int32_t* counts, const int32_t* idx,
                         unsigned long long* order, int num_sms, cudaStream_t st);

// bf16 tensor-core block-sparse attention.
cudaError_t launch_attn_tc(const Dims& D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const int32_t* counts, const int32_t* idx,
                           const unsigned long long* order, void* O, float* lse, int* status,
                           int num_sms, cudaStream_t st);

// fp32 CUDA-core block-sparse attention.
cudaError_t launch_attn_simt(const Dims& D, const float* Q, const float* K, const float* V,
                             const int32_t* counts, const int32_t* idx, float* O, float* lse,
                             cudaStream_t st);

}  // namespace xattn
