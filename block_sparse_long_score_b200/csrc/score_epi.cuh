// score_epi.cuh -- the parts of the scoring kernels ("XAttention: Block
// Sparse Attention with Antidiagonal Scoring", §2.1 and Algorithm 1) that do
// not depend on how a tile's GEMM is issued: the launch parameters and the
// epilogue, which reduces each row of a 256-column accumulator tile to one
// partial log2-sum-exp per key block. score_tc.cu (one CTA per 128 x 256
// tile) and score_tc_pair.cu (a CTA pair per 256 x 256 tile) both use it.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace scoring {

constexpr int kBN = 256;            // reshaped key columns per tile
constexpr int kBK = 64;             // features per stage (one 128-byte swizzle row)

struct Params {
  int R, S, r, NB, causal, hq, hkv, group;
  int MT, NT, tiles_per_head;
  long long total_tiles;
  float scale_log2;     // log2(e) / sqrt(d * S)
  PermArg perm;         // query sub-row of each key sub-row (antidiagonal: S-1-i)
  float* part;
  size_t part_head;     // floats per (batch, head)
  int* status;
};

// Reduces one 32-column chunk of a row into per-key-block partials.
// RP = reshaped columns per key block (r). For RP <= 32 each chunk holds whole
// blocks; for RP > 32 a block spans RP/32 chunks and (m, s) carry across.
template <int RP>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&v)[32], int c0, int rho,
                                               int R, int jmax, bool need_mask, bool causal,
                                               float sl2, float* prow, float& m_run,
                                               float& s_run) {
  float x[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float a = __uint_as_float(v[i]);
    if (need_mask) {
      const int c = c0 + i;
      if (c >= R || (causal && c > rho)) a = -INFINITY;
    }
    x[i] = a;
  }
  if constexpr (RP <= 32) {
#pragma unroll
    for (int g = 0; g < 32 / RP; ++g) {
      const int j = (c0 + g * RP) / RP;
      if (j > jmax) continue;
      float m = x[g * RP];
      if constexpr (RP == 2) m = fmaxf(m, x[g * RP + 1]);
#pragma unroll
      for (int i = 1; i + 1 < RP; i += 2) m = fmax3(m, x[g * RP + i], x[g * RP + i + 1]);
      if constexpr (RP > 2 && (RP % 2) == 0) m = fmaxf(m, x[g * RP + RP - 1]);
      if (m == -INFINITY) {  // no visible column (cannot happen for j <= jmax)
        prow[j] = -INFINITY;
        continue;
      }
      const float mb = m * sl2;
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < RP; ++i) s += ex2(fmaf(x[g * RP + i], sl2, -mb));
      prow[j] = mb + lg2(s);
    }
  } else {
    float m = x[0];
#pragma unroll
    for (int i = 1; i < 31; i += 2) m = fmax3(m, x[i], x[i + 1]);
    m = fmaxf(m, x[31]);
    const float mb = m * sl2;
    float s = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int i = 0; i < 32; ++i) s += ex2(fmaf(x[i], sl2, -mb));
    }
    // combine with the running (max, sum) of this key block
    if (mb > m_run) {
      s_run = s_run * ex2(m_run - mb) + s;
      m_run = mb;
    } else if (mb != -INFINITY) {
      s_run += s * ex2(mb - m_run);
    }
    const int j = c0 / RP;
    // the block ends with this chunk, or the row's columns do (a short last block)
    if (((c0 + 32) % RP) == 0 || c0 + 32 >= R) {
      if (j <= jmax) prow[j] = m_run + lg2(s_run);
      m_run = -INFINITY;
      s_run = 0.f;
    }
  }
}

template <int RP>
__device__ __forceinline__ void epilogue_tile(uint32_t tacc, int rho, int n0, const Params& p,
                                              float* prow, int jmax, bool row_ok,
                                              bool need_mask, int half) {
  float m_run = -INFINITY, s_run = 0.f;
  constexpr int kHalfChunks = kBN / 64;  // 32-column chunks per half tile
#pragma unroll 1
  for (int ch = half * kHalfChunks; ch < (half + 1) * kHalfChunks; ++ch) {
    uint32_t v[32];
    tmem_ld32(tacc + ch * 32, v);
    tmem_ld_wait();
    const int c0 = n0 + ch * 32;
    if (row_ok && c0 < p.R && (c0 / RP) <= jmax) {
      epilogue_chunk<RP>(v, c0, rho, p.R, jmax, need_mask, p.causal != 0, p.scale_log2, prow,
                         m_run, s_run);
    }
  }
}

}  // namespace scoring
}  // namespace xattn
