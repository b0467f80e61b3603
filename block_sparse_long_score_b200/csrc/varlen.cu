// varlen.cu -- xattn_prefill_varlen: the prefill step over a batch of
// sequences of different lengths, packed one after another.
//
// Sequence i is a contiguous [heads, L_i, d] array in each of Q, K, V and O,
// starting right after sequence i-1. Each sequence runs as a batch-1 problem
// of its own length through the same two calls as a fixed-length batch
// (xattn_score_select, then xattn_sparse_attn), so a length that B does not
// divide ends in a shorter last block as usual. The calls are queued one
// sequence after another on the caller's stream and share one workspace,
// sized for the longest sequence.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "host.cuh"

namespace xattn {
namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Regions of the workspace for a batch-1 problem of length L.
struct VarlenLayout {
  size_t mask, counts, idx, score_ws, attn_ws, total;
};

int layout_for(const xattn_shape& one, VarlenLayout* Lo) {
  Dims D;
  int rc = host::check_shape(&one, &D);
  if (rc != XATTN_OK) return rc;
  const size_t rows = static_cast<size_t>(D.hq) * D.NB;
  Lo->mask = round_up(rows * ((D.NB + 31) / 32) * sizeof(uint32_t));
  Lo->counts = round_up(rows * sizeof(int32_t));
  Lo->idx = round_up(rows * D.NB * sizeof(int32_t));
  Lo->score_ws = round_up(xattn_score_workspace_bytes(&one));
  Lo->attn_ws = round_up(xattn_attn_workspace_bytes(&one));
  Lo->total = Lo->mask + Lo->counts + Lo->idx + Lo->score_ws + Lo->attn_ws;
  return XATTN_OK;
}

// Checks every length (0 is allowed and skipped; others must make a valid
// batch-1 shape) and returns the workspace layout of the longest one.
int check_lengths(const xattn_shape* shape, int nseq, const int32_t* seqlens,
                  VarlenLayout* Lo, int* lmax) {
  if (!shape || nseq < 1 || !seqlens) return XATTN_ERR_INVALID_ARG;
  long long total = 0;
  int longest = 0;
  for (int i = 0; i < nseq; ++i) {
    if (seqlens[i] < 0) return XATTN_ERR_INVALID_ARG;
    if (seqlens[i] == 0) continue;
    xattn_shape one = *shape;
    one.batch = 1;
    one.L = seqlens[i];
    Dims D;
    const int rc = host::check_shape(&one, &D);
    if (rc != XATTN_OK) return rc;
    total += seqlens[i];
    if (seqlens[i] > longest) longest = seqlens[i];
  }
  if (longest == 0) return XATTN_ERR_INVALID_ARG;  // nothing to compute
  // every element offset must fit the kernels' 32-bit row arithmetic
  if (total * shape->hq > (1ll << 31) - 1) return XATTN_ERR_UNSUPPORTED;
  xattn_shape one = *shape;
  one.batch = 1;
  one.L = longest;
  *lmax = longest;
  return layout_for(one, Lo);
}

}  // namespace
}  // namespace xattn

using namespace xattn;
using namespace xattn::host;

extern "C" {

size_t xattn_prefill_varlen_workspace_bytes(const xattn_shape* shape, int nseq,
                                            const int32_t* seqlens) {
  VarlenLayout Lo;
  int lmax = 0;
  if (check_lengths(shape, nseq, seqlens, &Lo, &lmax) != XATTN_OK) return 0;
  return Lo.total;
}

int xattn_prefill_varlen(const void* Q, const void* K, const void* V, const xattn_shape* shape,
                         int nseq, const int32_t* seqlens, const float* tau, void* O,
                         float* lse, void* ws, size_t ws_bytes, void* stream) {
  VarlenLayout Lo;
  int lmax = 0;
  int rc = check_lengths(shape, nseq, seqlens, &Lo, &lmax);
  if (rc != XATTN_OK) return rc;
  if (!Q || !K || !V || !O || !tau) return XATTN_ERR_INVALID_ARG;
  for (int h = 0; h < shape->hq; ++h)
    if (!(tau[h] > 0.0f && tau[h] <= 1.0f)) return XATTN_ERR_INVALID_ARG;  // NaN too
  if (!ws || ws_bytes < Lo.total || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return XATTN_ERR_WORKSPACE;

  char* p = static_cast<char*>(ws);
  uint32_t* mask = reinterpret_cast<uint32_t*>(p); p += Lo.mask;
  int32_t* counts = reinterpret_cast<int32_t*>(p); p += Lo.counts;
  int32_t* idx = reinterpret_cast<int32_t*>(p); p += Lo.idx;
  void* score_ws = p; p += Lo.score_ws;
  void* attn_ws = p;

  const size_t es = shape->dtype == XATTN_BF16 ? 2 : 4;
  const size_t qrow = static_cast<size_t>(shape->hq) * shape->d * es;   // one token, all heads
  const size_t kvrow = static_cast<size_t>(shape->hkv) * shape->d * es;
  const char* Qp = static_cast<const char*>(Q);
  const char* Kp = static_cast<const char*>(K);
  const char* Vp = static_cast<const char*>(V);
  char* Op = static_cast<char*>(O);
  size_t tok = 0;  // tokens of the sequences before the current one
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < nseq; ++i) {
    const int L = seqlens[i];
    if (L == 0) continue;
    xattn_shape one = *shape;
    one.batch = 1;
    one.L = L;
    rc = xattn_score_select(Qp + tok * qrow, Kp + tok * kvrow, &one, tau, nullptr, mask, counts,
                            idx, score_ws, Lo.score_ws, st);
    if (rc != XATTN_OK) return rc;
    rc = xattn_sparse_attn(Qp + tok * qrow, Kp + tok * kvrow, Vp + tok * kvrow, &one, counts,
                           idx, Op + tok * qrow,
                           lse ? lse + tok * static_cast<size_t>(shape->hq) : nullptr, attn_ws,
                           Lo.attn_ws, st);
    if (rc != XATTN_OK) return rc;
    tok += static_cast<size_t>(L);
  }
  return XATTN_OK;
}

}  // extern "C"
