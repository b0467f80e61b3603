// varlen.cu -- xattn_prefill_varlen: the prefill step over a batch of
// sequences of different lengths, packed one after another.
//
// Sequence i is a contiguous [heads, L_i, d] array in each of Q, K, V and O,
// starting right after sequence i-1. Each sequence runs as a batch-1 problem
// of its own length through the same two calls as a fixed-length batch
// (xattn_score_select, then xattn_sparse_attn), so a length that B does not
// divide ends in a shorter last block as usual.
//
// A short sequence's kernels fill only part of the GPU (its persistent grids
// are sized by its own tiles and units), so the sequences are dealt over up
// to four lanes that run concurrently: lane 0 is the caller's stream, the
// others are streams the call creates, forks off the caller's stream with an
// event and joins back the same way. Each lane has its own scratch, sized for
// the longest sequence; within a lane the sequences run one after another.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "host.cuh"

namespace xattn {
namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxLanes = 4;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Regions of one lane's scratch for a batch-1 problem of length L.
struct VarlenLayout {
  size_t mask, counts, idx, score_ws, attn_ws, lane;  // lane = one lane's bytes
  int lanes;                                          // concurrent lanes
  size_t total;                                       // lanes * lane
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
  Lo->lane = Lo->mask + Lo->counts + Lo->idx + Lo->score_ws + Lo->attn_ws;
  return XATTN_OK;
}

// Checks every length (0 is allowed and skipped; others must make a valid
// batch-1 shape) and returns the workspace layout of the longest one.
int check_lengths(const xattn_shape* shape, int nseq, const int32_t* seqlens,
                  VarlenLayout* Lo, int* lmax) {
  if (!shape || nseq < 1 || !seqlens) return XATTN_ERR_INVALID_ARG;
  long long total = 0;
  int longest = 0, nonempty = 0;
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
    ++nonempty;
    if (seqlens[i] > longest) longest = seqlens[i];
  }
  if (longest == 0) return XATTN_ERR_INVALID_ARG;  // nothing to compute
  // every element offset must fit the kernels' 32-bit row arithmetic
  if (total * shape->hq > (1ll << 31) - 1) return XATTN_ERR_UNSUPPORTED;
  xattn_shape one = *shape;
  one.batch = 1;
  one.L = longest;
  *lmax = longest;
  const int rc = layout_for(one, Lo);
  if (rc != XATTN_OK) return rc;
  Lo->lanes = nonempty < kMaxLanes ? nonempty : kMaxLanes;
  Lo->total = Lo->lane * Lo->lanes;
  return XATTN_OK;
}

// The streams and events one call owns beyond the caller's stream; the
// destructor releases them (CUDA defers that until their work is done).
struct Lanes {
  cudaStream_t s[kMaxLanes] = {};
  cudaEvent_t start = nullptr, end[kMaxLanes] = {};
  int n = 0;
  int create(int lanes, cudaStream_t caller) {
    n = lanes;
    s[0] = caller;
    if (n <= 1) return XATTN_OK;
    if (cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(start, caller) != cudaSuccess)
      return XATTN_ERR_CUDA;
    for (int k = 1; k < n; ++k) {
      if (cudaStreamCreateWithFlags(&s[k], cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&end[k], cudaEventDisableTiming) != cudaSuccess ||
          cudaStreamWaitEvent(s[k], start, 0) != cudaSuccess)
        return XATTN_ERR_CUDA;
    }
    return XATTN_OK;
  }
  // the caller's stream waits for every other lane that was created
  int join() {
    int rc = XATTN_OK;
    for (int k = 1; k < n; ++k) {
      if (!s[k] || !end[k]) continue;
      if (cudaEventRecord(end[k], s[k]) != cudaSuccess ||
          cudaStreamWaitEvent(s[0], end[k], 0) != cudaSuccess)
        rc = XATTN_ERR_CUDA;
    }
    return rc;
  }
  ~Lanes() {
    if (start) cudaEventDestroy(start);
    for (int k = 1; k < kMaxLanes; ++k) {
      if (end[k]) cudaEventDestroy(end[k]);
      if (s[k]) cudaStreamDestroy(s[k]);
    }
  }
};

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

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Lanes lanes;
  if ((rc = lanes.create(Lo.lanes, st)) != XATTN_OK) {
    lanes.join();  // whatever was forked is joined back before returning
    return rc;
  }

  const size_t es = shape->dtype == XATTN_BF16 ? 2 : 4;
  const size_t qrow = static_cast<size_t>(shape->hq) * shape->d * es;   // one token, all heads
  const size_t kvrow = static_cast<size_t>(shape->hkv) * shape->d * es;
  const char* Qp = static_cast<const char*>(Q);
  const char* Kp = static_cast<const char*>(K);
  const char* Vp = static_cast<const char*>(V);
  char* Op = static_cast<char*>(O);
  size_t tok = 0;  // tokens of the sequences before the current one
  int j = 0;       // non-empty sequences so far
  for (int i = 0; i < nseq && rc == XATTN_OK; ++i) {
    const int L = seqlens[i];
    if (L == 0) continue;
    const int lane = j++ % Lo.lanes;
    char* p = static_cast<char*>(ws) + static_cast<size_t>(lane) * Lo.lane;
    uint32_t* mask = reinterpret_cast<uint32_t*>(p); p += Lo.mask;
    int32_t* counts = reinterpret_cast<int32_t*>(p); p += Lo.counts;
    int32_t* idx = reinterpret_cast<int32_t*>(p); p += Lo.idx;
    void* score_ws = p; p += Lo.score_ws;
    void* attn_ws = p;
    xattn_shape one = *shape;
    one.batch = 1;
    one.L = L;
    rc = score_select_host_tau(Qp + tok * qrow, Kp + tok * kvrow, &one, tau, nullptr, mask,
                               counts, idx, score_ws, Lo.score_ws, lanes.s[lane]);
    if (rc == XATTN_OK)
      rc = xattn_sparse_attn(Qp + tok * qrow, Kp + tok * kvrow, Vp + tok * kvrow, &one, counts,
                             idx, Op + tok * qrow,
                             lse ? lse + tok * static_cast<size_t>(shape->hq) : nullptr,
                             attn_ws, Lo.attn_ws, lanes.s[lane]);
    tok += static_cast<size_t>(L);
  }
  // join the lanes even after a failure, so nothing queued is left unordered
  const int jrc = lanes.join();
  return rc != XATTN_OK ? rc : jrc;
}

}  // extern "C"
