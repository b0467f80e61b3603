// prefill_host.cu -- xattn_prefill_host: the whole prefill step (score and
// select, then block-sparse attention) on Q, K, V held in host memory, with
// the host<->device copies overlapped with the compute.
//
// Every step of the method is independent across KV-head groups: a query head
// reads only its own KV head (grouped-query attention), scoring and selection
// work per head, and the attention units are (head, query block) pairs. So the
// layer is cut into chunks of whole KV heads (with their query heads) per
// batch entry. Each chunk is a contiguous range of Q, K, V and O in the
// [batch, heads, L, d] layout, so it moves with one copy per tensor.
//
// Three streams carry the chunks through a two-slot ring of device buffers:
//   copy-in  stream:  Q, K, V of chunk c        -> slot c % 2
//   compute  stream:  xattn_score_select + xattn_sparse_attn on slot c % 2
//                     (the caller's stream)
//   copy-out stream:  O (and lse) of slot c % 2 -> host
// Events order each slot's reuse: the copy-in of chunk c + 2 waits for the
// compute of chunk c to finish reading it, and the compute of chunk c + 2 waits
// for the copy-out of chunk c before it overwrites O. The copy-in and copy-out
// streams first wait for the caller's stream, and at the end the caller's
// stream waits for both, so the whole call is ordered on the caller's stream
// like any other call of the library.
//
// The selection's and the attention's scratch (mask, counts, idx, the scoring
// partials, the work order) is used on the compute stream alone, one chunk
// after another, so it needs one copy only.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "host.cuh"

namespace xattn {
namespace {

constexpr int kSlots = 2;
constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Byte sizes of the regions of the workspace for chunks of `ck` KV heads.
struct Layout {
  size_t q, kv, o, lse;          // per slot
  size_t mask, counts, idx;      // single copy
  size_t score_ws, attn_ws;      // single copy
  size_t total;
};

xattn_shape chunk_shape(const xattn_shape& s, int ck) {
  xattn_shape c = s;
  c.batch = 1;
  c.hkv = ck;
  c.hq = ck * (s.hq / s.hkv);
  return c;
}

size_t elem_bytes(int dtype) { return dtype == XATTN_BF16 ? 2 : 4; }

int layout_of(const xattn_shape& s, const Dims& D, int ck, Layout* Lo) {
  const xattn_shape cs = chunk_shape(s, ck);
  const size_t es = elem_bytes(D.dtype);
  const size_t hq_c = static_cast<size_t>(cs.hq);
  const size_t row = static_cast<size_t>(D.L) * D.d * es;
  Lo->q = round_up(hq_c * row);
  Lo->kv = round_up(static_cast<size_t>(ck) * row);
  Lo->o = Lo->q;
  Lo->lse = round_up(hq_c * D.L * sizeof(float));
  const size_t words = (static_cast<size_t>(D.NB) + 31) / 32;
  Lo->mask = round_up(hq_c * D.NB * words * sizeof(uint32_t));
  Lo->counts = round_up(hq_c * D.NB * sizeof(int32_t));
  Lo->idx = round_up(hq_c * D.NB * D.NB * sizeof(int32_t));
  Lo->score_ws = round_up(xattn_score_workspace_bytes(&cs));
  Lo->attn_ws = round_up(xattn_attn_workspace_bytes(&cs));
  if (Lo->score_ws == 0 || Lo->attn_ws == 0) return XATTN_ERR_INVALID_ARG;
  Lo->total = kSlots * (Lo->q + 2 * Lo->kv + Lo->o + Lo->lse) + Lo->mask + Lo->counts +
              Lo->idx + Lo->score_ws + Lo->attn_ws;
  return XATTN_OK;
}

// Resolves kv_heads_per_chunk (0 = one KV head per chunk) and checks it.
int chunk_heads(const Dims& D, int kv_heads_per_chunk, int* ck) {
  if (kv_heads_per_chunk < 0 || kv_heads_per_chunk > D.hkv) return XATTN_ERR_INVALID_ARG;
  *ck = kv_heads_per_chunk == 0 ? 1 : kv_heads_per_chunk;
  return XATTN_OK;
}

// The CUDA objects one call owns. The destructor releases them; CUDA defers the
// release of a stream or event until the work queued on it has finished.
struct CallObjects {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, in_end = nullptr, out_end = nullptr;
  cudaEvent_t in_done[kSlots] = {}, comp_done[kSlots] = {}, out_done[kSlots] = {};

  int create() {
    if (cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) != cudaSuccess)
      return XATTN_ERR_CUDA;
    cudaEvent_t* all[] = {&start,        &in_end,       &out_end,     &in_done[0],
                          &in_done[1],   &comp_done[0], &comp_done[1], &out_done[0],
                          &out_done[1]};
    for (cudaEvent_t* e : all)
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess)
        return XATTN_ERR_CUDA;
    return XATTN_OK;
  }
  ~CallObjects() {
    cudaEvent_t all[] = {start,        in_end,       out_end,     in_done[0], in_done[1],
                         comp_done[0], comp_done[1], out_done[0], out_done[1]};
    for (cudaEvent_t e : all)
      if (e) cudaEventDestroy(e);
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
  }
};

}  // namespace
}  // namespace xattn

using namespace xattn;
using namespace xattn::host;

extern "C" {

size_t xattn_prefill_host_workspace_bytes(const xattn_shape* shape, int kv_heads_per_chunk) {
  Dims D;
  if (check_shape(shape, &D) != XATTN_OK) return 0;
  int ck = 0;
  if (chunk_heads(D, kv_heads_per_chunk, &ck) != XATTN_OK) return 0;
  Layout Lo;
  if (layout_of(*shape, D, ck, &Lo) != XATTN_OK) return 0;
  return Lo.total;
}

int xattn_prefill_host(const void* Q, const void* K, const void* V, const xattn_shape* shape,
                       const float* tau, void* O, float* lse, int kv_heads_per_chunk, void* ws,
                       size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!Q || !K || !V || !O || !tau) return XATTN_ERR_INVALID_ARG;
  for (int h = 0; h < D.hq; ++h)
    if (!(tau[h] > 0.0f && tau[h] <= 1.0f)) return XATTN_ERR_INVALID_ARG;  // NaN too
  int ck = 0;
  if ((rc = chunk_heads(D, kv_heads_per_chunk, &ck)) != XATTN_OK) return rc;
  Layout Lo;
  if ((rc = layout_of(*shape, D, ck, &Lo)) != XATTN_OK) return rc;
  if (!ws || ws_bytes < Lo.total || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0)
    return XATTN_ERR_WORKSPACE;

  // carve the workspace
  char* p = static_cast<char*>(ws);
  char *q_d[kSlots], *k_d[kSlots], *v_d[kSlots], *o_d[kSlots];
  float* lse_d[kSlots];
  for (int s = 0; s < kSlots; ++s) {
    q_d[s] = p; p += Lo.q;
    k_d[s] = p; p += Lo.kv;
    v_d[s] = p; p += Lo.kv;
    o_d[s] = p; p += Lo.o;
    lse_d[s] = reinterpret_cast<float*>(p); p += Lo.lse;
  }
  uint32_t* mask = reinterpret_cast<uint32_t*>(p); p += Lo.mask;
  int32_t* counts = reinterpret_cast<int32_t*>(p); p += Lo.counts;
  int32_t* idx = reinterpret_cast<int32_t*>(p); p += Lo.idx;
  void* score_ws = p; p += Lo.score_ws;
  void* attn_ws = p;

  CallObjects co;
  if ((rc = co.create()) != XATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaEventRecord(co.start, st) != cudaSuccess ||
      cudaStreamWaitEvent(co.in, co.start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(co.out, co.start, 0) != cudaSuccess)
    return XATTN_ERR_CUDA;

  const size_t es = elem_bytes(D.dtype);
  const size_t row = static_cast<size_t>(D.L) * D.d * es;  // one head of one tensor
  const int G = D.group;
  const int groups = (D.hkv + ck - 1) / ck;
  const int chunks = D.batch * groups;
  const char* Qh = static_cast<const char*>(Q);
  const char* Kh = static_cast<const char*>(K);
  const char* Vh = static_cast<const char*>(V);
  char* Oh = static_cast<char*>(O);

  // A failure part-way still joins the side streams back to the caller's
  // stream below, so nothing the call queued is left unordered.
  for (int c = 0; c < chunks && rc == XATTN_OK; ++c) {
    const int slot = c % kSlots;
    const int b = c / groups;
    const int kv0 = (c % groups) * ck;
    const int nkv = D.hkv - kv0 < ck ? D.hkv - kv0 : ck;
    const int hq0 = kv0 * G;
    const size_t qoff = (static_cast<size_t>(b) * D.hq + hq0) * row;
    const size_t kvoff = (static_cast<size_t>(b) * D.hkv + kv0) * row;
    const size_t qbytes = static_cast<size_t>(nkv) * G * row;
    const size_t kvbytes = static_cast<size_t>(nkv) * row;
    const xattn_shape cs = chunk_shape(*shape, nkv);

    // copy in
    cudaError_t e = cudaSuccess;
    if (c >= kSlots) e = cudaStreamWaitEvent(co.in, co.comp_done[slot], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(q_d[slot], Qh + qoff, qbytes, cudaMemcpyDefault, co.in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(k_d[slot], Kh + kvoff, kvbytes, cudaMemcpyDefault, co.in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(v_d[slot], Vh + kvoff, kvbytes, cudaMemcpyDefault, co.in);
    if (e == cudaSuccess) e = cudaEventRecord(co.in_done[slot], co.in);
    // compute
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, co.in_done[slot], 0);
    if (e == cudaSuccess && c >= kSlots) e = cudaStreamWaitEvent(st, co.out_done[slot], 0);
    if (e != cudaSuccess) {
      rc = XATTN_ERR_CUDA;
      break;
    }
    rc = score_select_host_tau(q_d[slot], k_d[slot], &cs, tau + hq0, nullptr, mask, counts,
                               idx, score_ws, Lo.score_ws, st);
    if (rc != XATTN_OK) break;
    rc = xattn_sparse_attn(q_d[slot], k_d[slot], v_d[slot], &cs, counts, idx, o_d[slot],
                           lse ? lse_d[slot] : nullptr, attn_ws, Lo.attn_ws, st);
    if (rc != XATTN_OK) break;
    e = cudaEventRecord(co.comp_done[slot], st);
    // copy out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(co.out, co.comp_done[slot], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(Oh + qoff, o_d[slot], qbytes, cudaMemcpyDefault, co.out);
    if (e == cudaSuccess && lse) {
      const size_t loff = (static_cast<size_t>(b) * D.hq + hq0) * D.L;
      e = cudaMemcpyAsync(lse + loff, lse_d[slot],
                          static_cast<size_t>(nkv) * G * D.L * sizeof(float),
                          cudaMemcpyDefault, co.out);
    }
    if (e == cudaSuccess) e = cudaEventRecord(co.out_done[slot], co.out);
    if (e != cudaSuccess) rc = XATTN_ERR_CUDA;
  }

  // join the side streams back into the caller's stream
  bool joined = cudaEventRecord(co.in_end, co.in) == cudaSuccess &&
                cudaEventRecord(co.out_end, co.out) == cudaSuccess &&
                cudaStreamWaitEvent(st, co.in_end, 0) == cudaSuccess &&
                cudaStreamWaitEvent(st, co.out_end, 0) == cudaSuccess;
  if (!joined && rc == XATTN_OK) rc = XATTN_ERR_CUDA;
  return rc;
}

}  // extern "C"
