// api.cu -- the C ABI declared in include/xattn.h: host-side argument checks,
// TMA descriptor set-up, and the kernel launch sequence of each call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "host.cuh"

namespace xattn {

// Per-device status word. Kernels that give up a bounded wait write
// kStatusTimeout here; xattn_get_device_status reads and clears it.
__device__ int g_status_word;

namespace host {

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
std::mutex g_ctx_mu;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

int current_context_id(unsigned long long* id) {
  *id = 0;
  {
    std::lock_guard<std::mutex> lock(g_ctx_mu);
    if (!g_ctx_get_current || !g_ctx_get_id) {
      void* f1 = nullptr;
      void* f2 = nullptr;
      cudaDriverEntryPointQueryResult q1, q2;
      if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) !=
              cudaSuccess ||
          q1 != cudaDriverEntryPointSuccess || !f1 ||
          cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
          q2 != cudaDriverEntryPointSuccess || !f2)
        return XATTN_ERR_CUDA;
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
  }
  CUcontext c = nullptr;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS) return XATTN_ERR_CUDA;
  if (c == nullptr) return XATTN_OK;
  return g_ctx_get_id(c, id) == CUDA_SUCCESS ? XATTN_OK : XATTN_ERR_CUDA;
}

// Looks up the device state of the current device, creating it on first use
// and again whenever the device's context has changed since.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return XATTN_ERR_CUDA;
  unsigned long long ctx = 0;
  int rc = current_context_id(&ctx);
  if (rc != XATTN_OK) return rc;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready || ctx == 0 || s.ctx_id != ctx) {
    s.ready = false;
    void* addr = nullptr;
    // also makes the device's primary context current if there was none
    if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return XATTN_ERR_CUDA;
    if ((rc = current_context_id(&ctx)) != XATTN_OK || ctx == 0) return XATTN_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return XATTN_ERR_CUDA;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return XATTN_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    s.status = static_cast<int*>(addr);
    s.num_sms = sms;
    s.ctx_id = ctx;
    s.ready = true;
  }
  *out = &s;
  return XATTN_OK;
}

// Checks a shape and fills the derived sizes. Returns an xattn_status.
int check_shape(const xattn_shape* sh, Dims* D) {
  if (!sh) return XATTN_ERR_INVALID_ARG;
  const xattn_shape& s = *sh;
  if (s.batch < 1 || s.hq < 1 || s.hkv < 1 || s.L < 1 || s.d < 1 || s.B < 1 || s.S < 1)
    return XATTN_ERR_INVALID_ARG;
  if (s.hq % s.hkv != 0) return XATTN_ERR_INVALID_ARG;
  // L need not be a multiple of B (the last block is then shorter), but it
  // must be a multiple of S so that every reshaped row and column is whole
  if (s.L % s.S != 0 || s.B % s.S != 0) return XATTN_ERR_INVALID_ARG;
  if (s.dtype != XATTN_F32 && s.dtype != XATTN_BF16) return XATTN_ERR_INVALID_ARG;
  if (s.hq > XATTN_MAX_HEADS) return XATTN_ERR_UNSUPPORTED;
  const int NB = (s.L + s.B - 1) / s.B;
  if (NB > XATTN_MAX_BLOCKS) return XATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(s.batch) * s.hq * s.L > (1ll << 31) - 1) return XATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(s.batch) * s.hq * NB > (1ll << 24)) return XATTN_ERR_UNSUPPORTED;
  if (s.dtype == XATTN_BF16) {
    if (s.d != 128 || s.B != 128) return XATTN_ERR_UNSUPPORTED;
  } else {
    if (!(s.d == 32 || s.d == 64 || s.d == 128) || s.B > 256) return XATTN_ERR_UNSUPPORTED;
    if (static_cast<long long>(s.S) * s.d * 4 > 48 * 1024) return XATTN_ERR_UNSUPPORTED;
  }
  D->batch = s.batch;
  D->hq = s.hq;
  D->hkv = s.hkv;
  D->L = s.L;
  D->d = s.d;
  D->B = s.B;
  D->S = s.S;
  D->causal = s.causal ? 1 : 0;
  D->dtype = s.dtype;
  D->NB = NB;
  D->r = s.B / s.S;
  D->R = s.L / s.S;
  D->tail = s.L - (NB - 1) * s.B;
  D->group = s.hq / s.hkv;
  return XATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 2-D bf16 view [rows, 128] with 64 x 128 boxes and 128-byte swizzle.
int make_map_2d(CUtensorMap* m, const void* ptr, long long rows) {
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? XATTN_OK : XATTN_ERR_CUDA;
}

// 4-D bf16 view [heads][rho][s][feature] = [bh][L/S][S][128] of a [bh, L, 128]
// tensor, with boxes of 64 features x 1 s x box_rows reshaped rows.
int make_map_reshaped(CUtensorMap* m, const void* ptr, int S, int R, int bh, int box_rows) {
  cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(R),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[3] = {128 * 2, static_cast<cuuint64_t>(S) * 128 * 2,
                           static_cast<cuuint64_t>(R) * S * 128 * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? XATTN_OK : XATTN_ERR_CUDA;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? XATTN_OK : XATTN_ERR_CUDA; }

}  // namespace host
}  // namespace xattn

using namespace xattn;
using namespace xattn::host;

extern "C" {

size_t xattn_score_workspace_bytes(const xattn_shape* shape) {
  Dims D;
  if (check_shape(shape, &D) != XATTN_OK) return 0;
  return static_cast<size_t>(D.batch) * D.hq * part_head_elems(D.NB, D.r, D.R, D.causal != 0) *
             sizeof(float) +
         256;
}

}  // extern "C"

namespace {

// Host checks shared by the scoring calls (Q, K, workspace). probs may be
// required or optional.
int check_score_args(const void* Q, const void* K, const xattn_shape* shape, void* ws,
                     size_t ws_bytes, Dims* D) {
  int rc = check_shape(shape, D);
  if (rc != XATTN_OK) return rc;
  if (!Q || !K) return XATTN_ERR_INVALID_ARG;
  const size_t need = xattn_score_workspace_bytes(shape);
  if (!ws || ws_bytes < need) return XATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 3u) != 0) return XATTN_ERR_INVALID_ARG;  // fp32 partials
  if (D->dtype == XATTN_BF16 && (!aligned16(Q) || !aligned16(K))) return XATTN_ERR_INVALID_ARG;
  return XATTN_OK;
}

// Launches the scoring GEMM (partial log-sum-exp into the workspace).
int score_partials(const void* Q, const void* K, const Dims& D, const PermArg& perm,
                   float* part, cudaStream_t st) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != XATTN_OK) return rc;
  if (D.dtype == XATTN_BF16) {
    CUtensorMap tq, tk;
    // a CTA pair loads 128 of a tile's 256 key rows per CTA, a lone CTA all 256
    const bool pair = D.S >= kScorePairMinS;
    if ((rc = make_map_reshaped(&tq, Q, D.S, D.R, D.batch * D.hq, 128)) != XATTN_OK) return rc;
    if ((rc = make_map_reshaped(&tk, K, D.S, D.R, D.batch * D.hkv, pair ? 128 : 256)) !=
        XATTN_OK)
      return rc;
    const cudaError_t e =
        pair ? launch_score_tc_pair(D, tq, tk, perm, part, ds->status, ds->num_sms, st)
             : launch_score_tc(D, tq, tk, perm, part, ds->status, ds->num_sms, st);
    if ((rc = cuda_status(e)) != XATTN_OK) return rc;
  } else {
    if ((rc = cuda_status(launch_score_simt(D, static_cast<const float*>(Q),
                                            static_cast<const float*>(K), perm, part, st))) !=
        XATTN_OK)
      return rc;
  }
  return XATTN_OK;
}

// Scoring with an explicit sampling pattern (already validated).
int score_impl(const void* Q, const void* K, const xattn_shape* shape, const PermArg& perm,
               float* probs, void* ws, size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_score_args(Q, K, shape, ws, ws_bytes, &D);
  if (rc != XATTN_OK) return rc;
  if (!probs) return XATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  if ((rc = score_partials(Q, K, D, perm, part, st)) != XATTN_OK) return rc;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != XATTN_OK) return rc;
  return cuda_status(launch_score_reduce(D, part, probs, ds->status, st));
}

// Per-head thresholds from a host array; INVALID_ARG unless each is in (0, 1].
int tau_arg(const float* tau, int hq, TauArg* ta) {
  std::memset(ta, 0, sizeof(*ta));
  for (int h = 0; h < hq; ++h) {
    const float t = tau[h];
    if (!(t > 0.0f && t <= 1.0f)) return XATTN_ERR_INVALID_ARG;  // also rejects NaN
    ta->v[h] = t;
  }
  return XATTN_OK;
}

// Per-head thresholds read by the kernels from a device array; each kernel
// checks its head's value and reports one outside (0, 1] in the status word.
void tau_dev_arg(const float* tau_dev, int* status, TauArg* ta) {
  std::memset(ta, 0, sizeof(*ta));
  ta->dev = tau_dev;
  ta->status = status;
}

// Scoring, then the fused reduce + find_blocks, with validated thresholds.
int score_select_impl(const void* Q, const void* K, const xattn_shape* shape, const TauArg& ta,
                      float* probs, uint32_t* mask, int32_t* counts, int32_t* idx, void* ws,
                      size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_score_args(Q, K, shape, ws, ws_bytes, &D);
  if (rc != XATTN_OK) return rc;
  if (!mask || !counts || !idx) return XATTN_ERR_INVALID_ARG;
  if (D.S > 256) return XATTN_ERR_UNSUPPORTED;  // S divides B <= 256 for every valid shape
  PermArg perm;  // the antidiagonal
  std::memset(&perm, 0, sizeof(perm));
  for (int i = 0; i < D.S; ++i) perm.q[i] = static_cast<uint8_t>(D.S - 1 - i);
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != XATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  if ((rc = score_partials(Q, K, D, perm, part, st)) != XATTN_OK) return rc;
  return cuda_status(launch_score_select(D, part, probs, ta, mask, counts, idx, ds->status,
                                         ds->num_sms, st));
}

// Fixed-budget selection (arguments already validated into `budget`).
int select_budget_impl(const float* probs, const BudgetArg& budget, const Dims& D,
                       uint32_t* mask, int32_t* counts, int32_t* idx, void* stream) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != XATTN_OK) return rc;
  return cuda_status(launch_select_budget(D, probs, budget, mask, counts, idx,
                                          static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int xattn_score(const void* Q, const void* K, const xattn_shape* shape, float* probs, void* ws,
                size_t ws_bytes, void* stream) {
  Dims D;
  const int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (D.S > 256) return XATTN_ERR_UNSUPPORTED;  // S divides B <= 256 for every valid shape
  PermArg perm;  // the antidiagonal: chunk i reads query sub-row S-1-i
  std::memset(&perm, 0, sizeof(perm));
  for (int i = 0; i < D.S; ++i) perm.q[i] = static_cast<uint8_t>(D.S - 1 - i);
  return score_impl(Q, K, shape, perm, probs, ws, ws_bytes, stream);
}

int xattn_score_partials(const void* Q, const void* K, const xattn_shape* shape, void* ws,
                         size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_score_args(Q, K, shape, ws, ws_bytes, &D);
  if (rc != XATTN_OK) return rc;
  if (D.S > 256) return XATTN_ERR_UNSUPPORTED;  // S divides B <= 256 for every valid shape
  PermArg perm;  // the antidiagonal
  std::memset(&perm, 0, sizeof(perm));
  for (int i = 0; i < D.S; ++i) perm.q[i] = static_cast<uint8_t>(D.S - 1 - i);
  return score_partials(Q, K, D, perm, static_cast<float*>(ws),
                        static_cast<cudaStream_t>(stream));
}

int xattn_score_pattern(const void* Q, const void* K, const xattn_shape* shape,
                        const int32_t* perm, float* probs, void* ws, size_t ws_bytes,
                        void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!perm) return XATTN_ERR_INVALID_ARG;
  if (D.S > 256) return XATTN_ERR_UNSUPPORTED;
  PermArg pa;
  std::memset(&pa, 0, sizeof(pa));
  bool seen[256] = {};
  for (int i = 0; i < D.S; ++i) {
    const int32_t v = perm[i];
    if (v < 0 || v >= D.S || seen[v]) return XATTN_ERR_INVALID_ARG;
    seen[v] = true;
    pa.q[i] = static_cast<uint8_t>(v);
  }
  return score_impl(Q, K, shape, pa, probs, ws, ws_bytes, stream);
}

int xattn_select(const float* probs, const float* tau, const xattn_shape* shape, uint32_t* mask,
                 int32_t* counts, int32_t* idx, void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!probs || !tau || !mask || !counts || !idx) return XATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != XATTN_OK) return rc;
  TauArg ta;
  tau_dev_arg(tau, ds->status, &ta);
  return cuda_status(
      launch_select(D, probs, ta, mask, counts, idx, ds->num_sms, static_cast<cudaStream_t>(stream)));
}

int xattn_score_select(const void* Q, const void* K, const xattn_shape* shape, const float* tau,
                       float* probs, uint32_t* mask, int32_t* counts, int32_t* idx, void* ws,
                       size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_score_args(Q, K, shape, ws, ws_bytes, &D);  // every host check first
  if (rc != XATTN_OK) return rc;
  if (!tau || !mask || !counts || !idx) return XATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != XATTN_OK) return rc;
  TauArg ta;
  tau_dev_arg(tau, ds->status, &ta);
  return score_select_impl(Q, K, shape, ta, probs, mask, counts, idx, ws, ws_bytes, stream);
}

}  // extern "C"

namespace xattn {
namespace host {

int score_select_host_tau(const void* Q, const void* K, const xattn_shape* shape,
                          const float* tau_host, float* probs, uint32_t* mask, int32_t* counts,
                          int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  if (!tau_host || !shape) return XATTN_ERR_INVALID_ARG;
  if (shape->hq < 1 || shape->hq > XATTN_MAX_HEADS) return XATTN_ERR_INVALID_ARG;
  TauArg ta;
  const int rc = tau_arg(tau_host, shape->hq, &ta);
  if (rc != XATTN_OK) return rc;
  return score_select_impl(Q, K, shape, ta, probs, mask, counts, idx, ws, ws_bytes, stream);
}

}  // namespace host
}  // namespace xattn

extern "C" {

int xattn_select_topk(const float* probs, const int32_t* k, const xattn_shape* shape,
                      uint32_t* mask, int32_t* counts, int32_t* idx, void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!probs || !k || !mask || !counts || !idx) return XATTN_ERR_INVALID_ARG;
  BudgetArg ba;
  std::memset(&ba, 0, sizeof(ba));
  for (int h = 0; h < D.hq; ++h) {
    if (k[h] < 1) return XATTN_ERR_INVALID_ARG;
    ba.k[h] = k[h];
  }
  ba.use_ratio = 0;
  return select_budget_impl(probs, ba, D, mask, counts, idx, stream);
}

int xattn_select_topratio(const float* probs, const float* ratio, const xattn_shape* shape,
                          uint32_t* mask, int32_t* counts, int32_t* idx, void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!probs || !ratio || !mask || !counts || !idx) return XATTN_ERR_INVALID_ARG;
  BudgetArg ba;
  std::memset(&ba, 0, sizeof(ba));
  for (int h = 0; h < D.hq; ++h) {
    const float r = ratio[h];
    if (!(r > 0.0f && r <= 1.0f)) return XATTN_ERR_INVALID_ARG;  // also rejects NaN
    ba.ratio[h] = r;
  }
  ba.use_ratio = 1;
  return select_budget_impl(probs, ba, D, mask, counts, idx, stream);
}

size_t xattn_attn_workspace_bytes(const xattn_shape* shape) {
  Dims D;
  if (check_shape(shape, &D) != XATTN_OK) return 0;
  return sizeof(unsigned long long) * (static_cast<size_t>(D.batch) * D.hq * D.NB + 32);
}

int xattn_sparse_attn(const void* Q, const void* K, const void* V, const xattn_shape* shape,
                      const int32_t* counts, const int32_t* idx, void* O, float* lse, void* ws,
                      size_t ws_bytes, void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!Q || !K || !V || !counts || !idx || !O) return XATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < xattn_attn_workspace_bytes(shape)) return XATTN_ERR_WORKSPACE;
  if (D.dtype == XATTN_BF16 &&
      (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)))
    return XATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != XATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D.dtype == XATTN_BF16) {
    unsigned long long* order = static_cast<unsigned long long*>(ws);
    if ((rc = cuda_status(launch_sched(D, counts, idx, order, ds->num_sms, st))) != XATTN_OK) return rc;
    CUtensorMap tq, tk, tv;
    if ((rc = make_map_2d(&tq, Q, static_cast<long long>(D.batch) * D.hq * D.L)) != XATTN_OK)
      return rc;
    if ((rc = make_map_2d(&tk, K, static_cast<long long>(D.batch) * D.hkv * D.L)) != XATTN_OK)
      return rc;
    if ((rc = make_map_2d(&tv, V, static_cast<long long>(D.batch) * D.hkv * D.L)) != XATTN_OK)
      return rc;
    return cuda_status(launch_attn_tc(D, tq, tk, tv, counts, idx, order, O, lse, ds->status,
                                      ds->num_sms, st));
  }
  return cuda_status(launch_attn_simt(D, static_cast<const float*>(Q),
                                      static_cast<const float*>(K),
                                      static_cast<const float*>(V), counts, idx,
                                      static_cast<float*>(O), lse, st));
}

int xattn_selftest_timeout(void* stream) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != XATTN_OK) return rc;
  return cuda_status(launch_selftest_timeout(ds->status, static_cast<cudaStream_t>(stream)));
}

int xattn_get_device_status(void* stream) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != XATTN_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return XATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ds->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return XATTN_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(ds->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return XATTN_ERR_CUDA;
  }
  if (v == kStatusTimeout) return XATTN_ERR_TIMEOUT;
  if (v == kStatusBadTau) return XATTN_ERR_INVALID_ARG;
  return XATTN_OK;
}

const char* xattn_strerror(int status) {
  switch (status) {
    case XATTN_OK: return "ok";
    case XATTN_ERR_INVALID_ARG: return "invalid argument";
    case XATTN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case XATTN_ERR_CUDA: return "CUDA runtime error";
    case XATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case XATTN_ERR_TIMEOUT: return "a kernel wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
