// noalloc.cu -- xattn_sparse_attn_noalloc: block-sparse attention for callers
// that cannot allocate device memory.
//
// xattn_sparse_attn needs a small workspace for its work order (one 64-bit
// entry per work unit). Some callers have no way to provide it: a host program that
// has handed all device memory to another allocator, or a serving loop that may
// not allocate once it is running (cudaMalloc can synchronise the device and
// can fail under memory pressure). This entry point keeps that order list in a
// file-scope __device__ array instead, so it allocates nothing.
//
// The array holds XATTN_NOALLOC_MAX_UNITS entries (2 MiB). Every GPU that loads
// the library keeps it until the process exits. All calls on a device share it
// and it keeps the last call's contents; the schedule kernel rewrites every
// entry a call reads, so nothing needs clearing. Calls whose kernels overlap on
// the GPU (different streams, no ordering between them) race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "host.cuh"

namespace xattn {
namespace {

// Work-order scratch of xattn_sparse_attn_noalloc (device memory of the module).
static __device__ __align__(256) unsigned long long g_noalloc_order[XATTN_NOALLOC_MAX_UNITS];

std::mutex g_scratch_mu;
unsigned long long* g_scratch_ptr[host::kMaxDevices] = {};
unsigned long long g_scratch_ctx[host::kMaxDevices] = {};  // context of each cached address

// Device address of g_noalloc_order on the current device. In host code the
// symbol itself is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device and context, and cached. A new
// context on the device (after cudaDeviceReset, say) holds the array at a new
// address, so the cache is keyed by the context's process-unique ID.
int scratch_address(unsigned long long** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= host::kMaxDevices)
    return XATTN_ERR_CUDA;
  unsigned long long ctx = 0;
  int rc = host::current_context_id(&ctx);
  if (rc != XATTN_OK) return rc;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    g_scratch_ptr[dev] = nullptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_order) != cudaSuccess || p == nullptr)
      return XATTN_ERR_CUDA;
    if ((rc = host::current_context_id(&ctx)) != XATTN_OK || ctx == 0) return XATTN_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<unsigned long long*>(p);
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return XATTN_OK;
}

}  // namespace
}  // namespace xattn

using namespace xattn;
using namespace xattn::host;

extern "C" int xattn_sparse_attn_noalloc(const void* Q, const void* K, const void* V,
                                         const xattn_shape* shape, const int32_t* counts,
                                         const int32_t* idx, void* O, float* lse,
                                         void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!Q || !K || !V || !counts || !idx || !O) return XATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D.dtype != XATTN_BF16) {
    // the fp32 kernel maps rows to warps directly and needs no scratch, so
    // the unit limit does not apply to it
    return cuda_status(launch_attn_simt(D, static_cast<const float*>(Q),
                                        static_cast<const float*>(K),
                                        static_cast<const float*>(V), counts, idx,
                                        static_cast<float*>(O), lse, st));
  }
  const long long units = static_cast<long long>(D.batch) * D.hq * D.NB;
  if (units > XATTN_NOALLOC_MAX_UNITS) return XATTN_ERR_WORKSPACE;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return XATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != XATTN_OK) return rc;
  unsigned long long* order = nullptr;
  if ((rc = scratch_address(&order)) != XATTN_OK) return rc;
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
