// host.cuh -- host-side helpers of the C-ABI layer (argument checks, per-device
// state, TMA descriptors), shared by the entry-point files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace xattn {
namespace host {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  unsigned long long ctx_id = 0;  // context the addresses below belong to
  int* status = nullptr;          // device address of the status word
  int num_sms = 0;
};

// Process-unique ID of the current CUDA context (cuCtxGetId); 0 when the
// thread has no current context yet. Device addresses of module variables
// belong to one context: a cache keyed by this ID is rebuilt when the context
// changes (for example after cudaDeviceReset and a new primary context).
int current_context_id(unsigned long long* id);

// State of the current device, created on first use and rebuilt when the
// device's context changes. Returns an xattn_status.
int device_state(DeviceState** out);
// Checks a shape and fills the derived sizes. Returns an xattn_status.
int check_shape(const xattn_shape* sh, Dims* D);
bool aligned16(const void* p);
// xattn_score_select with the thresholds in HOST memory (checked on the host
// and passed to the kernels by value), for the whole-step calls that take
// tau from the host.
int score_select_host_tau(const void* Q, const void* K, const xattn_shape* shape,
                          const float* tau_host, float* probs, uint32_t* mask, int32_t* counts,
                          int32_t* idx, void* ws, size_t ws_bytes, void* stream);
// 2-D bf16 view [rows, 128] with 64 x 128 boxes and 128-byte swizzle.
int make_map_2d(CUtensorMap* m, const void* ptr, long long rows);
int cuda_status(cudaError_t e);

}  // namespace host
}  // namespace xattn
