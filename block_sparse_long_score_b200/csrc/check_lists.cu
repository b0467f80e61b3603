// check_lists.cu -- xattn_check_lists: validation of caller-provided block
// lists before xattn_sparse_attn.
//
// xattn_sparse_attn trusts its lists to have the layout xattn_select writes:
// a row's count is in [0, NB] and its first `count` entries are strictly
// ascending block indices in [0, NB). (Causal rows may end in blocks above the
// diagonal; the attention drops those.) A list that breaks this does not make
// the attention read outside its buffers -- counts are clamped to [0, NB], and
// a block index only moves a TMA coordinate, where out-of-range tiles read the
// fill value -- but it gives wrong rows: a repeated block is summed twice, and
// only a list's last entry is looked at for the diagonal and the short last
// block. This kernel reads every row once and counts the rows that break the
// layout; it writes nothing else.
#include <cuda_runtime.h>

#include "common.cuh"
#include "host.cuh"

namespace xattn {
namespace {

constexpr int kWarps = 8;

// One warp per row: the count, then the entries in chunks of 32 (each lane
// compares its entry with its left neighbour's).
__global__ void __launch_bounds__(kWarps * 32)
    check_lists_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ idx,
                       long long rows, int NB, int32_t* __restrict__ bad) {
  const int lane = threadIdx.x % 32;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + threadIdx.x / 32;
  if (row >= rows) return;
  const int n = counts[row];
  bool ok = n >= 0 && n <= NB;
  if (ok) {
    const int32_t* list = idx + row * NB;
    int prev = -1;  // the previous chunk's last entry
    for (int j0 = 0; j0 < n && ok; j0 += 32) {
      const int j = j0 + lane;
      const int v = j < n ? list[j] : 0;
      const int left = __shfl_up_sync(0xffffffffu, v, 1);
      bool good = true;
      if (j < n) {
        good = v >= 0 && v < NB;
        good = good && v > (lane == 0 ? prev : left);
      }
      ok = __all_sync(0xffffffffu, good);
      prev = __shfl_sync(0xffffffffu, v, 31);
    }
  }
  if (!ok && lane == 0) atomicAdd(bad, 1);
}

}  // namespace
}  // namespace xattn

using namespace xattn;
using namespace xattn::host;

extern "C" int xattn_check_lists(const int32_t* counts, const int32_t* idx,
                                 const xattn_shape* shape, int32_t* bad_rows, void* stream) {
  Dims D;
  int rc = check_shape(shape, &D);
  if (rc != XATTN_OK) return rc;
  if (!counts || !idx || !bad_rows) return XATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(bad_rows, 0, sizeof(int32_t), st) != cudaSuccess) return XATTN_ERR_CUDA;
  const long long rows = static_cast<long long>(D.batch) * D.hq * D.NB;
  const unsigned grid = static_cast<unsigned>((rows + kWarps - 1) / kWarps);
  check_lists_kernel<<<grid, kWarps * 32, 0, st>>>(counts, idx, rows, D.NB, bad_rows);
  return cuda_status(cudaGetLastError());
}
