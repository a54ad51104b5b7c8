// flexq_linear_static_scratch: the linear layer of flexq_linear for callers
// that cannot allocate device memory.
//
// When a linear layer's output grid is smaller than the GPU, flexq_linear
// splits K across CTAs and sums fp32 partial results in a caller-provided
// workspace.  Some callers have no way to provide one: a plug-in that a host
// framework calls with nothing but its input and output buffers while the
// framework's own pool owns the rest of device memory, or a latency-critical
// loop that must not pay for cudaMalloc/cudaFree (cudaFree waits for the whole
// device).  This entry point takes the same inputs and outputs and keeps the
// partial sums in a fixed array compiled into the library instead.
//
// Properties a user must know:
// * The array holds kStaticScratchBytes (8 MiB) of fp32 partial tiles; a shape
//   whose K-split scratch (flexq_linear_workspace) is larger is rejected with
//   FLEXQ_ERR_INVALID before anything is launched.  The 8 MiB are reserved
//   on a device from the first use of the library's device code there (with
//   lazy module loading, the first launch) until the process exits.
// * The first call on a device looks up the array's device address (with that
//   device current) and keeps it once the lookup succeeds; a failed lookup is
//   reported and retried by the next call.  Make that first call before any
//   stream capture begins.
// * All calls share the one array and it keeps the last call's contents; each
//   call clears the part it uses before accumulating.  Calls whose kernels
//   overlap on the GPU (other streams, other host threads) race on it and
//   produce wrong sums: serialise them.
// * Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library
//   routine.
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "flexq.h"
#include "kernels.h"

namespace flexq {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_ptr[kMaxDev];  // set once the lookup on that device succeeded
std::mutex g_scratch_mu;

// Device address of the static array on the current device.  In host code the
// name g_static_scratch is only a host-side stand-in, so the address must come
// from cudaGetSymbolAddress.  A successful lookup is kept for the device; a
// failed one (for example during a stream capture) is not, so a later call
// tries again.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();  // the failure is reported through the return value
      return e;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace flexq

using namespace flexq;

extern "C" flexq_status flexq_linear_static_scratch(const void* x_dev, int ldx, const void* w_dev, int w_bits,
                                                    int m, int n, int k, const void* bias_dev,
                                                    const void* residual_dev, int ld_res, int epilogue,
                                                    void* y_dev, int ldy, int force_splits, void* stream) {
  // The argument rules are those of flexq_linear; only the scratch differs.
  if (m < 0 || n <= 0 || k <= 0 || k % 64 != 0 || (w_bits != 4 && w_bits != 16) || force_splits < 0 ||
      force_splits > k / 64) {
    set_last_error("invalid shape, w_bits or force_splits");
    return FLEXQ_ERR_INVALID;
  }
  if (m == 0) return FLEXQ_OK;
  const size_t need = linear_workspace_bytes(m, n, k, w_bits, force_splits);
  if (need > kStaticScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "K-split partial sums need %zu bytes; the static scratch holds %zu", need,
             kStaticScratchBytes);
    set_last_error(msg);
    return FLEXQ_ERR_INVALID;
  }
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_on_current_device(&scratch);
    if (e != cudaSuccess || scratch == nullptr) {
      char msg[200];
      snprintf(msg, sizeof(msg), "static scratch address lookup failed: %s", cudaGetErrorString(e));
      set_last_error(msg);
      return FLEXQ_ERR_CUDA;
    }
  }
  return flexq_linear(x_dev, ldx, w_dev, w_bits, m, n, k, bias_dev, residual_dev, ld_res, epilogue, y_dev, ldy,
                      scratch, need > 0 ? kStaticScratchBytes : 0, force_splits, stream);
}
