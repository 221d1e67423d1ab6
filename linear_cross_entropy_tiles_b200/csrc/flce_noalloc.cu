// flce_noalloc.cu -- flce_fused_noalloc: the fused forward + backward for
// callers that cannot hand the library a workspace.
//
// Some callers have no way to obtain scratch device memory: a plugin running
// inside a host program whose memory manager owns all of the GPU's memory and
// does not let guests allocate, or a caller from another language that can
// pass only the tensors it was given.  This entry point needs nothing from
// them beyond inputs and outputs: its scratch space is the file-scope array
// below, of a fixed size, which every GPU that loads this module keeps for the
// life of the process.  It calls no allocator of any kind.
//
// The array is shared by every call on a device and keeps whatever the last
// call left in it.  The fused computation writes every scratch byte it later
// reads within the same call (the status word, N_valid, the shifted labels,
// the LSE partials, the q / G chunk, the dX accumulator or split slabs, and
// the dW running sum, whose first row chunk stores without reading), so
// nothing has to be cleared between calls.  Two calls whose GPU work overlaps in time (different streams, or
// different host threads on the same device) race on the array and give
// wrong results; serialise them.
#include <mutex>

#include <cuda_runtime.h>

#include "flce.h"

namespace {

// The scratch array.  In host code this name is only a handle for the
// runtime, not a device address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[FLCE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_looked_up[kMaxDevices] = {};

// Device address of g_scratch in the current device's context.  It is looked
// up on every call (cheap once the module is loaded), so a context that was
// torn down and made again, e.g. by cudaDeviceReset, never sees a stale
// address.  The first look-up on a device may load the module; it is refused
// while `st` is being captured into a graph, where loading is not allowed.
flce_status_t scratch_address(cudaStream_t st, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FLCE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_looked_up[dev]) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return FLCE_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return FLCE_ERR_INVALID_ARG;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return FLCE_ERR_CUDA;
  g_looked_up[dev] = true;
  *out = p;
  return FLCE_OK;
}

}  // namespace

extern "C" FLCE_API flce_status_t flce_fused_noalloc(const flce_problem_t* p, const void* X,
                                                      const void* W, const int64_t* labels,
                                                      float dloss, float* loss, void* dX,
                                                      void* dW, struct CUstream_st* stream) {
  const size_t need = flce_workspace_size(p, FLCE_OP_FUSED);
  if (need == 0) return FLCE_ERR_INVALID_ARG;
  if (need > size_t(FLCE_NOALLOC_SCRATCH_BYTES)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  flce_status_t s = scratch_address(reinterpret_cast<cudaStream_t>(stream), &ws);
  if (s != FLCE_OK) return s;
  return flce_fused(p, X, W, labels, dloss, loss, dX, dW, ws, size_t(FLCE_NOALLOC_SCRATCH_BYTES),
                    stream);
}
