// pft_build_no_ws: the PFT build for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory for pft_build: a process
// whose device memory is carved up entirely by another pool at start-up, or a
// fixed C interface that hands this library only its input and output
// pointers and has nowhere to size or pass a workspace.  This entry point
// serves them by using a scratch array that lives in the library itself: a
// file-scope __device__ array of PFMOE_PFT_NO_WS_SCRATCH_BYTES bytes, which
// every GPU that loads the library holds until the process exits.
//
// The array's name in host code is only a host-side stand-in, not a device
// address, so the device address is looked up with cudaGetSymbolAddress once
// per device (with that device current) on the first call made on it, cached,
// and handed to the kernels.  That first call should therefore come before
// any stream capture (a first call on a capturing stream is refused).  The
// cached address belongs to the device's current context: after
// cudaDeviceReset the process must not call this entry point on that device
// again.  Nothing here calls cudaMalloc, cudaFree or any routine
// that allocates.
//
// Every call on a device shares the one array and finds in it whatever the
// last call left there.  The PFT kernels write every scratch word they read,
// so nothing needs clearing first; calls whose work overlaps on the GPU (for
// example on two streams at once) race on the array and must be ordered by
// the caller.
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace pfmoe {
namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_pft_scratch[PFMOE_PFT_NO_WS_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_pft_scratch on the current device (looked up once per device).  The
// lookup may load the library's module on the device, which a stream under capture does not
// allow, so a first call on a capturing stream is refused with a clear message instead.
int scratch_address(cudaStream_t stream, void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PFMOE_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(PFMOE_ERR_UNSUPPORTED, "pft_build_no_ws supports device ordinals below 64");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cs);
    if (e != cudaSuccess) return fail(PFMOE_ERR_CUDA, std::string("cudaStreamIsCapturing: ") + cudaGetErrorString(e));
    if (cs != cudaStreamCaptureStatusNone)
      return fail(PFMOE_ERR_UNSUPPORTED,
                  "pft_build_no_ws: the first call on a device looks up the built-in scratch array and cannot run "
                  "during stream capture; make one call on this device before capturing");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pft_scratch);
    if (e != cudaSuccess || !p)
      return fail(PFMOE_ERR_CUDA, std::string("cudaGetSymbolAddress(pft scratch): ") + cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PFMOE_OK;
}

}  // namespace
}  // namespace pfmoe

extern "C" int pft_build_no_ws(const int32_t* topk_ids, const float* topk_w, int T, int E, int k,
                               int32_t* tokens_per_expert, int32_t* expert_offsets, int32_t* token_ids,
                               int32_t* expert_ids, float* combine_weights, int32_t* pos, int32_t* tile_offsets,
                               int32_t* err, void* stream) {
  using namespace pfmoe;
  set_error("");
  if (T < 0 || E <= 0 || k <= 0) return fail(PFMOE_ERR_ARG, "pft_build_no_ws: need T >= 0, E > 0, k > 0");
  const size_t need = pft_build_workspace_size(T, E, k);
  if (need > PFMOE_PFT_NO_WS_SCRATCH_BYTES)
    return fail(PFMOE_ERR_UNSUPPORTED,
                "pft_build_no_ws: this shape needs " + std::to_string(need) + " bytes of scratch but the built-in " +
                    "array holds " + std::to_string(PFMOE_PFT_NO_WS_SCRATCH_BYTES) +
                    " bytes; use pft_build with a caller workspace");
  void* scratch = nullptr;
  PFMOE_TRY(scratch_address(static_cast<cudaStream_t>(stream), &scratch));
  return pft_build(topk_ids, topk_w, T, E, k, tokens_per_expert, expert_offsets, token_ids, expert_ids,
                   combine_weights, pos, tile_offsets, scratch, PFMOE_PFT_NO_WS_SCRATCH_BYTES, err, stream);
}
