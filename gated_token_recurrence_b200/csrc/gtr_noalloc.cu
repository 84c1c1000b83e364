// Allocation-free entry point: gtr_gla_fwd_noalloc.
//
// Who needs it: callers that are not allowed to call cudaMalloc.  Examples are
// a plugin running inside an inference engine that hands out device memory
// only at build time and forbids allocation while serving, and a real-time
// loop that must not pay cudaMalloc's implicit device synchronisation and
// unpredictable latency after start-up.  Such a caller cannot use
// gtr_gla_fwd (whose cached workspace grows with cudaMalloc) and may not be
// able to set aside a workspace for gtr_gla_fwd_ex either.
//
// How: the split path's scratch (chunk summaries, chunk-start states and chunk
// log-decays) lives in a fixed array compiled into this library,
// g_noalloc_scratch, of kNoallocScratchBytes.  Every GPU that loads the library
// holds that array until the process exits.  Host code cannot use the array's
// name as a device address (on the host it names a host-side stand-in), so the
// first call on each device, with that device current, asks the runtime for
// the array's device address once (cudaGetSymbolAddress) and caches it.
#include <mutex>

#include "gtr_common.cuh"
#include "gtr_internal.h"

namespace gtr {
namespace {

// 20 MiB: the split path needs the shared workspace prefix plus kSplitUnitBytes per
// (batch, head, chunk) unit, so B * heads * ceil(L/64) <= 634 units fit (for example
// the 1024^2 image with 8 heads: 512 units).
constexpr size_t kNoallocScratchBytes = size_t(20) << 20;
constexpr size_t kNoallocMaxUnits = (kNoallocScratchBytes - kWsPrefixBytes) / kSplitUnitBytes;
static_assert(kNoallocMaxUnits == 634, "the documented unit limit matches the array size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set up on first use).
gtr_status_t scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GTR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GTR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // reset the runtime's last-error state for the caller's next check
      return GTR_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return GTR_OK;
}

}  // namespace
}  // namespace gtr

extern "C" gtr_status_t gtr_gla_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const float* log_gamma, void* out, int B, int heads,
                                            int grid_H, int grid_W, int d_k, int d_v, int direction,
                                            int in_dtype, int out_dtype, gtr_stream_t stream) {
  // The same argument checks as every other entry point, then the size limit: all on
  // the host, before anything touches the device.
  gtr_status_t st = gtr::validate_call(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v,
                                       direction, in_dtype, out_dtype);
  if (st != GTR_OK) return st;
  const long long L = (long long)grid_H * grid_W;
  const long long units = (long long)B * heads * ((L + gtr::kChunk - 1) / gtr::kChunk);
  if (units > (long long)gtr::kNoallocMaxUnits) return GTR_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = gtr::scratch_address(&scratch);
  if (st != GTR_OK) return st;
  // Nothing in the scratch has to start at zero: the split path writes every
  // summary, state and log-decay it reads earlier in the same call, and it never
  // touches the header.  Calls that overlap on the GPU (other streams, or other
  // threads) share this one array and race; order them.
  return gtr_gla_fwd_ex(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v, direction,
                        in_dtype, out_dtype, GTR_PATH_SPLIT, scratch, gtr::kNoallocScratchBytes,
                        stream);
}
