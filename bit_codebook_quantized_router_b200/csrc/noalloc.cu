// moe_q4_forward_noalloc: the MoE layer forward for callers that cannot
// allocate device memory.
//
// moe_q4_forward needs a caller-provided workspace.  Some callers have no way
// to get one: a serving loop that forbids cudaMalloc after start-up (it can
// synchronise the whole device and stall every stream), or code that only
// receives raw device pointers from another framework's allocator and has no
// allocator of its own.  For them this entry point runs the same kernels with
// the workspace placed in a fixed static device array of this library.
//
// The array (kNoAllocScratchBytes) is part of the library image: every GPU on
// which the library is loaded holds it until the process exits.  Host code
// cannot use the array's name as a device address (on the host it names a
// host-side stand-in), so the first call on each device looks the address up
// with cudaGetSymbolAddress while that device is current and caches it; make
// that first call outside any stream capture.  The cached address belongs to
// the device's primary context: after cudaDeviceReset on that device the
// library's module is loaded afresh at another address, so this entry point
// must not be used on a device that has been reset since its first call.
// All calls share the one
// array and it keeps the previous call's contents: the forward rewrites every
// word it reads (the status word is reset by the routing step itself), and
// two calls whose work overlaps on the GPU (different streams, or different
// host threads on one device) race on it and must be serialised by the caller.
#include <mutex>

#include "q4_api_internal.h"
#include "q4_common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set-up once per
// device), or nullptr on failure.
void* scratch_address(int dev) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" int moe_q4_forward_noalloc(const moe_q4_layer* layer, const void* x, const float* logits, int T,
                                      int top_k, void* out, float* out_f32, int32_t* status, void* stream) {
  const size_t need = moe_q4_forward_workspace(layer, T, top_k);
  if (need == 0) return MOE_Q4_EINVAL;
  if (need > kNoAllocScratchBytes) return MOE_Q4_ENOTSUP;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_Q4_ECUDA;
  void* ws = scratch_address(dev);
  if (!ws) return MOE_Q4_ECUDA;
  const int rc = q4_forward_in_workspace(layer, x, logits, T, top_k, out, out_f32, ws, kNoAllocScratchBytes,
                                         (cudaStream_t)stream);
  if (rc != MOE_Q4_OK || !status) return rc;
  // no tokens: nothing ran, so the status is OK (written, not left stale)
  if (T == 0)
    return cudaMemsetAsync(status, 0, sizeof(int32_t), (cudaStream_t)stream) == cudaSuccess ? MOE_Q4_OK
                                                                                            : MOE_Q4_ECUDA;
  // the status word is the workspace's first int32
  return cudaMemcpyAsync(status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, (cudaStream_t)stream) ==
                 cudaSuccess
             ? MOE_Q4_OK
             : MOE_Q4_ECUDA;
}
