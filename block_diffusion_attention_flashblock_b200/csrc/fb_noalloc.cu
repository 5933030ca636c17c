// fb_attn_outblock_noalloc: the dense block-external attention of
// fb_attn_outblock for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a scratch buffer at
// call time: code that runs under a host framework which has already claimed
// the whole device pool for its own allocator, plug-ins that may only use
// memory their host gives them, or services that forbid allocation once they
// are serving, so that a request can never fail for lack of memory. For them
// the split-KV partial results, the only scratch this call needs, live in a
// fixed array inside the library instead of in caller memory.
//
// The array is a file-scope __device__ variable of FB_NOALLOC_SCRATCH_BYTES.
// Every GPU on which the library is loaded holds it until the process exits.
// Host code cannot use the array's name as a device address, so the first
// call on each device looks the address up with cudaGetSymbolAddress, with
// that device current, and caches it.  That first call on a device should come
// before any stream capture on it.  Every call shares the one array and it
// keeps the last call's contents; this call fully writes every partial it later
// reads, so nothing needs clearing, but two calls whose work overlaps on the
// GPU (different streams, no ordering between them) race on the array.
#include <math.h>
#include <string.h>

#include <mutex>

#include "fb_internal.cuh"

namespace fb {
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[FB_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (set up once).
fb_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FB_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return FB_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FB_ECUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return FB_OK;
}

}  // namespace
}  // namespace fb

extern "C" fb_status fb_attn_outblock_noalloc(const fb_attn_desc* d, const void* q, const void* kp,
                                              const void* vp, int64_t prefix_len, float* a_out, float* l_out,
                                              cudaStream_t stream) {
  size_t need = 0;
  fb_status st = fb_outblock_workspace_bytes(d, prefix_len < 0 ? 0 : prefix_len, 0, &need);
  if (st != FB_OK) return st;
  if (need > (size_t)FB_NOALLOC_SCRATCH_BYTES) return FB_ENOSPACE;
  void* scratch = nullptr;
  if ((st = fb::scratch_address(&scratch)) != FB_OK) return st;
  return fb_attn_outblock(d, q, kp, vp, prefix_len, nullptr, 0, a_out, l_out, nullptr, nullptr, scratch,
                          (size_t)FB_NOALLOC_SCRATCH_BYTES, stream);
}
