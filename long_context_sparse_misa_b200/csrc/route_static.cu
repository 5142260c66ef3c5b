// The block-pooled router with library-owned scratch: misa_route_static.
//
// The router itself is the one of misa_route ("MISA: Mixture of Indexer
// Sparse Attention for Long-Context LLM Inference", gist.science summary,
// "Methodologie: MISA", Lightweight Block-Pooled Router); the paper has no
// counterpart for this entry point.  It exists for callers that cannot hand
// the library a workspace: a C or C++ serving loop that issues the router
// for every decode step from a host runtime with no device allocator of its
// own, or code that must not call cudaMalloc on that path (cudaMalloc can
// synchronise the device and can fail under memory pressure mid-request).
// Such a caller gets the same kernels, with their scratch in a file-scope
// device array of fixed size instead of a caller workspace.
//
// Scratch: kStaticScratchBytes (4 MiB) of device memory per device, part of
// the library's module image.  It holds the query-group table, the group
// scan's per-sequence scratch, and either the pooled-block range partial
// sums (CUDA-core router) or the split pooled keys (tensor-core router).
// Nothing in it needs to start at zero: every word a call reads was written
// earlier in the same call.  Problems whose router needs more are refused
// with MISA_ERR_UNSUPPORTED and a message giving both sizes.
//
// Set-up: the first call on each device, with that device current, looks up
// the array's device address (cudaGetSymbolAddress, which may load the
// module onto the device) and caches it; later calls launch kernels only.
// Make one call on each device before capturing a stream that uses it.
//
// Concurrency: there is one scratch array per device.  Two calls on the same
// device whose executions overlap (different streams, or different host
// threads without ordering) race on it and give wrong results; order them,
// for example by issuing them on one stream.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (set-up on the
// first call for that device).
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "misa_route_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    set_error("misa_route_static: device %d outside 0..%d", dev, kMaxDevices - 1);
    return MISA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "misa_route_static: cudaGetSymbolAddress");
    if (!p) {
      set_error("misa_route_static: cudaGetSymbolAddress returned NULL");
      return MISA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MISA_OK;
}

}  // namespace
}  // namespace misa

using namespace misa;

extern "C" int misa_route_static(const misa_problem_t* p, const uint16_t* q, const float* w,
                                 const uint16_t* K, const float* Kbar, int32_t m, int32_t* heads,
                                 uint16_t* q_r, float* w_r, float* router_scores,
                                 misa_stream_t stream) {
  // Problem and m checks (misa_workspace_size sets the message on failure).
  if (misa_workspace_size(p, m, 1, 0) == 0) return MISA_ERR_INVALID_ARG;
  if (tracing_enabled()) {
    set_error("misa_route_static: tracing is on; its CUDA events would be created in this call");
    return MISA_ERR_INVALID_ARG;
  }
  if (p->num_queries == 0) return MISA_OK;
  const size_t need = route_path_bytes(p);
  if (need > kStaticScratchBytes) {
    set_error("misa_route_static: this problem needs %zu bytes of router scratch, the static "
              "scratch holds %zu; use misa_route with a workspace",
              need, kStaticScratchBytes);
    return MISA_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc) return rc;
  // With need <= capacity misa_route takes the same path as with a caller
  // workspace of `need` bytes or more.
  return misa_route(p, q, w, K, Kbar, m, heads, q_r, w_r, router_scores, scratch,
                    kStaticScratchBytes, stream);
}
