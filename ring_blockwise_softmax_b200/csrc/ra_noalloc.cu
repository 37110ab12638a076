// ra_noalloc.cu - ra_ring_fwd_noalloc: the stepwise ring forward with its fp32 accumulator held
// in a fixed, library-owned device array instead of caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point of the call.  Examples:
// code running inside a host application whose caching allocator already owns all device memory
// and exposes no scratch interface (a cudaMalloc there fails, or fragments the pool), services that
// fix their memory budget at start-up and forbid allocations afterwards, and latency-critical
// paths that must not pay for the implicit device-wide synchronisation of cudaMalloc / cudaFree.
// The caller still passes the inputs and outputs; only the intermediate (O, LSE) accumulator
// moves into the library.
//
// The array lives for as long as the library is loaded, on every device that loads it.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "ra_attn.h"
#include "ra_internal.h"

namespace ra {
ra_status_t set_last_error(ra_status_t status, const char* message);  // defined in ra_attn.cu
}

namespace {

// Scratch for the stepwise ring's fp32 (O, LSE) accumulator; its size is RA_NOALLOC_SCRATCH_BYTES.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device ordinal, with the context it was looked up in.
struct ScratchAddr {
  void* ptr = nullptr;
  unsigned long long ctx = 0;
};
std::mutex g_noalloc_mu;
ScratchAddr g_noalloc_addr[64];

ra_status_t noalloc_fail(ra_status_t st, const std::string& msg) { return ra::set_last_error(st, msg.c_str()); }

}  // namespace

extern "C" ra_status_t ra_ring_fwd_noalloc(const ra_tensor_t* q, const ra_tensor_t* k, const ra_tensor_t* v, int P,
                                           int layout, int causal, float scale, const ra_tensor_t* o, float* lse,
                                           ra_stream_t stream) {
  size_t need = 0;
  ra_status_t st = ra_ring_workspace_size(q, P, RA_RING_STEPWISE, &need);
  if (st != RA_OK) return st;
  if (need > RA_NOALLOC_SCRATCH_BYTES)
    return noalloc_fail(RA_ERR_WORKSPACE,
                        "ra_ring_fwd_noalloc: the accumulator needs " + std::to_string(need) +
                            " bytes, more than the fixed scratch of " + std::to_string(RA_NOALLOC_SCRATCH_BYTES) +
                            " bytes; use ra_ring_fwd with a caller-allocated workspace");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(RA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return noalloc_fail(RA_ERR_UNSUPPORTED, "device ordinal out of range");
  void* ptr = nullptr;
  {
    // Set-up, once per device and context, with that device current: the symbol's device address
    // (the name itself is only a host-side stand-in and must never be handed to a kernel).  The
    // address is looked up again when the current context is not the one it was found in, e.g.
    // after cudaDeviceReset, which reloads the module.
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    const unsigned long long ctx = ra::current_context_id();
    ScratchAddr& a = g_noalloc_addr[dev];
    if (a.ptr == nullptr || ctx == 0 || ctx != a.ctx) {
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess)
        return noalloc_fail(RA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
      a.ptr = ptr;
      a.ctx = ra::current_context_id();
    }
    ptr = a.ptr;
  }
  // Step 0 of the stepwise ring writes every accumulator element that later steps read, so the
  // scratch needs no clearing between calls.
  const ra_stream_t streams[1] = {stream};
  return ra_ring_fwd(q, k, v, P, layout, causal, scale, RA_RING_STEPWISE, o, lse, streams, 1, ptr, need);
}
