// attn_bwd_static_workspace: the backward pass for callers that cannot
// allocate device memory.  Host code plus one file-scope device array.
//
// The backward needs scratch memory (fp32 row sums and the fp32 dQ
// accumulator).  attn_bwd takes it from the caller; this entry point takes it
// from `g_static_workspace` below instead, so the caller passes inputs and
// outputs only.  The array lives in every GPU that loads this library, for the
// life of the process.
#include <cuda_runtime.h>

#include <cstring>

#include "../../include/attn.h"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[ATTN_STATIC_WORKSPACE_BYTES];

// Device address of the stream's device's copy of the array.  Host code cannot
// use the symbol's name as a device pointer, so the address is looked up with
// that device current.  It is looked up on every call rather than cached: a
// reset of the device's primary context reloads the module and can move the
// array.
cudaError_t workspace_address(cudaStream_t stream, void** out) {
  int cur = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return e;
  dev = cur;
  if (stream != nullptr && (e = cudaStreamGetDevice(stream, &dev)) != cudaSuccess) return e;
  if (dev != cur && (e = cudaSetDevice(dev)) != cudaSuccess) return e;
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_static_workspace);
  if (dev != cur) {
    const cudaError_t r = cudaSetDevice(cur);  // the caller's device comes back either way
    if (e == cudaSuccess) e = r;
  }
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" int attn_bwd_static_workspace(const attn_bwd_params* params, void* stream_ptr) {
  if (!params || params->struct_size != sizeof(attn_bwd_params)) return cudaErrorInvalidValue;
  const size_t need = attn_bwd_workspace_size(params);
  if (need > (size_t)ATTN_STATIC_WORKSPACE_BYTES) return cudaErrorMemoryAllocation;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  void* ws = nullptr;
  cudaError_t e = workspace_address(stream, &ws);
  if (e != cudaSuccess) return e;
  attn_bwd_params p;
  std::memcpy(&p, params, sizeof(p));
  p.workspace = ws;
  p.workspace_bytes = ATTN_STATIC_WORKSPACE_BYTES;
  return attn_bwd(&p, stream_ptr);
}
