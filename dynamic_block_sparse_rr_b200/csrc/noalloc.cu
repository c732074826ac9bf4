// noalloc.cu — rr_search_static: the pattern search for callers that cannot
// give the library any device memory of its own.
//
// rr_search needs a caller-provided workspace (pooled keys, block masses and a
// status word).  Some callers have no way to provide one: an operator or plugin
// interface that hands over only the input and output tensors, or a process
// whose device memory is wholly owned by another allocator, so that no extra
// buffer can be requested at run time.  For them the search's scratch lives
// here, in one file-scope device array that every GPU loading this library
// holds until the process exits.
//
// The entry point itself allocates nothing: it calls no cudaMalloc, cudaFree or
// allocating library routine.  On every call it asks the runtime for the
// array's device address on the current device (cudaGetSymbolAddress, a lookup
// that allocates nothing) and then runs the same kernels as rr_search, with the
// workspace carved out of the array.  The address is not kept between calls, so
// a context that was reset in the meantime (cudaDeviceReset) gets the new one.
#include <cuda_runtime.h>

#include "rr.h"

namespace {

constexpr size_t kStaticScratchBytes = 32ull << 20;   // 32 MiB, see rr.h

// The scratch.  In host code this name is only a stand-in for the symbol, not a
// device address: it must never be passed to a kernel directly.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the scratch in the current device's context.  The first
// call in a context also loads this library's device code there.
rr_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return RR_ECUDA;
  *out = p;
  return RR_OK;
}

}  // namespace

extern "C" rr_status rr_search_static(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S,
                                      float tau, int32_t* count, int32_t* idx, void* stream) {
  size_t need = 0;
  rr_status st = rr_workspace_size(L, H, Hkv, d, B, S, &need);
  if (st != RR_OK) return st;
  if (need > kStaticScratchBytes) return RR_ESCRATCH;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != RR_OK) return st;
  return rr_search(q, k, L, H, Hkv, d, B, S, tau, count, idx, nullptr, scratch, kStaticScratchBytes, stream);
}
