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
// allocating library routine.  It resolves the array's device address once per
// device (cudaGetSymbolAddress, with that device current) and then runs the same
// kernels as rr_search, with the workspace carved out of the array.
#include <cuda_runtime.h>

#include <mutex>

#include "rr.h"

namespace {

constexpr size_t kStaticScratchBytes = 32ull << 20;   // 32 MiB, see rr.h
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a stand-in for the symbol, not a
// device address: it must never be passed to a kernel directly.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device (resolved on first use).
rr_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RR_ECUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return RR_ECUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
