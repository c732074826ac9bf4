// rr_internal.h — launchers shared between the kernel files and the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rr {

struct DeviceGuardArgs {
  unsigned int* status;   // workspace status word
  uint64_t limit_ns;      // bound of every device-side wait
};

// Stride pooling of keys: kbar = mean of the S keys of each stride, stored as a
// bf16 pair (hi = bf16(kbar), lo = bf16(kbar - hi)).  k: [L, Hkv, d].
cudaError_t launch_pool_keys(const void* k, void* khi, void* klo, int L, int Hkv, int d, int S,
                             cudaStream_t stream);

// Sampled-score search: block mass[h, I, J] (unnormalised) for J <= I.
cudaError_t launch_search(const void* q, const void* khi, const void* klo, float* mass, int L, int H,
                          int Hkv, int d, int B, int S, const DeviceGuardArgs& g, cudaStream_t stream);

// Adaptive Top-tau with protection of the last query block.
cudaError_t launch_top_tau(const float* mass, int H, int Nb, float tau, int32_t* count, int32_t* idx,
                           cudaStream_t stream);

// Causal block-sparse attention over the mask.
cudaError_t launch_bsfa(const void* q, const void* k, const void* v, const int32_t* count,
                        const int32_t* idx, void* o, int L, int H, int Hkv, int d, int B,
                        const DeviceGuardArgs& g, cudaStream_t stream);

// Share of each row's block mass kept by a mask (diagnostics).
cudaError_t launch_mask_recall(const float* mass, const int32_t* count, const int32_t* idx, int H, int Nb,
                               float* recall, cudaStream_t stream);

// Low byte of the workspace status word when a device-side wait ran out.
constexpr unsigned kStatusTimeoutCode = 5u;

// Largest Nb = L/B the kernels accept (bounded by the on-chip list / sort buffers).
constexpr int kMaxBlocks = 4096;

}  // namespace rr
