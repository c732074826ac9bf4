// recall.cu — mask diagnostics: the dense view of a block mask, and the share
// of a row's exact attention mass that a block mask keeps (the synthetic analogue of RRAttention's pattern
// visualisations, sciencestack page, Figures 4 and 5: full-attention ground
// truth against the RR selection).
//
// Input mass is an unnormalised block mass [H, Nb, Nb] (entries J <= I), such as
// rr_search returns at stride S = 1, where every query is sampled and every key
// is its own stride, so that the block mass is the exact full-attention mass.
// recall[h, I] = sum over the listed J of mass[h, I, J] / sum over J <= I.
// One warp per row; fp64 sums in a fixed order (lane-strided partial sums, then
// a butterfly), so the result is deterministic.
#include <stdint.h>

#include "rr_internal.h"

namespace rr {
namespace {

constexpr int kWarpsPerBlock = 8;

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    mask_recall_kernel(const float* __restrict__ mass, const int32_t* __restrict__ count,
                       const int32_t* __restrict__ idx, int H, int Nb, float* __restrict__ recall) {
  const long long row = static_cast<long long>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(H) * Nb) return;
  const int I = static_cast<int>(row % Nb);
  const float* m = mass + row * Nb;
  const int32_t* list = idx + row * Nb;
  int c = count[row];
  c = c < 0 ? 0 : (c > I + 1 ? I + 1 : c);
  double tot = 0.0, kept = 0.0;
  for (int J = lane; J <= I; J += 32) tot += static_cast<double>(m[J]);
  for (int t = lane; t < c; t += 32) {
    const int J = list[t];
    if (J >= 0 && J <= I) kept += static_cast<double>(m[J]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, off);
    kept += __shfl_xor_sync(0xffffffffu, kept, off);
  }
  if (lane == 0) recall[row] = tot > 0.0 ? static_cast<float>(kept / tot) : 0.0f;
}

// Dense view of a block mask: one warp per (h, I) row clears the row's Nb bytes,
// then sets dense[h, I, J] = 1 for each listed J in [0, Nb).
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    mask_to_dense_kernel(const int32_t* __restrict__ count, const int32_t* __restrict__ idx, int H, int Nb,
                         uint8_t* __restrict__ dense) {
  const long long row = static_cast<long long>(blockIdx.x) * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(H) * Nb) return;
  uint8_t* out = dense + row * Nb;
  for (int J = lane; J < Nb; J += 32) out[J] = 0;
  __syncwarp();
  const int32_t* list = idx + row * Nb;
  int c = count[row];
  c = c < 0 ? 0 : (c > Nb ? Nb : c);
  for (int t = lane; t < c; t += 32) {
    const int J = list[t];
    if (J >= 0 && J < Nb) out[J] = 1;
  }
}

}  // namespace

cudaError_t launch_mask_to_dense(const int32_t* count, const int32_t* idx, int H, int Nb, uint8_t* dense,
                                 cudaStream_t stream) {
  const long long rows = static_cast<long long>(H) * Nb;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
  mask_to_dense_kernel<<<blocks, kWarpsPerBlock * 32, 0, stream>>>(count, idx, H, Nb, dense);
  return cudaGetLastError();
}

cudaError_t launch_mask_recall(const float* mass, const int32_t* count, const int32_t* idx, int H, int Nb,
                               float* recall, cudaStream_t stream) {
  const long long rows = static_cast<long long>(H) * Nb;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((rows + kWarpsPerBlock - 1) / kWarpsPerBlock);
  mask_recall_kernel<<<blocks, kWarpsPerBlock * 32, 0, stream>>>(mass, count, idx, H, Nb, recall);
  return cudaGetLastError();
}

}  // namespace rr
