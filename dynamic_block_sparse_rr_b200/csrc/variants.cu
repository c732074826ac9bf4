// variants.cu — data movement for the search's sampling variants (RRAttention
// leaves open how the per-head offset behaves from stride to stride, what
// stands for the keys of a stride, and whether GQA heads share one mask):
//
//   gather_rotated: the rows at the rotating offsets p(h, i) = i*S + (h + i) mod S,
//     gathered into a dense [Ns, H, d] array the search reads with plain 3D tiles
//     (queries, and keys unless the stride-mean keys are asked for).
//     HBM-bound: reads and writes Ns*H*d*2 bytes; one thread per 16 bytes,
//     consecutive threads on consecutive addresses of one row.
//   group_mass: the block masses of the g query heads of a kv head summed, in
//     head order, into one [Nb, Nb] mass per kv head (one mask per GQA group).
//     HBM-bound: reads H*Nb^2*4 bytes, writes Hkv*Nb^2*4; float4 when Nb % 4 == 0.
#include <stdint.h>

#include "rr_internal.h"

namespace rr {
namespace {

__global__ void __launch_bounds__(256) gather_rotated_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                             long long n_out, int H, int src_heads, int div,
                                                             int row_vec, int S) {
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n_out;
       t += (long long)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(t % row_vec);
    const long long ih = t / row_vec;              // i * H + h
    const int h = static_cast<int>(ih % H);
    const long long i = ih / H;
    const long long p = i * S + (h + i) % S;       // rotating sampled position
    dst[t] = __ldg(src + (p * src_heads + h / div) * row_vec + c);
  }
}

template <bool VEC>
__global__ void __launch_bounds__(256) group_mass_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                                         int g, long long plane, long long n_out) {
  // plane = Nb*Nb floats (VEC: float4s); n_out = Hkv * plane
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n_out;
       t += (long long)gridDim.x * blockDim.x) {
    const long long kv = t / plane, e = t - kv * plane;
    const long long base = kv * g * plane + e;
    if (VEC) {
      const float4* s4 = reinterpret_cast<const float4*>(src);
      float4 a = __ldg(s4 + base);
      for (int u = 1; u < g; ++u) {
        const float4 b = __ldg(s4 + base + u * plane);
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
      reinterpret_cast<float4*>(dst)[t] = a;
    } else {
      float a = __ldg(src + base);
      for (int u = 1; u < g; ++u) a += __ldg(src + base + u * plane);
      dst[t] = a;
    }
  }
}

unsigned grid_for(long long n) {
  long long blocks = (n + 255) / 256;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  return static_cast<unsigned>(blocks);
}

}  // namespace

cudaError_t launch_gather_rotated(const void* src, void* dst, int L, int H, int src_heads, int div, int d, int S,
                                  cudaStream_t stream) {
  const int row_vec = d / 8;
  const long long n_out = static_cast<long long>(L / S) * H * row_vec;
  if (n_out == 0) return cudaSuccess;
  gather_rotated_kernel<<<grid_for(n_out), 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                            n_out, H, src_heads, div, row_vec, S);
  return cudaGetLastError();
}

cudaError_t launch_group_mass(const float* src, float* dst, int Hkv, int g, int Nb, cudaStream_t stream) {
  const long long plane = static_cast<long long>(Nb) * Nb;
  if (plane == 0 || Hkv <= 0) return cudaSuccess;
  const bool vec = (plane % 4) == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;
  if (vec) {
    const long long n = Hkv * (plane / 4);
    group_mass_kernel<true><<<grid_for(n), 256, 0, stream>>>(src, dst, g, plane / 4, n);
  } else {
    const long long n = Hkv * plane;
    group_mass_kernel<false><<<grid_for(n), 256, 0, stream>>>(src, dst, g, plane, n);
  }
  return cudaGetLastError();
}

}  // namespace rr
