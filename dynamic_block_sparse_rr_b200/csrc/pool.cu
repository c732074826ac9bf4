// pool.cu — stride-mean keys, the alternative reading of the search's key side
// (RRAttention page, Abstract: scores gathered per stride at O(L^2/S^2) cost;
// the pages do not say whether a stride's keys are sampled or averaged, and the
// default search samples them).  The S keys of stride j are averaged
// in fp32 (sequential order t = 0..S-1) and stored as a bf16 pair so that the
// tensor-core search sees the mean to about 16 significant bits:
//   hi = bf16_rn(mean), lo = bf16_rn(mean - hi).
// HBM-bound: reads L*Hkv*d*2 bytes, writes 2*Ns*Hkv*d*2 bytes; one thread per
// 8 consecutive elements (16-byte loads, consecutive threads on consecutive
// addresses).
#include <cuda_bf16.h>

#include "rr_internal.h"

namespace rr {
namespace {

__global__ void __launch_bounds__(256) pool_keys_kernel(const uint4* __restrict__ k, uint4* __restrict__ khi,
                                                        uint4* __restrict__ klo, long long n_out,
                                                        int row_vec, int S, float inv_s) {
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n_out;
       t += (long long)gridDim.x * blockDim.x) {
    const long long j = t / row_vec;
    const int c = static_cast<int>(t - j * row_vec);
    const uint4* src = k + j * S * (long long)row_vec + c;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int s = 0; s < S; ++s) {
      uint4 v = __ldg(src + (long long)s * row_vec);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
    uint4 hi, lo;
    __nv_bfloat162* ph = reinterpret_cast<__nv_bfloat162*>(&hi);
    __nv_bfloat162* pl = reinterpret_cast<__nv_bfloat162*>(&lo);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float m0 = acc[2 * e] * inv_s, m1 = acc[2 * e + 1] * inv_s;
      const __nv_bfloat162 h = __floats2bfloat162_rn(m0, m1);
      const float2 hf = __bfloat1622float2(h);
      ph[e] = h;
      pl[e] = __floats2bfloat162_rn(m0 - hf.x, m1 - hf.y);
    }
    khi[t] = hi;
    klo[t] = lo;
  }
}

}  // namespace

cudaError_t launch_pool_keys(const void* k, void* khi, void* klo, int L, int Hkv, int d, int S,
                             cudaStream_t stream) {
  const int row_vec = Hkv * d / 8;
  const long long n_out = static_cast<long long>(L / S) * row_vec;
  if (n_out == 0) return cudaSuccess;
  long long blocks = (n_out + 255) / 256;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  pool_keys_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<uint4*>(khi), static_cast<uint4*>(klo), n_out, row_vec, S,
      1.0f / static_cast<float>(S));
  return cudaGetLastError();
}

}  // namespace rr
