// topk.cu — adaptive Top-tau block selection with static protection of the
// last query block (RRAttention abstract: "adaptive Top-tau selection"; TL;DR:
// "Top-tau block selection and a static protection of the last query block").
//
// One CTA per (head h, query block I).  The I+1 block masses of the row are
// sorted by (mass descending, J ascending) with a bitonic network on 64-bit
// keys in shared memory, their running sum is taken in fp64, and the shortest
// prefix whose sum reaches tau * (row total) is kept; the selected J are then
// written in ascending order (flag + exclusive scan).  Row Nb-1, and every row
// when tau >= 1, keeps all J <= I.
#include <stdint.h>

#include "rr_internal.h"

namespace rr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Exclusive block scan of one value per thread; returns the exclusive prefix,
// writes the block total to *total.  Deterministic order.
template <typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T* warp_buf, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    T y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_buf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    T w = lane < kWarps ? warp_buf[lane] : T(0);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      T y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    if (lane < kWarps) warp_buf[lane] = w;  // inclusive warp prefixes
  }
  __syncthreads();
  const T before_warp = warp == 0 ? T(0) : warp_buf[warp - 1];
  *total = warp_buf[kWarps - 1];
  const T excl = before_warp + x - v;
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kThreads) top_tau_kernel(const float* __restrict__ mass, int H, int Nb,
                                                           float tau, int32_t* __restrict__ count,
                                                           int32_t* __restrict__ idx, int p2max, int rep) {
  extern __shared__ __align__(16) uint8_t smem[];
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem);
  unsigned char* sel = reinterpret_cast<unsigned char*>(keys + p2max);
  __shared__ double dbuf[kWarps];
  __shared__ int ibuf[kWarps];
  __shared__ int s_cut;

  // Heavier rows (larger I) first.
  const int I = Nb - 1 - static_cast<int>(blockIdx.x / H);
  const int h = static_cast<int>(blockIdx.x % H);
  const long long row = static_cast<long long>(h) * Nb + I;
  const int n = I + 1;
  // output rows: heads h*rep .. h*rep+rep-1 (rep > 1: one mask for a GQA group)
  const long long orow = static_cast<long long>(h) * rep * Nb + I;
  const long long ostride = static_cast<long long>(Nb) * Nb;   // between output heads
  int32_t* out = idx + orow * Nb;
  const int tid = threadIdx.x;

  if (I == Nb - 1 || !(tau < 1.0f)) {  // protected last row, or tau >= 1: every causal block
    for (int r = 0; r < rep; ++r)
      for (int t = tid; t < n; t += kThreads) out[r * ostride + t] = t;
    for (int r = tid; r < rep; r += kThreads) count[orow + static_cast<long long>(r) * Nb] = n;
    return;
  }

  int p2 = 1;
  while (p2 < n) p2 <<= 1;
  const float* m = mass + row * Nb;
  // Key = (mass bits, ~J) complemented, so an ascending sort gives mass
  // descending, then J ascending; padding sorts last.
  for (int i = tid; i < p2; i += kThreads) {
    unsigned long long key = ~0ull;
    if (i < n) {
      const unsigned mb = __float_as_uint(m[i]);
      key = ~((static_cast<unsigned long long>(mb) << 32) | static_cast<unsigned long long>(0xFFFFFFFFu - i));
    }
    keys[i] = key;
  }
  if (tid == 0) s_cut = n - 1;
  __syncthreads();
  for (int kk = 2; kk <= p2; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < p2; i += kThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          const bool up = (i & kk) == 0;
          if (up ? (a > b) : (a < b)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }

  // Running sum in fp64 over contiguous chunks, chunk order = thread order.
  const int per = (p2 + kThreads - 1) / kThreads;
  const int c0 = tid * per, c1 = min(c0 + per, n);
  double local = 0.0;
  for (int t = c0; t < c1; ++t) local += static_cast<double>(__uint_as_float(static_cast<unsigned>(~keys[t] >> 32)));
  double total;
  double run = block_exclusive_scan<double>(local, dbuf, &total);
  const double thr = static_cast<double>(tau) * total;
  for (int t = c0; t < c1; ++t) {
    run += static_cast<double>(__uint_as_float(static_cast<unsigned>(~keys[t] >> 32)));
    if (run >= thr) {
      atomicMin(&s_cut, t);
      break;
    }
  }
  for (int t = tid; t < n; t += kThreads) sel[t] = 0;
  __syncthreads();
  const int cnt = s_cut + 1;
  for (int t = tid; t < cnt; t += kThreads) {
    const unsigned j = 0xFFFFFFFFu - static_cast<unsigned>(~keys[t] & 0xFFFFFFFFull);
    sel[j] = 1;
  }
  __syncthreads();
  // Ascending output: exclusive scan of the flags in J order.
  const int q0 = tid * per, q1 = min(q0 + per, n);
  int flags = 0;
  for (int t = q0; t < q1; ++t) flags += sel[t];
  int tot;
  int pos = block_exclusive_scan<int>(flags, ibuf, &tot);
  for (int t = q0; t < q1; ++t)
    if (sel[t]) {
      for (int r = 0; r < rep; ++r) out[r * ostride + pos] = t;
      ++pos;
    }
  for (int r = tid; r < rep; r += kThreads) count[orow + static_cast<long long>(r) * Nb] = cnt;
}

}  // namespace

cudaError_t launch_top_tau(const float* mass, int H, int Nb, float tau, int32_t* count, int32_t* idx, int rep,
                           cudaStream_t stream) {
  if (H <= 0 || Nb <= 0) return cudaSuccess;
  int p2 = 1;
  while (p2 < Nb) p2 <<= 1;
  const size_t smem = static_cast<size_t>(p2) * 8 + static_cast<size_t>(Nb);
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = set_smem_limit_once(top_tau_kernel, static_cast<int>(8 * kMaxBlocks + kMaxBlocks), smem_set);
  if (e != cudaSuccess) return e;
  top_tau_kernel<<<static_cast<unsigned>(H) * Nb, kThreads, smem, stream>>>(mass, H, Nb, tau, count, idx, p2, rep);
  return cudaGetLastError();
}

}  // namespace rr
