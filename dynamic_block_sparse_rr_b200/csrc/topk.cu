// topk.cu — adaptive Top-tau block selection with the last query block always
// kept (RRAttention page, Abstract: the adaptive Top-tau cut; TL;DR: Top-tau
// selection plus a fixed protection of the final query block).
//
// The kept set of row (h, I) is the shortest prefix, in (mass descending, J
// ascending) order, of its I+1 block masses whose sum reaches tau * (row
// total).  That prefix is every block with mass above a threshold value T plus
// the lowest-J blocks with mass exactly T, so T is found without sorting.  The
// sums are exact integers: each mass is scaled to a fixed-point fraction of the
// row total (round(mass / total * 2^31) units, the total in fp64), which makes
// the selection deterministic; it can differ from an exact real-number cut only
// for a block within ~2^-31 of the row total from tau.  The masses are
// non-negative floats, whose bit patterns order like their values:
//   * rows of up to 1024 blocks: one warp per row, T by bisection over its 31
//     bits (a candidate is kept while the units of the masses at or above it
//     still reach the target);
//   * longer rows: one CTA per row, T by a radix select (4 passes of 8 bits,
//     each histogramming the units of the remaining candidates per digit).
// The selected J are written in ascending order.  Row Nb-1, and every row when
// tau >= 1, keeps all J <= I.
#include <stdint.h>

#include "rr_internal.h"

namespace rr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPerThread = (kMaxBlocks + kThreads - 1) / kThreads;   // masses owned by one thread
constexpr int kWarpRow = 1024;   // rows up to this length: one warp per row

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

struct SelectShared {
  uint32_t hsum[kWarps][256];   // per-warp histograms (units per digit) of the current pass
  double dbuf[kWarps];
  uint32_t ubuf[kWarps];
  uint32_t digit, base_sum;
};

// Rows longer than kWarpRow blocks: radix select, one CTA per row.  The launch
// covers rows I_top, I_top - 1, ..., heavier rows first.
__global__ void __launch_bounds__(kThreads, 4) top_tau_kernel(const float* __restrict__ mass, int H, int Nb,
                                                             float tau, int32_t* __restrict__ count,
                                                             int32_t* __restrict__ idx, int rep, int I_top) {
  const int I = I_top - static_cast<int>(blockIdx.x / H);
  const int h = static_cast<int>(blockIdx.x % H);
  const long long row = static_cast<long long>(h) * Nb + I;
  const int n = I + 1;
  // output rows: heads h*rep .. h*rep+rep-1 (rep > 1: one mask for a GQA group)
  const long long orow = static_cast<long long>(h) * rep * Nb + I;
  const long long ostride = static_cast<long long>(Nb) * Nb;   // between output heads
  int32_t* out = idx + orow * Nb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (I == Nb - 1 || !(tau < 1.0f)) {  // protected last row, or tau >= 1: every causal block
    for (int r = 0; r < rep; ++r)
      for (int t = tid; t < n; t += kThreads) out[r * ostride + t] = t;
    for (int r = tid; r < rep; r += kThreads) count[orow + static_cast<long long>(r) * Nb] = n;
    return;
  }

  {
    __shared__ SelectShared sh;

    // This thread's contiguous chunk of the row: masses as bit patterns, and the
    // row total in fp64 (fixed summation order).
    const int per = (n + kThreads - 1) / kThreads;
    const int c0 = min(tid * per, n), c1 = min(c0 + per, n);
    const float* m = mass + row * Nb;
    uint32_t key[kPerThread];
    double local = 0.0;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      key[e] = 0u;
      if (c0 + e < c1) {
        const float v = m[c0 + e];
        key[e] = __float_as_uint(v);
        local += static_cast<double>(v);
      }
    }
    double total;
    block_exclusive_scan<double>(local, sh.dbuf, &total);
    // Fixed point: a mass is round(mass / total * 2^31) units; the units sum to
    // 2^31 up to rounding (at most 2^31 + n/2 < 2^32).
    const double scale = total > 0.0 ? 2147483648.0 / total : 0.0;
    auto units = [&](uint32_t k) { return __double2uint_rn(static_cast<double>(__uint_as_float(k)) * scale); };
    uint32_t lsum = 0;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e)
      if (c0 + e < c1) lsum += units(key[e]);
    uint32_t total_i;
    block_exclusive_scan<uint32_t>(lsum, sh.ubuf, &total_i);

    uint32_t T = 0, sum_gt = 0, k_eq = 1;
    if (total_i == 0) {
      // no mass at all: the order is J ascending and the first block reaches it
      T = 0xFFFFFFFFu;   // nothing is above T; J = 0 is the one block kept
    } else {
      // target: the smallest integer prefix sum that is >= tau * total
      const uint32_t target = static_cast<uint32_t>(
          fmin(ceil(static_cast<double>(tau) * static_cast<double>(total_i)), static_cast<double>(total_i)));
      uint32_t prefix = 0, base_sum = 0;
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < kWarps * 256; b += kThreads) (&sh.hsum[0][0])[b] = 0u;
        __syncthreads();
        // histogram of the candidates: the masses whose higher digits equal the
        // digits chosen so far
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          if (c0 + e < c1) {
            const uint32_t k = key[e];
            if (pass == 0 || ((k ^ prefix) >> (shift + 8)) == 0u) {
              atomicAdd(&sh.hsum[warp][(k >> shift) & 255u], units(k));
            }
          }
        }
        __syncthreads();
        if (warp == 0) {
          // lane L holds digits 255-8L .. 248-8L (descending); the digit taken is
          // the one where the running sum from the top reaches the target
          uint32_t bs[8], ls = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int b = 255 - 8 * lane - k;
            uint32_t s = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) s += sh.hsum[w][b];
            bs[k] = s;
            ls += s;
          }
          uint32_t is = ls;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const uint32_t ys = __shfl_up_sync(0xffffffffu, is, off);
            if (lane >= off) is += ys;
          }
          const uint32_t need = target - base_sum;   // >= 1, reached inside these candidates
          uint32_t run = is - ls;
          if (run < need && need <= is) {            // exactly one lane
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (run + bs[k] >= need) {
                sh.digit = static_cast<uint32_t>(255 - 8 * lane - k);
                sh.base_sum = base_sum + run;
                break;
              }
              run += bs[k];
            }
          }
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        base_sum = sh.base_sum;
        __syncthreads();
      }
      T = prefix;
      sum_gt = base_sum;
      // the blocks of mass exactly T all have the same units; the lowest-J k_eq
      // of them complete the prefix
      const uint32_t t_val = units(T);
      k_eq = t_val > 0 ? (target - sum_gt + t_val - 1) / t_val : 1u;
    }

    // flags in J order: above T, or equal to T and among the first k_eq equal
    uint32_t my_eq = 0;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e)
      if (c0 + e < c1 && (total_i == 0 ? (c0 + e == 0) : key[e] == T)) ++my_eq;
    uint32_t tot_eq;
    uint32_t rank = block_exclusive_scan<uint32_t>(my_eq, sh.ubuf, &tot_eq);
    uint32_t sel_bits = 0, my_sel = 0;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      if (c0 + e < c1) {
        const bool eq = total_i == 0 ? (c0 + e == 0) : key[e] == T;
        bool s = total_i != 0 && key[e] > T;
        if (eq) s = (rank++ < k_eq);
        if (s) {
          sel_bits |= 1u << e;
          ++my_sel;
        }
      }
    }
    uint32_t cnt;
    uint32_t pos = block_exclusive_scan<uint32_t>(my_sel, sh.ubuf, &cnt);
#pragma unroll
    for (int e = 0; e < kPerThread; ++e)
      if (sel_bits & (1u << e)) {
        for (int r = 0; r < rep; ++r) out[r * ostride + pos] = c0 + e;
        ++pos;
      }
    for (int r = tid; r < rep; r += kThreads) count[orow + static_cast<long long>(r) * Nb] = static_cast<int32_t>(cnt);
  }
}

// Rows of up to kWarpRow blocks: one warp per row, with the selection of the
// radix path (the same fixed-point units, target, threshold T and lowest-J rule
// for masses equal to T) and T found by bisection over its 31 bits instead of
// histograms: bit by bit from the top, a candidate is kept when the units of
// the masses at or above it still reach the target.  Lane l holds elements
// l, l+32, l+64, ... (kSlots of them, unused slots mass 0 and 0 units), so that
// (slot, lane) order is J order, and ballots give the ranks among equal masses
// and the output positions.

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);   // same bits on every lane
  return v;
}
__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) { return __reduce_add_sync(0xffffffffu, v); }

template <int kSlots>
__global__ void __launch_bounds__(kThreads) top_tau_warp_kernel(const float* __restrict__ mass, int H, int Nb,
                                                                float tau, int32_t* __restrict__ count,
                                                                int32_t* __restrict__ idx, int rep, int I_top,
                                                                int n_rows) {
  const int lane = threadIdx.x & 31;
  const int gw = static_cast<int>(blockIdx.x) * kWarps + static_cast<int>(threadIdx.x >> 5);
  if (gw >= n_rows * H) return;   // whole warps only
  const int I = I_top - gw / H;   // heavier rows first
  const int h = gw % H;
  const long long row = static_cast<long long>(h) * Nb + I;
  const int n = I + 1;            // <= 32 * kSlots
  const long long orow = static_cast<long long>(h) * rep * Nb + I;
  const long long ostride = static_cast<long long>(Nb) * Nb;
  int32_t* out = idx + orow * Nb;
  if (I == Nb - 1 || !(tau < 1.0f)) {  // protected last row, or tau >= 1: every causal block
    for (int r = 0; r < rep; ++r)
      for (int t = lane; t < n; t += 32) out[r * ostride + t] = t;
    for (int r = lane; r < rep; r += 32) count[orow + static_cast<long long>(r) * Nb] = n;
    return;
  }
  const float* m = mass + row * Nb;
  uint32_t key[kSlots], un[kSlots];
  double local = 0.0;
#pragma unroll
  for (int e = 0; e < kSlots; ++e) {
    key[e] = 0u;
    const int i = e * 32 + lane;
    if (i < n) {
      const float v = m[i];
      key[e] = __float_as_uint(v);
      local += static_cast<double>(v);
    }
  }
  const double total = warp_sum_f64(local);
  // Fixed point: a mass is round(mass / total * 2^31) units (sum <= 2^31 + n/2).
  const double scale = total > 0.0 ? 2147483648.0 / total : 0.0;
  auto units = [&](uint32_t k) { return __double2uint_rn(static_cast<double>(__uint_as_float(k)) * scale); };
  uint32_t lsum = 0;
#pragma unroll
  for (int e = 0; e < kSlots; ++e) {
    un[e] = e * 32 + lane < n ? units(key[e]) : 0u;
    lsum += un[e];
  }
  const uint32_t total_i = warp_sum_u32(lsum);

  uint32_t T = 0xFFFFFFFFu, k_eq = 1;
  if (total_i != 0) {
    const uint32_t target = static_cast<uint32_t>(
        fmin(ceil(static_cast<double>(tau) * static_cast<double>(total_i)), static_cast<double>(total_i)));
    // the largest T whose masses at or above it reach the target (a mass
    // present in the row: the sum only changes at present values); unused
    // slots (key 0, 0 units) never count, since every candidate is >= 1
    uint32_t P = 0;
    for (int b = 30; b >= 0; --b) {
      const uint32_t cand = P | (1u << b);
      uint32_t sge = 0;
#pragma unroll
      for (int e = 0; e < kSlots; ++e) sge += key[e] >= cand ? un[e] : 0u;
      if (warp_sum_u32(sge) >= target) P = cand;
    }
    T = P;
    uint32_t sgt = 0;
#pragma unroll
    for (int e = 0; e < kSlots; ++e) sgt += key[e] > T ? un[e] : 0u;
    const uint32_t sum_gt = warp_sum_u32(sgt);
    const uint32_t t_val = units(T);
    k_eq = t_val > 0 ? (target - sum_gt + t_val - 1) / t_val : 1u;
  }

  // flags in J order: above T, or equal to T and among the first k_eq equal
  // (a row without mass keeps J = 0 alone)
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t eq_seen = 0, pos = 0;
#pragma unroll
  for (int e = 0; e < kSlots; ++e) {
    if (e * 32 < n) {   // uniform across the warp
      const int i = e * 32 + lane;
      const bool valid = i < n;
      const bool eq = valid && (total_i == 0 ? i == 0 : key[e] == T);
      const bool gt = valid && total_i != 0 && key[e] > T;
      const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
      const bool sel = gt || (eq && eq_seen + __popc(eqm & lt) < k_eq);
      eq_seen += __popc(eqm);
      const uint32_t sm = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const uint32_t p = pos + __popc(sm & lt);
        for (int r = 0; r < rep; ++r) out[r * ostride + p] = i;
      }
      pos += __popc(sm);
    }
  }
  for (int r = lane; r < rep; r += 32) count[orow + static_cast<long long>(r) * Nb] = static_cast<int32_t>(pos);
}

template <int kSlots>
cudaError_t launch_warp_rows(const float* mass, int H, int Nb, float tau, int32_t* count, int32_t* idx, int rep,
                             int I_top, int n_rows, cudaStream_t stream) {
  if (n_rows <= 0) return cudaSuccess;
  const long long warps = static_cast<long long>(H) * n_rows;
  top_tau_warp_kernel<kSlots><<<static_cast<unsigned>((warps + kWarps - 1) / kWarps), kThreads, 0, stream>>>(
      mass, H, Nb, tau, count, idx, rep, I_top, n_rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_top_tau(const float* mass, int H, int Nb, float tau, int32_t* count, int32_t* idx, int rep,
                           cudaStream_t stream) {
  if (H <= 0 || Nb <= 0) return cudaSuccess;
  if (Nb > kMaxBlocks) return cudaErrorInvalidValue;
  // Rows I >= kWarpRow: radix select, one CTA per row.  Shorter rows: one warp
  // per row, in three launches by length (8, 16 or 32 masses per lane).
  // Heavier rows first.
  if (Nb > kWarpRow) {
    top_tau_kernel<<<static_cast<unsigned>(H) * (Nb - kWarpRow), kThreads, 0, stream>>>(mass, H, Nb, tau, count,
                                                                                       idx, rep, Nb - 1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // rows [lo, hi) of the row range a launch covers
  auto range = [&](int lo, int hi, int& I_top, int& n_rows) {
    hi = hi < Nb ? hi : Nb;
    n_rows = hi > lo ? hi - lo : 0;
    I_top = hi - 1;
  };
  int top, nr;
  cudaError_t e;
  range(512, kWarpRow, top, nr);
  if ((e = launch_warp_rows<32>(mass, H, Nb, tau, count, idx, rep, top, nr, stream)) != cudaSuccess) return e;
  range(256, 512, top, nr);
  if ((e = launch_warp_rows<16>(mass, H, Nb, tau, count, idx, rep, top, nr, stream)) != cudaSuccess) return e;
  range(0, 256, top, nr);
  if ((e = launch_warp_rows<8>(mass, H, Nb, tau, count, idx, rep, top, nr, stream)) != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace rr
