// topk.cu — adaptive Top-tau block selection with static protection of the
// last query block (RRAttention abstract: "adaptive Top-tau selection"; TL;DR:
// "Top-tau block selection and a static protection of the last query block").
//
// One CTA per (head h, query block I).  The kept set of row I is the shortest
// prefix, in (mass descending, J ascending) order, of the I+1 block masses
// whose sum reaches tau * (row total).  Rows of up to 256 blocks are sorted
// outright (bitonic network on 64-bit keys, fp64 running sum).  Longer rows use
// that such a prefix is every block with mass above a threshold value T plus
// the lowest-J blocks with mass exactly T, and find T without sorting: the
// masses are non-negative floats, whose bit patterns order like their values,
// and a radix select over those bits (4 passes of 8 bits) walks down to T,
// each pass histogramming (count, mass sum) per digit of the remaining
// candidates and taking the digit where the running sum from the top crosses
// the target.  Those sums are exact integers (each mass scaled to a fixed-point
// fraction of the row total, 2^31 units), so the selection is deterministic.
// The selected J are written in ascending order (flag + exclusive scan).  Row
// Nb-1, and every row when tau >= 1, keeps all J <= I.
#include <stdint.h>

#include "rr_internal.h"

namespace rr {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPerThread = (kMaxBlocks + kThreads - 1) / kThreads;   // masses owned by one thread

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
  uint32_t hcnt[kWarps][256];   // per-warp histograms of the current pass
  uint32_t hsum[kWarps][256];
  double dbuf[kWarps];
  uint32_t ubuf[kWarps];
  uint32_t digit, base_sum, base_cnt;
};

// Rows up to this length are sorted outright (a 64-bit bitonic network in
// shared memory): for them the sort costs less than the radix passes' fixed
// work.
constexpr int kSmallRow = 256;

struct SmallShared {
  unsigned long long keys[kSmallRow];
  unsigned char sel[kSmallRow];
  double dbuf[kWarps];
  int ibuf[kWarps];
  int cut;
};

// The shortest prefix of the row in (mass descending, J ascending) order whose
// fp64 running sum reaches tau * total, for n <= kSmallRow; writes the selected
// J ascending to the rep output heads.
__device__ __forceinline__ void select_small(const float* __restrict__ m, int n, float tau, SmallShared& sh,
                                             int32_t* __restrict__ out, long long ostride, int rep,
                                             int32_t* __restrict__ count, long long orow, int Nb) {
  unsigned long long* keys = sh.keys;
  unsigned char* sel = sh.sel;
  const int tid = threadIdx.x;
  int p2 = 1;
  while (p2 < n) p2 <<= 1;
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
  if (tid == 0) sh.cut = n - 1;
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
  // Running sum in fp64 in sorted order (one entry per thread), first index
  // reaching tau * total.
  const double v = tid < n ? static_cast<double>(__uint_as_float(static_cast<unsigned>(~keys[tid] >> 32))) : 0.0;
  double total;
  const double run = block_exclusive_scan<double>(v, sh.dbuf, &total) + v;
  if (tid < n && run >= static_cast<double>(tau) * total) atomicMin(&sh.cut, tid);
  for (int t = tid; t < n; t += kThreads) sel[t] = 0;
  __syncthreads();
  const int cnt = sh.cut + 1;
  for (int t = tid; t < cnt; t += kThreads)
    sel[0xFFFFFFFFu - static_cast<unsigned>(~keys[t] & 0xFFFFFFFFull)] = 1;
  __syncthreads();
  // Ascending output: exclusive scan of the flags in J order.
  const int flag = tid < n ? sel[tid] : 0;
  int tot;
  const int pos = block_exclusive_scan<int>(flag, sh.ibuf, &tot);
  if (flag)
    for (int r = 0; r < rep; ++r) out[r * ostride + pos] = tid;
  for (int r = tid; r < rep; r += kThreads) count[orow + static_cast<long long>(r) * Nb] = cnt;
}

// kLarge: rows I >= kSmallRow (radix select); else rows I < kSmallRow (sort).
// The launch covers rows I_top, I_top - 1, ..., heavier rows first.
template <bool kLarge>
__global__ void __launch_bounds__(kThreads, kLarge ? 4 : 1) top_tau_kernel(const float* __restrict__ mass, int H,
                                                                          int Nb, float tau, int32_t* __restrict__ count,
                                                                          int32_t* __restrict__ idx, int rep,
                                                                          int I_top) {
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

  if constexpr (!kLarge) {
    __shared__ SmallShared ss;
    select_small(mass + row * Nb, n, tau, ss, out, ostride, rep, count, orow, Nb);
    return;
  } else {
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

    uint32_t T = 0, sum_gt = 0, cnt_gt = 0, k_eq = 1;
    if (total_i == 0) {
      // no mass at all: the order is J ascending and the first block reaches it
      T = 0xFFFFFFFFu;   // nothing is above T; J = 0 is the one block kept
    } else {
      // target: the smallest integer prefix sum that is >= tau * total
      const uint32_t target = static_cast<uint32_t>(
          fmin(ceil(static_cast<double>(tau) * static_cast<double>(total_i)), static_cast<double>(total_i)));
      uint32_t prefix = 0, base_sum = 0, base_cnt = 0;
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < kWarps * 256; b += kThreads) {
          (&sh.hcnt[0][0])[b] = 0u;
          (&sh.hsum[0][0])[b] = 0u;
        }
        __syncthreads();
        // histogram of the candidates: the masses whose higher digits equal the
        // digits chosen so far
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
          if (c0 + e < c1) {
            const uint32_t k = key[e];
            if (pass == 0 || ((k ^ prefix) >> (shift + 8)) == 0u) {
              const uint32_t d = (k >> shift) & 255u;
              atomicAdd(&sh.hcnt[warp][d], 1u);
              atomicAdd(&sh.hsum[warp][d], units(k));
            }
          }
        }
        __syncthreads();
        if (warp == 0) {
          // lane L holds digits 255-8L .. 248-8L (descending); the digit taken is
          // the one where the running sum from the top reaches the target
          uint32_t bs[8], bc[8], ls = 0, lc = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int b = 255 - 8 * lane - k;
            uint32_t s = 0, c = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
              s += sh.hsum[w][b];
              c += sh.hcnt[w][b];
            }
            bs[k] = s;
            bc[k] = c;
            ls += s;
            lc += c;
          }
          uint32_t is = ls, ic = lc;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const uint32_t ys = __shfl_up_sync(0xffffffffu, is, off);
            const uint32_t yc = __shfl_up_sync(0xffffffffu, ic, off);
            if (lane >= off) {
              is += ys;
              ic += yc;
            }
          }
          const uint32_t need = target - base_sum;   // >= 1, reached inside these candidates
          uint32_t run = is - ls, runc = ic - lc;
          if (run < need && need <= is) {            // exactly one lane
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (run + bs[k] >= need) {
                sh.digit = static_cast<uint32_t>(255 - 8 * lane - k);
                sh.base_sum = base_sum + run;
                sh.base_cnt = base_cnt + runc;
                break;
              }
              run += bs[k];
              runc += bc[k];
            }
          }
        }
        __syncthreads();
        prefix |= sh.digit << shift;
        base_sum = sh.base_sum;
        base_cnt = sh.base_cnt;
        __syncthreads();
      }
      T = prefix;
      sum_gt = base_sum;
      cnt_gt = base_cnt;
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

}  // namespace

cudaError_t launch_top_tau(const float* mass, int H, int Nb, float tau, int32_t* count, int32_t* idx, int rep,
                           cudaStream_t stream) {
  if (H <= 0 || Nb <= 0) return cudaSuccess;
  if (Nb > kMaxBlocks) return cudaErrorInvalidValue;
  // rows I >= kSmallRow by radix select, rows below by sorting: two launches
  const int n_large = Nb > kSmallRow ? Nb - kSmallRow : 0, n_small = Nb - n_large;
  if (n_large > 0) {
    top_tau_kernel<true><<<static_cast<unsigned>(H) * n_large, kThreads, 0, stream>>>(mass, H, Nb, tau, count, idx,
                                                                                      rep, Nb - 1);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  top_tau_kernel<false><<<static_cast<unsigned>(H) * n_small, kThreads, 0, stream>>>(mass, H, Nb, tau, count, idx,
                                                                                     rep, n_small - 1);
  return cudaGetLastError();
}

}  // namespace rr
