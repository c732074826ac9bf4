// decode.cu — decode-stage sparsification: one new token per sequence attends
// to its KV cache through a round-robin sampled search and block-sparse
// attention.  The RRAttention pages name decoding-stage sparsification only as
// a future extension (sciencestack page, TL;DR); the operator here carries the
// prefill rules over to a single query at position t = len - 1:
//   * head h scores the cached keys at its own sampled positions
//     j*S + (h mod S) <= t, softmax over them, block mass per key block;
//   * Top-tau over the key blocks J <= t/B as in prefill, and the block that
//     holds the query (the newest keys) is always kept;
//   * the query attends to every key <= t of the kept blocks.
//
// The path is bound by HBM (the sampled keys, then the kept K and V blocks); the
// kernels are sized for bytes in flight and kept lean in instructions:
//   decode_search_kernel   a few CTAs per (sequence, head), each over a run of
//                          the head's sampled key rows: 128-row TMA tiles of a
//                          zero-copy strided view (two-stage ring) scored on
//                          m16n8k16 tensor-core tiles (mma.sync, q as column 0),
//                          scores to the workspace, the run's max and block
//                          masses on that max.  The CTA that finishes a row
//                          last puts the row's masses on one scale and runs
//                          Top-tau on fixed-point units of the row total (the
//                          prefill rule), its threshold found by four passes
//                          over 8-bit digits of the mass bits; list and a
//                          bitmap of the kept blocks out.  One CTA also writes
//                          the prefix of the sequences' block counts;
//   decode_group_select_kernel  (one list per GQA group only) one CTA per
//                          (sequence, kv head): Top-tau on the group's summed
//                          masses, the list written to every head of the group;
//   decode_attn_kernel     one persistent CTA per SM over an equal share of the
//                          flattened (sequence, kv head, causal key block)
//                          space: a kept block's K and V tiles come in once by
//                          TMA (two-stage ring, running on across rows) for
//                          every query head of the GQA group that kept it.  The
//                          group's <= 8 heads are the 8 columns of m16n8k16
//                          tiles, so the two small contractions per block
//                          (scores of 128 keys, P V) are a few instructions per
//                          warp; each warp keeps an online softmax over its 16
//                          keys of every block.  At the end of each row the
//                          warps' partials merge into the CTA's partial for the
//                          row;
//   decode_combine_kernel  one CTA per (sequence, kv head): the partials of the
//                          CTAs that shared the row merged into the output.
#include <cuda_bf16.h>
#include <math.h>
#include <stdlib.h>

#include <algorithm>
#include <atomic>

#include "rr_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace rr {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kMaxPer = (kMaxBlocks + kDecThreads - 1) / kDecThreads;   // masses per thread

// Block-wide sums and max over the 256 threads (fixed order: warp trees, then
// warp 0 over the warp results).  `buf` holds kDecWarps slots; every thread
// gets the result.
template <typename T>
__device__ __forceinline__ T block_sum(T v, T* buf) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) buf[warp] = v;
  __syncthreads();
  T s = buf[0];
#pragma unroll
  for (int w = 1; w < kDecWarps; ++w) s += buf[w];
  return s;
}

__device__ __forceinline__ float block_max(float v, float* buf) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) buf[warp] = v;
  __syncthreads();
  float s = buf[0];
#pragma unroll
  for (int w = 1; w < kDecWarps; ++w) s = fmaxf(s, buf[w]);
  return s;
}

// Exclusive scan of one u32 per thread in thread order; *total gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* buf, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  __syncthreads();
  if (lane == 31) buf[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) {
    before += w < warp ? buf[w] : 0u;
    all += buf[w];
  }
  *total = all;
  return before + x - v;
}

constexpr int kSearchTile = 128;   // sampled keys per TMA tile of the search
constexpr int kSearchStages = 2;

// Byte offset of element (row, c) in a TMA tile of rows x D bf16 stored as D/64
// column blocks of rows x 128 bytes with the 128-byte swizzle (c a multiple of 8
// when used as a 16-byte row address).
template <int BN>
__device__ __forceinline__ uint32_t swz(int row, int c) {
  return static_cast<uint32_t>((c >> 6) * (BN * 128) + row * 128 + ((((c & 63) >> 3) ^ (row & 7)) << 4) + (c & 7) * 2);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col).
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct DecSearchShared {
  uint64_t full[kSearchStages];
  int abort;
  int last;
  double dbuf[kDecWarps];
  float fbuf[kDecWarps];
  uint32_t ubuf[kDecWarps];
  uint32_t hist[kDecThreads];   // radix digits of the threshold search
  uint32_t digit, above;
};

// Top-tau over the nb = Jt + 1 block masses in mass[] (shared memory), as in
// prefill (fixed-point units of the row total; the threshold, the largest mass
// whose masses at or above it reach the target, found digit by digit of the
// mass bits; equal masses to the lower J), plus the current block Jt.  wbits (shared memory, ceil(nb/32) words) collects the
// bitmap.  The ascending list goes to rep consecutive rows of out (row stride
// out_stride), the bitmap to rep consecutive rows of obits (W words each), the
// count to count[0 .. rep).  Called by every thread of the CTA.
__device__ __noinline__ void block_select(DecSearchShared& sh, const float* mass, uint32_t* wbits, int nb, int Jt,
                                          float tau, int32_t* out, long long out_stride, uint32_t* obits, int W,
                                          int32_t* count, int rep) {
  const int tid = threadIdx.x;
  for (int w = tid; w < (nb + 31) / 32; w += kDecThreads) wbits[w] = 0u;
  __syncthreads();
  // this thread's contiguous chunk of the row
  const int per = (nb + kDecThreads - 1) / kDecThreads;
  const int c0 = min(tid * per, nb), c1 = min(c0 + per, nb);
  uint32_t key[kMaxPer];
  double local = 0.0;
#pragma unroll
  for (int e = 0; e < kMaxPer; ++e) {
    key[e] = 0u;
    if (c0 + e < c1) {
      const float v = mass[c0 + e];
      key[e] = __float_as_uint(v);
      local += static_cast<double>(v);
    }
  }
  uint32_t sel_bits = 0;
  if (tau < 1.0f) {
    const double total = block_sum<double>(local, sh.dbuf);
    const double scale = total > 0.0 ? 2147483648.0 / total : 0.0;
    auto units = [&](uint32_t kk) { return __double2uint_rn(static_cast<double>(__uint_as_float(kk)) * scale); };
    uint32_t un[kMaxPer], lsum = 0;
#pragma unroll
    for (int e = 0; e < kMaxPer; ++e) {
      un[e] = c0 + e < c1 ? units(key[e]) : 0u;
      lsum += un[e];
    }
    const uint32_t total_i = block_sum<uint32_t>(lsum, sh.ubuf);
    if (total_i != 0) {
      const uint32_t target = static_cast<uint32_t>(
          fmin(ceil(static_cast<double>(tau) * static_cast<double>(total_i)), static_cast<double>(total_i)));
      // the largest mass T whose masses at or above it still reach the target,
      // one 8-bit digit of its bits at a time from the top: `above` holds the
      // units of the masses above the digits fixed so far, and the digit taken
      // is the largest whose masses, with `above`, reach the target
      uint32_t T = 0, above = 0;
      for (int shift = 24; shift >= 0; shift -= 8) {
        sh.hist[tid] = 0u;
        __syncthreads();
        const uint32_t hmask = shift == 24 ? 0u : (0xffffffffu << (shift + 8));
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e)
          if (c0 + e < c1 && (key[e] & hmask) == T) atomicAdd(&sh.hist[(key[e] >> shift) & 255u], un[e]);
        __syncthreads();
        const uint32_t v = sh.hist[255 - tid];   // thread i takes digit 255 - i
        uint32_t all;
        const uint32_t ex = block_excl_scan(v, sh.ubuf, &all);   // units of the digits above it
        if (above + ex < target && above + ex + v >= target) {
          sh.digit = 255u - tid;
          sh.above = above + ex;
        }
        __syncthreads();
        T |= sh.digit << shift;
        above = sh.above;
      }
      const uint32_t sum_gt = above;   // units of the masses above T
      uint32_t my_eq = 0;
#pragma unroll
      for (int e = 0; e < kMaxPer; ++e) my_eq += (c0 + e < c1 && key[e] == T) ? 1u : 0u;
      const uint32_t t_val = units(T);
      const uint32_t k_eq = t_val > 0 ? (target - sum_gt + t_val - 1) / t_val : 1u;
      uint32_t tot_eq;
      uint32_t rank = block_excl_scan(my_eq, sh.ubuf, &tot_eq);   // masses equal to T: lowest J first
#pragma unroll
      for (int e = 0; e < kMaxPer; ++e) {
        if (c0 + e < c1) {
          bool s = key[e] > T;
          if (key[e] == T) s = rank++ < k_eq;
          if (s) sel_bits |= 1u << e;
        }
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < kMaxPer; ++e)
      if (c0 + e < c1) sel_bits |= 1u << e;
  }
  if (Jt >= c0 && Jt < c1) sel_bits |= 1u << (Jt - c0);   // the block holding the query
  uint32_t my_sel = __popc(sel_bits), cnt;
  uint32_t pos = block_excl_scan(my_sel, sh.ubuf, &cnt);
#pragma unroll
  for (int e = 0; e < kMaxPer; ++e) {
    if (sel_bits & (1u << e)) {
      for (int r = 0; r < rep; ++r) out[r * out_stride + pos] = c0 + e;
      ++pos;
      atomicOr(&wbits[(c0 + e) >> 5], 1u << ((c0 + e) & 31));
    }
  }
  __syncthreads();
  for (int r = 0; r < rep; ++r)
    for (int w = tid; w < W; w += kDecThreads) obits[r * W + w] = w < (nb + 31) / 32 ? wbits[w] : 0u;
  if (tid < rep) count[tid] = static_cast<int32_t>(cnt);
}


// Exclusive prefix of the sequences' causal block counts (0 for a length
// outside [1, Lmax]): rowstart[n], and rowstart[N] the total.  Called by every
// thread of one CTA.
__device__ void block_count_prefix(const int32_t* __restrict__ lens, int N, int Lmax, int B,
                                   int32_t* __restrict__ rowstart, uint32_t* buf) {
  uint32_t carry = 0;
  for (int base = 0; base < N; base += kDecThreads) {
    const int n = base + static_cast<int>(threadIdx.x);
    uint32_t nbl = 0;
    if (n < N) {
      const int len = __ldg(lens + n);
      nbl = (len >= 1 && len <= Lmax) ? static_cast<uint32_t>((len - 1) / B + 1) : 0u;
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan(nbl, buf, &tot);
    if (n < N) rowstart[n] = static_cast<int32_t>(carry + ex);
    carry += tot;
  }
  if (threadIdx.x == 0) rowstart[N] = static_cast<int32_t>(carry);
}

// grid (N*H, SC): CTA (row, c) scores the sampled keys of tiles [c tpc, (c+1) tpc)
// of its (sequence, head) row and owns the key blocks those keys fall in
// (B/S divides the 128 strides of a tile).  Its max and its blocks' masses on
// that max go to the workspace; the CTA that arrives last on the row's counter
// (zeroed before the launch) rescales every chunk's masses to the row max and
// selects.
template <int D>
__global__ void __launch_bounds__(kDecThreads, 3) decode_search_kernel(
    const __grid_constant__ CUtensorMap mks, const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lens,
    int N, int Lmax, int H, int Hkv, int B, int S, float sl2, float tau, int tpc, float* __restrict__ scores,
    int Ns_max, float* __restrict__ cmax, unsigned int* __restrict__ arrive, float* __restrict__ mass, int group,
    int32_t* __restrict__ count, int32_t* __restrict__ idx, uint32_t* __restrict__ bits, int Nbm, int W,
    int32_t* __restrict__ rowstart, unsigned int* status, uint64_t limit_ns) {
  constexpr int kTileBytes = kSearchTile * D * 2;
  static_assert(kMaxBlocks * 4 + kMaxBlocks / 8 + kDecSearchChunks * 4 <= kSearchStages * kTileBytes,
                "selection arrays fit in the ring");
  __shared__ DecSearchShared sh;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int SC = static_cast<int>(gridDim.y), c = static_cast<int>(blockIdx.y);
  const long long row = blockIdx.x;
  const int n = static_cast<int>(row / H), h = static_cast<int>(row % H);
  const int kvh = h / (H / Hkv);
  int32_t* out = idx + row * Nbm;
  uint32_t* obits = bits + row * W;
  if (c == 0 && row == 0) block_count_prefix(lens, N, Lmax, B, rowstart, sh.ubuf);
  const int len = __ldg(lens + n);
  if (len < 1 || len > Lmax) {   // not a cache length this call can serve: nothing selected
    if (c == 0) {
      if (tid == 0) {
        count[row] = 0;
        atomicCAS(status, 0u, kStatusLenCode | (static_cast<unsigned>(n < (1 << 24) ? n : (1 << 24) - 1) << 8));
      }
      for (int w = tid; w < W; w += kDecThreads) obits[w] = 0u;
    }
    return;
  }
  const int t = len - 1, Jt = t / B, nb = Jt + 1, off = h % S, r = B / S;
  const int ns = t >= off ? (t - off) / S + 1 : 0;   // sampled keys at or before t
  const int nt = (ns + kSearchTile - 1) / kSearchTile;
  const int i0 = c * tpc, i1 = min(i0 + tpc, nt);      // this CTA's tiles
  const int bpc = tpc * (kSearchTile / r);
  const int J0 = min(c * bpc, nb), J1 = min(J0 + bpc, nb);   // and key blocks
  if (tid == 0) {
    for (int st = 0; st < kSearchStages; ++st) mbar_init(smem_u32(&sh.full[st]), 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  // warp w scores keys 16w .. 16w + 15 of a tile on m16n8k16 tiles: the keys
  // are A fragments (ldmatrix from the swizzled tile), q is column 0 of the B
  // fragments (the other seven columns are zero)
  const int warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;
  uint32_t qb[D / 16][2];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const __nv_bfloat16* qr = q + row * D + 16 * ks + 2 * tig;
    qb[ks][0] = gid == 0 ? __ldg(reinterpret_cast<const uint32_t*>(qr)) : 0u;
    qb[ks][1] = gid == 0 ? __ldg(reinterpret_cast<const uint32_t*>(qr + 8)) : 0u;
  }
  __syncthreads();
  const Guard guard{&sh.abort, status, limit_ns};
  // tile i: the sampled keys of strides 128 i .. 128 i + 127 of sequence n
  auto issue = [&](int i) {
    const int st = (i - i0) % kSearchStages;
    const uint32_t fb = smem_u32(&sh.full[st]);
    mbar_expect_tx(fb, kTileBytes);
    uint8_t* dst = smem + st * kTileBytes;
    for (int a = 0; a < D / 64; ++a)
      tma_load_4d(smem_u32(dst + a * kSearchTile * 128), &mks, fb, a * 64, kvh, off,
                  n * (Lmax / S) + i * kSearchTile);
  };
  int issued = i0;
  if (tid == 0 && i0 < i1) {
    tma_prefetch_desc(&mks);
    for (; issued < i1 && issued < i0 + kSearchStages; ++issued) issue(issued);
  }
  // scores (log2 units) of the sampled keys, to the workspace row
  float* sc = scores + row * Ns_max;
  float lmax = -INFINITY;
  bool ok = true;
  for (int i = i0; i < i1; ++i) {
    const int st = (i - i0) % kSearchStages;
    if (!wait_bar(smem_u32(&sh.full[st]), ((i - i0) / kSearchStages) & 1, guard, 1)) ok = false;
    if (!__syncthreads_and(ok)) break;
    const uint32_t tile = smem_u32(smem + st * kTileBytes);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(tile + swz<kSearchTile>(16 * warp + (mi & 1) * 8 + ri, 16 * ks + (mi >> 1) * 8), a);
      mma_bf16(acc, a, qb[ks][0], qb[ks][1]);
    }
    if (tig == 0) {   // column 0: keys 16w + gid (acc 0) and 16w + gid + 8 (acc 2)
      const int j = i * kSearchTile + 16 * warp + gid;
      if (j < ns) {
        sc[j] = acc[0] * sl2;
        lmax = fmaxf(lmax, acc[0] * sl2);
      }
      if (j + 8 < ns) {
        sc[j + 8] = acc[2] * sl2;
        lmax = fmaxf(lmax, acc[2] * sl2);
      }
    }
    __syncthreads();   // stage st is free again
    if (tid == 0 && issued < i1) issue(issued++);
  }
  if (tid == 0) {
    for (int i = (issued - i0 > kSearchStages ? issued - kSearchStages : i0); i < issued; ++i)
      drain_bar(smem_u32(&sh.full[(i - i0) % kSearchStages]), ((i - i0) / kSearchStages) & 1, kDrainLimitNs);
  }
  grid_dependents_launch();   // the next grid may take the SMs this one frees
  // a wait that ran out (status recorded) leaves this run without mass
  const bool good = __syncthreads_and(ok);
  const float cm = good ? block_max(lmax, sh.fbuf) : -INFINITY;
  __syncthreads();   // the scores of other threads are visible (global writes, same block)
  // this run's block masses on its own max: exp2 of the scores summed over the r
  // strides of each block
  float* mrow = mass + row * Nbm;
  for (int J = J0 + tid; J < J1; J += kDecThreads) {
    float m = 0.f;
    if (cm > -INFINITY) {
      const int j1 = min((J + 1) * r, ns);
      for (int j = J * r; j < j1; ++j) m += exp2f(sc[j] - cm);
    }
    mrow[J] = m;
  }
  if (tid == 0) cmax[row * SC + c] = cm;
  __threadfence();
  __syncthreads();
  if (tid == 0) sh.last = atomicAdd(arrive + row, 1u) == static_cast<unsigned>(SC - 1);
  __syncthreads();
  if (!sh.last) return;
  __threadfence();
  // the last CTA of the row: every run's masses on the row max, in the ring's
  // shared memory (every copy has landed)
  float* smass = reinterpret_cast<float*>(smem);
  uint32_t* swbits = reinterpret_cast<uint32_t*>(smem + kMaxBlocks * 4);
  float* scm = reinterpret_cast<float*>(smem + kMaxBlocks * 4 + kMaxBlocks / 8);
  // one round of loads (a load here waits behind the other CTAs' stream): the
  // runs' maxima and this thread's masses
  if (tid < SC) scm[tid] = __ldcg(cmax + row * SC + tid);
  float mv[kMaxPer];
#pragma unroll
  for (int e = 0; e < kMaxPer; ++e) {
    const int J = tid + e * kDecThreads;
    mv[e] = J < nb ? __ldcg(mrow + J) : 0.f;
  }
  __syncthreads();
  float M = -INFINITY;
  for (int k = 0; k < SC; ++k) M = fmaxf(M, scm[k]);
#pragma unroll
  for (int e = 0; e < kMaxPer; ++e) {
    const int J = tid + e * kDecThreads;
    if (J < nb) {
      const float ck = scm[J / bpc];
      smass[J] = ck > -INFINITY ? mv[e] * exp2f(ck - M) : 0.f;
    }
  }
  __syncthreads();

  if (group) {   // one mask per GQA group: the head's masses, normalised, for the group kernel
    float lsum = 0.f;
    for (int J = tid; J < nb; J += kDecThreads) lsum += smass[J];
    const float tot = block_sum<float>(lsum, sh.fbuf);
    const float inv = tot > 0.f ? 1.0f / tot : 0.f;
    for (int J = tid; J < nb; J += kDecThreads) mrow[J] = smass[J] * inv;
    return;
  }
  block_select(sh, smass, swbits, nb, Jt, tau, out, Nbm, obits, W, count + row, 1);
}

// One mask per GQA group (decode): the block masses of the group's g heads,
// written by the search kernels, summed in head order; the selection goes to
// every head of the group.  One CTA per (sequence, kv head).
__global__ void __launch_bounds__(kDecThreads) decode_group_select_kernel(const float* __restrict__ group_mass,
                                                                         const int32_t* __restrict__ lens, int Lmax,
                                                                         int H, int Hkv, int B, float tau,
                                                                         int32_t* __restrict__ count,
                                                                         int32_t* __restrict__ idx,
                                                                         uint32_t* __restrict__ bits, int Nbm, int W) {
  __shared__ DecSearchShared sh;
  __shared__ float smass[kMaxBlocks];
  __shared__ uint32_t swbits[kMaxBlocks / 32];
  const int tid = threadIdx.x;
  const int n = static_cast<int>(blockIdx.x) / Hkv, kvh = static_cast<int>(blockIdx.x) % Hkv;
  const int g = H / Hkv;
  const long long row0 = static_cast<long long>(n) * H + kvh * g;   // first head of the group
  const int len = __ldg(lens + n);
  if (len < 1 || len > Lmax) {   // the search recorded it; nothing selected
    if (tid < g) count[row0 + tid] = 0;
    for (int i = tid; i < g * W; i += kDecThreads) bits[row0 * W + i] = 0u;
    return;
  }
  const int Jt = (len - 1) / B, nb = Jt + 1;
  for (int J = tid; J < nb; J += kDecThreads) {
    float m = 0.f;
    for (int r = 0; r < g; ++r) m += group_mass[(row0 + r) * Nbm + J];
    smass[J] = m;
  }
  __syncthreads();
  block_select(sh, smass, swbits, nb, Jt, tau, idx + row0 * Nbm, Nbm, bits + row0 * W, W, count + row0, g);
}

// ------------------------------------------------------------------ attention
constexpr int kDecStages = 2;

template <int BN, int D>
struct DecAttnCfg {
  static constexpr int kTileBytes = BN * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;   // K and V
  static constexpr int kMergeLd = D / 2 + 4;            // merge rows: half of d, padded against bank conflicts
  static constexpr int kMergeBytes = (BN / 16) * 8 * kMergeLd * 4;
  static constexpr int kSmem = kDecStages * kStageBytes + kMergeBytes + 1024;
};

struct DecAttnCtrl {
  uint64_t full[kDecStages];
  uint64_t never;                          // fault injection: a barrier nothing arrives on
  int abort;
  float2 ml[kDecWarps][8];                 // warp partials: (max, sum) per head
  __nv_bfloat16 p[kDecWarps][8][24];       // per warp: P of its 16 keys, [head][key] (rows padded)
};

// The rows of one attention CTA's share [b0, b1) of the flattened space in which
// row (n, kvh) holds the causal key blocks 0 .. nbl_n - 1 of sequence n, rows
// n-major then kv head; rowstart is the exclusive prefix of nbl_n (a sequence
// of length outside [1, Lmax] has none).  A segment is the part [Ja, Jb) of one
// row inside the share.
struct SegWalk {
  const int32_t* rs;
  int Hkv;
  long long pos, b1;
  int n, kvh, Ja, Jb;
  __device__ __forceinline__ void load() {
    const long long base = static_cast<long long>(Hkv) * __ldcg(rs + n);
    const int nbl = __ldcg(rs + n + 1) - __ldcg(rs + n);
    const long long o = pos - base;
    kvh = static_cast<int>(o / nbl);
    Ja = static_cast<int>(o % nbl);
    const long long rend = base + static_cast<long long>(kvh + 1) * nbl;
    Jb = Ja + static_cast<int>((b1 < rend ? b1 : rend) - pos);
  }
  __device__ bool begin(const int32_t* rs_, int N, int Hkv_, long long b0, long long b1_) {
    rs = rs_;
    Hkv = Hkv_;
    pos = b0;
    b1 = b1_;
    if (pos >= b1) return false;
    // the last sequence whose rows start at or before b0 (it has blocks: b0 < total)
    int lo = 0, hi = N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<long long>(Hkv) * __ldcg(rs + mid) <= pos) lo = mid;
      else hi = mid - 1;
    }
    n = lo;
    load();
    return true;
  }
  __device__ bool next() {
    pos += Jb - Ja;
    if (pos >= b1) return false;
    if (pos == static_cast<long long>(Hkv) * __ldcg(rs + n + 1)) {   // the next sequence with blocks
      do ++n;
      while (__ldcg(rs + n + 1) == __ldcg(rs + n));
    }
    load();
    return true;
  }
};

// Bits of word w of a segment's blocks, and the union of the group's kept bits there.
__device__ __forceinline__ uint32_t seg_mask(const SegWalk& s, int w) {
  const int lo = max(s.Ja - 32 * w, 0), hi = min(s.Jb - 32 * w, 32);
  const uint32_t upto = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}
__device__ __forceinline__ uint32_t group_word(const uint32_t* __restrict__ bits, const SegWalk& s, int H, int g,
                                               int W, int w) {
  const uint32_t* b = bits + (static_cast<long long>(s.n) * H + s.kvh * g) * W + w;
  uint32_t u = 0u;
  for (int hh = 0; hh < g; ++hh) u |= __ldcg(b + static_cast<long long>(hh) * W);
  return u & seg_mask(s, w);
}

// The kept blocks of a CTA's share in order (the copy side's walk).
struct KeptWalk {
  SegWalk s;
  bool live;
  int w;
  uint32_t rem;
  __device__ void begin(const int32_t* rs, int N, int Hkv, long long b0, long long b1, const uint32_t* bits, int H,
                        int g, int W) {
    live = s.begin(rs, N, Hkv, b0, b1);
    if (live) {
      w = s.Ja >> 5;
      rem = group_word(bits, s, H, g, W, w);
    }
  }
  __device__ bool next(const uint32_t* bits, int H, int g, int W, int& n, int& J) {
    while (live) {
      if (rem) {
        J = 32 * w + __ffs(static_cast<int>(rem)) - 1;
        rem &= rem - 1u;
        n = s.n;
        return true;
      }
      if (++w <= (s.Jb - 1) >> 5) {
        rem = group_word(bits, s, H, g, W, w);
        continue;
      }
      live = s.next();
      if (live) {
        w = s.Ja >> 5;
        rem = group_word(bits, s, H, g, W, w);
      }
    }
    return false;
  }
};

// owner(x): the CTA whose share [c T / P, (c+1) T / P) holds flattened block x.
__device__ __forceinline__ int share_owner(long long x, long long T, int P) {
  return static_cast<int>(((x + 1) * P - 1) / T);
}
__device__ __forceinline__ long long share_start(int c, long long T, int P) {
  return static_cast<long long>(c) * T / P;
}

// grid P (one CTA per SM): CTA c walks its share [c T / P, (c+1) T / P) of the
// flattened (sequence, kv head, causal block) space, T = Hkv * rowstart[N].  Each
// kept block J of a row comes in once for the whole GQA group; the group's heads
// are the 8 columns of m16n8k16 tiles (heads beyond the group and heads that did
// not keep J are masked).  Warp w owns keys 16w..16w+15 of every block and keeps
// its own online softmax and O^T over them (a split over keys inside the CTA):
//   S^T [16 keys x heads] = K_J [16 keys x d] . Q^T [d x heads]
//   per head: running max and sum over the warp's keys, P (bf16) re-laid from
//   the accumulator fragment to the operand fragment through a small per-warp
//   buffer
//   O^T [d x heads] += V_J^T [d x 16 keys] . P^T [16 keys x heads]
// No cross-warp exchange per block: one barrier frees the stage.  At the end of
// each row segment the warp partials merge into the CTA's partial for the row,
// slot (row + c) of the workspace (row n Hkv + kvh; the slots of the (row, CTA)
// pairs that exist are distinct because rows and shares are both in order).
// Q^T stays in registers as B fragments; K comes in as A fragments by ldmatrix,
// V^T by ldmatrix.trans, both from the 128-byte swizzled TMA tiles.  The copies
// run ahead across rows.
template <int BN, int D>
__global__ void __launch_bounds__(kDecThreads, 1) decode_attn_kernel(
    const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lens, const int32_t* __restrict__ rowstart,
    const uint32_t* __restrict__ bits, int N, int Lmax, int H, int Hkv, int W, float sl2, float* __restrict__ part,
    unsigned int* status, uint64_t limit_ns, int inject_stall) {
  using C = DecAttnCfg<BN, D>;
  constexpr int kKeyWarps = BN / 16;  // warps that own keys (8 at B = 128, 4 at B = 64)
  constexpr int kDSteps = D / 16;     // k-steps of S (over d)
  constexpr int kOTiles = D / 16;     // d-row tiles of O^T
  constexpr int kLd = C::kMergeLd;
  __shared__ DecAttnCtrl ctl;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ow = reinterpret_cast<float*>(smem + kDecStages * C::kStageBytes);   // merge rows [warp][head][kLd]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;   // mma fragment coordinates
  const int P = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int g = H / Hkv;
  if (tid == 0) {
    for (int st = 0; st < kDecStages; ++st) mbar_init(smem_u32(&ctl.full[st]), 1);
    mbar_init(smem_u32(&ctl.never), 1);
    ctl.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
  }
  // the search's lists and block-count prefix (the grid ahead, launched so that
  // this one may start early) are read only past this point, through L2
  grid_dependency_wait();
  const long long T = static_cast<long long>(Hkv) * __ldcg(rowstart + N);
  const long long b0 = share_start(c, T, P), b1 = share_start(c + 1, T, P);
  if (b0 >= b1) return;
  __syncthreads();
  const Guard guard{&ctl.abort, status, limit_ns};

  // kept block number i of the share goes to stage i % kDecStages
  KeptWalk pk;   // thread 0's walk: the copies
  int issued = 0;
  auto issue_next = [&]() {
    int nn, J;
    if (!pk.next(bits, H, g, W, nn, J)) return;
    const int st = issued % kDecStages;
    const uint32_t fb = smem_u32(&ctl.full[st]);
    mbar_expect_tx(fb, C::kStageBytes);
    uint8_t* dst = smem + st * C::kStageBytes;
    const int r0 = nn * Lmax + J * BN;
    for (int a = 0; a < D / 64; ++a) {
      tma_load_3d(smem_u32(dst + a * BN * 128), &mk, fb, a * 64, pk.s.kvh, r0);
      tma_load_3d(smem_u32(dst + C::kTileBytes + a * BN * 128), &mv, fb, a * 64, pk.s.kvh, r0);
    }
    ++issued;
  };
  if (tid == 0) {
    pk.begin(rowstart, N, Hkv, b0, b1, bits, H, g, W);
    for (int i = 0; i < kDecStages; ++i) issue_next();
  }

  const int mi = lane >> 3, ri = lane & 7;   // ldmatrix: this lane's matrix and row
  bool ok = true;
  // Injected fault (tests only): thread 0 waits on a barrier that nothing arrives
  // on; the bounded wait gives up, and the CTA takes its abort path.
  if (inject_stall && tid == 0) ok = wait_bar(smem_u32(&ctl.never), 0, guard, 9);
  ok = __syncthreads_and(ok);
  int seq = 0;   // kept blocks consumed
  SegWalk cs;
  bool more = cs.begin(rowstart, N, Hkv, b0, b1);
  while (more) {
    const int n = cs.n, kvh = cs.kvh;
    const int t = __ldg(lens + n) - 1;
    // Q^T as B fragments: b0 = Q[head gid][16 ks + 2 tig, +1], b1 = the same at +8
    uint32_t qb[kDSteps][2];
    {
      const bool hv = gid < g;
      const __nv_bfloat16* qr = q + (static_cast<long long>(n) * H + kvh * g + (hv ? gid : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < kDSteps; ++ks) {
        qb[ks][0] = hv ? __ldg(reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * tig)) : 0u;
        qb[ks][1] = hv ? __ldg(reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * tig + 8)) : 0u;
      }
    }
    // This warp's running max and sum for the lane's two head columns (2 tig,
    // 2 tig + 1), and its O^T tiles (d rows 16 mt + gid and + 8, the same columns).
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o_acc[kOTiles][4];
#pragma unroll
    for (int mt = 0; mt < kOTiles; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o_acc[mt][e] = 0.f;
    const uint32_t* hrow = bits + (static_cast<long long>(n) * H + kvh * g) * W;
    for (int w = cs.Ja >> 5; ok && w <= (cs.Jb - 1) >> 5; ++w) {
      // the lane's two heads' kept bits in this word, and the group's union
      const uint32_t hb0 = 2 * tig < g ? __ldcg(hrow + static_cast<long long>(2 * tig) * W + w) : 0u;
      const uint32_t hb1 = 2 * tig + 1 < g ? __ldcg(hrow + static_cast<long long>(2 * tig + 1) * W + w) : 0u;
      uint32_t rem = group_word(bits, cs, H, g, W, w);
      while (rem) {
        const int jw = __ffs(static_cast<int>(rem)) - 1;
        rem &= rem - 1u;
        const int J = 32 * w + jw;
        const int st = seq % kDecStages;
        if (!wait_bar(smem_u32(&ctl.full[st]), (seq / kDecStages) & 1, guard, 1)) ok = false;
        if (!__syncthreads_and(ok)) {
          ok = false;
          break;
        }
        if (warp < kKeyWarps) {
          const uint32_t ks_base = smem_u32(smem + st * C::kStageBytes);
          const uint32_t vs_base = ks_base + C::kTileBytes;
          const bool keep0 = (hb0 >> jw) & 1u, keep1 = (hb1 >> jw) & 1u;
          // S^T tile: keys 16w + gid (acc 0, 1) and 16w + gid + 8 (acc 2, 3)
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < kDSteps; ++ks) {
            uint32_t a[4];
            ldsm_x4(ks_base + swz<BN>(16 * warp + (mi & 1) * 8 + ri, 16 * ks + (mi >> 1) * 8), a);
            mma_bf16(acc, a, qb[ks][0], qb[ks][1]);
          }
          const int key0 = J * BN + 16 * warp + gid;
          const bool v0 = key0 <= t, v1 = key0 + 8 <= t;
          const float s0 = (keep0 && v0) ? acc[0] * sl2 : -INFINITY;
          const float s1 = (keep1 && v0) ? acc[1] * sl2 : -INFINITY;
          const float s2 = (keep0 && v1) ? acc[2] * sl2 : -INFINITY;
          const float s3 = (keep1 && v1) ? acc[3] * sl2 : -INFINITY;
          // per head column: max over the warp's 16 keys
          float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
          for (int x = 4; x < 32; x <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, x));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, x));
          }
          const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
          // a column with nothing so far and nothing now keeps alpha 1 (its O is 0)
          const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m_run[0] - mn0);
          const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m_run[1] - mn1);
          const __nv_bfloat16 p0 = __float2bfloat16(s0 == -INFINITY ? 0.f : exp2f(s0 - mn0));
          const __nv_bfloat16 p1 = __float2bfloat16(s1 == -INFINITY ? 0.f : exp2f(s1 - mn1));
          const __nv_bfloat16 p2 = __float2bfloat16(s2 == -INFINITY ? 0.f : exp2f(s2 - mn0));
          const __nv_bfloat16 p3 = __float2bfloat16(s3 == -INFINITY ? 0.f : exp2f(s3 - mn1));
          // sums of the bf16 P that P V uses
          float sm0 = __bfloat162float(p0) + __bfloat162float(p2), sm1 = __bfloat162float(p1) + __bfloat162float(p3);
#pragma unroll
          for (int x = 4; x < 32; x <<= 1) {
            sm0 += __shfl_xor_sync(0xffffffffu, sm0, x);
            sm1 += __shfl_xor_sync(0xffffffffu, sm1, x);
          }
          l_run[0] = l_run[0] * al0 + sm0;
          l_run[1] = l_run[1] * al1 + sm1;
          m_run[0] = mn0;
          m_run[1] = mn1;
          // P from the accumulator layout (key rows, head columns) to the operand
          // layout (b0 = P[head gid][keys 2 tig, +1], b1 = keys + 8)
          __nv_bfloat16(*pw)[24] = ctl.p[warp];
          pw[2 * tig][gid] = p0;
          pw[2 * tig + 1][gid] = p1;
          pw[2 * tig][gid + 8] = p2;
          pw[2 * tig + 1][gid + 8] = p3;
          __syncwarp();
          const uint32_t pb0 = *reinterpret_cast<const uint32_t*>(&pw[gid][2 * tig]);
          const uint32_t pb1 = *reinterpret_cast<const uint32_t*>(&pw[gid][2 * tig + 8]);
          __syncwarp();
#pragma unroll
          for (int mt = 0; mt < kOTiles; ++mt) {
            o_acc[mt][0] *= al0;
            o_acc[mt][1] *= al1;
            o_acc[mt][2] *= al0;
            o_acc[mt][3] *= al1;
            uint32_t a[4];
            ldsm_x4_t(vs_base + swz<BN>(16 * warp + (mi >> 1) * 8 + ri, 16 * mt + (mi & 1) * 8), a);
            mma_bf16(o_acc[mt], a, pb0, pb1);
          }
        }
        __syncthreads();   // stage st is free again
        if (tid == 0) issue_next();
        ++seq;
      }
    }
    // the row's partial from this CTA: the warp partials merged (nothing after a
    // wait that ran out)
    const long long prow = (static_cast<long long>(n) * Hkv + kvh + c) * g;
    if (warp < kKeyWarps && gid == 0) {
      ctl.ml[warp][2 * tig] = make_float2(m_run[0], l_run[0]);
      ctl.ml[warp][2 * tig + 1] = make_float2(m_run[1], l_run[1]);
    }
    __syncthreads();
    const int hh = warp;   // one warp per head of the group
    float f[kKeyWarps];
    bool has = false;
    if (hh < g) {
      float Mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kKeyWarps; ++w) Mx = fmaxf(Mx, ctl.ml[w][hh].x);
      has = ok && Mx > -INFINITY;
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < kKeyWarps; ++w) {
        const float2 ml = ctl.ml[w][hh];
        f[w] = (has && ml.x > -INFINITY) ? exp2f(ml.x - Mx) : 0.f;
        L += ml.y * f[w];
      }
      if (lane == 0) {
        part[(prow + hh) * (D + 2)] = has ? Mx : -INFINITY;
        part[(prow + hh) * (D + 2) + 1] = has ? L : 0.f;
      }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {   // the two halves of d in turn through the merge rows
      if (warp < kKeyWarps) {
#pragma unroll
        for (int mt = hf * kOTiles / 2; mt < (hf + 1) * kOTiles / 2; ++mt) {
          const int d0 = 16 * mt + gid - hf * (D / 2);
          ow[(warp * 8 + 2 * tig) * kLd + d0] = o_acc[mt][0];
          ow[(warp * 8 + 2 * tig + 1) * kLd + d0] = o_acc[mt][1];
          ow[(warp * 8 + 2 * tig) * kLd + d0 + 8] = o_acc[mt][2];
          ow[(warp * 8 + 2 * tig + 1) * kLd + d0 + 8] = o_acc[mt][3];
        }
      }
      __syncthreads();
      if (hh < g) {
        for (int d = lane; d < D / 2; d += 32) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < kKeyWarps; ++w) acc += ow[(w * 8 + hh) * kLd + d] * f[w];
          part[(prow + hh) * (D + 2) + 2 + hf * (D / 2) + d] = has ? acc : 0.f;
        }
      }
      __syncthreads();
    }
    more = cs.next();
  }
  grid_dependents_launch();
  // copies still in flight land before the CTA exits (only after a wait ran out
  // can any be left)
  if (tid == 0) {
    for (int i = max(seq, issued - kDecStages); i < issued; ++i)
      drain_bar(smem_u32(&ctl.full[i % kDecStages]), (i / kDecStages) & 1, kDrainLimitNs);
  }
}

// The partials of the attention CTAs whose shares met row (n, kvh) merged into
// the output of the group's g heads: O = sum_c o_c 2^(m_c - M) / sum_c l_c
// 2^(m_c - M), M the largest m_c.  One CTA per row.  The row's g * D outputs are
// split into runs of 4 adjacent columns over nthr = g * D / 4 threads; the
// CTA's 256 threads form 256 / nthr groups (1 to 16) that merge disjoint runs
// of the row's partials, each run's loads (up to 16 partials) in flight at
// once; the groups' (max, sum, output) states combine through shared memory.
// A sequence with no blocks (a length outside [1, Lmax]) gets a zero output.
template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(const float* __restrict__ part,
                                                                    const int32_t* __restrict__ rowstart, int N,
                                                                    int H, int Hkv, int P,
                                                                    __nv_bfloat16* __restrict__ o) {
  constexpr int kBatch = 16;
  __shared__ float4 gs[2 * kDecThreads];   // per group and thread: (max, sum, o0, o1) and (o2, o3)
  const int tid = threadIdx.x;
  const long long r = blockIdx.x;
  const int n = static_cast<int>(r / Hkv), kvh = static_cast<int>(r % Hkv);
  const int g = H / Hkv;
  const int nthr = g * D / 4, groups = kDecThreads / nthr;
  const int grp = tid / nthr, e0 = 4 * (tid % nthr);
  const int hm = e0 / D, col = e0 % D;
  // the attention's partials (the grid ahead, launched so that this one may
  // start early) are read only past this point, through L2
  grid_dependency_wait();
  const int nbl = __ldcg(rowstart + n + 1) - __ldcg(rowstart + n);
  float Mx = -INFINITY, L = 0.f, O[4] = {0.f, 0.f, 0.f, 0.f};
  if (nbl > 0) {
    const long long T = static_cast<long long>(Hkv) * __ldcg(rowstart + N);
    const long long s0 = static_cast<long long>(Hkv) * __ldcg(rowstart + n) + static_cast<long long>(kvh) * nbl;
    const int clo = share_owner(s0, T, P), chi = share_owner(s0 + nbl - 1, T, P);
    const int per = (chi - clo + 1 + groups - 1) / groups;
    const int g0 = clo + grp * per, g1 = min(g0 + per, chi + 1);
    const float* pr = part + (r * g + hm) * (D + 2);   // + c g (D + 2) for CTA c
    const long long cs_stride = static_cast<long long>(g) * (D + 2);
    // with T >= P every share holds a block (and the 64-bit divisions of the
    // test stay out of the loop); otherwise an empty share wrote nothing
    const bool all_full = T >= P;
    for (int base = g0; base < g1; base += kBatch) {
      float mk[kBatch], lk[kBatch];
      float2 ok[kBatch][2];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int cc = base + u;
        const bool use = cc < g1 && (all_full || share_start(cc, T, P) != share_start(cc + 1, T, P));
        const float* pc = pr + static_cast<long long>(use ? cc : clo) * cs_stride;
        mk[u] = __ldcg(pc);
        lk[u] = __ldcg(pc + 1);
        ok[u][0] = __ldcg(reinterpret_cast<const float2*>(pc + 2 + col));
        ok[u][1] = __ldcg(reinterpret_cast<const float2*>(pc + 4 + col));
        if (!use) mk[u] = -INFINITY;
      }
      float bm = Mx;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) bm = fmaxf(bm, mk[u]);
      if (bm == -INFINITY) continue;
      const float a = Mx == -INFINITY ? 0.f : exp2f(Mx - bm);
      L *= a;
#pragma unroll
      for (int k = 0; k < 4; ++k) O[k] *= a;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float f = mk[u] == -INFINITY ? 0.f : exp2f(mk[u] - bm);
        L += lk[u] * f;
        O[0] += ok[u][0].x * f;
        O[1] += ok[u][0].y * f;
        O[2] += ok[u][1].x * f;
        O[3] += ok[u][1].y * f;
      }
      Mx = bm;
    }
  }
  if (grp < groups) {
    gs[grp * nthr + tid % nthr] = make_float4(Mx, L, O[0], O[1]);
    gs[kDecThreads + grp * nthr + tid % nthr] = make_float4(O[2], O[3], 0.f, 0.f);
  }
  __syncthreads();
  if (tid < nthr) {
    float M = -INFINITY;
    for (int k = 0; k < groups; ++k) M = fmaxf(M, gs[k * nthr + tid].x);
    float Ls = 0.f, A[4] = {0.f, 0.f, 0.f, 0.f};
    if (M > -INFINITY) {
      for (int k = 0; k < groups; ++k) {
        const float4 st = gs[k * nthr + tid], s2 = gs[kDecThreads + k * nthr + tid];
        const float f = st.x == -INFINITY ? 0.f : exp2f(st.x - M);
        Ls += st.y * f;
        A[0] += st.z * f;
        A[1] += st.w * f;
        A[2] += s2.x * f;
        A[3] += s2.y * f;
      }
    }
    const float inv = Ls > 0.f ? 1.0f / Ls : 0.f;
    __nv_bfloat16* orow = o + (static_cast<long long>(n) * H + kvh * g + hm) * D + col;
    *reinterpret_cast<__nv_bfloat162*>(orow) = __floats2bfloat162_rn(A[0] * inv, A[1] * inv);
    *reinterpret_cast<__nv_bfloat162*>(orow + 2) = __floats2bfloat162_rn(A[2] * inv, A[3] * inv);
  }
}

template <int BN, int D>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const int32_t* lens, int N, int Lmax, int H,
                            int Hkv, int S, float tau, bool gqa, int32_t* count, int32_t* idx, void* o,
                            const DecodeScratch& w, const DeviceGuardArgs& g, cudaStream_t stream) {
  const int Nbm = Lmax / BN, W = (Nbm + 31) / 32;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  CUtensorMap mks, mk, mv;
  const uint64_t rows = static_cast<uint64_t>(N) * Lmax;
  if (!make_tmap_sampled(&mks, k, rows, Hkv, D, S, kSearchTile) || !make_tmap_rows(&mk, k, rows, Hkv, D, BN) ||
      !make_tmap_rows(&mv, v, rows, Hkv, D, BN))
    return cudaErrorInvalidValue;
  constexpr int kSearchSmem = kSearchStages * kSearchTile * D * 2 + 1024;
  static std::atomic<uint64_t> search_smem_set{0};
  if ((e = set_smem_limit_once(decode_search_kernel<D>, kSearchSmem, search_smem_set)) != cudaSuccess) return e;
  static std::atomic<int> search_occ{0};   // resident search CTAs per SM
  int occ = search_occ.load(std::memory_order_relaxed);
  if (occ == 0) {
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_search_kernel<D>, kDecThreads, kSearchSmem)) !=
        cudaSuccess)
      return e;
    occ = std::max(occ, 1);
    search_occ.store(occ, std::memory_order_relaxed);
  }
  // search: as many CTAs per row as keep the whole grid resident at once
  const int Ns_max = Lmax / S, nt_max = (Ns_max + kSearchTile - 1) / kSearchTile;
  const long long NH = static_cast<long long>(N) * H;
  int SC = static_cast<int>(std::min<long long>(static_cast<long long>(occ) * sms / NH, kDecSearchChunks));
  SC = std::max(1, std::min(SC, nt_max));
  const int tpc = (nt_max + SC - 1) / SC;
  SC = (nt_max + tpc - 1) / tpc;
  decode_search_kernel<D><<<dim3(static_cast<unsigned>(NH), SC), kDecThreads, kSearchSmem, stream>>>(
      mks, static_cast<const __nv_bfloat16*>(q), lens, N, Lmax, H, Hkv, BN, S, sl2, tau, tpc, w.scores, Ns_max, w.cmax,
      w.arrive, w.mass, gqa ? 1 : 0, count, idx, w.bits, Nbm, W, w.rowstart, g.status, g.limit_ns);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (gqa) {
    decode_group_select_kernel<<<static_cast<unsigned>(N) * Hkv, kDecThreads, 0, stream>>>(
        w.mass, lens, Lmax, H, Hkv, BN, tau, count, idx, w.bits, Nbm, W);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  using C = DecAttnCfg<BN, D>;
  static std::atomic<uint64_t> smem_set{0};
  if ((e = set_smem_limit_once(decode_attn_kernel<BN, D>, C::kSmem, smem_set)) != cudaSuccess) return e;
  const int P = std::max(1, std::min(sms, kDecAttnCTAs));
  // attention and combine may start while the grid ahead finishes (programmatic
  // dependent launch); each waits for it before reading what it wrote
  cudaLaunchAttribute early[1];
  early[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  early[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(P);
  lc.blockDim = dim3(kDecThreads);
  lc.dynamicSmemBytes = C::kSmem;
  lc.stream = stream;
  lc.attrs = early;
  lc.numAttrs = 1;
  // RR_DEBUG_STALL_WAIT=1 injects a wait that never completes (tests of the
  // bounded-wait path); unset in normal use.
  const char* inj = getenv("RR_DEBUG_STALL_WAIT");
  const int inject = (inj && inj[0] == '1') ? 1 : 0;
  if ((e = cudaLaunchKernelEx(&lc, decode_attn_kernel<BN, D>, mk, mv, static_cast<const __nv_bfloat16*>(q), lens,
                              static_cast<const int32_t*>(w.rowstart), static_cast<const uint32_t*>(w.bits), N, Lmax,
                              H, Hkv, W, sl2, w.part, g.status, g.limit_ns, inject)) != cudaSuccess)
    return e;
  lc.gridDim = dim3(static_cast<unsigned>(N) * Hkv);
  lc.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&lc, decode_combine_kernel<D>, static_cast<const float*>(w.part),
                            static_cast<const int32_t*>(w.rowstart), N, H, Hkv, P, static_cast<__nv_bfloat16*>(o));
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const int32_t* lens, int N, int Lmax, int H,
                          int Hkv, int d, int B, int S, float tau, bool gqa, int32_t* count, int32_t* idx, void* o,
                          const DecodeScratch& w, const DeviceGuardArgs& g, cudaStream_t stream) {
  if (B == 128 && d == 128) return launch_decode_t<128, 128>(q, k, v, lens, N, Lmax, H, Hkv, S, tau, gqa, count, idx, o, w, g, stream);
  if (B == 128 && d == 64) return launch_decode_t<128, 64>(q, k, v, lens, N, Lmax, H, Hkv, S, tau, gqa, count, idx, o, w, g, stream);
  if (B == 64 && d == 128) return launch_decode_t<64, 128>(q, k, v, lens, N, Lmax, H, Hkv, S, tau, gqa, count, idx, o, w, g, stream);
  if (B == 64 && d == 64) return launch_decode_t<64, 64>(q, k, v, lens, N, Lmax, H, Hkv, S, tau, gqa, count, idx, o, w, g, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rr
