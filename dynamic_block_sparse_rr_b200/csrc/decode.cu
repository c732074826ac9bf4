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
//   decode_search_kernel   one CTA per (sequence, head): the head's sampled key
//                          rows come in as 128-row TMA tiles of a zero-copy
//                          strided view (two-stage ring), scores to the
//                          workspace, block mass in shared memory, Top-tau by
//                          bisection over the
//                          mass bits with block-wide sums of fixed-point units
//                          (the prefill rule), list and a bitmap of the kept
//                          blocks out;
//   decode_attn_kernel     one CTA per (sequence, kv head, 16 key blocks): a
//                          kept block's K and V tiles come in once by TMA
//                          (three-stage ring) for every query head of the GQA
//                          group that kept it.  The group's <= 8 heads are the 8
//                          columns of m16n8k16 tensor-core tiles (mma.sync), so
//                          the two small contractions per block (scores of 128
//                          keys, P V) are a few instructions per warp; each warp
//                          keeps an online softmax over its 16 keys of every
//                          block, and the warps' partials merge into the
//                          chunk's partial (max, sum, output);
//   decode_combine_kernel  one CTA per (sequence, head): the partials merged.
#include <cuda_bf16.h>
#include <math.h>

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

// Byte offset of element (row, c) of a 128-row TMA tile (128-byte swizzle, D/64
// column blocks of 128 rows x 128 bytes); c a multiple of 8.
__device__ __forceinline__ uint32_t swz128(int row, int c) {
  return static_cast<uint32_t>((c >> 6) * (128 * 128) + row * 128 + ((((c & 63) >> 3) ^ (row & 7)) << 4));
}

struct DecSearchShared {
  uint64_t full[kSearchStages];
  int abort;
  float mass[kMaxBlocks];
  double dbuf[kDecWarps];
  float fbuf[kDecWarps];
  uint32_t ubuf[kDecWarps];
  uint32_t bits[kMaxBlocks / 32];
};

// Top-tau over the nb = Jt + 1 block masses in sh.mass, as in prefill (fixed-point
// units of the row total, the threshold by bisection over the mass bits with
// block-wide sums, equal masses to the lower J), plus the current block Jt.
// The ascending list goes to rep consecutive rows of out (row stride
// out_stride), the bitmap to rep consecutive rows of obits (W words each), the
// count to count[0 .. rep).  Called by every thread of the CTA.
__device__ __noinline__ void block_select(DecSearchShared& sh, int nb, int Jt, float tau, int32_t* out,
                                          long long out_stride, uint32_t* obits, int W, int32_t* count, int rep) {
  const int tid = threadIdx.x;
  for (int w = tid; w < (nb + 31) / 32; w += kDecThreads) sh.bits[w] = 0u;
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
      const float v = sh.mass[c0 + e];
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
      // the largest mass T whose masses at or above it still reach the target
      uint32_t P = 0;
      for (int b = 30; b >= 0; --b) {
        const uint32_t cand = P | (1u << b);
        uint32_t sge = 0;
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) sge += key[e] >= cand ? un[e] : 0u;
        if (block_sum<uint32_t>(sge, sh.ubuf) >= target) P = cand;
      }
      const uint32_t T = P;
      uint32_t sgt = 0, my_eq = 0;
#pragma unroll
      for (int e = 0; e < kMaxPer; ++e) {
        sgt += key[e] > T ? un[e] : 0u;
        my_eq += (c0 + e < c1 && key[e] == T) ? 1u : 0u;
      }
      const uint32_t sum_gt = block_sum<uint32_t>(sgt, sh.ubuf);
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
      atomicOr(&sh.bits[(c0 + e) >> 5], 1u << ((c0 + e) & 31));
    }
  }
  __syncthreads();
  for (int r = 0; r < rep; ++r)
    for (int w = tid; w < W; w += kDecThreads) obits[r * W + w] = w < (nb + 31) / 32 ? sh.bits[w] : 0u;
  if (tid < rep) count[tid] = static_cast<int32_t>(cnt);
}


template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_search_kernel(
    const __grid_constant__ CUtensorMap mks, const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lens,
    int Lmax, int H, int Hkv, int B, int S, float sl2, float tau, float* __restrict__ scores, int Ns_max,
    int32_t* __restrict__ count, int32_t* __restrict__ idx, uint32_t* __restrict__ bits, int Nbm, int W,
    float* __restrict__ group_mass, unsigned int* status, uint64_t limit_ns) {
  constexpr int kTileBytes = kSearchTile * D * 2;
  __shared__ DecSearchShared sh;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int n = static_cast<int>(blockIdx.x) / H, h = static_cast<int>(blockIdx.x) % H;
  const int kvh = h / (H / Hkv);
  const long long row = static_cast<long long>(n) * H + h;
  int32_t* out = idx + row * Nbm;
  uint32_t* obits = bits + row * W;
  const int len = __ldg(lens + n);
  if (len < 1 || len > Lmax) {   // not a cache length this call can serve: nothing selected
    if (tid == 0) {
      count[row] = 0;
      atomicCAS(status, 0u, kStatusLenCode | (static_cast<unsigned>(n < (1 << 24) ? n : (1 << 24) - 1) << 8));
    }
    for (int w = tid; w < W; w += kDecThreads) obits[w] = 0u;
    return;
  }
  const int t = len - 1, Jt = t / B, nb = Jt + 1, off = h % S, r = B / S;
  const int ns = t >= off ? (t - off) / S + 1 : 0;   // sampled keys at or before t
  const int nt = (ns + kSearchTile - 1) / kSearchTile;
  if (tid == 0) {
    for (int st = 0; st < kSearchStages; ++st) mbar_init(smem_u32(&sh.full[st]), 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  // lanes 2k and 2k+1 score key k of a tile, each over half of d; the half of
  // q they need stays in registers
  const int kr = tid >> 1, half = tid & 1;
  float qr[D / 2];
#pragma unroll
  for (int c = 0; c < D / 2; c += 2) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + row * D + half * (D / 2) + c));
    qr[c] = f.x * sl2;
    qr[c + 1] = f.y * sl2;
  }
  __syncthreads();
  const Guard guard{&sh.abort, status, limit_ns};
  // tile i: the sampled keys of strides 128 i .. 128 i + 127 of sequence n
  auto issue = [&](int i) {
    const int st = i % kSearchStages;
    const uint32_t fb = smem_u32(&sh.full[st]);
    mbar_expect_tx(fb, kTileBytes);
    uint8_t* dst = smem + st * kTileBytes;
    for (int a = 0; a < D / 64; ++a)
      tma_load_4d(smem_u32(dst + a * kSearchTile * 128), &mks, fb, a * 64, kvh, off,
                  n * (Lmax / S) + i * kSearchTile);
  };
  int issued = 0;
  if (tid == 0) {
    tma_prefetch_desc(&mks);
    for (; issued < nt && issued < kSearchStages; ++issued) issue(issued);
  }
  // scores (log2 units) of the sampled keys, to the workspace row
  float* sc = scores + row * Ns_max;
  float lmax = -INFINITY;
  bool ok = true;
  for (int i = 0; i < nt; ++i) {
    const int st = i % kSearchStages;
    if (!wait_bar(smem_u32(&sh.full[st]), (i / kSearchStages) & 1, guard, 1)) ok = false;
    if (!__syncthreads_and(ok)) break;
    const uint8_t* tile = smem + st * kTileBytes;
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int c = 0; c < D / 2; c += 8) {
      const uint4 v4 = *reinterpret_cast<const uint4*>(tile + swz128(kr, half * (D / 2) + c));
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p2[e]);
        acc0 = fmaf(f.x, qr[c + 2 * e], acc0);
        acc1 = fmaf(f.y, qr[c + 2 * e + 1], acc1);
      }
    }
    float sv = acc0 + acc1;
    sv += __shfl_xor_sync(0xffffffffu, sv, 1);
    const int j = i * kSearchTile + kr;
    if (j < ns) {
      if (half == 0) sc[j] = sv;
      lmax = fmaxf(lmax, sv);
    }
    __syncthreads();   // stage st is free again
    if (tid == 0 && issued < nt) issue(issued++);
  }
  if (tid == 0) {
    for (int i = (issued > kSearchStages ? issued - kSearchStages : 0); i < issued; ++i)
      drain_bar(smem_u32(&sh.full[i % kSearchStages]), (i / kSearchStages) & 1, kDrainLimitNs);
  }
  if (!__syncthreads_and(ok)) {   // a wait ran out (status recorded): nothing selected
    if (tid == 0) count[row] = 0;
    for (int w = tid; w < W; w += kDecThreads) obits[w] = 0u;
    return;
  }
  const float mx = block_max(lmax, sh.fbuf);
  __syncthreads();   // the scores of other threads are visible (global writes, same block)
  // block mass: exp2 of the scores summed over the r strides of each block
  for (int J = tid; J < nb; J += kDecThreads) {
    float m = 0.f;
    const int j1 = min((J + 1) * r, ns);
    for (int j = J * r; j < j1; ++j) m += exp2f(sc[j] - mx);
    sh.mass[J] = m;
  }
  __syncthreads();

  if (group_mass) {   // one mask per GQA group: the head's masses, normalised, for the group kernel
    float lsum = 0.f;
    for (int J = tid; J < nb; J += kDecThreads) lsum += sh.mass[J];
    const float tot = block_sum<float>(lsum, sh.fbuf);
    const float inv = tot > 0.f ? 1.0f / tot : 0.f;
    float* mrow = group_mass + row * Nbm;
    for (int J = tid; J < nb; J += kDecThreads) mrow[J] = sh.mass[J] * inv;
    return;
  }
  block_select(sh, nb, Jt, tau, out, Nbm, obits, W, count + row, 1);
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
    sh.mass[J] = m;
  }
  __syncthreads();
  block_select(sh, nb, Jt, tau, idx + row0 * Nbm, Nbm, bits + row0 * W, W, count + row0, g);
}

// ------------------------------------------------------------------ attention
constexpr int kDecChunk = 16;   // key blocks per attention CTA (half a bitmap word)
constexpr int kDecStages = 3;

template <int BN, int D>
struct DecAttnCfg {
  static constexpr int kTileBytes = BN * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;   // K and V
  static constexpr int kSmem = kDecStages * kStageBytes + 1024;
  static_assert(kDecWarps * 8 * D * 4 <= kStageBytes, "the warp partials fit in one stage");
};

struct DecAttnCtrl {
  uint64_t full[kDecStages];
  int abort;
  uint32_t hbits[8];
  float2 ml[kDecWarps][8];                 // warp partials: (max, sum) per head
  __nv_bfloat16 p[kDecWarps][8][24];       // per warp: P of its 16 keys, [head][key] (rows padded)
};

// Position of the (i+1)-th set bit of `set` (i < popcount).
__device__ __forceinline__ int nth_bit(uint32_t set, int i) {
  for (int k = 0; k < i; ++k) set &= set - 1u;
  return __ffs(static_cast<int>(set)) - 1;
}

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

// One CTA per (sequence n, kv head, 16 key blocks).  Each kept block J comes in
// once for the whole GQA group; the group's heads are the 8 columns of
// m16n8k16 tiles (heads beyond the group and heads that did not keep J are
// masked).  Warp w owns keys 16w..16w+15 of every block and keeps its own
// online softmax and O^T over them (a split over keys inside the CTA):
//   S^T [16 keys x heads] = K_J [16 keys x d] . Q^T [d x heads]
//   per head: running max and sum over the warp's keys, P (bf16) re-laid from
//   the accumulator fragment to the operand fragment through a small per-warp
//   buffer
//   O^T [d x heads] += V_J^T [d x 16 keys] . P^T [16 keys x heads]
// No cross-warp exchange per block: one barrier frees the stage.  At the end the
// eight warp partials are merged into the chunk's partial.  Q^T stays in
// registers as B fragments; K comes in as A fragments by ldmatrix, V^T by
// ldmatrix.trans, both from the 128-byte swizzled TMA tiles.
template <int BN, int D>
__global__ void __launch_bounds__(kDecThreads, 1) decode_attn_kernel(
    const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ lens, const uint32_t* __restrict__ bits,
    int Lmax, int H, int Hkv, int W, int NC, float sl2, float* __restrict__ part, unsigned int* status,
    uint64_t limit_ns) {
  using C = DecAttnCfg<BN, D>;
  constexpr int kKeyWarps = BN / 16;  // warps that own keys (8 at B = 128, 4 at B = 64)
  constexpr int kDSteps = D / 16;     // k-steps of S (over d)
  constexpr int kOTiles = D / 16;     // d-row tiles of O^T
  __shared__ DecAttnCtrl ctl;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;   // mma fragment coordinates
  const int chunk = static_cast<int>(blockIdx.x), kvh = static_cast<int>(blockIdx.y), n = static_cast<int>(blockIdx.z);
  const int g = H / Hkv;
  const int len = __ldg(lens + n);
  const int t = len - 1;
  const int J0 = chunk * kDecChunk;
  const bool live = len >= 1 && len <= Lmax && J0 <= t / BN;
  if (tid < 8) {
    uint32_t b = 0u;
    if (live && tid < g) b = __ldg(bits + (static_cast<long long>(n) * H + kvh * g + tid) * W + (J0 >> 5));
    ctl.hbits[tid] = (b >> (J0 & 31)) & ((1u << kDecChunk) - 1u);
  }
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(smem_u32(&ctl.full[s]), 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
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
  __syncthreads();
  uint32_t any = 0;
  for (int hh = 0; hh < g; ++hh) any |= ctl.hbits[hh];
  const Guard guard{&ctl.abort, status, limit_ns};

  // the chunk's kept blocks, ascending; block i of the sequence goes to stage i % kDecStages
  auto issue = [&](int i) {
    const int J = J0 + nth_bit(any, i);
    const int st = i % kDecStages;
    const uint32_t fb = smem_u32(&ctl.full[st]);
    mbar_expect_tx(fb, C::kStageBytes);
    uint8_t* dst = smem + st * C::kStageBytes;
    const int r0 = n * Lmax + J * BN;
    for (int a = 0; a < D / 64; ++a) {
      tma_load_3d(smem_u32(dst + a * BN * 128), &mk, fb, a * 64, kvh, r0);
      tma_load_3d(smem_u32(dst + C::kTileBytes + a * BN * 128), &mv, fb, a * 64, kvh, r0);
    }
  };
  const int n_blk = __popc(any);
  int issued = 0;   // thread 0: copies issued so far
  if (tid == 0) {
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
    for (; issued < n_blk && issued < kDecStages; ++issued) issue(issued);
  }

  // This warp's running max and sum for the lane's two head columns (2 tig,
  // 2 tig + 1), and its O^T tiles (d rows 16 mt + gid and + 8, the same columns).
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o_acc[kOTiles][4];
#pragma unroll
  for (int mt = 0; mt < kOTiles; ++mt)
#pragma unroll
    for (int c = 0; c < 4; ++c) o_acc[mt][c] = 0.f;
  const int mi = lane >> 3, ri = lane & 7;   // ldmatrix: this lane's matrix and row
  bool ok = true;
  for (int i = 0; i < n_blk; ++i) {
    const int J = J0 + nth_bit(any, i);
    const uint32_t jb = 1u << (J - J0);
    const int st = i % kDecStages;
    if (!wait_bar(smem_u32(&ctl.full[st]), (i / kDecStages) & 1, guard, 1)) ok = false;
    if (!__syncthreads_and(ok)) break;
    if (warp < kKeyWarps) {
      const uint32_t ks_base = smem_u32(smem + st * C::kStageBytes);
      const uint32_t vs_base = ks_base + C::kTileBytes;
      const bool keep0 = 2 * tig < g && (ctl.hbits[2 * tig] & jb);
      const bool keep1 = 2 * tig + 1 < g && (ctl.hbits[2 * tig + 1] & jb);
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
      const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&pw[gid][2 * tig]);
      const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&pw[gid][2 * tig + 8]);
      __syncwarp();
#pragma unroll
      for (int mt = 0; mt < kOTiles; ++mt) {
        o_acc[mt][0] *= al0;
        o_acc[mt][1] *= al1;
        o_acc[mt][2] *= al0;
        o_acc[mt][3] *= al1;
        uint32_t a[4];
        ldsm_x4_t(vs_base + swz<BN>(16 * warp + (mi >> 1) * 8 + ri, 16 * mt + (mi & 1) * 8), a);
        mma_bf16(o_acc[mt], a, b0, b1);
      }
    }
    __syncthreads();   // stage st is free again
    if (tid == 0 && issued < n_blk) issue(issued++);
  }
  // in-flight copies land before the CTA exits (only after an abort can any be left)
  if (tid == 0) {
    for (int i = (issued > kDecStages ? issued - kDecStages : 0); i < issued; ++i)
      drain_bar(smem_u32(&ctl.full[i % kDecStages]), (i / kDecStages) & 1, kDrainLimitNs);
  }
  const bool done = __syncthreads_and(ok) && live;
  // merge the warp partials: stage 0 holds each warp's O^T as [warp][head][d] fp32
  float* ow = reinterpret_cast<float*>(smem);
  if (warp < kKeyWarps) {
    if (gid == 0) {
      ctl.ml[warp][2 * tig] = make_float2(m_run[0], l_run[0]);
      ctl.ml[warp][2 * tig + 1] = make_float2(m_run[1], l_run[1]);
    }
#pragma unroll
    for (int mt = 0; mt < kOTiles; ++mt) {
      const int d0 = 16 * mt + gid;
      ow[(warp * 8 + 2 * tig) * D + d0] = o_acc[mt][0];
      ow[(warp * 8 + 2 * tig + 1) * D + d0] = o_acc[mt][1];
      ow[(warp * 8 + 2 * tig) * D + d0 + 8] = o_acc[mt][2];
      ow[(warp * 8 + 2 * tig + 1) * D + d0 + 8] = o_acc[mt][3];
    }
  }
  __syncthreads();
  // thread layout: head hh = tid / 32 (one warp per head), d columns lane, lane + 32, ...
  const int hh = warp;
  if (hh < g) {
    const long long prow = ((static_cast<long long>(n) * H + kvh * g + hh) * NC + chunk) * (D + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kKeyWarps; ++w) M = fmaxf(M, ctl.ml[w][hh].x);
    const bool has = done && M > -INFINITY;
    float f[kKeyWarps], L = 0.f;
#pragma unroll
    for (int w = 0; w < kKeyWarps; ++w) {
      const float2 ml = ctl.ml[w][hh];
      f[w] = (has && ml.x > -INFINITY) ? exp2f(ml.x - M) : 0.f;
      L += ml.y * f[w];
    }
    if (lane == 0) {
      part[prow] = has ? M : -INFINITY;
      part[prow + 1] = has ? L : 0.f;
    }
    for (int d = lane; d < D; d += 32) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kKeyWarps; ++w) acc += ow[(w * 8 + hh) * D + d] * f[w];
      part[prow + 2 + d] = has ? acc : 0.f;
    }
  }
}

// Partials of the chunks of one (sequence, head) merged: O = sum_c o_c 2^(m_c - M)
// / sum_c l_c 2^(m_c - M), M the largest m_c.  One thread per output column.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ part, const int32_t* __restrict__ lens,
                                                          int Lmax, int B, int NC, __nv_bfloat16* __restrict__ o) {
  const int n = static_cast<int>(blockIdx.y);
  const long long row = static_cast<long long>(n) * gridDim.x + blockIdx.x;   // n * H + h
  const int c = threadIdx.x;
  const int len = __ldg(lens + n);
  const int nc = (len >= 1 && len <= Lmax) ? ((len - 1) / B) / kDecChunk + 1 : 0;
  const float* p = part + row * NC * (D + 2);
  float M = -INFINITY;
  for (int k = 0; k < nc; ++k) M = fmaxf(M, p[k * (D + 2)]);
  float L = 0.f, O = 0.f;
  if (M > -INFINITY) {
    for (int k = 0; k < nc; ++k) {
      const float mk = p[k * (D + 2)];
      if (mk == -INFINITY) continue;
      const float f = exp2f(mk - M);
      L += p[k * (D + 2) + 1] * f;
      O += p[k * (D + 2) + 2 + c] * f;
    }
  }
  o[row * D + c] = __float2bfloat16(L > 0.f ? O / L : 0.f);
}

template <int BN, int D>
cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const int32_t* lens, int N, int Lmax, int H,
                            int Hkv, int S, float tau, bool gqa, int32_t* count, int32_t* idx, void* o,
                            const DecodeScratch& w, const DeviceGuardArgs& g, cudaStream_t stream) {
  const int Nbm = Lmax / BN, W = (Nbm + 31) / 32;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  CUtensorMap mks, mk, mv;
  const uint64_t rows = static_cast<uint64_t>(N) * Lmax;
  if (!make_tmap_sampled(&mks, k, rows, Hkv, D, S, kSearchTile) || !make_tmap_rows(&mk, k, rows, Hkv, D, BN) ||
      !make_tmap_rows(&mv, v, rows, Hkv, D, BN))
    return cudaErrorInvalidValue;
  constexpr int kSearchSmem = kSearchStages * kSearchTile * D * 2 + 1024;
  static std::atomic<uint64_t> search_smem_set{0};
  cudaError_t e = set_smem_limit_once(decode_search_kernel<D>, kSearchSmem, search_smem_set);
  if (e != cudaSuccess) return e;
  decode_search_kernel<D><<<static_cast<unsigned>(N) * H, kDecThreads, kSearchSmem, stream>>>(
      mks, static_cast<const __nv_bfloat16*>(q), lens, Lmax, H, Hkv, BN, S, sl2, tau, w.scores, Lmax / S, count, idx,
      w.bits, Nbm, W, gqa ? w.mass : nullptr, g.status, g.limit_ns);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (gqa) {
    decode_group_select_kernel<<<static_cast<unsigned>(N) * Hkv, kDecThreads, 0, stream>>>(
        w.mass, lens, Lmax, H, Hkv, BN, tau, count, idx, w.bits, Nbm, W);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  using C = DecAttnCfg<BN, D>;
  static std::atomic<uint64_t> smem_set{0};
  if ((e = set_smem_limit_once(decode_attn_kernel<BN, D>, C::kSmem, smem_set)) != cudaSuccess) return e;
  const int NC = (Nbm + kDecChunk - 1) / kDecChunk;
  decode_attn_kernel<BN, D><<<dim3(NC, Hkv, N), kDecThreads, C::kSmem, stream>>>(
      mk, mv, static_cast<const __nv_bfloat16*>(q), lens, w.bits, Lmax, H, Hkv, W, NC, sl2, w.part, g.status,
      g.limit_ns);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  decode_combine_kernel<D><<<dim3(H, N), D, 0, stream>>>(w.part, lens, Lmax, BN, NC, static_cast<__nv_bfloat16*>(o));
  return cudaGetLastError();
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
