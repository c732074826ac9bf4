// search.cu — the round-robin sampled-score pass and block-mass aggregation
// (RRAttention page, Abstract: per-head round-robin sampling, scores gathered
// per stride, a search cost of O(L^2/S^2); Figure 2 caption: stages 1 and 2).
//
// Head h samples, in stride i, position p(h, i) = i*S + (h mod S).  Its Ns = L/S
// sampled queries are scored against the Ns keys at the same positions of its
// kv head: s[i, j] = q_p(h,i) . k_p(h,j) / sqrt(d) for j <= i.  That is a causal
// attention over the head's strided subsequence, computed in 128 x 128 tiles:
//
//   * one CTA per (head, tile of 128 sampled rows); heavier tiles launch first;
//   * the sampled rows and keys are read zero-copy through 4D TMA views
//     (d, heads, S, Ns), so no sampled copy is ever materialised;
//   * S = Qs Ks^T runs on tcgen05 (bf16 in, fp32 accumulate in TMEM); with the
//     stride-mean keys of the alternative reading it is two MMA chains,
//     Qs*Khi^T + Qs*Klo^T, so the pooled keys enter at ~16 bits;
//   * pass 1 walks the row's key tiles for the row log-sum-exp (online), pass 2
//     recomputes the identical scores, forms P = exp(s - lse) and sums P over
//     the r x r (sampled row, stride) pairs of each B x B block with warp
//     shuffles; the block masses go to global memory.
//
// Warp roles: warp 0 issues TMA, warp 1 issues MMAs (one thread) and owns the
// TMEM allocation, warps 2..5 (128 threads, thread = sampled row = TMEM lane)
// do the softmax and reductions.  TMEM: two 128-column fp32 score buffers, so
// the MMA of tile n+1 overlaps the softmax of tile n.  Small shared memory
// lets two CTAs share an SM, whose tensor core then alternates between them.
#include <cuda_bf16.h>

#include "rr_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace rr {
namespace {

constexpr int kTile = 128;
constexpr int kThreads = 192;

template <int D>
struct SearchCfg {
  static constexpr int kStages = D == 128 ? 2 : 4;       // pooled-key tiles (hi or lo) in flight
  static constexpr int kTileBytes = kTile * D * 2;       // one 128 x D bf16 tile
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kTileBytes;
  static constexpr int kCtrlOff = kStageOff + kStages * kTileBytes;
  static constexpr int kSmem = kCtrlOff + 1024 + 1024;   // control block + alignment slack
};

struct SearchCtrl {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t s_empty[2];
  uint64_t drain;
  uint64_t red_bar;   // the 128 reduction threads meet here (bounded, unlike bar.sync)
  uint32_t tmem_base;
  int abort;
  float red[4][4];   // cross-warp partial block sums when r > 32
};

template <int D, int LOGR>
__global__ void __launch_bounds__(kThreads, 2)
    search_kernel(const __grid_constant__ CUtensorMap mqs, const __grid_constant__ CUtensorMap mkh,
                  const __grid_constant__ CUtensorMap mkl, float* __restrict__ mass, int H, int Hkv, int S,
                  int Ns, int Nb, float sl2, int q_mode, int k_mode, int head0, unsigned int* status, uint64_t limit_ns) {
  using C = SearchCfg<D>;
  constexpr int R = 1 << LOGR;                 // sampled rows (and strides) per block
  constexpr int GPT = kTile / R;               // key blocks per 128-stride tile
  constexpr int KSTEPS = D / 16;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTile, false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sStage = smem + C::kStageOff;
  SearchCtrl* ctl = reinterpret_cast<SearchCtrl*>(smem + C::kCtrlOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_row_tiles = (Ns + kTile - 1) / kTile;
  const int rt = n_row_tiles - 1 - static_cast<int>(blockIdx.x / H);   // row tile, heavy first
  const int h = static_cast<int>(blockIdx.x % H);
  const int kvh = h / (H / Hkv);
  const int n_key_tiles = rt + 1;
  const int n_seq = 2 * n_key_tiles;           // pass 1 then pass 2
  // q_mode 0: sampled rows read through the 4D view (d, H, S, Ns) at offset h mod S;
  //        1: rows gathered beforehand into [Ns, H, d] (rotating offsets).
  // k_mode 0: stride means as a bf16 (hi, lo) pair [Ns, Hkv, d], two MMA chains;
  //        1: one sampled key per stride through the 4D view of k at offset h mod S;
  //        2: sampled keys gathered beforehand into [Ns, H, d].
  const int parts = k_mode == 0 ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->q_full), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->s_full[b]), 1);
      mbar_init(smem_u32(&ctl->s_empty[b]), 128);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    mbar_init(smem_u32(&ctl->red_bar), 128);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ctl->tmem_base;
  const Guard guard{&ctl->abort, status, limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mqs);
      tma_prefetch_desc(&mkh);
      tma_prefetch_desc(&mkl);
      const uint32_t qb = smem_u32(&ctl->q_full);
      mbar_expect_tx(qb, C::kTileBytes);
      for (int a = 0; a < D / 64; ++a) {
        if (q_mode == 0)
          tma_load_4d(smem_u32(sQ + a * kTile * 128), &mqs, qb, a * 64, h, (h + head0) % S, rt * kTile);
        else
          tma_load_3d(smem_u32(sQ + a * kTile * 128), &mqs, qb, a * 64, h, rt * kTile);
      }
      int k = 0;
      bool ok = true;
      for (int n = 0; n < n_seq && ok; ++n) {
        const int c = n % n_key_tiles;
        for (int part = 0; part < parts && ok; ++part) {
          const int st = k % C::kStages;
          const uint32_t ph = (k / C::kStages) & 1;
          if (!wait_bar(smem_u32(&ctl->empty[st]), ph ^ 1, guard, 1)) { ok = false; break; }
          const uint32_t fb = smem_u32(&ctl->full[st]);
          mbar_expect_tx(fb, C::kTileBytes);
          uint8_t* dst = sStage + st * C::kTileBytes;
          for (int a = 0; a < D / 64; ++a) {
            const uint32_t da = smem_u32(dst + a * kTile * 128);
            if (k_mode == 0)
              tma_load_3d(da, part == 0 ? &mkh : &mkl, fb, a * 64, kvh, c * kTile);
            else if (k_mode == 1)
              tma_load_4d(da, &mkh, fb, a * 64, kvh, (h + head0) % S, c * kTile);
            else
              tma_load_3d(da, &mkh, fb, a * 64, h, c * kTile);
          }
          ++k;
        }
      }
      // drain: every issued load has landed before the CTA may exit
      drain_bar(qb, 0, kDrainLimitNs);
      for (int kk = (k > C::kStages ? k - C::kStages : 0); kk < k; ++kk)
        drain_bar(smem_u32(&ctl->full[kk % C::kStages]), (kk / C::kStages) & 1, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = wait_bar(smem_u32(&ctl->q_full), 0, guard, 2);
      // descriptor bases (K-major, 128-byte swizzle), stepped with 32-bit adds
      const uint32_t q_lo = sdesc_sw128_lo(smem_u32(sQ), 16);
      const uint32_t k_lo = sdesc_sw128_lo(smem_u32(sStage), 16);
      constexpr uint32_t d_hi = sdesc_sw128_hi(1024);
      int k = 0;
      for (int n = 0; n < n_seq && ok; ++n) {
        const int b = n & 1;
        if (!wait_bar(smem_u32(&ctl->s_empty[b]), ((n >> 1) & 1) ^ 1, guard, 3)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tm + b * kTile;
        for (int part = 0; part < parts; ++part) {
          const int st = k % C::kStages;
          if (!wait_bar(smem_u32(&ctl->full[st]), (k / C::kStages) & 1, guard, 4)) { ok = false; break; }
          const uint32_t kb = k_lo + st * (C::kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk)
            umma_ss_lh(dcol, q_lo + (kk >> 2) * (kTile * 128 >> 4) + 2 * (kk & 3), d_hi,
                       kb + (kk >> 2) * (kTile * 128 >> 4) + 2 * (kk & 3), d_hi, kIdesc,
                       (part > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&ctl->empty[st]));
          ++k;
        }
        if (!ok) break;
        umma_commit(smem_u32(&ctl->s_full[b]));
      }
      umma_commit(smem_u32(&ctl->drain));
      drain_bar(smem_u32(&ctl->drain), 0, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / reduction
    const int wq = warp & 3;                    // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;             // sampled row within the tile
    const int i = rt * kTile + row;             // sampled row index (stride of the query)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f, lse = 0.f;
    uint32_t red_phase = 0;
    bool ok = true;
    for (int n = 0; n < n_seq; ++n) {
      const int b = n & 1;
      const int c = n % n_key_tiles;
      const bool pass2 = n >= n_key_tiles;
      if (!wait_bar_warp(smem_u32(&ctl->s_full[b]), (n >> 1) & 1, guard, 5)) { ok = false; break; }
      tc_fence_after();
      uint32_t raw[128];
      tmem_ld128(tm + lane_off + b * kTile, raw);
      tc_fence_before();
      mbar_arrive(smem_u32(&ctl->s_empty[b]));
      // scores of this tile as loaded (scaled inside the exponentials below:
      // x = s * sl2 - m in one fused multiply-add, the same in both passes)
      float v[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) v[j] = __uint_as_float(raw[j]);
      if (c == rt) {   // the diagonal tile (uniform across the CTA): stride-causal, j <= i
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (j > row) v[j] = -INFINITY;
      }
      const uint64_t sl2x2 = f2pack(sl2, sl2);
      if (!pass2) {
        // row max: eight independent three-input chains (sl2 > 0 commutes with max)
        float m8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) m8[a] = fmaxf(v[2 * a], v[2 * a + 1]);
#pragma unroll
        for (int j = 16; j < 128; j += 16) {
#pragma unroll
          for (int a = 0; a < 8; ++a) m8[a] = max3(m8[a], v[j + 2 * a], v[j + 2 * a + 1]);
        }
        const float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * sl2;
        const float m_new = fmaxf(m_run, mx);
        const uint64_t negm = f2pack(-m_new, -m_new);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // four packed partial sums
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) {
          float x0, x1;
          f2unpack(fma2(f2pack(v[2 * jj], v[2 * jj + 1]), sl2x2, negm), x0, x1);
          acc[jj & 3] = add2(acc[jj & 3], f2pack(ex2(x0), ex2(x1)));
        }
        float s0, s1;
        f2unpack(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), s0, s1);
        l_run = l_run * ex2(m_run - m_new) + (s0 + s1);
        m_run = m_new;
        if (n == n_key_tiles - 1) lse = m_run + lg2(l_run);
        continue;
      }
      // pass 2: probabilities, summed over each key block's R strides (in place: v[g])
      const uint64_t negl = f2pack(-lse, -lse);
      if constexpr (R == 1) {
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) {
          float x0, x1;
          f2unpack(fma2(f2pack(v[2 * jj], v[2 * jj + 1]), sl2x2, negl), x0, x1);
          v[2 * jj] = ex2(x0);
          v[2 * jj + 1] = ex2(x1);
        }
      } else {
#pragma unroll
        for (int g = 0; g < GPT; ++g) {
          uint64_t acc = 0ull;
#pragma unroll
          for (int t = 0; t < R / 2; ++t) {
            const int jj = g * (R / 2) + t;
            float x0, x1;
            f2unpack(fma2(f2pack(v[2 * jj], v[2 * jj + 1]), sl2x2, negl), x0, x1);
            acc = add2(acc, f2pack(ex2(x0), ex2(x1)));
          }
          float s0, s1;
          f2unpack(acc, s0, s1);
          v[g] = s0 + s1;
        }
      }
      // ... and over the R sampled rows of each query block
      if constexpr (R <= 32) {
#pragma unroll
        for (int g = 0; g < GPT; ++g) {
#pragma unroll
          for (int off = 1; off < R; off <<= 1) v[g] += __shfl_xor_sync(0xffffffffu, v[g], off);
        }
        const int I = i >> LOGR;
        if ((lane & (R - 1)) == 0 && I < Nb) {
          float* dst = mass + (static_cast<long long>(h) * Nb + I) * Nb + c * GPT;
#pragma unroll
          for (int g = 0; g < GPT; ++g)
            if (c * GPT + g < Nb) dst[g] = v[g];
        }
      } else {
#pragma unroll
        for (int g = 0; g < GPT; ++g) {
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) v[g] += __shfl_xor_sync(0xffffffffu, v[g], off);
        }
        if (lane == 0) {
#pragma unroll
          for (int g = 0; g < GPT; ++g) ctl->red[wq][g] = v[g];
        }
        mbar_arrive(smem_u32(&ctl->red_bar));
        if (!wait_bar_warp(smem_u32(&ctl->red_bar), red_phase++ & 1, guard, 6)) { ok = false; break; }
        constexpr int WPB = R / 32;             // warps per query block
        const int t = threadIdx.x - 64;
        if (t < (4 / WPB) * GPT) {
          const int qb = t / GPT, g = t % GPT;
          float acc = 0.f;
          for (int w = 0; w < WPB; ++w) acc += ctl->red[qb * WPB + w][g];
          const int I = (rt * kTile) / R + qb;
          if (I < Nb && c * GPT + g < Nb) mass[(static_cast<long long>(h) * Nb + I) * Nb + c * GPT + g] = acc;
        }
        mbar_arrive(smem_u32(&ctl->red_bar));
        if (!wait_bar_warp(smem_u32(&ctl->red_bar), red_phase++ & 1, guard, 7)) { ok = false; break; }
      }
    }
    (void)ok;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tm, 256);
}

template <int D, int LOGR>
cudaError_t launch_search_t(const CUtensorMap& mqs, const CUtensorMap& mkh, const CUtensorMap& mkl, float* mass,
                            int H, int Hkv, int S, int Ns, int Nb, float sl2, int q_mode, int k_mode,
                            int head0, const DeviceGuardArgs& g, cudaStream_t stream) {
  using C = SearchCfg<D>;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = set_smem_limit_once(search_kernel<D, LOGR>, C::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  const int n_row_tiles = (Ns + kTile - 1) / kTile;
  search_kernel<D, LOGR><<<static_cast<unsigned>(n_row_tiles) * H, kThreads, C::kSmem, stream>>>(
      mqs, mkh, mkl, mass, H, Hkv, S, Ns, Nb, sl2, q_mode, k_mode, head0, g.status, g.limit_ns);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_r(int logr, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, float* mass,
                       int H, int Hkv, int S, int Ns, int Nb, float sl2, int qm, int km, int h0, const DeviceGuardArgs& g,
                       cudaStream_t st) {
  switch (logr) {
    case 0: return launch_search_t<D, 0>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 1: return launch_search_t<D, 1>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 2: return launch_search_t<D, 2>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 3: return launch_search_t<D, 3>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 4: return launch_search_t<D, 4>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 5: return launch_search_t<D, 5>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 6: return launch_search_t<D, 6>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    case 7: return launch_search_t<D, 7>(a, b, c, mass, H, Hkv, S, Ns, Nb, sl2, qm, km, h0, g, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_search(const SearchSources& src, float* mass, int L, int H, int Hkv, int d, int B, int S,
                          const DeviceGuardArgs& g, cudaStream_t stream) {
  const int Ns = L / S, Nb = L / B, r = B / S;
  int logr = 0;
  while ((1 << logr) < r) ++logr;
  CUtensorMap mqs, mkh, mkl;
  bool ok = src.q_mode == 0 ? make_tmap_sampled(&mqs, src.q, L, H, d, S, kTile)
                            : make_tmap_rows(&mqs, src.q, Ns, H, d, kTile);
  if (src.k_mode == 0) {
    ok = ok && make_tmap_rows(&mkh, src.k_a, Ns, Hkv, d, kTile) && make_tmap_rows(&mkl, src.k_b, Ns, Hkv, d, kTile);
  } else if (src.k_mode == 1) {
    ok = ok && make_tmap_sampled(&mkh, src.k_a, L, Hkv, d, S, kTile);
    mkl = mkh;
  } else {
    ok = ok && make_tmap_rows(&mkh, src.k_a, Ns, H, d, kTile);
    mkl = mkh;
  }
  if (!ok) return cudaErrorInvalidValue;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  if (d == 128)
    return dispatch_r<128>(logr, mqs, mkh, mkl, mass, H, Hkv, S, Ns, Nb, sl2, src.q_mode, src.k_mode, src.head0, g, stream);
  return dispatch_r<64>(logr, mqs, mkh, mkl, mass, H, Hkv, S, Ns, Nb, sl2, src.q_mode, src.k_mode, src.head0, g, stream);
}

}  // namespace rr
