// bsfa.cu — causal block-sparse FlashAttention forward over the selected
// blocks (RRAttention page, Abstract: about half of the blocks computed and a
// 2.4x speedup at 128K on the pages' workloads; Figure 2 caption: stage 3;
// Figure 3 caption, panel a).
//
// One CTA per (head h, query block I), launched kv head by kv head, longest
// rows first: a 128-row query tile (the B = 64 case
// uses the first 64 rows), the key blocks J listed for (h, I) visited in
// ascending order.  Both contractions per block run on tcgen05 with fp32
// accumulators in TMEM:
//     S = Q K_J^T           (A = Q, B = K_J from shared memory, K-major)
//     O += P V_J            (A = P from TMEM as bf16, B = V_J, MN-major)
// The block list is split between two softmax warpgroups (even / odd list
// positions), each with its own S buffer and O accumulator, so the tensor core
// works on one group's blocks while the other group runs its softmax.  Each
// group keeps its own running max / sum; the two partial results are merged
// exactly in the epilogue:  O = (O_a 2^(m_a-m) + O_b 2^(m_b-m)) / (l_a 2^(m_a-m)
// + l_b 2^(m_b-m)).
//
// Online softmax in the exp2 domain with a lazy running max: a group's first
// block sets it to that block's row max; later blocks are exponentiated with
// it directly, and a row's max moves (with O and l rescaled) only when the
// block's sum of P passes 2^16.  That keeps P < 2^16, which bf16 and fp32 hold
// without loss, and is exact after the final division because P and l always
// use the same max.
//
// Warp roles (384 threads, three warpgroups): warp 0 TMA producer; warps 1 and
// 3 MMA issuers (one thread each) for softmax groups 0 and 1, taking strict
// turns by whole MMA brackets (warp 1 also owns the 512-column TMEM
// allocation); warp 2 idle; warps 4-7 softmax group 0, warps 8-11 softmax
// group 1.  The first warpgroup gives registers back so that the softmax
// groups can hold a full score row: setmaxnreg 56 / 224 at B = 128 and
// 80 / 200 at B = 64, both within the launch's 384 * 168 registers
// (128*56 + 256*224 = 64512, 128*80 + 256*200 = 61440).
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512);
// P_x overwrites the last B/2 columns of S_x, so that the first half of the
// scores is still there when a row's block has to be redone.
// K/V tiles stream through a 4-stage shared-memory ring in the order the MMA
// consumes them: K0, K1, V0, K2, V1, K3, ...
#include <cuda_bf16.h>
#include <stdlib.h>

#include "rr_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace rr {
namespace {

constexpr int kThreads = 384;
constexpr int kStages = 4;

template <int BN, int D>
struct FaCfg {
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kTileBytes = BN * D * 2;
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kListOff = kStageOff + kStages * kTileBytes;
  static constexpr int kCtrlOff = kListOff + kMaxBlocks * 4;
  static constexpr int kUsed = kCtrlOff + 2048 + 1024;
  // At least ~120 KB so that one CTA holds an SM (it allocates all 512 TMEM columns).
  static constexpr int kSmem = kUsed > 122880 ? kUsed : 122880;
};

struct FaCtrl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t merge;
  uint64_t drain[2];
  uint64_t never;      // fault injection: a barrier nothing arrives on
  uint32_t tmem_base;
  int abort;
  int turn;            // which issuer may issue its next MMA bracket (0 or 1)
  int issuer_done[2];  // an issuer with no bracket left never takes the turn
  float2 ml[2][128];
};

// Exponentiate one row of scores into P = 2^(s*sl2 - m) (bf16, written to TMEM
// at p_col) and return the row sum of P in fp32.
template <int BN>
__device__ __forceinline__ float exp_store(const float (&s)[BN], float sl2, float m_run, uint32_t p_col) {
  const uint64_t scale2 = f2pack(sl2, sl2);
  const uint64_t negm2 = f2pack(-m_run, -m_run);
  uint64_t acc[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = 0ull;   // (+0.0f, +0.0f)
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int jj = c * 16 + j;
      const uint64_t xp = fma2(f2pack(s[2 * jj], s[2 * jj + 1]), scale2, negm2);
      float x0, x1;
      f2unpack(xp, x0, x1);
      const uint64_t pp = f2pack(ex2(x0), ex2(x1));
      acc[j & 3] = add2(acc[j & 3], pp);
      float p0, p1;
      f2unpack(pp, p0, p1);
      pk[j] = pack_bf16x2(p0, p1);
    }
    tmem_st16(p_col + c * 16, pk);
  }
  const uint64_t t = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  float lo, hi;
  f2unpack(t, lo, hi);
  return lo + hi;
}

// Row max of BN scores: eight independent three-input max chains.
template <int BN>
__device__ __forceinline__ float row_max(const float (&s)[BN]) {
  float m8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m8[j] = fmaxf(s[2 * j], s[2 * j + 1]);
#pragma unroll
  for (int j = 16; j < BN; j += 16) {
#pragma unroll
    for (int a = 0; a < 8; ++a) m8[a] = max3(m8[a], s[j + 2 * a], s[j + 2 * a + 1]);
  }
  return max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
}

template <int BN, int D>
__global__ void __launch_bounds__(kThreads, 1)
    bsfa_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, const int32_t* __restrict__ count,
                const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o, int H, int Hkv, int Nb,
                float sl2, unsigned int* status, uint64_t limit_ns, int inject_stall) {
  using C = FaCfg<BN, D>;
  constexpr uint32_t kIdS = idesc_bf16_f32(128, BN, false, false);
  constexpr uint32_t kIdO = idesc_bf16_f32(128, D, false, true);
  // A row's running max moves only when one block's exponentials sum past
  // this bound, so every P stays below 2^16: bf16 and fp32 share the 8-bit
  // exponent, and P, O and the row sum lose nothing at that size.
  constexpr float kSumLimit = 65536.0f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sStage = smem + C::kStageOff;
  int32_t* sList = reinterpret_cast<int32_t*>(smem + C::kListOff);
  FaCtrl* ctl = reinterpret_cast<FaCtrl*>(smem + C::kCtrlOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA order: kv head by kv head, and inside one kv head longer rows first
  // with the g query heads of a row side by side.  The CTAs resident at any time
  // then share one kv head's K and V (64 MB at L = 128K, d = 128), which stay
  // in L2 instead of being re-read from HBM by every row.
  const int g = H / Hkv;
  const int per_kv = g * Nb;
  const int kvh = static_cast<int>(blockIdx.x / per_kv);
  const int r = static_cast<int>(blockIdx.x % per_kv);
  const int I = Nb - 1 - r / g;
  const int h = kvh * g + r % g;
  const long long row_id = static_cast<long long>(h) * Nb + I;
  int cnt = count[row_id];
  const int32_t* list = idx + row_id * Nb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->q_full), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(smem_u32(&ctl->s_full[x]), 1);
      mbar_init(smem_u32(&ctl->p_full[x]), 128);
    }
    mbar_init(smem_u32(&ctl->merge), 256);
    mbar_init(smem_u32(&ctl->drain[0]), 1);
    mbar_init(smem_u32(&ctl->drain[1]), 1);
    mbar_init(smem_u32(&ctl->never), 1);
    ctl->abort = 0;
    ctl->turn = 0;
    ctl->issuer_done[0] = ctl->issuer_done[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), 512);
    tmem_relinquish();
  }
  // The row's block list, read coalesced into shared memory by every thread and
  // checked against the mask format: count in [1, I+1], entries strictly
  // ascending inside [0, I].  A list that breaks it (a key block above the
  // diagonal would attend to future keys, one past Nb would read past the
  // tensor) is not computed: the row's output is zero and the status word
  // records the mask error with the row.
  int bad = (cnt < 1 || cnt > I + 1) ? 1 : 0;
  if (!bad) {
    for (int t = threadIdx.x; t < cnt; t += kThreads) {
      const int J = __ldg(list + t);
      const int prev = t > 0 ? __ldg(list + t - 1) : -1;
      if (J < 0 || J > I || J <= prev) bad = 1;
      sList[t] = J;
    }
  }
  tc_fence_before();
  bad = __syncthreads_or(bad);
  tc_fence_after();
  if (bad) {
    if (threadIdx.x == 0)
      atomicCAS(status, 0u, kStatusMaskCode | (static_cast<unsigned>(row_id < (1 << 24) ? row_id : (1 << 24) - 1) << 8));
    cnt = 0;
  }
  const uint32_t tm = ctl->tmem_base;
  const Guard guard{&ctl->abort, status, limit_ns};
  if (warp < 4) {
    if constexpr (BN == 128) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
    } else {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n" ::: "memory");
    }
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && cnt > 0) {
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      const uint32_t qb = smem_u32(&ctl->q_full);
      mbar_expect_tx(qb, C::kQBytes);
      for (int a = 0; a < D / 64; ++a) tma_load_3d(smem_u32(sQ + a * 128 * 128), &mq, qb, a * 64, h, I * BN);
    }
    if (lane == 0 && cnt > 0) {
      int k = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* m, int J) {
        const int st = k % kStages;
        if (!wait_bar(smem_u32(&ctl->empty[st]), ((k / kStages) & 1) ^ 1, guard, 1)) return false;
        const uint32_t fb = smem_u32(&ctl->full[st]);
        mbar_expect_tx(fb, C::kTileBytes);
        uint8_t* dst = sStage + st * C::kTileBytes;
        for (int a = 0; a < D / 64; ++a) tma_load_3d(smem_u32(dst + a * BN * 128), m, fb, a * 64, kvh, J * BN);
        ++k;
        return true;
      };
      // tile order = MMA order: K0, K1, V0, K2, V1, K3, ...
      ok = load(&mk, sList[0]);
      if (ok && cnt > 1) ok = load(&mk, sList[1]);
      for (int t = 0; t < cnt && ok; ++t) {
        ok = load(&mv, sList[t]);
        if (ok && t + 2 < cnt) ok = load(&mk, sList[t + 2]);
      }
      drain_bar(smem_u32(&ctl->q_full), 0, kDrainLimitNs);
      for (int kk = (k > kStages ? k - kStages : 0); kk < k; ++kk)
        drain_bar(smem_u32(&ctl->full[kk % kStages]), (kk / kStages) & 1, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp & 1) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues softmax group 0's MMAs, warp 3 group 1's.  A tcgen05.mma
    // issue occupies its thread for nearly the MMA's own run time, so any other
    // instruction between two MMAs of one thread (even a satisfied barrier
    // test) leaves the tensor core idle.  The two issuers therefore take strict
    // turns by whole brackets (P V of one block and S of that group's next):
    // while one issues back to back, the other does its waits.  Strict turns
    // also keep the two groups half a period apart.
    const int x = warp >> 1;
    const int n_x = x == 0 ? (cnt + 1) >> 1 : cnt >> 1;   // list positions x, x+2, ...
    if (lane == 0 && n_x > 0) {
      bool ok = true;
      // Injected fault (tests only): wait on a barrier that nothing arrives
      // on; the bounded wait gives up, and the CTA takes its abort path.
      if (inject_stall) ok = wait_bar(smem_u32(&ctl->never), 0, guard, 9);
      if (ok) ok = wait_bar(smem_u32(&ctl->q_full), 0, guard, 2);
      // Descriptor bases, computed once.  K-major tiles step 32 bytes (2 in the
      // start-address field) per 16-wide K slice and one 64-column atom per 4
      // slices; the V tile (MN-major) steps 16 rows (128 in the field) per slice.
      const uint32_t q_lo = sdesc_sw128_lo(smem_u32(sQ), 16);
      const uint32_t k_lo = sdesc_sw128_lo(smem_u32(sStage), 16);
      const uint32_t v_lo = sdesc_sw128_lo(smem_u32(sStage), BN * 128);
      constexpr uint32_t q_hi = sdesc_sw128_hi(1024), k_hi = sdesc_sw128_hi(1024), v_hi = sdesc_sw128_hi(1024);
      constexpr uint32_t kStageStep = C::kTileBytes >> 4;
      const uint32_t s_tm = tm + x * 128, o_tm = tm + 256 + x * 128;
      // Position of a tile in the producer's order: K0, K1 (if cnt > 1), then
      // for t = 0..cnt-1: V(t), and K(t+2) while t+2 < cnt.
      const int c1 = cnt > 1 ? 1 : 0, tail = cnt > 2 ? cnt - 2 : 0;
      auto pos_v = [&](int t) { return 1 + c1 + t + (t < tail ? t : tail); };
      auto pos_k = [&](int t) { return t < 2 ? t : pos_v(t - 2) + 1; };
      auto wait_tile = [&](int pos, int site) {
        return wait_bar(smem_u32(&ctl->full[pos % kStages]), (pos / kStages) & 1, guard, site);
      };
      auto emit_s = [&](int t) {
        const int st = pos_k(t) % kStages;
        const uint32_t kb = k_lo + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss_lh(s_tm, q_lo + (kk >> 2) * (128 * 128 >> 4) + 2 * (kk & 3), q_hi,
                     kb + (kk >> 2) * (BN * 128 >> 4) + 2 * (kk & 3), k_hi, kIdS, kk > 0 ? 1u : 0u);
        umma_commit(smem_u32(&ctl->empty[st]));
      };
      auto emit_pv = [&](int t, bool acc) {
        const int st = pos_v(t) % kStages;
        const uint32_t vb = v_lo + st * kStageStep;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts_lh(o_tm, s_tm + BN / 2 + kk * 8, vb + kk * (16 * 128 >> 4), v_hi, kIdO, (acc || kk > 0) ? 1u : 0u);
        umma_commit(smem_u32(&ctl->empty[st]));
      };
      volatile int* turn = &ctl->turn;
      volatile int* other_done = &ctl->issuer_done[x ^ 1];
      // Wait for this issuer's turn (bounded; the other issuer may have finished).
      auto take_turn = [&]() {
        const uint64_t t0 = global_ns();
        for (uint32_t it = 0;; ++it) {
          if (*turn == x || *other_done) return true;
          if ((it & 255) == 255) {
            if (*guard.abort) return false;
            if (global_ns() - t0 > guard.limit_ns) {
              *guard.abort = 1;
              atomicCAS(guard.status, 0u, kStatusTimeout | (11u << 8));
              return false;
            }
          }
        }
      };
      auto give_turn = [&]() { *turn = x ^ 1; };
      // first S of this group: issuer 0 goes first, then issuer 1
      if (ok) ok = wait_tile(pos_k(x), 3);
      if (ok) ok = take_turn();
      if (ok) {
        emit_s(x);
        umma_commit(smem_u32(&ctl->s_full[x]));
        give_turn();
      }
      for (int i = 0; i < n_x && ok; ++i) {
        const int t = 2 * i + x;
        const bool more = i + 1 < n_x;
        // everything this bracket needs, while the other issuer's bracket runs:
        // the tiles first (they landed long ago; each satisfied test still
        // costs the thread ~150 cycles), then P, then the turn
        if (!wait_tile(pos_v(t), 4)) { ok = false; break; }
        if (more && !wait_tile(pos_k(t + 2), 3)) { ok = false; break; }
        if (!wait_bar(smem_u32(&ctl->p_full[x]), i & 1, guard, 5)) { ok = false; break; }
        tc_fence_after();   // P was written to TMEM by the softmax threads
        if (!take_turn()) { ok = false; break; }
        emit_pv(t, i > 0);
        if (more) emit_s(t + 2);
        umma_commit(smem_u32(&ctl->s_full[x]));
        if (!more) ctl->issuer_done[x] = 1;
        give_turn();
      }
      if (!ok) ctl->issuer_done[x] = 1;
      umma_commit(smem_u32(&ctl->drain[x]));
      drain_bar(smem_u32(&ctl->drain[x]), 0, kDrainLimitNs);
    } else if (lane == 0) {
      ctl->issuer_done[x] = 1;   // no bracket for this group
    }
    __syncwarp();
  }
  } else {
    if constexpr (BN == 128) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 224;\n" ::: "memory");
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    }
    // ------------------------------------------------------------ softmax groups
    const int x = (warp - 4) >> 2;              // group 0: warps 4-7, group 1: warps 8-11
    const int wq = warp & 3;                    // TMEM lane quarter
    const int row = wq * 32 + lane;             // row of the query tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_col = tm + lane_off + x * 128;
    const uint32_t p_col = s_col + BN / 2;
    const uint32_t o_col = tm + lane_off + 256 + x * 128;
    const int n_a = (cnt + 1) >> 1, n_b = cnt >> 1;
    const int n_x = x == 0 ? n_a : n_b;
    const bool diag_last = cnt > 0 && sList[cnt - 1] == I;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int u = 0; u < n_x; ++u) {
      const int t = 2 * u + x;
      if (!wait_bar_warp(smem_u32(&ctl->s_full[x]), u & 1, guard, 6)) { ok = false; break; }
      tc_fence_after();
      uint32_t raw[BN];
      if constexpr (BN == 128) {
        tmem_ld128(s_col, raw);
      } else {
        tmem_ld32x2(s_col, s_col + 32, raw);
      }
      float s[BN];
#pragma unroll
      for (int j = 0; j < BN; ++j) s[j] = __uint_as_float(raw[j]);
      const bool diag = diag_last && t == cnt - 1;   // uniform across the CTA
      if (diag) {
#pragma unroll
        for (int j = 0; j < BN; ++j)
          if (j > row) s[j] = -INFINITY;                // causal mask inside block J == I
      }
      // Online softmax with a lazy running max.  A group's first block sets it
      // to the block's row max.  Later blocks are exponentiated with it at
      // once, with no max pass: only when a row's block sum passes kSumLimit
      // (some score grew far above the running max) does that row take its
      // exact block max, rescale O and l, and redo the block.
      auto expo = [&]() { return exp_store<BN>(s, sl2, m_run, p_col); };
      bool rescale = false;
      float alpha = 1.0f;
      if (u == 0) m_run = row_max<BN>(s) * sl2;
      float sum = expo();
      if (u > 0) {
        const bool need = !(sum <= kSumLimit);
        rescale = __any_sync(0xffffffffu, need);
        if (rescale) {
          tmem_wait_st();
          // The P stores overwrote the second half of the scores in TMEM; the
          // first half is reloaded, so those registers need not live across
          // the first pass.
          if constexpr (BN == 128) {
            uint32_t r[64];
            tmem_ld32x2(s_col, s_col + 32, r);
#pragma unroll
            for (int j = 0; j < 64; ++j) s[j] = __uint_as_float(r[j]);
          } else {
            uint32_t r[32];
            tmem_ld32(s_col, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(r[j]);
          }
          if (diag) {
#pragma unroll
            for (int j = 0; j < BN / 2; ++j)
              if (j > row) s[j] = -INFINITY;
          }
          if (need) {
            const float m_new = fmaxf(m_run, row_max<BN>(s) * sl2);
            alpha = ex2(m_run - m_new);
            l_run *= alpha;
            m_run = m_new;
          }
          sum = expo();
        }
      }
      // O of this group is quiescent here (its last P V completed before this S
      // was signalled), and the next P V is issued only after p_full.
      if (rescale) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {   // rare: not unrolled, so it holds 32 registers only
          uint32_t ov[32];
          tmem_ld32(o_col + c * 32, ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tmem_st32(o_col + c * 32, ov);
        }
      }
      l_run += sum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&ctl->p_full[x]));
    }
    // the group's last P V has completed once its S barrier fires one more time
    if (ok && n_x > 0) ok = wait_bar_warp(smem_u32(&ctl->s_full[x]), n_x & 1, guard, 7);
    tc_fence_after();
    ctl->ml[x][row] = make_float2(n_x > 0 ? m_run : -INFINITY, n_x > 0 ? l_run : 0.f);
    tc_fence_before();
    mbar_arrive(smem_u32(&ctl->merge));
    if (!wait_bar(smem_u32(&ctl->merge), 0, guard, 8)) ok = false;
    tc_fence_after();
    const bool go = __all_sync(0xffffffffu, ok && !ctl->abort);
    if (cnt > 0 && go && row < BN) {
      const float2 a = ctl->ml[0][row], b = ctl->ml[1][row];
      const float mm = fmaxf(a.x, b.x);
      const float fa = a.y > 0.f ? ex2(a.x - mm) : 0.f;
      const float fb = b.y > 0.f ? ex2(b.x - mm) : 0.f;
      const float denom = a.y * fa + b.y * fb;
      const float inv = denom > 0.f ? 1.0f / denom : 0.f;
      const float ca = fa * inv, cb = fb * inv;
      __nv_bfloat16* dst = o + ((static_cast<long long>(I) * BN + row) * H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col = x * (D / 2) + c * 32;
        uint32_t va[32], vb[32];
        tmem_ld32(tm + lane_off + 256 + col, va);
        if (n_b > 0) {
          tmem_ld32(tm + lane_off + 384 + col, vb);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) vb[j] = 0u;
        }
        uint4 pk[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float o0 = __uint_as_float(va[2 * j]) * ca + __uint_as_float(vb[2 * j]) * cb;
          const float o1 = __uint_as_float(va[2 * j + 1]) * ca + __uint_as_float(vb[2 * j + 1]) * cb;
          pw[j] = pack_bf16x2(o0, o1);
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
        for (int j = 0; j < 4; ++j) d4[j] = pk[j];
      }
    } else if (cnt == 0 && row < BN) {
      // a row whose list broke the mask format: zero output (status recorded above)
      __nv_bfloat16* dst = o + ((static_cast<long long>(I) * BN + row) * H + h) * D;
      for (int c = x * (D / 2); c < (x + 1) * (D / 2); c += 8)
        *reinterpret_cast<uint4*>(dst + c) = make_uint4(0, 0, 0, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tm, 512);
}

template <int BN, int D>
cudaError_t launch_bsfa_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const int32_t* count, const int32_t* idx, void* o, int H, int Hkv, int Nb, float sl2,
                          const DeviceGuardArgs& g, int inject, cudaStream_t stream) {
  using C = FaCfg<BN, D>;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = set_smem_limit_once(bsfa_kernel<BN, D>, C::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  bsfa_kernel<BN, D><<<static_cast<unsigned>(H) * Nb, kThreads, C::kSmem, stream>>>(
      mq, mk, mv, count, idx, static_cast<__nv_bfloat16*>(o), H, Hkv, Nb, sl2, g.status, g.limit_ns, inject);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bsfa(const void* q, const void* k, const void* v, const int32_t* count, const int32_t* idx,
                        void* o, int L, int H, int Hkv, int d, int B, const DeviceGuardArgs& g,
                        cudaStream_t stream) {
  const int Nb = L / B;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_rows(&mq, q, L, H, d, 128) || !make_tmap_rows(&mk, k, L, Hkv, d, B) ||
      !make_tmap_rows(&mv, v, L, Hkv, d, B))
    return cudaErrorInvalidValue;
  const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  // RR_DEBUG_STALL_WAIT=1 injects a wait that never completes (tests of the
  // bounded-wait path); unset in normal use.
  const char* inj = getenv("RR_DEBUG_STALL_WAIT");
  const int inject = (inj && inj[0] == '1') ? 1 : 0;
  if (B == 128 && d == 128) return launch_bsfa_t<128, 128>(mq, mk, mv, count, idx, o, H, Hkv, Nb, sl2, g, inject, stream);
  if (B == 128 && d == 64) return launch_bsfa_t<128, 64>(mq, mk, mv, count, idx, o, H, Hkv, Nb, sl2, g, inject, stream);
  if (B == 64 && d == 128) return launch_bsfa_t<64, 128>(mq, mk, mv, count, idx, o, H, Hkv, Nb, sl2, g, inject, stream);
  if (B == 64 && d == 64) return launch_bsfa_t<64, 64>(mq, mk, mv, count, idx, o, H, Hkv, Nb, sl2, g, inject, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rr
