// rr_abi.cu — the C ABI declared in include/rr.h: host-side validation,
// workspace carving and stream-ordered launches.  No device memory is
// allocated here; every buffer is the caller's.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <vector>

#include "rr.h"
#include "rr_internal.h"

namespace {

uint64_t g_wait_limit_ns = 2000000000ull;

// An NVTX range around the host-side enqueue of one stage (visible in a
// timeline tool next to the kernels it launched; a no-op without one).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

constexpr unsigned kVarAll = RR_VAR_ROTATE | RR_VAR_MEAN_KEYS | RR_VAR_GQA_MASK;

// Workspace regions (byte offsets).  With flags 0 only status and mass are
// present (the rr_search layout); the pooled-key pair khi/klo only with
// RR_VAR_MEAN_KEYS, the gathered rows only when rotating.
struct Layout {
  size_t status, khi, klo, qs, ks, mass, gmass, total;
};

Layout carve(int L, int H, int Hkv, int d, int B, int S, unsigned flags = 0) {
  Layout w;
  const size_t Ns = static_cast<size_t>(L / S), Nb = static_cast<size_t>(L / B);
  const bool pooled = (flags & RR_VAR_MEAN_KEYS) != 0;
  const bool rotate = (flags & RR_VAR_ROTATE) != 0;
  const size_t kbar = pooled ? round_up(Ns * Hkv * d * 2) : 0;
  const size_t gathered = round_up(Ns * H * d * 2);
  size_t off = kAlign;
  w.status = 0;
  w.khi = off; off += kbar;
  w.klo = off; off += kbar;
  w.qs = off; off += rotate ? gathered : 0;
  w.ks = off; off += (rotate && !pooled) ? gathered : 0;
  w.mass = off; off += round_up(static_cast<size_t>(H) * Nb * Nb * 4);
  w.gmass = off; off += (flags & RR_VAR_GQA_MASK) ? round_up(static_cast<size_t>(Hkv) * Nb * Nb * 4) : 0;
  w.total = off;
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

rr_status check_shape(int L, int H, int Hkv, int d, int B, int S, bool need_s) {
  if (L <= 0 || H <= 0 || Hkv <= 0 || d <= 0 || B <= 0) return RR_EINVAL;
  if (H % Hkv != 0) return RR_EINVAL;
  if (L % B != 0) return RR_EINVAL;
  if (need_s && (S <= 0 || B % S != 0)) return RR_EINVAL;
  if (d != 64 && d != 128) return RR_EUNSUPPORTED;
  if (B != 64 && B != 128) return RR_EUNSUPPORTED;
  if (L / B > rr::kMaxBlocks) return RR_EUNSUPPORTED;
  if (static_cast<long long>(L) * H * d >= (1ll << 40)) return RR_EUNSUPPORTED;
  return RR_OK;
}

// Enqueues the search (pooling or gathers, scores and block mass, Top-tau) with
// its scratch at ws laid out by w; the caller has validated everything and
// reset the status word g.status points to.
rr_status enqueue_search(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S, float tau,
                         unsigned flags, int head0, int32_t* count, int32_t* idx, float* mass, uint8_t* ws,
                         const Layout& w, const rr::DeviceGuardArgs& g, cudaStream_t s) {
  float* m = mass ? mass : reinterpret_cast<float*>(ws + w.mass);
  const bool rotate = (flags & RR_VAR_ROTATE) != 0, sampled = (flags & RR_VAR_MEAN_KEYS) == 0;
  const int g_heads = H / Hkv;
  rr::SearchSources src{q, ws + w.khi, ws + w.klo, 0, 0, head0};
  if (rotate) {
    if (rr::launch_gather_rotated(q, ws + w.qs, L, H, H, 1, d, S, s) != cudaSuccess) return RR_ECUDA;
    src.q = ws + w.qs;
    src.q_mode = 1;
  }
  if (!sampled) {
    if (rr::launch_pool_keys(k, ws + w.khi, ws + w.klo, L, Hkv, d, S, s) != cudaSuccess) return RR_ECUDA;
  } else if (rotate) {
    if (rr::launch_gather_rotated(k, ws + w.ks, L, H, Hkv, g_heads, d, S, s) != cudaSuccess) return RR_ECUDA;
    src.k_a = src.k_b = ws + w.ks;
    src.k_mode = 2;
  } else {
    src.k_a = src.k_b = k;
    src.k_mode = 1;
  }
  if (rr::launch_search(src, m, L, H, Hkv, d, B, S, g, s) != cudaSuccess) return RR_ECUDA;
  const int Nb = L / B;
  if (flags & RR_VAR_GQA_MASK) {
    float* gm = reinterpret_cast<float*>(ws + w.gmass);
    if (rr::launch_group_mass(m, gm, Hkv, g_heads, Nb, s) != cudaSuccess) return RR_ECUDA;
    if (rr::launch_top_tau(gm, Hkv, Nb, tau, count, idx, g_heads, s) != cudaSuccess) return RR_ECUDA;
  } else {
    if (rr::launch_top_tau(m, H, Nb, tau, count, idx, 1, s) != cudaSuccess) return RR_ECUDA;
  }
  return RR_OK;
}

// Workspace of rr_attention_host: the status word, two slots of one kv head's
// device copies (q [L, g, d], k and v [L, 1, d], o [L, g, d]), and the search
// scratch of one kv head's g heads (its own status word unused).
struct HostLayout {
  size_t status, slot[2], q, k, v, o, search, total;
  Layout sl;
};

HostLayout carve_host(int L, int H, int Hkv, int d, int B, int S) {
  HostLayout w;
  const int g = H / Hkv;
  const size_t qb = round_up(static_cast<size_t>(L) * g * d * 2), kb = round_up(static_cast<size_t>(L) * d * 2);
  w.status = 0;
  w.q = 0;
  w.k = qb;
  w.v = qb + kb;
  w.o = qb + 2 * kb;
  const size_t slot_bytes = 2 * qb + 2 * kb;
  w.slot[0] = kAlign;
  w.slot[1] = kAlign + slot_bytes;
  w.search = kAlign + 2 * slot_bytes;
  w.sl = carve(L, g, 1, d, B, S);
  w.total = w.search + w.sl.total;
  return w;
}

// Decode workspace: the status word and the search's arrival counters (per
// sequence and head), zeroed by one memset per call, the sampled scores [N, H, Lmax/S] fp32,
// the kept-block bitmaps [N, H, W] u32 (W = ceil(Lmax/B / 32)), the attention
// partials [(N Hkv + P) H/Hkv, d+2] fp32 (one per (row, attention CTA) pair, P
// <= kDecAttnCTAs), the block masses [N, H, Lmax/B] fp32, the search CTAs' maxima
// [N, H, kDecSearchChunks] fp32 and the prefix of block counts [N+1] i32.
struct DecodeLayout {
  size_t status, arrive, zero_bytes, scores, bits, part, mass, cmax, rowstart, total;
};

DecodeLayout carve_decode(int N, int Lmax, int H, int Hkv, int d, int B, int S) {
  DecodeLayout w;
  const size_t rows = static_cast<size_t>(N) * H;
  const size_t W = (static_cast<size_t>(Lmax / B) + 31) / 32;
  w.status = 0;
  w.arrive = 16;
  w.zero_bytes = w.arrive + rows * 4;
  size_t off = round_up(w.zero_bytes);
  w.scores = off; off += round_up(rows * (Lmax / S) * 4);
  w.bits = off; off += round_up(rows * W * 4);
  w.part = off;
  off += round_up((static_cast<size_t>(N) * Hkv + rr::kDecAttnCTAs) * static_cast<size_t>(H / Hkv) * (d + 2) * 4);
  w.mass = off; off += round_up(rows * static_cast<size_t>(Lmax / B) * 4);
  w.cmax = off; off += round_up(rows * rr::kDecSearchChunks * 4);
  w.rowstart = off; off += round_up((static_cast<size_t>(N) + 1) * 4);
  w.total = off;
  return w;
}

rr_status check_decode_shape(int N, int Lmax, int H, int Hkv, int d, int B, int S) {
  if (N <= 0 || Lmax <= 0 || H <= 0 || Hkv <= 0 || S <= 0) return RR_EINVAL;
  if (H % Hkv != 0 || B <= 0 || B % S != 0 || Lmax % B != 0) return RR_EINVAL;
  if (d != 64 && d != 128) return RR_EUNSUPPORTED;
  if (B != 64 && B != 128) return RR_EUNSUPPORTED;
  if (H / Hkv > 8) return RR_EUNSUPPORTED;
  if (Lmax / B > rr::kMaxBlocks) return RR_EUNSUPPORTED;
  if (static_cast<long long>(N) * Lmax >= (1ll << 31)) return RR_EUNSUPPORTED;
  return RR_OK;
}

rr_status check_ws(void* ws, size_t ws_bytes, const Layout& w) {
  if (!ws) return RR_EINVAL;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return RR_EALIGN;
  if (ws_bytes < w.total) return RR_EINVAL;
  return RR_OK;
}

}  // namespace

extern "C" {

rr_status rr_workspace_size(int L, int H, int Hkv, int d, int B, int S, size_t* bytes) {
  if (!bytes) return RR_EINVAL;
  rr_status st = check_shape(L, H, Hkv, d, B, S, true);
  if (st != RR_OK) return st;
  *bytes = carve(L, H, Hkv, d, B, S).total;
  return RR_OK;
}

rr_status rr_workspace_size_variant(int L, int H, int Hkv, int d, int B, int S, unsigned flags, size_t* bytes) {
  if (!bytes || (flags & ~kVarAll)) return RR_EINVAL;
  rr_status st = check_shape(L, H, Hkv, d, B, S, true);
  if (st != RR_OK) return st;
  *bytes = carve(L, H, Hkv, d, B, S, flags).total;
  return RR_OK;
}

rr_status rr_search_variant(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S, float tau,
                            unsigned flags, int32_t* count, int32_t* idx, float* mass, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (flags & ~kVarAll) return RR_EINVAL;
  rr_status st = check_shape(L, H, Hkv, d, B, S, true);
  if (st != RR_OK) return st;
  if (!(tau > 0.0f) || tau != tau) return RR_EINVAL;
  if (!q || !k || !count || !idx) return RR_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(count) || !aligned16(idx) || (mass && !aligned16(mass)))
    return RR_EALIGN;
  const Layout w = carve(L, H, Hkv, d, B, S, flags);
  if ((st = check_ws(workspace, workspace_bytes, w)) != RR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned int* status = reinterpret_cast<unsigned int*>(ws + w.status);
  const rr::DeviceGuardArgs g{status, g_wait_limit_ns};
  const Range range("rr_search");
  if (cudaMemsetAsync(status, 0, sizeof(unsigned int), s) != cudaSuccess) return RR_ECUDA;
  return enqueue_search(q, k, L, H, Hkv, d, B, S, tau, flags, 0, count, idx, mass, ws, w, g, s);
}

rr_status rr_search(const void* q, const void* k, int L, int H, int Hkv, int d, int B, int S, float tau,
                    int32_t* count, int32_t* idx, float* mass, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return rr_search_variant(q, k, L, H, Hkv, d, B, S, tau, 0u, count, idx, mass, workspace, workspace_bytes,
                           stream);
}

rr_status rr_sparse_attn(const void* q, const void* k, const void* v, int L, int H, int Hkv, int d, int B,
                         const int32_t* count, const int32_t* idx, void* o, void* workspace,
                         size_t workspace_bytes, void* stream) {
  rr_status st = check_shape(L, H, Hkv, d, B, 1, false);
  if (st != RR_OK) return st;
  if (!q || !k || !v || !count || !idx || !o || !workspace) return RR_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(count) || !aligned16(idx))
    return RR_EALIGN;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return RR_EALIGN;
  if (workspace_bytes < kAlign) return RR_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int* status = static_cast<unsigned int*>(workspace);
  const rr::DeviceGuardArgs g{status, g_wait_limit_ns};
  const Range range("rr_sparse_attn");
  if (cudaMemsetAsync(status, 0, sizeof(unsigned int), s) != cudaSuccess) return RR_ECUDA;
  if (rr::launch_bsfa(q, k, v, count, idx, o, L, H, Hkv, d, B, g, s) != cudaSuccess) return RR_ECUDA;
  return RR_OK;
}

rr_status rr_attention(const void* q, const void* k, const void* v, int L, int H, int Hkv, int d, int B, int S,
                       float tau, int32_t* count, int32_t* idx, void* o, void* workspace, size_t workspace_bytes,
                       void* stream) {
  rr_status st = check_shape(L, H, Hkv, d, B, S, true);
  if (st != RR_OK) return st;
  if (!v || !o) return RR_EINVAL;
  if (!aligned16(v) || !aligned16(o)) return RR_EALIGN;
  st = rr_search(q, k, L, H, Hkv, d, B, S, tau, count, idx, nullptr, workspace, workspace_bytes, stream);
  if (st != RR_OK) return st;
  // the search's status word stays in place: attention does not reset it
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int* status = static_cast<unsigned int*>(workspace);
  const rr::DeviceGuardArgs g{status, g_wait_limit_ns};
  const Range range("rr_attention: sparse attention");
  if (rr::launch_bsfa(q, k, v, count, idx, o, L, H, Hkv, d, B, g, s) != cudaSuccess) return RR_ECUDA;
  return RR_OK;
}

rr_status rr_mask_recall(const float* mass, const int32_t* count, const int32_t* idx, int H, int Nb,
                         float* recall, void* stream) {
  if (!mass || !count || !idx || !recall || H <= 0 || Nb <= 0) return RR_EINVAL;
  if (Nb > rr::kMaxBlocks) return RR_EUNSUPPORTED;
  if (!aligned16(mass) || !aligned16(count) || !aligned16(idx) || !aligned16(recall)) return RR_EALIGN;
  if (rr::launch_mask_recall(mass, count, idx, H, Nb, recall, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RR_ECUDA;
  return RR_OK;
}

rr_status rr_workspace_size_host(int L, int H, int Hkv, int d, int B, int S, size_t* bytes) {
  if (!bytes) return RR_EINVAL;
  rr_status st = check_shape(L, H, Hkv, d, B, S, true);
  if (st != RR_OK) return st;
  *bytes = carve_host(L, H, Hkv, d, B, S).total;
  return RR_OK;
}

rr_status rr_attention_host(const void* q_host, const void* k_host, const void* v_host, int L, int H, int Hkv,
                            int d, int B, int S, float tau, int32_t* count, int32_t* idx, void* o_host,
                            void* workspace, size_t workspace_bytes, void* stream, void* copy_stream) {
  rr_status st = check_shape(L, H, Hkv, d, B, S, true);
  if (st != RR_OK) return st;
  if (!(tau > 0.0f) || tau != tau) return RR_EINVAL;
  if (!q_host || !k_host || !v_host || !o_host || !count || !idx || !workspace) return RR_EINVAL;
  if (!aligned16(count) || !aligned16(idx)) return RR_EALIGN;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return RR_EALIGN;
  const HostLayout hl = carve_host(L, H, Hkv, d, B, S);
  if (workspace_bytes < hl.total) return RR_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = static_cast<cudaStream_t>(copy_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned int* status = reinterpret_cast<unsigned int*>(ws + hl.status);
  const rr::DeviceGuardArgs g{status, g_wait_limit_ns};
  const int gq = H / Hkv, Nb = L / B;
  const size_t row_q = static_cast<size_t>(H) * d * 2, row_kv = static_cast<size_t>(Hkv) * d * 2;
  const size_t wkv = static_cast<size_t>(d) * 2;

  // events: start (prior work on `stream` before the first copy), qk[slot]
  // (q and k of a kv head landed: its search may start), in[slot] (v landed
  // too), out[slot] (its kernels done), end (last copy)
  cudaEvent_t ev[8] = {};
  for (int i = 0; i < 8; ++i) {
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return RR_ECUDA;
    }
  }
  cudaEvent_t ev_start = ev[0], ev_end = ev[5];
  cudaEvent_t ev_in[2] = {ev[1], ev[2]}, ev_out[2] = {ev[3], ev[4]}, ev_qk[2] = {ev[6], ev[7]};
  // Work items: (kv head c, query heads h0 .. h0+gn of its group).  A kv head
  // is one item, except that the first item holds a single query head (its
  // inputs land sooner, so the kernels start sooner) and so does the last (its
  // O copy, which trails the last kernel, is smaller).  Each query head's search
  // and attention are independent of the others', so the results do not depend
  // on this split.
  struct Item { int c, h0, gn; };
  std::vector<Item> items;
  for (int c = 0; c < Hkv; ++c) {
    int h0 = 0, rem = gq;
    if (c == 0 && rem > 1) { items.push_back({c, 0, 1}); h0 = 1; --rem; }
    if (c == Hkv - 1 && rem > 1) {
      items.push_back({c, h0, rem - 1});
      items.push_back({c, h0 + rem - 1, 1});
    } else {
      items.push_back({c, h0, rem});
    }
  }
  const int n_items = static_cast<int>(items.size());
  auto h2d = [&](int n) {
    const Item& it = items[n];
    uint8_t* base = ws + hl.slot[n & 1];
    const size_t w = static_cast<size_t>(it.gn) * d * 2;   // this item's q (and o) row
    const uint8_t* qh = static_cast<const uint8_t*>(q_host) + (static_cast<size_t>(it.c) * gq + it.h0) * d * 2;
    const uint8_t* kh = static_cast<const uint8_t*>(k_host) + it.c * wkv;
    const uint8_t* vh = static_cast<const uint8_t*>(v_host) + it.c * wkv;
    return cudaMemcpy2DAsync(base + hl.k, wkv, kh, row_kv, wkv, L, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
           cudaMemcpy2DAsync(base + hl.q, w, qh, row_q, w, L, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
           cudaEventRecord(ev_qk[n & 1], cs) == cudaSuccess &&
           cudaMemcpy2DAsync(base + hl.v, wkv, vh, row_kv, wkv, L, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
           cudaEventRecord(ev_in[n & 1], cs) == cudaSuccess;
  };
  bool ok = cudaMemsetAsync(status, 0, sizeof(unsigned int), s) == cudaSuccess &&
            cudaEventRecord(ev_start, s) == cudaSuccess && cudaStreamWaitEvent(cs, ev_start, 0) == cudaSuccess;
  for (int n = 0; n < 2 && n < n_items && ok; ++n) ok = h2d(n);
  for (int n = 0; n < n_items && ok; ++n) {
    const Item& it = items[n];
    const int slot = n & 1;
    uint8_t* base = ws + hl.slot[slot];
    const int h_first = it.c * gq + it.h0;   // global index of the item's first query head
    const size_t w = static_cast<size_t>(it.gn) * d * 2;
    int32_t* cc = count + static_cast<size_t>(h_first) * Nb;
    int32_t* ic = idx + static_cast<size_t>(h_first) * Nb * Nb;
    const Range range("rr_attention_host: item");
    ok = cudaStreamWaitEvent(s, ev_qk[slot], 0) == cudaSuccess;
    if (ok) {
      ok = enqueue_search(base + hl.q, base + hl.k, L, it.gn, 1, d, B, S, tau, 0u, h_first, cc, ic, nullptr,
                          ws + hl.search, hl.sl, g, s) == RR_OK;
    }
    ok = ok && cudaStreamWaitEvent(s, ev_in[slot], 0) == cudaSuccess;
    ok = ok && rr::launch_bsfa(base + hl.q, base + hl.k, base + hl.v, cc, ic, base + hl.o, L, it.gn, 1, d, B, g,
                               s) == cudaSuccess;
    ok = ok && cudaEventRecord(ev_out[slot], s) == cudaSuccess && cudaStreamWaitEvent(cs, ev_out[slot], 0) == cudaSuccess;
    ok = ok && cudaMemcpy2DAsync(static_cast<uint8_t*>(o_host) + static_cast<size_t>(h_first) * d * 2, row_q,
                                 base + hl.o, w, w, L, cudaMemcpyDeviceToHost, cs) == cudaSuccess;
    // the slot's inputs are free once its kernels are done (waited above)
    if (ok && n + 2 < n_items) ok = h2d(n + 2);
  }
  ok = ok && cudaEventRecord(ev_end, cs) == cudaSuccess && cudaStreamWaitEvent(s, ev_end, 0) == cudaSuccess;
  for (int i = 0; i < 8; ++i) cudaEventDestroy(ev[i]);   // released once their work completes
  return ok ? RR_OK : RR_ECUDA;
}

rr_status rr_decode_workspace_size(int N, int Lmax, int H, int Hkv, int d, int B, int S, size_t* bytes) {
  if (!bytes) return RR_EINVAL;
  const rr_status st = check_decode_shape(N, Lmax, H, Hkv, d, B, S);
  if (st != RR_OK) return st;
  *bytes = carve_decode(N, Lmax, H, Hkv, d, B, S).total;
  return RR_OK;
}

rr_status rr_decode_variant(const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, int N,
                            int Lmax, int H, int Hkv, int d, int B, int S, float tau, unsigned flags, int32_t* count,
                            int32_t* idx, void* o, void* workspace, size_t workspace_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(RR_VAR_GQA_MASK)) return RR_EINVAL;
  rr_status st = check_decode_shape(N, Lmax, H, Hkv, d, B, S);
  if (st != RR_OK) return st;
  if (!(tau > 0.0f) || tau != tau) return RR_EINVAL;
  if (!q || !k_cache || !v_cache || !lens || !count || !idx || !o || !workspace) return RR_EINVAL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(count) ||
      !aligned16(idx) || (reinterpret_cast<uintptr_t>(lens) & 3u))
    return RR_EALIGN;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return RR_EALIGN;
  const DecodeLayout w = carve_decode(N, Lmax, H, Hkv, d, B, S);
  if (workspace_bytes < w.total) return RR_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned int* status = reinterpret_cast<unsigned int*>(ws + w.status);
  const rr::DeviceGuardArgs g{status, g_wait_limit_ns};
  const rr::DecodeScratch sc{reinterpret_cast<float*>(ws + w.scores),       reinterpret_cast<uint32_t*>(ws + w.bits),
                             reinterpret_cast<float*>(ws + w.part),         reinterpret_cast<float*>(ws + w.mass),
                             reinterpret_cast<float*>(ws + w.cmax),         reinterpret_cast<unsigned int*>(ws + w.arrive),
                             reinterpret_cast<int32_t*>(ws + w.rowstart)};
  const Range range("rr_decode");
  if (cudaMemsetAsync(ws, 0, w.zero_bytes, s) != cudaSuccess) return RR_ECUDA;   // status and arrival counters
  if (rr::launch_decode(q, k_cache, v_cache, lens, N, Lmax, H, Hkv, d, B, S, tau, (flags & RR_VAR_GQA_MASK) != 0,
                        count, idx, o, sc, g, s) != cudaSuccess)
    return RR_ECUDA;
  return RR_OK;
}

rr_status rr_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* lens, int N, int Lmax,
                    int H, int Hkv, int d, int B, int S, float tau, int32_t* count, int32_t* idx, void* o,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return rr_decode_variant(q, k_cache, v_cache, lens, N, Lmax, H, Hkv, d, B, S, tau, 0u, count, idx, o, workspace,
                           workspace_bytes, stream);
}

rr_status rr_mask_to_dense(const int32_t* count, const int32_t* idx, int H, int Nb, uint8_t* dense, void* stream) {
  if (!count || !idx || !dense || H <= 0 || Nb <= 0) return RR_EINVAL;
  if (Nb > rr::kMaxBlocks) return RR_EUNSUPPORTED;
  if (!aligned16(count) || !aligned16(idx)) return RR_EALIGN;
  if (rr::launch_mask_to_dense(count, idx, H, Nb, dense, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RR_ECUDA;
  return RR_OK;
}

rr_status rr_check_status(void* workspace, void* stream) {
  if (!workspace) return RR_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int host = 0;
  if (cudaMemcpyAsync(&host, workspace, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return RR_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RR_ECUDA;
  if ((host & 0xFFu) == rr::kStatusTimeoutCode) return RR_ETIMEOUT;
  if ((host & 0xFFu) == rr::kStatusMaskCode) return RR_EMASK;
  if ((host & 0xFFu) == rr::kStatusLenCode) return RR_EINVAL;
  return host == 0 ? RR_OK : RR_ECUDA;
}

uint64_t rr_set_wait_limit_ns(uint64_t ns) {
  const uint64_t prev = g_wait_limit_ns;
  g_wait_limit_ns = ns;
  return prev;
}

const char* rr_status_string(rr_status s) {
  switch (s) {
    case RR_OK: return "ok";
    case RR_EINVAL: return "invalid argument";
    case RR_EUNSUPPORTED: return "unsupported shape (d and B must be 64 or 128, L/B <= 4096)";
    case RR_EALIGN: return "misaligned pointer (16 bytes; workspace 256 bytes)";
    case RR_ECUDA: return "CUDA error";
    case RR_ETIMEOUT: return "device-side wait timed out";
    case RR_ESCRATCH: return "shape needs more scratch than rr_search_static's 32 MiB array";
    case RR_EMASK: return "block list outside the mask format (row not computed)";
  }
  return "unknown status";
}

}  // extern "C"
