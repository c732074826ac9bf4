// rr_internal.h — launchers shared between the kernel files and the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace rr {

struct DeviceGuardArgs {
  unsigned int* status;   // workspace status word
  uint64_t limit_ns;      // bound of every device-side wait
};

// Stride pooling of keys: kbar = mean of the S keys of each stride, stored as a
// bf16 pair (hi = bf16(kbar), lo = bf16(kbar - hi)).  k: [L, Hkv, d].
cudaError_t launch_pool_keys(const void* k, void* khi, void* klo, int L, int Hkv, int d, int S,
                             cudaStream_t stream);

// Sampled-score search: block mass[h, I, J] (unnormalised) for J <= I.
//   q_mode 0: q is [L, H, d], rows read at offset h mod S in each stride;
//          1: q holds the sampled rows, gathered into [Ns, H, d].
//   k_mode 0: k_a / k_b are the stride means' bf16 (hi, lo) parts [Ns, Hkv, d];
//          1: k_a is k [L, Hkv, d], one key per stride at offset h mod S;
//          2: k_a holds the sampled keys, gathered into [Ns, H, d].
// head0: global index of head 0 of this launch (the sampled offsets of q_mode 0
// and k_mode 1 are (h + head0) mod S), for searches run on a slice of the heads.
struct SearchSources {
  const void* q;
  const void* k_a;
  const void* k_b;
  int q_mode;
  int k_mode;
  int head0;
};
cudaError_t launch_search(const SearchSources& src, float* mass, int L, int H, int Hkv, int d, int B, int S,
                          const DeviceGuardArgs& g, cudaStream_t stream);

// Rows at the rotating offsets: dst[i, h, :] = src[i*S + (h + i) mod S, h / div, :]
// for i < L/S, h < H (src [L, heads, d], dst [L/S, H, d], bf16).
cudaError_t launch_gather_rotated(const void* src, void* dst, int L, int H, int src_heads, int div, int d, int S,
                                  cudaStream_t stream);

// GQA group mass: dst[kv, I, J] = sum of src[kv*g + t, I, J] over t < g (all I, J).
cudaError_t launch_group_mass(const float* src, float* dst, int Hkv, int g, int Nb, cudaStream_t stream);

// Adaptive Top-tau with protection of the last query block.
// rows = heads of `mass` ([rows, Nb, Nb]); each row's selection is written to the
// rep output heads rows*rep.. (rep = 1: one output head per mass head).
cudaError_t launch_top_tau(const float* mass, int rows, int Nb, float tau, int32_t* count, int32_t* idx, int rep,
                           cudaStream_t stream);

// Causal block-sparse attention over the mask.
cudaError_t launch_bsfa(const void* q, const void* k, const void* v, const int32_t* count,
                        const int32_t* idx, void* o, int L, int H, int Hkv, int d, int B,
                        const DeviceGuardArgs& g, cudaStream_t stream);

// Dense uint8 view [H, Nb, Nb] of a block mask (diagnostics).
cudaError_t launch_mask_to_dense(const int32_t* count, const int32_t* idx, int H, int Nb, uint8_t* dense,
                                 cudaStream_t stream);

// Share of each row's block mass kept by a mask (diagnostics).
cudaError_t launch_mask_recall(const float* mass, const int32_t* count, const int32_t* idx, int H, int Nb,
                               float* recall, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit to `bytes` once per device
// (the attribute belongs to the current device's context): `done` holds one
// bit per device index below 64; higher indices set it on every call.
template <typename Kernel>
cudaError_t set_smem_limit_once(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Low byte of the workspace status word when a device-side wait ran out.
constexpr unsigned kStatusTimeoutCode = 5u;
// Low byte of the workspace status word when the attention kernel met a block
// list outside the mask format (bits 8..31: the row h*Nb + I, saturated).
constexpr unsigned kStatusMaskCode = 7u;

// Low byte of the workspace status word when a decode call met a cache length
// outside [1, Lmax] (bits 8..31: the sequence, saturated).
constexpr unsigned kStatusLenCode = 8u;

// Decode-stage scratch (workspace regions): sampled scores [N, H, Lmax/S] fp32,
// kept-block bitmaps [N, H, W] u32 (W = ceil(Lmax/B / 32)), and the attention
// partials [N, H, NC, d + 2] fp32 (max, sum, output columns per 16-block chunk,
// NC = ceil(Lmax/B / 16)).
struct DecodeScratch {
  float* scores;          // sampled scores [N, H, Lmax/S] fp32
  uint32_t* bits;         // kept-block bitmaps [N, H, W] u32
  float* part;            // attention partials [(N Hkv + P) H/Hkv, d + 2] fp32
  float* mass;            // block masses [N, H, Lmax/B] fp32
  float* cmax;            // per search CTA: its max [N, H, kDecSearchChunks] fp32
  unsigned int* arrive;   // per (sequence, head): search CTAs done [N, H] u32, zero before the launch
  int32_t* rowstart;      // prefix of the sequences' block counts [N + 1] i32
};

// Search CTAs per (sequence, head) and attention CTAs per launch, at most.
constexpr int kDecSearchChunks = 32;
constexpr int kDecAttnCTAs = 1024;

// Decode stage: search, block-sparse attention and combine for one new token per
// sequence.  q, o: [N, H, d]; k, v: [N, Lmax, Hkv, d]; lens: [N] cache lengths.
// gqa: one mask per GQA group, selected on the group's summed block mass.
cudaError_t launch_decode(const void* q, const void* k, const void* v, const int32_t* lens, int N, int Lmax, int H,
                          int Hkv, int d, int B, int S, float tau, bool gqa, int32_t* count, int32_t* idx, void* o,
                          const DecodeScratch& w, const DeviceGuardArgs& g, cudaStream_t stream);

// Largest Nb = L/B the kernels accept (bounded by the on-chip list / sort buffers).
constexpr int kMaxBlocks = 4096;

}  // namespace rr
