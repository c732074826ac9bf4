// tmap.h — host-side construction of TMA tensor maps (bf16, 128-byte swizzle).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rr {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// A bf16 tensor of `rank` dims (dims[0] innermost, contiguous), byte strides
// for dims 1..rank-1, box `box` (box[0] * 2 bytes must be <= 128), 128B swizzle,
// out-of-range elements read as zero.
inline bool make_tmap_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                  const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [rows, heads, d] bf16 tensor viewed as (d, heads, rows); box (64, 1, box_rows):
// one head, box_rows consecutive rows, 64 columns of d per load.
inline bool make_tmap_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads, uint64_t d,
                           uint32_t box_rows) {
  const uint64_t dims[3] = {d, heads, rows};
  const uint64_t strides[2] = {d * 2, heads * d * 2};
  const uint32_t box[3] = {64, 1, box_rows};
  return make_tmap_bf16(m, base, 3, dims, strides, box);
}

// The round-robin sampled-query view of q [L, H, d]: (d, H, S, Ns) with
// element (x, h, t, i) = q[i*S + t, h, x]; box (64, 1, 1, box_rows).
inline bool make_tmap_sampled(CUtensorMap* m, const void* q, uint64_t L, uint64_t H, uint64_t d,
                              uint64_t S, uint32_t box_rows) {
  const uint64_t dims[4] = {d, H, S, L / S};
  const uint64_t strides[3] = {d * 2, H * d * 2, S * H * d * 2};
  const uint32_t box[4] = {64, 1, 1, box_rows};
  return make_tmap_bf16(m, q, 4, dims, strides, box);
}

}  // namespace rr
