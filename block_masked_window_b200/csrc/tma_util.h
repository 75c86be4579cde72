// Host-side TMA tensor-map construction for the tcgen05 attention kernel.
//
// The K and V caches [B, Hkv, S, 128] bf16 are described as 2-D tensors of B*Hkv*S rows of
// 128 channels; a box is 64 channels (128 bytes, the SWIZZLE_128B atom width) by kTileKeys
// rows, so one key tile is two boxes per operand. Q [B, W, Hq, 128] is a 3-D tensor
// (channel, head, b*W + window row); a box of (64, G, W) gathers the R = W*G rows that share
// one KV head in window-row-major order, i.e. row r = i*G + g.
//
// cuTensorMapEncodeTiled is reached through the runtime's driver entry point, so the library
// does not link libcuda directly.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "pbd_common.cuh"

namespace la {

constexpr int kTileKeys = 128;  // keys per tile of the tcgen05 kernel

struct TmaMaps {
  alignas(64) CUtensorMap k;
  alignas(64) CUtensorMap v;
  alignas(64) CUtensorMap q;
  alignas(64) CUtensorMap o;   // output rows, store map (no swizzle, whole 256-byte rows)
};

int tc_ctas_per_sm();
int tc_tile_keys();
int tc_segment_units();

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
  }
  return fn;
}

// pool_rows > 0: paged caches, K/V are page pools of pool_rows rows read as 64-row boxes (one
// box per page piece of a key tile).
inline cudaError_t make_tma_maps(const Problem& p, TmaMaps* m, long long pool_rows = 0) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t rows = pool_rows > 0 ? (cuuint64_t)pool_rows : (cuuint64_t)p.B * p.Hkv * p.S;
  {
    cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, rows};
    cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)(pool_rows > 0 ? 64 : kTileKeys)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&m->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)p.k, dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    r = enc(&m->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)p.v, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.W};
    cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)p.Hq * kHeadDim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)p.G, (cuuint32_t)p.W};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&m->q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)p.q, dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // Same geometry over `out`, whole 128-channel rows, for the epilogue's TMA stores.
    cuuint32_t obox[3] = {(cuuint32_t)kHeadDim, (cuuint32_t)p.G, (cuuint32_t)p.W};
    r = enc(&m->o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)p.out, dims, strides, obox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

// Prefill maps: q [B*T rows, Hq, 128] with a box of (64 channels, 1 head, 128 tokens); the K
// and V caches as for the decode kernel (64 channels x 128 rows), and the fp16 copy of V
// [B*Hkv*Tp rows, 128] the same way, all with the 128-byte swizzle.
inline cudaError_t make_prefill_maps(const PrefillProblem& p, CUtensorMap* mq, CUtensorMap* mk,
                                     CUtensorMap* mv, CUtensorMap* mv16) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  {
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.T};
    cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)p.Hq * kHeadDim * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)p.q, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const cuuint64_t rows = (cuuint64_t)p.B * p.Hkv * p.S;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (enc(mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)p.k, dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)p.v, dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cuuint64_t dims16[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)p.B * p.Hkv * p.Tp};
  if (enc(mv16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)p.v16, dims16, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

}  // namespace la
