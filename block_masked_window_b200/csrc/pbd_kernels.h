// Host-side launchers of the PBD kernels (internal to the library; the public C ABI is
// include/la_pbd.h).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "pbd_common.cuh"

namespace la {

// Launch with programmatic stream serialization allowed (see pdl_wait in pbd_common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seq_lens, const int32_t* window_lens, int B, int W,
                             int Hkv, int S, cudaStream_t stream);

// Empty kernel with programmatic dependent launch (launch-floor measurements).
cudaError_t launch_noop(int ctas, int threads, cudaStream_t stream);

// CUDA-core split-KV attention (any R = W * G <= 128).
int simt_rows_per_thread(int R);
int simt_tile_keys();
size_t simt_smem_bytes(int R, int B);
cudaError_t simt_max_ctas_per_sm(int R, int B, int* ctas);
cudaError_t launch_attn_simt(const Problem& p, cudaStream_t stream);

// tcgen05 + TMA split-KV attention (R <= 80).
size_t tc_smem_bytes(int R, int B);
cudaError_t launch_attn_tc(const Problem& p, const void* tmap_k, const void* tmap_v,
                           const void* tmap_q, const void* tmap_o, cudaStream_t stream);

// tcgen05 + TMA block-causal prefill (one CTA per 128 query rows of a (sequence, head)).
size_t prefill_smem_bytes();
// Launches the V conversion (prefill_v16_kernel) and then the prefill kernel.
cudaError_t launch_prefill_tc(const PrefillProblem& p, const void* tmap_q, const void* tmap_k,
                              const void* tmap_v, const void* tmap_v16, cudaStream_t stream);

// Merge of the per-split partials into the bf16 output.
cudaError_t launch_combine(const Problem& p, cudaStream_t stream);

// Workspace carve-up shared by the launchers and the C ABI.
constexpr size_t kPrefixOffset = kHeaderBytes;                               // int[B+1]
constexpr size_t kPrefixBytes = ((size_t)(kMaxBatch + 1) * 4 + 255) / 256 * 256;
constexpr size_t kSlotsOffset = kPrefixOffset + kPrefixBytes;
constexpr int kMaxCtasPerSm = 4;

}  // namespace la
