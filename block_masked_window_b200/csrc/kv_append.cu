// Step a1: window K/V append into the cache (RK3588 model card, "How it differs from the
// original", item 1: the prefix KV is reused and the window's tokens are written after it,
// with no explicit rollback of stale speculative rows).
//
// One warp per (b, w, kv head): lanes 0..15 move the 256-byte K row as 16-byte vectors,
// lanes 16..31 the V row. Pure data movement, bit-exact.
#include "pbd_common.cuh"
#include "pbd_kernels.h"

namespace la {

__global__ void __launch_bounds__(256) kv_append_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ window_lens, int B, int W, int Hkv, int S) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long rows = (long long)B * W * Hkv;
  if (row >= rows) return;
  const int h = (int)(row % Hkv);
  const int w = (int)((row / Hkv) % W);
  const int b = (int)(row / ((long long)Hkv * W));
  const int P = __ldg(seq_lens + b);
  const int wb = window_lens ? __ldg(window_lens + b) : W;   // this sequence's window
  if (P < 0 || wb < 1 || wb > W || (long long)P + wb > S) return;  // flagged by the attention kernels
  if (w >= wb) return;                         // padding row of a shorter window
  constexpr int kVec = kHeadDim * 2 / 16;      // 16 vectors of 16 bytes per row
  const int c = lane & (kVec - 1);
  const size_t src = (size_t)row * kVec + c;   // [B, W, Hkv, D] row-major
  const size_t dst = (((size_t)b * Hkv + h) * S + (size_t)(P + w)) * kVec + c;
  if (lane < kVec) {
    k_cache[dst] = __ldg(k_new + src);
  } else {
    v_cache[dst] = __ldg(v_new + src);
  }
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seq_lens, const int32_t* window_lens, int B,
                             int W, int Hkv, int S, cudaStream_t stream) {
  const long long rows = (long long)B * W * Hkv;
  const int warps_per_block = 8;
  const unsigned grid = (unsigned)((rows + warps_per_block - 1) / warps_per_block);
  return launch_pdl(kv_append_kernel, dim3(grid), dim3(32 * warps_per_block), 0, stream,
                    static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                    static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), seq_lens,
                    window_lens, B, W, Hkv, S);
}

}  // namespace la
