// la_pbd_attn_static: the window-attention entry point for callers that cannot allocate
// device memory.
//
// Some callers have no way to provide the scratch buffer that la_pbd_attn needs: a plugin
// hosted by an inference engine that owns all device memory and hands its kernels no
// workspace, or a latency-critical decode loop that forbids cudaMalloc because the call can
// synchronise the whole device and take an unbounded time. This entry point serves them: it
// runs exactly the same kernels as la_pbd_attn, but their scratch (error header, prefix sums
// and split partials) lives in one file-scope device array, kStaticScratchBytes (32 MiB)
// large, that every GPU holds from the moment the library's code is loaded on it until the
// process exits. No device memory is allocated or freed by the call.
#include <cstdint>

#include "la_pbd.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;

// The shared scratch. In host code this name is only a stand-in for the symbol: its device
// address must come from cudaGetSymbolAddress with the device current.
static __device__ __align__(256) unsigned char g_pbd_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device. Looked up on every call (a
// table lookup once the module is loaded), so no address outlives a device reset. Under CUDA
// lazy module loading (the default since CUDA 12.2) the first lookup on a device loads this
// module there and reserves the array: that first call belongs in set-up code.
la_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_pbd_scratch) != cudaSuccess || p == nullptr) return LA_ERR_CUDA;
  *out = p;
  return LA_OK;
}

}  // namespace

extern "C" la_status la_pbd_attn_static(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                                        const void* v_cache, const int32_t* seq_lens,
                                        int32_t window_len, void* out, void* stream) {
  // Configuration errors first, as la_pbd_attn reports them (nothing is enqueued).
  const int32_t algo = la_pbd_algo(cfg, window_len);
  if (algo < 0) return (la_status)(-algo);
  const size_t need = la_pbd_workspace_bytes(cfg, window_len);
  if (need == 0) return LA_ERR_CUDA;   // valid configuration, but the device query failed
  if (need > kStaticScratchBytes) return LA_ERR_WORKSPACE;
  void* scratch = nullptr;
  la_status st = scratch_address(&scratch);
  if (st != LA_OK) return st;
  return la_pbd_attn(cfg, q, k_cache, v_cache, seq_lens, window_len, out, scratch,
                     kStaticScratchBytes, stream);
}
