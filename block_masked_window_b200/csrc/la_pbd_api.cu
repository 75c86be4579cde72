// C ABI of the PBD window-attention library (declared in include/la_pbd.h): argument
// validation, workspace sizing, kernel selection and launch. Nothing here allocates device
// memory or synchronises, except la_pbd_check.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <mutex>

#include "la_pbd.h"
#include "pbd_common.cuh"
#include "pbd_kernels.h"
#include "tma_util.h"

namespace {

using la::Problem;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
std::mutex g_mu;

cudaError_t sm_count(int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_sm_count[dev] = n;
  }
  *out = g_sm_count[dev];
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Encoded TMA tensor maps of recent calls. Encoding the four maps of a call is host work of
// the same order as the launches themselves, and a decode loop calls with the same few
// buffers again and again (one set per layer). A map holds only the addresses, sizes and
// strides it was made from, all of which are in the key, so an entry is valid for any call
// with an equal key, on any device.
struct MapKey {
  const void* ptr[4];            // k, v, q, out
  int B, Hq, Hkv, G, W, S;
  long long pool_rows;
};
struct MapEntry {
  MapKey key;
  la::TmaMaps maps;
  bool used;
};
constexpr int kMapCache = 128;
MapEntry g_map_cache[kMapCache];
int g_map_next = 0;
std::mutex g_map_mu;

cudaError_t tma_maps_for(const Problem& p, long long pool_rows, la::TmaMaps* out) {
  MapKey key;
  std::memset(&key, 0, sizeof(key));   // (padding too: keys are compared bytewise)
  key.ptr[0] = p.k;
  key.ptr[1] = p.v;
  key.ptr[2] = p.q;
  key.ptr[3] = p.out;
  key.B = p.B;
  key.Hq = p.Hq;
  key.Hkv = p.Hkv;
  key.G = p.G;
  key.W = p.W;
  key.S = p.S;
  key.pool_rows = pool_rows;
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (const MapEntry& e : g_map_cache) {
      if (e.used && std::memcmp(&e.key, &key, sizeof(key)) == 0) {
        *out = e.maps;
        return cudaSuccess;
      }
    }
  }
  la::TmaMaps m;
  const cudaError_t e = la::make_tma_maps(p, &m, pool_rows);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_map_mu);
  MapEntry& slot = g_map_cache[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCache;
  slot.key = key;
  slot.maps = m;
  slot.used = true;
  *out = m;
  return cudaSuccess;
}

la_status check_cfg(const la_pbd_cfg* cfg, int32_t W) {
  if (!cfg) return LA_ERR_INVALID_ARG;
  if (cfg->batch < 1 || cfg->batch > la::kMaxBatch) return LA_ERR_INVALID_ARG;
  if (cfg->num_kv_heads < 1 || cfg->num_q_heads < 1) return LA_ERR_INVALID_ARG;
  if (cfg->max_seq < 1) return LA_ERR_INVALID_ARG;
  if (!std::isfinite(cfg->scale)) return LA_ERR_INVALID_ARG;
  if (W < 1 || W > la::kMaxWindow) return LA_ERR_INVALID_ARG;
  if (cfg->mask_mode != LA_MASK_PBD && cfg->mask_mode != LA_MASK_CAUSAL_WINDOW)
    return LA_ERR_INVALID_ARG;
  if (cfg->algo != LA_ALGO_AUTO && cfg->algo != LA_ALGO_TCGEN05 && cfg->algo != LA_ALGO_SIMT)
    return LA_ERR_INVALID_ARG;
  if (cfg->head_dim != la::kHeadDim) return LA_ERR_UNSUPPORTED;
  if (cfg->num_q_heads % cfg->num_kv_heads != 0) return LA_ERR_UNSUPPORTED;
  // Per-head prefix sums and TMA row coordinates are int32: B * Hkv * S_max < 2^31.
  if ((long long)cfg->batch * cfg->num_kv_heads * cfg->max_seq >= (1LL << 31))
    return LA_ERR_UNSUPPORTED;
  if ((long long)cfg->batch * cfg->num_kv_heads > 65535) return LA_ERR_UNSUPPORTED;
  const long long R = (long long)W * (cfg->num_q_heads / cfg->num_kv_heads);
  if (R > 128) return LA_ERR_UNSUPPORTED;
  if (cfg->algo == LA_ALGO_TCGEN05 && R > 80) return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

// Kernel choice for a validated configuration.
int pick_algo(const la_pbd_cfg* cfg, int R) {
  if (cfg->algo != LA_ALGO_AUTO) return cfg->algo;
  return (R <= 80) ? LA_ALGO_TCGEN05 : LA_ALGO_SIMT;
}

size_t slots_for(const la_pbd_cfg* cfg, int sms) {
  return (size_t)sms * la::kMaxCtasPerSm + (size_t)cfg->batch * cfg->num_kv_heads;
}

la_status fill_problem(const la_pbd_cfg* cfg, int32_t W, Problem* p) {
  std::memset(p, 0, sizeof(*p));
  p->B = cfg->batch;
  p->Hq = cfg->num_q_heads;
  p->Hkv = cfg->num_kv_heads;
  p->G = cfg->num_q_heads / cfg->num_kv_heads;
  p->W = W;
  p->S = cfg->max_seq;
  p->R = W * p->G;
  p->rows_pad = la::round_up(p->R, 16);
  p->mask_mode = cfg->mask_mode;
  p->scale_log2 = cfg->scale * 1.4426950408889634f;
  p->wait_limit_ns = la::kDefaultWaitLimitNs;
  return LA_OK;
}

// Grid size: the resident capacity, but no more CTAs than the largest possible unit stream
// (every sequence at full capacity) can keep busy at c_min units each.
int grid_for(const Problem& p, int capacity) {
  const long long max_units =
      (long long)p.B * p.Hkv * ((p.S + p.unit - 1) / p.unit + p.seg_units);
  const long long useful = (max_units + p.c_min - 1) / p.c_min;
  return (int)(useful < capacity ? (useful < 1 ? 1 : useful) : capacity);
}

}  // namespace

extern "C" {

int32_t la_version(void) { return 100; }

const char* la_status_string(la_status s) {
  switch (s) {
    case LA_OK: return "ok";
    case LA_ERR_INVALID_ARG: return "invalid argument";
    case LA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LA_ERR_WORKSPACE: return "workspace missing or too small";
    case LA_ERR_CUDA: return "CUDA error";
    case LA_ERR_SEQ_OVERFLOW: return "a sequence had seq_len < 0 or seq_len + window > max_seq";
    case LA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
  }
  return "unknown status";
}

int32_t la_pbd_algo(const la_pbd_cfg* cfg, int32_t W) {
  const la_status st = check_cfg(cfg, W);
  if (st != LA_OK) return -(int32_t)st;
  return pick_algo(cfg, W * (cfg->num_q_heads / cfg->num_kv_heads));
}

size_t la_pbd_workspace_bytes(const la_pbd_cfg* cfg, int32_t W) {
  if (check_cfg(cfg, W) != LA_OK) return 0;
  int sms = 0;
  if (sm_count(&sms) != cudaSuccess) return 0;
  const int G = cfg->num_q_heads / cfg->num_kv_heads;
  const int rows_pad = la::round_up(W * G, 16);
  return la::kSlotsOffset + slots_for(cfg, sms) * la::slot_floats(rows_pad) * sizeof(float);
}

static la_status check_attn_args(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* seq_lens, int32_t W,
                                 const void* out, const void* workspace,
                                 size_t workspace_bytes) {
  la_status st = check_cfg(cfg, W);
  if (st != LA_OK) return st;
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return LA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(seq_lens, 4))
    return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return LA_ERR_WORKSPACE;
  const size_t need = la_pbd_workspace_bytes(cfg, W);
  if (need == 0) return LA_ERR_CUDA;
  if (workspace_bytes < need) return LA_ERR_WORKSPACE;
  return LA_OK;
}

la_status la_pbd_workspace_init(void* workspace, size_t bytes, void* stream) {
  if (!workspace || bytes < la::kSlotsOffset || !aligned(workspace, 256)) return LA_ERR_WORKSPACE;
  cudaError_t e = cudaMemsetAsync(workspace, 0, la::kHeaderBytes, (cudaStream_t)stream);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_kv_append(const la_pbd_cfg* cfg, const void* k_new, const void* v_new, void* k_cache,
                       void* v_cache, const int32_t* seq_lens, int32_t W, void* stream) {
  la_status st = check_cfg(cfg, W);
  if (st != LA_OK) return st;
  if (!k_new || !v_new || !k_cache || !v_cache || !seq_lens) return LA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(seq_lens, 4))
    return LA_ERR_INVALID_ARG;
  cudaError_t e = la::launch_kv_append(k_new, v_new, k_cache, v_cache, seq_lens, nullptr, cfg->batch, W,
                                       cfg->num_kv_heads, cfg->max_seq, (cudaStream_t)stream);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

}  // extern "C"

namespace {

// Attention launch (attention kernel + merge) for validated arguments. With k_new / v_new
// non-null the caller has chosen the tcgen05 kernel, which then also appends the window
// (caches written through k_cache / v_cache).
// Paged caches for attn_launch (null block_table: contiguous caches).
struct Paging {
  const int32_t* block_table = nullptr;
  int pages_per_seq = 0, page_size = 0, num_pages = 0;
};

// Self-test of the device-side failure detection (la_pbd_selftest_timeout).
struct Selftest {
  long long wait_limit_ns = la::kDefaultWaitLimitNs;
  int stall = 0;
};

la_status attn_launch(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens,
                      const int32_t* window_lens, int32_t W, void* out, void* workspace,
                      const void* k_new, const void* v_new, void* stream,
                      const Paging& pg = Paging(), const Selftest& st = Selftest()) {
  Problem p;
  fill_problem(cfg, W, &p);
  p.wait_limit_ns = st.wait_limit_ns;
  p.stall_test = st.stall;
  p.window_lens = window_lens;
  if (pg.block_table) {
    p.block_table = pg.block_table;
    p.pages_per_seq = pg.pages_per_seq;
    p.page_size = pg.page_size;
    p.S = pg.pages_per_seq * pg.page_size;   // key capacity of a sequence
  }
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k_cache);
  p.v = static_cast<const __nv_bfloat16*>(v_cache);
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  char* ws = static_cast<char*>(workspace);
  p.hdr = reinterpret_cast<la::WsHeader*>(ws);
  p.pre_g = reinterpret_cast<int*>(ws + la::kPrefixOffset);
  p.partials = reinterpret_cast<float*>(ws + la::kSlotsOffset);

  int sms = 0;
  if (sm_count(&sms) != cudaSuccess) return LA_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  const int algo = pick_algo(cfg, p.R);
  if (k_new && algo != LA_ALGO_TCGEN05) return LA_ERR_INVALID_ARG;
  if (pg.block_table && algo != LA_ALGO_TCGEN05) return LA_ERR_UNSUPPORTED;
  if (algo == LA_ALGO_TCGEN05) {
    p.k_new = static_cast<const __nv_bfloat16*>(k_new);
    p.v_new = static_cast<const __nv_bfloat16*>(v_new);
    p.kc = const_cast<__nv_bfloat16*>(p.k);
    p.vc = const_cast<__nv_bfloat16*>(p.v);
    la::TmaMaps maps;
    const long long pool_rows =
        pg.block_table ? (long long)pg.num_pages * p.Hkv * pg.page_size : 0;
    if (tma_maps_for(p, pool_rows, &maps) != cudaSuccess) return LA_ERR_CUDA;
    p.unit = la::tc_tile_keys();
    p.c_min = 1;
    p.seg_units = 0;
    const int cap = sms * la::tc_ctas_per_sm();
    // The fixed segment cost only matters when a CTA can get several tiles. When even full
    // caches have no more tiles than the grid has CTAs, every CTA gets at most one tile, and
    // the cost would only add CTAs without work.
    if ((long long)p.B * p.Hkv * ((p.S + p.unit - 1) / p.unit) > cap)
      p.seg_units = la::tc_segment_units();
    p.num_ctas = grid_for(p, cap);
    e = la::launch_attn_tc(p, &maps.k, &maps.v, &maps.q, &maps.o, s);
  } else {
    int per_sm = 0;
    e = la::simt_max_ctas_per_sm(p.R, p.B, &per_sm);
    if (e != cudaSuccess) return LA_ERR_CUDA;
    if (per_sm < 1) return LA_ERR_UNSUPPORTED;
    if (per_sm > la::kMaxCtasPerSm) per_sm = la::kMaxCtasPerSm;
    p.unit = la::simt_tile_keys();
    p.c_min = 1;
    p.seg_units = 0;
    p.num_ctas = grid_for(p, sms * per_sm);
    e = la::launch_attn_simt(p, s);
  }
  if (e != cudaSuccess) return LA_ERR_CUDA;
  e = la::launch_combine(p, s);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

}  // namespace

extern "C" {

la_status la_pbd_attn(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, int32_t W, void* out,
                      void* workspace, size_t workspace_bytes, void* stream) {
  la_status st = check_attn_args(cfg, q, k_cache, v_cache, seq_lens, W, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  return attn_launch(cfg, q, k_cache, v_cache, seq_lens, nullptr, W, out, workspace, nullptr, nullptr,
                     stream);
}

la_status la_noop_chain(int32_t launches, int32_t ctas, int32_t threads, void* stream) {
  if (launches < 0 || ctas < 1 || threads < 1 || threads > 1024) return LA_ERR_INVALID_ARG;
  for (int i = 0; i < launches; ++i)
    if (la::launch_noop(ctas, threads, (cudaStream_t)stream) != cudaSuccess) return LA_ERR_CUDA;
  return LA_OK;
}

la_status la_pbd_plan_params(int32_t algo, int32_t* unit_keys, int32_t* seg_units) {
  if (!unit_keys || !seg_units) return LA_ERR_INVALID_ARG;
  if (algo == LA_ALGO_TCGEN05) {
    *unit_keys = la::tc_tile_keys();
    *seg_units = la::tc_segment_units();
  } else if (algo == LA_ALGO_SIMT) {
    *unit_keys = la::simt_tile_keys();
    *seg_units = 0;
  } else {
    return LA_ERR_INVALID_ARG;
  }
  return LA_OK;
}

int32_t la_pbd_plan(const la_pbd_cfg* cfg, int32_t W, const int32_t* seq_lens_host,
                    int32_t num_ctas, int32_t unit_keys, int32_t seg_units,
                    int32_t* segments, int32_t max_segments) {
  la_status st = check_cfg(cfg, W);
  if (st != LA_OK) return -(int32_t)st;
  if (!seq_lens_host || num_ctas < 1 || unit_keys < 1 || seg_units < 0 || max_segments < 0 ||
      (max_segments > 0 && !segments))
    return -(int32_t)LA_ERR_INVALID_ARG;
  Problem p;
  fill_problem(cfg, W, &p);
  p.seq_lens = seq_lens_host;
  p.unit = unit_keys;
  p.c_min = 1;
  p.seg_units = seg_units;
  p.num_ctas = num_ctas;
  std::vector<int> pre(p.B + 1, 0);
  for (int b = 0; b < p.B; ++b) pre[b + 1] = pre[b] + la::plan_units_of(p, la::visible_len(p, b));
  const long long T = (long long)p.Hkv * pre[p.B];
  int32_t count = 0;
  for (int c = 0; c < num_ctas; ++c) {
    la::SegmentIter it = la::plan_begin(p, pre.data(), c, T);
    la::Segment sg;
    while (it.next(p, pre.data(), c, sg)) {
      if (count < max_segments) {
        int32_t* r = segments + 6 * (size_t)count;
        r[0] = c; r[1] = sg.b; r[2] = sg.h; r[3] = sg.j0; r[4] = sg.j1;
        r[5] = sg.whole ? -1 : sg.slot;
      }
      ++count;
    }
  }
  return count;
}

la_status la_pbd_step(const la_pbd_cfg* cfg, const void* q, const void* k_new, const void* v_new,
                      void* k_cache, void* v_cache, const int32_t* seq_lens, int32_t W,
                      void* out, void* workspace, size_t workspace_bytes, void* stream) {
  // Validate both halves before enqueuing anything.
  la_status st = check_attn_args(cfg, q, k_cache, v_cache, seq_lens, W, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return LA_ERR_INVALID_ARG;
  // The tcgen05 kernel appends the window itself (one launch less per layer); the CUDA-core
  // kernel runs after the append kernel.
  if (pick_algo(cfg, W * (cfg->num_q_heads / cfg->num_kv_heads)) == LA_ALGO_TCGEN05)
    return attn_launch(cfg, q, k_cache, v_cache, seq_lens, nullptr, W, out, workspace, k_new, v_new,
                       stream);
  st = la_kv_append(cfg, k_new, v_new, k_cache, v_cache, seq_lens, W, stream);
  if (st != LA_OK) return st;
  return attn_launch(cfg, q, k_cache, v_cache, seq_lens, nullptr, W, out, workspace, nullptr, nullptr,
                     stream);
}

la_status la_pbd_attn_varwin(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* seq_lens,
                             const int32_t* window_lens, int32_t W_max, void* out,
                             void* workspace, size_t workspace_bytes, void* stream) {
  la_status st = check_attn_args(cfg, q, k_cache, v_cache, seq_lens, W_max, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  if (!window_lens || !aligned(window_lens, 4)) return LA_ERR_INVALID_ARG;
  return attn_launch(cfg, q, k_cache, v_cache, seq_lens, window_lens, W_max, out, workspace,
                     nullptr, nullptr, stream);
}

la_status la_pbd_step_varwin(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                             const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seq_lens, const int32_t* window_lens,
                             int32_t W_max, void* out, void* workspace, size_t workspace_bytes,
                             void* stream) {
  la_status st = check_attn_args(cfg, q, k_cache, v_cache, seq_lens, W_max, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  if (!window_lens || !aligned(window_lens, 4)) return LA_ERR_INVALID_ARG;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return LA_ERR_INVALID_ARG;
  if (pick_algo(cfg, W_max * (cfg->num_q_heads / cfg->num_kv_heads)) == LA_ALGO_TCGEN05)
    return attn_launch(cfg, q, k_cache, v_cache, seq_lens, window_lens, W_max, out, workspace,
                       k_new, v_new, stream);
  cudaError_t e = la::launch_kv_append(k_new, v_new, k_cache, v_cache, seq_lens, window_lens,
                                       cfg->batch, W_max, cfg->num_kv_heads, cfg->max_seq,
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return LA_ERR_CUDA;
  return attn_launch(cfg, q, k_cache, v_cache, seq_lens, window_lens, W_max, out, workspace,
                     nullptr, nullptr, stream);
}

// Prefill workspace: the header, one flag per 128-row V tile [B, Hkv, ntiles] (int32), then
// V as fp16 [B, Hkv, Tp, D] at a 1024-byte boundary (Tp = ntiles * 128 >= t_max).
struct PrefillWs {
  size_t flags, v16, total;
  int ntiles, Tp;
};
static PrefillWs prefill_ws(const la_pbd_cfg* cfg, int32_t t_max) {
  PrefillWs w;
  w.ntiles = (t_max + 127) / 128;
  w.Tp = w.ntiles * 128;
  const size_t tiles = (size_t)cfg->batch * cfg->num_kv_heads * w.ntiles;
  w.flags = (size_t)la::kHeaderBytes;
  w.v16 = (w.flags + tiles * sizeof(int32_t) + 1023) / 1024 * 1024;
  w.total = w.v16 + tiles * 128 * (size_t)la::kHeadDim * 2;
  return w;
}

size_t la_block_prefill_workspace_bytes(const la_pbd_cfg* cfg, int32_t t_max) {
  if (check_cfg(cfg, 1) != LA_OK || t_max < 1) return 0;
  if ((long long)cfg->batch * cfg->num_kv_heads * (((long long)t_max + 127) / 128 * 128) >= (1LL << 31))
    return 0;
  return prefill_ws(cfg, t_max).total;
}

static la_status prefill_launch(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* seq_lens, int32_t t_max,
                                int32_t block_size, void* out, void* workspace,
                                size_t workspace_bytes, void* stream, long long wait_limit_ns,
                                int stall) {
  la_status st = check_cfg(cfg, 1);
  if (st != LA_OK) return st;
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return LA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(seq_lens, 4))
    return LA_ERR_INVALID_ARG;
  if (t_max < 1 || block_size < 1) return LA_ERR_INVALID_ARG;
  if ((long long)cfg->batch * t_max >= (1LL << 31)) return LA_ERR_UNSUPPORTED;
  if ((long long)cfg->batch * cfg->num_kv_heads * (((long long)t_max + 127) / 128 * 128) >= (1LL << 31))
    return LA_ERR_UNSUPPORTED;
  if (!workspace || !aligned(workspace, 256)) return LA_ERR_WORKSPACE;
  const PrefillWs w = prefill_ws(cfg, t_max);
  if (workspace_bytes < w.total) return LA_ERR_WORKSPACE;
  la::PrefillProblem p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k_cache);
  p.v = static_cast<const __nv_bfloat16*>(v_cache);
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.hdr = static_cast<la::WsHeader*>(workspace);
  p.B = cfg->batch;
  p.Hq = cfg->num_q_heads;
  p.Hkv = cfg->num_kv_heads;
  p.G = cfg->num_q_heads / cfg->num_kv_heads;
  p.S = cfg->max_seq;
  p.T = t_max;
  p.bs = block_size;
  p.scale_log2 = cfg->scale * 1.4426950408889634f;
  p.wait_limit_ns = wait_limit_ns;
  p.stall_test = stall;
  p.v16_ok = reinterpret_cast<int*>(static_cast<char*>(workspace) + w.flags);
  p.v16 = reinterpret_cast<__half*>(static_cast<char*>(workspace) + w.v16);
  p.ntiles = w.ntiles;
  p.Tp = w.Tp;
  CUtensorMap mq, mk, mv, mv16;
  if (la::make_prefill_maps(p, &mq, &mk, &mv, &mv16) != cudaSuccess) return LA_ERR_CUDA;
  cudaError_t e = la::launch_prefill_tc(p, &mq, &mk, &mv, &mv16, (cudaStream_t)stream);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_block_prefill(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* seq_lens, int32_t t_max,
                           int32_t block_size, void* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return prefill_launch(cfg, q, k_cache, v_cache, seq_lens, t_max, block_size, out, workspace,
                        workspace_bytes, stream, la::kDefaultWaitLimitNs, 0);
}

la_status la_block_prefill_selftest_timeout(const la_pbd_cfg* cfg, const void* q,
                                            const void* k_cache, const void* v_cache,
                                            const int32_t* seq_lens, int32_t t_max,
                                            int32_t block_size, void* out, void* workspace,
                                            size_t workspace_bytes, int64_t wait_limit_ns,
                                            void* stream) {
  if (wait_limit_ns < 1000 || wait_limit_ns > la::kDefaultWaitLimitNs) return LA_ERR_INVALID_ARG;
  return prefill_launch(cfg, q, k_cache, v_cache, seq_lens, t_max, block_size, out, workspace,
                        workspace_bytes, stream, wait_limit_ns, 1);
}

static la_status check_paging(const la_pbd_cfg* cfg, int32_t W, const int32_t* block_table,
                              int32_t pages_per_seq, int32_t page_size, int32_t num_pages) {
  if (!block_table || !aligned(block_table, 4)) return LA_ERR_INVALID_ARG;
  if (pages_per_seq < 1 || num_pages < 1 || page_size < 64 || page_size % 64 != 0)
    return LA_ERR_INVALID_ARG;
  if ((long long)num_pages * cfg->num_kv_heads * page_size >= (1LL << 31)) return LA_ERR_UNSUPPORTED;
  if ((long long)cfg->batch * cfg->num_kv_heads * pages_per_seq * page_size >= (1LL << 31))
    return LA_ERR_UNSUPPORTED;
  if (pick_algo(cfg, W * (cfg->num_q_heads / cfg->num_kv_heads)) != LA_ALGO_TCGEN05)
    return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

la_status la_pbd_attn_paged(const la_pbd_cfg* cfg, const void* q, const void* k_pool,
                            const void* v_pool, const int32_t* block_table,
                            int32_t pages_per_seq, int32_t page_size, int32_t num_pages,
                            const int32_t* seq_lens, int32_t W, void* out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  la_status st = check_attn_args(cfg, q, k_pool, v_pool, seq_lens, W, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  st = check_paging(cfg, W, block_table, pages_per_seq, page_size, num_pages);
  if (st != LA_OK) return st;
  Paging pg;
  pg.block_table = block_table;
  pg.pages_per_seq = pages_per_seq;
  pg.page_size = page_size;
  pg.num_pages = num_pages;
  return attn_launch(cfg, q, k_pool, v_pool, seq_lens, nullptr, W, out, workspace, nullptr,
                     nullptr, stream, pg);
}

la_status la_pbd_step_paged(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                            const void* v_new, void* k_pool, void* v_pool,
                            const int32_t* block_table, int32_t pages_per_seq,
                            int32_t page_size, int32_t num_pages, const int32_t* seq_lens,
                            int32_t W, void* out, void* workspace, size_t workspace_bytes,
                            void* stream) {
  la_status st = check_attn_args(cfg, q, k_pool, v_pool, seq_lens, W, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  st = check_paging(cfg, W, block_table, pages_per_seq, page_size, num_pages);
  if (st != LA_OK) return st;
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return LA_ERR_INVALID_ARG;
  Paging pg;
  pg.block_table = block_table;
  pg.pages_per_seq = pages_per_seq;
  pg.page_size = page_size;
  pg.num_pages = num_pages;
  return attn_launch(cfg, q, k_pool, v_pool, seq_lens, nullptr, W, out, workspace, k_new,
                     v_new, stream, pg);
}

la_status la_pbd_selftest_timeout(const la_pbd_cfg* cfg, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* seq_lens, int32_t W,
                                   void* out, void* workspace, size_t workspace_bytes,
                                   int64_t wait_limit_ns, void* stream) {
  if (wait_limit_ns < 1000 || wait_limit_ns > la::kDefaultWaitLimitNs) return LA_ERR_INVALID_ARG;
  la_status st = check_attn_args(cfg, q, k_cache, v_cache, seq_lens, W, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  if (pick_algo(cfg, W * (cfg->num_q_heads / cfg->num_kv_heads)) != LA_ALGO_TCGEN05)
    return LA_ERR_UNSUPPORTED;
  Selftest t;
  t.wait_limit_ns = wait_limit_ns;
  t.stall = 1;
  return attn_launch(cfg, q, k_cache, v_cache, seq_lens, nullptr, W, out, workspace, nullptr,
                     nullptr, stream, Paging(), t);
}

la_status la_pbd_selftest_replan(const la_pbd_cfg* cfg, const void* q, const void* k_new,
                                 const void* v_new, void* k_cache, void* v_cache,
                                 const int32_t* seq_lens, int32_t W, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  la_status st = check_attn_args(cfg, q, k_cache, v_cache, seq_lens, W, out, workspace,
                                 workspace_bytes);
  if (st != LA_OK) return st;
  if ((k_new == nullptr) != (v_new == nullptr)) return LA_ERR_INVALID_ARG;
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16))) return LA_ERR_INVALID_ARG;
  if (pick_algo(cfg, W * (cfg->num_q_heads / cfg->num_kv_heads)) != LA_ALGO_TCGEN05)
    return LA_ERR_UNSUPPORTED;
  Selftest t;
  t.stall = 2;
  return attn_launch(cfg, q, k_cache, v_cache, seq_lens, nullptr, W, out, workspace, k_new,
                     v_new, stream, Paging(), t);
}

la_status la_pbd_check(void* workspace, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return LA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t err = 0;
  cudaError_t e = cudaMemcpyAsync(&err, workspace, sizeof(err), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return LA_ERR_CUDA;
  if (err & la::kErrTimeout) return LA_ERR_TIMEOUT;
  if (err & la::kErrSeqOverflow) return LA_ERR_SEQ_OVERFLOW;
  return LA_OK;
}

}  // extern "C"
