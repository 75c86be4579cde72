// Shared device-side pieces of the PBD window-attention kernels: constants, the workspace
// header, the partial-result slot layout and the flattened split-KV work plan.
//
// Work plan ("stream-K" over key tiles). Sequence s = b * Hkv + h (batch b, KV head h) has
// N_b = P_b + W visible keys (0 if P_b is invalid), cut into U_b = ceil(N_b / unit) units of
// `unit` keys (the attention kernel's key tile; only a sequence's last unit is partial). All
// sequences are laid end to end in one flattened stream of T = Hkv * sum_b U_b units. CTA c
// of a grid of G CTAs owns units [lo(c), lo(c + 1)) with lo(c) = floor(c * T / G) when
// T >= G, so every CTA gets floor(T / G) or ceil(T / G) whole tiles (at least one) whatever
// the mix of prefix lengths; when T < G, CTA c takes unit c alone. No tile is ever shared by
// two CTAs, and every CTA between the first and the last of a sequence holds a piece of it.
// The part of a sequence that falls in one CTA is a segment; a CTA
// that holds a whole sequence writes its final output directly, every other segment writes
// an (m, l, acc) partial to slot c + s, and the combine kernel merges them. Slot c + s is
// unique because CTAs and sequences advance together along the stream.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace la {

constexpr int kHeadDim = 128;
constexpr int kMaxBatch = 4096;
constexpr int kMaxWindow = 16;
constexpr int kHeaderBytes = 256;
constexpr long long kDefaultWaitLimitNs = 2000000000LL;   // bounded device-side waits: ~2 s

// Sticky error bits in the workspace header (first 32-bit word).
constexpr uint32_t kErrSeqOverflow = 1u;
constexpr uint32_t kErrTimeout = 2u;

struct WsHeader {
  uint32_t err;
  uint32_t pad[63];
};

// Launch-wide parameters shared by the attention and combine kernels.
struct Problem {
  const __nv_bfloat16* q;       // [B, W, Hq, D]
  const __nv_bfloat16* k;       // [B, Hkv, S, D]
  const __nv_bfloat16* v;       // [B, Hkv, S, D]
  const int32_t* seq_lens;      // [B]
  const int32_t* window_lens;   // [B] window length W_b <= W of each sequence, or null (all W)
  // Paged caches (tcgen05 kernel only): k and v are page pools [num_pages, Hkv, page_size, D]
  // and key j of sequence b lives in page block_table[b * pages_per_seq + j / page_size];
  // null block_table = contiguous caches [B, Hkv, S, D].
  const int32_t* block_table;
  int pages_per_seq, page_size;
  __nv_bfloat16* out;           // [B, W, Hq, D]
  // Fused window append (tcgen05 kernel only; null otherwise): the window's keys/values are
  // read from k_new / v_new [B, W, Hkv, D] and written into the caches kc / vc (= k, v).
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* kc;
  __nv_bfloat16* vc;
  float* partials;              // slots, see slot_floats
  WsHeader* hdr;
  int* pre_g;                   // [B+1] prefix sums of plan units, written by attention CTA 0
  int B, Hq, Hkv, G, W, S;      // G = Hq / Hkv; W = the (longest) window length
  int R;                        // rows per sequence = W * G
  int rows_pad;                 // R rounded up to 16: rows per partial slot
  int mask_mode;                // 0 = PBD window, 1 = causal window
  int num_ctas;                 // grid size of the attention kernel (fixes the chunk size)
  int unit;                     // keys per plan unit (the attention kernel's key tile)
  int c_min;                    // minimum units per CTA
  int seg_units;                // plan units charged per (sequence, KV head) besides its tiles
  float scale_log2;             // scale * log2(e)
  long long wait_limit_ns;      // limit of every bounded device-side wait (tcgen05 kernel)
  int stall_test;               // self-tests: 1 = the first S^T completion is never signalled,
                                //             2 = the plan made before the wait is rejected
};

// Launch parameters of the block-causal prefill kernel.
struct PrefillProblem {
  const __nv_bfloat16* q;       // [B, T, Hq, D]
  const __nv_bfloat16* k;       // [B, Hkv, S, D], rows [0, T_b) hold the sequence
  const __nv_bfloat16* v;       // [B, Hkv, S, D]
  const int32_t* seq_lens;      // [B] tokens T_b of each sequence
  __nv_bfloat16* out;           // [B, T, Hq, D]
  WsHeader* hdr;
  int B, Hq, Hkv, G, S, T;      // T = padded token count of q / out
  int bs;                       // block size of the block mask
  float scale_log2;
  long long wait_limit_ns;      // limit of every bounded device-side wait
  int stall_test;               // self-test: 1 = the first S_0 completion is never signalled
  // V as fp16 (workspace): [B, Hkv, Tp, D], rows [0, T_b) of each (sequence, KV head), and one
  // flag per 128-row tile, [B, Hkv, ntiles]: 1 when the tile converted exactly enough for the
  // fp16 product (see prefill_v16_kernel).
  __half* v16;
  int* v16_ok;
  int Tp, ntiles;               // Tp = ntiles * 128 >= T
};

__host__ __device__ inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

__host__ __device__ inline size_t slot_floats(int rows_pad) {
  return (size_t)rows_pad * (kHeadDim + 2);
}
// Slot layout: m[rows_pad] (log2 domain), l[rows_pad], acc[rows_pad][D].
__device__ inline float* slot_ptr(const Problem& p, int slot) {
  return p.partials + (size_t)slot * slot_floats(p.rows_pad);
}

// Loads of seq_lens / window_lens. kL2 = true reads through L2 only (ld.global.cg): the only
// form used before a kernel's dependency wait, so that no L1 line of a value the previous
// kernel may still write can be hit after the wait. (Host-callable for the plan inspection
// entry point, where the arrays are host memory.)
template <bool kL2 = false>
__host__ __device__ inline int load_len(const int32_t* a) {
#ifdef __CUDA_ARCH__
  return kL2 ? __ldcg(a) : __ldg(a);
#else
  return *a;
#endif
}

// Window length of sequence b (W when all sequences share it).
template <bool kL2 = false>
__host__ __device__ inline int window_of(const Problem& p, int b) {
  if (!p.window_lens) return p.W;
  return load_len<kL2>(p.window_lens + b);
}

// Visible keys P + w of a sequence with prefix P and window w (0 marks an invalid prefix or
// window length).
__host__ __device__ inline int visible_of(const Problem& p, int P, int w) {
  if (P < 0 || w < 1 || w > p.W || (long long)P + w > (long long)p.S) return 0;
  return P + w;
}

// Visible keys of sequence b, P_b + W_b.
template <bool kL2 = false>
__host__ __device__ inline int visible_len(const Problem& p, int b) {
  return visible_of(p, load_len<kL2>(p.seq_lens + b), window_of<kL2>(p, b));
}

// Key tiles of a sequence with n visible keys.
__host__ __device__ inline int units_of(const Problem& p, int n) { return (n + p.unit - 1) / p.unit; }

// Plan units of one (sequence, KV head) with n visible keys: seg_units units that stand for
// the fixed cost of a segment (loading Q, the first tile's exact maximum, the epilogue),
// followed by one unit per key tile. Charging the fixed cost in the plan gives a CTA whose
// run crosses sequence starts fewer tiles, so that CTAs with several segments do not finish
// last. An invalid sequence (n = 0) has no units.
__host__ __device__ inline int plan_units_of(const Problem& p, int n) {
  return n > 0 ? units_of(p, n) + p.seg_units : 0;
}

// Block-wide prefix sum of the plan units U_b (plan_units_of) into pre[0..B] (pre[0] = 0,
// pre[b+1] = U_0 + ... + U_b).
// Every thread of the block must call it. `warp_tot` needs one int per warp (<= 32).
template <bool kL2 = false>
__device__ inline void plan_prefix(const Problem& p, int* pre, int* warp_tot) {
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, wid = tid >> 5;
  const int nwarps = (nthr + 31) >> 5;
  int carry = 0;
  if (tid == 0) pre[0] = 0;
  for (int base = 0; base < p.B; base += nthr) {
    int b = base + tid;
    int x = (b < p.B) ? plan_units_of(p, visible_len<kL2>(p, b)) : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int t = (lane < nwarps) ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      if (lane < nwarps) warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    int add = carry + (wid > 0 ? warp_tot[wid - 1] : 0);
    if (b < p.B) pre[b + 1] = x + add;
    carry += warp_tot[nwarps - 1];
    __syncthreads();
  }
}

// First unit of CTA c (c in [0, num_ctas]) for a stream of T units (identical in every kernel
// that uses the plan): floor(c * T / G) when T >= G, else min(c, T).
__host__ __device__ inline long long plan_lo(const Problem& p, long long T, int c) {
  if (T < p.num_ctas) return c < T ? (long long)c : T;
  return (long long)c * T / p.num_ctas;
}

// The CTA that owns unit x (0 <= x < T): the largest c with plan_lo(c) <= x, i.e.
// c * T < (x + 1) * G when T >= G, else x.
__host__ __device__ inline int plan_cta_of(const Problem& p, long long T, long long x) {
  if (T < p.num_ctas) return (int)x;
  return (int)(((x + 1) * p.num_ctas - 1) / T);
}

// Largest b with Hkv * pre[b] <= pos (pos < T). Never returns a zero-length sequence.
__host__ __device__ inline int plan_find_batch(const Problem& p, const int* pre, long long pos) {
  int lo = 0, hi = p.B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((long long)p.Hkv * pre[mid] <= pos) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct Segment {
  int b, h;        // batch, KV head
  int n;           // visible keys of the sequence (N_b = P_b + W_b)
  int w;           // window length of the sequence (W_b)
  int j0, j1;      // key range of this segment, 0 <= j0 < j1 <= n, j0 a multiple of unit
  bool whole;      // the segment is the whole sequence
  int slot;        // partial slot (when !whole)
};

// Iterator over the segments of CTA `c`. The units of (b, h) start at s0: seg_units fixed-cost
// units, then its key tiles from t0 = s0 + seg_units on. A CTA whose run holds only fixed-cost
// units of (b, h) gets no segment of it; the CTA holding tile 0 does the sequence's first
// segment.
struct SegmentIter {
  long long pos, end;
  int b, h;
  template <bool kL2 = false>
  __host__ __device__ bool next(const Problem& p, const int* pre, int c, Segment& sg) {
    while (pos < end) {
      int u = pre[b + 1] - pre[b];
      long long s0 = (long long)p.Hkv * pre[b] + (long long)h * u;
      if (u == 0 || pos >= s0 + u) {  // advance to the next sequence
        if (++h == p.Hkv) { h = 0; ++b; }
        continue;
      }
      const long long t0 = s0 + p.seg_units;
      const long long hi = (end < s0 + u) ? end : s0 + u;
      const long long lo = pos > t0 ? pos : t0;
      pos = hi;
      if (hi <= t0) continue;  // only fixed-cost units of (b, h) in this CTA
      const int n = visible_len<kL2>(p, b);
      sg.b = b; sg.h = h; sg.n = n; sg.w = window_of<kL2>(p, b);
      sg.j0 = (int)(lo - t0) * p.unit;
      const int e = (int)(hi - t0) * p.unit;
      sg.j1 = e < n ? e : n;
      sg.whole = (lo == t0 && hi == s0 + u);
      sg.slot = c + b * p.Hkv + h;
      return true;
    }
    return false;
  }
};

// CTAs that hold the first and the last key tile of (b, h), whose units start at s0 = off
// and number u > 0 (stream of T units): the sequence is split iff they differ, and its partial
// results sit in slots c + b * Hkv + h for c in [first, last].
__host__ __device__ inline void plan_tile_ctas(const Problem& p, long long off, int u, long long T,
                                               int* first, int* last) {
  *first = plan_cta_of(p, T, off + p.seg_units);
  *last = plan_cta_of(p, T, off + u - 1);
}

__host__ __device__ inline SegmentIter plan_begin(const Problem& p, const int* pre, int c, long long T) {
  SegmentIter it;
  it.pos = plan_lo(p, T, c);
  it.end = plan_lo(p, T, c + 1);
  it.b = 0; it.h = 0;
  if (it.pos < T) {
    int b = plan_find_batch(p, pre, it.pos);
    int u = pre[b + 1] - pre[b];
    long long off = it.pos - (long long)p.Hkv * pre[b];
    it.b = b;
    it.h = u > 0 ? (int)(off / u) : 0;
    if (it.h >= p.Hkv) it.h = p.Hkv - 1;
  }
  return it;
}

// Output row r of sequence (b, h): window row i = r / G, query head h*G + r % G.
__device__ inline size_t out_row_offset(const Problem& p, int b, int h, int r) {
  int i = r / p.G, g = r - i * p.G;
  return (((size_t)b * p.W + i) * p.Hq + (size_t)h * p.G + g) * kHeadDim;
}

// Number of keys visible to row r (window row i = r / G) of a sequence of n = P + w visible
// keys with a window of w rows: all n (PBD mask) or P + i + 1 (causal window); rows of the
// padding (i >= w) see nothing.
__device__ inline int row_limit(const Problem& p, int n, int w, int r) {
  const int i = r / p.G;
  if (i >= w) return 0;
  if (p.mask_mode == 0) return n;
  return n - w + i + 1;
}

// Rows need their own key limits: the causal-window mask or per-sequence windows.
__host__ __device__ inline bool row_limits(const Problem& p) {
  return p.mask_mode != 0 || p.window_lens != nullptr;
}

// Programmatic dependent launch. Every kernel of the library is launched so that it may start
// while the previous kernel of the stream is still running, and waits for its predecessor
// (completion and memory visibility) before the first access to global memory that a
// predecessor may have written. Every CTA executes the wait before it can exit, so a kernel
// completes only after its predecessor did: the ordering is transitive along the stream.
// A kernel signals that its successor may start right away, except the attention kernels,
// which signal after their wait: when the merge kernel starts, everything before the
// attention kernel has completed, so the merge may read seq_lens and window_lens (which the
// attention kernel does not write) before its own wait. Launched without the attribute, both
// instructions are no-ops.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ inline float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace la
