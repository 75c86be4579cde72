// tcgen05 + TMA split-KV PBD window attention for sm_100a.
//
// Steps a2..a5 of one PBD decode step (LocateAnything-3B for RK3588 model card, "How it
// differs from the original", item 1: the window attends bidirectionally to itself and
// causally to the prefix, so every window row sees keys [0, P_b + W)). The R = W * G query
// rows that share one KV head (window row i, grouped head g -> row q = i*G + g) are the
// narrow N side of two tensor-core products per 128-key tile, and the keys (or channels) are
// the full-rate M = 128 side:
//   S^T = K  Q^T   (M = 128 keys,     N = NQ rows,       K = 128 channels) -> TMEM fp32
//   O^T = V^T P^T  (M = 128 channels, N = 2 NQ (hi, lo), K = 128 keys)     -> TMEM fp32
// The softmax row sums are not a tensor-core product: softmax thread t (key t of every tile)
// adds its fp32 p values to NQ partial sums kept in its own TMEM lane, after it has handed
// the tile's P^T to the MMA, and the 128 lanes are reduced once per segment. So the single
// MMA-issuing thread issues 16 instructions per tile, not 24.
// NQ = R rounded up to 16 (48 for the PBD window of 6 rows x 8 grouped heads; up to 80, the
// window of 10 rows that the RKLLM engine sends after 5 accepted tokens). P is split
// into P_hi + P_lo (both bf16, residual ~2^-17 P) so that the bf16 tensor-core product keeps
// fp32-level accuracy; both halves ride in one N = 2 NQ MMA that reads the V tile once.
//
// Online softmax with a lazy reference maximum: per row q the kernel keeps a reference m_q
// (log2 domain) and uses p = 2^(x - m_q). The reference is raised (and O, l rescaled) only
// when some score of a tile exceeds it by more than 2^8, which a CTA-wide vote detects
// without reducing across keys; the full cross-key maximum is computed only then (always on a
// segment's first tile). O accumulates in TMEM over the whole segment, so a tile without a
// rescale touches O only through the MMA.
//
// Roles (224 threads, 1 CTA per SM):
//   warp 0      TMA producer of Q (once per segment, double-buffered) and the K ring
//   warp 6      TMA producer of the V ring (so neither ring waits on the other)
//   warp 1      TMEM owner and single-thread MMA issuer (non-blocking: issues whichever of
//               the next S^T or the next O^T product is ready first)
//   warps 2..5  softmax: thread t of the 128 reads TMEM lane t, i.e. key t of the S^T tile,
//               channel t of the O^T accumulator and the row-sum partials of key lane t
//
// Shared-memory operand layouts: K, V and Q use the 128-byte swizzle written by TMA (K-major
// for K and Q, MN-major for V as the A operand of O^T); P^T is written by the softmax
// threads as an MN-major, non-swizzled operand (8x8 core matrices: rows of 16 bytes, key
// groups 128 bytes apart, row groups 2048 bytes apart), one 16-byte store per 8 rows.
//
// Options of the same kernel: the window append fused into the producers (la_pbd_step), key
// limits per row (causal-window mask, per-sequence window lengths), and paged caches (a
// template parameter, so that the contiguous kernels' code is unchanged). Before waiting for
// the previous kernel of the stream, a small batch's first key tiles are prefetched into L2
// from a guess of the plan. The epilogue stages a whole sequence's bf16 output rows in shared
// memory for one TMA store; a split sequence's fp32 partial rows go straight from registers
// to their slot.
//
// Every mbarrier wait is bounded: after a limit (2 s by default, set per call) the CTA raises
// the sticky timeout flag in the workspace header, the other roles stop at their next wait,
// in-flight copies and MMAs are drained with bounded waits, TMEM is freed and the kernel
// returns. A self-test option withholds the first S^T completion signal so that this path
// runs (la_pbd_selftest_timeout).
#include "pbd_common.cuh"
#include "pbd_kernels.h"
#include "tc_util.cuh"
#include "tma_util.h"

namespace la {
namespace {

using namespace tc;

constexpr int kNT = kTileKeys;          // 128 keys per tile
constexpr int kSegUnits = 3;            // plan units charged per segment (tc_segment_units)
constexpr int kKStages = 2;
constexpr int kSBufs = 4;               // S^T buffers in TMEM (most): QK may run kSBufs-1 tiles ahead
constexpr int kThreadsTc = 224;
constexpr int kTmemCols = 512;
constexpr int kHalfBytes = kNT * 128;   // 128 rows x 128 B: one swizzle column of a K/V tile
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr float kLazyThreshold = 8.f;   // log2 units: p stays <= 2^8 between rescales
constexpr int kNamedBarSoftmax = 1;

// Barrier indices (K ring, V ring sized at run time up to kMaxVStages). Every barrier is waited
// with a phase parity, which is only sound if its producer can never complete two phases
// ahead of a waiter. Each ring below is sized so that refilling a slot requires its previous
// consumer to have finished: e.g. the softmax can only refill a P^T buffer after the PV
// product that read it completed, so P-full is per buffer (a single P-full barrier could be
// lapped while the MMA issuer is busy).
constexpr int kMaxVStages = 3;
constexpr int kBarKFull = 0;
constexpr int kBarKEmpty = kBarKFull + kKStages;
constexpr int kBarVFull = kBarKEmpty + kKStages;
constexpr int kBarVEmpty = kBarVFull + kMaxVStages;
constexpr int kBarQFull = kBarVEmpty + kMaxVStages;   // [2]: Q is double-buffered
constexpr int kBarQEmpty = kBarQFull + 2;            // [2]
constexpr int kBarSFull = kBarQEmpty + 2;            // [kSBufs]
constexpr int kBarPFull = kBarSFull + kSBufs;            // [2]: one per P^T buffer
constexpr int kBarOFull = kBarPFull + 2;            // [2]: one per P^T buffer
constexpr int kBarDrain = kBarOFull + 2;
constexpr int kBarKRaw = kBarDrain + 1;              // [kKStages]: K tiles of a fused append
constexpr int kBarVRaw = kBarKRaw + kKStages;         // [kMaxVStages]: V tiles of a fused append
constexpr int kNumBars = kBarVRaw + kMaxVStages;

// Buffers of the rows' operands for a given NQ: up to 64 rows, four S^T buffers in TMEM and
// a double-buffered P^T in shared memory (the softmax of tile t + 1 writes P^T while the PV
// product of tile t reads the other buffer); at 80 rows TMEM holds three S^T buffers
// ((3 + 3) x 80 of its 512 columns) and P^T is single-buffered, so that the K and V rings still
// fit in shared memory (the softmax of tile t + 1 computes its probabilities first and waits
// for the PV product of tile t only before storing them).
__host__ __device__ constexpr int tc_sbufs(int nq) { return nq <= 64 ? kSBufs : 3; }
__host__ __device__ constexpr int tc_pbufs(int nq) { return nq <= 64 ? 2 : 1; }

// Shared-memory plan for a given NQ and V ring depth.
struct TcLayout {
  int k, v, q, p, bar, misc, vote, wmax, lim, mref, alpha, pre, end;
};
__host__ __device__ inline TcLayout tc_layout(int nq, int vstages, int qbufs, int B) {
  // Operand buffers are 1024-byte multiples from a 1024-aligned base; every small region is
  // rounded to 16 bytes (the per-row references are read as float4).
  auto a16 = [](int x) { return (x + 15) & ~15; };
  TcLayout L;
  L.k = 0;
  L.v = L.k + kKStages * kTileBytes;
  L.q = L.v + vstages * kTileBytes;
  L.p = L.q + qbufs * 2 * nq * 128;         // Q: qbufs buffers x two 64-channel halves
  L.bar = L.p + tc_pbufs(nq) * nq * 512;    // P^T: buffers of 2*nq/8 row groups of 2048 B
  L.misc = a16(L.bar + kNumBars * 8);       // tmem slot, abort flag
  L.vote = L.misc + 16;                     // (unused slot kept for alignment)
  L.wmax = L.vote + 32;                     // [2][4][nq] floats
  L.lim = a16(L.wmax + 2 * 4 * nq * 4);     // [3][nq] ints: (unused), output offsets, key limits
  L.mref = a16(L.lim + 3 * nq * 4);         // [2][nq]: per-row references
  L.alpha = a16(L.mref + 2 * nq * 4);       // [nq]: rescale factors of the last reference update
  L.pre = a16(L.alpha + nq * 4);            // plan: [B+1], 32 ints, first segment (16 x 8 B)
  L.end = L.pre + (round_up(B + 1, 4) + 32) * 4 + 16 * 8;
  return L;
}

__device__ __forceinline__ void softmax_bar() {
  asm volatile("bar.sync %0, 128;" ::"n"(kNamedBarSoftmax) : "memory");
}

// OR of a predicate over the 128 softmax threads (named barrier 1), returned to all of them.
__device__ __forceinline__ bool softmax_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kNamedBarSoftmax)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ int tiles_of(const Segment& sg) { return (sg.j1 - sg.j0 + kNT - 1) / kNT; }

// P^T rows 16c..16c+15 of one key (thread): bf16 hi and lo halves, one 16-byte store per
// group of 8 rows. `prow` addresses this key's 16-byte slot in row group 0 of the hi half;
// row groups are 2048 bytes apart and the lo half follows the NQ/8 hi groups.
template <int NQ>
__device__ __forceinline__ void store_pt16_impl(uint32_t prow, int c, const float (&x)[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = x[8 * h + 2 * e], b = x[8 * h + 2 * e + 1];
      hi[e] = pack_bf16x2(a, b);
      const float ha = __uint_as_float(hi[e] << 16), hb = __uint_as_float(hi[e] & 0xFFFF0000u);
      lo[e] = pack_bf16x2(a - ha, b - hb);
    }
    const int m = 2 * c + h;
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + m * 2048), "r"(hi[0]),
                 "r"(hi[1]), "r"(hi[2]), "r"(hi[3]));
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + (NQ / 8 + m) * 2048),
                 "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3]));
  }
}

// Row of key j of (b, h) in the K/V tensor maps: contiguous caches, or the page pool (the key
// must lie in one of the sequence's pages, j < pages_per_seq * page_size).
template <bool PAGED>
__device__ __forceinline__ int kv_row(const Problem& p, int b, int h, int j) {
  if (!PAGED) return (b * p.Hkv + h) * p.S + j;
  const int page = __ldg(p.block_table + (size_t)b * p.pages_per_seq + j / p.page_size);
  return (page * p.Hkv + h) * p.page_size + (j % p.page_size);
}

// Issues the two (contiguous) or four (paged: one 64-row box per page piece) TMA loads of key
// tile [jt, jt + 128) of segment sg into `dst`, all on barrier `fb`. Paged halves that lie
// wholly past the segment's keys read the segment's last page instead (their rows are never
// used), so no block-table entry beyond the sequence is touched. Every key tile is read once
// per call: contiguous loads carry an L2 evict-first policy.
template <bool PAGED>
__device__ __forceinline__ void load_kv_tile(const Problem& p, const Segment& sg,
                                             const CUtensorMap* map, uint32_t dst, uint32_t fb,
                                             int jt, uint64_t policy) {
  if (!PAGED) {
    const int row = (sg.b * p.Hkv + sg.h) * p.S + jt;
    tma_load_2d_hint(dst, map, fb, 0, row, policy);
    tma_load_2d_hint(dst + kHalfBytes, map, fb, 64, row, policy);
    return;
  }
  const int jl = sg.j1 - 1;   // last key of the segment
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int j = min(jt + 64 * hr, jl);
    const int row = kv_row<true>(p, sg.b, sg.h, j);
    const uint32_t off = (uint32_t)hr * 64u * 128u;
    tma_load_2d(dst + off, map, fb, 0, row);
    tma_load_2d(dst + kHalfBytes + off, map, fb, 64, row);
  }
}

// ---- Fused window append (step a1 inside the attention launch).
// The window's keys [P, P + W) of a sequence (n = P + W visible keys) come from k_new / v_new.
// The producer warp of K (or V) loads the rows that fall in key tile [jt, jt + kNT) into
// registers, writes them to their cache rows (the append), and, once the tile's TMA copy of
// the cache (whose window rows are stale) has landed, writes them over those rows in shared
// memory before it releases the tile to the MMA. Each window row lies in exactly one tile of
// one CTA, so every row is appended once.
constexpr int kWinRegs = kMaxWindow * 16 / 32;   // 16-byte chunks per lane: W rows x 16 chunks

__device__ __forceinline__ bool tile_window(const Problem& p, const Segment& sg, int jt, int& w0,
                                            int& w1) {
  const int P = sg.n - sg.w;
  const int lo = max(jt, P), hi = min(jt + kNT, sg.j1);
  w0 = lo - P;
  w1 = hi - P;
  return lo < hi;
}

// Lane l holds chunks l, l + 32, ... of the rows [w0, w1) (16 chunks of 16 bytes per row).
template <bool PAGED>
__device__ __forceinline__ void window_load_append(const Problem& p, const Segment& sg,
                                                   const __nv_bfloat16* src,
                                                   __nv_bfloat16* cache, int w0, int w1,
                                                   int lane, uint4 (&v)[kWinRegs]) {
  const int P = sg.n - sg.w;
  const int cnt = (w1 - w0) * 16;
#pragma unroll
  for (int u = 0; u < kWinRegs; ++u) {
    const int idx = lane + 32 * u;
    if (idx < cnt) {
      const int w = w0 + (idx >> 4), ch = idx & 15;
      const uint4* s = reinterpret_cast<const uint4*>(
          src + (((size_t)sg.b * p.W + w) * p.Hkv + sg.h) * kHeadDim) + ch;
      v[u] = __ldg(s);
      uint4* d = reinterpret_cast<uint4*>(
          cache + (size_t)kv_row<PAGED>(p, sg.b, sg.h, P + w) * kHeadDim) + ch;
      *d = v[u];
    }
  }
}

// Writes the held rows into the tile at `tile` (two 64-channel halves, 128-byte swizzle:
// 16-byte chunk c of row r of a half sits at r * 128 + ((c ^ (r & 7)) * 16)).
__device__ __forceinline__ void window_patch(uint32_t tile, const Problem& p, const Segment& sg,
                                             int jt, int w0, int w1, int lane,
                                             const uint4 (&v)[kWinRegs]) {
  const int P = sg.n - sg.w;
  const int cnt = (w1 - w0) * 16;
#pragma unroll
  for (int u = 0; u < kWinRegs; ++u) {
    const int idx = lane + 32 * u;
    if (idx < cnt) {
      const int r = P + w0 + (idx >> 4) - jt, ch = idx & 15;
      const uint32_t a = tile + (uint32_t)((ch >> 3) * kHalfBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v[u].x), "r"(v[u].y),
                   "r"(v[u].z), "r"(v[u].w));
    }
  }
}

}  // namespace

template <int NQ, bool CAUSAL, bool PAGED>
__global__ void __launch_bounds__(kThreadsTc, 1)
    pbd_attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmo,
                       Problem p, int ring) {
  static_assert(NQ % 16 == 0 && NQ >= 16 && NQ <= 80, "NQ");
  constexpr int kQHalf = NQ * 128;                 // bytes of one 64-channel half of Q
  constexpr int kSB = tc_sbufs(NQ);                // S^T buffers
  constexpr int kPB = tc_pbufs(NQ);                // P^T buffers
  constexpr int kColS = 0;                         // S^T buffers at [0, kSB NQ)
  constexpr int kColO = kSB * NQ;                  // O^T (hi | lo)
  constexpr int kColL = (kSB + 2) * NQ;            // row-sum partials of each key lane
  static_assert((kSB + 3) * NQ <= kTmemCols, "TMEM columns");
  static_assert(kSB <= kSBufs, "S barriers");
  constexpr uint32_t kIdescQK = idesc_f16(128, NQ, 0, 0);
  constexpr uint32_t kIdescPV = idesc_f16(128, 2 * NQ, 1, 1);

  extern __shared__ __align__(1024) char smem_raw[];
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int vstages = ring & 0xff, qbufs = ring >> 8;   // V ring depth, Q buffers
  const TcLayout L = tc_layout(NQ, vstages, qbufs, p.B);
  const uint32_t sb = smem_u32(base);
  const uint32_t sK = sb + L.k, sV = sb + L.v, sQ = sb + L.q, sP = sb + L.p;
  auto bar = [&](int i) { return sb + (uint32_t)L.bar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.misc + 8);
  float* wmax = reinterpret_cast<float*>(base + L.wmax);
  int* lim_s = reinterpret_cast<int*>(base + L.lim);
  int* pre = reinterpret_cast<int*>(base + L.pre);           // the plan's prefix sums
  int* warp_tot = pre + round_up(p.B + 1, 4);
  // First segment of this CTA and the plan iterator after it: b, h, n, w, j0, j1, whole, slot,
  // have, pos, end, iterator b, iterator h.
  long long* spec = reinterpret_cast<long long*>(warp_tot + 32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Ctl ctl{abort_flag, p.hdr, p.wait_limit_ns};
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmq)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmo)) : "memory");
  }

  // Q rows R..NQ-1 must read as zero: clear them in both Q buffers once (TMA writes only rows
  // < R, so no generic store ever meets a copy in flight).
  {
    const int per_half = (NQ - p.R) * 8;   // 16-byte chunks of rows [R, NQ) in one half
    for (int i = tid; i < 4 * per_half; i += kThreadsTc) {
      const int half = i / per_half, c = i - half * per_half;
      reinterpret_cast<uint4*>(base + L.q + half * kQHalf + p.R * 128)[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
  }
  auto init_barriers = [&]() {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < kMaxVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarQFull + s), 1);
      mbar_init(bar(kBarQEmpty + s), 1);
    }
    for (int s = 0; s < kSBufs; ++s) mbar_init(bar(kBarSFull + s), 1);
    mbar_init(bar(kBarPFull + 0), 128);
    mbar_init(bar(kBarPFull + 1), 128);
    mbar_init(bar(kBarOFull + 0), 1);
    mbar_init(bar(kBarOFull + 1), 1);
    mbar_init(bar(kBarDrain), 1);
    for (int s = 0; s < kKStages; ++s) mbar_init(bar(kBarKRaw + s), 1);
    for (int s = 0; s < kMaxVStages; ++s) mbar_init(bar(kBarVRaw + s), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  };
  if (tid == 0) {
    init_barriers();
    *abort_flag = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // The plan before the wait (speculative). Made from seq_lens / window_lens as they are now,
  // read through L2 only, while the previous kernel of the stream finishes: the prefix sums,
  // this CTA's first segment (thread 0, shared through shared memory so that every role
  // sees the same values) and, for contiguous caches, an L2 prefetch of its Q and first key
  // tiles. Right after the wait the producers issue the copies of that first segment, and
  // the plan is checked against the values read after the wait. If anything the plan or the
  // first segment depends on differs (a sequence's number of plan units, or the prefix and
  // window length of the first segment's sequence), the producers drain those copies, the
  // barriers are initialised again and the kernel continues from the plan made anew;
  // otherwise the copies are already in flight.
  plan_prefix<true>(p, pre, warp_tot);
  long long T = (long long)p.Hkv * pre[p.B];
  if (tid == 0) {
    SegmentIter it0 = plan_begin(p, pre, blockIdx.x, T);
    Segment s0{};
    const bool have0 = it0.next<true>(p, pre, blockIdx.x, s0);
    spec[0] = s0.b; spec[1] = s0.h; spec[2] = s0.n; spec[3] = s0.w; spec[4] = s0.j0;
    spec[5] = s0.j1; spec[6] = s0.whole; spec[7] = s0.slot; spec[8] = have0;
    spec[9] = it0.pos; spec[10] = it0.end; spec[11] = it0.b; spec[12] = it0.h;
    if (!PAGED && have0) {
      // L2 hint only (no shared memory written, no barrier): Q and the first two key tiles.
      tma_prefetch_3d(&tmq, 0, s0.h * p.G, s0.b * p.W);
      tma_prefetch_3d(&tmq, 64, s0.h * p.G, s0.b * p.W);
      const int nt = min(tiles_of(s0), 2);
      for (int t = 0; t < nt; ++t) {
        const int row = (s0.b * p.Hkv + s0.h) * p.S + s0.j0 + t * kNT;
        tma_prefetch_2d(&tmk, 0, row);
        tma_prefetch_2d(&tmk, 64, row);
        tma_prefetch_2d(&tmv, 0, row);
        tma_prefetch_2d(&tmv, 64, row);
      }
    }
  }
  __syncthreads();
  Segment sg0;
  sg0.b = (int)spec[0]; sg0.h = (int)spec[1]; sg0.n = (int)spec[2]; sg0.w = (int)spec[3];
  sg0.j0 = (int)spec[4]; sg0.j1 = (int)spec[5]; sg0.whole = spec[6] != 0; sg0.slot = (int)spec[7];
  bool have0 = spec[8] != 0;
  // Everything above is on-chip (or an L2 hint); from here on global memory written by the
  // previous kernel of the stream is read. The merge kernel after this one may start only
  // once every CTA is past the wait (it reads seq_lens before its own wait).
  pdl_wait();
  pdl_trigger();
  const uint64_t kv_policy = l2_policy_evict_first();
  // Speculative copies of the first segment's Q and first key tile (on the barriers the
  // producers would use for them).
  bool spec_issued = false;
  if ((warp == 0 || warp == 6) && lane == 0 && have0) {
    int w0 = 0, w1 = 0;
    if (warp == 0) {
      mbar_expect_tx(bar(kBarQFull), 2u * p.R * 128u);
      tma_load_3d(sQ, &tmq, bar(kBarQFull), 0, sg0.h * p.G, sg0.b * p.W);
      tma_load_3d(sQ + kQHalf, &tmq, bar(kBarQFull), 64, sg0.h * p.G, sg0.b * p.W);
      const bool fuse = p.k_new != nullptr && tile_window(p, sg0, sg0.j0, w0, w1);
      const uint32_t fb = bar(fuse ? kBarKRaw : kBarKFull);
      mbar_expect_tx(fb, (uint32_t)kTileBytes);
      load_kv_tile<PAGED>(p, sg0, &tmk, sK, fb, sg0.j0, kv_policy);
    } else {
      const bool fuse = p.v_new != nullptr && tile_window(p, sg0, sg0.j0, w0, w1);
      const uint32_t fb = bar(fuse ? kBarVRaw : kBarVFull);
      mbar_expect_tx(fb, (uint32_t)kTileBytes);
      load_kv_tile<PAGED>(p, sg0, &tmv, sV, fb, sg0.j0, kv_policy);
    }
    spec_issued = true;
  }
  // Check the plan against the values as they are after the wait: the plan is the same if
  // every sequence has the same number of plan units (hence the same prefix sums), and the
  // first segment is the same if its sequence also has the same prefix and window length.
  // (Later segments read their lengths after the wait in any case.) One read per sequence
  // and the barrier that also orders the tensor-memory allocation before its use.
  bool differs = (p.stall_test & 2) != 0;   // (self-test of the path below)
  for (int b = tid; b < p.B; b += kThreadsTc) {
    const int w = window_of(p, b);
    const int n = visible_of(p, load_len(p.seq_lens + b), w);
    differs |= plan_units_of(p, n) != pre[b + 1] - pre[b];
    if (have0 && b == sg0.b) differs |= n != sg0.n || w != sg0.w;
  }
  fence_async_smem();
  tc_fence_before();
  if (__syncthreads_or(differs)) {
    // Rare: the plan changed. Drain the speculative copies, start the barriers afresh and
    // make the plan from the values read after the wait.
    if (spec_issued) {
      int w0 = 0, w1 = 0;
      if (warp == 0) {
        mbar_drain(bar(kBarQFull), 0, 100000000LL);
        const bool fuse = p.k_new != nullptr && tile_window(p, sg0, sg0.j0, w0, w1);
        mbar_drain(bar(fuse ? kBarKRaw : kBarKFull), 0, 100000000LL);
      } else {
        const bool fuse = p.v_new != nullptr && tile_window(p, sg0, sg0.j0, w0, w1);
        mbar_drain(bar(fuse ? kBarVRaw : kBarVFull), 0, 100000000LL);
      }
      spec_issued = false;
    }
    plan_prefix<false>(p, pre, warp_tot);   // (starts and ends with a barrier)
    if (tid == 0) {
      for (int i = 0; i < kNumBars; ++i) mbar_inval(bar(i));
      init_barriers();
      T = (long long)p.Hkv * pre[p.B];
      SegmentIter it0 = plan_begin(p, pre, blockIdx.x, T);
      Segment s0{};
      const bool h0 = it0.next(p, pre, blockIdx.x, s0);
      spec[0] = s0.b; spec[1] = s0.h; spec[2] = s0.n; spec[3] = s0.w; spec[4] = s0.j0;
      spec[5] = s0.j1; spec[6] = s0.whole; spec[7] = s0.slot; spec[8] = h0;
      spec[9] = it0.pos; spec[10] = it0.end; spec[11] = it0.b; spec[12] = it0.h;
    }
    __syncthreads();
    T = (long long)p.Hkv * pre[p.B];
    sg0.b = (int)spec[0]; sg0.h = (int)spec[1]; sg0.n = (int)spec[2]; sg0.w = (int)spec[3];
    sg0.j0 = (int)spec[4]; sg0.j1 = (int)spec[5]; sg0.whole = spec[6] != 0; sg0.slot = (int)spec[7];
    have0 = spec[8] != 0;
  }
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (blockIdx.x == 0) {
    for (int i = tid; i <= p.B; i += kThreadsTc) p.pre_g[i] = pre[i];
  }
  // Every role starts from the first segment above and continues the plan after it.
  SegmentIter it0;
  it0.pos = spec[9]; it0.end = spec[10]; it0.b = (int)spec[11]; it0.h = (int)spec[12];

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer: Q, K
    // Lane 0 issues the copies; the whole warp moves the window rows of a fused append.
    SegmentIter it = it0;
    Segment sg = sg0;
    int g = 0, nseg = 0;
    uint32_t raw_par = 0;   // phase parity of each stage's fused-append barrier
    bool ok = true;
    for (bool have = have0; ok && have; have = it.next(p, pre, blockIdx.x, sg)) {
      if (lane == 0 && !(spec_issued && nseg == 0)) {
        const int qs = nseg % qbufs, qu = nseg / qbufs;
        if (qu > 0 && !mbar_wait(bar(kBarQEmpty + qs), (qu - 1) & 1, ctl)) {
          ok = false;
        } else {
          const uint32_t dq = sQ + qs * 2 * kQHalf;
          mbar_expect_tx(bar(kBarQFull + qs), 2u * p.R * 128u);
          tma_load_3d(dq, &tmq, bar(kBarQFull + qs), 0, sg.h * p.G, sg.b * p.W);
          tma_load_3d(dq + kQHalf, &tmq, bar(kBarQFull + qs), 64, sg.h * p.G, sg.b * p.W);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int nt = tiles_of(sg);
      for (int t = 0; t < nt; ++t, ++g) {
        const int jt = sg.j0 + t * kNT;
        const int ks = g % kKStages, ku = g / kKStages;
        int w0 = 0, w1 = 0;
        const bool fuse = p.k_new != nullptr && tile_window(p, sg, jt, w0, w1);
        if (lane == 0 && !(spec_issued && g == 0)) {
          if (ku > 0 && !mbar_wait(bar(kBarKEmpty + ks), (ku - 1) & 1, ctl)) {
            ok = false;
          } else {
            const uint32_t dk = sK + ks * kTileBytes;
            const uint32_t fb = bar((fuse ? kBarKRaw : kBarKFull) + ks);
            mbar_expect_tx(fb, (uint32_t)kTileBytes);
            load_kv_tile<PAGED>(p, sg, &tmk, dk, fb, jt, kv_policy);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (fuse) {
          // While the tile is in flight: fetch the window rows and append them to the cache.
          uint4 win[kWinRegs];
          window_load_append<PAGED>(p, sg, p.k_new, p.kc, w0, w1, lane, win);
          const uint32_t fb = bar(kBarKRaw + ks);
          if (lane == 0 && !mbar_wait(fb, (raw_par >> ks) & 1u, ctl)) {
            mbar_drain(fb, (raw_par >> ks) & 1u, 100000000LL);
            ok = false;
          }
          raw_par ^= 1u << ks;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          window_patch(sK + ks * kTileBytes, p, sg, jt, w0, w1, lane, win);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarKFull + ks));
        }
      }
      ++nseg;
    }
    // Drain: the copies issued last must have landed before shared memory is released.
    if (lane == 0) {
      for (int back = 1; back <= kKStages && g - back >= 0; ++back) {
        const int gg = g - back;
        mbar_drain(bar(kBarKFull + gg % kKStages), (gg / kKStages) & 1, 100000000LL);
      }
      if (nseg > 0) mbar_drain(bar(kBarQFull + (nseg - 1) % qbufs), ((nseg - 1) / qbufs) & 1, 100000000LL);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------------ TMA producer: V
    SegmentIter it = it0;
    Segment sg = sg0;
    int g = 0;
    uint32_t raw_par = 0;
    bool ok = true;
    for (bool have = have0; ok && have; have = it.next(p, pre, blockIdx.x, sg)) {
      const int nt = tiles_of(sg);
      for (int t = 0; t < nt; ++t, ++g) {
        const int jt = sg.j0 + t * kNT;
        const int vs = g % vstages, vu = g / vstages;
        int w0 = 0, w1 = 0;
        const bool fuse = p.v_new != nullptr && tile_window(p, sg, jt, w0, w1);
        if (lane == 0 && !(spec_issued && g == 0)) {
          if (vu > 0 && !mbar_wait(bar(kBarVEmpty + vs), (vu - 1) & 1, ctl)) {
            ok = false;
          } else {
            const uint32_t dv = sV + vs * kTileBytes;
            const uint32_t fb = bar((fuse ? kBarVRaw : kBarVFull) + vs);
            mbar_expect_tx(fb, (uint32_t)kTileBytes);
            load_kv_tile<PAGED>(p, sg, &tmv, dv, fb, jt, kv_policy);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (fuse) {
          // While the tile is in flight: fetch the window rows and append them to the cache.
          uint4 win[kWinRegs];
          window_load_append<PAGED>(p, sg, p.v_new, p.vc, w0, w1, lane, win);
          const uint32_t fb = bar(kBarVRaw + vs);
          if (lane == 0 && !mbar_wait(fb, (raw_par >> vs) & 1u, ctl)) {
            mbar_drain(fb, (raw_par >> vs) & 1u, 100000000LL);
            ok = false;
          }
          raw_par ^= 1u << vs;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          window_patch(sV + vs * kTileBytes, p, sg, jt, w0, w1, lane, win);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarVFull + vs));
        }
      }
    }
    if (lane == 0) {
      for (int back = 1; back <= vstages && g - back >= 0; ++back) {
        const int gg = g - back;
        mbar_drain(bar(kBarVFull + gg % vstages), (gg / vstages) & 1, 100000000LL);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      SegmentIter it = it0;
      Segment sg = sg0;
      int g = 0, nseg = 0;
      bool ok = true;
      uint32_t sQseg = sQ;   // Q buffer of the current segment
      auto issue_qk = [&](int gg) {
        const uint32_t kb = sK + (gg % kKStages) * kTileBytes;
        const uint32_t d = tmem + kColS + (uint32_t)((gg % kSB) * NQ);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t ka = kb + (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint32_t qa = sQseg + (kk >> 2) * kQHalf + (kk & 3) * 32;
          umma(d, sdesc(ka, 16, 1024, 2), sdesc(qa, 16, 1024, 2), kIdescQK, kk > 0);
        }
      };
      auto issue_pv = [&](int gg, bool first) {
        const uint32_t vb = sV + (gg % vstages) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kNT / 16; ++kk) {
          const uint64_t pdesc = sdesc(sP + (gg % kPB) * (NQ * 512) + kk * 256, 128, 2048, 0);
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          umma(tmem + kColO, sdesc(vb + kk * 2048, kHalfBytes, 1024, 2), pdesc, kIdescPV, acc);
        }
      };
      for (bool have = have0; ok && have; have = it.next(p, pre, blockIdx.x, sg)) {
        const int nt = tiles_of(sg);
        const int qs = nseg % qbufs;
        if (!mbar_wait(bar(kBarQFull + qs), (nseg / qbufs) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        sQseg = sQ + qs * 2 * kQHalf;
        // Issue S^T(t) as soon as K(t) has landed and its S buffer is free (P(t-kSB+1) consumed),
        // and O^T += V^T P^T(t) as soon as P(t) and V(t) are ready, whichever comes first.
        const int g0 = g;
        int nqk = 0, npv = 0;
        long long t_prog = now_ns();
        uint32_t spins = 0;
        while (npv < nt) {
          bool prog = false;
          const bool want_qk = nqk < nt && nqk <= npv + kSB - 1;
          const bool want_pv = npv < nqk;
          if (want_qk != want_pv) {
            // One event pending: a (bounded) blocking wait is cheaper than polling.
            const bool got = want_qk
                ? mbar_wait(bar(kBarKFull + (g0 + nqk) % kKStages), ((g0 + nqk) / kKStages) & 1, ctl)
                : (mbar_wait(bar(kBarPFull + (g0 + npv) % kPB), ((g0 + npv) / kPB) & 1, ctl) &&
                   mbar_wait(bar(kBarVFull + (g0 + npv) % vstages), ((g0 + npv) / vstages) & 1, ctl));
            if (!got) { ok = false; break; }
          }
          if (want_qk) {
            const int gq = g0 + nqk;
            if (mbar_test(bar(kBarKFull + gq % kKStages), (gq / kKStages) & 1)) {
              tc_fence_after();
              issue_qk(gq);
              // (Self-test of the failure detection: the first completion is withheld, so the
              // softmax warps' bounded wait for it runs out.)
              if (!((p.stall_test & 1) && gq == 0)) umma_commit(bar(kBarSFull + gq % kSB));
              umma_commit(bar(kBarKEmpty + gq % kKStages));
              if (nqk == nt - 1) umma_commit(bar(kBarQEmpty + qs));
              ++nqk;
              prog = true;
            }
          }
          if (want_pv) {
            const int gp = g0 + npv;
            if (mbar_test(bar(kBarPFull + gp % kPB), (gp / kPB) & 1) &&
                mbar_test(bar(kBarVFull + gp % vstages), (gp / vstages) & 1)) {
              tc_fence_after();
              issue_pv(gp, npv == 0);
              umma_commit(bar(kBarOFull + gp % kPB));
              umma_commit(bar(kBarVEmpty + gp % vstages));
              ++npv;
              prog = true;
            }
          }
          if (prog) {
            spins = 0;
            t_prog = now_ns();
            continue;
          }
          // Idle poll: back off so this thread does not take issue slots from the softmax
          // warp that shares its scheduler.
          __nanosleep(32);
          if ((++spins & 63u) == 0) {
            if (*abort_flag) { ok = false; break; }
            if (now_ns() - t_prog > p.wait_limit_ns) {
              *abort_flag = 1;
              atomicOr(&p.hdr->err, kErrTimeout);
              ok = false;
              break;
            }
          }
        }
        g = g0 + nt;
        ++nseg;
      }
      // Drain all issued MMAs before TMEM can be released.
      umma_commit(bar(kBarDrain));
      mbar_drain(bar(kBarDrain), 0, 100000000LL);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    // Per tile each thread holds its key's NQ scores. The per-row references m (log2 units,
    // shared by all threads) live in shared memory, double-buffered; row sums accumulate in
    // TMEM next to O.
    const int sub = warp & 3;                   // TMEM sub-partition of this warp
    const int w4 = warp - 2;                    // 0..3 within the softmax group
    const int row = 32 * sub + lane;            // key of the S^T tile / channel of O^T
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * sub) << 16);
    const int stid = tid - 64;                  // 0..127
    float* rowst = reinterpret_cast<float*>(base + L.mref);   // [2][NQ]
    float* alpha_s = reinterpret_cast<float*>(base + L.alpha); // [NQ]
    const float c2 = p.scale_log2;
    SegmentIter it = it0;
    Segment sg = sg0;
    int g = 0;
    bool ok = true;
    for (bool have = have0; ok && have; have = it.next(p, pre, blockIdx.x, sg)) {
      const int nt = tiles_of(sg);
      for (int q = stid; q < NQ; q += 128) {
        if (CAUSAL) lim_s[2 * NQ + q] = (q < p.R) ? min(row_limit(p, sg.n, sg.w, q), sg.j1) : 0;
        rowst[q] = -INFINITY;            // no reference yet
      }
      softmax_bar();
      const int* lim_q = lim_s + 2 * NQ;
      int cur = 0;

      for (int t = 0; t < nt; ++t) {
        const int gt = g + t;
        const int jt = sg.j0 + t * kNT;
        const int key = jt + row;
        const bool key_ok = key < sg.j1;
        const uint32_t s_addr = lane_addr + kColS + (gt % kSB) * NQ;
        if (!mbar_wait(bar(kBarSFull + gt % kSB), (gt / kSB) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        // P^T is written as hi/lo row groups, one 16-byte store per 8 rows.
        const uint32_t prow = sP + (gt % kPB) * (NQ * 512) + (uint32_t)((row >> 3) * 128 + (row & 7) * 16);
        // A segment's first tile has no references yet: it always takes the exact-maximum
        // path below.
        bool rescale = true;
        bool hot = false;     // p of this tile kept in xs, row sums still to be added
        float xs[NQ];
        if (t > 0) {
          // The common path (hot, fully unrolled): all NQ scores of this key at once,
          // p = 2^(score * scale_log2 - reference); the vote asks whether some exponent exceeds
          // the lazy threshold. Padding rows (q >= R) need no mask: their Q rows are zero, so
          // their scores are exactly 0.
          float x[NQ];
#pragma unroll
          for (int c = 0; c < NQ / 16; ++c) tmem_ld16(s_addr + 16 * c, x + 16 * c);
          tc_wait_ld();
          const float4* mr4 = reinterpret_cast<const float4*>(rowst + cur * NQ);
          bool exceeds = false;
#pragma unroll
          for (int c4 = 0; c4 < NQ / 4; ++c4) {
            const float4 m4 = mr4[c4];
            const float mq[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = 4 * c4 + e;
              const float y = fmaf(x[q], c2, -mq[e]);
              const bool v = CAUSAL ? (key < lim_q[q]) : key_ok;
              exceeds |= v && (y > kLazyThreshold);
              x[q] = v ? fast_exp2(y) : 0.f;
            }
          }
          // CTA-wide vote: raise the references only if some score is far above them.
          rescale = softmax_bar_or(exceeds);
          if (!rescale) {
            hot = true;
            // The product that last read this P^T buffer (tile gt - kPB) must be done.
            if (gt >= kPB) {
              const int gr = gt - kPB;
              if (!mbar_wait(bar(kBarOFull + gr % kPB), (gr / kPB) & 1, ctl)) { ok = false; break; }
              tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < NQ / 16; ++c)
              store_pt16_impl<NQ>(prow, c, *reinterpret_cast<const float(*)[16]>(x + 16 * c));
#pragma unroll
            for (int q = 0; q < NQ; ++q) xs[q] = x[q];
          }
        }
        if (rescale) {
          // The rare path (always taken on a segment's first tile), 16 rows at a time straight
          // from TMEM in rolled loops: it runs cold, where instruction fetch rather than
          // arithmetic sets its speed, so small code wins.
          // Exact tile maxima per row (log2 units): warp reduction, then across the warps.
          float* wm = wmax + (gt & 1) * 4 * NQ;
#pragma unroll 1
          for (int c = 0; c < NQ / 16; ++c) {
            float x[16];
            tmem_ld16(s_addr + 16 * c, x);
            tc_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const bool v = CAUSAL ? (key < lim_q[16 * c + k]) : key_ok;
              const float m = warp_max_f32(v ? x[k] * c2 : -INFINITY);
              if (k == (lane & 15) && (lane >> 4) == 0) wm[w4 * NQ + 16 * c + k] = m;
            }
          }
          softmax_bar();
          // Thread q publishes the new reference of row q and the factor that rescales what
          // was accumulated against the old one.
          float* mw = rowst + (cur ^ 1) * NQ;
          if (stid < NQ) {
            const int q = stid;
            const float tm = fmaxf(fmaxf(wm[q], wm[NQ + q]), fmaxf(wm[2 * NQ + q], wm[3 * NQ + q]));
            const float mo = rowst[cur * NQ + q];
            const float mn = fmaxf(mo, tm);
            mw[q] = mn;
            alpha_s[q] = (mn == -INFINITY) ? 1.f : fast_exp2(mo - mn);
          }
          // The previous PV product (and so every earlier one) must be complete before O and l
          // are rescaled in place (and before a single P^T buffer is rewritten).
          if (gt > 0) {
            if (!mbar_wait(bar(kBarOFull + (gt - 1) % kPB), ((gt - 1) / kPB) & 1, ctl)) { ok = false; break; }
            tc_fence_after();
          }
          softmax_bar();
#pragma unroll 1
          for (int c = 0; c < NQ / 16; ++c) {
            float x[16];
            tmem_ld16(s_addr + 16 * c, x);
            tc_wait_ld();
            const float4* mn4 = reinterpret_cast<const float4*>(mw + 16 * c);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const float4 m4 = mn4[c4];
              const float mq[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int k = 4 * c4 + e;
                const bool v = CAUSAL ? (key < lim_q[16 * c + k]) : key_ok;
                const float safe = (mq[e] == -INFINITY) ? 0.f : mq[e];
                x[k] = v ? fast_exp2(fmaf(x[k], c2, -safe)) : 0.f;
              }
            }
            store_pt16_impl<NQ>(prow, c, x);
            if (t == 0) {
              tmem_st16(lane_addr + kColL + 16 * c, x);   // row-sum partials start here
            } else {
              // O hi, O lo and the row-sum partials of these 16 rows move to the new
              // references; this tile's p joins the partials.
              const float4* al4 = reinterpret_cast<const float4*>(alpha_s + 16 * c);
              float al[16];
#pragma unroll
              for (int e4 = 0; e4 < 4; ++e4) {
                const float4 a4 = al4[e4];
                al[4 * e4] = a4.x; al[4 * e4 + 1] = a4.y; al[4 * e4 + 2] = a4.z; al[4 * e4 + 3] = a4.w;
              }
#pragma unroll 1
              for (int blk = 0; blk < 3; ++blk) {
                float o[16];
                const uint32_t col = kColO + blk * NQ + 16 * c;
                tmem_ld16(lane_addr + col, o);
                tc_wait_ld();
                if (blk < 2) {
#pragma unroll
                  for (int e = 0; e < 16; ++e) o[e] *= al[e];
                } else {
#pragma unroll
                  for (int e = 0; e < 16; ++e) o[e] = fmaf(o[e], al[e], x[e]);
                }
                tmem_st16(lane_addr + col, o);
              }
            }
          }
          tc_wait_st();
          // Nobody reads the old references after the barrier above, and the next writer of
          // this buffer waits at the next tile's vote barrier.
          cur ^= 1;
        }
        // Rows of the V tile past the segment end hold other data: zero them so 0 * x
        // cannot turn into NaN in the tensor-core product.
        const int valid = min(kNT, sg.j1 - jt);
        if (valid < kNT) {
          // The tile's V copy must have landed before its tail is overwritten.
          if (!mbar_wait(bar(kBarVFull + gt % vstages), (gt / vstages) & 1, ctl)) { ok = false; break; }
          const uint32_t vbase = sV + (gt % vstages) * kTileBytes;
          for (int idx = stid; idx < (kNT - valid) * 16; idx += 128) {
            const int r = valid + (idx >> 4), ch = idx & 15;
            const uint32_t a = vbase + (ch >> 3) * kHalfBytes + r * 128 + (ch & 7) * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(0u), "r"(0u),
                         "r"(0u), "r"(0u));
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + gt % kPB));
        if (hot) {
          // Off the MMA's critical path: this tile's p joins the row-sum partials of this
          // key lane (the previous tile's partial stores have completed: every tile ends
          // with a wait on them).
#pragma unroll
          for (int c = 0; c < NQ / 16; ++c) {
            float lp[16];
            tmem_ld16(lane_addr + kColL + 16 * c, lp);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) lp[e] += xs[16 * c + e];
            tmem_st16(lane_addr + kColL + 16 * c, lp);
          }
          tc_wait_st();
        }
      }
      if (!ok) break;
      const int glast = g + nt - 1;
      g += nt;
      if (!mbar_wait(bar(kBarOFull + glast % kPB), (glast / kPB) & 1, ctl)) { ok = false; break; }
      tc_fence_after();

      // Epilogue: O^T row `row` (one channel) of a whole sequence is normalised, staged in the
      // idle P^T buffer as [R][128] bf16 output rows and written by one TMA store; a partial
      // is written straight to its slot.
      float* slot = sg.whole ? nullptr : slot_ptr(p, sg.slot);
      const uint32_t stg = sP;
      const uint64_t keep = l2_policy_evict_last();
      if (!sg.whole) {
        // A partial's O is not normalised, so it is written first, straight from registers
        // to its slot, and its stores drain while the row sums are reduced: for each row the
        // warp writes 32 consecutive channels (128 bytes). The merge reads it back after this
        // kernel: kept in L2 (evict-last) while the rest of the K/V stream passes through.
        float* accp = slot + 2 * p.rows_pad;
#pragma unroll 1
        for (int c = 0; c < NQ / 16; ++c) {
          float ohi[16], olo[16];
          tmem_ld16(lane_addr + kColO + 16 * c, ohi);
          tmem_ld16(lane_addr + kColO + NQ + 16 * c, olo);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int q = 16 * c + e;
            if (q >= p.R) break;
            st_global_hint(accp + (size_t)q * kHeadDim + row, ohi[e] + olo[e], keep);
          }
        }
      }
      // Row sums: reduce the 128 key lanes' partials, 16 rows at a time. Within a warp a
      // butterfly halves the values each lane holds at every step (16 + 8 + 4 + 2 + 1
      // shuffles leave lane l with the warp's sum of row l & 15); the four warps' sums meet in
      // shared memory.
      float* wsum = wmax + NQ;         // [4][NQ] per-warp sums
#pragma unroll 1
      for (int c = 0; c < NQ / 16; ++c) {
        float v[16];
        tmem_ld16(lane_addr + kColL + 16 * c, v);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] += __shfl_xor_sync(0xffffffffu, v[e], 16);
#pragma unroll
        for (int h = 8; h >= 1; h >>= 1) {
          const bool upper = (lane & h) != 0;
#pragma unroll
          for (int e = 0; e < h; ++e) {
            const float give = upper ? v[e] : v[e + h];
            const float keep = upper ? v[e + h] : v[e];
            v[e] = keep + __shfl_xor_sync(0xffffffffu, give, h);
          }
        }
        if (lane < 16) wsum[w4 * NQ + 16 * c + lane] = v[0];
      }
      softmax_bar();
      float* linv = wmax + 5 * NQ;     // [NQ] reciprocals of the row sums
      if (!sg.whole) {
        if (stid < p.R) {
          const float l = (wsum[stid] + wsum[NQ + stid]) + (wsum[2 * NQ + stid] + wsum[3 * NQ + stid]);
          st_global_hint(slot + stid, rowst[cur * NQ + stid], keep);
          st_global_hint(slot + p.rows_pad + stid, l, keep);
        }
      } else {
        if (stid < NQ) {
          const float l = (wsum[stid] + wsum[NQ + stid]) + (wsum[2 * NQ + stid] + wsum[3 * NQ + stid]);
          linv[stid] = 1.f / l;
        }
        softmax_bar();
        const int rows_w = sg.w * p.G;
#pragma unroll 1
        for (int c = 0; c < NQ / 16; ++c) {
          float ohi[16], olo[16];
          tmem_ld16(lane_addr + kColO + 16 * c, ohi);
          tmem_ld16(lane_addr + kColO + NQ + 16 * c, olo);
          tc_wait_ld();
          const float4* l4 = reinterpret_cast<const float4*>(linv + 16 * c);
          float res[16];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 a4 = l4[e4];
            const float li[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) res[4 * e4 + e] = (ohi[4 * e4 + e] + olo[4 * e4 + e]) * li[e];
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int q = 16 * c + e;
            if (q >= p.R) break;
            // Padding rows of a shorter window (no visible key) are written as zeros.
            const __nv_bfloat16 v = __float2bfloat16_rn(q < rows_w ? res[e] : 0.f);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg + (uint32_t)(q * kHeadDim + row) * 2u),
                         "h"(*reinterpret_cast<const unsigned short*>(&v)));
          }
        }
        fence_async_smem();
        softmax_bar();
        if (stid == 0) {
          asm volatile(
              "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                  reinterpret_cast<uint64_t>(&tmo)),
              "r"(stg), "r"(0), "r"(sg.h * p.G), "r"(sg.b * p.W)
              : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          // The staging buffer is reused as P^T by the next segment: wait until it was read.
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
      }
      // O, l and the shared per-segment buffers are reused by the next segment.
      tc_fence_before();
      softmax_bar();
    }
  }

  // Epilogue stores issued by this thread must be complete before the CTA retires.
  if (tid == 64) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  tc_fence_before();
  __syncthreads();

  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

int tc_ctas_per_sm() { return 1; }
int tc_tile_keys() { return kNT; }
// Fixed cost of a segment in tile times: a CTA pays it for each segment (Q load, the first
// tile's exact-maximum pass, the epilogue, and the refill of the rings it leaves behind).
int tc_segment_units() { return kSegUnits; }

static int tc_nq(int R) { return round_up(R, 16); }

// V ring depth and Q buffers that fit: the V ring depth matters most (a V tile is held until
// its PV product completes), a second Q buffer only hides segment changes (measured: no gain
// on a ragged batch of 64 sequences when it costs a V stage).
static int tc_ring(int nq, int B) {
  const int limit = 227 * 1024 - 1024;
  const int options[5][2] = {{3, 2}, {3, 1}, {2, 2}, {2, 1}, {1, 1}};   // {V stages, Q buffers}
  for (auto& o : options)
    if (tc_layout(nq, o[0], o[1], B).end <= limit) return o[0] | (o[1] << 8);
  return 0;
}

size_t tc_smem_bytes(int R, int B) {
  const int nq = tc_nq(R);
  const int ring = tc_ring(nq, B);
  return ring ? (size_t)1024 + tc_layout(nq, ring & 0xff, ring >> 8, B).end : 0;
}

template <int NQ, bool CAUSAL, bool PAGED>
static cudaError_t launch_nq(const Problem& p, const CUtensorMap& k, const CUtensorMap& v,
                             const CUtensorMap& q, const CUtensorMap& o, cudaStream_t stream) {
  const int ring = tc_ring(NQ, p.B);
  if (ring == 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)1024 + tc_layout(NQ, ring & 0xff, ring >> 8, p.B).end;
  cudaError_t e = cudaFuncSetAttribute(pbd_attn_tc_kernel<NQ, CAUSAL, PAGED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(pbd_attn_tc_kernel<NQ, CAUSAL, PAGED>, dim3(p.num_ctas), dim3(kThreadsTc), smem,
                    stream, k, v, q, o, p, ring);
}

cudaError_t launch_attn_tc(const Problem& p, const void* tmap_k, const void* tmap_v,
                           const void* tmap_q, const void* tmap_o, cudaStream_t stream) {
  const CUtensorMap& k = *static_cast<const CUtensorMap*>(tmap_k);
  const CUtensorMap& v = *static_cast<const CUtensorMap*>(tmap_v);
  const CUtensorMap& q = *static_cast<const CUtensorMap*>(tmap_q);
  const CUtensorMap& o = *static_cast<const CUtensorMap*>(tmap_o);
  const bool causal = row_limits(p);   // per-row key limits
  // Paged caches get their own instantiations so that the contiguous kernels' code (and its
  // instruction-cache footprint on the latency-bound single-tile path) is unchanged.
  const bool paged = p.block_table != nullptr;
#define LA_TC_CASE(N)                                                                      \
  case N:                                                                                  \
    if (paged) return causal ? launch_nq<N, true, true>(p, k, v, q, o, stream)            \
                             : launch_nq<N, false, true>(p, k, v, q, o, stream);          \
    return causal ? launch_nq<N, true, false>(p, k, v, q, o, stream)                      \
                  : launch_nq<N, false, false>(p, k, v, q, o, stream);
  switch (tc_nq(p.R)) {
    LA_TC_CASE(16)
    LA_TC_CASE(32)
    LA_TC_CASE(48)
    LA_TC_CASE(64)
    LA_TC_CASE(80)
    default: return cudaErrorInvalidValue;
  }
#undef LA_TC_CASE
}

}  // namespace la
