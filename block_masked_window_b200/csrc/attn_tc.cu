// tcgen05 + TMA split-KV PBD window attention for sm_100a.
//
// Steps a2..a5 of one PBD decode step (LocateAnything-3B for RK3588 model card, "How it
// differs from the original", item 1: the window attends bidirectionally to itself and
// causally to the prefix, so every window row sees keys [0, P_b + W)). The R = W * G query
// rows that share one KV head (window row i, grouped head g -> row i*G + g; G = Hq / Hkv) form
// the M = 64 side of two tensor-core products per 64-key tile:
//   S  = Q  K^T   (M=64 rows, N=64 keys,     K=128 channels)  -> TMEM, fp32
//   O  = P  V     (M=64 rows, N=128 channels, K=64 keys)       -> TMEM, fp32
// P is the online-softmax probability tile. To keep fp32-level accuracy through a bf16
// tensor-core product, P is split as P = P_hi + P_lo with both halves bf16 (error ~2^-17 P)
// and O takes two MMAs per k-step; the tensor core has ample headroom at this arithmetic
// intensity (48 flop per byte of K/V at W = 6), so the path stays bound by HBM.
//
// Roles (192 threads, 2 CTAs per SM, 256 TMEM columns each):
//   warp 0      TMA producer: Q once per segment, K/V tiles into a 2-stage ring
//   warp 1      TMEM owner and single-thread MMA issuer
//   warps 2..5  softmax / accumulation: warp w reads TMEM sub-partition w % 4, i.e. rows
//               16*(w%4) .. +15 of the 64-row accumulators, through 16x256b loads whose
//               per-thread layout is (row t/4 and t/4+8, columns 2*(t%4) + {0,1} per 8)
// The softmax warps keep the running output in registers: every PV product lands in a fresh
// TMEM tile that they fold in as O <- alpha * O + PV, so no TMEM read-modify-write is needed.
//
// Shared-memory tiles use the 128-byte swizzle written by TMA, which is also the canonical
// SWIZZLE_128B operand layout of the tensor core: K-major for Q, K and P, MN-major for V.
//
// Every mbarrier wait is bounded: after ~2 s of waiting the CTA raises the sticky timeout
// flag in the workspace header, the other roles stop at their next wait, in-flight copies
// and MMAs are drained with bounded waits, TMEM is freed and the kernel returns.
#include "pbd_common.cuh"
#include "pbd_kernels.h"
#include "tma_util.h"

namespace la {
namespace {

constexpr int kNT = kTileKeys;         // keys per tile
constexpr int kStages = 2;
constexpr int kThreadsTc = 192;
constexpr int kTmemCols = 256;
constexpr int kColO = 128;             // O accumulator columns [128, 256); S buffers at 0, 64

constexpr int kHalfBytes = 64 * 128;            // 64 rows x 128 B (one swizzle column)
constexpr int kQBytes = 2 * kHalfBytes;         // Q: 2 halves of 64 channels
constexpr int kTileBytes = 2 * kHalfBytes;      // one K (or V) tile: 2 halves
constexpr int kStageBytes = 2 * kTileBytes;     // K + V
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffPhi = kOffStage + kStages * kStageBytes;
constexpr int kOffPlo = kOffPhi + kHalfBytes;
constexpr int kOffBar = kOffPlo + kHalfBytes;
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem slot, abort flag
constexpr int kOffPre = kOffMisc + 64;

// Barrier indices.
constexpr int kBarFull = 0;     // [kStages]
constexpr int kBarEmpty = 2;    // [kStages]
constexpr int kBarQFull = 4;
constexpr int kBarQEmpty = 5;
constexpr int kBarSFull = 6;    // [2]
constexpr int kBarPFull = 8;
constexpr int kBarOFull = 9;
constexpr int kBarDrain = 10;

constexpr long long kWaitLimitNs = 2000000000LL;   // 2 s

// Instruction descriptors (kind::f16): D fp32 (bit 4), A bf16 (bits 7..9 = 1),
// B bf16 (bits 10..12 = 1), B major bit 16, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kNT >> 3) << 17) |
                              ((uint32_t)(64 >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(64 >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor, SWIZZLE_128B (layout type 2), descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ long long now_ns() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

struct Ctl {
  volatile int* abort_flag;
  WsHeader* hdr;
};

// Bounded wait for the completion of phase `parity`. Returns false when the CTA is aborting.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Ctl& ctl) {
  const long long limit_ns = kWaitLimitNs;
  if (mbar_try(bar, parity)) return true;
  const long long t0 = now_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*ctl.abort_flag) return false;
      if (now_ns() - t0 > limit_ns) {
        *ctl.abort_flag = 1;
        atomicOr(&ctl.hdr->err, kErrTimeout);
        return false;
      }
    }
  }
}

// Wait used while tearing down: ignores the abort flag, gives up after `limit_ns`.
__device__ __noinline__ void mbar_drain(uint32_t bar, uint32_t parity, long long limit_ns) {
  const long long t0 = now_ns();
  while (!mbar_try(bar, parity)) {
    if (now_ns() - t0 > limit_ns) return;
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 lanes x 256 bits, repeated 8 times: 32 registers (columns 8k + 2(t%4) + {0,1}).
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Same shape repeated 4 times: 16 registers.
__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, float (&v)[16]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ int tiles_of(const Segment& sg) { return (sg.j1 - sg.j0 + kNT - 1) / kNT; }

}  // namespace

__global__ void __launch_bounds__(kThreadsTc, 2)
    pbd_attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmq, Problem p) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  const uint32_t sQ = sb + kOffQ, sStage = sb + kOffStage, sPhi = sb + kOffPhi, sPlo = sb + kOffPlo;
  const uint32_t sBar = sb + kOffBar;
  auto bar = [&](int i) { return sBar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 8);
  int* pre = reinterpret_cast<int*>(base + kOffPre);
  int* warp_tot = pre + round_up(p.B + 1, 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Ctl ctl{abort_flag, p.hdr};

  // Q padding rows R..63 must read as zero: clear the Q tile once (TMA rewrites rows < R).
  for (int i = tid; i < kQBytes / 16; i += kThreadsTc)
    reinterpret_cast<uint4*>(base + kOffQ)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    mbar_init(bar(kBarSFull + 0), 1);
    mbar_init(bar(kBarSFull + 1), 1);
    mbar_init(bar(kBarPFull), 128);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  plan_prefix(p, pre, warp_tot);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const long long T = (long long)p.Hkv * pre[p.B];
  if (blockIdx.x == 0) {
    for (int i = tid; i <= p.B; i += kThreadsTc) p.pre_g[i] = pre[i];
  }
  const long long C = plan_chunk(p, T);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SegmentIter it = plan_begin(p, pre, blockIdx.x, C, T);
      Segment sg;
      int g = 0, nseg = 0;
      bool ok = true;
      while (ok && it.next(p, pre, blockIdx.x, sg)) {
        if (nseg > 0 && !mbar_wait(bar(kBarQEmpty), (nseg - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(bar(kBarQFull), 2u * p.R * 128u);
        tma_load_3d(sQ, &tmq, bar(kBarQFull), 0, sg.h * p.G, sg.b * p.W);
        tma_load_3d(sQ + kHalfBytes, &tmq, bar(kBarQFull), 64, sg.h * p.G, sg.b * p.W);
        const int row0 = (sg.b * p.Hkv + sg.h) * p.S + sg.j0;
        const int nt = tiles_of(sg);
        for (int t = 0; t < nt; ++t, ++g) {
          const int st = g % kStages, use = g / kStages;
          if (use > 0 && !mbar_wait(bar(kBarEmpty + st), (use - 1) & 1, ctl)) { ok = false; break; }
          const uint32_t dk = sStage + st * kStageBytes, dv = dk + kTileBytes;
          mbar_expect_tx(bar(kBarFull + st), (uint32_t)kStageBytes);
          const int row = row0 + t * kNT;
          tma_load_2d(dk, &tmk, bar(kBarFull + st), 0, row);
          tma_load_2d(dk + kHalfBytes, &tmk, bar(kBarFull + st), 64, row);
          tma_load_2d(dv, &tmv, bar(kBarFull + st), 0, row);
          tma_load_2d(dv + kHalfBytes, &tmv, bar(kBarFull + st), 64, row);
        }
        ++nseg;
      }
      // Drain: the copies issued last must have landed before shared memory is released.
      for (int back = 1; back <= kStages && g - back >= 0; ++back) {
        const int gg = g - back;
        mbar_drain(bar(kBarFull + gg % kStages), (gg / kStages) & 1, 100000000LL);
      }
      if (nseg > 0) mbar_drain(bar(kBarQFull), (nseg - 1) & 1, 100000000LL);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      SegmentIter it = plan_begin(p, pre, blockIdx.x, C, T);
      Segment sg;
      int g = 0, nseg = 0;
      bool ok = true;
      const uint64_t sbo = 1024;
      auto issue_qk = [&](int gg) {
        const int st = gg % kStages;
        const uint32_t d = tmem + (uint32_t)((gg & 1) * kNT);
        const uint32_t kb = sStage + st * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kHalfBytes + (kk & 3) * 32);
          umma(d, sdesc(sQ + off, 16, sbo), sdesc(kb + off, 16, sbo), kIdescQK, kk > 0);
        }
      };
      auto issue_pv = [&](int gg) {
        const int st = gg % kStages;
        const uint32_t vb = sStage + st * kStageBytes + kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kNT / 16; ++kk) {
          const uint64_t bdesc = sdesc(vb + kk * 2048, kHalfBytes, sbo);
          umma(tmem + kColO, sdesc(sPhi + kk * 32, 16, sbo), bdesc, kIdescPV, kk > 0);
          umma(tmem + kColO, sdesc(sPlo + kk * 32, 16, sbo), bdesc, kIdescPV, 1);
        }
      };
      while (ok && it.next(p, pre, blockIdx.x, sg)) {
        const int nt = tiles_of(sg);
        if (!mbar_wait(bar(kBarQFull), nseg & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const int g0 = g;
        if (!mbar_wait(bar(kBarFull + g0 % kStages), (g0 / kStages) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        issue_qk(g0);
        umma_commit(bar(kBarSFull + (g0 & 1)));
        if (nt == 1) umma_commit(bar(kBarQEmpty));
        for (int t = 0; t < nt; ++t) {
          const int gt = g0 + t;
          if (t + 1 < nt) {
            const int gn = gt + 1;
            if (!mbar_wait(bar(kBarFull + gn % kStages), (gn / kStages) & 1, ctl)) { ok = false; break; }
            tc_fence_after();
            issue_qk(gn);
            umma_commit(bar(kBarSFull + (gn & 1)));
            if (t + 2 == nt) umma_commit(bar(kBarQEmpty));
          }
          if (!mbar_wait(bar(kBarPFull), gt & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          issue_pv(gt);
          umma_commit(bar(kBarOFull));
          umma_commit(bar(kBarEmpty + gt % kStages));
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
    const int q4 = warp & 3;
    const int t0 = lane & 3, t1 = lane >> 2;
    const int ra = 16 * q4 + t1, rb = ra + 8;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int stid = tid - 64;  // 0..127
    SegmentIter it = plan_begin(p, pre, blockIdx.x, C, T);
    Segment sg;
    int g = 0;
    bool ok = true;
    while (ok && it.next(p, pre, blockIdx.x, sg)) {
      const int nt = tiles_of(sg);
      const int lim_a = (ra < p.R) ? min(row_limit(p, sg.n, ra), sg.j1) : 0;
      const int lim_b = (rb < p.R) ? min(row_limit(p, sg.n, rb), sg.j1) : 0;
      float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
      float alpha_a = 0.f, alpha_b = 0.f;
      float o[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) o[i] = 0.f;

      auto fold_o = [&](int gg, float aa, float ab) -> bool {
        if (!mbar_wait(bar(kBarOFull), gg & 1, ctl)) return false;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[16];
          tmem_ld_x4(tmem + lane_base + kColO + 32 * c, v);
          tc_wait_ld();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = 16 * c + 4 * k;
            o[i + 0] = fmaf(o[i + 0], aa, v[4 * k + 0]);
            o[i + 1] = fmaf(o[i + 1], aa, v[4 * k + 1]);
            o[i + 2] = fmaf(o[i + 2], ab, v[4 * k + 2]);
            o[i + 3] = fmaf(o[i + 3], ab, v[4 * k + 3]);
          }
        }
        return true;
      };

      for (int t = 0; t < nt; ++t) {
        const int gt = g + t;
        const int jt = sg.j0 + t * kNT;
        if (!mbar_wait(bar(kBarSFull + (gt & 1)), (gt >> 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        float s[32];
        tmem_ld_x8(tmem + lane_base + (uint32_t)((gt & 1) * kNT), s);
        tc_wait_ld();

        // Mask and row maxima (log2 domain). Column of s[4k+e]: 8k + 2*t0 + (e & 1).
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = jt + 8 * k + 2 * t0 + e;
            float xa = (j < lim_a) ? s[4 * k + e] * p.scale_log2 : -INFINITY;
            float xb = (j < lim_b) ? s[4 * k + 2 + e] * p.scale_log2 : -INFINITY;
            s[4 * k + e] = xa;
            s[4 * k + 2 + e] = xb;
            mx_a = fmaxf(mx_a, xa);
            mx_b = fmaxf(mx_b, xb);
          }
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float na = (mn_a == -INFINITY) ? 1.f : fast_exp2(m_a - mn_a);
        const float nb = (mn_b == -INFINITY) ? 1.f : fast_exp2(m_b - mn_b);
        const float ref_a = (mn_a == -INFINITY) ? 0.f : mn_a;
        const float ref_b = (mn_b == -INFINITY) ? 0.f : mn_b;
        m_a = mn_a;
        m_b = mn_b;
        float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float pa = fast_exp2(s[4 * k + e] - ref_a);
            const float pb = fast_exp2(s[4 * k + 2 + e] - ref_b);
            s[4 * k + e] = pa;
            s[4 * k + 2 + e] = pb;
            sum_a += pa;
            sum_b += pb;
          }
        }
        l_a = l_a * na + sum_a;
        l_b = l_b * nb + sum_b;

        // Fold the previous tile's PV (its P buffer is then free), remember this tile's alpha.
        if (t > 0 && !fold_o(gt - 1, alpha_a, alpha_b)) { ok = false; break; }
        alpha_a = na;
        alpha_b = nb;

        // P = P_hi + P_lo as bf16 into the swizzled K-major operand tiles.
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          __nv_bfloat162 ha = __floats2bfloat162_rn(s[4 * k + 0], s[4 * k + 1]);
          __nv_bfloat162 hb = __floats2bfloat162_rn(s[4 * k + 2], s[4 * k + 3]);
          float2 fa = __bfloat1622float2(ha), fb = __bfloat1622float2(hb);
          __nv_bfloat162 la2 = __floats2bfloat162_rn(s[4 * k + 0] - fa.x, s[4 * k + 1] - fa.y);
          __nv_bfloat162 lb2 = __floats2bfloat162_rn(s[4 * k + 2] - fb.x, s[4 * k + 3] - fb.y);
          const uint32_t offa = (uint32_t)(ra * 128 + ((k ^ (ra & 7)) << 4) + 4 * t0);
          const uint32_t offb = (uint32_t)(rb * 128 + ((k ^ (rb & 7)) << 4) + 4 * t0);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPhi + offa), "r"(pack_bf16x2(ha)));
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPhi + offb), "r"(pack_bf16x2(hb)));
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPlo + offa), "r"(pack_bf16x2(la2)));
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPlo + offb), "r"(pack_bf16x2(lb2)));
        }
        // Rows of the V tile past the segment end hold other data: zero them so 0 * x
        // cannot turn into NaN in the tensor-core product.
        const int valid = min(kNT, sg.j1 - jt);
        if (valid < kNT) {
          const uint32_t vb = sStage + (gt % kStages) * kStageBytes + kTileBytes;
          for (int idx = stid; idx < (kNT - valid) * 16; idx += 128) {
            const int row = valid + (idx >> 4), ch = idx & 15;
            const uint32_t a = vb + (ch >> 3) * kHalfBytes + row * 128 + (ch & 7) * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(0u), "r"(0u),
                         "r"(0u), "r"(0u));
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kBarPFull));
      }
      if (!ok) break;
      if (!fold_o(g + nt - 1, alpha_a, alpha_b)) { ok = false; break; }
      g += nt;

      // Row sums across the quad, then the output or the partial.
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = half ? rb : ra;
        if (r >= p.R) continue;
        const float l = half ? l_b : l_a;
        const float m = half ? m_b : m_a;
        if (sg.whole) {
          const float inv = 1.f / l;
          __nv_bfloat16* dst = p.out + out_row_offset(p, sg.b, sg.h, r);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int d = 8 * k + 2 * t0;
            __nv_bfloat162 v2 = __floats2bfloat162_rn(o[4 * k + 2 * half] * inv,
                                                      o[4 * k + 2 * half + 1] * inv);
            *reinterpret_cast<__nv_bfloat162*>(dst + d) = v2;
          }
        } else {
          float* slot = slot_ptr(p, sg.slot);
          if (t0 == 0) {
            slot[r] = m;
            slot[p.rows_pad + r] = l;
          }
          float* acc = slot + 2 * p.rows_pad + (size_t)r * kHeadDim;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int d = 8 * k + 2 * t0;
            *reinterpret_cast<float2*>(acc + d) = make_float2(o[4 * k + 2 * half], o[4 * k + 2 * half + 1]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

int tc_ctas_per_sm() { return 2; }
int tc_min_chunk() { return kNT; }

size_t tc_smem_bytes(int B) {
  const size_t pre_ints = (size_t)round_up(B + 1, 4) + 32;
  return 1024 + kOffPre + pre_ints * 4;
}

cudaError_t launch_attn_tc(const Problem& p, const void* tmap_k, const void* tmap_v,
                           const void* tmap_q, cudaStream_t stream) {
  const size_t smem = tc_smem_bytes(p.B);
  cudaError_t e = cudaFuncSetAttribute(pbd_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  pbd_attn_tc_kernel<<<p.num_ctas, kThreadsTc, smem, stream>>>(
      *static_cast<const CUtensorMap*>(tmap_k), *static_cast<const CUtensorMap*>(tmap_v),
      *static_cast<const CUtensorMap*>(tmap_q), p);
  return cudaGetLastError();
}

}  // namespace la
