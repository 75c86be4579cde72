// tcgen05 + TMA block-causal prefill attention for sm_100a.
//
// The prefill of a block-diffusion decoder uses a block mask over whole sequences: token i
// attends key j when j <= i or when both lie in the same block of `block_size` consecutive
// tokens (SDLM-style block mask; the PBD window is the last block of it). For contiguous
// blocks this is one key limit per row: row i sees keys [0, min(T, (i / bs + 1) * bs)).
//
// One CTA computes 128 query rows of one (sequence, query head) against the keys they may
// see, flash-attention style, on the tensor cores, per tile of 128 keys and per key half h:
//   S_h = Q K_h^T  (M = 128 query rows, N = 64 keys,       K = 128 channels) -> TMEM fp32
//   O_h += P_h V_h (M = 128 query rows, N = 128 channels,  K = 64 keys)      -> TMEM fp32
// The two key halves are processed independently, as two interleaved split-KV streams: half
// h's probabilities multiply V rows [64h, 64h + 64) into their own accumulator O_h (TMEM: two
// S buffers and O_0, O_1 fill the 512 columns), with their own reference maximum and row sum,
// and the two are merged once at the end. Two softmax threads own query row r (TMEM lane r),
// one per key half: each reads its 64 scores from TMEM, keeps its lazy reference maximum
// (raised only when a score exceeds it by 2^8; the warp then rescales its O_h rows after the
// previous PV product has completed) and row sum in registers, and writes its half of the row
// of P back into tensor memory, over the 64 score columns it has just read, packed two keys
// per 32-bit column; the PV product reads it there (A from tensor memory). A single bf16
// rounding of P would add a relative L2 error of ~1e-3 to the output, on top of the ~1.7e-3 of
// the output's own bf16 rounding, so P is kept more precisely in one of two ways, chosen per
// CTA:
//   * fp16 P (relative rounding 2^-11, 8x finer than bf16) times V converted to fp16 once per
//     call by prefill_v16_kernel. The conversion is exact for 2^-17 <= |v| <= 65504, so it is
//     used when every V tile the CTA reads has its largest |v| in [2^-6, 65520) (or is all
//     zeros): smaller elements then err by at most 2^-25 <= 2^-19 of the tile's largest. One
//     product per key half and tile.
//   * otherwise P = P_hi + P_lo, two bf16 parts (P_lo = bf16(P - P_hi), residual ~2^-17 P;
//     P_hi in the first 32 columns, P_lo in the next 32), each multiplied by the bf16 V tile:
//     two products per key half and tile.
// P lives in the S buffer of its tile, so it is double-buffered with S, and shared memory
// holds only Q and the K and V rings (three stages each). S_h of tile t + 2 reuses its
// columns once PV_h of tile t has completed.
// Each half has its own S and P barriers, so nothing ties the two halves together until the
// end: the two softmax warps sharing a scheduler (one per half) drift apart by about half a
// tile, and one's exponentials overlap the other's maxima, TMEM traffic and waits instead of
// both queueing on the MUFU at once (measured: the softmax of a tile took ~1200 cycles with
// the halves apart, ~1750 in step). The price is QK^T as N = 64 products, which keep the
// tensor core nearly as long as N = 128 ones (53 against 64 cycles each). At the end the
// pair merges (m, l, O_0, O_1) and each thread normalises and stores 64 of the row's 128
// output channels. The softmax uses paired fp32 instructions (one FMA and one add per two
// scores) and three-input maxima.
//
// Roles (384 threads, 1 CTA per SM): warp 0 TMA for Q and the K ring, warp 10 TMA for the V
// ring, warp 1 TMEM owner and QK^T issuer, warp 11 PV issuer, warps 2..9 softmax (warps w and
// w + 4 share the TMEM lane quarter w % 4, one per key half). Query tiles are scheduled
// longest first (the last tiles see the most keys). Every wait is bounded (sticky timeout
// flag, drain, TMEM freed, return).
#include "pbd_common.cuh"
#include "pbd_kernels.h"
#include "tc_util.cuh"
#include "tma_util.h"

namespace la {
namespace {

using namespace tc;

constexpr int kBM = 128;                 // query rows per CTA
constexpr int kBN = 128;                 // keys per tile
constexpr int kPfThreads = 384;         // 12 warps
constexpr int kPfStages = 3;             // K and V ring depth
constexpr int kPHalf = 128 * 128;        // one 64-column half of a 128-row bf16 tile (16 KB)
constexpr int kPTile = 2 * kPHalf;       // 32 KB: a 128-row x 128-channel bf16 operand tile
constexpr float kPfLazy = 8.f;           // log2 units
constexpr int kPfTmemCols = 512;
constexpr int kColS = 0;                 // S (then P_hi | P_lo per key half): 2 buffers x 128
constexpr int kColO = 2 * kBN;           // O of key half 0 (128 columns), then of key half 1

constexpr int kBQFull = 0;
constexpr int kBKFull = 1;                        // [kPfStages]
constexpr int kBKEmpty = kBKFull + kPfStages;     // [kPfStages]
constexpr int kBVFull = kBKEmpty + kPfStages;     // [kPfStages]
constexpr int kBVEmpty = kBVFull + kPfStages;     // [kPfStages]
constexpr int kBSFull = kBVEmpty + kPfStages;     // [key half][tile parity]: S_h of the tile
constexpr int kBPFull = kBSFull + 4;              // [key half][tile parity], one arrival per warp
constexpr int kBOFull = kBPFull + 4;              // [key half][tile parity]
constexpr int kBDrain = kBOFull + 4;
constexpr int kBNum = kBDrain + 1;

// Shared memory: Q | K ring | V ring | barriers | misc.
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kPTile;
constexpr int kOffV = kOffK + kPfStages * kPTile;
constexpr int kOffBar = kOffV + kPfStages * kPTile;
constexpr int kOffMisc = kOffBar + kBNum * 8;
constexpr int kPfSmem = kOffMisc + 16;
// The final (m, l) exchange of the two halves ([2][2 halves][128 rows] floats) reuses the Q
// tile: it happens after every product of the CTA has completed.
constexpr int kOffX = kOffQ;
constexpr size_t kPfSmemAlloc = (size_t)kPfSmem + 1024;   // + alignment slack

// Named barrier 1 over the 256 softmax threads.
__device__ __forceinline__ void pf_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// The 64 probabilities of one key half of a row as fp16, two keys per 32-bit word (the lower
// key in the low half), into 32 tensor-memory columns from `taddr`.
__device__ __forceinline__ void store_p16_tmem(uint32_t taddr, const float (&x)[64]) {
  uint32_t w[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    __half2 h2 = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t*>(&h2);
  }
  tmem_st32(taddr, w);
}

// The same as bf16 P_hi and P_lo, into 32 + 32 tensor-memory columns from `taddr`.
__device__ __forceinline__ void store_p_tmem(uint32_t taddr, const float (&x)[64]) {
  uint32_t hi[32], lo[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float a = x[2 * e], b = x[2 * e + 1];
    __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
    hi[e] = *reinterpret_cast<uint32_t*>(&h2);
    const float ha = __uint_as_float(hi[e] << 16), hb = __uint_as_float(hi[e] & 0xFFFF0000u);
    __nv_bfloat162 l2 = __floats2bfloat162_rn(a - ha, b - hb);
    lo[e] = *reinterpret_cast<uint32_t*>(&l2);
  }
  tmem_st32(taddr, hi);
  tmem_st32(taddr + 32, lo);
}

// Maximum of three (one instruction; a NaN operand is ignored, as by fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Paired fp32 arithmetic (two lanes of a 64-bit register).
__device__ __forceinline__ uint64_t pack_f32x2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}


// Bounded wait of an MMA-issuing thread for one phase of a barrier (hardware-suspended
// try_wait). The limit is counted in SM clock cycles, a cheap register read (a %globaltimer
// read costs tens of nanoseconds, on these threads' critical path): limit_ns * 2 cycles last
// at least limit_ns at the 1.965 GHz maximum SM clock.
constexpr long long kPfCyclesPerNs = 2;
__device__ __forceinline__ bool mma_poll(uint32_t bar, uint32_t parity, const Ctl& ctl) {
  if (mbar_test(bar, parity)) return true;
  const long long c0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*ctl.abort_flag) return false;
      if (clock64() - c0 > ctl.limit_ns * kPfCyclesPerNs) {
        *ctl.abort_flag = 1;
        atomicOr(&ctl.hdr->err, kErrTimeout);
        return false;
      }
    }
  }
}

}  // namespace

// V rows [0, T_b) of every (sequence, KV head) as fp16 in the workspace, one 128-row tile per
// block, with the tile's flag: 1 when its largest |v| lies in [2^-6, 65520) or the tile holds
// only zeros (NaN elements are carried over and do not count), i.e. when the fp16 product
// is as accurate as the bf16 P_hi + P_lo one (see above). bf16 -> fp16 is exact for
// 2^-17 <= |v| <= 65504.
__global__ void __launch_bounds__(256) prefill_v16_kernel(PrefillProblem p) {
  const int t = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  pdl_wait();   // V and seq_lens may come from the previous kernel of the stream
  pdl_trigger();
  int Tb = __ldg(p.seq_lens + b);
  if (Tb < 0 || Tb > p.T || Tb > p.S) Tb = 0;   // (the attention kernel flags it)
  const int r0 = t * kBN;
  const int rows = max(0, min(kBN, Tb - r0));
  const uint4* src = reinterpret_cast<const uint4*>(p.v + ((size_t)(b * p.Hkv + hk) * p.S + r0) * kHeadDim);
  uint4* dst = reinterpret_cast<uint4*>(p.v16 + ((size_t)(b * p.Hkv + hk) * p.Tp + r0) * kHeadDim);
  float vmax = 0.f;
  for (int c = threadIdx.x; c < rows * (kHeadDim / 8); c += blockDim.x) {
    const uint4 x = __ldg(src + c);   // 8 bf16
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
      vmax = fmaxf(vmax, fmaxf(fabsf(lo), fabsf(hi)));
      __half2 h2 = __floats2half2_rn(lo, hi);
      o[e] = *reinterpret_cast<uint32_t*>(&h2);
    }
    dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  __shared__ float wmax[8];
  vmax = warp_max_f32(vmax);
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = vmax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
    p.v16_ok[(size_t)(b * p.Hkv + hk) * p.ntiles + t] = (m < 65520.f && (m >= 0x1p-6f || m == 0.f)) ? 1 : 0;
  }
}

__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmv16,
                      PrefillProblem p) {
  extern __shared__ __align__(1024) char smem_raw[];
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  const uint32_t sQ = sb + kOffQ, sK = sb + kOffK, sV = sb + kOffV;
  auto bar = [&](int i) { return sb + (uint32_t)kOffBar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = (p.T + kBM - 1) / kBM;
  const int tile = ntiles - 1 - (int)blockIdx.x;   // longest first
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.G;
  const int i0 = tile * kBM;
  Ctl ctl{abort_flag, p.hdr, p.wait_limit_ns};

  pdl_trigger();
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmq)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmv16)) : "memory");
    mbar_init(bar(kBQFull), 1);
    for (int s = 0; s < kPfStages; ++s) {
      mbar_init(bar(kBKFull + s), 1);
      mbar_init(bar(kBKEmpty + s), 1);
      mbar_init(bar(kBVFull + s), 1);
      mbar_init(bar(kBVEmpty + s), 1);
    }
    for (int s = 0; s < 4; ++s) mbar_init(bar(kBSFull + s), 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(bar(kBPFull + s), 4);   // one arrival per softmax warp of the half
      mbar_init(bar(kBOFull + s), 1);
    }
    mbar_init(bar(kBDrain), 2);   // both issuing threads
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kPfTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  pdl_wait();

  // Tokens of this sequence; an invalid length gives zero rows and the sticky flag.
  int Tb = __ldg(p.seq_lens + b);
  if (Tb < 0 || Tb > p.T || Tb > p.S) {
    if (tid == 0 && h == 0 && tile == ntiles - 1) atomicOr(&p.hdr->err, kErrSeqOverflow);
    Tb = 0;
  }
  const int rows_here = min(kBM, p.T - i0);   // rows of `out` this CTA owns
  const int ilast = min(i0 + kBM, Tb) - 1;    // last valid query row of the tile
  const int kmax = (ilast >= i0) ? min(Tb, (ilast / p.bs + 1) * p.bs) : 0;
  const int nk = (kmax + kBN - 1) / kBN;      // key tiles (0: nothing to compute)
  // fp16 P and V when every V tile this CTA reads converted exactly enough.
  int ok16 = 1;
  for (int t = tid; t < nk; t += kPfThreads) ok16 &= __ldcg(p.v16_ok + (size_t)(b * p.Hkv + hk) * p.ntiles + t);
  tc_fence_before();
  const bool f16 = __syncthreads_and(ok16) != 0;
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (nk > 0 && warp == 0) {
    // ------------------------------------------------------------------ TMA: Q, K
    if (lane == 0) {
      bool ok = true;
      mbar_expect_tx(bar(kBQFull), (uint32_t)kPTile);
      tma_load_3d(sQ, &tmq, bar(kBQFull), 0, h, b * p.T + i0);
      tma_load_3d(sQ + kPHalf, &tmq, bar(kBQFull), 64, h, b * p.T + i0);
      const int row0 = (b * p.Hkv + hk) * p.S;
      int t = 0;
      for (; ok && t < nk; ++t) {
        const int s = t % kPfStages, u = t / kPfStages;
        if (u > 0 && !mbar_wait(bar(kBKEmpty + s), (u - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(bar(kBKFull + s), (uint32_t)kPTile);
        tma_load_2d(sK + s * kPTile, &tmk, bar(kBKFull + s), 0, row0 + t * kBN);
        tma_load_2d(sK + s * kPTile + kPHalf, &tmk, bar(kBKFull + s), 64, row0 + t * kBN);
      }
      for (int back = 1; back <= kPfStages && t - back >= 0; ++back) {
        const int tt = t - back;
        mbar_drain(bar(kBKFull + tt % kPfStages), (tt / kPfStages) & 1, 100000000LL);
      }
      mbar_drain(bar(kBQFull), 0, 100000000LL);
    }
  } else if (nk > 0 && warp == 10) {
    // ------------------------------------------------------------------ TMA: V
    if (lane == 0) {
      bool ok = true;
      // (The fp16 copy has the same layout with Tp rows per (sequence, KV head).)
      const CUtensorMap* vmap = f16 ? &tmv16 : &tmv;
      const int row0 = (b * p.Hkv + hk) * (f16 ? p.Tp : p.S);
      int t = 0;
      for (; ok && t < nk; ++t) {
        const int s = t % kPfStages, u = t / kPfStages;
        if (u > 0 && !mbar_wait(bar(kBVEmpty + s), (u - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(bar(kBVFull + s), (uint32_t)kPTile);
        tma_load_2d(sV + s * kPTile, vmap, bar(kBVFull + s), 0, row0 + t * kBN);
        tma_load_2d(sV + s * kPTile + kPHalf, vmap, bar(kBVFull + s), 64, row0 + t * kBN);
      }
      for (int back = 1; back <= kPfStages && t - back >= 0; ++back) {
        const int tt = t - back;
        mbar_drain(bar(kBVFull + tt % kPfStages), (tt / kPfStages) & 1, 100000000LL);
      }
    }
  } else if (nk > 0 && (warp == 1 || warp == 11)) {
    // ------------------------------------------------------------------ MMA issuers
    // Two issuing threads, each in a fixed order: warp 1 issues every QK^T, warp 11 every PV
    // (each commits and drains its own products). A tcgen05.mma returns to its thread only
    // at the tensor core's pace (~65 cycles per M128 N128 K16 product, a few queued), so with
    // one issuer PV(t) queued behind QK^T(t + 1), and QK^T(t + 2) waits for PV(t) (P(t) lives
    // in S's columns): that chain, not a pipe, set the pace.
    if (lane == 0) {
      constexpr uint32_t kIdS64 = idesc_f16(128, 64, 0, 0);    // Q K-major, K K-major, N = 64 keys
      constexpr uint32_t kIdO = idesc_f16(128, 128, 0, 1);     // P (tensor memory), V MN-major
      constexpr uint32_t kIdO16 = idesc_f16(128, 128, 0, 1, kOpFp16);   // the same in fp16
      // Operand descriptors, computed once and advanced by their offsets (the start-address
      // field holds the shared-memory byte address / 16 in 14 bits; every operand lies below
      // 256 KB, so adding offset / 16 never carries out of it).
      const uint64_t dq = sdesc(sQ, 16, 1024, 2), dk = sdesc(sK, 16, 1024, 2);
      const uint64_t dv = sdesc(sV, kPHalf, 1024, 2);
      bool ok = true;
      if (warp == 1) {
        // Per tile, once K(t) has landed: S_0(t), then S_1(t), into buffer t & 1, each after
        // its own half's PV(t - 2) has completed; then the K tile is released.
        ok = mma_poll(bar(kBQFull), 0, ctl);
        for (int t = 0; ok && t < nk; ++t) {
          const int s = t % kPfStages;
          ok = mma_poll(bar(kBKFull + s), (t / kPfStages) & 1, ctl);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            // S_h(t): the scores of key half h (N = 64) into columns [64h, 64h + 64) of the
            // buffer, once PV_h(t - 2) (which reads P_h(t - 2) from them) has completed.
            if (t >= 2) {
              const int tp = t - 2;
              ok = ok && mma_poll(bar(kBOFull + 2 * hh + (tp & 1)), (tp >> 1) & 1, ctl);
            }
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tmem + kColS + (uint32_t)((t & 1) * kBN + 64 * hh);
            const uint64_t kb = dk + ((uint32_t)(s * kPTile + hh * 64 * 128) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (uint32_t)((kk >> 2) * kPHalf + (kk & 3) * 32) >> 4;
              umma(d, dq + off, kb + off, kIdS64, kk > 0);
            }
            // (Self-test of the failure detection: the first completion is withheld, so the
            // half-0 softmax warps' bounded wait for it runs out.)
            if (!((p.stall_test & 1) && t == 0 && hh == 0)) umma_commit(bar(kBSFull + 2 * hh + (t & 1)));
          }
          if (!ok) break;
          umma_commit(bar(kBKEmpty + s));
        }
      } else {
        // O_h += P_h(t) V_h(t) for each half as its P lands: P columns (keys) [64h, 64h + 64)
        // times V rows [64h, 64h + 64), in fp16, or once for each bf16 part of P.
        for (int t = 0; ok && t < nk; ++t) {
          const int s = t % kPfStages;
          ok = mma_poll(bar(kBVFull + s), (t / kPfStages) & 1, ctl);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (!ok) break;
            ok = mma_poll(bar(kBPFull + 2 * hh + (t & 1)), (t >> 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            const uint32_t pa = tmem + kColS + (uint32_t)((t & 1) * kBN + 64 * hh);   // P (P_hi)
            const uint64_t vb = dv + ((uint32_t)(s * kPTile + hh * 4 * 2048) >> 4);
            if (f16) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_ts(tmem + kColO + hh * 128, pa + kk * 8, vb + kk * (2048 >> 4), kIdO16, (t > 0 || kk > 0) ? 1u : 0u);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t vd = vb + kk * (2048 >> 4);
                umma_ts(tmem + kColO + hh * 128, pa + kk * 8, vd, kIdO, (t > 0 || kk > 0) ? 1u : 0u);
                umma_ts(tmem + kColO + hh * 128, pa + 32 + kk * 8, vd, kIdO, 1u);
              }
            }
            umma_commit(bar(kBOFull + 2 * hh + (t & 1)));
          }
          if (!ok) break;
          umma_commit(bar(kBVEmpty + s));   // the V tile is free once both products complete
        }
      }
      // Drain this thread's products before TMEM can be released.
      umma_commit(bar(kBDrain));
      mbar_drain(bar(kBDrain), 0, 100000000LL);
    }
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------------ softmax warps
    const int sub = warp & 3;
    const int half = (warp - 2) >> 2;              // key half of every tile
    const int r = 32 * sub + lane;                 // query row of this thread (TMEM lane)
    const int i = i0 + r;
    const int st = 128 * half + r;                 // softmax thread index 0..255
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * sub) << 16);
    const uint32_t o_addr = lane_addr + kColO + 128 * half;   // this half's accumulator O_h
    const int lim = (i < Tb) ? min(Tb, (i / p.bs + 1) * p.bs) : 0;   // keys [0, lim)
    const float c2 = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;              // this half's reference and row sum
    bool ok = true;
    for (int t = 0; t < nk; ++t) {
      const int j0 = t * kBN + 64 * half;          // first key of this thread's half
      const uint32_t s_addr = lane_addr + kColS + (uint32_t)((t & 1) * kBN + 64 * half);
      // (Every lane waits on the same barrier; the vote keeps the error path warp-uniform.)
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBSFull + 2 * half + (t & 1)), (t >> 1) & 1, ctl))) { ok = false; break; }
      tc_fence_after();
      // This half's 64 scores: two 32-column TMEM reads, one wait.
      float x[64];
      tmem_ld32(s_addr, x);
      tmem_ld32(s_addr + 32, x + 32);
      tc_wait_ld();
      // Halves wholly below this row's limit need no mask (all but the last one or two).
      // (Eight independent partial maxima: a single 64-long dependency chain would leave the
      // issue slots idle.)
      const bool full = j0 + 64 <= lim;
      if (!full) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (j0 + e >= lim) x[e] = -INFINITY;
      }
      // (Three-input maxima: 36 instructions for the 64 scores.)
      float mp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = fmax3(x[u], x[u + 8], x[u + 16]);
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = fmax3(mp[u], x[u + 24], x[u + 32]);
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = fmax3(mp[u], x[u + 40], x[u + 48]);
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = fmaxf(mp[u], x[u + 56]);
      const float mt = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) * c2;
      // Lazy reference: raise it only when a score exceeds it by more than 2^8.
      const bool raise = mt > m_ref + kPfLazy || (m_ref == -INFINITY && mt > -INFINITY);
      float alpha = 1.f;
      if (raise) {
        alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mt);
        l *= alpha;
        m_ref = mt;
      }
      // Rows whose reference moved rescale their O_h row (warp-uniform TMEM access), once
      // this half's previous PV product is complete.
      if (t > 0 && __any_sync(0xffffffffu, raise)) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBOFull + 2 * half + ((t - 1) & 1)), ((t - 1) >> 1) & 1, ctl))) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 128 / 16; ++c) {
          float o[16];
          tmem_ld16(o_addr + 16 * c, o);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= alpha;
          tmem_st16(o_addr + 16 * c, o);
        }
        tc_wait_st();
      }
      // p = 2^(x c2 - m_ref) in fp32 (masked scores are -inf: ex2.approx gives exactly 0 for
      // them), and this tile's part of the row sum.
      const float mref = (m_ref == -INFINITY) ? 0.f : m_ref;
      // (Paired fp32 instructions: one FMA and one add per two scores.)
      const uint64_t c2v = pack_f32x2(c2, c2), nmv = pack_f32x2(-mref, -mref);
      uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        float y0, y1;
        unpack_f32x2(fma_f32x2(pack_f32x2(x[e], x[e + 1]), c2v, nmv), y0, y1);
        x[e] = fast_exp2(y0);
        x[e + 1] = fast_exp2(y1);
        ls[(e >> 1) & 3] = add_f32x2(ls[(e >> 1) & 3], pack_f32x2(x[e], x[e + 1]));
      }
      float l0, l1, l2, l3, l4, l5, l6, l7;
      unpack_f32x2(ls[0], l0, l1);
      unpack_f32x2(ls[1], l2, l3);
      unpack_f32x2(ls[2], l4, l5);
      unpack_f32x2(ls[3], l6, l7);
      l += ((l0 + l1) + (l2 + l3)) + ((l4 + l5) + (l6 + l7));
      // P (fp16, or P_hi and P_lo) over this half's scores in the S buffer of the tile.
      if (f16) store_p16_tmem(s_addr, x);
      else store_p_tmem(s_addr, x);
      tc_wait_st();
      // Keys of this half past the visible range (last tile): zero their V rows so that
      // 0 * x cannot become NaN in the product (those rows may hold anything).
      const int valid = min(kBN, kmax - t * kBN);
      const int zlo = max(valid, 64 * half), zhi = 64 * half + 64;
      if (zlo < zhi) {
        const int s = t % kPfStages;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBVFull + s), (t / kPfStages) & 1, ctl))) { ok = false; break; }
        const uint32_t vbase = sV + s * kPTile;
        for (int idx = r; idx < (zhi - zlo) * 16; idx += 128) {
          const int rr = zlo + (idx >> 4), ch = idx & 15;
          const uint32_t a = vbase + (ch >> 3) * kPHalf + rr * 128 + (ch & 7) * 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(0u), "r"(0u),
                       "r"(0u), "r"(0u));
        }
        // (Only these generic stores need ordering before the async proxy's reads; P went to
        // tensor memory.)
        fence_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBPFull + 2 * half + (t & 1)));
    }
    // Epilogue: both halves' last products complete, then the pair merges
    //   M = max(m_0, m_1), a_h = 2^(m_h - M), out = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1)
    // and each thread stores 64 of the row's 128 channels (128 bytes) as bf16.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(kBOFull + ((nk - 1) & 1)), ((nk - 1) >> 1) & 1, ctl));
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(kBOFull + 2 + ((nk - 1) & 1)), ((nk - 1) >> 1) & 1, ctl));
    tc_fence_after();
    float* xs = reinterpret_cast<float*>(base + kOffX);   // [2 halves][128 rows] x (m, l)
    xs[st] = m_ref;
    xs[256 + st] = l;
    pf_bar();
    const float m0 = half ? xs[st ^ 128] : m_ref, m1 = half ? m_ref : xs[st ^ 128];
    const float l0 = half ? xs[256 + (st ^ 128)] : l, l1 = half ? l : xs[256 + (st ^ 128)];
    const float M = fmaxf(m0, m1);
    const float a0 = (m0 == -INFINITY) ? 0.f : fast_exp2(m0 - M);
    const float a1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - M);
    const float L = a0 * l0 + a1 * l1;
    const float inv = (ok && i < Tb && L > 0.f) ? 1.f / L : 0.f;
    const float w0 = a0 * inv, w1 = a1 * inv;
    __nv_bfloat16* dst = p.out + (((size_t)b * p.T + i) * p.Hq + h) * kHeadDim + 64 * half;
#pragma unroll 1
    for (int c = 0; c < 64 / 16; ++c) {
      float o0[16], o1[16];
      if (ok) {   // (warp-uniform)
        tmem_ld16(lane_addr + kColO + 64 * half + 16 * c, o0);
        tmem_ld16(lane_addr + kColO + 128 + 64 * half + 16 * c, o1);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) o0[e] = o1[e] = 0.f;
      }
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        __nv_bfloat162 v2 = __floats2bfloat162_rn(fmaf(o0[e], w0, o1[e] * w1),
                                                  fmaf(o0[e + 1], w0, o1[e + 1] * w1));
        pk[e >> 1] = *reinterpret_cast<uint32_t*>(&v2);
      }
      if (r < rows_here) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 16 * c);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
  if (nk == 0 && warp >= 2 && warp <= 9) {
    // No valid row in this tile: the owned rows of `out` are zeros (each thread 64 channels).
    const int r = 32 * (warp & 3) + lane, half = (warp - 2) >> 2;
    if (r < rows_here) {
      uint4* d4 = reinterpret_cast<uint4*>(p.out + (((size_t)b * p.T + i0 + r) * p.Hq + h) * kHeadDim +
                                           64 * half);
#pragma unroll
      for (int c = 0; c < 8; ++c) d4[c] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPfTmemCols));
  }
}

size_t prefill_smem_bytes() { return kPfSmemAlloc; }

cudaError_t launch_prefill_tc(const PrefillProblem& p, const void* tmap_q, const void* tmap_k,
                              const void* tmap_v, const void* tmap_v16, cudaStream_t stream) {
  const CUtensorMap& q = *static_cast<const CUtensorMap*>(tmap_q);
  const CUtensorMap& k = *static_cast<const CUtensorMap*>(tmap_k);
  const CUtensorMap& v = *static_cast<const CUtensorMap*>(tmap_v);
  const CUtensorMap& v16 = *static_cast<const CUtensorMap*>(tmap_v16);
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kPfSmemAlloc);
  if (e != cudaSuccess) return e;
  e = launch_pdl(prefill_v16_kernel, dim3(p.ntiles, p.Hkv, p.B), dim3(256), 0, stream, p);
  if (e != cudaSuccess) return e;
  const int ntiles = (p.T + kBM - 1) / kBM;
  return launch_pdl(prefill_tc_kernel, dim3(ntiles, p.Hq, p.B), dim3(kPfThreads), kPfSmemAlloc,
                    stream, q, k, v, v16, p);
}

}  // namespace la
