// Step a6: merge of the split-KV partials of every sequence into the bf16 output.
//
// For a row with partials (m_k, l_k, acc_k), k over the CTAs that held part of the sequence,
// with m in the log2 domain:
//   M = max_k m_k,  w_k = 2^(m_k - M),  out = (sum_k w_k acc_k) / (sum_k w_k l_k),
// rounded to bf16 (RNE). Sequences held whole by one CTA were written by the attention kernel
// and are skipped here. Sequences with an invalid prefix length (no visible keys) get zero
// rows and raise the sticky overflow flag.
//
// One warp per output row (4 rows per 128-thread block): lane k holds partial k's maximum and
// sum, the warp reduces them (weights kept in shared memory), and each lane accumulates 4 of
// the 128 channels over the partials with independent 16-byte loads. The first KM partial rows
// are loaded in one round trip with the maxima and sums: KM = 16, or 40 where a sequence can
// be split into more than 16 pieces at a small batch (one sequence over up to 40 CTAs, e.g. a
// 4096-token prefix at one tile per CTA), where a second round trip would otherwise follow.
#include "pbd_common.cuh"
#include "pbd_kernels.h"

namespace la {

constexpr int kCombineRows = 4;
constexpr int kCombineMaxSlots = 1024;   // >= partials of one sequence (<= grid size)
// kMerge partials are loaded in the first round trip; with kMerge = 4 the kernel needs so few
// registers that 12 blocks fit on an SM, so a batch of many short split sequences (thousands
// of rows, two or three partials each) is merged in one wave of blocks.
template <int kMerge>
__global__ void __launch_bounds__(32 * kCombineRows, kMerge <= 4 ? 12 : 1) pbd_combine_kernel(Problem p) {
  __shared__ float s_w[kCombineRows][kCombineMaxSlots];   // (16 KB)
  pdl_trigger();
  const int s = blockIdx.y;            // sequence = b * Hkv + h
  const int b = s / p.Hkv, h = s - b * p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kCombineRows + warp;
  // The plan of sequence b: its units u, the units pb before it and the total. For a batch of
  // up to 256 sequences each warp derives it before the dependency wait from seq_lens and
  // window_lens, 32 sequences at a time (L2 reads; the attention kernel before this one does
  // not write them, and it lets this kernel start only after its own wait, so their last
  // writer has completed). After the wait only the partials remain to be read. A larger batch
  // reads the prefix sums that attention CTA 0 published.
  int u = 0, pb = 0, ptot = 0, wb = p.W;
  const bool early = p.B <= 256;
  if (early) {
    int carry = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      int x = 0, w = p.W;
      if (b0 + lane < p.B) {
        const int P = __ldcg(p.seq_lens + b0 + lane);
        if (p.window_lens) w = __ldcg(p.window_lens + b0 + lane);
        x = plan_units_of(p, visible_of(p, P, w));
      }
      int incl = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b >= b0 && b < b0 + 32) {   // (warp-uniform)
        u = __shfl_sync(0xffffffffu, x, b - b0);
        pb = carry + __shfl_sync(0xffffffffu, incl - x, b - b0);
        wb = __shfl_sync(0xffffffffu, w, b - b0);
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    ptot = carry;
  }
  pdl_wait();
  if (!early) {
    pb = p.pre_g[b];
    u = p.pre_g[b + 1] - pb;
    ptot = p.pre_g[p.B];
    wb = window_of(p, b);
  }
  if (r >= p.R) return;
  __nv_bfloat16* dst = p.out + out_row_offset(p, b, h, r);
  const long long T = (long long)p.Hkv * ptot;
  const long long off = (long long)p.Hkv * pb + (long long)h * u;
  if (u > 0 && r / p.G >= wb) {
    // Padding row of a shorter window: written as zeros by whichever kernel owns the
    // sequence (here if it was split; the attention kernel if it was whole).
    int f0, l0;
    plan_tile_ctas(p, off, u, T, &f0, &l0);
    if (f0 != l0) reinterpret_cast<uint2*>(dst)[lane] = make_uint2(0u, 0u);
    return;
  }
  if (u == 0) {
    reinterpret_cast<uint2*>(dst)[lane] = make_uint2(0u, 0u);
    if (lane == 0 && r == 0 && h == 0) atomicOr(&p.hdr->err, kErrSeqOverflow);
    return;
  }
  int c0, c1;
  plan_tile_ctas(p, off, u, T, &c0, &c1);
  if (c0 == c1) return;
  const int ns = c1 - c0 + 1;
  const size_t stride = slot_floats(p.rows_pad);
  const float* base = p.partials + (size_t)(c0 + s) * stride;

  // Latency, not bandwidth, decides this kernel: the partials were just written and sit in
  // L2. So the first kMerge partial rows are loaded together with the maxima and sums (one
  // round trip for all of them), and the weights are applied afterwards.
  const float* acc0 = base + 2 * p.rows_pad + (size_t)r * kHeadDim + 4 * lane;
  float4 a[kMerge];
#pragma unroll
  for (int u = 0; u < kMerge; ++u)
    if (u < ns) a[u] = *reinterpret_cast<const float4*>(acc0 + (size_t)u * stride);
  // Maxima and sums of partials lane and lane + 32, in the same round trip (up to 64
  // partials; more take further round trips).
  float mk0 = -INFINITY, lk0 = 0.f, mk1 = -INFINITY, lk1 = 0.f;
  if (lane < ns) {
    mk0 = base[(size_t)lane * stride + r];
    lk0 = base[(size_t)lane * stride + p.rows_pad + r];
  }
  if (lane + 32 < ns) {
    mk1 = base[(size_t)(lane + 32) * stride + r];
    lk1 = base[(size_t)(lane + 32) * stride + p.rows_pad + r];
  }
  float M = fmaxf(mk0, mk1);
  for (int k = lane + 64; k < ns; k += 32) M = fmaxf(M, base[(size_t)k * stride + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = (mk0 == -INFINITY) ? 0.f : fast_exp2(mk0 - M);
  const float w1 = (mk1 == -INFINITY) ? 0.f : fast_exp2(mk1 - M);
  if (lane < ns) s_w[warp][lane] = w0;
  if (lane + 32 < ns) s_w[warp][lane + 32] = w1;
  float L = fmaf(w0, lk0, w1 * lk1);
  for (int k = lane + 64; k < ns; k += 32) {
    const float m2 = base[(size_t)k * stride + r];
    const float w2 = (m2 == -INFINITY) ? 0.f : fast_exp2(m2 - M);
    s_w[warp][k] = w2;
    L = fmaf(w2, base[(size_t)k * stride + p.rows_pad + r], L);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  __syncwarp();

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kMerge; ++u) {
    if (u < ns) {
      const float w = s_w[warp][u];
      acc.x = fmaf(w, a[u].x, acc.x);
      acc.y = fmaf(w, a[u].y, acc.y);
      acc.z = fmaf(w, a[u].z, acc.z);
      acc.w = fmaf(w, a[u].w, acc.w);
    }
  }
  for (int k = kMerge; k < ns; ++k) {
    const float4 v = *reinterpret_cast<const float4*>(acc0 + (size_t)k * stride);
    const float w = s_w[warp][k];
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
  }
  const float inv = 1.f / L;
  __nv_bfloat162 o01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  __nv_bfloat162 o23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t*>(&o01);
  packed.y = *reinterpret_cast<uint32_t*>(&o23);
  reinterpret_cast<uint2*>(dst)[lane] = packed;
}

cudaError_t launch_combine(const Problem& p, cudaStream_t stream) {
  if (p.num_ctas > kCombineMaxSlots) return cudaErrorInvalidValue;
  dim3 grid((p.R + kCombineRows - 1) / kCombineRows, p.B * p.Hkv);
  // A sequence is split into at most one piece per key tile of its capacity, and (with C >= 1
  // units per CTA) at most one per CTA; the larger first batch pays off only where that bound
  // exceeds 16 and the batch is small enough for the merge to be latency-bound.
  const long long tiles = (p.S + p.unit - 1) / p.unit;
  const long long pieces = tiles < p.num_ctas ? tiles : p.num_ctas;
  if (pieces > 16 && (long long)p.B * p.Hkv <= 4)
    return launch_pdl(pbd_combine_kernel<40>, grid, dim3(32 * kCombineRows), 0, stream, p);
  // With at least half as many (sequence, KV head) pairs as attention CTAs, a pair spans few
  // CTAs (a longer one still merges correctly, through the loop past the first batch).
  if (2LL * p.B * p.Hkv >= p.num_ctas)
    return launch_pdl(pbd_combine_kernel<4>, grid, dim3(32 * kCombineRows), 0, stream, p);
  return launch_pdl(pbd_combine_kernel<16>, grid, dim3(32 * kCombineRows), 0, stream, p);
}

}  // namespace la
