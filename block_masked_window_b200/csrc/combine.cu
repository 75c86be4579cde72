// Step a6: merge of the split-KV partials of every sequence into the bf16 output.
//
// For a row with partials (m_k, l_k, acc_k), k over the CTAs that held part of the sequence,
// with m in the log2 domain:
//   M = max_k m_k,  w_k = 2^(m_k - M),  out = (sum_k w_k acc_k) / (sum_k w_k l_k),
// rounded to bf16 (RNE). Sequences held whole by one CTA were written by the attention kernel
// and are skipped here. Sequences with an invalid prefix length (no visible keys) get zero
// rows and raise the sticky overflow flag.
#include "pbd_common.cuh"
#include "pbd_kernels.h"

namespace la {

__global__ void __launch_bounds__(256) pbd_combine_kernel(Problem p) {
  const int s = blockIdx.x;            // sequence = b * Hkv + h
  const int b = s / p.Hkv, h = s - b * p.Hkv;
  const int n = p.pre_g[b + 1] - p.pre_g[b];
  const int nthr = blockDim.x;
  if (n == 0) {
    for (int idx = threadIdx.x; idx < p.R * (kHeadDim / 8); idx += nthr) {
      int r = idx / (kHeadDim / 8), c = idx % (kHeadDim / 8);
      *reinterpret_cast<uint4*>(p.out + out_row_offset(p, b, h, r) + c * 8) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    if (threadIdx.x == 0 && h == 0) atomicOr(&p.hdr->err, kErrSeqOverflow);
    return;
  }
  const long long T = (long long)p.Hkv * p.pre_g[p.B];
  const long long C = plan_chunk(p, T);
  const long long off = (long long)p.Hkv * p.pre_g[b] + (long long)h * n;
  const int c0 = (int)(off / C), c1 = (int)((off + n - 1) / C);
  if (c0 == c1) return;

  // One thread per (row, 4 channels).
  for (int idx = threadIdx.x; idx < p.R * (kHeadDim / 4); idx += nthr) {
    const int r = idx / (kHeadDim / 4), d = (idx % (kHeadDim / 4)) * 4;
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c) M = fmaxf(M, slot_ptr(p, c + s)[r]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = c0; c <= c1; ++c) {
      const float* sl = slot_ptr(p, c + s);
      const float mk = sl[r];
      if (mk == -INFINITY) continue;
      const float w = fast_exp2(mk - M);
      L = fmaf(w, sl[p.rows_pad + r], L);
      const float4 a = *reinterpret_cast<const float4*>(sl + 2 * p.rows_pad + (size_t)r * kHeadDim + d);
      acc.x = fmaf(w, a.x, acc.x);
      acc.y = fmaf(w, a.y, acc.y);
      acc.z = fmaf(w, a.z, acc.z);
      acc.w = fmaf(w, a.w, acc.w);
    }
    const float inv = 1.f / L;
    __nv_bfloat162 o01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 o23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&o01);
    packed.y = *reinterpret_cast<uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(p.out + out_row_offset(p, b, h, r) + d) = packed;
  }
}

cudaError_t launch_combine(const Problem& p, cudaStream_t stream) {
  pbd_combine_kernel<<<p.B * p.Hkv, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace la
