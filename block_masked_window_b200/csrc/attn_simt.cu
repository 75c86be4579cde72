// CUDA-core (fp32 FFMA) split-KV PBD window attention.
//
// Steps a2..a5 of one PBD decode step for every (sequence, KV head) segment of this CTA's
// share of the flattened key stream (see pbd_common.cuh): scores of the R = W * G query rows
// that share a KV head (W window rows x G grouped query heads) against 32-key tiles, the
// window mask as a per-row key limit, an online softmax in the log2 domain, and the PV
// product. Everything after the bf16 loads is fp32, including the probabilities, so this
// kernel is also the numerical yardstick of the tensor-core path.
//
// Tiles of K and V are double-buffered in shared memory with cp.async (16-byte vectors, zero
// fill past the segment end, so no row outside [j0, j1) is ever read from global memory).
//
// Thread roles, 256 threads:
//  * scores: warp w, half-warp hf, lane t in the half: row group rg = 2w + hf owns rows
//    [rg*RPT, rg*RPT + RPT) and keys t and t + 16 of the tile;
//  * PV: warp w owns rows w, w + 8, ... (2*RPT rows) and each lane 4 of the 128 channels.
#include "pbd_common.cuh"
#include "pbd_kernels.h"

namespace la {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;            // keys per tile
constexpr int kKStride = kHeadDim + 8;  // bf16 elements per K row in smem (272 B, conflict-free)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
               "l"(gmem), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

struct SimtSmem {
  int* pre;
  int* warp_tot;
  float* q;        // [16*RPT][128]
  __nv_bfloat16* k[2];  // [kTile][kKStride]
  __nv_bfloat16* v[2];  // [kTile][128]
  float* pr;       // [16*RPT][kTile]
  float* alpha;    // [16*RPT]
  float* m;        // [16*RPT]
  float* l;        // [16*RPT]
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) / 16 * 16; }

__host__ __device__ inline size_t simt_layout(int rpt, int B, SimtSmem* s, char* base) {
  const int rows = 16 * rpt;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align16(off + bytes);
    return o;
  };
  size_t o_pre = take((size_t)(B + 1) * 4);
  size_t o_wt = take(32 * 4);
  size_t o_q = take((size_t)rows * kHeadDim * 4);
  size_t o_k0 = take((size_t)kTile * kKStride * 2);
  size_t o_k1 = take((size_t)kTile * kKStride * 2);
  size_t o_v0 = take((size_t)kTile * kHeadDim * 2);
  size_t o_v1 = take((size_t)kTile * kHeadDim * 2);
  size_t o_p = take((size_t)rows * kTile * 4);
  size_t o_a = take((size_t)rows * 4);
  size_t o_m = take((size_t)rows * 4);
  size_t o_l = take((size_t)rows * 4);
  if (s) {
    s->pre = reinterpret_cast<int*>(base + o_pre);
    s->warp_tot = reinterpret_cast<int*>(base + o_wt);
    s->q = reinterpret_cast<float*>(base + o_q);
    s->k[0] = reinterpret_cast<__nv_bfloat16*>(base + o_k0);
    s->k[1] = reinterpret_cast<__nv_bfloat16*>(base + o_k1);
    s->v[0] = reinterpret_cast<__nv_bfloat16*>(base + o_v0);
    s->v[1] = reinterpret_cast<__nv_bfloat16*>(base + o_v1);
    s->pr = reinterpret_cast<float*>(base + o_p);
    s->alpha = reinterpret_cast<float*>(base + o_a);
    s->m = reinterpret_cast<float*>(base + o_m);
    s->l = reinterpret_cast<float*>(base + o_l);
  }
  return off;
}

// Issue the cp.async loads of key tile [jt, jt + kTile) of segment `sg` into buffer `buf`.
__device__ __forceinline__ void load_tile(const Problem& p, const SimtSmem& s, const Segment& sg,
                                          int jt, int buf) {
  const size_t head = ((size_t)sg.b * p.Hkv + sg.h) * p.S;
  // 32 rows x 16 vectors x {K, V} = 1024 vectors, 4 per thread.
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    int idx = threadIdx.x + it * kThreads;
    int isv = idx >> 9;            // 0..1
    int r = (idx >> 4) & 31;       // row in tile
    int c = idx & 15;              // 16-byte vector in row
    int j = jt + r;
    bool ok = j < sg.j1;
    size_t row = head + (size_t)(ok ? j : sg.j0);
    const __nv_bfloat16* src = (isv ? p.v : p.k) + row * kHeadDim + c * 8;
    __nv_bfloat16* dst = isv ? (s.v[buf] + r * kHeadDim + c * 8) : (s.k[buf] + r * kKStride + c * 8);
    cp_async16(dst, src, ok ? 16 : 0);
  }
  cp_async_commit();
}

template <int RPT>
__global__ void __launch_bounds__(kThreads) pbd_attn_simt_kernel(Problem p) {
  extern __shared__ __align__(16) char smem_raw[];
  SimtSmem s;
  simt_layout(RPT, p.B, &s, smem_raw);
  constexpr int ROWS = 16 * RPT;
  constexpr int PROWS = 2 * RPT;  // rows per thread in the PV phase

  pdl_wait();
  pdl_trigger();   // after the wait: the merge kernel reads seq_lens before its own wait
  plan_prefix(p, s.pre, s.warp_tot);
  __syncthreads();
  const long long T = (long long)p.Hkv * s.pre[p.B];
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i <= p.B; i += blockDim.x) p.pre_g[i] = s.pre[i];
  }
  SegmentIter it = plan_begin(p, s.pre, blockIdx.x, T);

  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int hf = lane >> 4, tl = lane & 15;
  const int rg = wid * 2 + hf;        // score-phase row group
  const int d0 = (lane) * 4;          // PV-phase channels d0..d0+3

  Segment sg;
  while (it.next(p, s.pre, blockIdx.x, sg)) {
    // ---- Q rows of this (b, h) as fp32; padding rows are zero.
    for (int idx = tid; idx < ROWS * (kHeadDim / 8); idx += kThreads) {
      int r = idx / (kHeadDim / 8), c = idx % (kHeadDim / 8);
      float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
      if (r < p.R) {
        uint4 raw = *reinterpret_cast<const uint4*>(p.q + out_row_offset(p, sg.b, sg.h, r) + c * 8);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
        float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
        lo = make_float4(f0.x, f0.y, f1.x, f1.y);
        hi = make_float4(f2.x, f2.y, f3.x, f3.y);
      }
      float4* dst = reinterpret_cast<float4*>(s.q + r * kHeadDim + c * 8);
      dst[0] = lo;
      dst[1] = hi;
    }

    float m_run[RPT], l_run[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) { m_run[k] = -INFINITY; l_run[k] = 0.f; }
    float acc[PROWS][4];
#pragma unroll
    for (int k = 0; k < PROWS; ++k) acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.f;

    const int ntiles = (sg.j1 - sg.j0 + kTile - 1) / kTile;
    load_tile(p, s, sg, sg.j0, 0);
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t & 1;
      const int jt = sg.j0 + t * kTile;
      if (t + 1 < ntiles) {
        load_tile(p, s, sg, jt + kTile, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();

      // ---- scores for rows rg*RPT.. and keys tl, tl+16 of the tile
      float sc[RPT][2];
#pragma unroll
      for (int k = 0; k < RPT; ++k) sc[k][0] = sc[k][1] = 0.f;
      const __nv_bfloat16* k0 = s.k[buf] + tl * kKStride;
      const __nv_bfloat16* k1 = s.k[buf] + (tl + 16) * kKStride;
#pragma unroll 4
      for (int d = 0; d < kHeadDim; d += 8) {
        uint4 ra = *reinterpret_cast<const uint4*>(k0 + d);
        uint4 rb = *reinterpret_cast<const uint4*>(k1 + d);
        const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&ra);
        const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&rb);
        float ka[8], kb[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 fa = __bfloat1622float2(ha[e]), fb = __bfloat1622float2(hb[e]);
          ka[2 * e] = fa.x; ka[2 * e + 1] = fa.y;
          kb[2 * e] = fb.x; kb[2 * e + 1] = fb.y;
        }
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
          const float4* qr = reinterpret_cast<const float4*>(s.q + (rg * RPT + k) * kHeadDim + d);
          float4 q0 = qr[0], q1 = qr[1];
          float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            sc[k][0] = fmaf(qv[e], ka[e], sc[k][0]);
            sc[k][1] = fmaf(qv[e], kb[e], sc[k][1]);
          }
        }
      }

      // ---- mask, online softmax (log2 domain), probabilities to smem
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int r = rg * RPT + k;
        const int lim = (r < p.R) ? row_limit(p, sg.n, sg.w, r) : 0;
        const int lim_seg = lim < sg.j1 ? lim : sg.j1;
        float x0 = (jt + tl < lim_seg) ? sc[k][0] * p.scale_log2 : -INFINITY;
        float x1 = (jt + tl + 16 < lim_seg) ? sc[k][1] * p.scale_log2 : -INFINITY;
        float mx = fmaxf(x0, x1);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m_run[k], mx);
        float alpha, p0, p1;
        if (m_new == -INFINITY) {
          alpha = 1.f; p0 = 0.f; p1 = 0.f;
        } else {
          alpha = fast_exp2(m_run[k] - m_new);
          p0 = fast_exp2(x0 - m_new);
          p1 = fast_exp2(x1 - m_new);
        }
        m_run[k] = m_new;
        l_run[k] = l_run[k] * alpha + p0 + p1;
        s.pr[r * kTile + tl] = p0;
        s.pr[r * kTile + tl + 16] = p1;
        if (tl == 0) s.alpha[r] = alpha;
      }
      __syncthreads();

      // ---- PV: acc[row][d0..d0+3] = alpha * acc + sum_j p[row][j] * v[j][d0..]
      const int nvalid = (sg.j1 - jt) < kTile ? (sg.j1 - jt) : kTile;
#pragma unroll
      for (int k = 0; k < PROWS; ++k) {
        const float a = s.alpha[wid + 8 * k];
        acc[k][0] *= a; acc[k][1] *= a; acc[k][2] *= a; acc[k][3] *= a;
      }
      const __nv_bfloat16* vb = s.v[buf] + d0;
      for (int j = 0; j < nvalid; j += 4) {
        float vv[4][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint2 raw = *reinterpret_cast<const uint2*>(vb + (j + e) * kHeadDim);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
          float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
          vv[e][0] = f0.x; vv[e][1] = f0.y; vv[e][2] = f1.x; vv[e][3] = f1.y;
        }
#pragma unroll
        for (int k = 0; k < PROWS; ++k) {
          float4 pp = *reinterpret_cast<const float4*>(s.pr + (wid + 8 * k) * kTile + j);
          float pj[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[k][c] = fmaf(pj[e], vv[e][c], acc[k][c]);
          }
        }
      }
      __syncthreads();
    }

    // ---- finish: reduce l over the half-warp, publish m and l per row
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      float lsum = l_run[k];
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
      if (tl == 0) {
        s.m[rg * RPT + k] = m_run[k];
        s.l[rg * RPT + k] = lsum;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < PROWS; ++k) {
      const int r = wid + 8 * k;
      if (r >= p.R) continue;
      if (sg.whole) {
        // Padding rows of a shorter window (no visible key, l = 0) are written as zeros.
        const float inv = (r / p.G < sg.w) ? 1.f / s.l[r] : 0.f;
        __nv_bfloat162 o01 = __floats2bfloat162_rn(acc[k][0] * inv, acc[k][1] * inv);
        __nv_bfloat162 o23 = __floats2bfloat162_rn(acc[k][2] * inv, acc[k][3] * inv);
        uint2 packed;
        packed.x = *reinterpret_cast<uint32_t*>(&o01);
        packed.y = *reinterpret_cast<uint32_t*>(&o23);
        *reinterpret_cast<uint2*>(p.out + out_row_offset(p, sg.b, sg.h, r) + d0) = packed;
      } else {
        float* slot = slot_ptr(p, sg.slot);
        if (lane == 0) {
          slot[r] = s.m[r];
          slot[p.rows_pad + r] = s.l[r];
        }
        *reinterpret_cast<float4*>(slot + 2 * p.rows_pad + (size_t)r * kHeadDim + d0) =
            make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
      }
    }
    __syncthreads();
  }
}

template <int RPT>
cudaError_t launch_rpt(const Problem& p, cudaStream_t stream) {
  size_t smem = simt_layout(RPT, p.B, nullptr, nullptr);
  cudaError_t e = cudaFuncSetAttribute(pbd_attn_simt_kernel<RPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(pbd_attn_simt_kernel<RPT>, dim3(p.num_ctas), dim3(kThreads), smem, stream, p);
}

template <int RPT>
cudaError_t occupancy_rpt(int B, int* ctas) {
  size_t smem = simt_layout(RPT, B, nullptr, nullptr);
  cudaError_t e = cudaFuncSetAttribute(pbd_attn_simt_kernel<RPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, pbd_attn_simt_kernel<RPT>, kThreads,
                                                       smem);
}

}  // namespace

int simt_rows_per_thread(int R) { return (R + 15) / 16; }
int simt_tile_keys() { return kTile; }

size_t simt_smem_bytes(int R, int B) {
  return simt_layout(simt_rows_per_thread(R), B, nullptr, nullptr);
}

cudaError_t simt_max_ctas_per_sm(int R, int B, int* ctas) {
  switch (simt_rows_per_thread(R)) {
    case 1: return occupancy_rpt<1>(B, ctas);
    case 2: return occupancy_rpt<2>(B, ctas);
    case 3: return occupancy_rpt<3>(B, ctas);
    case 4: return occupancy_rpt<4>(B, ctas);
    case 5: return occupancy_rpt<5>(B, ctas);
    case 6: return occupancy_rpt<6>(B, ctas);
    case 7: return occupancy_rpt<7>(B, ctas);
    case 8: return occupancy_rpt<8>(B, ctas);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_simt(const Problem& p, cudaStream_t stream) {
  switch (simt_rows_per_thread(p.R)) {
    case 1: return launch_rpt<1>(p, stream);
    case 2: return launch_rpt<2>(p, stream);
    case 3: return launch_rpt<3>(p, stream);
    case 4: return launch_rpt<4>(p, stream);
    case 5: return launch_rpt<5>(p, stream);
    case 6: return launch_rpt<6>(p, stream);
    case 7: return launch_rpt<7>(p, stream);
    case 8: return launch_rpt<8>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace la
