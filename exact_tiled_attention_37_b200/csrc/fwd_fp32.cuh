// Forward attention for fp32 storage (head dimension 64) on the CUDA cores.
//
// The tensor cores have no fp32 product: tf32 keeps 10 mantissa bits, which
// puts the logsumexp of N(0,1) inputs about 1.5e-3 away from the exact value,
// above the 1e-3 bar.  This kernel keeps the same tiled online-softmax
// algorithm as the tensor-core kernels (K/V tiles staged in shared memory,
// running row maximum and sum, one division at the end) with fp32 FMAs.
//
// CTA: 4 warps, 32 query rows (8 per warp), 64-key tiles.  Lane l of a warp
// computes the scores of keys l and l + 32 for the warp's 8 rows and owns
// output columns l and l + 32 of those rows.
#pragma once

#include "fwd.cuh"

namespace eta {

constexpr int kF32Rows = 32;   // query rows per CTA
constexpr int kF32Keys = 64;   // keys per tile
constexpr int kF32D = 64;

__global__ void __launch_bounds__(128) fwd_fp32_kernel(const float* __restrict__ q,
                                                       const float* __restrict__ k,
                                                       const float* __restrict__ v,
                                                       long long qsb, long long qsh, long long qsn,
                                                       long long ksb, long long ksh, long long ksn,
                                                       long long vsb, long long vsh, long long vsn,
                                                       const FwdParams p) {
  __shared__ float sq[kF32Rows][kF32D];
  __shared__ float sk[kF32D][kF32Keys];  // transposed: lanes read consecutive keys
  __shared__ float sv[kF32Keys][kF32D];
  __shared__ float sp[4][8][kF32Keys];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const int q0 = blockIdx.x * kF32Rows;
  const float* qb = q + b * qsb + h * qsh;
  const float* kb = k + b * ksb + hk * ksh;
  const float* vb = v + b * vsb + hk * vsh;

  for (int e = threadIdx.x; e < kF32Rows * kF32D; e += blockDim.x) {
    const int r = e / kF32D, d = e % kF32D;
    sq[r][d] = (q0 + r < p.N) ? qb[(q0 + r) * qsn + d] : 0.f;
  }

  float m[8], l[8], o0[8], o1[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
    o0[r] = 0.f;
    o1[r] = 0.f;
  }
  const int row0 = warp * 8;
  const int2 kr = window_keys(q0, min(p.N, q0 + kF32Rows), p.N, p.wl, p.wr);
  for (int kt = (kr.x / kF32Keys) * kF32Keys; kt < kr.y; kt += kF32Keys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kF32Keys * kF32D; e += blockDim.x) {
      const int r = e / kF32D, d = e % kF32D;
      const bool in = kt + r < p.N;
      sk[d][r] = in ? kb[(kt + r) * ksn + d] : 0.f;
      sv[r][d] = in ? vb[(kt + r) * vsn + d] : 0.f;
    }
    __syncthreads();
    float s0[8], s1[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) s0[r] = s1[r] = 0.f;
#pragma unroll 8
    for (int d = 0; d < kF32D; ++d) {
      const float k0v = sk[d][lane], k1v = sk[d][lane + 32];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float qv = sq[row0 + r][d];
        s0[r] = fmaf(qv, k0v, s0[r]);
        s1[r] = fmaf(qv, k1v, s1[r]);
      }
    }
    const int key0 = kt + lane, key1 = kt + lane + 32;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int qrow = q0 + row0 + r;
      float a = s0[r] * p.scale, c = s1[r] * p.scale;
      const int2 cw = col_window(0, qrow, p.N, p.wl, p.wr);  // visible keys [cw.x, cw.y)
      if (key0 < cw.x || key0 >= cw.y) a = -INFINITY;
      if (key1 < cw.x || key1 >= cw.y) c = -INFINITY;
      float mx = fmaxf(a, c);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[r], mx);
      const float ref = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m[r] == -INFINITY) ? 0.f : expf(m[r] - ref);
      const float pa = expf(a - ref), pc = expf(c - ref);
      float sum = pa + pc;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[r] = l[r] * alpha + sum;
      o0[r] *= alpha;
      o1[r] *= alpha;
      m[r] = m_new;
      sp[warp][r][lane] = pa;
      sp[warp][r][lane + 32] = pc;
    }
    __syncwarp();
#pragma unroll 4
    for (int key = 0; key < kF32Keys; ++key) {
      const float v0 = sv[key][lane], v1 = sv[key][lane + 32];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float pr = sp[warp][r][key];
        o0[r] = fmaf(pr, v0, o0[r]);
        o1[r] = fmaf(pr, v1, o1[r]);
      }
    }
    __syncwarp();
  }
  float* ob = static_cast<float*>(p.o) + b * p.osb + h * p.osh;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int qrow = q0 + row0 + r;
    if (qrow < p.N) {
      const float inv = 1.f / l[r];
      ob[qrow * p.osn + lane] = o0[r] * inv;
      ob[qrow * p.osn + lane + 32] = o1[r] * inv;
      if (lane == 0) p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] = m[r] + logf(l[r]);
    }
  }
}

}  // namespace eta
