// merge.cuh -- the standalone merge / finalize kernel for caller-held states.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "tile.cuh"

namespace gqa {

// ============================================================================
// merge / finalize
// ============================================================================

struct MergeArgs {
  const float* m;            // state (r, i) at r * row_stride + i * state_stride
  const float* l;
  const float* acc;          // ... times D
  int32_t rows, S;
  int64_t row_stride;        // S for [rows, S] (split-major), 1 for [S, rows] (gathered)
  int64_t state_stride;      // 1 for [rows, S], rows for [S, rows]
  const float* cm;           // carry [rows] / [rows, D], or null
  const float* cl;
  const float* cacc;
  float* om;                 // merged state out, or null (may alias the carry)
  float* ol;
  float* oacc;
  void* out;                 // [rows, D] or null
  int32_t out_bf16;
};

template <int D>
__global__ void __launch_bounds__(128) gqa_merge_kernel(const MergeArgs a) {
  constexpr int W = 4, E = D / 32;
  __shared__ float red[W];
  __shared__ float accs[W][D];
  __shared__ float lsum[W];
  const int r = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nS = a.S;
  const size_t base = static_cast<size_t>(r) * a.row_stride;
  const size_t ss = static_cast<size_t>(a.state_stride);
  // pass 1: the largest maximum among non-empty states (and the carry)
  float M = -INFINITY;
  for (int i = threadIdx.x; i < nS; i += blockDim.x)
    if (a.l[base + i * ss] != 0.f) M = fmaxf(M, a.m[base + i * ss]);
  for (int x = 16; x >= 1; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const bool has_carry = a.cl != nullptr && a.cl[r] != 0.f;
  float cmr = 0.f, clr = 0.f;
  if (has_carry) {
    cmr = a.cm[r];
    clr = a.cl[r];
    M = fmaxf(M, cmr);
  }
  // pass 2: rescaled sums; warp w takes states w, w+4, ...; lanes split D
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float L = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int i = warp; i < nS; i += W) {
      const float li = a.l[base + i * ss];
      if (li == 0.f) continue;
      const float w = expf(a.m[base + i * ss] - M);
      L += li * w;
      const float* src = a.acc + (base + i * ss) * D + lane * E;
      if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(v.x, w, acc[0]);
        acc[1] = fmaf(v.y, w, acc[1]);
        acc[2] = fmaf(v.z, w, acc[2]);
        acc[3] = fmaf(v.w, w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(v.x, w, acc[0]);
        acc[1] = fmaf(v.y, w, acc[1]);
      }
    }
    if (has_carry && warp == 0) {
      const float w = expf(cmr - M);
      L += clr * w;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(a.cacc[static_cast<size_t>(r) * D + lane * E + e], w, acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) accs[warp][lane * E + e] = acc[e];
  if (lane == 0) lsum[warp] = L;
  __syncthreads();
  const float Lt = (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const float A = (accs[0][d] + accs[1][d]) + (accs[2][d] + accs[3][d]);
    if (a.oacc) a.oacc[static_cast<size_t>(r) * D + d] = A;
    if (a.out) {
      const float y = (Lt == 0.f) ? 0.f : __fdiv_rn(A, Lt);
      if (a.out_bf16)
        static_cast<__nv_bfloat16*>(a.out)[static_cast<size_t>(r) * D + d] = __float2bfloat16_rn(y);
      else
        static_cast<float*>(a.out)[static_cast<size_t>(r) * D + d] = y;
    }
  }
  if (threadIdx.x == 0 && a.om) {
    a.om[r] = (Lt == 0.f) ? -INFINITY : M;
    a.ol[r] = Lt;
  }
}

}  // namespace gqa
