// partition_f32.cuh -- the fp32 CUDA-core partition kernel.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "tile.cuh"

namespace gqa {

// ============================================================================
// fp32 K/V: CUDA-core partition kernel
// ============================================================================

template <int D, int HMAX>
struct F32Cfg {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kE = D / 32;  // elements per lane
  static constexpr int kSmemBytes = (kWarps + 1) * HMAX * (D + 4 + 2) * 4;
  static constexpr int kWeightCap = kSmemBytes / 4 / 2;
};

template <int D, int HMAX>
__global__ void __launch_bounds__(F32Cfg<D, HMAX>::kThreads)
gqa_partition_f32_kernel(const PartitionArgs a) {
  using C = F32Cfg<D, HMAX>;
  constexpr int E = C::kE, W = C::kWarps, HP = HMAX, P = D + 4;
  extern __shared__ float fsm[];
  __shared__ float smM[16], smL[16], smC[16], smN[16];
  __shared__ int smFlag;
  const Tile t = tile_of(a, blockIdx.x);
  ptx::grid_dependency_wait();
  if (t.kbeg >= t.kend) {
    if (a.write_empty) write_empty_states<D>(a, t);
    if (a.merge && t.n == 0 && t.c == 0)
      merge_segment<D, HMAX>(a, t, 0, threadIdx.x, smM, smL, smC, fsm, C::kWeightCap, BlockSync{});
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* qg = static_cast<const float*>(a.q) +
                    (static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * a.hpk) * D;
  float qv[HMAX][E];
#pragma unroll
  for (int h = 0; h < HMAX; ++h)
#pragma unroll
    for (int e = 0; e < E; ++e) qv[h][e] = (h < a.hpk) ? __ldg(qg + h * D + lane * E + e) : 0.f;
  float m[HMAX], l[HMAX], o[HMAX][E];
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[h][e] = 0.f;
  }
  const float* kg = static_cast<const float*>(a.k);
  const float* vg = static_cast<const float*>(a.v);
  const size_t rs = static_cast<size_t>(a.G) * D;
  if (t.append) {
    write_appended_row(a, t, D, threadIdx.x, C::kThreads);
    for (int h = warp; h < a.hpk; h += W) {
      const float s2 = appended_logit2<D, float>(a, t, h, lane);
      if (lane == 0) smN[h] = s2;
    }
    __syncthreads();   // smN is read by other warps in the epilogue (a warp may have no keys)
  }
  // U keys per warp step (32 floats of K and of V per lane: 16 keys at d 64,
  // 8 at d 128): their loads are issued together, their per-head dot products
  // reduced together (U-way interleaved butterflies), and the running state
  // rescaled once per step.
  constexpr int U = 32 / E;
#pragma unroll 1
  for (int key0 = t.kbeg + warp; key0 < t.kstream; key0 += W * U) {
    float kv[U][E], vv[U][E];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int key = key0 + u * W;
      const bool live = key < t.kstream;
      const size_t base = (static_cast<size_t>(t.o0) + (live ? key : t.kbeg)) * rs +
                          static_cast<size_t>(t.g) * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        kv[u][e] = live ? __ldg(kg + base + e) : 0.f;
        vv[u][e] = live ? __ldg(vg + base + e) : 0.f;
      }
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= a.hpk) break;
      float sc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) d = fmaf(qv[h][e], kv[u][e], d);
        sc[u] = d;
      }
#pragma unroll
      for (int x = 16; x >= 1; x >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], x);
      float mx = m[h];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int key = key0 + u * W;
        sc[u] = (key < t.kstream) ? fmaf(sc[u], a.scale_log2, bias2(a, t, key)) : -INFINITY;
        mx = fmaxf(mx, sc[u]);
      }
      // every logit so far may be -inf (a masking bias): keep exp2 away from -inf - -inf
      const float mu = (mx == -INFINITY) ? 0.f : mx;
      const float al = exp2f(m[h] - mu);
      float lsum = l[h] * al;
#pragma unroll
      for (int e = 0; e < E; ++e) o[h][e] *= al;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float p = exp2f(sc[u] - mu);
        lsum += p;
#pragma unroll
        for (int e = 0; e < E; ++e) o[h][e] = fmaf(p, vv[u][e], o[h][e]);
      }
      l[h] = lsum;
      m[h] = mx;
    }
  }
  if (threadIdx.x == 0) ptx::grid_launch_dependents();   // cache stream done (see the bf16 kernel)
  // slots: W warps, plus the appended key when this tile owns it
  float* ms = fsm;
  float* ls = ms + (W + 1) * HP;
  float* accs = ls + (W + 1) * HP;
  const int nslots = W + (t.append ? 1 : 0);
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      ms[warp * HP + h] = m[h];
      ls[warp * HP + h] = l[h];
    }
  }
  if (t.append)
    for (int h = threadIdx.x; h < HP; h += C::kThreads) {
      ms[W * HP + h] = h < a.hpk ? smN[h] : -INFINITY;
      ls[W * HP + h] = h < a.hpk ? 1.f : 0.f;
    }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    if (h >= a.hpk) break;
    float M = -INFINITY;
    for (int w = 0; w < nslots; ++w) M = fmaxf(M, ms[w * HP + h]);
    const float f = exp2f(m[h] - ((M == -INFINITY) ? 0.f : M));
#pragma unroll
    for (int e = 0; e < E; ++e) accs[(warp * HP + h) * P + lane * E + e] = o[h][e] * f;
  }
  if (t.append)
    for (int i = threadIdx.x; i < a.hpk * D; i += C::kThreads) {
      const int h = i / D, d = i % D;
      float M = -INFINITY;
      for (int w = 0; w < nslots; ++w) M = fmaxf(M, ms[w * HP + h]);
      const float vn = static_cast<const float*>(a.v_new)[(static_cast<size_t>(t.b) * a.G + t.g) * D + d];
      accs[(W * HP + h) * P + d] = vn * exp2f(ms[W * HP + h] - (M == -INFINITY ? 0.f : M));
    }
  __syncthreads();
  store_partial<D, W, HP>(a, t, ms, ls, accs, threadIdx.x, C::kThreads, nslots);
  if (a.merge) {
    __syncthreads();                         // store_partial done with the scratch
    finish_segment<D, HMAX>(a, t, threadIdx.x, smM, smL, smC, &smFlag, fsm, C::kWeightCap, 0u,
                            BlockSync{});
  }
}

}  // namespace gqa
