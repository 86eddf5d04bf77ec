// topk.cuh -- index rows -> additive bias.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "tile.cuh"

namespace gqa {

// ============================================================================
// index rows -> additive bias (metrale glm5next_dsa_ref, topk_to_mask)
// ============================================================================

// One CTA per sequence b: rows offsets[b]..offsets[b+1]-1 of `bias` become -inf,
// then 0 at every in-range position named by idx[b, 0..width) (relative to the
// sequence; -1 is the INVALID sentinel, repeats collapse, out-of-range entries
// are dropped). Rows outside every sequence are not touched. Malformed offsets
// leave the sequence alone and flag kErrBadOffsets.
__global__ void __launch_bounds__(256) gqa_topk_to_bias_kernel(const int32_t* idx, int32_t width,
                                                               const int32_t* offsets, int32_t max_len,
                                                               float* bias, uint32_t* err) {
  const int b = blockIdx.x;
  const int o0 = offsets[b], o1 = offsets[b + 1];
  if (!(0 <= o0 && o0 <= o1 && o1 <= max_len)) {
    if (threadIdx.x == 0 && err) atomicOr(err, kErrBadOffsets);
    return;
  }
  for (int r = o0 + threadIdx.x; r < o1; r += blockDim.x) bias[r] = -INFINITY;
  __syncthreads();
  const int n = o1 - o0;
  for (int w = threadIdx.x; w < width; w += blockDim.x) {
    const int t = idx[static_cast<size_t>(b) * width + w];
    if (t >= 0 && t < n) bias[o0 + t] = 0.f;
  }
}

}  // namespace gqa
