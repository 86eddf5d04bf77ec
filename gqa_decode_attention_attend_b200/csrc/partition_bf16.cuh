// partition_bf16.cuh -- the bf16 TMA-staged tensor-core partition kernel.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "tile.cuh"

namespace gqa {

// ============================================================================
// bf16 K/V: TMA-staged, tensor-core partition kernel
// ============================================================================

template <int D, int NT>
struct TcCfg {
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kKeysPerWarp = 16;
  static constexpr int kStageKeys = kKeysPerWarp * kConsumerWarps;  // 64 rows per stage
  static constexpr int kHalves = D / 64;                            // 128-byte column blocks
  static constexpr int kHalfTileBytes = kStageKeys * 128;
  static constexpr int kStageBytes = 2 * kHalves * kHalfTileBytes;  // K and V
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kHP = 8 * NT;                                // padded heads
  static constexpr int kScratchBytes = (kConsumerWarps + 1) * kHP * (D + 4 + 2) * 4;
  static constexpr int kDataBytes = kRingBytes > kScratchBytes ? kRingBytes : kScratchBytes;
  static constexpr int kBarOffset = kDataBytes;                     // 2*kStages + 1 mbarriers
  static constexpr int kAbortOffset = kBarOffset + (2 * kStages + 1 + 1) * 8;
  static constexpr int kFlagOffset = kAbortOffset + 4;
  static constexpr int kMergeOffset = kAbortOffset + 16;            // 4 x 16 floats
  static constexpr int kSmemBytes = 1024 + kMergeOffset + 4 * 16 * 4;   // + alignment slack
  // The merge's split weights reuse the ring (idle once the tile is consumed).
  static constexpr int kWeightCap = kRingBytes / 4 / 2;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(kScratchBytes <= kRingBytes, "epilogue scratch reuses the ring");
};

// Address of 16-byte chunk `chunk` (0..7) of row `r` of a 128B-swizzled half tile.
__device__ __forceinline__ uint32_t swz(uint32_t tile, int r, int chunk) {
  return tile + r * 128 + ((chunk ^ (r & 7)) << 4);
}

template <int D, int NT>
__global__ void __launch_bounds__(TcCfg<D, NT>::kThreads)
gqa_partition_bf16_kernel(const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const PartitionArgs a) {
  using C = TcCfg<D, NT>;
  extern __shared__ uint8_t smem_raw[];
  // aligned by an offset from the array itself (the compiler keeps accesses
  // through it in the shared state space)
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t ring = ptx::smem_u32(smem);
  const uint32_t bar_full = ring + C::kBarOffset;
  const uint32_t bar_empty = bar_full + C::kStages * 8;
  const uint32_t bar_merge = bar_empty + C::kStages * 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbortOffset);

  float* smM = reinterpret_cast<float*>(smem + C::kMergeOffset);
  float* smL = smM + 16;
  float* smC = smM + 32;
  float* smN = smM + 48;                         // appended key's base-2 logit per head
  int* smFlag = reinterpret_cast<int*>(smem + C::kFlagOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const Tile t = tile_of(a, blockIdx.x);
  if (t.kbeg >= t.kend) {
    ptx::grid_dependency_wait();
    if (a.write_empty) write_empty_states<D>(a, t);
    // A sequence without keys: split 0 still writes its rows (carry or zeros).
    if (a.merge && t.n == 0 && t.c == 0 && warp < C::kConsumerWarps)
      merge_segment<D, C::kHP>(a, t, 0, threadIdx.x, smM, smL, smC, reinterpret_cast<float*>(smem),
                               C::kWeightCap, NamedSync128{});
    return;
  }
  const int nst = (t.kstream - t.kbeg + C::kStageKeys - 1) / C::kStageKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(bar_full + 8 * s, 1);
      ptx::mbar_init(bar_empty + 8 * s, C::kConsumerWarps);
    }
    ptx::mbar_init(bar_merge, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer warp
  if (warp == C::kConsumerWarps) {
    if (lane == 0) {
      ptx::prefetch_tensormap(&tm_k);
      ptx::prefetch_tensormap(&tm_v);
      const uint64_t pol = ptx::l2_policy_evict_first();
      int issued = 0;
      for (int it = 0; it < nst; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (it >= C::kStages &&
            !ptx::mbar_wait_bounded(bar_empty + 8 * s, ph ^ 1, abort_flag, kWaitLimitNs)) {
          atomicOr(a.err, kErrTimeout);
          *abort_flag = 1;
          break;
        }
        const uint32_t full = bar_full + 8 * s;
        ptx::mbar_arrive_expect_tx(full, C::kStageBytes);
        const int row = t.o0 + t.kbeg + it * C::kStageKeys;
        const uint32_t st = ring + s * C::kStageBytes;
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
          ptx::tma_load_2d(st + h * C::kHalfTileBytes, &tm_k, t.g * D + h * 64, row, full, pol);
          ptx::tma_load_2d(st + (C::kHalves + h) * C::kHalfTileBytes, &tm_v, t.g * D + h * 64, row,
                           full, pol);
        }
        ++issued;
      }
      // Every load of the tile is issued (its last stages are in flight): the
      // next kernel on the stream may now be scheduled. It still waits for this
      // grid before reading what it writes, so its first cache loads overlap
      // this grid's last stages, epilogue and merges.
      if (a.trigger_at_last_load) ptx::grid_launch_dependents();
      if (*abort_flag) {
        // Drain the copies still in flight before the CTA's shared memory goes away.
        for (int it = max(0, issued - C::kStages); it < issued; ++it)
          ptx::mbar_wait_bounded(bar_full + 8 * (it % C::kStages), (it / C::kStages) & 1,
                                 nullptr, kWaitLimitNs);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  // Everything the previous kernel on the stream may have written (q, carry,
  // bias, the appended K/V, the workspace) is read only after this wait; the
  // producer's cache loads above may run ahead of it (early-start launches).
  ptx::grid_dependency_wait();
  // Q^T as the B operand of S^T = K Q^T: b0 = q[head][k0 + 2*(lane%4) + {0,1}],
  // b1 = the same 8 columns further, head = nt*8 + lane/4 (zero past hpk).
  uint32_t qf[D / 16][NT][2];
  {
    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) +
                              (static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * a.hpk) * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int head = nt * 8 + (lane >> 2);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int d0 = kk * 16 + (lane & 3) * 2;
        if (head < a.hpk) {
          qf[kk][nt][0] = __ldg(reinterpret_cast<const unsigned int*>(qg + head * D + d0));
          qf[kk][nt][1] = __ldg(reinterpret_cast<const unsigned int*>(qg + head * D + d0 + 8));
        } else {
          qf[kk][nt][0] = qf[kk][nt][1] = 0u;
        }
      }
    }
  }

  float o[D / 16][NT][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[mt][nt][j] = 0.f;
  float mrun[NT][2], lrun[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mrun[nt][0] = mrun[nt][1] = -INFINITY;
    lrun[nt][0] = lrun[nt][1] = 0.f;
  }
  const float sl2 = a.scale_log2;
  bool aborted = false;
  if (t.append) {
    write_appended_row(a, t, D, threadIdx.x, 32 * C::kConsumerWarps);
    for (int h = warp; h < a.hpk; h += C::kConsumerWarps) {
      const float s2 = appended_logit2<D, __nv_bfloat16>(a, t, h, lane);
      if (lane == 0) smN[h] = s2;
    }
  }

#pragma unroll 1
  for (int it = 0; it < nst; ++it) {
    const int s = it % C::kStages;
    const uint32_t ph = (it / C::kStages) & 1;
    if (!aborted && !ptx::mbar_wait_bounded(bar_full + 8 * s, ph, abort_flag, kWaitLimitNs)) {
      if (lane == 0) atomicOr(a.err, kErrTimeout);
      *abort_flag = 1;
      aborted = true;
    }
    if (aborted) break;
    const int key0 = t.kbeg + it * C::kStageKeys + warp * C::kKeysPerWarp;
    const int nvalid = min(C::kKeysPerWarp, t.kstream - key0);
    const uint32_t kt = ring + s * C::kStageBytes;
    const uint32_t vt = kt + C::kHalves * C::kHalfTileBytes;
    const int wrow = warp * C::kKeysPerWarp;

    if (nvalid > 0) {
      if (nvalid < C::kKeysPerWarp) {
        // Rows past the sequence end hold another sequence's (or no) data; zero
        // their V so that 0-weight * garbage cannot become NaN in the MMA.
        uint8_t* vtile = smem + s * C::kStageBytes + C::kHalves * C::kHalfTileBytes;
        const int nz = (C::kKeysPerWarp - nvalid) * C::kHalves * 8;
        for (int i = lane; i < nz; i += 32) {
          const int r = wrow + nvalid + i / (C::kHalves * 8);
          const int rem = i % (C::kHalves * 8);
          *reinterpret_cast<uint4*>(vtile + (rem >> 3) * C::kHalfTileBytes + r * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }

      // S^T[16 keys x 8*NT heads] = K[16 x D] . Q^T[D x 8*NT]
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
      {
        const int r = wrow + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int dcol = kk * 16 + (lane >> 4) * 8;
          uint32_t af[4];
          ptx::ldmatrix_x4(af, swz(kt + (dcol >> 6) * C::kHalfTileBytes, r, (dcol & 63) >> 3));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) ptx::mma_bf16_16816(sacc[nt], af, qf[kk][nt][0], qf[kk][nt][1]);
        }
      }

      // Online softmax update (base 2). Fragment: sacc[nt][e] is key lane/4,
      // sacc[nt][e+2] key lane/4+8, both for head column nt*8 + 2*(lane%4) + e.
      const int kr = lane >> 2;
      const float b0 = (kr < nvalid) ? bias2(a, t, key0 + kr) : 0.f;
      const float b1 = (kr + 8 < nvalid) ? bias2(a, t, key0 + kr + 8) : 0.f;
      uint32_t ph_hi[NT][2], ph_lo[NT][2];
      float alpha[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float p[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float s0 = (kr < nvalid) ? fmaf(sacc[nt][e], sl2, b0) : -INFINITY;
          const float s1 = (kr + 8 < nvalid) ? fmaf(sacc[nt][e + 2], sl2, b1) : -INFINITY;
          float mx = fmaxf(s0, s1);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float mnew = fmaxf(mrun[nt][e], mx);
          const float mu = (mnew == -INFINITY) ? 0.f : mnew;
          alpha[nt][e] = exp2f(mrun[nt][e] - mu);
          mrun[nt][e] = mnew;
          p[e] = exp2f(s0 - mu);
          p[e + 2] = exp2f(s1 - mu);
          lrun[nt][e] = lrun[nt][e] * alpha[nt][e] + (p[e] + p[e + 2]);
        }
        // P^T as the B operand of O^T += V^T P^T: split p = hi + lo, both bf16,
        // so the product keeps ~16 significant bits of each weight.
        const uint32_t h01 = ptx::pack_bf16x2(p[0], p[1]);
        const uint32_t h23 = ptx::pack_bf16x2(p[2], p[3]);
        const uint32_t l01 = ptx::pack_bf16x2(p[0] - ptx::bf16lo_to_f32(h01), p[1] - ptx::bf16hi_to_f32(h01));
        const uint32_t l23 = ptx::pack_bf16x2(p[2] - ptx::bf16lo_to_f32(h23), p[3] - ptx::bf16hi_to_f32(h23));
        ph_hi[nt][0] = ptx::movmatrix_trans(h01);
        ph_hi[nt][1] = ptx::movmatrix_trans(h23);
        ph_lo[nt][0] = ptx::movmatrix_trans(l01);
        ph_lo[nt][1] = ptx::movmatrix_trans(l23);
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][0] *= alpha[nt][0];
          o[mt][nt][1] *= alpha[nt][1];
          o[mt][nt][2] *= alpha[nt][0];
          o[mt][nt][3] *= alpha[nt][1];
        }

      // O^T[D x 8*NT] += V^T[D x 16 keys] . P^T[16 keys x 8*NT]
      {
        const int j = lane >> 3;
        const int r = wrow + (lane & 7) + (j >> 1) * 8;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int dcol = mt * 16 + (j & 1) * 8;
          uint32_t af[4];
          ptx::ldmatrix_x4_trans(af, swz(vt + (dcol >> 6) * C::kHalfTileBytes, r, (dcol & 63) >> 3));
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            ptx::mma_bf16_16816(o[mt][nt], af, ph_hi[nt][0], ph_hi[nt][1]);
            ptx::mma_bf16_16816(o[mt][nt], af, ph_lo[nt][0], ph_lo[nt][1]);
          }
        }
      }
      if (nvalid < C::kKeysPerWarp) ptx::fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * s);
  }

  // ------------------------------------------------------------ epilogue
  // Otherwise the next kernel may be scheduled once the tile's cache stream is
  // done, overlapping this grid's epilogue and merges.
  if (!a.trigger_at_last_load && threadIdx.x == 0) ptx::grid_launch_dependents();
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = lrun[nt][e];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      lrun[nt][e] = l;
    }
  constexpr int W = C::kConsumerWarps, HP = C::kHP, P = D + 4;
  const int ctid = threadIdx.x;                   // 0 .. 32*W-1
  ptx::named_barrier_sync(1, 32 * W);             // ring no longer read by anyone
  // slots: W warps, plus the appended key when this tile owns it
  float* ms = reinterpret_cast<float*>(smem);
  float* ls = ms + (W + 1) * HP;
  float* accs = ls + (W + 1) * HP;
  const int nslots = W + (t.append ? 1 : 0);
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        ms[warp * HP + nt * 8 + lane * 2 + e] = mrun[nt][e];
        ls[warp * HP + nt * 8 + lane * 2 + e] = lrun[nt][e];
      }
  }
  if (t.append)   // the appended key as one more slot: m = its logit, l = 1
    for (int h = ctid; h < HP; h += 32 * W) {
      ms[W * HP + h] = h < a.hpk ? smN[h] : -INFINITY;
      ls[W * HP + h] = h < a.hpk ? 1.f : 0.f;
    }
  ptx::named_barrier_sync(1, 32 * W);
  float f[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hc = nt * 8 + (lane & 3) * 2 + e;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W + 1; ++w)
        if (w < nslots) M = fmaxf(M, ms[w * HP + hc]);
      const float Mu = (M == -INFINITY) ? 0.f : M;
      f[nt][e] = exp2f(mrun[nt][e] - Mu);
    }
  if (t.append)
    for (int i = ctid; i < a.hpk * D; i += 32 * W) {
      const int h = i / D, d = i % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W + 1; ++w) M = fmaxf(M, ms[w * HP + h]);
      const float vn = __bfloat162float(static_cast<const __nv_bfloat16*>(a.v_new)[(static_cast<size_t>(t.b) * a.G + t.g) * D + d]);
      accs[(W * HP + h) * P + d] = vn * exp2f(ms[W * HP + h] - (M == -INFINITY ? 0.f : M));
    }
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int d = mt * 16 + (lane >> 2);
      const int hc = nt * 8 + (lane & 3) * 2;
      accs[(warp * HP + hc) * P + d] = o[mt][nt][0] * f[nt][0];
      accs[(warp * HP + hc + 1) * P + d] = o[mt][nt][1] * f[nt][1];
      accs[(warp * HP + hc) * P + d + 8] = o[mt][nt][2] * f[nt][0];
      accs[(warp * HP + hc + 1) * P + d + 8] = o[mt][nt][3] * f[nt][1];
    }
  ptx::named_barrier_sync(1, 32 * W);
  // A tile whose pipeline gave up (GQA_ERR_TIMEOUT is set) stores no partial
  // state, but still takes its merge ticket, so that the segment's ticket
  // counter returns to zero as after any other call.
  const bool tile_aborted = *abort_flag != 0;
  // The sequence's only split, with the partial states the call's own: the
  // output straight from the slots above (no partial state stored, no ticket).
  if (a.merge && a.partials_internal && !tile_aborted && t.kbeg == 0 && t.kend == t.n) {
    finalize_single_split<D, W, HP>(a, t, ms, ls, accs, nslots, ctid, smM, smL, smC, smN, NamedSync128{});
    return;
  }
  if (!tile_aborted) store_partial<D, W, HP>(a, t, ms, ls, accs, ctid, 32 * W, nslots);
  static_assert(C::kConsumerWarps == 4, "NamedSync128 spans the four consumer warps");
  if (a.merge) {
    ptx::named_barrier_sync(1, 32 * W);     // store_partial done with the ring scratch
    finish_segment<D, HP>(a, t, ctid, smM, smL, smC, smFlag, reinterpret_cast<float*>(smem),
                          C::kWeightCap, bar_merge, NamedSync128{}, tile_aborted);
  }
}

}  // namespace gqa
