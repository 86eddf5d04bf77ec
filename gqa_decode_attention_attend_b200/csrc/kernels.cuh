// kernels.cuh -- the sm_100a kernels of the decode-attention hot path.
//
//  * gqa_partition_bf16_kernel<D, NT>: one CTA owns one (sequence b, KV head g,
//    key chunk c) tile. A producer warp streams the chunk's K/V rows of head g
//    through a ring of shared-memory stages with TMA (2-D tiled loads, 128-byte
//    swizzle, no multicast); four consumer warps each take 16 keys of every
//    stage and, for ALL heads_per_kv query heads of the group at once, compute
//    the logits S^T = K Q^T and the value sum O^T += V^T P^T on the tensor cores
//    (mma.sync m16n8k16, bf16 in, fp32 accumulate), with the online softmax
//    (running max m, partition l) in fp32 registers. K/V rows are read from HBM
//    once per group and broadcast to its query heads (cortiq_engine
//    NystromState: every Q head of a group reads the same K/V rows; needle_core
//    attn.rs: broadcast, not repeat-copy).
//  * gqa_partition_f32_kernel<D, HMAX>: the fp32 K/V variant on CUDA cores
//    (fp32 FMA keeps the fp32 tolerance; no tensor-core format is exact here).
//  * gqa_merge_kernel<D>: numerically stable merge of per-split states and the
//    carry (USearch linear algebra, DenseAttendConfig::carry: partial-softmax
//    rescaling), optional state out, optional out = acc / l.
//
// Inside the partition kernels logits are kept in base 2 (scale * log2 e folded
// into one multiply) so that exp2 is the only transcendental; every state that
// leaves a kernel stores m in natural-log units (the largest logit).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace gqa {

constexpr uint32_t kErrBadOffsets = 1u;
constexpr uint32_t kErrTimeout = 2u;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per pipeline wait
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

struct PartitionArgs {
  const void* q;             // [B, H, D]
  const void* k;             // [max_len, G, D] (fp32 kernel only; bf16 uses tensor maps)
  const void* v;
  const int32_t* offsets;    // [B+1]
  int32_t B, H, G, hpk, max_len;
  int32_t chunk_len, num_splits;
  float scale_log2;          // score_scale * log2(e)
  float* part_m;             // [B*H, S]
  float* part_l;             // [B*H, S]
  float* part_acc;           // [B*H, S, D]
  int32_t write_empty;       // write empty states for splits without keys
  uint32_t* err;             // device error word
};

// Work item of a CTA: flattened index -> (b, split c, g), g fastest so that the
// CTAs reading the KV heads of the same cache rows run side by side.
struct Tile {
  int b, c, g;
  int o0;           // first cache row of the sequence
  int kbeg, kend;   // key range of the tile, relative to the sequence
};

__device__ __forceinline__ Tile tile_of(const PartitionArgs& a, int bid) {
  Tile t;
  t.g = bid % a.G;
  const int rest = bid / a.G;
  t.c = rest % a.num_splits;
  t.b = rest / a.num_splits;
  int o0 = __ldg(a.offsets + t.b);
  int o1 = __ldg(a.offsets + t.b + 1);
  if (!(0 <= o0 && o0 <= o1 && o1 <= a.max_len)) {
    if (t.c == 0 && t.g == 0 && threadIdx.x == 0) atomicOr(a.err, kErrBadOffsets);
    o0 = o1 = 0;
  }
  const int n = o1 - o0;
  t.o0 = o0;
  t.kbeg = t.c * a.chunk_len;
  t.kend = (t.c == a.num_splits - 1) ? n : min(n, t.kbeg + a.chunk_len);
  return t;
}

__device__ __forceinline__ size_t state_index(const PartitionArgs& a, const Tile& t, int h) {
  return (static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * a.hpk + h) * a.num_splits + t.c;
}

template <int D>
__device__ __forceinline__ void write_empty_states(const PartitionArgs& a, const Tile& t) {
  for (int i = threadIdx.x; i < a.hpk * D; i += blockDim.x) {
    const int h = i / D, d = i % D;
    const size_t s = state_index(a, t, h);
    a.part_acc[s * D + d] = 0.f;
    if (d == 0) {
      a.part_m[s] = -INFINITY;
      a.part_l[s] = 0.f;
    }
  }
}

// Cross-warp combine of per-warp states held in shared memory, then store of the
// tile's partial state. ms/ls: [W][HP] base-2 maxima and partitions; accs:
// [W][HP][D + 4], already rescaled to the tile maximum. Threads 0..nthreads-1.
template <int D, int W, int HP>
__device__ __forceinline__ void store_partial(const PartitionArgs& a, const Tile& t,
                                              const float* ms, const float* ls, const float* accs,
                                              int tid, int nthreads) {
  constexpr int P = D + 4;
  for (int i = tid; i < a.hpk * D; i += nthreads) {
    const int h = i / D, d = i % D;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) s += accs[(w * HP + h) * P + d];
    a.part_acc[state_index(a, t, h) * D + d] = s;
  }
  for (int h = tid; h < a.hpk; h += nthreads) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, ms[w * HP + h]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) L += ls[w * HP + h] * exp2f(ms[w * HP + h] - Mu);
    const size_t s = state_index(a, t, h);
    a.part_m[s] = (L == 0.f) ? -INFINITY : M * kLn2;
    a.part_l[s] = L;
  }
}

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
  static constexpr int kScratchBytes = kConsumerWarps * kHP * (D + 4 + 2) * 4;
  static constexpr int kDataBytes = kRingBytes > kScratchBytes ? kRingBytes : kScratchBytes;
  static constexpr int kBarOffset = kDataBytes;                     // 2*kStages mbarriers
  static constexpr int kAbortOffset = kBarOffset + 2 * kStages * 8;
  static constexpr int kSmemBytes = 1024 + kAbortOffset + 16;       // + alignment slack
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
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = ptx::smem_u32(smem);
  const uint32_t bar_full = ring + C::kBarOffset;
  const uint32_t bar_empty = bar_full + C::kStages * 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbortOffset);

  const Tile t = tile_of(a, blockIdx.x);
  if (t.kbeg >= t.kend) {
    if (a.write_empty) write_empty_states<D>(a, t);
    return;
  }
  const int nst = (t.kend - t.kbeg + C::kStageKeys - 1) / C::kStageKeys;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(bar_full + 8 * s, 1);
      ptx::mbar_init(bar_empty + 8 * s, C::kConsumerWarps);
    }
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
    const int nvalid = min(C::kKeysPerWarp, t.kend - key0);
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
      uint32_t ph_hi[NT][2], ph_lo[NT][2];
      float alpha[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float p[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float s0 = (kr < nvalid) ? sacc[nt][e] * sl2 : -INFINITY;
          const float s1 = (kr + 8 < nvalid) ? sacc[nt][e + 2] * sl2 : -INFINITY;
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
  float* ms = reinterpret_cast<float*>(smem);
  float* ls = ms + W * HP;
  float* accs = ls + W * HP;
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        ms[warp * HP + nt * 8 + lane * 2 + e] = mrun[nt][e];
        ls[warp * HP + nt * 8 + lane * 2 + e] = lrun[nt][e];
      }
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
      for (int w = 0; w < W; ++w) M = fmaxf(M, ms[w * HP + hc]);
      const float Mu = (M == -INFINITY) ? 0.f : M;
      f[nt][e] = exp2f(mrun[nt][e] - Mu);
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
  if (*abort_flag) return;
  store_partial<D, W, HP>(a, t, ms, ls, accs, ctid, 32 * W);
}

// ============================================================================
// fp32 K/V: CUDA-core partition kernel
// ============================================================================

template <int D, int HMAX>
struct F32Cfg {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kE = D / 32;  // elements per lane
  static constexpr int kSmemBytes = kWarps * HMAX * (D + 4 + 2) * 4;
};

template <int D, int HMAX>
__global__ void __launch_bounds__(F32Cfg<D, HMAX>::kThreads)
gqa_partition_f32_kernel(const PartitionArgs a) {
  using C = F32Cfg<D, HMAX>;
  constexpr int E = C::kE, W = C::kWarps, HP = HMAX, P = D + 4;
  extern __shared__ float fsm[];
  const Tile t = tile_of(a, blockIdx.x);
  if (t.kbeg >= t.kend) {
    if (a.write_empty) write_empty_states<D>(a, t);
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
#pragma unroll 1
  for (int key = t.kbeg + warp; key < t.kend; key += W) {
    const size_t base = (static_cast<size_t>(t.o0) + key) * rs + static_cast<size_t>(t.g) * D + lane * E;
    float kv[E], vv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kv[e] = __ldg(kg + base + e);
      vv[e] = __ldg(vg + base + e);
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= a.hpk) break;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) s = fmaf(qv[h][e], kv[e], s);
#pragma unroll
      for (int x = 16; x >= 1; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
      const float s2 = s * a.scale_log2;
      const float mn = fmaxf(m[h], s2);
      const float al = exp2f(m[h] - mn);
      const float p = exp2f(s2 - mn);
      l[h] = l[h] * al + p;
#pragma unroll
      for (int e = 0; e < E; ++e) o[h][e] = fmaf(p, vv[e], o[h][e] * al);
      m[h] = mn;
    }
  }
  float* ms = fsm;
  float* ls = ms + W * HP;
  float* accs = ls + W * HP;
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      ms[warp * HP + h] = m[h];
      ls[warp * HP + h] = l[h];
    }
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    if (h >= a.hpk) break;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, ms[w * HP + h]);
    const float f = exp2f(m[h] - ((M == -INFINITY) ? 0.f : M));
#pragma unroll
    for (int e = 0; e < E; ++e) accs[(warp * HP + h) * P + lane * E + e] = o[h][e] * f;
  }
  __syncthreads();
  store_partial<D, W, HP>(a, t, ms, ls, accs, threadIdx.x, C::kThreads);
}

// ============================================================================
// merge / finalize
// ============================================================================

struct MergeArgs {
  const float* m;            // [rows, S]
  const float* l;            // [rows, S]
  const float* acc;          // [rows, S, D]
  int32_t rows, S;
  // When offsets != nullptr the states are the partition kernel's splits and row
  // r = b*H + h uses only the first ceil(N_b / chunk_len) of them (clamped to S).
  const int32_t* offsets;
  int32_t H, chunk_len, max_len;
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
  int nS = a.S;
  if (a.offsets != nullptr) {
    const int b = r / a.H;
    const int o0 = __ldg(a.offsets + b), o1 = __ldg(a.offsets + b + 1);
    const int n = (0 <= o0 && o0 <= o1 && o1 <= a.max_len) ? o1 - o0 : 0;
    nS = (n == 0) ? 0 : min(a.S, (n + a.chunk_len - 1) / a.chunk_len);
  }
  const size_t base = static_cast<size_t>(r) * a.S;
  // pass 1: the largest maximum among non-empty states (and the carry)
  float M = -INFINITY;
  for (int i = threadIdx.x; i < nS; i += blockDim.x)
    if (a.l[base + i] != 0.f) M = fmaxf(M, a.m[base + i]);
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
      const float li = a.l[base + i];
      if (li == 0.f) continue;
      const float w = expf(a.m[base + i] - M);
      L += li * w;
      const float* src = a.acc + (base + i) * D + lane * E;
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
