// coded.cuh -- the partition kernel over a dictionary-coded cache.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "tile.cuh"

namespace gqa {

// ============================================================================
// dictionary-coded cache (qualiaDB KvDictionary read path)
// ============================================================================

// Every cache row of every KV head is `words` code words: atom index in the
// high 16 bits, the coefficient's binary16 bits in the low 16 (a zero
// coefficient, as in padding words, contributes nothing). The row is
// sum_w coeff_w * atom[index_w] (KvDictionary::reconstruct_from_words).
struct CodedArgs {
  const uint32_t* k_codes;   // [max_len, G, words]
  const uint32_t* v_codes;
  const float* k_atoms;      // [n_atoms, D] fp32
  const float* v_atoms;
  int32_t words, n_atoms;
  int32_t q_bf16;
};

constexpr int kMaxCodeWords = 16;

// The words of one code row into registers (16-byte loads when the row is a
// multiple of 4 words, else word by word); words past `words` are zero.
__device__ __forceinline__ void load_code_row(const uint32_t* row, int words, uint32_t (&w)[kMaxCodeWords]) {
  if ((words & 3) == 0) {
#pragma unroll
    for (int q = 0; q < kMaxCodeWords / 4; ++q) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (4 * q < words) v = __ldg(reinterpret_cast<const uint4*>(row) + q);
      w[4 * q] = v.x;
      w[4 * q + 1] = v.y;
      w[4 * q + 2] = v.z;
      w[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kMaxCodeWords; ++i) w[i] = i < words ? __ldg(row + i) : 0u;
  }
}

__device__ __forceinline__ float code_coeff(uint32_t word) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(word & 0xFFFFu)));
}

// Decode attention straight from the codes, never rebuilding a row:
//   q.K_j = sum_w c_jw (q . katom[i_jw])  -- a table qa[h][atom] of the CTA's
//     query heads against every K atom, built once per CTA, then lookups;
//   sum_j p_j V_j = sum_atom (sum_{j,w: i'_jw = atom} p_j c'_jw) vatom[atom]
//     -- per-atom weights Wt[h][atom] accumulated per key (shared atomics),
//     multiplied by the V atoms once at the end.
// The online softmax runs per block of 256 keys (one key per thread, its K and
// V code rows fetched together): the block's maximum per head, a rescale of l
// and Wt when it grows, then the block's weights. The atom tables are built
// and applied by whole warps (lanes across D, one coalesced row per atom), so
// both cost a few trips to L2 rather than one per atom. Same tiles, partial
// states and fused merge as the other partition kernels; the Wt sums are not
// bit-reproducible (atomic order). Two CTAs per SM (registers capped at 128),
// as the split plan assumes.
template <int D, int HMAX>
__global__ void __launch_bounds__(256, 2) gqa_partition_coded_kernel(const PartitionArgs a, const CodedArgs c) {
  constexpr int NT = 256, NW = NT / 32, E = D / 32;
  extern __shared__ float csm[];
  __shared__ float qs[HMAX * D];
  __shared__ float accb[HMAX * D];
  __shared__ float red[NW][HMAX];
  __shared__ float Mrun[HMAX], Lrun[HMAX], fac[HMAX];
  __shared__ float smM[16], smL[16], smC[16];
  __shared__ int smFlag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hpk = a.hpk, NA = c.n_atoms;
  float* qa = csm;                  // [hpk][NA]
  float* Wt = csm + hpk * NA;       // [hpk][NA]

  const Tile t = tile_of(a, blockIdx.x);
  ptx::grid_dependency_wait();
  if (t.kbeg >= t.kend) {
    if (a.write_empty) write_empty_states<D>(a, t);
    if (a.merge && t.n == 0 && t.c == 0 && tid < 128)
      merge_segment<D, HMAX>(a, t, 0, tid, smM, smL, smC, csm, hpk * NA, NamedSync128{});
    return;
  }
  // query rows of the group
  const size_t qrow = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * hpk;
  for (int i = tid; i < hpk * D; i += NT) {
    qs[i] = c.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qrow * D + i])
                     : static_cast<const float*>(a.q)[qrow * D + i];
    accb[i] = 0.f;
  }
  if (tid < HMAX) {
    Mrun[tid] = -INFINITY;
    Lrun[tid] = 0.f;
  }
  for (int i = tid; i < hpk * NA; i += NT) Wt[i] = 0.f;
  __syncthreads();
  // the logit table: warp w takes atoms w, w+8, ...; lanes split D
  {
    float qreg[HMAX][E];
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
#pragma unroll
      for (int e = 0; e < E; ++e) qreg[h][e] = h < hpk ? qs[h * D + lane * E + e] : 0.f;
#pragma unroll 2
    for (int at = warp; at < NA; at += NW) {
      float kv[E];
#pragma unroll
      for (int e = 0; e < E; ++e) kv[e] = __ldg(c.k_atoms + static_cast<size_t>(at) * D + lane * E + e);
#pragma unroll
      for (int h = 0; h < HMAX; ++h) {
        if (h >= hpk) break;
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) d = fmaf(qreg[h][e], kv[e], d);
#pragma unroll
        for (int x = 16; x >= 1; x >>= 1) d += __shfl_xor_sync(0xffffffffu, d, x);
        if (lane == 0) qa[h * NA + at] = d * a.scale_log2;
      }
    }
  }
  __syncthreads();

  const int W = c.words;
  bool bad = false;
#pragma unroll 1
  for (int kb = t.kbeg; kb < t.kend; kb += NT) {
    const int key = kb + tid;
    const bool live = key < t.kend;
    const size_t crow = (static_cast<size_t>(t.o0) + (live ? key : t.kbeg)) * a.G + t.g;
    uint32_t kw[kMaxCodeWords], vw[kMaxCodeWords];
    if (live) {
      load_code_row(c.k_codes + crow * W, W, kw);
      load_code_row(c.v_codes + crow * W, W, vw);
    }
    float sc[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) sc[h] = live ? 0.f : -INFINITY;
    if (live) {
#pragma unroll
      for (int w = 0; w < kMaxCodeWords; ++w) {
        const int idx = static_cast<int>(kw[w] >> 16);
        const float cf = code_coeff(kw[w]);
        if (cf == 0.f) continue;
        if (idx >= NA) {
          bad = true;
          continue;
        }
#pragma unroll
        for (int h = 0; h < HMAX; ++h)
          if (h < hpk) sc[h] = fmaf(cf, qa[h * NA + idx], sc[h]);
      }
      const float bb = bias2(a, t, key);
#pragma unroll
      for (int h = 0; h < HMAX; ++h) sc[h] += bb;
    }
    // block maximum per head
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
      float v = sc[h];
      for (int x = 16; x >= 1; x >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, x));
      if (lane == 0) red[warp][h] = v;
    }
    __syncthreads();
    if (tid < hpk) {
      float bm = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) bm = fmaxf(bm, red[w][tid]);
      const float mo = Mrun[tid], mn = fmaxf(mo, bm);
      const float f = (mn == -INFINITY) ? 1.f : exp2f(mo - mn);
      fac[tid] = f;
      Mrun[tid] = mn;
      Lrun[tid] *= f;
    }
    __syncthreads();
    for (int i = tid; i < hpk * NA; i += NT) {
      const float f = fac[i / NA];
      if (f != 1.f) Wt[i] *= f;
    }
    float p[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      const float mu = (h < hpk && Mrun[h] != -INFINITY) ? Mrun[h] : 0.f;
      p[h] = (h < hpk) ? exp2f(sc[h] - mu) : 0.f;
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
      float v = p[h];
      for (int x = 16; x >= 1; x >>= 1) v += __shfl_xor_sync(0xffffffffu, v, x);
      if (lane == 0) red[warp][h] = v;
    }
    __syncthreads();                 // rescale of Wt done, partial sums of p in red
    if (tid < hpk) {
      float ssum = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) ssum += red[w][tid];
      Lrun[tid] += ssum;
    }
    if (live) {
#pragma unroll
      for (int w = 0; w < kMaxCodeWords; ++w) {
        const int idx = static_cast<int>(vw[w] >> 16);
        const float cf = code_coeff(vw[w]);
        if (cf == 0.f) continue;
        if (idx >= NA) {
          bad = true;
          continue;
        }
#pragma unroll
        for (int h = 0; h < HMAX; ++h)
          if (h < hpk && p[h] != 0.f) atomicAdd(Wt + h * NA + idx, p[h] * cf);
      }
    }
    __syncthreads();                 // Wt and red are reused by the next block
  }
  if (bad) atomicOr(a.err, kErrBadCodes);
  if (threadIdx.x == 0) ptx::grid_launch_dependents();

  // acc[h][d] = sum over atoms of Wt[h][atom] * vatom[atom][d]: warp w takes
  // atoms w, w+8, ... with lanes across D, then the warps add into accb
  {
    float acc[HMAX][E];
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
#pragma unroll 2
    for (int at = warp; at < NA; at += NW) {
      float vv[E];
#pragma unroll
      for (int e = 0; e < E; ++e) vv[e] = __ldg(c.v_atoms + static_cast<size_t>(at) * D + lane * E + e);
#pragma unroll
      for (int h = 0; h < HMAX; ++h) {
        if (h >= hpk) break;
        const float wgt = Wt[h * NA + at];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = fmaf(wgt, vv[e], acc[h][e]);
      }
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
#pragma unroll
      for (int e = 0; e < E; ++e) atomicAdd(accb + h * D + lane * E + e, acc[h][e]);
    }
  }
  __syncthreads();
  // the state goes out exactly as store_partial writes a single slot
  for (int i = tid; i < hpk * D; i += NT) {
    const int h = i / D, d = i % D;
    a.part_acc[state_index(a, t, h) * D + d] = accb[i];
  }
  if (tid < hpk) {
    const size_t si = state_index(a, t, tid);
    a.part_m[si] = (Lrun[tid] == 0.f) ? -INFINITY : Mrun[tid] * kLn2;
    a.part_l[si] = Lrun[tid];
  }
  if (a.merge) {
    __syncthreads();
    if (tid < 128)
      finish_segment<D, HMAX>(a, t, tid, smM, smL, smC, &smFlag, csm, hpk * NA, 0u, NamedSync128{});
  }
}

}  // namespace gqa
