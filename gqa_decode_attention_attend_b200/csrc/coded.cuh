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

// Word w of a code row: rows of a multiple of 4 words are read 16 bytes at a
// time (the compiler merges the four reads of one quad), others word by word.
__device__ __forceinline__ uint32_t code_word(const uint32_t* row, int w, int words) {
  if ((words & 3) == 0) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(row) + (w >> 2));
    const int r = w & 3;
    return r == 0 ? q.x : r == 1 ? q.y : r == 2 ? q.z : q.w;
  }
  return __ldg(row + w);
}

// Decode attention straight from the codes, never rebuilding a row:
//   q.K_j = sum_w c_jw (q . katom[i_jw])  -- a table qa[h][atom] of the CTA's
//     query heads against every K atom, built once per CTA, then lookups;
//   sum_j p_j V_j = sum_atom (sum_{j,w: i'_jw = atom} p_j c'_jw) vatom[atom]
//     -- per-atom weights Wt[h][atom] accumulated per key (shared atomics),
//     multiplied by the V atoms once at the end.
// The online softmax runs per block of 256 keys (one key per thread): the
// block's maximum per head, a rescale of l and Wt when it grows, then the
// block's weights. Same tiles, partial states and fused merge as the other
// partition kernels; the Wt sums are not bit-reproducible (atomic order).
// Two CTAs per SM (registers capped at 128), as the split plan assumes.
template <int D, int HMAX>
__global__ void __launch_bounds__(256, 2) gqa_partition_coded_kernel(const PartitionArgs a, const CodedArgs c) {
  constexpr int NT = 256, NW = NT / 32;
  extern __shared__ float csm[];
  __shared__ float qs[HMAX * D];
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
  // query rows of the group, then the logit table against every K atom
  const size_t qrow = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * hpk;
  for (int i = tid; i < hpk * D; i += NT)
    qs[i] = c.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qrow * D + i])
                     : static_cast<const float*>(a.q)[qrow * D + i];
  if (tid < HMAX) {
    Mrun[tid] = -INFINITY;
    Lrun[tid] = 0.f;
  }
  __syncthreads();
  for (int at = tid; at < NA; at += NT) {
    float dot[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) dot[h] = 0.f;
    const float4* ka = reinterpret_cast<const float4*>(c.k_atoms + static_cast<size_t>(at) * D);
#pragma unroll 4
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 kv = __ldg(ka + d4);
#pragma unroll
      for (int h = 0; h < HMAX; ++h) {
        if (h >= hpk) break;
        const float* qh = qs + h * D + d4 * 4;
        dot[h] = fmaf(qh[0], kv.x, fmaf(qh[1], kv.y, fmaf(qh[2], kv.z, fmaf(qh[3], kv.w, dot[h]))));
      }
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
      if (h < hpk) {
        qa[h * NA + at] = dot[h] * a.scale_log2;
        Wt[h * NA + at] = 0.f;
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
    float sc[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) sc[h] = live ? 0.f : -INFINITY;
    if (live) {
      const uint32_t* kc = c.k_codes + crow * W;
      for (int w = 0; w < W; ++w) {
        const uint32_t word = code_word(kc, w, W);
        const int idx = static_cast<int>(word >> 16);
        const float cf = __half2float(__ushort_as_half(static_cast<unsigned short>(word & 0xFFFFu)));
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
      const uint32_t* vc = c.v_codes + crow * W;
      for (int w = 0; w < W; ++w) {
        const uint32_t word = code_word(vc, w, W);
        const int idx = static_cast<int>(word >> 16);
        const float cf = __half2float(__ushort_as_half(static_cast<unsigned short>(word & 0xFFFFu)));
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

  // acc[h][d] = sum over atoms of Wt[h][atom] * vatom[atom][d]; the state goes
  // out exactly as store_partial writes a single slot
  for (int i = tid; i < hpk * D; i += NT) {
    const int h = i / D, d = i % D;
    const float* wr = Wt + h * NA;
    float acc = 0.f;
#pragma unroll 8
    for (int at = 0; at < NA; ++at) acc = fmaf(wr[at], __ldg(c.v_atoms + static_cast<size_t>(at) * D + d), acc);
    a.part_acc[state_index(a, t, h) * D + d] = acc;
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
