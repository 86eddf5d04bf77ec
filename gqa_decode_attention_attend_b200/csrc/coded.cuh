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
constexpr int kCodedThreads = 256;     // one key per thread per block of keys
// Largest heads_per_kv * n_atoms: three tables of that many words (logits,
// value weights, the block's integer weights) in shared memory.
constexpr int kCodedMaxTableEntries = 12288;

// Code rows are prefetched into a ring of blocks: three slots (two blocks
// ahead) up to 8 words per row, two slots (one block ahead) above.
__host__ __device__ constexpr int coded_code_slots(int words) { return words <= 8 ? 3 : 2; }

// Dynamic shared memory of the coded kernel: the code ring, then the three tables.
__host__ __device__ constexpr size_t coded_smem_bytes(int words, int hpk, int n_atoms) {
  return static_cast<size_t>(coded_code_slots(words)) * 2 * words * kCodedThreads * 4 +
         static_cast<size_t>(3) * hpk * n_atoms * 4;
}

__device__ __forceinline__ float code_coeff(uint32_t word) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(word & 0xFFFFu)));
}

// Fixed-point scale of one head's value weights in a block. The weights of
// any atom sum, in absolute value, to at most bound = sum_j p_j sum_w |c_jw|
// over the block's keys, so weights scaled by 2^e with bound * 2^e <= 2^30
// (and each rounded by at most 1/2) sum without overflow in 32-bit integers;
// the rounding errors stay below 2^-30 * bound per weight, relative to the
// block's whole value sum.
__device__ __forceinline__ float block_weight_scale(float bound) {
  if (!(bound > 0.f)) return 1073741824.f;                   // no weight this block (or NaN)
  if (!(bound < INFINITY)) return 0.f;
  // ceil(log2(bound)) from the bits: the exponent, plus one unless a power of 2
  const int bits = __float_as_int(bound);
  int cl = ((bits >> 23) & 0xFF) - 127 + ((bits & 0x7FFFFF) != 0 ? 1 : 0);
  if ((bits >> 23) == 0) cl = -126;                          // subnormal: below 2^-126
  const int e = max(-126, min(30, 30 - cl));
  return __int_as_float((e + 127) << 23);                     // 2^e
}

// Decode attention straight from the codes, never rebuilding a row:
//   q.K_j = sum_w c_jw (q . katom[i_jw])  -- a table qa[atom][h] of the CTA's
//     query heads against every K atom, built once per CTA, then lookups;
//   sum_j p_j V_j = sum_atom (sum_{j,w: i'_jw = atom} p_j c'_jw) vatom[atom]
//     -- per-atom weights Wt[h][atom], multiplied by the V atoms once at the end.
// Keys go in blocks of 256 (one per thread). Each thread copies the K and V
// code rows of the blocks ahead into shared memory (cp.async, its own slots)
// while the current block runs. Per block: logits by table lookup, the
// block's maximum per head (barrier), the weights p, the bound on each head's
// weight sums (barrier), then every weight p * c is added to an integer table
// Wb in fixed point scaled to that bound (32-bit shared atomics, which B200
// executes several times faster than float ones, and whose sums do not
// depend on their order; barrier); at the next block's start Wb is folded
// into the float table Wt, rescaled to the new running maximum. The partition
// l is kept per thread and reduced once. So the coded kernel's results are
// bit-reproducible. The logit table is built by whole warps, lanes across D
// (coalesced atom rows), with a warp reduce-scatter of the partial dot
// products; the V atoms are applied by whole warps the same way (lanes across
// D, no cross-lane sums). Same tiles, partial states and
// fused merge as the other partition kernels. Two CTAs per SM for the usual
// table sizes (registers capped at 128), as the split plan assumes.
// MW: a compile-time bound on the words per row (4, 8 or 16) for the per-key loops.
template <int D, int HMAX, int MW>
__global__ void __launch_bounds__(kCodedThreads, 2)
gqa_partition_coded_kernel(const PartitionArgs a, const CodedArgs c) {
  static_assert(MW == 4 || MW == 8 || MW == 16, "words bound 4, 8 or 16");
  constexpr int NT = kCodedThreads, NW = NT / 32, E = D / 32;
  extern __shared__ __align__(16) uint32_t dsm[];
  __shared__ __align__(16) float qs[HMAX * D];
  __shared__ float accb[HMAX * D];
  __shared__ float red[NW][HMAX];        // per warp: maxima per head (then partitions)
  __shared__ float red2[NW][HMAX];       // per warp: weight bounds per head
  __shared__ float smM[16], smL[16], smC[16];
  __shared__ int smFlag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hpk = a.hpk, NA = c.n_atoms, W = c.words;
  const int slots = coded_code_slots(W);
  uint32_t* cbuf = dsm;                                        // [slots][2][W][NT] code ring
  float* qa = reinterpret_cast<float*>(dsm + slots * 2 * W * NT);   // [NA][hpk] logits (base 2)
  float* Wt = qa + hpk * NA;                                   // [hpk][NA] value weights
  uint32_t* Wb = reinterpret_cast<uint32_t*>(Wt + hpk * NA);   // [hpk][NA] block weights, fixed point

  const Tile t = tile_of(a, blockIdx.x);
  ptx::grid_dependency_wait();
  if (t.kbeg >= t.kend) {
    if (a.write_empty) write_empty_states<D>(a, t);
    if (a.merge && t.n == 0 && t.c == 0 && tid < 128)
      merge_segment<D, HMAX>(a, t, 0, tid, smM, smL, smC, qa, hpk * NA, NamedSync128{});
    return;
  }

  // This thread's code rows of block number `blk` (keys kbeg + 256 blk ..) go
  // to its own slots of ring slot blk % slots: K then V, as 16-byte quads
  // (quad-major, then thread) when the row is a multiple of 4 words, else word
  // by word (word-major). One commit group per block, empty past the tile.
  const bool quads = (W & 3) == 0;
  const uint32_t cbuf_u32 = ptx::smem_u32(cbuf);
  const int nblk = (t.kend - t.kbeg + NT - 1) / NT;
  auto stage_codes = [&](int blk) {
    const int key = t.kbeg + blk * NT + tid;
    if (blk < nblk && key < t.kend) {
      const size_t row = ((static_cast<size_t>(t.o0) + key) * a.G + t.g) * W;
      const uint32_t base = cbuf_u32 + (blk - (blk / slots) * slots) * 2 * W * NT * 4;
      if (quads) {
        for (int q = 0; q < W / 4; ++q) {
          ptx::cp_async_16(base + ((0 * (W / 4) + q) * NT + tid) * 16, c.k_codes + row + 4 * q);
          ptx::cp_async_16(base + ((1 * (W / 4) + q) * NT + tid) * 16, c.v_codes + row + 4 * q);
        }
      } else {
        for (int w = 0; w < W; ++w) {
          ptx::cp_async_4(base + ((0 * W + w) * NT + tid) * 4, c.k_codes + row + w);
          ptx::cp_async_4(base + ((1 * W + w) * NT + tid) * 4, c.v_codes + row + w);
        }
      }
    }
    ptx::cp_async_commit();
  };
  // this thread's K (kv = 0) or V (kv = 1) code row of a block out of its ring slot
  auto load_row = [&](const uint32_t* sl, int kv, uint32_t (&r)[MW]) {
    if (quads) {
#pragma unroll
      for (int q = 0; q < MW / 4; ++q) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (4 * q < W) v = reinterpret_cast<const uint4*>(sl)[(kv * (W / 4) + q) * NT + tid];
        r[4 * q] = v.x;
        r[4 * q + 1] = v.y;
        r[4 * q + 2] = v.z;
        r[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int w = 0; w < MW; ++w) r[w] = w < W ? sl[(kv * W + w) * NT + tid] : 0u;
    }
  };
  for (int blk = 0; blk < slots - 1; ++blk) stage_codes(blk);

  // query rows of the group
  const size_t qrow = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * hpk;
  for (int i = tid; i < hpk * D; i += NT) {
    qs[i] = c.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qrow * D + i])
                     : static_cast<const float*>(a.q)[qrow * D + i];
    accb[i] = 0.f;
  }
  for (int i = tid; i < hpk * NA; i += NT) {
    Wt[i] = 0.f;
    Wb[i] = 0u;
  }
  __syncthreads();
  // the logit table: a warp takes A = 32 / HMAX atoms per pass, lanes across D
  // (coalesced rows, two passes of loads in flight). Each lane's A x HMAX
  // partial dot products are summed across the warp by a reduce-scatter: at
  // each of 5 steps a lane keeps half of its values and adds the other half
  // from the lane `off` away, so lane L ends with atom L / HMAX, head L % HMAX.
  {
    constexpr int A = 32 / HMAX;
    float qreg[HMAX][E];
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
#pragma unroll
      for (int e = 0; e < E; ++e) qreg[h][e] = h < hpk ? qs[h * D + lane * E + e] : 0.f;
#pragma unroll 2
    for (int a0 = warp * A; a0 < NA; a0 += NW * A) {
      float v[32];
#pragma unroll
      for (int i = 0; i < A; ++i) {
        float kv[E];
        const int at = a0 + i;
#pragma unroll
        for (int e = 0; e < E; ++e)
          kv[e] = at < NA ? __ldg(c.k_atoms + static_cast<size_t>(at) * D + lane * E + e) : 0.f;
#pragma unroll
        for (int h = 0; h < HMAX; ++h) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) d = fmaf(qreg[h][e], kv[e], d);
          v[i * HMAX + h] = d;
        }
      }
#pragma unroll
      for (int st = 0; st < 5; ++st) {
        const int off = 16 >> st;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
          const float send = upper ? v[i] : v[i + off];
          const float keep = upper ? v[i + off] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      const int at = a0 + lane / HMAX, h = lane % HMAX;
      if (at < NA && h < hpk) qa[at * hpk + h] = v[0] * a.scale_log2;
    }
  }
  __syncthreads();

  // running maximum per head (identical in every thread), this thread's share
  // of the partition, and the previous block's rescale and scale for the fold
  float mrun[HMAX], lthr[HMAX], fprev[HMAX], inv_prev[HMAX];
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    mrun[h] = -INFINITY;
    lthr[h] = 0.f;
    fprev[h] = 1.f;
    inv_prev[h] = 0.f;
  }
  bool bad = false;
  const bool quad_heads = (hpk & 3) == 0;
#pragma unroll 1
  for (int blk = 0; blk < nblk; ++blk) {
    const int kb = t.kbeg + blk * NT;
    const int key = kb + tid;
    const bool live = key < t.kend;
    // this block's group has landed when at most slots - 2 later ones are pending
    if (slots == 3)
      ptx::cp_async_wait_group<1>();
    else
      ptx::cp_async_wait_group<0>();
    uint32_t kw[MW], vw[MW];
    const int slot = blk - (blk / slots) * slots;
    load_row(cbuf + slot * 2 * W * NT, 0, kw);
    load_row(cbuf + slot * 2 * W * NT, 1, vw);
    if (!live)
#pragma unroll
      for (int w = 0; w < MW; ++w) kw[w] = vw[w] = 0u;
    // the slot of the previous block, already read: own slots only, no barrier
    stage_codes(blk + slots - 1);
    // fold the previous block's integer weights into Wt (rescaled to the
    // maximum they were taken against) and clear them
    if (kb > t.kbeg)
#pragma unroll
      for (int h = 0; h < HMAX; ++h) {
        if (h >= hpk) break;
        for (int i = tid; i < NA; i += NT) {
          const int j = h * NA + i;
          Wt[j] = fmaf(Wt[j], fprev[h], static_cast<float>(static_cast<int32_t>(Wb[j])) * inv_prev[h]);
          Wb[j] = 0u;
        }
      }
    float sc[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) sc[h] = live ? 0.f : -INFINITY;
    float csum = 0.f;                // sum of |V coefficient| of the key
    if (live) {
#pragma unroll
      for (int w = 0; w < MW; ++w) {
        const int idx = static_cast<int>(kw[w] >> 16);
        const float cf = code_coeff(kw[w]);
        if (cf == 0.f) continue;
        if (idx >= NA) {
          bad = true;
          continue;
        }
        // an atom's logits of all heads sit side by side: 16-byte loads when
        // heads_per_kv is a multiple of 4
        const float* row = qa + idx * hpk;
        if (quad_heads) {
#pragma unroll
          for (int q4 = 0; q4 < HMAX / 4; ++q4)
            if (4 * q4 < hpk) {
              const float4 t4 = *reinterpret_cast<const float4*>(row + 4 * q4);
              sc[4 * q4] = fmaf(cf, t4.x, sc[4 * q4]);
              sc[4 * q4 + 1] = fmaf(cf, t4.y, sc[4 * q4 + 1]);
              sc[4 * q4 + 2] = fmaf(cf, t4.z, sc[4 * q4 + 2]);
              sc[4 * q4 + 3] = fmaf(cf, t4.w, sc[4 * q4 + 3]);
            }
        } else {
#pragma unroll
          for (int h = 0; h < HMAX; ++h)
            if (h < hpk) sc[h] = fmaf(cf, row[h], sc[h]);
        }
      }
      const float bb = bias2(a, t, key);
#pragma unroll
      for (int h = 0; h < HMAX; ++h) sc[h] += bb;
#pragma unroll
      for (int w = 0; w < MW; ++w) csum += fabsf(code_coeff(vw[w]));
    }
    // block maxima per head
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
      float v = sc[h];
      for (int x = 16; x >= 1; x >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, x));
      if (lane == 0) red[warp][h] = v;
    }
    __syncthreads();                 // red complete; Wb folded and clear
    float p[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) {
        p[h] = 0.f;
        continue;
      }
      float bm = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) bm = fmaxf(bm, red[w][h]);
      const float mn = fmaxf(mrun[h], bm);
      const float f = (mn == -INFINITY) ? 1.f : exp2f(mrun[h] - mn);
      mrun[h] = mn;
      fprev[h] = f;
      p[h] = exp2f(sc[h] - (mn == -INFINITY ? 0.f : mn));
      lthr[h] = fmaf(lthr[h], f, p[h]);
    }
    // per head: bound on the block's weight sums, summed in a fixed order
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
      float v = p[h] * csum;
      for (int x = 16; x >= 1; x >>= 1) v += __shfl_xor_sync(0xffffffffu, v, x);
      if (lane == 0) red2[warp][h] = v;
    }
    __syncthreads();                 // red2 complete
    float scale[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      float bound = 0.f;
      if (h < hpk)
#pragma unroll
        for (int w = 0; w < NW; ++w) bound += red2[w][h];
      scale[h] = block_weight_scale(bound);
      inv_prev[h] = scale[h] > 0.f ? 1.f / scale[h] : 0.f;
    }
    float ps[HMAX];                  // weights already in fixed-point units
#pragma unroll
    for (int h = 0; h < HMAX; ++h) ps[h] = p[h] * scale[h];
    if (live) {
#pragma unroll
      for (int w = 0; w < MW; ++w) {
        const int idx = static_cast<int>(vw[w] >> 16);
        const float cf = code_coeff(vw[w]);
        if (cf == 0.f) continue;
        if (idx >= NA) {
          bad = true;
          continue;
        }
#pragma unroll
        for (int h = 0; h < HMAX; ++h)
          if (h < hpk && p[h] != 0.f)
            atomicAdd(Wb + h * NA + idx, static_cast<uint32_t>(__float2int_rn(ps[h] * cf)));
      }
    }
    __syncthreads();                 // Wb complete before the next fold; red, red2 free
  }
  // the last block's weights
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    if (h >= hpk) break;
    for (int i = tid; i < NA; i += NT) {
      const int j = h * NA + i;
      Wt[j] = fmaf(Wt[j], fprev[h], static_cast<float>(static_cast<int32_t>(Wb[j])) * inv_prev[h]);
    }
  }
  // the partition: every thread's share, summed in a fixed order
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    if (h >= hpk) break;
    float v = lthr[h];
    for (int x = 16; x >= 1; x >>= 1) v += __shfl_xor_sync(0xffffffffu, v, x);
    if (lane == 0) red[warp][h] = v;
  }
  __syncthreads();
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
#pragma unroll 16
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
    // the warps' sums in warp order (deterministic), through accb
    for (int w = 0; w < NW; ++w) {
      if (warp == w) {
#pragma unroll
        for (int h = 0; h < HMAX; ++h) {
          if (h >= hpk) break;
#pragma unroll
          for (int e = 0; e < E; ++e) accb[h * D + lane * E + e] += acc[h][e];
        }
      }
      __syncthreads();
    }
  }
  // the state goes out exactly as store_partial writes a single slot
  for (int i = tid; i < hpk * D; i += NT) {
    const int h = i / D, d = i % D;
    a.part_acc[state_index(a, t, h) * D + d] = accb[i];
  }
#pragma unroll
  for (int h = 0; h < HMAX; ++h)
    if (h < hpk && tid == h) {
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) L += red[w][h];
      const size_t si = state_index(a, t, h);
      a.part_m[si] = (L == 0.f) ? -INFINITY : mrun[h] * kLn2;
      a.part_l[si] = L;
    }
  if (a.merge) {
    __syncthreads();
    if (tid < 128)
      finish_segment<D, HMAX>(a, t, tid, smM, smL, smC, &smFlag, qa, hpk * NA, 0u, NamedSync128{});
  }
}

}  // namespace gqa
