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
//  * The CTA that completes the last split of a (sequence, KV head) segment
//    merges the segment's partial states and the carry and writes the output
//    (ticket counter per segment), so one launch does the whole call.
//  * gqa_merge_kernel<D>: the standalone merge of caller-held states and a
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
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace gqa {

constexpr uint32_t kErrBadOffsets = 1u;
constexpr uint32_t kErrTimeout = 2u;
constexpr uint32_t kErrBadCodes = 4u;
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
  // Fused merge: when `merge` is set, the CTA that completes the last split of a
  // (sequence, KV head) segment folds all its partial states and the carry and
  // writes out / state_out. counters[B*G] are per-segment tickets, zero between
  // calls (the merging CTA resets its own).
  int32_t merge;
  uint32_t* counters;
  const float* cm;           // carry [B*H] / [B*H, D], or null
  const float* cl;
  const float* cacc;
  float* om;                 // state out, or null (may alias the carry)
  float* ol;
  float* oacc;
  void* out;                 // [B*H, D] or null
  int32_t out_bf16;
  // Additive logit bias per cache row (fp32 [max_len], natural-log units, -inf
  // masks the key), or null (needle_core attn.rs, self_attn_incremental: attn_bias).
  const float* bias;
  // Append (needle_core attn.rs, KvCache::push_kv before the attention): when
  // k_new is set, the new token of sequence b is its last key, row
  // offsets[b+1]-1: the CTA owning that key writes k_new/v_new [B, G, D] into
  // kw/vw (the caches) and folds the key in from k_new/v_new directly.
  const void* k_new;
  const void* v_new;
  void* kw;
  void* vw;
  int32_t kv_elem;           // bytes per cache element (2 or 4)
  // Where a CTA lets the next kernel on the stream be scheduled (early-start
  // launches): 1 = once its producer has issued the tile's last load, 0 = once
  // its consumers have finished the tile's cache stream.
  int32_t trigger_at_last_load;
};

// Work item of a CTA: flattened index -> (b, split c, g), g fastest so that the
// CTAs reading the KV heads of the same cache rows run side by side.
struct Tile {
  int b, c, g;
  int o0;           // first cache row of the sequence
  int n;            // keys of the sequence (0 if its offsets are malformed)
  int kbeg, kend;   // key range of the tile, relative to the sequence
  int kstream;      // end of the keys read from the cache (kend, or n-1 for the append tile)
  bool append;      // this tile owns the appended (last) key of the sequence
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
  t.n = n;
  t.kbeg = t.c * a.chunk_len;
  t.kend = (t.c == a.num_splits - 1) ? n : min(n, t.kbeg + a.chunk_len);
  t.append = a.k_new != nullptr && t.kbeg < t.kend && t.kend == n;
  t.kstream = t.append ? n - 1 : t.kend;
  if (a.k_new != nullptr && n == 0 && t.c == 0 && t.g == 0 && threadIdx.x == 0)
    atomicOr(a.err, kErrBadOffsets);     // no row for the appended token
  return t;
}

// Logit bias of key `key` (relative to the sequence) in base-2 units.
__device__ __forceinline__ float bias2(const PartitionArgs& a, const Tile& t, int key) {
  return a.bias != nullptr ? __ldg(a.bias + t.o0 + key) * kLog2e : 0.f;
}

// Append tile: copy the new token's K and V rows of head g into the caches.
__device__ __forceinline__ void write_appended_row(const PartitionArgs& a, const Tile& t, int D,
                                                   int tid, int nthreads) {
  const size_t row_bytes = static_cast<size_t>(D) * a.kv_elem;
  const size_t src = (static_cast<size_t>(t.b) * a.G + t.g) * row_bytes;
  const size_t dst = ((static_cast<size_t>(t.o0) + t.n - 1) * a.G + t.g) * row_bytes;
  const int chunks = static_cast<int>(row_bytes / 16);
  for (int i = tid; i < 2 * chunks; i += nthreads) {
    const bool isv = i >= chunks;
    const int j = isv ? i - chunks : i;
    const uint4 val = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(isv ? a.v_new : a.k_new) + src + 16 * j);
    *reinterpret_cast<uint4*>(static_cast<uint8_t*>(isv ? a.vw : a.kw) + dst + 16 * j) = val;
  }
}

// Base-2 logit of the appended key for query head h of the tile's group,
// computed by one warp (lanes split D); q and k_new in the cache dtype.
template <int D, typename T>
__device__ __forceinline__ float appended_logit2(const PartitionArgs& a, const Tile& t, int h, int lane) {
  const T* q = static_cast<const T*>(a.q) + (static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * a.hpk + h) * D;
  const T* k = static_cast<const T*>(a.k_new) + (static_cast<size_t>(t.b) * a.G + t.g) * D;
  float s = 0.f;
  for (int d = lane; d < D; d += 32) s = fmaf(static_cast<float>(q[d]), static_cast<float>(k[d]), s);
  for (int x = 16; x >= 1; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
  return s * a.scale_log2 + bias2(a, t, t.n - 1);
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
// tile's partial state. ms/ls: [nslots][HP] base-2 maxima and partitions; accs:
// [nslots][HP][D + 4], already rescaled to the tile maximum; nslots is W, or
// W + 1 when the appended key occupies an extra slot. Threads 0..nthreads-1.
template <int D, int W, int HP>
__device__ __forceinline__ void store_partial(const PartitionArgs& a, const Tile& t,
                                              const float* ms, const float* ls, const float* accs,
                                              int tid, int nthreads, int nslots = W) {
  constexpr int P = D + 4;
  for (int i = tid; i < a.hpk * D; i += nthreads) {
    const int h = i / D, d = i % D;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < W + 1; ++w)
      if (w < nslots) s += accs[(w * HP + h) * P + d];
    a.part_acc[state_index(a, t, h) * D + d] = s;
  }
  for (int h = tid; h < a.hpk; h += nthreads) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W + 1; ++w)
      if (w < nslots) M = fmaxf(M, ms[w * HP + h]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < W + 1; ++w)
      if (w < nslots) L += ls[w * HP + h] * exp2f(ms[w * HP + h] - Mu);
    const size_t s = state_index(a, t, h);
    a.part_m[s] = (L == 0.f) ? -INFINITY : M * kLn2;
    a.part_l[s] = L;
  }
}

// Splits of the segment that hold keys: ceil(n / chunk_len), at most S (the
// last split takes any remainder).
__device__ __forceinline__ int live_splits(const PartitionArgs& a, const Tile& t) {
  return t.n == 0 ? 0 : min(a.num_splits, (t.n + a.chunk_len - 1) / a.chunk_len);
}

// Final merge of one segment's hpk query rows (USearch linear algebra,
// DenseAttendConfig::carry: partial-softmax rescaling), run by the 128 threads
// `tid` of the CTA that completed the segment: for each row,
//   M = max over non-empty splits and the carry of m,
//   L = sum l e^{m - M},  ACC = sum acc e^{m - M},  out = ACC / L (0 if L == 0).
// The merge sits on the kernel's critical path (uniform batches finish all
// their splits together), so it is built to wait on memory about twice:
//  1. every (row, split) pair's (m, l) is fetched at once into shared memory;
//     a warp per row then forms the weights e^{m - M} in place, M and L;
//  2. thread (column quad qd, split group cg) keeps one float4 accumulator per
//     row and fetches all its splits' acc quads of all rows back to back;
//     the split groups of a quad sit in adjacent lanes and add up by shuffles.
// When 2 * hpk * nsplit exceeds the shared scratch (2 * wcap floats) a slower
// path recomputes the weights from global memory. smM/smL/smC: >= hpk floats.
// Partial states written by other CTAs are read with ld.global.cg (L2).
template <int D, int HP, class Sync>
__device__ __forceinline__ void merge_segment(const PartitionArgs& a, const Tile& t, int nsplit,
                                              int tid, float* smM, float* smL, float* smC,
                                              float* wts, int wcap, Sync sync) {
  constexpr int NT = 128;
  constexpr int Q = D / 4;             // column quads
  constexpr int GC = NT / Q;           // split groups: 4 (D=128) or 8 (D=64)
  const int warp = tid >> 5, lane = tid & 31;
  const size_t row0 = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * a.hpk;
  const int S = a.num_splits;
  const int hpk = a.hpk;
  const int pairs = hpk * nsplit;
  const bool staged = pairs <= wcap;
  float* wm = wts;                     // [hpk][nsplit]: m, then the weight
  float* wl = wts + wcap;              // [hpk][nsplit]: l
  if (staged) {
    for (int p = tid; p < pairs; p += NT) {
      const int h = p / nsplit, c = p - h * nsplit;
      const size_t si = (row0 + h) * S + c;
      wm[p] = __ldcg(a.part_m + si);
      wl[p] = __ldcg(a.part_l + si);
    }
    sync();
  }
  for (int h = warp; h < hpk; h += NT / 32) {
    const size_t r = row0 + h;
    float M = -INFINITY;
    for (int c = lane; c < nsplit; c += 32) {
      const float lc = staged ? wl[h * nsplit + c] : __ldcg(a.part_l + r * S + c);
      const float mc = staged ? wm[h * nsplit + c] : __ldcg(a.part_m + r * S + c);
      if (lc != 0.f) M = fmaxf(M, mc);
    }
    for (int x = 16; x >= 1; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    const bool has_carry = a.cl != nullptr && a.cl[r] != 0.f;
    if (has_carry) M = fmaxf(M, a.cm[r]);
    float L = 0.f;
    for (int c = lane; c < nsplit; c += 32) {
      const float lc = staged ? wl[h * nsplit + c] : __ldcg(a.part_l + r * S + c);
      const float mc = staged ? wm[h * nsplit + c] : __ldcg(a.part_m + r * S + c);
      const float w = (lc != 0.f && M != -INFINITY) ? expf(mc - M) : 0.f;
      L = fmaf(lc, w, L);
      if (staged) wm[h * nsplit + c] = w;
    }
    for (int x = 16; x >= 1; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
    float wc = 0.f;
    if (has_carry) {
      wc = expf(a.cm[r] - M);
      L = fmaf(a.cl[r], wc, L);
    }
    if (lane == 0) {
      smM[h] = M;
      smL[h] = L;
      smC[h] = wc;
    }
  }
  sync();

  const int qd = tid / GC, cg = tid % GC;
  float4 acc[HP];
#pragma unroll
  for (int h = 0; h < HP; ++h) acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (staged) {
    // Issue every load of a batch of U splits x HP rows before any arithmetic:
    // the loads are independent, so the batch costs one trip to L2.
    constexpr int U = HP <= 8 ? 2 : 1;
#pragma unroll 1
    for (int c0 = cg; c0 < nsplit; c0 += U * GC) {
      float4 v[U][HP];
      float w[U][HP];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * GC;
#pragma unroll
        for (int h = 0; h < HP; ++h) {
          const bool live = h < hpk && c < nsplit;
          w[u][h] = live ? wm[h * nsplit + c] : 0.f;
          v[u][h] = live ? __ldcg(reinterpret_cast<const float4*>(a.part_acc + ((row0 + h) * S + c) * D) + qd)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int h = 0; h < HP; ++h) {
          acc[h].x = fmaf(v[u][h].x, w[u][h], acc[h].x);
          acc[h].y = fmaf(v[u][h].y, w[u][h], acc[h].y);
          acc[h].z = fmaf(v[u][h].z, w[u][h], acc[h].z);
          acc[h].w = fmaf(v[u][h].w, w[u][h], acc[h].w);
        }
    }
  } else {
    // Too many splits to stage their weights: recompute them (slower).
    for (int c = cg; c < nsplit; c += GC) {
      for (int h = 0; h < hpk && h < HP; ++h) {
        const size_t si = (row0 + h) * S + c;
        const float lc = __ldcg(a.part_l + si);
        const float w = (lc != 0.f && smM[h] != -INFINITY) ? expf(__ldcg(a.part_m + si) - smM[h]) : 0.f;
        if (w == 0.f) continue;
        const float4 vv = __ldcg(reinterpret_cast<const float4*>(a.part_acc + si * D) + qd);
        acc[h].x = fmaf(vv.x, w, acc[h].x);
        acc[h].y = fmaf(vv.y, w, acc[h].y);
        acc[h].z = fmaf(vv.z, w, acc[h].z);
        acc[h].w = fmaf(vv.w, w, acc[h].w);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HP; ++h) {
    if (h >= hpk) break;
#pragma unroll
    for (int x = 1; x < GC; x <<= 1) {
      acc[h].x += __shfl_xor_sync(0xffffffffu, acc[h].x, x);
      acc[h].y += __shfl_xor_sync(0xffffffffu, acc[h].y, x);
      acc[h].z += __shfl_xor_sync(0xffffffffu, acc[h].z, x);
      acc[h].w += __shfl_xor_sync(0xffffffffu, acc[h].w, x);
    }
  }
  if (cg == 0) {
#pragma unroll
    for (int h = 0; h < HP; ++h) {
      if (h >= hpk) break;
      const size_t r = row0 + h;
      const float wc = smC[h];
      float y[4] = {acc[h].x, acc[h].y, acc[h].z, acc[h].w};
      if (wc != 0.f) {
        const float4 cv = *reinterpret_cast<const float4*>(a.cacc + r * D + qd * 4);
        y[0] = fmaf(cv.x, wc, y[0]);
        y[1] = fmaf(cv.y, wc, y[1]);
        y[2] = fmaf(cv.z, wc, y[2]);
        y[3] = fmaf(cv.w, wc, y[3]);
      }
      if (a.oacc) *reinterpret_cast<float4*>(a.oacc + r * D + qd * 4) = make_float4(y[0], y[1], y[2], y[3]);
      if (a.out) {
        const float L = smL[h];
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = (L == 0.f) ? 0.f : __fdiv_rn(y[e], L);
        if (a.out_bf16) {
          __nv_bfloat162* dst =
              reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.out) + r * D + qd * 4);
          dst[0] = __floats2bfloat162_rn(o[0], o[1]);
          dst[1] = __floats2bfloat162_rn(o[2], o[3]);
        } else {
          *reinterpret_cast<float4*>(static_cast<float*>(a.out) + r * D + qd * 4) =
              make_float4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }
  // m and l of the state out are written after every thread has read the carry
  // (state out may alias it).
  sync();
  if (a.om)
    for (int h = tid; h < hpk; h += NT) {
      a.om[row0 + h] = (smL[h] == 0.f) ? -INFINITY : smM[h];
      a.ol[row0 + h] = smL[h];
    }
}

// The same merge with the segment's partial acc rows brought into shared
// memory by TMA bulk copies (one per query row: its nsplit splits are
// contiguous), issued before the (m, l) loads so that both round trips to L2
// overlap; the weighted sums then run out of shared memory. Needs
// hpk * nsplit * (D + 2) floats of `ring` (bytes `cap`) and the mbarrier `bar`
// (initialised with count 1, phase 0 unused). Returns false, doing nothing,
// when the segment does not fit.
template <int D, class Sync>
__device__ __forceinline__ bool merge_segment_smem(const PartitionArgs& a, const Tile& t, int nsplit,
                                                   int tid, float* smM, float* smL, float* smC,
                                                   uint8_t* ring, int cap, uint32_t bar, Sync sync) {
  constexpr int NT = 128;
  constexpr int Q = D / 4;
  constexpr int GC = NT / Q;
  const int hpk = a.hpk;
  const int pairs = hpk * nsplit;
  if (nsplit == 0 || static_cast<size_t>(pairs) * (D + 2) * 4 > static_cast<size_t>(cap)) return false;
  const int warp = tid >> 5, lane = tid & 31;
  const size_t row0 = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * a.hpk;
  const int S = a.num_splits;
  float* accS = reinterpret_cast<float*>(ring);           // [hpk][nsplit][D]
  float* wm = accS + static_cast<size_t>(pairs) * D;       // [hpk][nsplit]
  float* wl = wm + pairs;
  ptx::fence_proxy_async_smem();    // this thread's earlier generic writes to the ring
  sync();
  if (tid == 0) {
    ptx::fence_proxy_async_global();
    const uint32_t row_bytes = static_cast<uint32_t>(nsplit) * D * 4;
    ptx::mbar_arrive_expect_tx(bar, row_bytes * hpk);
    for (int h = 0; h < hpk; ++h)
      ptx::bulk_load_1d(ptx::smem_u32(accS) + h * row_bytes, a.part_acc + (row0 + h) * S * D, row_bytes, bar);
  }
  for (int p = tid; p < pairs; p += NT) {
    const int h = p / nsplit, c = p - h * nsplit;
    const size_t si = (row0 + h) * S + c;
    wm[p] = __ldcg(a.part_m + si);
    wl[p] = __ldcg(a.part_l + si);
  }
  sync();
  for (int h = warp; h < hpk; h += NT / 32) {
    const size_t r = row0 + h;
    float M = -INFINITY;
    for (int c = lane; c < nsplit; c += 32)
      if (wl[h * nsplit + c] != 0.f) M = fmaxf(M, wm[h * nsplit + c]);
    for (int x = 16; x >= 1; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
    const bool has_carry = a.cl != nullptr && a.cl[r] != 0.f;
    if (has_carry) M = fmaxf(M, a.cm[r]);
    float L = 0.f;
    for (int c = lane; c < nsplit; c += 32) {
      const float lc = wl[h * nsplit + c];
      const float w = (lc != 0.f && M != -INFINITY) ? expf(wm[h * nsplit + c] - M) : 0.f;
      L = fmaf(lc, w, L);
      wm[h * nsplit + c] = w;
    }
    for (int x = 16; x >= 1; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
    float wc = 0.f;
    if (has_carry) {
      wc = expf(a.cm[r] - M);
      L = fmaf(a.cl[r], wc, L);
    }
    if (lane == 0) {
      smM[h] = M;
      smL[h] = L;
      smC[h] = wc;
    }
  }
  sync();
  const bool landed = ptx::mbar_wait_bounded(bar, 0, nullptr, kWaitLimitNs);
  if (!landed) {
    // Record the failure, give the copies one more bounded wait so none is
    // left writing into a finished CTA's shared memory, and skip the output.
    if (tid == 0) atomicOr(a.err, kErrTimeout);
    ptx::mbar_wait_bounded(bar, 0, nullptr, kWaitLimitNs);
    return true;
  }
  // thread (column quad qd, row group hg): whole rows out of shared memory
  const int qd = tid % Q, hg = tid / Q;
  for (int h = hg; h < hpk; h += GC) {
    const size_t r = row0 + h;
    const float* src = accS + static_cast<size_t>(h) * nsplit * D + qd * 4;
    const float* w = wm + h * nsplit;
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int c = 0; c < nsplit; ++c) {
      const float4 v = *reinterpret_cast<const float4*>(src + static_cast<size_t>(c) * D);
      const float wc = w[c];
      y.x = fmaf(v.x, wc, y.x);
      y.y = fmaf(v.y, wc, y.y);
      y.z = fmaf(v.z, wc, y.z);
      y.w = fmaf(v.w, wc, y.w);
    }
    const float cw = smC[h];
    if (cw != 0.f) {
      const float4 cv = *reinterpret_cast<const float4*>(a.cacc + r * D + qd * 4);
      y.x = fmaf(cv.x, cw, y.x);
      y.y = fmaf(cv.y, cw, y.y);
      y.z = fmaf(cv.z, cw, y.z);
      y.w = fmaf(cv.w, cw, y.w);
    }
    if (a.oacc) *reinterpret_cast<float4*>(a.oacc + r * D + qd * 4) = y;
    if (a.out) {
      const float L = smL[h];
      const float o0 = (L == 0.f) ? 0.f : __fdiv_rn(y.x, L);
      const float o1 = (L == 0.f) ? 0.f : __fdiv_rn(y.y, L);
      const float o2 = (L == 0.f) ? 0.f : __fdiv_rn(y.z, L);
      const float o3 = (L == 0.f) ? 0.f : __fdiv_rn(y.w, L);
      if (a.out_bf16) {
        __nv_bfloat162* dst =
            reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.out) + r * D + qd * 4);
        dst[0] = __floats2bfloat162_rn(o0, o1);
        dst[1] = __floats2bfloat162_rn(o2, o3);
      } else {
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + r * D + qd * 4) = make_float4(o0, o1, o2, o3);
      }
    }
  }
  sync();
  if (a.om)
    for (int h = tid; h < hpk; h += NT) {
      a.om[row0 + h] = (smL[h] == 0.f) ? -INFINITY : smM[h];
      a.ol[row0 + h] = smL[h];
    }
  return true;
}

// After the CTA's partial state is stored: take a ticket on the segment and,
// if this CTA completed it, merge. All participating threads call this.
template <int D, int HP, class Sync>
__device__ __forceinline__ void finish_segment(const PartitionArgs& a, const Tile& t, int tid,
                                               float* smM, float* smL, float* smC, int* smFlag,
                                               float* wts, int wcap, uint32_t bulk_bar, Sync sync) {
  const int nsplit = live_splits(a, t);
  if (nsplit > 1) {
    // The barrier orders every thread's partial-state stores before thread 0's
    // ticket; the ticket's release makes them visible device-wide to the CTA
    // that draws the last ticket, whose acquire (and the barrier after it)
    // orders its reads of the other splits' states after their stores.
    sync();
    if (tid == 0) {
      const unsigned seg = static_cast<unsigned>(t.b) * a.G + t.g;
      const unsigned ticket = ptx::atomic_add_acq_rel_gpu(a.counters + seg, 1u);
      const int last = (ticket == static_cast<unsigned>(nsplit - 1));
      if (last) a.counters[seg] = 0u;   // every split has counted: reset for the next call
      *smFlag = last;
    }
    sync();
    if (!*smFlag) return;
  } else {
    sync();                     // a single split: the CTA merges its own partial
  }
  if (bulk_bar != 0u &&
      merge_segment_smem<D>(a, t, nsplit, tid, smM, smL, smC, reinterpret_cast<uint8_t*>(wts),
                            2 * wcap * 4, bulk_bar, sync))
    return;
  merge_segment<D, HP>(a, t, nsplit, tid, smM, smL, smC, wts, wcap, sync);
}

struct NamedSync128 {
  __device__ __forceinline__ void operator()() const { ptx::named_barrier_sync(1, 128); }
};
struct BlockSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

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
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
  if (*abort_flag) return;
  store_partial<D, W, HP>(a, t, ms, ls, accs, ctid, 32 * W, nslots);
  static_assert(C::kConsumerWarps == 4, "NamedSync128 spans the four consumer warps");
  if (a.merge) {
    ptx::named_barrier_sync(1, 32 * W);     // store_partial done with the ring scratch
    finish_segment<D, HP>(a, t, ctid, smM, smL, smC, smFlag, reinterpret_cast<float*>(smem),
                          C::kWeightCap, bar_merge, NamedSync128{});
  }
}

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
  }
  // U keys per warp step: their loads are issued together, their per-head dot
  // products reduced together (U-way interleaved butterflies), and the running
  // state rescaled once per step.
  constexpr int U = 4;
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
template <int D, int HMAX>
__global__ void __launch_bounds__(256) gqa_partition_coded_kernel(const PartitionArgs a, const CodedArgs c) {
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
        const uint32_t word = __ldg(kc + w);
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
        const uint32_t word = __ldg(vc + w);
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
