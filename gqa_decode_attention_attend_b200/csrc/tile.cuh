// tile.cuh -- what the partition kernels share: their arguments, the (sequence, split,
// KV head) tile of a CTA, partial-state stores and the fused per-segment merge.
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
  // The partial states are the call's own scratch (no partials_out): a tile
  // that is its sequence's only split may then finalise without storing one.
  int32_t partials_internal;
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
  // heads in groups of HB (at most 8 float4 accumulators per thread)
  constexpr int HB = HP > 8 ? 8 : HP;
#pragma unroll 1
  for (int h0 = 0; h0 < hpk; h0 += HB) {
    float4 acc[HB];
#pragma unroll
    for (int hh = 0; hh < HB; ++hh) acc[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (staged) {
      // Issue every load of a batch of U splits x HB rows before any arithmetic:
      // the loads are independent, so the batch costs one trip to L2.
      constexpr int U = HB <= 4 ? 2 : 1;
#pragma unroll 1
      for (int c0 = cg; c0 < nsplit; c0 += U * GC) {
        float4 v[U][HB];
        float w[U][HB];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + u * GC;
#pragma unroll
          for (int hh = 0; hh < HB; ++hh) {
            const int h = h0 + hh;
            const bool live = h < hpk && c < nsplit;
            w[u][hh] = live ? wm[h * nsplit + c] : 0.f;
            v[u][hh] = live ? __ldcg(reinterpret_cast<const float4*>(a.part_acc + ((row0 + h) * S + c) * D) + qd)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int hh = 0; hh < HB; ++hh) {
            acc[hh].x = fmaf(v[u][hh].x, w[u][hh], acc[hh].x);
            acc[hh].y = fmaf(v[u][hh].y, w[u][hh], acc[hh].y);
            acc[hh].z = fmaf(v[u][hh].z, w[u][hh], acc[hh].z);
            acc[hh].w = fmaf(v[u][hh].w, w[u][hh], acc[hh].w);
          }
      }
    } else {
      // Too many splits to stage their weights: recompute them (slower).
      for (int c = cg; c < nsplit; c += GC) {
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
          const int h = h0 + hh;
          if (h >= hpk) break;
          const size_t si = (row0 + h) * S + c;
          const float lc = __ldcg(a.part_l + si);
          const float w = (lc != 0.f && smM[h] != -INFINITY) ? expf(__ldcg(a.part_m + si) - smM[h]) : 0.f;
          if (w == 0.f) continue;
          const float4 vv = __ldcg(reinterpret_cast<const float4*>(a.part_acc + si * D) + qd);
          acc[hh].x = fmaf(vv.x, w, acc[hh].x);
          acc[hh].y = fmaf(vv.y, w, acc[hh].y);
          acc[hh].z = fmaf(vv.z, w, acc[hh].z);
          acc[hh].w = fmaf(vv.w, w, acc[hh].w);
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < HB; ++hh) {
      if (h0 + hh >= hpk) break;
#pragma unroll
      for (int x = 1; x < GC; x <<= 1) {
        acc[hh].x += __shfl_xor_sync(0xffffffffu, acc[hh].x, x);
        acc[hh].y += __shfl_xor_sync(0xffffffffu, acc[hh].y, x);
        acc[hh].z += __shfl_xor_sync(0xffffffffu, acc[hh].z, x);
        acc[hh].w += __shfl_xor_sync(0xffffffffu, acc[hh].w, x);
      }
    }
    if (cg == 0) {
#pragma unroll
      for (int hh = 0; hh < HB; ++hh) {
        const int h = h0 + hh;
        if (h >= hpk) break;
        const size_t r = row0 + h;
        const float wc = smC[h];
        float y[4] = {acc[hh].x, acc[hh].y, acc[hh].z, acc[hh].w};
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

// A segment with one split, finalised by its CTA straight from the per-slot
// states in shared memory (ms, ls [slots][HP] base-2; accs [slots][HP][D + 4]
// rescaled to the tile maximum): store_partial's arithmetic followed by
// merge_segment_smem's for one split and the carry, in the same order, without
// the partial state's store and reload. Run by the 128 threads tid; smW holds
// a per-head weight.
template <int D, int W, int HP, class Sync>
__device__ __forceinline__ void finalize_single_split(const PartitionArgs& a, const Tile& t, const float* ms,
                                                      const float* ls, const float* accs, int nslots, int tid,
                                                      float* smM, float* smL, float* smC, float* smW, Sync sync) {
  constexpr int NT = 128, P = D + 4, Q = D / 4, GC = NT / Q;
  const int hpk = a.hpk;
  const size_t row0 = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * hpk;
  for (int h = tid; h < hpk; h += NT) {
    // the tile's state, as store_partial forms it
    float Mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < W + 1; ++w)
      if (w < nslots) Mt = fmaxf(Mt, ms[w * HP + h]);
    const float Mu = (Mt == -INFINITY) ? 0.f : Mt;
    float Lt = 0.f;
#pragma unroll
    for (int w = 0; w < W + 1; ++w)
      if (w < nslots) Lt += ls[w * HP + h] * exp2f(ms[w * HP + h] - Mu);
    const float mt = (Lt == 0.f) ? -INFINITY : Mt * kLn2;
    // one split and the carry, as merge_segment_smem folds them
    const size_t r = row0 + h;
    float M = (Lt != 0.f) ? mt : -INFINITY;
    const bool has_carry = a.cl != nullptr && a.cl[r] != 0.f;
    if (has_carry) M = fmaxf(M, a.cm[r]);
    const float wt = (Lt != 0.f && M != -INFINITY) ? expf(mt - M) : 0.f;
    float L = fmaf(Lt, wt, 0.f);
    float wc = 0.f;
    if (has_carry) {
      wc = expf(a.cm[r] - M);
      L = fmaf(a.cl[r], wc, L);
    }
    smM[h] = M;
    smL[h] = L;
    smC[h] = wc;
    smW[h] = wt;
  }
  sync();
  const int qd = tid % Q, hg = tid / Q;
  for (int h = hg; h < hpk; h += GC) {
    const size_t r = row0 + h;
    float sv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < W + 1; ++w)
        if (w < nslots) acc += accs[(w * HP + h) * P + qd * 4 + e];
      sv[e] = acc;
    }
    const float wt = smW[h];
    float4 y = make_float4(fmaf(sv[0], wt, 0.f), fmaf(sv[1], wt, 0.f), fmaf(sv[2], wt, 0.f), fmaf(sv[3], wt, 0.f));
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
  // m and l of the state out after every thread has read the carry (state out
  // may alias it)
  sync();
  if (a.om)
    for (int h = tid; h < hpk; h += NT) {
      a.om[row0 + h] = (smL[h] == 0.f) ? -INFINITY : smM[h];
      a.ol[row0 + h] = smL[h];
    }
}

// After the CTA's partial state is stored: take a ticket on the segment and,
// if this CTA completed it, merge. All participating threads call this.
// `aborted` (a tile whose pipeline gave up, with GQA_ERR_TIMEOUT already set):
// the ticket is still taken, and the counter still reset by the last CTA, but
// an aborted CTA merges nothing.
template <int D, int HP, class Sync>
__device__ __forceinline__ void finish_segment(const PartitionArgs& a, const Tile& t, int tid,
                                               float* smM, float* smL, float* smC, int* smFlag,
                                               float* wts, int wcap, uint32_t bulk_bar, Sync sync,
                                               bool aborted = false) {
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
      *smFlag = last && !aborted;
    }
    sync();
    if (!*smFlag) return;
  } else {
    sync();                     // a single split: the CTA merges its own partial
    if (aborted) return;
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

}  // namespace gqa
