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
constexpr int kCodedThreads = 512;     // threads of a coded-kernel CTA (one CTA per SM)
// Largest heads_per_kv * n_atoms: three tables of that many words (logits,
// value weights, the round's integer weights) in shared memory.
constexpr int kCodedMaxTableEntries = 12288;
// Dynamic shared memory budget of the coded kernel (under the 227 KB a CTA may
// hold, with room for its static shared memory).
constexpr int kCodedSmemBudget = 212 * 1024;
// 128 bytes of alignment slack, then a 256-byte header (mbarriers)
constexpr int kCodedFixedBytes = 384;
constexpr int kCodedMaxRoundKeys = 8192;

// Shared memory plan of the coded kernel, the same on host and device. In
// words, after the header:
//   ring    P x W x 512: a thread's next P code rows (P = 4, 2 or 1, as many
//           as fit with a round of 512 keys);
//   round   KR x (hpk + 1): the round's logits and |V coefficient| sums, KR
//           keys, a multiple of 512, at most 8192, as many as fit. The round
//           region also stages atom rows;
//   tables  3 x hpk x n_atoms: logit table, value weights, round weights.
__host__ __device__ constexpr int coded_table_words(int hpk, int n_atoms) { return 3 * hpk * n_atoms; }
__host__ __device__ constexpr int coded_free_words() { return (kCodedSmemBudget - kCodedFixedBytes) / 4; }
// words of the round region per key: its logits and its |V coefficient| sum
__host__ __device__ constexpr int coded_key_words(int hpk) { return hpk + 1; }
__host__ __device__ constexpr bool coded_ring_fits(int rows, int words, int hpk, int n_atoms) {
  return rows * words * kCodedThreads + kCodedThreads * coded_key_words(hpk) +
             coded_table_words(hpk, n_atoms) <=
         coded_free_words();
}
__host__ __device__ constexpr int coded_ring_rows(int words, int hpk, int n_atoms) {
  return coded_ring_fits(4, words, hpk, n_atoms)   ? 4
         : coded_ring_fits(2, words, hpk, n_atoms) ? 2
                                                   : 1;
}
__host__ __device__ constexpr int coded_round_keys_uncapped(int words, int hpk, int n_atoms) {
  return (coded_free_words() - coded_ring_rows(words, hpk, n_atoms) * words * kCodedThreads -
          coded_table_words(hpk, n_atoms)) / coded_key_words(hpk) / kCodedThreads * kCodedThreads;
}
__host__ __device__ constexpr int coded_round_keys(int words, int hpk, int n_atoms) {
  return coded_round_keys_uncapped(words, hpk, n_atoms) > kCodedMaxRoundKeys
             ? kCodedMaxRoundKeys
             : coded_round_keys_uncapped(words, hpk, n_atoms);
}
__host__ __device__ constexpr size_t coded_smem_bytes(int words, int hpk, int n_atoms) {
  return kCodedFixedBytes +
         4 * (static_cast<size_t>(coded_ring_rows(words, hpk, n_atoms)) * words * kCodedThreads +
              static_cast<size_t>(coded_round_keys(words, hpk, n_atoms)) * coded_key_words(hpk) +
              coded_table_words(hpk, n_atoms));
}

__device__ __forceinline__ float code_coeff(uint32_t word) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(word & 0xFFFFu)));
}

// Fixed-point scale of one head's value weights in a round of keys. The
// weights of any atom sum, in absolute value, to at most bound = sum_j p_j
// sum_w |c_jw| over the round's keys, so weights scaled by 2^e with
// bound * 2^e <= 2^30 (and each rounded by at most 1/2) sum without overflow
// in 32-bit integers. The chosen e puts bound * 2^e in (2^29, 2^30], so the
// rounding error of a weight (half a unit, 2^-e / 2) stays below 2^-30 * bound.
__device__ __forceinline__ float round_weight_scale(float bound) {
  if (!(bound > 0.f)) return 1073741824.f;                   // no weight this round (or NaN)
  if (!(bound < INFINITY)) return 0.f;
  // ceil(log2(bound)) from the bits: the exponent, plus one unless a power of 2
  const int bits = __float_as_int(bound);
  int cl = ((bits >> 23) & 0xFF) - 127 + ((bits & 0x7FFFFF) != 0 ? 1 : 0);
  if ((bits >> 23) == 0) cl = -126;                          // subnormal: below 2^-126
  const int e = max(-126, min(30, 30 - cl));
  return __int_as_float((e + 127) << 23);                     // 2^e
}

// Per head h < hpk (unrolled up to HMAX): reduce v[h][w] over the NW warps
// of the CTA with op, in a fixed order (lane w holds warp w's value, then a
// butterfly), so every thread gets the same result.
template <int HMAX, int NW, class Op>
__device__ __forceinline__ void cta_reduce_heads(const float (*v)[NW], int hpk, int lane, float init,
                                                 float (&out)[HMAX], Op op) {
  static_assert(NW <= 32, "one lane per warp");
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    if (h >= hpk) break;
    float x = lane < NW ? v[h][lane] : init;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = op(x, __shfl_xor_sync(0xffffffffu, x, o));
    out[h] = x;
  }
}

// Decode attention straight from the codes, never rebuilding a row:
//   q.K_j = sum_w c_jw (q . katom[i_jw])  -- a table qa[atom][h] of the CTA's
//     query heads against every K atom, built once per CTA, then lookups;
//   sum_j p_j V_j = sum_atom (sum_{j,w: i'_jw = atom} p_j c'_jw) vatom[atom]
//     -- per-atom weights Wt[h][atom], multiplied by the V atoms once at the end.
// One CTA of 512 threads per SM. Atom rows come into shared memory by TMA bulk
// copies, two chunks in flight, for the logit table (warps take atoms, lanes
// across D, a warp reduce-scatter sums the partial dot products) and for the
// value epilogue (threads own 4 columns of up to 4 heads for a share of the
// atoms, then the shares add in a fixed order).
// Keys go in rounds of KR (a multiple of 512); thread tid takes keys tid, tid
// + 512, ... of a round. Code rows pass through a P-row ring by cp.async, each
// warp copying its 32 keys' rows together in whole 32-byte sectors into its
// own part of a slot (the next pass's first rows are issued before each
// barrier, so they run across it). Per round, two passes and one barrier
// between them:
//   A. the K and V rows of each key in turn: logits by table lookups into the
//      round's logit store, each key's sum of |V coefficient|, and the
//      thread's maxima per head; then, out of its own keys' entries of the
//      store, its share of the bound sum_j p_j sum_w |c'_jw| on any atom's
//      weight sum, relative to its own maxima. The warps combine (maximum,
//      bound) pairs -> barrier;
//   C. the new running maximum and the round's bound relative to it; each
//      key's weights p, the partition, and every weight p * c' added to the
//      integer table Wb in fixed point, scaled by a power of two that keeps
//      the bound below 2^30 (32-bit shared atomics, which B200 runs several
//      times faster than float ones, and whose sums do not depend on their
//      order).
// After a barrier each thread folds its atoms of Wb into the value weights Wt,
// both rescaled to the new running maximum, and clears them.
// Cross-warp maxima and sums go through a fixed-order lane butterfly, so the
// results are bit-reproducible. A segment with one split (the tile is the
// whole sequence) folds the carry and writes out / state_out directly; others
// go through the same partial states and fused merge as the other partition
// kernels. HMAX: a compile-time bound on heads_per_kv (4, 8 or 16); MW: on
// the words per row (4, 8 or 16); EXACT: the rows have exactly MW words and
// heads_per_kv is HMAX, so that both counts and everything derived from them
// are constants.
template <int D, int HMAX, int MW, bool EXACT = false>
__global__ void __launch_bounds__(kCodedThreads, 1)
gqa_partition_coded_kernel(const PartitionArgs a, const CodedArgs c) {
  static_assert(MW == 4 || MW == 8 || MW == 16, "words bound 4, 8 or 16");
  constexpr int NT = kCodedThreads, NW = NT / 32, E = D / 32;
  extern __shared__ uint8_t dsm_raw[];
  // aligned by an offset from the array itself, so that every access through
  // these pointers stays a shared-memory access for the compiler
  uint32_t* dsm = reinterpret_cast<uint32_t*>(dsm_raw + ((128u - (ptx::smem_u32(dsm_raw) & 127u)) & 127u));
  __shared__ float red[HMAX][NW];        // per head, per warp: maxima (then partitions)
  __shared__ float red2[HMAX][NW];       // per head, per warp: weight bounds
  __shared__ float smM[16], smL[16], smC[16];
  __shared__ float hM[16], hL[16];       // per head: base-2 running maximum, partition
  // Above 8 heads the per-head values every thread shares (running maximum,
  // the round's weight maximum, scale and rescale factor) live here, set by
  // one thread per head, instead of in every thread's registers.
  constexpr bool SH = HMAX > 8;
  __shared__ float cM[HMAX], cMn[HMAX], cSc[HMAX], cFr[HMAX];
  __shared__ int smFlag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hpk = EXACT ? HMAX : a.hpk, NA = c.n_atoms, W = EXACT ? MW : c.words;
  const int P = coded_ring_rows(W, hpk, NA);
  const int KR = coded_round_keys(W, hpk, NA);
  const uint32_t bar0 = ptx::smem_u32(dsm);                    // atom copies into buffer 0 / 1
  const uint32_t bar1 = bar0 + 8;
  uint32_t* ring = dsm + 64;                                   // [P][W or W/4 quads][NT] K rows
  float* lg = reinterpret_cast<float*>(ring + P * W * NT);    // [KR][hpk] logits
  float* cs = lg + KR * hpk;                                   // [KR] sums of |V coefficient|
  float* qa = cs + KR;                                         // [NA][hpk] logits (base 2)
  float* Wt = qa + hpk * NA;                                   // [hpk][NA] value weights
  uint32_t* Wb = reinterpret_cast<uint32_t*>(Wt + hpk * NA);   // [hpk][NA] round weights, fixed point

  const Tile t = tile_of(a, blockIdx.x);
  ptx::grid_dependency_wait();
  if (t.kbeg >= t.kend) {
    if (a.write_empty) write_empty_states<D>(a, t);
    if (a.merge && t.n == 0 && t.c == 0 && tid < 128)
      merge_segment<D, HMAX>(a, t, 0, tid, smM, smL, smC, qa, hpk * NA, NamedSync128{});
    return;
  }
  if (tid == 0) {
    ptx::mbar_init(bar0, 1);
    ptx::mbar_init(bar1, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const bool quads = (W & 3) == 0;
  const int nround = (t.kend - t.kbeg + KR - 1) / KR;
  const size_t row_stride = static_cast<size_t>(a.G) * W;
  const uint32_t* kbase = c.k_codes + (static_cast<size_t>(t.o0) * a.G + t.g) * W;
  const uint32_t* vbase = c.v_codes + (static_cast<size_t>(t.o0) * a.G + t.g) * W;
  auto round_keys = [&](int rd) { return min(KR, t.kend - t.kbeg - rd * KR); };
  // keys of a round in warp w's rows: tid + i * NT for i < rows_of(nk), the
  // count of the warp's lane 0 (the most in the warp), so that loops over a
  // warp's rows run the same count in every lane; a lane whose key is past the
  // round (j >= nk) takes part in the copies and warp syncs and nothing else
  auto rows_of = [&](int nk) { return nk > warp * 32 ? (nk - warp * 32 + NT - 1) / NT : 0; };

  // ---- code rows: a stream of rows through the ring's P slots, one commit
  // group per row (empty past the stream's end), row n of a stream in slot
  // n % P. Pass A's stream is the K and V rows of the thread's keys in turn
  // (K, V of key tid, then of key tid + NT, ...), pass C's its V rows. Each
  // warp's part of a slot holds its 32 keys' rows ([32][W] words), copied by
  // the lanes together: 16-byte units u = lane + 32 k (quad u % QR of row
  // u / QR, QR = W / 4), so that a copy instruction reads whole 32-byte
  // sectors; quad q of row r sits at q ^ ((r >> s) & (QR - 1)) when QR is a
  // power of two (8 >> s = 8 / QR rows a 128-byte line), which keeps each lane's
  // reads of its own row free of bank conflicts. Rows of W not a multiple of
  // 4 are copied word by word, each lane its own. A warp sync after the wait
  // makes the lanes' copies visible to the warp, and one before each copy
  // keeps it off a row that a lane still reads.
  const uint32_t ring_u32 = ptx::smem_u32(ring);
  const int QR = W / 4;
  const bool qswz = quads && (QR & (QR - 1)) == 0;
  const int qsh = QR == 4 ? 1 : (QR == 2 ? 2 : 3);
  auto qpos = [&](int q, int r) { return qswz ? (q ^ ((r >> qsh) & (QR - 1))) : q; };
  int u_row[MW / 4], u_src[MW / 4], u_dst[MW / 4];   // this lane's units: row, source and slot words
#pragma unroll
  for (int k = 0; k < MW / 4; ++k) {
    const int u = lane + 32 * k;
    u_row[k] = quads ? u / max(QR, 1) : 32;
    const int q = quads ? u % max(QR, 1) : 0;
    u_src[k] = u_row[k] * static_cast<int>(a.G) * W + 4 * q;
    u_dst[k] = u_row[k] * W + 4 * qpos(q, u_row[k]);
  }
  // row n of the round starting at key kb with nk keys: pass A (two rows a
  // key) or pass C (V rows)
  auto issue = [&](bool pass_a, int kb, int nk, int n) {
    __syncwarp();
    const int i = pass_a ? n >> 1 : n;
    const int j0 = warp * 32 + i * NT;             // the warp's first key of the step
    if (j0 < nk) {
      const uint32_t dst = ring_u32 + ((n % P) * NW + warp) * 32 * W * 4;
      const uint32_t* src = ((pass_a && (n & 1) == 0) ? kbase : vbase) + static_cast<size_t>(kb + j0) * row_stride;
      if (quads) {
#pragma unroll
        for (int k = 0; k < MW / 4; ++k)
          if (k < QR && j0 + u_row[k] < nk) ptx::cp_async_16(dst + u_dst[k] * 4, src + u_src[k]);
      } else if (j0 + lane < nk) {
        for (int w = 0; w < W; ++w) ptx::cp_async_4(dst + (lane * W + w) * 4, src + lane * row_stride + w);
      }
    }
    ptx::cp_async_commit();
  };
  auto prime = [&](bool pass_a, int kb, int nk) {
    for (int n = 0; n < P; ++n) issue(pass_a, kb, nk, n);
  };
  auto fetch = [&](int n, uint32_t (&r)[MW]) {   // wait for row n, read this lane's
    if (P >= 4)
      ptx::cp_async_wait_group<3>();
    else if (P == 2)
      ptx::cp_async_wait_group<1>();
    else
      ptx::cp_async_wait_group<0>();
    __syncwarp();
    const uint32_t* row = ring + ((n % P) * NW + warp) * 32 * W + lane * W;
    if (quads) {
#pragma unroll
      for (int q = 0; q < MW / 4; ++q) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (q < QR) v = reinterpret_cast<const uint4*>(row)[qpos(q, lane)];
        r[4 * q] = v.x;
        r[4 * q + 1] = v.y;
        r[4 * q + 2] = v.z;
        r[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int w = 0; w < MW; ++w) r[w] = w < W ? row[w] : 0u;
    }
  };
  // ---- atom rows: chunks of `chunk` atoms through two buffers in the logit
  // store region, by bulk copies completing on bar0 / bar1. A chunk's copy is
  // issued once every thread is done with the buffer (a barrier, and a proxy
  // fence for the generic accesses before it); a wait that gives up flags
  // GQA_ERR_TIMEOUT, lets the copy land (bounded) and turns `ok` false in every
  // thread (a vote).
  uint32_t phase0 = 0u, phase1 = 0u;
  float* abuf = lg;
  const int region = KR * (hpk + 1);                  // words of lg + cs (free outside rounds)
  const int vwords = P * W * NT + KR * coded_key_words(hpk);   // ring + round region: V atom staging
  auto issue_atoms = [&](const float* atoms, int a0, int n, int b, float* base) {
    if (tid == 0 && n > 0) {
      const uint32_t bb = b ? bar1 : bar0;
      ptx::mbar_arrive_expect_tx(bb, static_cast<uint32_t>(n) * D * 4);
      ptx::bulk_load_1d(ptx::smem_u32(base), atoms + static_cast<size_t>(a0) * D, static_cast<uint32_t>(n) * D * 4, bb);
    }
  };
  auto wait_atoms = [&](int b) -> bool {
    const uint32_t bb = b ? bar1 : bar0;
    const uint32_t ph = b ? phase1 : phase0;
    const bool landed = ptx::mbar_wait_bounded(bb, ph, nullptr, kWaitLimitNs);
    const bool all = __syncthreads_and(landed) != 0;
    if (!all) {
      if (tid == 0) atomicOr(a.err, kErrTimeout);
      if (!landed) ptx::mbar_wait_bounded(bb, ph, nullptr, kWaitLimitNs);
    }
    if (b)
      phase1 ^= 1u;
    else
      phase0 ^= 1u;
    return all;
  };
  // Run body(chunk start, count, rows) over all atoms of `atoms`, two chunks in flight.
  bool ok = true;
  // Atoms per buffer: as many as half the words hold, a multiple of 128 when
  // that many fit (the table's 16 warps take 8 atoms a step, so a chunk of
  // 130 would leave one warp a second step for 2 atoms).
  auto atoms_per_chunk = [&](int words) {
    const int n = words / 2 / D;
    return n >= 128 ? n / 128 * 128 : n;
  };
  // The first two chunks' copies (thread 0), into buffers nobody uses any more.
  auto start_atoms = [&](const float* atoms, float* base, int words) {
    const int chunk = atoms_per_chunk(words);
    issue_atoms(atoms, 0, min(chunk, NA), 0, base);
    if (NA > chunk) issue_atoms(atoms, chunk, min(chunk, NA - chunk), 1, base + static_cast<size_t>(chunk) * D);
  };
  // started: start_atoms has run already (else every thread's accesses to the
  // buffers are fenced and waited for here first)
  auto over_atoms = [&](const float* atoms, float* base, int words, bool started, auto&& body) {
    const int chunk = atoms_per_chunk(words);           // atoms per buffer
    float* const buf1 = base + static_cast<size_t>(chunk) * D;
    const int nchunk = (NA + chunk - 1) / chunk;
    if (!started) {
      ptx::fence_proxy_async_smem();
      __syncthreads();
      start_atoms(atoms, base, words);
    }
    for (int k = 0; k < nchunk && ok; ++k) {
      const int b = k & 1;
      float* const bufk = b ? buf1 : base;
      ok = wait_atoms(b);
      if (!ok) break;
      body(k * chunk, min(chunk, NA - k * chunk), bufk);
      if (k + 2 < nchunk) {
        ptx::fence_proxy_async_smem();
        __syncthreads();                               // buffer b read by everyone
        issue_atoms(atoms, (k + 2) * chunk, min(chunk, NA - (k + 2) * chunk), b, bufk);
      }
    }
  };

  // The logit table's first atom rows are on their way (the logit store is
  // untouched so far) before the first code rows are requested.
  start_atoms(c.k_atoms, abuf, region);
  // the first two rows before the table, the rest after it: issuing copies
  // holds a warp, and the table should start as soon as its atoms land
  const int early_rows = P < 2 ? P : 2;
  if (nround > 0)
    for (int n = 0; n < early_rows; ++n) issue(true, t.kbeg, round_keys(0), n);
  for (int i = tid; i < hpk * NA; i += NT) {
    Wt[i] = 0.f;
    Wb[i] = 0u;
  }
  // the logit table, HT heads at a time (at most 8, for registers): a warp
  // takes A = 32 / HT atoms per pass, lanes across D (the rows out of shared
  // memory). Each lane's A x HT partial dot products are summed across the
  // warp by a reduce-scatter: at each of 5 steps a lane keeps half of its
  // values and adds the other half from the lane `off` away, so lane L ends
  // with atom L / HT, head L % HT of the pass.
  {
    constexpr int HT = HMAX > 8 ? 8 : HMAX;
    constexpr int A = 32 / HT;
    const size_t qrow = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * hpk;
    // this lane's columns of HT query heads from h0; the first HT are loaded
    // before the atom copies are waited for, and kept when they are all
    float qreg[HT][E];
    auto load_q = [&](int h0) {
#pragma unroll
      for (int h = 0; h < HT; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const size_t qi = (qrow + h0 + h) * D + lane * E + e;
          qreg[h][e] = h0 + h >= hpk ? 0.f
                       : c.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qi])
                                  : static_cast<const float*>(a.q)[qi];
        }
    };
    load_q(0);
    over_atoms(c.k_atoms, abuf, region, true, [&](int c0, int n, const float* rows) {
#pragma unroll 1
      for (int h0 = 0; h0 < hpk; h0 += HT) {
        if (hpk > HT) load_q(h0);
        for (int a0 = warp * A; a0 < n; a0 += NW * A) {
          float v[32];
#pragma unroll
          for (int i = 0; i < A; ++i) {
            const int at = a0 + i;
            float kv[E];
            if (E == 4) {
              const float4 k4 = at < n ? *reinterpret_cast<const float4*>(rows + at * D + lane * 4)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
              kv[0] = k4.x;
              kv[1 % E] = k4.y;
              kv[2 % E] = k4.z;
              kv[3 % E] = k4.w;
            } else {
#pragma unroll
              for (int e = 0; e < E; ++e) kv[e] = at < n ? rows[at * D + lane * E + e] : 0.f;
            }
#pragma unroll
            for (int h = 0; h < HT; ++h) {
              float d = 0.f;
#pragma unroll
              for (int e = 0; e < E; ++e) d = fmaf(qreg[h][e], kv[e], d);
              v[i * HT + h] = d;
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
          const int at = a0 + lane / HT, h = h0 + lane % HT;
          if (at < n && h < hpk) qa[(c0 + at) * hpk + h] = v[0] * a.scale_log2;
        }
      }
    });
  }
  if (nround > 0)
    for (int n = early_rows; n < P; ++n) issue(true, t.kbeg, round_keys(0), n);
  __syncthreads();                   // the table is complete; the logit store is free

  // Running maximum per head (identical in every thread) and this thread's
  // share of the partition. Per round, one barrier between the passes:
  //   A. K rows: logits by table lookup into lg[key][h] and this thread's
  //      maxima; V rows: the sum of |coefficient| of each key into cs. Then,
  //      from its own keys in shared memory, the thread's share of the bound
  //      sum_j p_j sum_w |c'_jw| relative to its own maxima. Warps combine
  //      (maximum, bound) pairs -> barrier;
  //   C. the round's maximum and bound from the warps' pairs in a fixed order;
  //      weights p, the partition, and the weights into Wb in fixed point.
  // After a barrier, each thread folds its atoms of Wb into Wt (both rescaled
  // to the new running maximum) and clears them.
  float mrun[HMAX], lthr[HMAX];
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    mrun[h] = -INFINITY;
    lthr[h] = 0.f;
  }
  if (SH && tid < HMAX) cM[tid] = -INFINITY;   // read after the first round's barrier
  // (maximum, bound) pairs: the bound rescaled to the larger maximum; the
  // combination is symmetric, so a butterfly leaves the same bits in every lane
  auto pair_combine = [](float& m, float& s, float m2, float s2) {
    const float mm = fmaxf(m, m2);
    const float a = m == -INFINITY ? 0.f : s * exp2f(m - mm);
    const float b = m2 == -INFINITY ? 0.f : s2 * exp2f(m2 - mm);
    m = mm;
    s = a + b;
  };
  auto fadd_op = [](float x, float y) { return x + y; };
  bool bad = false;
  const bool quad_heads = (hpk & 3) == 0;
  auto load_heads = [&](const float* src, float (&x)[HMAX]) {
    if (quad_heads) {
#pragma unroll
      for (int q4 = 0; q4 < HMAX / 4; ++q4)
        if (4 * q4 < hpk) {
          const float4 t4 = *reinterpret_cast<const float4*>(src + 4 * q4);
          x[4 * q4] = t4.x;
          x[4 * q4 + 1] = t4.y;
          x[4 * q4 + 2] = t4.z;
          x[4 * q4 + 3] = t4.w;
        }
    } else {
#pragma unroll
      for (int h = 0; h < HMAX; ++h)
        if (h < hpk) x[h] = src[h];
    }
  };
#pragma unroll 1
  for (int rd = 0; rd < nround && ok; ++rd) {
    const int kb = t.kbeg + rd * KR;
    const int nk = round_keys(rd);
    const int mine = rows_of(nk);
    // ---- pass A
    float tmax[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) tmax[h] = -INFINITY;
#pragma unroll 1
    for (int i = 0; i < mine; ++i) {
      const int j = tid + i * NT;
      const bool live = j < nk;
      uint32_t kw[MW];
      fetch(2 * i, kw);
      float s[HMAX];
#pragma unroll
      for (int h = 0; h < HMAX; ++h) s[h] = 0.f;
#pragma unroll
      for (int w = 0; w < MW; ++w) {
        const int idx = static_cast<int>(kw[w] >> 16);
        const bool in = idx < NA;
        bad |= live && !in;
        const float cf = in ? code_coeff(kw[w]) : 0.f;
        // an atom's logits of all heads sit side by side: 16-byte loads when
        // heads_per_kv is a multiple of 4
        const float* row = qa + (in ? idx : 0) * hpk;
        if (quad_heads) {
#pragma unroll
          for (int q4 = 0; q4 < HMAX / 4; ++q4)
            if (4 * q4 < hpk) {
              const float4 t4 = *reinterpret_cast<const float4*>(row + 4 * q4);
              s[4 * q4] = fmaf(cf, t4.x, s[4 * q4]);
              s[4 * q4 + 1] = fmaf(cf, t4.y, s[4 * q4 + 1]);
              s[4 * q4 + 2] = fmaf(cf, t4.z, s[4 * q4 + 2]);
              s[4 * q4 + 3] = fmaf(cf, t4.w, s[4 * q4 + 3]);
            }
        } else {
#pragma unroll
          for (int h = 0; h < HMAX; ++h)
            if (h < hpk) s[h] = fmaf(cf, row[h], s[h]);
        }
      }
      issue(true, kb, nk, 2 * i + P);            // the K row's slot is free
      uint32_t vw[MW];
      fetch(2 * i + 1, vw);
      float csum = 0.f;                          // sum of |V coefficient| of the key
#pragma unroll
      for (int w = 0; w < MW; ++w) csum += fabsf(code_coeff(vw[w]));
      issue(true, kb, nk, 2 * i + 1 + P);        // the V row's slot is free
      if (!live) continue;
      cs[j] = csum;
      const float bb = bias2(a, t, kb + j);
      float* dst = lg + j * hpk;
      if (quad_heads) {
#pragma unroll
        for (int q4 = 0; q4 < HMAX / 4; ++q4)
          if (4 * q4 < hpk)
            *reinterpret_cast<float4*>(dst + 4 * q4) =
                make_float4(s[4 * q4] + bb, s[4 * q4 + 1] + bb, s[4 * q4 + 2] + bb, s[4 * q4 + 3] + bb);
      } else {
#pragma unroll
        for (int h = 0; h < HMAX; ++h)
          if (h < hpk) dst[h] = s[h] + bb;
      }
#pragma unroll
      for (int h = 0; h < HMAX; ++h) tmax[h] = fmaxf(tmax[h], s[h] + bb);
    }
    prime(false, kb, nk);            // pass C's V rows come in across the barrier
    // this thread's bound relative to its own maxima, from its keys' logits
    // and coefficient sums (no copy involved)
    float tb[HMAX];
#pragma unroll
    for (int h = 0; h < HMAX; ++h) tb[h] = 0.f;
#pragma unroll 2
    for (int i = 0; i < mine; ++i) {
      const int j = tid + i * NT;
      if (j >= nk) break;
      float l[HMAX];
      load_heads(lg + j * hpk, l);
      const float c = cs[j];
#pragma unroll
      for (int h = 0; h < HMAX; ++h)
        if (h < hpk && tmax[h] != -INFINITY) tb[h] = fmaf(exp2f(l[h] - tmax[h]), c, tb[h]);
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
      float m = tmax[h], sb = tb[h];
#pragma unroll
      for (int x = 16; x >= 1; x >>= 1)
        pair_combine(m, sb, __shfl_xor_sync(0xffffffffu, m, x), __shfl_xor_sync(0xffffffffu, sb, x));
      if (lane == 0) {
        red[h][warp] = m;
        red2[h][warp] = sb;
      }
    }
    __syncthreads();                 // red, red2 complete
    // ---- pass C
    float mn[HMAX], scale[HMAX], fr[HMAX];
    if (SH) {
      // thread h combines head h's pairs over the warps in order
      if (tid < hpk) {
        const int h = tid;
        float m = red[h][0], sb = red2[h][0];
        for (int w = 1; w < NW; ++w) pair_combine(m, sb, red[h][w], red2[h][w]);
        const float mold = cM[h];
        const float mnew = fmaxf(mold, m);
        cFr[h] = (mnew == -INFINITY) ? 1.f : exp2f(mold - mnew);
        cM[h] = mnew;
        cSc[h] = round_weight_scale(m == -INFINITY ? 0.f : sb * exp2f(m - mnew));
        cMn[h] = mnew == -INFINITY ? 0.f : mnew;
      }
      __syncthreads();               // cFr, cSc, cMn set
#pragma unroll
      for (int h = 0; h < HMAX; ++h)
        if (h < hpk) lthr[h] *= cFr[h];
    }
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (SH) break;
      mn[h] = 0.f;
      scale[h] = 0.f;
      fr[h] = 1.f;
      if (h >= hpk) continue;
      float m = lane < NW ? red[h][lane] : -INFINITY;
      float sb = lane < NW ? red2[h][lane] : 0.f;
#pragma unroll
      for (int x = 16; x >= 1; x >>= 1)
        pair_combine(m, sb, __shfl_xor_sync(0xffffffffu, m, x), __shfl_xor_sync(0xffffffffu, sb, x));
      const float mnew = fmaxf(mrun[h], m);
      fr[h] = (mnew == -INFINITY) ? 1.f : exp2f(mrun[h] - mnew);
      mrun[h] = mnew;
      lthr[h] *= fr[h];
      // weights relative to the running maximum are at most those relative
      // to the round's, so the round's bound still bounds them
      scale[h] = round_weight_scale(m == -INFINITY ? 0.f : sb * exp2f(m - mnew));
      mn[h] = mnew == -INFINITY ? 0.f : mnew;    // all masked so far: weights 0
    }
#pragma unroll 1
    for (int i = 0; i < mine; ++i) {
      const int j = tid + i * NT;
      uint32_t vw[MW];
      fetch(i, vw);
      if (j >= nk) {                 // past the round: the warp's copies and syncs only
        issue(false, kb, nk, i + P);
        continue;
      }
      float l[HMAX], ps[HMAX];       // weights in fixed-point units
      load_heads(lg + j * hpk, l);
#pragma unroll
      for (int h = 0; h < HMAX; ++h) {
        ps[h] = 0.f;
        if (h < hpk) {
          const float p = exp2f(l[h] - (SH ? cMn[h] : mn[h]));
          lthr[h] += p;
          ps[h] = p * (SH ? cSc[h] : scale[h]);
        }
      }
      // every word adds its weights, zero ones included (no branch); an index
      // out of range is flagged and adds zeros to atom 0
#pragma unroll
      for (int w = 0; w < MW; ++w) {
        if (w >= W) break;
        const int idx = static_cast<int>(vw[w] >> 16);
        const bool in = idx < NA;
        bad |= !in;
        const float cf = in ? code_coeff(vw[w]) : 0.f;
        uint32_t* wrow = Wb + (in ? idx : 0);
#pragma unroll
        for (int h = 0; h < HMAX; ++h)
          if (h < hpk) atomicAdd(wrow + h * NA, static_cast<uint32_t>(__float2int_rn(ps[h] * cf)));
      }
      issue(false, kb, nk, i + P);
    }
    // the next round's rows start coming in across the barrier; after the
    // last round, the V atoms' first chunks do (ring and store are free then)
    if (rd + 1 < nround)
      prime(true, kb + KR, round_keys(rd + 1));
    else
      ptx::fence_proxy_async_smem();
    __syncthreads();                 // the round's atomics done
    if (rd + 1 == nround) start_atoms(c.v_atoms, reinterpret_cast<float*>(ring), vwords);
    // fold: Wt and Wb relative to the new running maximum; Wb cleared
#pragma unroll
    for (int h = 0; h < HMAX; ++h) {
      if (h >= hpk) break;
      const float sch = SH ? cSc[h] : scale[h], frh = SH ? cFr[h] : fr[h];
      const float u = sch > 0.f ? 1.f / sch : 0.f;
      for (int i = h * NA + tid; i < (h + 1) * NA; i += NT) {
        Wt[i] = fmaf(Wt[i], frh, static_cast<float>(static_cast<int32_t>(Wb[i])) * u);
        Wb[i] = 0u;
      }
    }
  }
  ptx::cp_async_wait_group<0>();     // no copy left in flight
  // the partition: every thread's share, summed in a fixed order
#pragma unroll
  for (int h = 0; h < HMAX; ++h) {
    if (h >= hpk) break;
    float v = lthr[h];
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) v += __shfl_xor_sync(0xffffffffu, v, x);
    if (lane == 0) red[h][warp] = v;
  }
  __syncthreads();
  {
    float L[HMAX];
    cta_reduce_heads<HMAX, NW>(red, hpk, lane, 0.f, L, fadd_op);
#pragma unroll
    for (int h = 0; h < HMAX; ++h)
      if (h < hpk && tid == h) {
        hM[h] = SH ? cM[h] : mrun[h];
        hL[h] = L[h];
      }
  }
  // (hM, hL are read after the barriers of the atom copies below)
  if (bad) atomicOr(a.err, kErrBadCodes);
  if (threadIdx.x == 0) ptx::grid_launch_dependents();

  // acc[h][d] = sum over atoms of Wt[h][atom] * vatom[atom][d]: the V atoms
  // come through the ring and round region in chunks. Thread tid owns column
  // quad qd = tid % Q of the HG heads hg * HG .. hg * HG + HG - 1 (hg = (tid /
  // Q) % NG) for atom share ag = tid / (Q * NG) (atoms ag, ag + AG, ...): it
  // reads an atom's quad once for its HG heads and sums its atoms in order.
  // Then thread (qd, hg, ag < HG) adds head hg * HG + ag over the AG shares in
  // order.
  constexpr int Q = D / 4;
  constexpr int HG = HMAX < 4 ? HMAX : 4;              // heads per thread
  constexpr int NG = HMAX / HG;                        // head groups
  constexpr int AG = NT / (Q * NG);                    // atom shares: 4 .. 32
  static_assert(Q * NG * AG == NT && AG >= HG, "threads cover quads x head groups x shares");
  // the shares' sums, NT x HG float4, fit the V staging region: it is at least
  // the free words less the largest tables and one 512-key round's rounding
  static_assert(coded_free_words() - 3 * kCodedMaxTableEntries - kCodedThreads * (16 + 1) >= NT * HG * 4,
                "the shares' sums fit the V staging region");
  const int qd = tid % Q, hg = (tid / Q) % NG, ag = tid / (Q * NG);
  float4 acc4[HG];
#pragma unroll
  for (int k = 0; k < HG; ++k) acc4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ok)
    over_atoms(c.v_atoms, reinterpret_cast<float*>(ring), vwords, true,
               [&](int c0, int n, const float* rows) {
                 if (hg * HG < hpk) {
                   const float* wr = Wt + hg * HG * NA + c0;
#pragma unroll 2
                   for (int at = ag; at < n; at += AG) {
                     const float4 vv = *reinterpret_cast<const float4*>(rows + at * D + qd * 4);
#pragma unroll
                     for (int k = 0; k < HG; ++k) {
                       const float wgt = hg * HG + k < hpk ? wr[k * NA + at] : 0.f;
                       acc4[k].x = fmaf(wgt, vv.x, acc4[k].x);
                       acc4[k].y = fmaf(wgt, vv.y, acc4[k].y);
                       acc4[k].z = fmaf(wgt, vv.z, acc4[k].z);
                       acc4[k].w = fmaf(wgt, vv.w, acc4[k].w);
                     }
                   }
                 }
               });
  if (!ok) return;                   // a copy never landed (flagged): no state out
  __syncthreads();                   // the atom buffers are free
  float4* sh = reinterpret_cast<float4*>(ring);        // [AG][NG][HG][Q]
#pragma unroll
  for (int k = 0; k < HG; ++k) sh[((ag * NG + hg) * HG + k) * Q + qd] = acc4[k];
  __syncthreads();
  const int hh = hg * HG + ag;                          // this thread's head of the sum (ag < HG)
  const bool owner = ag < HG && hh < hpk;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (owner)
    for (int g2 = 0; g2 < AG; ++g2) {
      const float4 o = sh[((g2 * NG + hg) * HG + ag) * Q + qd];
      acc.x += o.x;
      acc.y += o.y;
      acc.z += o.z;
      acc.w += o.w;
    }

  // The state goes out as store_partial writes a single slot (m in natural-log units).
  if (owner) *reinterpret_cast<float4*>(a.part_acc + state_index(a, t, hh) * D + qd * 4) = acc;
  if (tid < hpk) {
    const size_t si = state_index(a, t, tid);
    a.part_m[si] = (hL[tid] == 0.f) ? -INFINITY : hM[tid] * kLn2;
    a.part_l[si] = hL[tid];
  }
  if (!a.merge) return;
  if (t.kbeg == 0 && t.kend == t.n) {
    // The tile is the whole sequence: fold the carry (USearch linear algebra,
    // DenseAttendConfig::carry) and write out / state_out from here.
    const size_t row0 = static_cast<size_t>(t.b) * a.H + static_cast<size_t>(t.g) * hpk;
    if (owner) {
      const size_t r = row0 + hh;
      const float Lh = hL[hh];
      float Mh = Lh == 0.f ? -INFINITY : hM[hh] * kLn2;
      const bool has_carry = a.cl != nullptr && a.cl[r] != 0.f;
      float wt = Lh == 0.f ? 0.f : 1.f, wc = 0.f;
      if (has_carry) {
        const float cmr = a.cm[r];
        const float M = fmaxf(Mh, cmr);
        wt = Lh == 0.f ? 0.f : expf(Mh - M);
        wc = expf(cmr - M);
        Mh = M;
      }
      const float Lt = fmaf(Lh, wt, has_carry ? a.cl[r] * wc : 0.f);
      float y[4] = {acc.x * wt, acc.y * wt, acc.z * wt, acc.w * wt};
      if (has_carry) {
        const float4 cv = *reinterpret_cast<const float4*>(a.cacc + r * D + qd * 4);
        y[0] = fmaf(cv.x, wc, y[0]);
        y[1] = fmaf(cv.y, wc, y[1]);
        y[2] = fmaf(cv.z, wc, y[2]);
        y[3] = fmaf(cv.w, wc, y[3]);
      }
      if (a.oacc) *reinterpret_cast<float4*>(a.oacc + r * D + qd * 4) = make_float4(y[0], y[1], y[2], y[3]);
      if (a.out) {
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = Lt == 0.f ? 0.f : __fdiv_rn(y[e], Lt);
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
      if (qd == 0) {
        smM[hh] = Lt == 0.f ? -INFINITY : Mh;
        smL[hh] = Lt;
      }
    }
    // m and l of the state out are written after every thread has read the
    // carry (state out may alias it)
    __syncthreads();
    if (a.om && tid < hpk) {
      a.om[row0 + tid] = smM[tid];
      a.ol[row0 + tid] = smL[tid];
    }
    return;
  }
  __syncthreads();
  if (tid < 128)
    finish_segment<D, HMAX>(a, t, tid, smM, smL, smC, &smFlag, qa, hpk * NA, 0u, NamedSync128{});
}

}  // namespace gqa
