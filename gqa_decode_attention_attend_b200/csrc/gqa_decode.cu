// gqa_decode.cu -- C ABI of the decode-attention library (include/gqa_decode.h):
// argument validation, the split heuristic, workspace sizing, TMA descriptor
// encoding and the kernel launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/gqa_decode.h"
#include "kernels.cuh"

namespace {

using gqa::MergeArgs;
using gqa::PartitionArgs;

constexpr int kVersion = 100;          // 0.1.0
constexpr size_t kHeaderBytes = 256;   // error word + reserved
// Merge tickets live in a fixed region right after the header that nothing else
// ever uses, so the zeros left by gqa_workspace_init and by every completed call
// survive calls of any shape. Batches with more (sequence, KV head) segments
// than it holds get a region after the partial states, cleared on each call.
constexpr size_t kTicketSlots = 65536;
constexpr int kChunkQuantum = 64;      // rows per pipeline stage of the bf16 kernel
constexpr int kMaxHeadsPerKv = 16;
constexpr int kMaxDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------------ device info

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  int resident_bf16[2][2] = {{0, 0}, {0, 0}};   // [D==128][NT-1]
  int resident_f32[2] = {0, 0};                 // [D==128], HMAX=16 worst case
  cudaError_t err = cudaSuccess;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

template <int D, int NT>
cudaError_t prepare_bf16(int* resident) {
  using C = gqa::TcCfg<D, NT>;
  cudaError_t e = cudaFuncSetAttribute(gqa::gqa_partition_bf16_kernel<D, NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(resident, gqa::gqa_partition_bf16_kernel<D, NT>,
                                                       C::kThreads, C::kSmemBytes);
}

template <int D, int HMAX>
cudaError_t prepare_f32(int* resident) {
  using C = gqa::F32Cfg<D, HMAX>;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(resident, gqa::gqa_partition_f32_kernel<D, HMAX>,
                                                       C::kThreads, C::kSmemBytes);
}

// the coded kernel's dynamic shared memory: every call's plan fits its budget,
// which leaves room under the 227 KB of a CTA for the kernel's static shared
// memory (3.4 KB at most); the largest tables still leave a ring row and the
// smallest round store
constexpr int kCodedMaxSmem = gqa::kCodedSmemBudget;
static_assert(kCodedMaxSmem + 4096 <= 227 * 1024, "coded shared memory under the per-CTA limit");
static_assert(gqa::coded_ring_fits(1, gqa::kMaxCodeWords, 1, gqa::kCodedMaxTableEntries) &&
                  gqa::coded_ring_fits(1, gqa::kMaxCodeWords, 16, gqa::kCodedMaxTableEntries / 16),
              "the largest coded tables fit beside a ring row and the smallest round store");

// Every bound also has a variant for exactly HMAX heads per KV head and MW
// words per row: its constant counts fold the loops' guards (on 16 x 4096
// keys, 4 heads, 8 words: 38.5 -> 33.9 us a call, measured on B200) and spill
// as much or less than the general one at most bounds. The switch stays per
// bound.
template <int HMAX, int MW>
constexpr bool kCodedExact = true;

template <int D, int HMAX, int MW>
cudaError_t prepare_coded() {
  if constexpr (kCodedExact<HMAX, MW>) {
    cudaError_t e = cudaFuncSetAttribute(gqa::gqa_partition_coded_kernel<D, HMAX, MW, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kCodedMaxSmem);
    if (e != cudaSuccess) return e;
  }
  return cudaFuncSetAttribute(gqa::gqa_partition_coded_kernel<D, HMAX, MW>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kCodedMaxSmem);
}

template <int D, int HMAX>
cudaError_t prepare_coded_words() {
  cudaError_t e = prepare_coded<D, HMAX, 4>();
  if (e == cudaSuccess) e = prepare_coded<D, HMAX, 8>();
  if (e == cudaSuccess) e = prepare_coded<D, HMAX, 16>();
  return e;
}

cudaError_t prepare_coded_all() {
  cudaError_t e = prepare_coded_words<64, 4>();
  if (e == cudaSuccess) e = prepare_coded_words<64, 8>();
  if (e == cudaSuccess) e = prepare_coded_words<64, 16>();
  if (e == cudaSuccess) e = prepare_coded_words<128, 4>();
  if (e == cudaSuccess) e = prepare_coded_words<128, 8>();
  if (e == cudaSuccess) e = prepare_coded_words<128, 16>();
  return e;
}

// Per-device one-time set-up (kernel attributes, occupancy, SM count).
const DeviceInfo* device_info(int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.ready) return &di;
  cudaDeviceProp prop;
  cudaError_t e = cudaGetDeviceProperties(&prop, dev);
  if (e == cudaSuccess && prop.major < 10) e = cudaErrorInvalidDevice;   // sm_100a code only
  if (e == cudaSuccess) e = prepare_bf16<64, 1>(&di.resident_bf16[0][0]);
  if (e == cudaSuccess) e = prepare_bf16<64, 2>(&di.resident_bf16[0][1]);
  if (e == cudaSuccess) e = prepare_bf16<128, 1>(&di.resident_bf16[1][0]);
  if (e == cudaSuccess) e = prepare_bf16<128, 2>(&di.resident_bf16[1][1]);
  if (e == cudaSuccess) e = prepare_coded_all();
  if (e == cudaSuccess) e = prepare_f32<64, 16>(&di.resident_f32[0]);
  if (e == cudaSuccess) e = prepare_f32<128, 16>(&di.resident_f32[1]);
  if (e != cudaSuccess) {
    cudaGetLastError();
    di.err = e;
    return nullptr;
  }
  di.sm_count = prop.multiProcessorCount;
  di.ready = true;
  return &di;
}

// ------------------------------------------------------------------ driver entry point

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// K or V cache [max_len, G, D] bf16 as a 2-D tensor (G*D columns, max_len rows);
// box = 64 columns (128 bytes, one swizzle span) x 64 rows. The last few
// encodings are kept per thread and reused for an identical cache.
bool make_kv_map(CUtensorMap* m, const void* base, int max_len, int G, int D) {
  struct Entry {
    const void* base;
    int max_len, G, D;
    CUtensorMap map;
  };
  constexpr int kKept = 4;
  thread_local Entry kept[kKept] = {};
  thread_local int next = 0;
  for (int i = 0; i < kKept; ++i)
    if (kept[i].base == base && kept[i].max_len == max_len && kept[i].G == G && kept[i].D == D) {
      *m = kept[i].map;
      return true;
    }
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(G) * D, static_cast<cuuint64_t>(max_len)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(G) * D * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kChunkQuantum)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  kept[next] = Entry{base, max_len, G, D, *m};
  next = (next + 1) % kKept;
  return true;
}

// ------------------------------------------------------------------ validation helpers

// Whether `p` is device (or managed) memory. Addresses already seen to be
// device memory are remembered in a small per-thread ring (64 entries), so a
// decode loop that passes the same buffers call after call pays for the
// driver query once; host addresses are never remembered.
bool is_device_ptr(const void* p) {
  if (p == nullptr) return true;
  constexpr int kSeen = 64;
  thread_local const void* seen[kSeen] = {};
  thread_local int seen_dev[kSeen] = {};
  thread_local int next = 0;
  int dev = -1;
  cudaGetDevice(&dev);
  for (int i = 0; i < kSeen; ++i)
    if (seen[i] == p && seen_dev[i] == dev) return true;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const bool ok = at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
  if (ok) {
    seen[next] = p;
    seen_dev[next] = dev;
    next = (next + 1) % kSeen;
  }
  return ok;
}

bool state_present(const gqa_state& s) { return s.m || s.l || s.acc; }
bool state_complete(const gqa_state& s) { return s.m && s.l && s.acc; }

struct Resolved {
  int B, H, G, hpk, D, max_len, max_seq_len;
  bool bf16;
  int out_bf16;
  float scale;
  bool want_merge;      // out or state_out requested
  bool has_partials;    // caller's partials_out
  int S, chunk;         // split plan
  int sm_count;         // SMs of the device (0 when not queried)
  int per_sm;           // partition CTAs resident per SM
  size_t bytes;         // workspace bytes
  size_t off_m, off_l, off_acc, off_counters;
  bool clear_counters;  // counters outside the fixed ticket region
};

int nt_of(int hpk) { return hpk <= 8 ? 1 : 2; }

// Split heuristic. A split is a chunk of chunk_len keys (a multiple of the
// 64-row pipeline stage) of one sequence; one CTA owns one (sequence, KV head,
// split) tile, so a call launches batch * num_kv_heads * num_splits CTAs.
//
// Equal-length batch: the kernel is HBM-bound as soon as about one CTA per SM
// is streaming, and every CTA does the same work, so the time is set by how
// the CTAs fill the `resident` slots. A last partial wave costs as much as
// max(its CTAs, sm_count) CTAs would (each CTA's own stream is bounded). The
// plan minimises
//     waves * (chunk_len + 128) + 4 * num_splits + merge
// (128 rows ~ a CTA's fixed prologue/epilogue, 4 rows ~ one more partial state
// in the merge), ties going to fewer splits. merge = 256 rows when the
// sequences are long (>= 2048 keys) and there is more than one split: the
// segment's last CTA takes its ticket and pulls the other splits' states from
// L2 after its own stream, about 3-4 us on B200, which only counts against
// long streams (short ones are bound by each CTA's latency, and splitting
// them pays). Measured on B200, 16 sequences x 8 KV heads x 4096 keys: 1
// split (128 CTAs) streams as fast as 2 back to back and ends a lone call
// ~4 us sooner.
// Ragged batch (total_rows below batch * max_seq_len): the tiles are uneven, so
// the plan aims at ~8 waves of CTAs and lets the block scheduler balance them.
gqa_status plan_impl(int32_t batch, int32_t G, int32_t max_seq_len, int64_t total_rows,
                     int32_t sm_count, int32_t ctas_per_sm, int32_t* chunk_len, int32_t* num_splits) {
  if (batch < 0 || G <= 0 || max_seq_len < 0 || sm_count <= 0 || ctas_per_sm <= 0 || !chunk_len ||
      !num_splits)
    return GQA_ERR_INVALID_ARGUMENT;
  const int64_t q = kChunkQuantum;
  if (max_seq_len == 0 || batch == 0) {
    *chunk_len = kChunkQuantum;
    *num_splits = 1;
    return GQA_OK;
  }
  const int64_t resident = static_cast<int64_t>(sm_count) * ctas_per_sm;
  const int64_t N = max_seq_len;
  const int64_t full = static_cast<int64_t>(batch) * N;
  if (total_rows <= 0 || total_rows > full) total_rows = full;
  const int64_t max_splits = (N + q - 1) / q;
  if (total_rows < full) {
    const int64_t target = resident * 8;
    int64_t chunk = (total_rows * G + target - 1) / target;
    chunk = (chunk + q - 1) / q * q;
    if (chunk < 4 * q) chunk = 4 * q;
    if (chunk > max_splits * q) chunk = max_splits * q;
    int64_t splits = (N + chunk - 1) / chunk;
    chunk = ((N + splits - 1) / splits + q - 1) / q * q;
    *chunk_len = static_cast<int32_t>(chunk);
    *num_splits = static_cast<int32_t>((N + chunk - 1) / chunk);
    return GQA_OK;
  }
  const int64_t segs = static_cast<int64_t>(batch) * G;
  double best = 0.0;
  int64_t best_chunk = 0, best_splits = 0;
  const int64_t limit = std::min<int64_t>(max_splits, 4 * resident / segs + 2);
  for (int64_t S = 1; S <= limit; ++S) {
    const int64_t chunk = ((N + S - 1) / S + q - 1) / q * q;
    const int64_t splits = (N + chunk - 1) / chunk;
    if (splits != S) continue;                      // same plan as a smaller S
    const int64_t ctas = segs * S;
    const int64_t rem = ctas % resident;
    const double waves = static_cast<double>(ctas / resident) +
                         (rem ? static_cast<double>(std::max<int64_t>(rem, sm_count)) / resident : 0.0);
    const double merge = (S > 1 && N >= 2048) ? 256.0 : 0.0;
    const double cost = waves * static_cast<double>(chunk + 128) + 4.0 * S + merge;
    if (best_splits == 0 || cost < best) {
      best = cost;
      best_chunk = chunk;
      best_splits = S;
    }
  }
  *chunk_len = static_cast<int32_t>(best_chunk);
  *num_splits = static_cast<int32_t>(best_splits);
  return GQA_OK;
}

// Host-side validation and planning shared by workspace_size and attend.
gqa_status resolve(const gqa_decode_params* p, Resolved* r, bool need_device, int per_sm_override = 0) {
  if (!p || p->struct_size != sizeof(gqa_decode_params)) return GQA_ERR_INVALID_ARGUMENT;
  r->B = p->batch;
  r->H = p->num_heads;
  r->G = p->num_kv_heads == 0 ? p->num_heads : p->num_kv_heads;
  r->D = p->head_dim;
  r->max_len = p->max_len;
  if (r->B < 0 || r->H <= 0 || r->G <= 0 || r->H % r->G != 0) return GQA_ERR_INVALID_ARGUMENT;
  r->hpk = r->H / r->G;
  if (r->hpk > kMaxHeadsPerKv) return GQA_ERR_INVALID_ARGUMENT;
  if (r->D != 64 && r->D != 128) return GQA_ERR_INVALID_ARGUMENT;
  if (r->max_len < 0 || p->max_seq_len < 0 || p->num_splits < 0) return GQA_ERR_INVALID_ARGUMENT;
  r->max_seq_len = p->max_seq_len == 0 ? r->max_len : p->max_seq_len;
  if (r->max_seq_len > r->max_len) r->max_seq_len = r->max_len;
  // q and an output are needed only when there is a sequence; K and V only
  // when the cache has rows (an empty tensor may have a null data pointer).
  if (!p->offsets) return GQA_ERR_INVALID_ARGUMENT;
  if (r->B > 0 && !p->q) return GQA_ERR_INVALID_ARGUMENT;
  if (r->max_len > 0 && (!p->k || !p->v)) return GQA_ERR_INVALID_ARGUMENT;
  const bool has_carry = state_present(p->carry_in);
  const bool has_state_out = state_present(p->state_out);
  r->has_partials = state_present(p->partials_out);
  if ((has_carry && !state_complete(p->carry_in)) || (has_state_out && !state_complete(p->state_out)) ||
      (r->has_partials && !state_complete(p->partials_out)))
    return GQA_ERR_INVALID_ARGUMENT;
  if (r->B > 0 && !p->out && !has_state_out && !r->has_partials) return GQA_ERR_INVALID_ARGUMENT;
  r->want_merge = p->out || has_state_out;
  if (p->q_dtype != GQA_F32 && p->q_dtype != GQA_BF16) return GQA_ERR_SHAPE_MISMATCH;
  if (p->kv_dtype != GQA_F32 && p->kv_dtype != GQA_BF16) return GQA_ERR_SHAPE_MISMATCH;
  if (p->q_dtype != p->kv_dtype) return GQA_ERR_SHAPE_MISMATCH;
  if (p->out && p->out_dtype != GQA_F32 && p->out_dtype != GQA_BF16) return GQA_ERR_SHAPE_MISMATCH;
  r->bf16 = p->kv_dtype == GQA_BF16;
  r->out_bf16 = p->out_dtype == GQA_BF16 ? 1 : 0;
  // q/K/V feed 32-bit and TMA loads; out and every acc array are read and
  // written four floats (or four bf16) at a time.
  const uintptr_t align_or =
      reinterpret_cast<uintptr_t>(p->q) | reinterpret_cast<uintptr_t>(p->k) |
      reinterpret_cast<uintptr_t>(p->v) | reinterpret_cast<uintptr_t>(p->out) |
      reinterpret_cast<uintptr_t>(p->carry_in.acc) | reinterpret_cast<uintptr_t>(p->state_out.acc) |
      reinterpret_cast<uintptr_t>(p->partials_out.acc);
  if (align_or & 15u) return GQA_ERR_SHAPE_MISMATCH;
  if (reinterpret_cast<uintptr_t>(p->bias) & 3u) return GQA_ERR_SHAPE_MISMATCH;
  if (!std::isfinite(p->score_scale)) return GQA_ERR_INVALID_ARGUMENT;
  if (p->flags & ~static_cast<uint32_t>(GQA_FLAG_EARLY_START)) return GQA_ERR_INVALID_ARGUMENT;
  r->scale = p->score_scale != 0.f ? p->score_scale : 1.0f / sqrtf(static_cast<float>(r->D));
  if (static_cast<int64_t>(r->B) * r->H * r->D > INT32_MAX) return GQA_ERR_INVALID_ARGUMENT;

  r->sm_count = 148;     // B200; replaced by the device's own count below
  r->per_sm = 2;
  if (need_device) {
    int dev;
    const DeviceInfo* di = device_info(&dev);
    if (!di) return GQA_ERR_DEVICE;
    const int per_sm = r->bf16 ? di->resident_bf16[r->D == 128][nt_of(r->hpk) - 1]
                               : di->resident_f32[r->D == 128];
    r->sm_count = di->sm_count;
    r->per_sm = per_sm > 0 ? per_sm : 1;
  }
  if (per_sm_override > 0) r->per_sm = per_sm_override;
  // split plan
  if (p->num_splits > 0) {
    r->S = p->num_splits;
    int64_t chunk = r->max_seq_len == 0 ? kChunkQuantum : (static_cast<int64_t>(r->max_seq_len) + r->S - 1) / r->S;
    chunk = (chunk + kChunkQuantum - 1) / kChunkQuantum * kChunkQuantum;
    r->chunk = static_cast<int>(chunk);
  } else {
    int32_t c, s;
    gqa_status st = plan_impl(r->B, r->G, r->max_seq_len, r->max_len, r->sm_count, r->per_sm, &c, &s);
    if (st != GQA_OK) return st;
    r->S = s;
    r->chunk = c;
  }
  if (static_cast<int64_t>(r->B) * r->S * r->G > INT32_MAX) return GQA_ERR_INVALID_ARGUMENT;
  // workspace: header, then internal partial states when merging without the caller's
  r->bytes = kHeaderBytes;
  r->off_m = r->off_l = r->off_acc = r->off_counters = 0;
  r->clear_counters = false;
  const size_t segs = static_cast<size_t>(r->B) * r->G;
  if (r->want_merge) {
    r->off_counters = r->bytes;
    r->bytes += kTicketSlots * sizeof(uint32_t);
  }
  if (r->want_merge && !r->has_partials) {
    const size_t n = static_cast<size_t>(r->B) * r->H * r->S;
    r->off_m = r->bytes;
    r->bytes += align256(n * sizeof(float));
    r->off_l = r->bytes;
    r->bytes += align256(n * sizeof(float));
    r->off_acc = r->bytes;
    r->bytes += align256(n * r->D * sizeof(float));
  }
  if (r->want_merge && segs > kTicketSlots) {
    r->off_counters = r->bytes;
    r->bytes += align256(segs * sizeof(uint32_t));
    r->clear_counters = true;
  }
  return GQA_OK;
}

template <int D>
cudaError_t launch_merge(const MergeArgs& m, cudaStream_t st) {
  if (m.rows == 0) return cudaSuccess;
  gqa::gqa_merge_kernel<D><<<m.rows, 128, 0, st>>>(m);
  return cudaGetLastError();
}

cudaError_t launch_merge_any(int D, const MergeArgs& m, cudaStream_t st) {
  return D == 128 ? launch_merge<128>(m, st) : launch_merge<64>(m, st);
}

// Launch configuration shared by the partition kernels. With early_start the
// launch carries programmatic stream serialization: the kernel may begin while
// the previous kernel on the stream finishes (see GQA_FLAG_EARLY_START).
struct Launch {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  Launch(unsigned grid, unsigned threads, size_t smem, cudaStream_t st, bool early_start) {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = early_start ? 1 : 0;
  }
};

template <int D, int NT>
cudaError_t launch_bf16(const PartitionArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                        unsigned grid, cudaStream_t st, bool early) {
  using C = gqa::TcCfg<D, NT>;
  Launch l(grid, C::kThreads, C::kSmemBytes, st, early);
  return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_bf16_kernel<D, NT>, tk, tv, a);
}

template <int D, int HMAX>
cudaError_t launch_f32(const PartitionArgs& a, unsigned grid, cudaStream_t st, bool early) {
  using C = gqa::F32Cfg<D, HMAX>;
  Launch l(grid, C::kThreads, C::kSmemBytes, st, early);
  return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_f32_kernel<D, HMAX>, a);
}

// The coded kernel for heads_per_kv bound hp (4, 8, 16) and words bound mw (4, 8, 16).
template <int D, int HMAX>
cudaError_t launch_coded_hp(Launch& l, int mw, const PartitionArgs& a, const gqa::CodedArgs& c) {
  // rows of exactly the bound's words, with the bound's heads per KV head,
  // take the variant compiled for them
  const bool ex = c.words == mw && a.hpk == HMAX;
  if (mw == 4) {
    if constexpr (kCodedExact<HMAX, 4>)
      if (ex) return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_coded_kernel<D, HMAX, 4, true>, a, c);
    return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_coded_kernel<D, HMAX, 4>, a, c);
  }
  if (mw == 8) {
    if constexpr (kCodedExact<HMAX, 8>)
      if (ex) return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_coded_kernel<D, HMAX, 8, true>, a, c);
    return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_coded_kernel<D, HMAX, 8>, a, c);
  }
  if constexpr (kCodedExact<HMAX, 16>)
    if (ex) return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_coded_kernel<D, HMAX, 16, true>, a, c);
  return cudaLaunchKernelEx(&l.cfg, gqa::gqa_partition_coded_kernel<D, HMAX, 16>, a, c);
}

template <int D>
cudaError_t launch_coded(Launch& l, int hp, int mw, const PartitionArgs& a, const gqa::CodedArgs& c) {
  if (hp == 4) return launch_coded_hp<D, 4>(l, mw, a, c);
  if (hp == 8) return launch_coded_hp<D, 8>(l, mw, a, c);
  return launch_coded_hp<D, 16>(l, mw, a, c);
}


cudaError_t launch_partition(const Resolved& r, const PartitionArgs& a, const CUtensorMap* tk,
                             const CUtensorMap* tv, cudaStream_t st, bool early) {
  const unsigned grid = static_cast<unsigned>(r.B) * r.S * r.G;
  if (grid == 0) return cudaSuccess;
  if (r.bf16) {
    const int nt = nt_of(r.hpk);
    if (r.D == 128)
      return nt == 1 ? launch_bf16<128, 1>(a, *tk, *tv, grid, st, early) : launch_bf16<128, 2>(a, *tk, *tv, grid, st, early);
    return nt == 1 ? launch_bf16<64, 1>(a, *tk, *tv, grid, st, early) : launch_bf16<64, 2>(a, *tk, *tv, grid, st, early);
  }
  if (r.D == 128) {
    if (r.hpk <= 4) return launch_f32<128, 4>(a, grid, st, early);
    if (r.hpk <= 8) return launch_f32<128, 8>(a, grid, st, early);
    return launch_f32<128, 16>(a, grid, st, early);
  }
  if (r.hpk <= 4) return launch_f32<64, 4>(a, grid, st, early);
  if (r.hpk <= 8) return launch_f32<64, 8>(a, grid, st, early);
  return launch_f32<64, 16>(a, grid, st, early);
}

// Kernel arguments of a decode call whose scratch is at `ws`.
PartitionArgs make_args(const gqa_decode_params* p, const Resolved& r, uint8_t* ws, const void* k_new,
                        const void* v_new) {
  PartitionArgs a{};
  a.q = p->q;
  a.k = p->k;
  a.v = p->v;
  a.offsets = p->offsets;
  a.B = r.B;
  a.H = r.H;
  a.G = r.G;
  a.hpk = r.hpk;
  a.max_len = r.max_len;
  a.chunk_len = r.chunk;
  a.num_splits = r.S;
  a.scale_log2 = r.scale * gqa::kLog2e;
  if (r.has_partials) {
    a.part_m = p->partials_out.m;
    a.part_l = p->partials_out.l;
    a.part_acc = p->partials_out.acc;
    a.write_empty = 1;
  } else {
    a.part_m = reinterpret_cast<float*>(ws + r.off_m);
    a.part_l = reinterpret_cast<float*>(ws + r.off_l);
    a.part_acc = reinterpret_cast<float*>(ws + r.off_acc);
    a.write_empty = 0;
  }
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.merge = r.want_merge ? 1 : 0;
  a.partials_internal = r.has_partials ? 0 : 1;
  a.counters = r.want_merge ? reinterpret_cast<uint32_t*>(ws + r.off_counters) : nullptr;
  const bool has_carry = state_present(p->carry_in);
  a.cm = has_carry ? p->carry_in.m : nullptr;
  a.cl = has_carry ? p->carry_in.l : nullptr;
  a.cacc = has_carry ? p->carry_in.acc : nullptr;
  const bool has_so = state_present(p->state_out);
  a.om = has_so ? p->state_out.m : nullptr;
  a.ol = has_so ? p->state_out.l : nullptr;
  a.oacc = has_so ? p->state_out.acc : nullptr;
  a.out = p->out;
  a.out_bf16 = r.out_bf16;
  a.bias = p->bias;
  a.k_new = k_new;
  a.v_new = v_new;
  a.kw = const_cast<void*>(p->k);
  a.vw = const_cast<void*>(p->v);
  a.kv_elem = r.bf16 ? 2 : 4;
  // A grid that fills most of the GPU's CTA slots lets the next kernel start
  // when its last loads are issued (the next grid then only takes the few free
  // slots and the stragglers' slots); a grid that leaves many slots free waits
  // until its streams are done, or the next grid would split into an early and
  // a late half (measured on B200: +2 % on 256 CTAs, -2..5 % on 160 CTAs).
  const int64_t grid = static_cast<int64_t>(r.B) * r.S * r.G;
  const int64_t slots = static_cast<int64_t>(r.sm_count) * r.per_sm;
  a.trigger_at_last_load = (grid * 5 >= slots * 4) ? 1 : 0;
  return a;
}

// Pointer checks and the single launch of a decode call, with the scratch at `ws`
// (the caller's workspace, or the library's static array).
gqa_status attend_impl(const gqa_decode_params* p, const Resolved& r, uint8_t* ws, cudaStream_t cs,
                       const void* k_new = nullptr, const void* v_new = nullptr) {
  const void* ptrs[] = {p->q, p->k, p->v, p->offsets, p->out,
                        p->carry_in.m, p->carry_in.l, p->carry_in.acc,
                        p->state_out.m, p->state_out.l, p->state_out.acc,
                        p->partials_out.m, p->partials_out.l, p->partials_out.acc,
                        p->bias, k_new, v_new};
  for (const void* q : ptrs)
    if (!is_device_ptr(q)) return GQA_ERR_DEVICE;
  if (r.B == 0) return GQA_OK;

  PartitionArgs a = make_args(p, r, ws, k_new, v_new);

  // With no cache rows every tile is empty and no load is issued, but a tensor
  // map still needs a non-zero extent and a valid aligned base: the scratch
  // stands in for the (possibly null) empty caches.
  CUtensorMap tk, tv;
  const int map_rows = r.max_len > 0 ? r.max_len : 1;
  const void* kb = r.max_len > 0 ? p->k : static_cast<const void*>(ws);
  const void* vb = r.max_len > 0 ? p->v : static_cast<const void*>(ws);
  if (r.bf16 && (!make_kv_map(&tk, kb, map_rows, r.G, r.D) || !make_kv_map(&tv, vb, map_rows, r.G, r.D)))
    return GQA_ERR_DEVICE;
  if (r.clear_counters &&
      cudaMemsetAsync(a.counters, 0, static_cast<size_t>(r.B) * r.G * sizeof(uint32_t), cs) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  if (launch_partition(r, a, &tk, &tv, cs, (p->flags & GQA_FLAG_EARLY_START) != 0) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  return GQA_OK;
}

}  // namespace

extern "C" {

const char* gqa_status_string(gqa_status s) {
  switch (s) {
    case GQA_OK: return "GQA_OK";
    case GQA_ERR_INVALID_ARGUMENT: return "GQA_ERR_INVALID_ARGUMENT";
    case GQA_ERR_SHAPE_MISMATCH: return "GQA_ERR_SHAPE_MISMATCH";
    case GQA_ERR_DEVICE: return "GQA_ERR_DEVICE";
    case GQA_ERR_WORKSPACE: return "GQA_ERR_WORKSPACE";
    case GQA_ERR_BAD_OFFSETS: return "GQA_ERR_BAD_OFFSETS";
    case GQA_ERR_TIMEOUT: return "GQA_ERR_TIMEOUT";
    case GQA_ERR_BAD_CODES: return "GQA_ERR_BAD_CODES";
  }
  return "GQA_ERR_UNKNOWN";
}

int32_t gqa_version(void) { return kVersion; }

gqa_status gqa_plan_splits(int32_t batch, int32_t num_kv_heads, int32_t max_seq_len, int64_t total_rows,
                           int32_t sm_count, int32_t ctas_per_sm, int32_t* chunk_len, int32_t* num_splits) {
  return plan_impl(batch, num_kv_heads, max_seq_len, total_rows, sm_count, ctas_per_sm, chunk_len,
                   num_splits);
}

gqa_status gqa_decode_workspace_size(const gqa_decode_params* params, size_t* bytes, int32_t* num_splits,
                                     int32_t* chunk_len) {
  Resolved r;
  gqa_status st = resolve(params, &r, true);
  if (st != GQA_OK) return st;
  if (bytes) *bytes = r.bytes;
  if (num_splits) *num_splits = r.S;
  if (chunk_len) *chunk_len = r.chunk;
  return GQA_OK;
}

gqa_status gqa_workspace_init(void* workspace, size_t workspace_bytes, gqa_stream_t stream) {
  if (!workspace || workspace_bytes < kHeaderBytes) return GQA_ERR_WORKSPACE;
  if (!is_device_ptr(workspace)) return GQA_ERR_DEVICE;
  if (cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  return GQA_OK;
}

gqa_status gqa_decode_attend(const gqa_decode_params* p, gqa_stream_t stream) {
  Resolved r;
  gqa_status st = resolve(p, &r, true);
  if (st != GQA_OK) return st;
  if (!p->workspace || p->workspace_bytes < r.bytes) return GQA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(p->workspace) & 255u) return GQA_ERR_WORKSPACE;
  if (!is_device_ptr(p->workspace)) return GQA_ERR_DEVICE;
  return attend_impl(p, r, static_cast<uint8_t*>(p->workspace), reinterpret_cast<cudaStream_t>(stream));
}

gqa_status gqa_decode_append_attend(const gqa_decode_params* p, const void* k_new, const void* v_new,
                                    gqa_stream_t stream) {
  Resolved r;
  gqa_status st = resolve(p, &r, true);
  if (st != GQA_OK) return st;
  if (r.B > 0 && (!k_new || !v_new || r.max_len == 0)) return GQA_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15u)
    return GQA_ERR_SHAPE_MISMATCH;
  if (!p->workspace || p->workspace_bytes < r.bytes) return GQA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(p->workspace) & 255u) return GQA_ERR_WORKSPACE;
  if (!is_device_ptr(p->workspace)) return GQA_ERR_DEVICE;
  return attend_impl(p, r, static_cast<uint8_t*>(p->workspace), reinterpret_cast<cudaStream_t>(stream),
                     k_new, v_new);
}

// Validation and the split plan of a coded call: everything as gqa_decode_attend
// would check it, with the code arrays standing in for the caches (their dtype
// is the queries'), and the plan made for the coded kernel's occupancy (one
// CTA of 512 threads per SM).
static gqa_status resolve_coded(const gqa_decode_params* p, const gqa_kv_codes* codes, gqa_decode_params* pc,
                                Resolved* r) {
  if (!p || !codes || p->struct_size != sizeof(gqa_decode_params)) return GQA_ERR_INVALID_ARGUMENT;
  if (codes->words < 1 || codes->words > 16 || codes->n_atoms < 1 || codes->n_atoms > 65536)
    return GQA_ERR_INVALID_ARGUMENT;
  *pc = *p;
  pc->k = codes->k_codes;
  pc->v = codes->v_codes;
  pc->kv_dtype = p->q_dtype;
  gqa_status st = resolve(pc, r, true, 1);
  if (st != GQA_OK) return st;
  if (r->B > 0 && r->max_len > 0 && (!codes->k_atoms || !codes->v_atoms)) return GQA_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(codes->k_atoms) | reinterpret_cast<uintptr_t>(codes->v_atoms)) & 15u)
    return GQA_ERR_SHAPE_MISMATCH;
  // rows of 4k words are read 16 bytes at a time
  if ((codes->words & 3) == 0 &&
      ((reinterpret_cast<uintptr_t>(codes->k_codes) | reinterpret_cast<uintptr_t>(codes->v_codes)) & 15u))
    return GQA_ERR_SHAPE_MISMATCH;
  if (static_cast<int64_t>(r->hpk) * codes->n_atoms > gqa::kCodedMaxTableEntries ||
      !gqa::coded_ring_fits(1, codes->words, r->hpk, codes->n_atoms))
    return GQA_ERR_INVALID_ARGUMENT;
  return GQA_OK;
}

gqa_status gqa_decode_coded_workspace_size(const gqa_decode_params* p, const gqa_kv_codes* codes, size_t* bytes,
                                           int32_t* num_splits, int32_t* chunk_len) {
  gqa_decode_params pc;
  Resolved r;
  gqa_status st = resolve_coded(p, codes, &pc, &r);
  if (st != GQA_OK) return st;
  if (bytes) *bytes = r.bytes;
  if (num_splits) *num_splits = r.S;
  if (chunk_len) *chunk_len = r.chunk;
  return GQA_OK;
}

gqa_status gqa_decode_attend_coded(const gqa_decode_params* p, const gqa_kv_codes* codes,
                                   gqa_stream_t stream) {
  gqa_decode_params pc;
  Resolved r;
  gqa_status st = resolve_coded(p, codes, &pc, &r);
  if (st != GQA_OK) return st;
  const size_t smem = gqa::coded_smem_bytes(codes->words, r.hpk, codes->n_atoms);
  if (!p->workspace || p->workspace_bytes < r.bytes) return GQA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(p->workspace) & 255u) return GQA_ERR_WORKSPACE;
  const void* ptrs[] = {p->q, p->offsets, p->out, p->workspace, p->bias, codes->k_codes, codes->v_codes,
                        codes->k_atoms, codes->v_atoms, p->carry_in.m, p->carry_in.l, p->carry_in.acc,
                        p->state_out.m, p->state_out.l, p->state_out.acc, p->partials_out.m,
                        p->partials_out.l, p->partials_out.acc};
  for (const void* q : ptrs)
    if (!is_device_ptr(q)) return GQA_ERR_DEVICE;
  if (r.B == 0) return GQA_OK;
  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  PartitionArgs a = make_args(&pc, r, ws, nullptr, nullptr);
  a.k = a.v = nullptr;
  a.kw = a.vw = nullptr;
  gqa::CodedArgs c{codes->k_codes, codes->v_codes, codes->k_atoms, codes->v_atoms, codes->words,
                   codes->n_atoms, r.bf16 ? 1 : 0};
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (r.clear_counters &&
      cudaMemsetAsync(a.counters, 0, static_cast<size_t>(r.B) * r.G * sizeof(uint32_t), cs) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  const unsigned grid = static_cast<unsigned>(r.B) * r.S * r.G;
  Launch l(grid, gqa::kCodedThreads, smem, cs, (p->flags & GQA_FLAG_EARLY_START) != 0);
  cudaError_t e;
  const int hp = r.hpk <= 4 ? 4 : (r.hpk <= 8 ? 8 : 16);
  const int mw = codes->words <= 4 ? 4 : (codes->words <= 8 ? 8 : 16);
  e = r.D == 128 ? launch_coded<128>(l, hp, mw, a, c) : launch_coded<64>(l, hp, mw, a, c);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  return GQA_OK;
}

gqa_status gqa_topk_to_bias(const int32_t* idx, int32_t batch, int32_t width, const int32_t* offsets,
                            int32_t max_len, float* bias, void* workspace, gqa_stream_t stream) {
  if (batch < 0 || width < 0 || max_len < 0) return GQA_ERR_INVALID_ARGUMENT;
  if (batch == 0) return GQA_OK;
  if (!offsets || !bias || (width > 0 && !idx)) return GQA_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(bias) & 3u) return GQA_ERR_SHAPE_MISMATCH;
  const void* ptrs[] = {idx, offsets, bias, workspace};
  for (const void* q : ptrs)
    if (!is_device_ptr(q)) return GQA_ERR_DEVICE;
  gqa::gqa_topk_to_bias_kernel<<<batch, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      idx, width, offsets, max_len, bias, static_cast<uint32_t*>(workspace));
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_DEVICE;
  return GQA_OK;
}

static gqa_status merge_common(const gqa_state* states, int32_t rows, int32_t num_states, int32_t head_dim,
                               const gqa_state* carry_in, const gqa_state* merged_out, void* out,
                               int32_t out_dtype, gqa_stream_t stream, bool gathered = false) {
  if (rows < 0 || num_states < 0 || (head_dim != 64 && head_dim != 128)) return GQA_ERR_INVALID_ARGUMENT;
  if (num_states > 0 && (!states || !state_complete(*states))) return GQA_ERR_INVALID_ARGUMENT;
  const bool has_carry = carry_in && state_present(*carry_in);
  const bool has_out_state = merged_out && state_present(*merged_out);
  if ((has_carry && !state_complete(*carry_in)) || (has_out_state && !state_complete(*merged_out)))
    return GQA_ERR_INVALID_ARGUMENT;
  if (!has_out_state && !out) return GQA_ERR_INVALID_ARGUMENT;
  if (out && out_dtype != GQA_F32 && out_dtype != GQA_BF16) return GQA_ERR_SHAPE_MISMATCH;
  if (static_cast<int64_t>(rows) * num_states * head_dim > (int64_t(1) << 40)) return GQA_ERR_INVALID_ARGUMENT;
  // the merge kernel reads acc rows with 8- (D=64) or 16-byte (D=128) vector loads
  if (num_states > 0 && (reinterpret_cast<uintptr_t>(states->acc) & 15u)) return GQA_ERR_SHAPE_MISMATCH;
  const void* ptrs[] = {num_states > 0 ? states->m : nullptr, num_states > 0 ? states->l : nullptr,
                        num_states > 0 ? states->acc : nullptr, has_carry ? carry_in->m : nullptr,
                        has_carry ? carry_in->l : nullptr, has_carry ? carry_in->acc : nullptr,
                        has_out_state ? merged_out->m : nullptr, has_out_state ? merged_out->l : nullptr,
                        has_out_state ? merged_out->acc : nullptr, out};
  for (const void* q : ptrs)
    if (!is_device_ptr(q)) return GQA_ERR_DEVICE;
  if (has_out_state && num_states > 0 &&
      (merged_out->m == states->m || merged_out->l == states->l || merged_out->acc == states->acc))
    return GQA_ERR_INVALID_ARGUMENT;
  if (rows == 0) return GQA_OK;
  MergeArgs m;
  m.m = num_states > 0 ? states->m : nullptr;
  m.l = num_states > 0 ? states->l : nullptr;
  m.acc = num_states > 0 ? states->acc : nullptr;
  m.rows = rows;
  m.S = num_states;
  m.row_stride = gathered ? 1 : num_states;
  m.state_stride = gathered ? rows : 1;
  m.cm = has_carry ? carry_in->m : nullptr;
  m.cl = has_carry ? carry_in->l : nullptr;
  m.cacc = has_carry ? carry_in->acc : nullptr;
  m.om = has_out_state ? merged_out->m : nullptr;
  m.ol = has_out_state ? merged_out->l : nullptr;
  m.oacc = has_out_state ? merged_out->acc : nullptr;
  m.out = out;
  m.out_bf16 = out_dtype == GQA_BF16 ? 1 : 0;
  if (launch_merge_any(head_dim, m, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GQA_ERR_DEVICE;
  return GQA_OK;
}

gqa_status gqa_softmax_merge(const gqa_state* states, int32_t rows, int32_t num_states, int32_t head_dim,
                             const gqa_state* carry_in, const gqa_state* merged_out, void* out,
                             int32_t out_dtype, gqa_stream_t stream) {
  return merge_common(states, rows, num_states, head_dim, carry_in, merged_out, out, out_dtype, stream);
}

gqa_status gqa_softmax_merge_gathered(const gqa_state* states, int32_t rows, int32_t num_states,
                                      int32_t head_dim, const gqa_state* carry_in,
                                      const gqa_state* merged_out, void* out, int32_t out_dtype,
                                      gqa_stream_t stream) {
  return merge_common(states, rows, num_states, head_dim, carry_in, merged_out, out, out_dtype, stream, true);
}

gqa_status gqa_state_finalize(const gqa_state* state, int32_t rows, int32_t head_dim, void* out,
                              int32_t out_dtype, gqa_stream_t stream) {
  if (!out || !state) return GQA_ERR_INVALID_ARGUMENT;
  return merge_common(state, rows, 1, head_dim, nullptr, nullptr, out, out_dtype, stream);
}

gqa_status gqa_get_device_error(void* workspace, gqa_stream_t stream) {
  if (!workspace) return GQA_ERR_WORKSPACE;
  if (!is_device_ptr(workspace)) return GQA_ERR_DEVICE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof word, cs) != cudaSuccess || cudaStreamSynchronize(cs) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_DEVICE;
    }
  }
  if (word & gqa::kErrBadOffsets) return GQA_ERR_BAD_OFFSETS;
  if (word & gqa::kErrTimeout) return GQA_ERR_TIMEOUT;
  if (word & gqa::kErrBadCodes) return GQA_ERR_BAD_CODES;
  return GQA_OK;
}

}  // extern "C"

// ============================================================================
// Decode attention without a caller-supplied workspace.
//
// Some callers cannot hand the library scratch memory: code that runs where a
// device allocation is not allowed or not safe (a plugin inside a host engine
// that owns every device buffer and offers no workspace, a fixed-budget or
// real-time deployment that forbids allocation after start-up, or a callback
// in which cudaMalloc would implicitly synchronise the device). For them the
// scratch of gqa_decode_attend (the error word and the per-split partial
// states) lives in the file-scope device array below, which the CUDA module
// loader sets aside, zero-filled, on every GPU that loads this library and
// keeps until the process exits.
// ============================================================================

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB per GPU
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry point (the library links
// no driver import), or null.
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

std::mutex g_static_mu;
struct StaticScratch {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
StaticScratch g_static_scratch_addr[kMaxDevices];

// Device address of g_static_scratch on the current device. The host-side
// symbol is only a stand-in, so the address is looked up once per device, with
// that device current, and cached together with its context: a new context
// (the old one reset) has its own copy of the array and gets a new lookup.
void* static_scratch_address(int dev) {
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current();
  if (get == nullptr || get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticScratch& e = g_static_scratch_addr[dev];
  if (e.addr == nullptr || ctx != e.ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if (get != nullptr && get(&ctx) != CUDA_SUCCESS) ctx = nullptr;   // the lookup may create it
    e.addr = p;
    e.ctx = ctx;
  }
  return e.addr;
}

}  // namespace

extern "C" gqa_status gqa_decode_attend_static_workspace(const gqa_decode_params* p,
                                                         gqa_stream_t stream) {
  Resolved r;
  gqa_status st = resolve(p, &r, true);
  if (st != GQA_OK) return st;
  if (r.bytes > kStaticScratchBytes) return GQA_ERR_WORKSPACE;   // scratch need above the array
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return GQA_ERR_DEVICE;
  }
  uint8_t* ws = static_cast<uint8_t*>(static_scratch_address(dev));
  if (ws == nullptr) return GQA_ERR_DEVICE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left in it. The error word and
  // the tickets of this call's segments (in the fixed region right after the
  // header; larger batches use a region attend_impl clears itself) must start
  // at zero, so both are cleared here, whatever an earlier call left; the
  // partial states are written before they are read.
  if (r.B > 0) {
    size_t clear = sizeof(uint32_t);
    if (r.want_merge && !r.clear_counters)
      clear = kHeaderBytes + static_cast<size_t>(r.B) * r.G * sizeof(uint32_t);
    if (cudaMemsetAsync(ws, 0, clear, cs) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_DEVICE;
    }
  }
  return attend_impl(p, r, ws, cs);
}

#ifdef GQA_TEST_HOOKS
// Test support, compiled only into the test copy of the library: fill the
// static scratch's header and ticket region with the byte `fill` on `stream`,
// as a call that stopped half way could have left it.
extern "C" gqa_status gqa_test_soil_static_scratch(int32_t fill, gqa_stream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_DEVICE;
  uint8_t* ws = static_cast<uint8_t*>(static_scratch_address(dev));
  if (ws == nullptr) return GQA_ERR_DEVICE;
  if (cudaMemsetAsync(ws, fill & 0xFF, kHeaderBytes + kTicketSlots * sizeof(uint32_t),
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GQA_ERR_DEVICE;
  return GQA_OK;
}
#endif
