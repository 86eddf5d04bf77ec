/*
 * gqa_decode.h -- C ABI of the B200 (sm_100a) grouped-query decode attention library.
 *
 * One query token per sequence attends over that sequence's cached keys. Each
 * query head h scores every cached key of its KV group g = h / (H / G) at scale
 * score_scale (1/sqrt(head_dim) when 0), folds it into a running maximum m, a
 * partition l and a weighted value sum acc, and the output is acc / l.
 *
 * Sources (the math and the argument conventions follow these pages):
 *   [attn.rs]   needle_core `attn.rs` (docs.rs needle-core 0.3.1 source):
 *               `KvCache` -- keys/values [max_len, num_kv_heads, head_dim];
 *               `self_attn_incremental` -- kv head of Q head hi is hi / kv_repeat,
 *               scale head_dim^-0.5, score -> softmax -> weighted sum of V;
 *               `cross_attn_incremental` -- the same decode over a fixed cache.
 *   [usearch]   USearch Rust docs, "Linear algebra", § Attention and the API
 *               tables: `attend` folds every scored key into each head's running
 *               maximum, partition and weighted value sum; outputs are already
 *               divided by the partition, in the queries' scalar type; a carry of
 *               one `DenseSoftmaxState` per query row folds the call into another
 *               over the same queries; `score_scale` zero derives 1/sqrt(d);
 *               `head_count` zero means one; ragged runs use Apache Arrow offsets;
 *               refusals are `Status::ShapeMismatch`, `Status::Device`,
 *               `Status::InvalidArgument`.
 *   [cortiq]    cortiq_engine `NystromState` (docs.rs): under GQA every Q head of
 *               a group reads the same K/V rows, so they are stored and read once
 *               per group.
 *   [dsa]       metrale `glm5next_dsa_ref/mod.rs`, `pool_states`: a softmax with
 *               no valid entry gives weight 0, not NaN.
 *
 * Conventions for every entry point:
 *   - Every tensor pointer is CALLER-OWNED DEVICE memory (cudaMalloc or a
 *     framework allocator). The library allocates nothing, never synchronises
 *     (except gqa_get_device_error) and enqueues all work on the caller's stream.
 *   - Errors found on the host are returned synchronously and nothing is
 *     launched. A launch failure returns GQA_ERR_DEVICE.
 *   - Device-side findings (bad offsets, a pipeline wait that gave up) set bits
 *     in the error word at the head of the workspace; gqa_get_device_error reads
 *     and clears it.
 *   - Dtypes: q/K/V are (fp32, fp32) or (bf16, bf16); any other pair is
 *     GQA_ERR_SHAPE_MISMATCH. Accumulation is fp32 in both cases.
 *   - head_dim is 64 or 128; heads per KV head (H / G) is 1..16.
 *   - q, K, V, out and every acc array start on a 16-byte boundary
 *     (GQA_ERR_SHAPE_MISMATCH otherwise).
 */
#ifndef GQA_DECODE_H
#define GQA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream). NULL is the legacy default stream. */
typedef struct CUstream_st* gqa_stream_t;

/* Status codes. Refusals mirror [usearch] Status::InvalidArgument,
 * Status::ShapeMismatch and Status::Device. */
typedef enum {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARGUMENT = 1, /* a size, count or required pointer is wrong  */
  GQA_ERR_SHAPE_MISMATCH = 2,   /* unsupported dtype pair or misaligned tensor */
  GQA_ERR_DEVICE = 3,           /* pointer not device memory, no device, launch failure */
  GQA_ERR_WORKSPACE = 4,        /* workspace missing or smaller than required  */
  GQA_ERR_BAD_OFFSETS = 5,      /* device-detected: offsets not monotone / beyond max_len */
  GQA_ERR_TIMEOUT = 6,          /* device-detected: a pipeline wait gave up    */
  GQA_ERR_BAD_CODES = 7         /* device-detected: a code word names a missing atom */
} gqa_status;

typedef enum { GQA_F32 = 0, GQA_BF16 = 1 } gqa_dtype;

/* Flags of gqa_decode_params.flags.
 * GQA_FLAG_EARLY_START: launch with programmatic stream serialization, so the
 *   call's kernel may start -- and begin streaming K/V cache rows -- while the
 *   kernel before it on the stream is still finishing. Everything else that
 *   kernel may write (q, the carry, the bias, the appended K/V, the workspace)
 *   is read only after it completes. The caller promises that the kernel
 *   immediately before this call does not write the offsets or any cache row
 *   this call reads from the cache (the row an append call writes itself is
 *   not read from the cache). Without the flag, ordinary stream order. */
enum { GQA_FLAG_EARLY_START = 1u };

/* An online-softmax state per query row, structure of arrays, fp32 device memory:
 *   m   [rows]        running maximum of the logits scale*q.k, natural-log units
 *                     ([usearch] DenseSoftmaxState::maximum_score)
 *   l   [rows]        partition: sum of e^{logit - m}  ([usearch] ::partition)
 *   acc [rows, D]     unnormalised weighted value sum, sum e^{logit - m} v
 * The output of a state is acc / l. A state with l == 0 is EMPTY whatever its m
 * (identity of the merge); the library writes empty states as (-inf, 0, 0).
 * A gqa_state with all three pointers NULL means "absent". */
typedef struct {
  float* m;
  float* l;
  float* acc;
} gqa_state;

/* Arguments of gqa_decode_attend. Set struct_size = sizeof(gqa_decode_params). */
typedef struct {
  uint32_t struct_size;
  /* q [batch, num_heads, head_dim]; row b*H + h is head h of sequence b ([usearch]
   * "row t * head_count + h of the queries is head h of token t"). */
  const void* q;
  int32_t q_dtype;           /* gqa_dtype */
  /* K and V caches [max_len, num_kv_heads, head_dim], row stride
   * num_kv_heads*head_dim ([attn.rs] KvCache). 16-byte aligned. */
  const void* k;
  const void* v;
  int32_t kv_dtype;          /* gqa_dtype */
  /* Arrow offsets [batch + 1], device int32: sequence b owns cache rows
   * offsets[b] .. offsets[b+1]-1. Must satisfy 0 <= offsets[b] <= offsets[b+1]
   * <= max_len; a violating sequence is treated as empty and flags
   * GQA_ERR_BAD_OFFSETS in the device error word. */
  const int32_t* offsets;
  int32_t batch;             /* B >= 0; 0 is a no-op */
  int32_t max_len;           /* rows allocated in the K/V caches (>= offsets[B]) */
  int32_t max_seq_len;       /* host hint: longest sequence; 0 => max_len. A hint
                                that is too small stays correct, only slower. */
  int32_t num_heads;         /* H >= 1 */
  int32_t num_kv_heads;      /* G; 0 => G = H. H % G must be 0, H / G <= 16 */
  int32_t head_dim;          /* D: 64 or 128 */
  float score_scale;         /* logit scale; 0 => 1/sqrt(head_dim); finite */
  /* Optional carry, one state per query row [B*H], folded into this call
   * ([usearch] DenseAttendConfig::carry). All-NULL = no carry. */
  gqa_state carry_in;
  /* Optional merged state out [B*H]; may alias carry_in exactly. */
  gqa_state state_out;
  /* Optional output [B, H, D] in out_dtype (acc / l, rounded to nearest even
   * for bf16; 0 for a row with no keys and no carry). */
  void* out;
  int32_t out_dtype;         /* gqa_dtype; conventionally q_dtype */
  /* Optional raw per-split states [B*H, num_splits] (m, l) and
   * [B*H, num_splits, D] (acc): split s of a sequence covers its keys
   * [s*chunk_len, (s+1)*chunk_len) (the last split also takes any remainder).
   * Splits with no keys are written as empty states. The carry is NOT folded
   * into these; merge them with gqa_softmax_merge. */
  gqa_state partials_out;
  int32_t num_splits;        /* 0 => chosen by the library's heuristic */
  /* Scratch: at least gqa_decode_workspace_size() bytes, 256-byte aligned,
   * initialised once with gqa_workspace_init. Not shared by calls that overlap. */
  void* workspace;
  size_t workspace_bytes;
  /* Optional additive logit bias, fp32 [max_len], one value per cache row, added
   * to scale*q.k of that row for every query head ([attn.rs] self_attn_incremental
   * `attn_bias`); -inf masks the key out. NULL = no bias. 4-byte aligned. */
  const float* bias;
  uint32_t flags;            /* GQA_FLAG_* bits; 0 = none */
} gqa_decode_params;

/* Bytes of workspace gqa_decode_attend needs for these params, and the
 * split plan it will use (either may be NULL). Host only; reads the current
 * device's SM count. At least out, state_out or partials_out must be set. */
gqa_status gqa_decode_workspace_size(const gqa_decode_params* params, size_t* bytes,
                                     int32_t* num_splits, int32_t* chunk_len);

/* Zero a workspace (its error word and its per-sequence merge tickets). Call
 * once after allocating a workspace. A call that reported GQA_ERR_TIMEOUT
 * produced no valid output, but it still leaves the tickets at zero: every
 * tile, including one whose pipeline wait gave up, takes its merge ticket and
 * the last one resets the counter, so the workspace stays usable as it is. */
gqa_status gqa_workspace_init(void* workspace, size_t workspace_bytes, gqa_stream_t stream);

/* Decode attention with a mergeable online-softmax state ([attn.rs]
 * self_attn_incremental / cross_attn_incremental without the projections;
 * [usearch] § Attention with its carry). One kernel launch on `stream`: the
 * split-KV partition kernel, whose last CTA per (sequence, KV head) merges that
 * sequence's splits and the carry when out or state_out is requested.
 * Asynchronous. */
gqa_status gqa_decode_attend(const gqa_decode_params* params, gqa_stream_t stream);

/* Decode attention exactly as gqa_decode_attend, for callers that cannot
 * provide scratch memory. The pages this library follows have no counterpart
 * of this entry point; it exists for deployment reasons only.
 *
 * Who needs it: code that must not allocate device memory or cannot obtain it
 * -- a plugin living inside a host engine that owns every device buffer and
 * gives the plugin no workspace, a fixed-budget or real-time service that
 * forbids allocations after start-up, or a callback in which cudaMalloc would
 * synchronise the device.
 *
 * params->workspace and params->workspace_bytes are ignored; every other field
 * means what it means for gqa_decode_attend, and the caller still passes all
 * inputs and outputs. The scratch is a 16 MiB device array inside the library
 * (the CUDA loader reserves it on every GPU that loads the library, until the
 * process exits). The call allocates nothing itself.
 *   - A call whose scratch need (gqa_decode_workspace_size) exceeds 16 MiB is
 *     refused with GQA_ERR_WORKSPACE.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it with the CUDA context it belongs to;
 *     make that first call before any stream capture. A later call under a
 *     different context of that device (after cudaDeviceReset, say) looks the
 *     address up again.
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls that may run at the same time on the GPU (different streams, or
 *     different host threads) race on it and must be serialised by the caller.
 *   - Each call starts by clearing, on the stream, the device error word and
 *     the merge tickets it will use, so nothing an earlier call left behind
 *     (an aborted call included) reaches its result. The error word is not
 *     readable through gqa_get_device_error; use gqa_decode_attend with a
 *     workspace to diagnose malformed offsets. */
gqa_status gqa_decode_attend_static_workspace(const gqa_decode_params* params, gqa_stream_t stream);

/* One decode step with the new token appended first ([attn.rs]
 * KvCache::push_kv, then self_attn_incremental): for every sequence b, cache row
 * offsets[b+1]-1 -- the caller's offsets already count the new token -- receives
 * k_new[b] and v_new[b] ([batch, num_kv_heads, head_dim], kv dtype, device,
 * 16-byte aligned), and the attention covers offsets[b]..offsets[b+1]-1 with the
 * new key included. params->k and params->v are WRITTEN (that one row per
 * sequence and KV head). A sequence with no row (offsets[b] == offsets[b+1]) has
 * no place for its token: it is skipped and GQA_ERR_BAD_OFFSETS is flagged in
 * the device error word (the pages' push_kv drops a token when the cache is
 * full). Everything else is as gqa_decode_attend. */
gqa_status gqa_decode_append_attend(const gqa_decode_params* params, const void* k_new,
                                    const void* v_new, gqa_stream_t stream);

/* A dictionary-coded KV cache (qualiaDB KvDictionary: a learned dictionary of
 * atoms; `reconstruct_from_words` is the f16-coefficient inverse of
 * `encode_to_words`, the compressed-cache read path). Every cache row of every
 * KV head is `words` 32-bit code words; a word holds the atom index in its high
 * 16 bits and the coefficient's IEEE binary16 bits in its low 16, and the row is
 * sum_w coeff_w * atoms[index_w] (a zero coefficient, as in padding words,
 * contributes nothing). K and V have their own dictionaries (pass the same
 * pointer twice for one shared dictionary). All device memory. */
typedef struct {
  const uint32_t* k_codes;   /* [max_len, num_kv_heads, words] */
  const uint32_t* v_codes;   /* [max_len, num_kv_heads, words] */
  int32_t words;             /* code words per row, 1..16 */
  const float* k_atoms;      /* [n_atoms, head_dim] fp32, 16-byte aligned */
  const float* v_atoms;      /* [n_atoms, head_dim] fp32, 16-byte aligned */
  int32_t n_atoms;           /* 1..65536, and heads_per_kv * n_atoms <= 12288 */
} gqa_kv_codes;

/* Decode attention over a dictionary-coded cache: exactly gqa_decode_attend on
 * the reconstructed rows, computed from the codes without rebuilding them
 * (logits from a table of each query head against every K atom; values as
 * per-atom weights applied to the V atoms once). params->k, ->v and ->kv_dtype
 * are ignored; q is fp32 or bf16; everything else (offsets, carry, bias,
 * partials, outputs, workspace, flags) as gqa_decode_attend. A code word naming
 * an atom >= n_atoms contributes nothing and flags GQA_ERR_BAD_CODES in the
 * device error word. The per-atom value weights are summed per round of keys (a
 * multiple of 512, at most 8192, as many as shared memory holds) in 32-bit fixed
 * point, scaled by a power of two to the round's largest possible sum
 * sum_j p_j sum_w |coeff_jw| (rounding error below 2^-30 of it per weight), so
 * results are bit-reproducible. The split plan is the coded kernel's own (one
 * CTA of 512 threads per SM), so size the workspace with
 * gqa_decode_coded_workspace_size. */
gqa_status gqa_decode_attend_coded(const gqa_decode_params* params, const gqa_kv_codes* codes,
                                   gqa_stream_t stream);

/* Workspace bytes and split plan of gqa_decode_attend_coded for these params
 * and codes (any output pointer may be NULL). Host only; reads the current
 * device's SM count. Validates as gqa_decode_attend_coded does. */
gqa_status gqa_decode_coded_workspace_size(const gqa_decode_params* params, const gqa_kv_codes* codes,
                                           size_t* bytes, int32_t* num_splits, int32_t* chunk_len);

/* Index-selected attention as an additive bias (metrale glm5next_dsa_ref,
 * `topk_to_mask`: the attention reads a mask built from an index row; repeated
 * indices collapse, the INVALID sentinel -1 and out-of-range entries drop).
 *   idx      device int32 [batch, width]: key positions relative to sequence b
 *   offsets  device int32 [batch + 1], as for gqa_decode_attend
 *   bias     device fp32 [max_len]: rows of every sequence become -inf except
 *            the selected ones, which become 0; other rows are not touched
 *   workspace  NULL, or a workspace whose error word takes GQA_ERR_BAD_OFFSETS
 * Pass the result as gqa_decode_params.bias. width may be 0 (everything masked). */
gqa_status gqa_topk_to_bias(const int32_t* idx, int32_t batch, int32_t width,
                            const int32_t* offsets, int32_t max_len, float* bias,
                            void* workspace, gqa_stream_t stream);

/* Merge num_states states per row ([usearch] carry: partial-softmax rescaling):
 *   M = max m_i,  L = sum l_i e^{m_i - M},  ACC = sum acc_i e^{m_i - M}
 * over the non-empty states (l_i != 0) of each row, plus carry_in when given.
 *   states      m, l [rows, num_states], acc [rows, num_states, head_dim]
 *   carry_in    NULL or a state [rows]
 *   merged_out  NULL or a state [rows]; may alias carry_in, not states
 *   out         NULL or [rows, head_dim] in out_dtype: ACC / L (0 when L == 0)
 * At least one of merged_out / out must be given. rows may be 0. */
gqa_status gqa_softmax_merge(const gqa_state* states, int32_t rows, int32_t num_states,
                             int32_t head_dim, const gqa_state* carry_in,
                             const gqa_state* merged_out, void* out, int32_t out_dtype,
                             gqa_stream_t stream);

/* The same merge for states laid out [num_states, rows] (m, l) and
 * [num_states, rows, head_dim] (acc) -- one block per contributor, the layout an
 * all-gather of per-rank states produces (context-parallel decode: each rank
 * attends over its slice of every sequence's keys, the states are exchanged,
 * and this merge folds them with the carry). Arguments otherwise as
 * gqa_softmax_merge. */
gqa_status gqa_softmax_merge_gathered(const gqa_state* states, int32_t rows, int32_t num_states,
                                      int32_t head_dim, const gqa_state* carry_in,
                                      const gqa_state* merged_out, void* out, int32_t out_dtype,
                                      gqa_stream_t stream);

/* out = acc / l per row (0 when l == 0), cast to out_dtype ([usearch]: outputs
 * land already divided by the partition). state [rows], out [rows, head_dim]. */
gqa_status gqa_state_finalize(const gqa_state* state, int32_t rows, int32_t head_dim, void* out,
                              int32_t out_dtype, gqa_stream_t stream);

/* Synchronise `stream`, read and clear the workspace's device error word.
 * Returns GQA_OK, GQA_ERR_BAD_OFFSETS, GQA_ERR_TIMEOUT or GQA_ERR_BAD_CODES
 * (the first set, in that order). */
gqa_status gqa_get_device_error(void* workspace, gqa_stream_t stream);

/* The split plan of the heuristic, exposed for inspection and tests (host only):
 * chunk_len is a multiple of 64 and num_splits = ceil(max_seq_len / chunk_len).
 * total_rows is the expected sum of sequence lengths (<= batch*max_seq_len;
 * equal means every sequence has max_seq_len keys); sm_count and ctas_per_sm
 * describe how many partition CTAs the GPU holds at once. */
gqa_status gqa_plan_splits(int32_t batch, int32_t num_kv_heads, int32_t max_seq_len,
                           int64_t total_rows, int32_t sm_count, int32_t ctas_per_sm,
                           int32_t* chunk_len, int32_t* num_splits);

/* Human-readable name of a status. Never NULL. */
const char* gqa_status_string(gqa_status status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t gqa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_DECODE_H */
