// gqa_oracle.cpp -- f64 CPU oracle for single-token grouped-query decode attention.
//
// TEST INFRASTRUCTURE ONLY. This file is the checker the CUDA path is compared
// against. Only the test suite, the smoke check and the benchmark's CPU-baseline
// leg may load it; the library's product path never does. It shares no code,
// header, table or constant with the CUDA sources, and includes none of them.
//
// What it computes (plain definition, no blocking, fusion or reordering):
//
//   For every sequence b and query head h, with kv_repeat = H / G and the group
//   g = floor(h / kv_repeat)  (needle_core attn.rs, `self_attn_incremental`:
//   "which KV head serves this Q head"), and every cached key j of sequence b,
//   i.e. j in [offsets[b], offsets[b+1])  (USearch linear algebra: ragged runs
//   as Apache Arrow offsets):
//
//     s_j   = scale * sum_c q[b,h,c] * K[j,g,c]         (attn.rs: dot * scale,
//             scale = score_scale, or head_dim^-0.5 when score_scale == 0
//             -- USearch `DenseAttendConfig::score_scale`, attn.rs `powf(hd,-0.5)`)
//     m     = max( max_j s_j , m_carry )                (running maximum)
//     l     = sum_j e^{s_j - m} + l_carry e^{m_carry - m}   (partition)
//     acc   = sum_j e^{s_j - m} V[j,g,:] + acc_carry e^{m_carry - m}
//     out   = acc / l                                   (USearch § Attention:
//             outputs already divided by the partition)
//
//   With an additive bias row (needle_core attn.rs `self_attn_incremental`,
//   `attn_bias`: added to the scaled score of position t), the logit of key j
//   is s_j = scale * q.k_j + bias[j], bias indexed by cache row; a bias of
//   -inf masks the key out (weight 0).
//
//   The max-shifted exponentials follow the exact-softmax recipe of the
//   cortiq_engine NystromState example `trial` (f64 exp of logit - max).
//   A carry state with l == 0 is the empty state and contributes nothing,
//   whatever its m. A row with no keys and no carry yields m = -inf, l = 0,
//   acc = 0 and out = 0 (an all-masked softmax gives weight 0, not NaN:
//   metrale glm5next_dsa_ref `pool_states`).
//
// Inputs arrive as stored: fp32, or bf16 bit patterns (uint16) which are
// widened exactly to f64. All arithmetic is f64, two passes per row (max, then
// sums), multithreaded over (b, h) rows with std::thread.
//
// Build: oracle/build.py (gcc, plain C++17). ORACLE_MUTATION=<n> compiles a
// deliberately wrong variant used only by the mutation test that proves the
// pins are sensitive.

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif

namespace {

// bf16 -> f64: a bf16 value is the upper half of an IEEE binary32 pattern, so
// shifting it into place and widening is exact.
inline double bf16_bits_to_f64(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// IEEE binary16 bits -> f64, from the format's definition (sign, 5-bit biased
// exponent, 10-bit fraction; exponent 0 is subnormal, 31 is inf/NaN).
inline double f16_bits_to_f64(uint16_t bits) {
  const int sign = bits >> 15;
  const int e = (bits >> 10) & 0x1F;
  const int f = bits & 0x3FF;
  double v;
  if (e == 0)
#if ORACLE_MUTATION == 16
    v = std::ldexp(static_cast<double>(f), -25);                // subnormals halved
#else
    v = std::ldexp(static_cast<double>(f), -24);
#endif
  else if (e == 31)
    v = f ? std::numeric_limits<double>::quiet_NaN() : std::numeric_limits<double>::infinity();
  else
    v = std::ldexp(static_cast<double>(1024 + f), e - 25);
  return sign ? -v : v;
}

// Element of a stored array: kind 0 = fp32, 1 = bf16 bits, 2 = f64.
inline double load_elem(const void* base, int is_bf16, int64_t idx) {
  if (is_bf16 == 1) return bf16_bits_to_f64(static_cast<const uint16_t*>(base)[idx]);
  if (is_bf16 == 2) return static_cast<const double*>(base)[idx];
  return static_cast<double>(static_cast<const float*>(base)[idx]);
}

const double kNegInf = -std::numeric_limits<double>::infinity();

struct AttendArgs {
  const void* q; int q_bf16;
  const void* k; const void* v; int kv_bf16;
  const int32_t* offsets;
  int B, H, G, D;
  double scale;
  const float* bias;      // [rows] additive logit bias per cache row, or null
  const float* cm; const float* cl; const float* cacc;
  double* om; double* ol; double* oacc; double* out;
};

// One query row (b, h) -> (m, l, acc, out), written at output index r.
void attend_one_row(const AttendArgs& a, int64_t row, int64_t r, std::vector<double>& s) {
  const int b = static_cast<int>(row / a.H);
  const int h = static_cast<int>(row % a.H);
  const int kv_repeat = a.H / a.G;
#if ORACLE_MUTATION == 1
  const int g = h % a.G;                      // wrong head map (interleaved)
#else
  const int g = h / kv_repeat;                // contiguous groups
#endif
  const int D = a.D;
  int64_t j0 = a.offsets[b];
  int64_t j1 = a.offsets[b + 1];
#if ORACLE_MUTATION == 7
  if (j1 > j0) j1 -= 1;                       // drops the last key
#endif
  const int64_t n = j1 > j0 ? j1 - j0 : 0;
  const int64_t kv_row_stride = static_cast<int64_t>(a.G) * D;

  // Pass 1: logits and their maximum.
  s.resize(static_cast<size_t>(n));
  double m = kNegInf;
  for (int64_t t = 0; t < n; ++t) {
    const int64_t j = j0 + t;
#if ORACLE_MUTATION == 5
    const int64_t kbase = static_cast<int64_t>(g) * (a.offsets[a.B]) * D + j * D;  // [G, rows, D] misread
#else
    const int64_t kbase = j * kv_row_stride + static_cast<int64_t>(g) * D;
#endif
    double dot = 0.0;
    for (int c = 0; c < D; ++c)
      dot += load_elem(a.q, a.q_bf16, row * D + c) * load_elem(a.k, a.kv_bf16, kbase + c);
#if ORACLE_MUTATION == 2
    s[t] = dot;                               // scale dropped
#else
    s[t] = a.scale * dot;
#endif
    if (a.bias != nullptr) {
#if ORACLE_MUTATION == 9
      s[t] = a.scale * (dot + static_cast<double>(a.bias[j]));   // bias inside the scale
#elif ORACLE_MUTATION == 13
      s[t] += static_cast<double>(a.bias[t]);                     // bias row of the sequence position
#else
      s[t] += static_cast<double>(a.bias[j]);
#endif
    }
    if (s[t] > m) m = s[t];
  }

  const bool has_carry = a.cl != nullptr && a.cl[row] != 0.0f;
  double mc = 0.0, lc = 0.0;
  if (has_carry) {
    mc = static_cast<double>(a.cm[row]);
    lc = static_cast<double>(a.cl[row]);
    if (mc > m) m = mc;
  }
#if ORACLE_MUTATION == 14
  if (a.cl != nullptr && !has_carry && static_cast<double>(a.cm[row]) > m) m = a.cm[row];   // empty carry in the max
#endif

  double* acc = a.oacc + r * D;
  for (int c = 0; c < D; ++c) acc[c] = 0.0;
  double l = 0.0;

  if (m != kNegInf) {
    // Pass 2: max-shifted exponentials, partition and weighted value sum.
    for (int64_t t = 0; t < n; ++t) {
      const int64_t j = j0 + t;
      const double p = std::exp(s[t] - m);
      l += p;
#if ORACLE_MUTATION == 8
      const void* vsrc = a.k;                 // keys used as values
#else
      const void* vsrc = a.v;
#endif
      const int64_t vbase = j * kv_row_stride + static_cast<int64_t>(g) * D;
      for (int c = 0; c < D; ++c) acc[c] += p * load_elem(vsrc, a.kv_bf16, vbase + c);
    }
    if (has_carry) {
#if ORACLE_MUTATION == 3
      const double w = std::exp(m - mc);      // rescale factor with the sign flipped
#else
      const double w = std::exp(mc - m);
#endif
      l += lc * w;
#if ORACLE_MUTATION == 12
      for (int c = 0; c < D; ++c) acc[c] += static_cast<double>(a.cacc[row * D + c]);   // acc not rescaled
#else
      for (int c = 0; c < D; ++c) acc[c] += static_cast<double>(a.cacc[row * D + c]) * w;
#endif
    }
  }

  a.om[r] = (l == 0.0) ? kNegInf : m;
  a.ol[r] = l;
  double* out = a.out + r * D;
  for (int c = 0; c < D; ++c) {
#if ORACLE_MUTATION == 4
    out[c] = acc[c];                          // not divided by the partition
#else
    out[c] = (l == 0.0) ? 0.0 : acc[c] / l;
#endif
  }
}

template <class F>
void parallel_rows(int64_t n_rows, int n_threads, F&& fn) {
  if (n_threads <= 0) {
    unsigned hc = std::thread::hardware_concurrency();
    n_threads = hc == 0 ? 1 : static_cast<int>(hc);
  }
  if (n_threads > n_rows) n_threads = static_cast<int>(n_rows > 0 ? n_rows : 1);
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (;;) {
      const int64_t r = next.fetch_add(1);
      if (r >= n_rows) break;
      fn(r);
    }
  };
  if (n_threads == 1) {
    worker();
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(static_cast<size_t>(n_threads));
  for (int t = 0; t < n_threads; ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Returns the number of worker threads a call with n_threads <= 0 uses.
int oracle_default_threads(void) {
  unsigned hc = std::thread::hardware_concurrency();
  return hc == 0 ? 1 : static_cast<int>(hc);
}

// Exact decode attention (definition at the top of this file).
//   q        [B, H, D]            fp32 or bf16 bits (q_bf16)
//   k, v     [rows, G, D]         fp32 or bf16 bits (kv_bf16)
//   offsets  [B+1]                host int32, Arrow offsets into the rows
//   carry    cm/cl [B*H], cacc [B*H, D] fp32, or all null
//   row_list the (b*H + h) rows to evaluate, or null for all B*H rows
//   outputs  om/ol [n], oacc/out [n, D] f64 for the n evaluated rows
// Returns 0 on success, -1 on a malformed argument.
int oracle_decode_attend(const void* q, int q_bf16, const void* k, const void* v, int kv_bf16,
                         const int32_t* offsets, int B, int H, int G, int D, double score_scale,
                         const float* bias, const float* cm, const float* cl, const float* cacc,
                         const int64_t* row_list, int64_t n_rows, double* om, double* ol,
                         double* oacc, double* out, int n_threads) {
  if (B < 0 || H <= 0 || G <= 0 || D <= 0 || H % G != 0) return -1;
  if (!q || !k || !v || !offsets || !om || !ol || !oacc || !out) return -1;
  if ((cm == nullptr) != (cl == nullptr) || (cm == nullptr) != (cacc == nullptr)) return -1;
  AttendArgs a{q, q_bf16, k, v, kv_bf16, offsets, B, H, G, D,
               score_scale != 0.0 ? score_scale : 1.0 / std::sqrt(static_cast<double>(D)), bias,
               cm, cl, cacc, om, ol, oacc, out};
  const int64_t total = static_cast<int64_t>(B) * H;
  const int64_t n = row_list ? n_rows : total;
  for (int64_t i = 0; row_list && i < n; ++i)
    if (row_list[i] < 0 || row_list[i] >= total) return -1;
  parallel_rows(n, n_threads, [&](int64_t i) {
    thread_local std::vector<double> s;
    attend_one_row(a, row_list ? row_list[i] : i, i, s);
  });
  return 0;
}

// Merge of online-softmax states over the same query rows (USearch linear
// algebra, `DenseAttendConfig::carry` / `DenseSoftmaxState`: partial-softmax
// rescaling). For each row, with states i = 0..S-1 (and the carry, if given)
// and only the non-empty ones (l_i != 0) taking part:
//     M   = max_i m_i
//     L   = sum_i l_i e^{m_i - M}
//     ACC = sum_i acc_i e^{m_i - M}
//     out = ACC / L          (0 when every state is empty)
// States are fp32 as stored, row-major [rows, S] (m, l) and [rows, S, D] (acc).
int oracle_softmax_merge(const float* m, const float* l, const float* acc, int64_t rows, int S,
                         int D, const float* cm, const float* cl, const float* cacc, double* om,
                         double* ol, double* oacc, double* out, int n_threads) {
  if (rows < 0 || S < 0 || D <= 0 || !om || !ol || !oacc || !out) return -1;
  if (S > 0 && (!m || !l || !acc)) return -1;
  if ((cm == nullptr) != (cl == nullptr) || (cm == nullptr) != (cacc == nullptr)) return -1;
  parallel_rows(rows, n_threads, [&](int64_t r) {
    double M = kNegInf;
    for (int i = 0; i < S; ++i) {
      const int64_t si = r * S + i;
#if ORACLE_MUTATION == 15
      if (static_cast<double>(m[si]) > M) M = m[si];                // empty states in the max
#else
      if (l[si] != 0.0f && static_cast<double>(m[si]) > M) M = m[si];
#endif
    }
    const bool has_carry = cl != nullptr && cl[r] != 0.0f;
    if (has_carry && static_cast<double>(cm[r]) > M) M = cm[r];
    double L = 0.0;
    double* a = oacc + r * D;
    for (int c = 0; c < D; ++c) a[c] = 0.0;
    if (M != kNegInf) {
      for (int i = 0; i < S; ++i) {
        const int64_t si = r * S + i;
        if (l[si] == 0.0f) continue;
#if ORACLE_MUTATION == 6
        const double w = 1.0;                 // partials added without rescaling
#else
        const double w = std::exp(static_cast<double>(m[si]) - M);
#endif
        L += static_cast<double>(l[si]) * w;
        for (int c = 0; c < D; ++c) a[c] += static_cast<double>(acc[si * D + c]) * w;
      }
      if (has_carry) {
        const double w = std::exp(static_cast<double>(cm[r]) - M);
        L += static_cast<double>(cl[r]) * w;
        for (int c = 0; c < D; ++c) a[c] += static_cast<double>(cacc[r * D + c]) * w;
      }
    }
    om[r] = (L == 0.0) ? kNegInf : M;
    ol[r] = L;
    for (int c = 0; c < D; ++c) out[r * D + c] = (L == 0.0) ? 0.0 : a[c] / L;
  });
  return 0;
}

// Index-selected attention as a mask (metrale glm5next_dsa_ref, `topk_to_mask`:
// the attention reads a visibility mask built from an index row; repeated
// indices collapse, the INVALID sentinel -1 and out-of-range entries are
// dropped). For decode, sequence b's index row idx[b, 0..width) holds key
// positions relative to the sequence; the result is an additive bias per cache
// row: 0 for a selected key of b, -inf for every other row of b. Rows outside
// every sequence are left untouched.
int oracle_topk_to_bias(const int32_t* idx, int B, int width, const int32_t* offsets, float* bias,
                        int64_t rows) {
  if (B < 0 || width < 0 || !offsets || !bias || (width > 0 && !idx)) return -1;
  const float ninf = -std::numeric_limits<float>::infinity();
  for (int b = 0; b < B; ++b) {
    const int64_t o0 = offsets[b], o1 = offsets[b + 1];
    if (o0 < 0 || o1 < o0 || o1 > rows) return -1;
    for (int64_t r = o0; r < o1; ++r) bias[r] = ninf;
    for (int w = 0; w < width; ++w) {
      const int64_t t = idx[static_cast<int64_t>(b) * width + w];
#if ORACLE_MUTATION == 10
      if (t >= 0 && o0 + t <= o1) bias[o0 + t] = 0.0f;    // admits one past the end
#else
      if (t >= 0 && t < o1 - o0) bias[o0 + t] = 0.0f;
#endif
    }
  }
  return 0;
}

// Reconstruction of a dictionary-coded cache (qualiaDB KvDictionary:
// `reconstruct_from_words`, the f16-coefficient inverse of `encode_to_words`;
// `reconstruct`: sum of coeff * atom). Every cache row of every KV head is
// `words` code words; word w holds the atom index in its high 16 bits and the
// coefficient's IEEE binary16 bits in its low 16 bits (a zero coefficient,
// as in padding words, reconstructs to nothing). atoms [n_atoms, D] fp32.
// out [rows*G, D] f64: out_r = sum_w f16(coeff_w) * atoms[index_w].
// Returns -1 if an index is out of range.
int oracle_reconstruct_words(const uint32_t* codes, int64_t rows_x_heads, int words, const float* atoms,
                             int n_atoms, int D, double* out) {
  if (!codes || !atoms || !out || words <= 0 || n_atoms <= 0 || D <= 0) return -1;
  for (int64_t r = 0; r < rows_x_heads; ++r) {
    double* o = out + r * D;
    for (int c = 0; c < D; ++c) o[c] = 0.0;
    for (int w = 0; w < words; ++w) {
      const uint32_t word = codes[r * words + w];
#if ORACLE_MUTATION == 11
      const int idx = static_cast<int>(word & 0xFFFF);              // fields swapped
      const double coeff = f16_bits_to_f64(static_cast<uint16_t>(word >> 16));
#else
      const int idx = static_cast<int>(word >> 16);
      const double coeff = f16_bits_to_f64(static_cast<uint16_t>(word & 0xFFFF));
#endif
      if (coeff == 0.0) continue;
      if (idx >= n_atoms) return -1;
      for (int c = 0; c < D; ++c) o[c] += coeff * static_cast<double>(atoms[static_cast<int64_t>(idx) * D + c]);
    }
  }
  return 0;
}

double oracle_f16_to_f64(uint16_t bits) { return f16_bits_to_f64(bits); }

// bf16 bits -> f64, exposed so the pins can check the widening on fixed patterns.
double oracle_bf16_to_f64(uint16_t bits) { return bf16_bits_to_f64(bits); }

}  // extern "C"
