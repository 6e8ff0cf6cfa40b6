// Plain fp64 CPU oracle for exact attention.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct reference that the
// CUDA path is checked against.  Only the tests, the smoke check and the benchmark's CPU
// baseline may load it; the library never does.  It shares no code with the CUDA path.
//
// What it computes is the plain definition, materialised row by row in the three steps of
// standard attention ("FlashAttention notes", section 2 "Standard Attention IO bottleneck";
// "LLM basics: from Attention to FlashAttention", chapter 3 section 4):
//
//   s_j  = scale * <q_i, k_j>                  for every allowed key j   (the S row)
//   m    = max_j s_j,  p_j = exp(s_j - m),  l = sum_j p_j                 (the P row,
//          safe softmax, chapter 3 section 1 of the same tutorial)
//   o_i  = sum_j p_j v_j / l,  lse_i = m + ln l                           (P times V)
//
// Allowed keys: j < nk (the sequence's key count); causal adds j <= i + (nk - nq), the
// bottom-right alignment that makes a single query see the whole cache (chapter 1 section 7
// "Masked Self-Attention" says token t sees tokens 1..t).  GQA maps query head h to key/value
// head h / (Hq / Hkv) (chapter 2 section 7).  A row with no allowed key gives o = 0 and
// lse = -inf.
//
// The online (m, l) merge ("FlashAttention notes", section 4 equations for m_new and l_new)
// is provided separately for the self-checks and the split-KV merge checks; the attention
// function never merges.
//
// Planted-mistake switches (ORACLE_PLANT_*) exist only so that a test can build broken
// copies of this file and show that the pins catch each mistake.  The normal build defines
// none of them.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <limits>
#include <thread>
#include <vector>

namespace {

constexpr double kNegInf = -std::numeric_limits<double>::infinity();

struct Problem {
  const float* q;
  const float* k;
  const float* v;
  int B, Hq, Hkv, Nq, Nk, d;
  double scale;
  int causal;
  const int32_t* cu;       // varlen offsets (B+1) or null
  const int32_t* kv_lens;  // per-batch key count limit or null
};

// Row geometry of query (b, h, i): pointers to its q row and to the first key/value rows
// of its head, the stride between consecutive keys, and the allowed key range [0, jmax).
struct RowView {
  const float* qrow;
  const float* kbase;
  const float* vbase;
  int64_t kstride;
  int64_t jmax;  // allowed keys are j in [0, jmax); may be <= 0
  int64_t orow;  // index of this row in o (units of d) and lse position
  int64_t lse_index;
  bool valid;
};

RowView view_row(const Problem& P, int b, int h, int64_t i) {
  RowView r{};
  const int G = P.Hq / P.Hkv;
#ifdef ORACLE_PLANT_GQA_MODULO
  const int g = h % P.Hkv;
#else
  const int g = h / G;
#endif
  int64_t q0, k0, nq, nk;
  if (P.cu) {
    q0 = P.cu[b];
    k0 = P.cu[b];
    nq = P.cu[b + 1] - P.cu[b];
#ifdef ORACLE_PLANT_VARLEN_SHORT_KEYS
    nk = nq > 0 ? nq - 1 : 0;
#else
    nk = nq;
#endif
  } else {
    q0 = (int64_t)b * P.Nq;
    k0 = (int64_t)b * P.Nk;
    nq = P.Nq;
    nk = P.Nk;
  }
  if (P.kv_lens) nk = std::min<int64_t>(nk, P.kv_lens[b]);
  r.valid = i < nq;
  if (!r.valid) return r;
  r.qrow = P.q + ((q0 + i) * P.Hq + h) * (int64_t)P.d;
  r.kbase = P.k + (k0 * P.Hkv + g) * (int64_t)P.d;
  r.vbase = P.v + (k0 * P.Hkv + g) * (int64_t)P.d;
  r.kstride = (int64_t)P.Hkv * P.d;
  int64_t jmax = nk;
  if (P.causal) {
#ifdef ORACLE_PLANT_CAUSAL_OFF_BY_ONE
    jmax = std::min<int64_t>(jmax, i + (nk - nq));
#else
    jmax = std::min<int64_t>(jmax, i + (nk - nq) + 1);
#endif
  }
  r.jmax = jmax;
  r.orow = (q0 + i) * P.Hq + h;
  r.lse_index = P.cu ? (int64_t)h * P.Nq + q0 + i : ((int64_t)b * P.Hq + h) * P.Nq + i;
  return r;
}

// One query row, materialised: S row, then P row, then P times V.
void attend_row(const Problem& P, const RowView& r, std::vector<double>& s, double* o, double* lse) {
  const int d = P.d;
  if (r.jmax <= 0) {
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    *lse = kNegInf;
    return;
  }
  s.resize((size_t)r.jmax);
  // step 1: scores
  for (int64_t j = 0; j < r.jmax; ++j) {
#ifdef ORACLE_PLANT_QV_SWAP
    const float* kr = r.vbase + j * r.kstride;
#else
    const float* kr = r.kbase + j * r.kstride;
#endif
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += (double)r.qrow[c] * (double)kr[c];
#ifdef ORACLE_PLANT_NO_SCALE
    s[(size_t)j] = acc;
#else
    s[(size_t)j] = P.scale * acc;
#endif
  }
  // step 2: safe softmax numerators and their sum
  double m = kNegInf;
  for (int64_t j = 0; j < r.jmax; ++j) m = std::max(m, s[(size_t)j]);
  double l = 0.0;
  for (int64_t j = 0; j < r.jmax; ++j) {
#ifdef ORACLE_PLANT_SIGN
    s[(size_t)j] = std::exp(m - s[(size_t)j]);
#else
    s[(size_t)j] = std::exp(s[(size_t)j] - m);
#endif
    l += s[(size_t)j];
  }
  // step 3: P times V, normalised
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  for (int64_t j = 0; j < r.jmax; ++j) {
#ifdef ORACLE_PLANT_QV_SWAP
    const float* vr = r.kbase + j * r.kstride;
#else
    const float* vr = r.vbase + j * r.kstride;
#endif
    const double p = s[(size_t)j];
    for (int c = 0; c < d; ++c) o[c] += p * (double)vr[c];
  }
  for (int c = 0; c < d; ++c) o[c] /= l;
#ifdef ORACLE_PLANT_LSE_NO_MAX
  *lse = std::log(l);
#else
  *lse = m + std::log(l);
#endif
}

int check_problem(const Problem& P) {
  if (!P.q || !P.k || !P.v) return 1;
  if (P.B < 0 || P.Hq <= 0 || P.Hkv <= 0 || P.Nq < 0 || P.Nk < 0 || P.d <= 0) return 1;
  if (P.Hq % P.Hkv != 0) return 1;
  if (P.cu && P.Nq != P.Nk) return 1;
  return 0;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F&& body) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  nthreads = (int)std::min<int64_t>(nthreads, std::max<int64_t>(n, 1));
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    std::vector<double> scratch;
    for (;;) {
      const int64_t t = next.fetch_add(1);
      if (t >= n) break;
      body(t, scratch);
    }
  };
  if (nthreads == 1) {
    worker();
    return;
  }
  std::vector<std::thread> pool;
  for (int t = 0; t < nthreads; ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Safe softmax of one row ("LLM basics", chapter 3 section 1: subtract the row max; the
// factor exp(-m) cancels between numerator and denominator).
int oracle_softmax(const double* x, int64_t n, double* p) {
  if (n <= 0 || !x || !p) return 1;
  double m = kNegInf;
  for (int64_t j = 0; j < n; ++j) m = std::max(m, x[j]);
  if (m == kNegInf) {
    for (int64_t j = 0; j < n; ++j) p[j] = 0.0;
    return 0;
  }
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    p[j] = std::exp(x[j] - m);
    l += p[j];
  }
  for (int64_t j = 0; j < n; ++j) p[j] /= l;
  return 0;
}

// The statistics a block carries: m = max x, l = sum exp(x - m) ("FlashAttention notes",
// section 4).  An empty or fully masked block has m = -inf and l = 0.
int oracle_row_stats(const double* x, int64_t n, double* m_out, double* l_out) {
  if (n < 0 || !m_out || !l_out) return 1;
  double m = kNegInf;
  for (int64_t j = 0; j < n; ++j) m = std::max(m, x[j]);
  double l = 0.0;
  if (m != kNegInf)
    for (int64_t j = 0; j < n; ++j) l += std::exp(x[j] - m);
  *m_out = m;
  *l_out = l;
  return 0;
}

// Merge of two blocks' statistics, the rule of "FlashAttention notes" section 4:
//   m_new = max(m1, m2);  l_new = exp(m1 - m_new) l1 + exp(m2 - m_new) l2.
// A block with m = -inf contributes weight 0.
void oracle_merge_stats(double m1, double l1, double m2, double l2, double* m_out, double* l_out) {
  const double mn = std::max(m1, m2);
  if (mn == kNegInf) {
    *m_out = kNegInf;
    *l_out = 0.0;
    return;
  }
  const double w1 = (m1 == kNegInf) ? 0.0 : std::exp(m1 - mn);
  const double w2 = (m2 == kNegInf) ? 0.0 : std::exp(m2 - mn);
  *m_out = mn;
  *l_out = w1 * l1 + w2 * l2;
}

// Merge of n partial results (m_s, l_s, acc_s[d]), each acc_s the un-normalised sum
// sum_j exp(s_j - m_s) v_j over its block, applied pairwise in order with the rule above
// (the accumulators are rescaled by the same weights as l).  Writes the merged m, l and the
// normalised output acc / l (zero when l == 0).
int oracle_merge_partials(const double* m, const double* l, const double* acc, int64_t n, int d,
                          double* m_out, double* l_out, double* o_out) {
  if (n < 0 || d <= 0) return 1;
  double M = kNegInf, L = 0.0;
  std::vector<double> A((size_t)d, 0.0);
  for (int64_t s = 0; s < n; ++s) {
    double mn, ln;
    oracle_merge_stats(M, L, m[s], l[s], &mn, &ln);
    if (mn == kNegInf) continue;
    const double wa = (M == kNegInf) ? 0.0 : std::exp(M - mn);
    const double wb = (m[s] == kNegInf) ? 0.0 : std::exp(m[s] - mn);
    for (int c = 0; c < d; ++c) A[(size_t)c] = wa * A[(size_t)c] + wb * acc[s * (int64_t)d + c];
    M = mn;
    L = ln;
  }
  *m_out = M;
  *l_out = L;
  for (int c = 0; c < d; ++c) o_out[c] = (L > 0.0) ? A[(size_t)c] / L : 0.0;
  return 0;
}

// Full attention.  Layouts (d innermost everywhere):
//   fixed length: q, o [B, Nq, Hq, d]; k, v [B, Nk, Hkv, d]; lse [B, Hq, Nq]
//   varlen (cu != null, Nq == Nk == total rows): q, o [total, Hq, d]; k, v [total, Hkv, d];
//            lse [Hq, total]; sequence b owns rows [cu[b], cu[b+1])
//   kv_lens (optional, fixed length only): batch b uses keys j < kv_lens[b]
// Inputs are float32 arrays holding the stored (bf16 or fp32) values exactly; all
// arithmetic is fp64.  Threads run over (b, h) rows; nthreads <= 0 uses all cores.
int oracle_attention(const float* q, const float* k, const float* v, int B, int Hq, int Hkv, int Nq,
                     int Nk, int d, double scale, int causal, const int32_t* cu_seqlens,
                     const int32_t* kv_lens, double* o, double* lse, int nthreads) {
  Problem P{q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal, cu_seqlens, kv_lens};
  if (check_problem(P) || !o || !lse) return 1;
  if (cu_seqlens && kv_lens) return 1;
  const int64_t rows_per_seq = Nq;  // varlen: an upper bound, rows past the sequence are skipped
  const int64_t units = (int64_t)B * Hq;
  parallel_for(units, nthreads, [&](int64_t u, std::vector<double>& s) {
    const int b = (int)(u / Hq), h = (int)(u % Hq);
    for (int64_t i = 0; i < rows_per_seq; ++i) {
      RowView r = view_row(P, b, h, i);
      if (!r.valid) break;
      attend_row(P, r, s, o + r.orow * d, lse + r.lse_index);
    }
  });
  return 0;
}

// Selected rows only: rows holds nrows triples (b, h, i) (i is the row within sequence b).
// Row r's output goes to o[r*d .. r*d+d) and lse[r].
int oracle_attention_rows(const float* q, const float* k, const float* v, int B, int Hq, int Hkv,
                          int Nq, int Nk, int d, double scale, int causal, const int32_t* cu_seqlens,
                          const int32_t* kv_lens, const int64_t* rows, int64_t nrows, double* o,
                          double* lse, int nthreads) {
  Problem P{q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal, cu_seqlens, kv_lens};
  if (check_problem(P) || !o || !lse || !rows || nrows < 0) return 1;
  for (int64_t t = 0; t < nrows; ++t) {
    const int64_t b = rows[3 * t], h = rows[3 * t + 1], i = rows[3 * t + 2];
    if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0) return 1;
    if (!view_row(P, (int)b, (int)h, i).valid) return 1;
  }
  parallel_for(nrows, nthreads, [&](int64_t t, std::vector<double>& s) {
    RowView r = view_row(P, (int)rows[3 * t], (int)rows[3 * t + 1], rows[3 * t + 2]);
    attend_row(P, r, s, o + t * d, lse + t);
  });
  return 0;
}

// Gradients of the attention above with respect to q, k and v, for an upstream gradient dout
// of o (same layout as o).  "FlashAttention notes", section 5.2 (backward): the backward
// rebuilds P from q, k and the softmax statistics instead of storing it, then dV = P^T dO and
// dP = dO V^T; the remaining steps are the derivative of the row softmax.  Here every row is
// materialised again in fp64 from q, k, v alone (this oracle keeps no forward state):
//
//   p_j  = softmax_j(s),  o_i = sum_j p_j v_j                       (as in the forward)
//   dp_j = <dout_i, v_j>,  D_i = sum_j p_j dp_j  (= <dout_i, o_i>)
//   ds_j = p_j (dp_j - D_i)                      (softmax derivative)
//   dq_i  = scale * sum_j ds_j k_j
//   dk_j += scale * ds_j q_i,   dv_j += p_j dout_i                  (summed over rows and over
//                                                                  the query heads of the group)
// Layouts as in oracle_attention (dq like q, dk/dv like k/v); fixed length or varlen.  Threads
// run over (sequence, key/value head) groups, which own disjoint dk/dv and dq rows.
int oracle_attention_bwd(const float* q, const float* k, const float* v, const float* dout, int B, int Hq,
                         int Hkv, int Nq, int Nk, int d, double scale, int causal, const int32_t* cu_seqlens,
                         double* dq, double* dk, double* dv, int nthreads) {
  Problem P{q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal, cu_seqlens, nullptr};
  if (check_problem(P) || !dout || !dq || !dk || !dv) return 1;
  const int G = Hq / Hkv;
  const int64_t rows_q = cu_seqlens ? (int64_t)Nq : (int64_t)B * Nq;
  const int64_t rows_k = cu_seqlens ? (int64_t)Nk : (int64_t)B * Nk;
  for (int64_t t = 0; t < rows_q * Hq * d; ++t) dq[t] = 0.0;
  for (int64_t t = 0; t < rows_k * Hkv * d; ++t) dk[t] = dv[t] = 0.0;
  const int64_t units = (int64_t)B * Hkv;
  parallel_for(units, nthreads, [&](int64_t u, std::vector<double>& scratch) {
    const int b = (int)(u / Hkv), g = (int)(u % Hkv);
    std::vector<double> o((size_t)d);
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int64_t i = 0; i < Nq; ++i) {
        RowView r = view_row(P, b, h, i);
        if (!r.valid) break;
        if (r.jmax <= 0) continue;  // no allowed key: o = 0 and no gradient flows
        const int64_t n = r.jmax;
        scratch.resize((size_t)(3 * n));
        double* s = scratch.data();
        double* pr = s + n;
        double* dp = pr + n;
        for (int64_t j = 0; j < n; ++j) {
          const float* kj = r.kbase + j * r.kstride;
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += (double)r.qrow[c] * (double)kj[c];
          s[j] = P.scale * acc;
        }
        double m = kNegInf;
        for (int64_t j = 0; j < n; ++j) m = std::max(m, s[j]);
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
          pr[j] = std::exp(s[j] - m);
          l += pr[j];
        }
        for (int64_t j = 0; j < n; ++j) pr[j] /= l;
        const float* dorow = dout + r.orow * d;
        for (int c = 0; c < d; ++c) o[(size_t)c] = 0.0;
        for (int64_t j = 0; j < n; ++j) {
          const float* vj = r.vbase + j * r.kstride;
          double acc = 0.0;
          for (int c = 0; c < d; ++c) {
            o[(size_t)c] += pr[j] * (double)vj[c];
            acc += (double)dorow[c] * (double)vj[c];
          }
          dp[j] = acc;
        }
        double D = 0.0;
        for (int64_t j = 0; j < n; ++j) D += pr[j] * dp[j];
        double* dqrow = dq + r.orow * d;
        // dk/dv row of key j: same place in the k/v layout as the key row itself
        const int64_t kvrow0 = (r.kbase - P.k) / d;  // (k0 * Hkv + g)
        for (int64_t j = 0; j < n; ++j) {
#ifdef ORACLE_PLANT_BWD_NO_D
          const double ds = pr[j] * dp[j];
#else
          const double ds = pr[j] * (dp[j] - D);
#endif
          const float* kj = r.kbase + j * r.kstride;
          double* dkj = dk + (kvrow0 + j * Hkv) * d;
          double* dvj = dv + (kvrow0 + j * Hkv) * d;
          for (int c = 0; c < d; ++c) {
#ifdef ORACLE_PLANT_BWD_DQ_NO_SCALE
            dqrow[c] += ds * (double)kj[c];
#else
            dqrow[c] += P.scale * ds * (double)kj[c];
#endif
#ifdef ORACLE_PLANT_BWD_DK_FROM_P
            dkj[c] += P.scale * pr[j] * (double)r.qrow[c];
#else
            dkj[c] += P.scale * ds * (double)r.qrow[c];
#endif
            dvj[c] += pr[j] * (double)dorow[c];
          }
        }
      }
    }
  });
  return 0;
}

int oracle_hardware_threads(void) { return (int)std::thread::hardware_concurrency(); }

}  // extern "C"
