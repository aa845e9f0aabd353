// CPU oracle for pooled block-sparse attention with a hybrid Top-k / Top-p
// block mask, and for its sparse + linear mix.
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, single-threaded
// restatement of what the method computes. Only the test suite, the smoke
// check and the benchmark's CPU-baseline leg may load it. It shares no code,
// header, table or constant with the CUDA library, and the CUDA library never
// calls it.
//
// Sources (the articles print no formula; each step restates their prose):
//   [SA2 s1]  SpargeAttention2 article ("Tsinghua invents an AI
//             attention-slimming technique", arXiv:2602.13515), section 1:
//             Top-k keeps a fixed number of the most important items; Top-p
//             keeps items until their summed importance reaches a threshold;
//             the hybrid runs both and merges (unions) the two selections.
//   [SA2 s4]  same article, section 4: a pre-filter pools neighbouring tokens
//             to score blocks cheaply, a selection stage applies the hybrid
//             rule, and attention runs block by block, each block either fully
//             computed or fully skipped, under a block-level mask.
//   [SLA2 s1] SLA2 article (arXiv:2602.12675), section 1: important regions get
//             sparse (softmax) attention, the rest get linear attention.
//   [SLA2 s2] same article, section 2: the sparse branch is renormalised over
//             the kept region only; the output is alpha * sparse output plus
//             (1 - alpha) * linear output, alpha a learnt ratio.
//
// Readings where the articles are silent (each one is listed with its reason
// in the design notes of the repository):
//   * pooling is the mean over a block's valid rows (a ragged last block
//     averages only the rows it has);
//   * block importance is softmax_J(qbar_I . kbar_J / sqrt(d)) along each
//     query-block row;
//   * Top-k keeps ceil(k * Nkb) blocks (computed as ceil(k*Nkb - 1e-9) to
//     absorb representation error), k = 0 disables it;
//   * Top-p keeps the shortest prefix of the (P descending, index ascending)
//     order whose running sum is >= p, p = 0 disables it;
//   * both selections are prefixes of the same order, so their union is the
//     longer prefix; every row keeps at least one block;
//   * the linear branch uses phi(x) = elu(x) + 1 on the keys outside the kept
//     blocks, normalised: O_l = sum_j (phi(q).phi(k_j)) v_j / sum_j phi(q).phi(k_j);
//     an empty complement gives O_l = 0;
//   * no causal masking (bidirectional video attention).
//
// Precision: everything is computed in double from the exactly widened bf16
// inputs. The block selection is an integer decision taken from floating
// point; it is the double-precision definition (pool, score, softmax, order,
// running sums), with no single-precision variant.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

namespace {

double widen(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

float widen_f(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// phi(x) = elu(x) + 1: x + 1 for x > 0, exp(x) otherwise [SLA2 s1, reading].
double phi(double x) { return x > 0.0 ? x + 1.0 : std::exp(x); }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

enum { OK = 0, ERR_ARG = 1 };

bool shape_ok(int64_t BH, int64_t N, int d, int blk) {
  return BH > 0 && N > 0 && d > 0 && blk > 0;
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Pooling [SA2 s4]: mean of each block's valid rows.
// X: bf16 bits, [BH, N, d] contiguous. out: [BH, ceil(N/blk), d].
// ---------------------------------------------------------------------------
int oracle_pool_f64(const uint16_t* X, int64_t BH, int64_t N, int d, int blk, double* out) {
  if (!X || !out || !shape_ok(BH, N, d, blk)) return ERR_ARG;
  const int64_t nb = ceil_div(N, blk);
  for (int64_t bh = 0; bh < BH; ++bh)
    for (int64_t I = 0; I < nb; ++I) {
      const int64_t r0 = I * blk, r1 = std::min<int64_t>(N, r0 + blk);
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int64_t r = r0; r < r1; ++r) acc += widen(X[(bh * N + r) * d + c]);
        out[(bh * nb + I) * d + c] = acc / static_cast<double>(r1 - r0);
      }
    }
  return OK;
}

// ---------------------------------------------------------------------------
// Pooled block importance [SA2 s4]: P[I, J] = softmax_J(qbar_I . kbar_J / sqrt d).
// qbar [BH, Nqb, d], kbar [BH, Nkb, d], P [BH, Nqb, Nkb].
// ---------------------------------------------------------------------------
int oracle_block_probs_f64(const double* qbar, const double* kbar, int64_t BH, int64_t Nqb,
                           int64_t Nkb, int d, double* P) {
  if (!qbar || !kbar || !P || BH <= 0 || Nqb <= 0 || Nkb <= 0 || d <= 0) return ERR_ARG;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  std::vector<double> s(Nkb);
  for (int64_t bh = 0; bh < BH; ++bh)
    for (int64_t I = 0; I < Nqb; ++I) {
      const double* q = qbar + (bh * Nqb + I) * d;
      double mx = -std::numeric_limits<double>::infinity();
      for (int64_t J = 0; J < Nkb; ++J) {
        const double* k = kbar + (bh * Nkb + J) * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * k[c];
        s[J] = dot * scale;
        mx = std::max(mx, s[J]);
      }
      double sum = 0.0;
      for (int64_t J = 0; J < Nkb; ++J) {
        s[J] = std::exp(s[J] - mx);
        sum += s[J];
      }
      double* row = P + (bh * Nqb + I) * Nkb;
      for (int64_t J = 0; J < Nkb; ++J) row[J] = s[J] / sum;
    }
  return OK;
}

// ---------------------------------------------------------------------------
// Hybrid Top-k / Top-p selection on one row of block probabilities [SA2 s1].
//
// P: Nkb probabilities. kept: receives the kept block indices in ascending
// order (capacity Nkb). Optional outputs: m (kept count), kc and pc (the Top-k
// and Top-p counts), order (the full (P desc, index asc) order), cum (cum[m] =
// running sum of the first m sorted probabilities, m = 0..Nkb, in double).
// ---------------------------------------------------------------------------
int oracle_select_row(const double* P, int64_t Nkb, double topk, double topp, int32_t* kept,
                      int64_t* m_out, int64_t* kc_out, int64_t* pc_out, int32_t* order_out,
                      double* cum_out) {
  if (!P || !kept || Nkb <= 0) return ERR_ARG;
  if (!(topk >= 0.0 && topk <= 1.0) || !(topp >= 0.0 && topp <= 1.0)) return ERR_ARG;
  // Order: most important first; equal importance goes to the lower index.
  std::vector<int32_t> order(Nkb);
  for (int64_t j = 0; j < Nkb; ++j) order[j] = static_cast<int32_t>(j);
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return P[a] > P[b]; });

  // Top-k: a fixed count regardless of how importance is spread.
  int64_t kc = 0;
  if (topk > 0.0) {
    kc = static_cast<int64_t>(std::ceil(topk * static_cast<double>(Nkb) - 1e-9));
    kc = std::min<int64_t>(std::max<int64_t>(kc, 0), Nkb);
  }
  // Top-p: the shortest prefix whose summed importance reaches p.
  std::vector<double> cum(Nkb + 1, 0.0);
  for (int64_t m = 1; m <= Nkb; ++m) cum[m] = cum[m - 1] + P[order[m - 1]];
  int64_t pc = 0;
  if (topp > 0.0) {
    pc = Nkb;
    for (int64_t m = 1; m <= Nkb; ++m)
      if (cum[m] >= topp) {
        pc = m;
        break;
      }
  }
  // Union of two prefixes of one order = the longer prefix; keep >= 1 block.
  const int64_t m = std::max<int64_t>(std::max(kc, pc), 1);
  std::vector<int32_t> sel(order.begin(), order.begin() + m);
  std::sort(sel.begin(), sel.end());
  for (int64_t i = 0; i < m; ++i) kept[i] = sel[i];
  if (m_out) *m_out = m;
  if (kc_out) *kc_out = kc;
  if (pc_out) *pc_out = pc;
  if (order_out)
    for (int64_t j = 0; j < Nkb; ++j) order_out[j] = order[j];
  if (cum_out)
    for (int64_t j = 0; j <= Nkb; ++j) cum_out[j] = cum[j];
  return OK;
}

// ---------------------------------------------------------------------------
// Block mask with a learnt router [SLA2 s2]: the article replaces the
// heuristic routing by a router with two learnable projection matrices that
// map the query and key features into a space suited to the routing
// decision. Reading: the pooled block vectors are projected,
//   qhat_I = qbar_I Wq_h,  khat_J = kbar_J Wk_h   (W: [d, dr] per head h),
// and the block importance is softmax_J(qhat_I . khat_J / sqrt(dr)), followed
// by the same hybrid selection. Every step in double.
// Q, K: bf16 bits [B*H, N, d]. Wq / Wk: fp32 [H, d, dr] (row c, column c'),
// H = BH / (batches); both null for the plain mask. kv_idx [B*H, Nqb, Nkb]
// (first kv_cnt entries valid, ascending), kv_cnt [B*H, Nqb]. P_out:
// optional [B*H, Nqb, Nkb].
// ---------------------------------------------------------------------------
int oracle_mask_router(const uint16_t* Q, const uint16_t* K, int64_t BH, int64_t N, int d, int bq, int bk,
                       const float* Wq, const float* Wk, int64_t H, int dr, double topk, double topp,
                       int32_t* kv_idx, int32_t* kv_cnt, double* P_out) {
  if (!Q || !K || !kv_idx || !kv_cnt || !shape_ok(BH, N, d, bq) || bk <= 0) return ERR_ARG;
  const bool routed = Wq != nullptr || Wk != nullptr;
  if (routed && (!Wq || !Wk || H <= 0 || BH % H != 0 || dr <= 0)) return ERR_ARG;
  const int dd = routed ? dr : d;
  const int64_t Nqb = ceil_div(N, bq), Nkb = ceil_div(N, bk);
  std::vector<double> P(static_cast<size_t>(BH * Nqb * Nkb));
  std::vector<double> qb(static_cast<size_t>(BH * Nqb * d)), kb(static_cast<size_t>(BH * Nkb * d));
  oracle_pool_f64(Q, BH, N, d, bq, qb.data());
  oracle_pool_f64(K, BH, N, d, bk, kb.data());
  if (routed) {
    std::vector<double> qh(static_cast<size_t>(BH * Nqb * dr)), kh(static_cast<size_t>(BH * Nkb * dr));
    for (int pass = 0; pass < 2; ++pass) {
      const std::vector<double>& in = pass == 0 ? qb : kb;
      std::vector<double>& out = pass == 0 ? qh : kh;
      const float* W = pass == 0 ? Wq : Wk;
      const int64_t nb = pass == 0 ? Nqb : Nkb;
      for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t I = 0; I < nb; ++I)
          for (int c2 = 0; c2 < dr; ++c2) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
              acc += in[(bh * nb + I) * d + c] * static_cast<double>(W[((bh % H) * d + c) * dr + c2]);
            out[(bh * nb + I) * dr + c2] = acc;
          }
    }
    oracle_block_probs_f64(qh.data(), kh.data(), BH, Nqb, Nkb, dd, P.data());
  } else {
    oracle_block_probs_f64(qb.data(), kb.data(), BH, Nqb, Nkb, dd, P.data());
  }
  for (int64_t row = 0; row < BH * Nqb; ++row) {
    int64_t m = 0;
    int rc = oracle_select_row(P.data() + row * Nkb, Nkb, topk, topp, kv_idx + row * Nkb, &m,
                               nullptr, nullptr, nullptr, nullptr);
    if (rc != OK) return rc;
    for (int64_t j = m; j < Nkb; ++j) kv_idx[row * Nkb + j] = 0;
    kv_cnt[row] = static_cast<int32_t>(m);
  }
  if (P_out) std::memcpy(P_out, P.data(), P.size() * sizeof(double));
  return OK;
}

// Block mask without a router [SA2 s1, s4]: pool, score, select, for every
// query-block row, the pooled vectors scored directly.
int oracle_mask(const uint16_t* Q, const uint16_t* K, int64_t BH, int64_t N, int d, int bq,
                int bk, double topk, double topp, int32_t* kv_idx, int32_t* kv_cnt, double* P_out) {
  return oracle_mask_router(Q, K, BH, N, d, bq, bk, nullptr, nullptr, 0, 0, topk, topp, kv_idx, kv_cnt, P_out);
}

// ---------------------------------------------------------------------------
// Attention outputs for a list of rows, in double.
//
// mode 0: sparse branch [SA2 s4, SLA2 s2] - softmax over the keys of the kept
//         blocks only (renormalised over that region), scale 1/sqrt(d).
// mode 1: linear branch [SLA2 s1] - phi-feature attention over the keys of
//         the blocks NOT kept, normalised; 0 when that set is empty.
// mode 2: the mix [SLA2 s2] - alpha_h * sparse + (1 - alpha_h) * linear.
// mode 3: dense softmax attention over all keys (all blocks kept).
//
// rows: flat row ids r = bh*N + i. O: [nrows, d]. lse (optional, modes 0 and
// 3): natural-log sum of exp of the scaled scores, -inf for an empty set.
// kv_idx / kv_cnt as produced by oracle_mask; entries must lie in [0, Nkb).
// ---------------------------------------------------------------------------
int oracle_attention_rows(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t BH,
                          int64_t N, int d, int bq, int bk, const int32_t* kv_idx,
                          const int32_t* kv_cnt, const float* alpha, int64_t H, int mode,
                          const int64_t* rows, int64_t nrows, double* O, double* lse) {
  if (!Q || !K || !V || !rows || !O || !shape_ok(BH, N, d, bq) || bk <= 0) return ERR_ARG;
  if (mode < 0 || mode > 3) return ERR_ARG;
  if (mode != 3 && (!kv_idx || !kv_cnt)) return ERR_ARG;
  if (mode == 2 && (!alpha || H <= 0 || BH % H != 0)) return ERR_ARG;
  const int64_t Nqb = ceil_div(N, bq), Nkb = ceil_div(N, bk);
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));

  // Rows are grouped by head so each head's widened K, V and phi(K) are built once.
  std::vector<int64_t> idx(nrows);
  for (int64_t i = 0; i < nrows; ++i) {
    if (rows[i] < 0 || rows[i] >= BH * N) return ERR_ARG;
    idx[i] = i;
  }
  std::stable_sort(idx.begin(), idx.end(), [&](int64_t a, int64_t b) { return rows[a] / N < rows[b] / N; });

  std::vector<double> Kd, Vd, phiK, q(d), phiq(d), s, acc(d), acc_s(d), acc_l(d);
  std::vector<char> kept(Nkb);
  int64_t cur_bh = -1;
  for (int64_t t = 0; t < nrows; ++t) {
    const int64_t ri = idx[t];
    const int64_t bh = rows[ri] / N, i = rows[ri] % N, I = i / bq;
    if (bh != cur_bh) {
      cur_bh = bh;
      Kd.assign(static_cast<size_t>(N * d), 0.0);
      Vd.assign(static_cast<size_t>(N * d), 0.0);
      for (int64_t e = 0; e < N * d; ++e) {
        Kd[e] = widen(K[bh * N * d + e]);
        Vd[e] = widen(V[bh * N * d + e]);
      }
      if (mode == 1 || mode == 2) {
        phiK.assign(static_cast<size_t>(N * d), 0.0);
        for (int64_t e = 0; e < N * d; ++e) phiK[e] = phi(Kd[e]);
      }
    }
    for (int c = 0; c < d; ++c) {
      q[c] = widen(Q[(bh * N + i) * d + c]);
      phiq[c] = phi(q[c]);
    }
    // Block membership of this row's query block.
    if (mode == 3) {
      std::fill(kept.begin(), kept.end(), 1);
    } else {
      std::fill(kept.begin(), kept.end(), 0);
      const int64_t cnt = kv_cnt[bh * Nqb + I];
      if (cnt < 0 || cnt > Nkb) return ERR_ARG;
      for (int64_t e = 0; e < cnt; ++e) {
        const int32_t J = kv_idx[(bh * Nqb + I) * Nkb + e];
        if (J < 0 || J >= Nkb) return ERR_ARG;
        kept[J] = 1;
      }
    }

    // Softmax branch over the kept keys (two passes: max, then exp-weighted sums).
    double lse_row = -std::numeric_limits<double>::infinity();
    std::fill(acc_s.begin(), acc_s.end(), 0.0);
    if (mode != 1) {
      double mx = -std::numeric_limits<double>::infinity();
      s.assign(static_cast<size_t>(N), 0.0);
      for (int64_t j = 0; j < N; ++j) {
        if (!kept[j / bk]) continue;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * Kd[j * d + c];
        s[j] = dot * scale;
        mx = std::max(mx, s[j]);
      }
      if (mx > -std::numeric_limits<double>::infinity()) {
        double l = 0.0;
        for (int64_t j = 0; j < N; ++j) {
          if (!kept[j / bk]) continue;
          const double e = std::exp(s[j] - mx);
          l += e;
          for (int c = 0; c < d; ++c) acc_s[c] += e * Vd[j * d + c];
        }
        for (int c = 0; c < d; ++c) acc_s[c] /= l;
        lse_row = mx + std::log(l);
      }
    }
    // Linear branch over the complement.
    std::fill(acc_l.begin(), acc_l.end(), 0.0);
    if (mode == 1 || mode == 2) {
      double den = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        if (kept[j / bk]) continue;
        double w = 0.0;
        for (int c = 0; c < d; ++c) w += phiq[c] * phiK[j * d + c];
        den += w;
        for (int c = 0; c < d; ++c) acc_l[c] += w * Vd[j * d + c];
      }
      if (den > 0.0)
        for (int c = 0; c < d; ++c) acc_l[c] /= den;
    }
    double a = 1.0;
    if (mode == 2) a = static_cast<double>(alpha[bh % H]);
    for (int c = 0; c < d; ++c) {
      double v;
      if (mode == 0 || mode == 3) v = acc_s[c];
      else if (mode == 1) v = acc_l[c];
      else v = a * acc_s[c] + (1.0 - a) * acc_l[c];
      O[ri * d + c] = v;
    }
    if (lse) lse[ri] = lse_row;
  }
  return OK;
}

}  // extern "C"

// ===========================================================================
// Low-bit sparse branch [SLA2 s3]: the article quantises the sparse branch's
// queries, keys, attention probabilities and values to a low-bit format
// ("for example 8-bit integers"), scaling into the low-bit range before the
// products and back after. It fixes neither the formats nor the scale
// granularity; the readings taken here:
//   * Q and K: int8, symmetric, one scale per (batch, head, block): the
//     block's max |x| maps to 127; q8 = rint(x * s) (ties to even), clamped
//     to [-127, 127]; s = 127 / amax in float (1 when amax = 0), the product
//     x * s in float. S = q8 . k8 is an exact integer.
//   * V: fp8 e4m3, one scale per (batch, head, channel) over all keys: the
//     channel's max |v| maps to 448; v8 = e4m3(v * s_v), the product in float.
//   * P: e4m3, scaled into the format's range by a power of two: the row's
//     largest value lands in (2^7, 2^8], the top binade below e4m3's largest
//     finite value 448. In two passes over the keys of the row's kept blocks
//     (in any order):
//       x_j   = float(S_j) * c, c = float(log2(e)/sqrt(d)) / (s_q * s_k) in float
//               (s_k the scale of key j's block);
//       m     = ceil(max_j x_j) over every kept key of the row (first pass);
//       e_j   = 2^(x_j - (m - 8)), x_j - (m - 8) in float, so e_j <= 2^8;
//       p_j   = e4m3(e_j) (second pass);
//       l     = sum_j e_j (the normaliser is not quantised: only the operands
//               of the two products are); acc = sum_j p_j v8_j;
//     O = acc / (l * s_v). Keys more than 14 binades below the row's max fall
//     into e4m3's subnormal range (below 2^-6).
// e4m3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; largest finite 448,
// subnormals down to 2^-9; rounding to nearest, ties to even; magnitudes
// above 448 saturate to 448.
// ===========================================================================

namespace {

double e4m3_rne(double x) {
  if (x == 0.0 || std::isnan(x)) return x;
  const double a = std::fabs(x);
  if (a >= 448.0) return std::copysign(448.0, x);
  int k;
  std::frexp(a, &k);                    // a = f * 2^k, f in [0.5, 1): binade exponent k - 1
  const int e = std::max(k - 1, -6);    // below 2^-6 the spacing stays 2^-9 (subnormals)
  const double q = std::ldexp(1.0, e - 3);
  const double r = std::nearbyint(a / q) * q;  // default rounding mode: to nearest, ties to even
  return std::copysign(std::min(r, 448.0), x);
}

float quant_scale(float amax, float top) { return amax > 0.0f ? top / amax : 1.0f; }

int8_t quant_i8(float x, float s) {
  float v = x * s;
  float r = std::nearbyint(v);
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return static_cast<int8_t>(r);
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Quantised operands of the low-bit sparse branch (readings above).
// Q, K, V: bf16 bits [BH, N, d]. q8 / k8: int8 [BH, N, d]; sq: [BH, ceil(N/bq)];
// sk: [BH, ceil(N/bk)]; v8: the e4m3 values as double [BH, N, d]; sv: [BH, d].
// ---------------------------------------------------------------------------
int oracle_quant_q8(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t BH, int64_t N, int d, int bq,
                    int bk, int8_t* q8, float* sq, int8_t* k8, float* sk, double* v8, float* sv) {
  if (!Q || !K || !V || !q8 || !sq || !k8 || !sk || !v8 || !sv || !shape_ok(BH, N, d, bq) || bk <= 0) return ERR_ARG;
  const int64_t nqb = ceil_div(N, bq), nkb = ceil_div(N, bk);
  for (int64_t bh = 0; bh < BH; ++bh) {
    for (int pass = 0; pass < 2; ++pass) {
      const uint16_t* X = pass == 0 ? Q : K;
      int8_t* out = pass == 0 ? q8 : k8;
      float* sc = pass == 0 ? sq : sk;
      const int blk = pass == 0 ? bq : bk;
      const int64_t nb = pass == 0 ? nqb : nkb;
      for (int64_t I = 0; I < nb; ++I) {
        const int64_t r0 = I * blk, r1 = std::min<int64_t>(N, r0 + blk);
        float amax = 0.0f;
        for (int64_t r = r0; r < r1; ++r)
          for (int c = 0; c < d; ++c) amax = std::max(amax, std::fabs(widen_f(X[(bh * N + r) * d + c])));
        const float s = quant_scale(amax, 127.0f);
        sc[bh * nb + I] = s;
        for (int64_t r = r0; r < r1; ++r)
          for (int c = 0; c < d; ++c) out[(bh * N + r) * d + c] = quant_i8(widen_f(X[(bh * N + r) * d + c]), s);
      }
    }
    for (int c = 0; c < d; ++c) {
      float amax = 0.0f;
      for (int64_t r = 0; r < N; ++r) amax = std::max(amax, std::fabs(widen_f(V[(bh * N + r) * d + c])));
      const float s = quant_scale(amax, 448.0f);
      sv[bh * d + c] = s;
      for (int64_t r = 0; r < N; ++r) {
        const float v = widen_f(V[(bh * N + r) * d + c]) * s;
        v8[(bh * N + r) * d + c] = e4m3_rne(static_cast<double>(v));
      }
    }
  }
  return OK;
}

// Nearest e4m3 value of each x (ties to even, saturating at 448).
int oracle_e4m3(const double* x, int64_t n, double* out) {
  if (!x || !out || n < 0) return ERR_ARG;
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_rne(x[i]);
  return OK;
}

// ---------------------------------------------------------------------------
// Low-bit sparse branch outputs for selected rows (readings above).
// rows: flat row ids bh*N + i. O: [nrows, d] double.
// ---------------------------------------------------------------------------
int oracle_attention_q8_rows(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t BH, int64_t N,
                             int d, int bq, int bk, const int32_t* kv_idx, const int32_t* kv_cnt,
                             const int64_t* rows, int64_t nrows, double* O) {
  if (!Q || !K || !V || !rows || !O || !kv_idx || !kv_cnt || !shape_ok(BH, N, d, bq) || bk <= 0) return ERR_ARG;
  const int64_t Nqb = ceil_div(N, bq), Nkb = ceil_div(N, bk);
  std::vector<int8_t> q8(static_cast<size_t>(BH * N * d)), k8(static_cast<size_t>(BH * N * d));
  std::vector<float> sq(static_cast<size_t>(BH * Nqb)), sk(static_cast<size_t>(BH * Nkb)), sv(static_cast<size_t>(BH * d));
  std::vector<double> v8(static_cast<size_t>(BH * N * d));
  const int rc = oracle_quant_q8(Q, K, V, BH, N, d, bq, bk, q8.data(), sq.data(), k8.data(), sk.data(), v8.data(),
                                 sv.data());
  if (rc != OK) return rc;
  const float c0 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  std::vector<double> acc(d);
  std::vector<float> x;        // x_j of the row's kept keys
  std::vector<int64_t> keys;   // their key indices
  for (int64_t t = 0; t < nrows; ++t) {
    const int64_t r = rows[t];
    if (r < 0 || r >= BH * N) return ERR_ARG;
    const int64_t bh = r / N, i = r % N, I = i / bq;
    const int64_t cnt = kv_cnt[bh * Nqb + I];
    if (cnt < 0 || cnt > Nkb) return ERR_ARG;
    const int8_t* qi = &q8[static_cast<size_t>((bh * N + i) * d)];
    // Pass 1: scaled integer scores of every kept key, and their maximum.
    x.clear();
    keys.clear();
    float mx = -std::numeric_limits<float>::infinity();
    for (int64_t e = 0; e < cnt; ++e) {
      const int64_t J = kv_idx[(bh * Nqb + I) * Nkb + e];
      if (J < 0 || J >= Nkb) return ERR_ARG;
      const float c = c0 / (sq[bh * Nqb + I] * sk[bh * Nkb + J]);
      for (int64_t j = J * bk; j < std::min<int64_t>(N, (J + 1) * bk); ++j) {
        const int8_t* kj = &k8[static_cast<size_t>((bh * N + j) * d)];
        int64_t S = 0;
        for (int cc = 0; cc < d; ++cc) S += static_cast<int64_t>(qi[cc]) * kj[cc];
        x.push_back(static_cast<float>(S) * c);
        keys.push_back(j);
        mx = std::max(mx, x.back());
      }
    }
    // Pass 2: codes of 2^(x - (m - 8)) for the integer reference m.
    const float ref = std::ceil(mx) - 8.0f;
    double l = 0.0;
    std::fill(acc.begin(), acc.end(), 0.0);
    for (size_t u = 0; u < x.size(); ++u) {
      const double ej = std::exp2(static_cast<double>(x[u] - ref));
      const double pj = e4m3_rne(ej);
      l += ej;
      for (int cc = 0; cc < d; ++cc) acc[cc] += pj * v8[static_cast<size_t>((bh * N + keys[u]) * d + cc)];
    }
    for (int cc = 0; cc < d; ++cc)
      O[t * d + cc] = l > 0.0 ? acc[cc] / (l * static_cast<double>(sv[bh * d + cc])) : 0.0;
  }
  return OK;
}

}  // extern "C"


// ===========================================================================
// Gradients [SA2 s1 (trainable sparse attention), SLA2 s2]: for a loss L with
// dL/dO = dO, the gradients of Q, K, V (and of alpha) through the forward of
// oracle_attention_rows, written out from the chain rule in double:
//
//   sparse branch (g_i = alpha * dO_i; alpha = 1 outside the mix):
//     P_ij = softmax over the kept keys of s_ij = q_i.k_j / sqrt(d),
//     O_s,i = sum_j P_ij v_j,
//     dV_j += P_ij g_i,      dP_ij = g_i . v_j,
//     dS_ij = P_ij (dP_ij - g_i . O_s,i),
//     dQ_i += sum_j dS_ij k_j / sqrt(d),   dK_j += dS_ij q_i / sqrt(d);
//   linear branch (h_i = (1 - alpha) dO_i; dO_i outside the mix), over the
//   keys j outside the kept blocks, w_ij = phi(q_i).phi(k_j),
//   den_i = sum_j w_ij, O_l,i = sum_j w_ij v_j / den_i:
//     dV_j += (w_ij / den_i) h_i,
//     dw_ij = h_i . (v_j - O_l,i) / den_i,
//     dQ_i += (sum_j dw_ij phi(k_j)) * phi'(q_i),
//     dK_j += dw_ij phi(q_i) * phi'(k_j),   phi'(x) = 1 (x > 0), e^x (x <= 0);
//     an empty complement (O_l = 0 by the forward's reading) gives nothing;
//   the mix: dalpha_h = sum over the rows of head h of dO_i . (O_s,i - O_l,i).
//
// mode as in oracle_attention_rows (0 sparse, 1 linear, 2 mix, 3 dense).
// dO: bf16 bits [BH, N, d] (widened exactly). Outputs:
//   dQ [n_rows, d] for the flat rows q_rows[] (bh*N + i), if dQ is not null;
//   dK, dV [n_blocks, bk, d] for the flat key blocks k_blocks[] (bh*Nkb + J),
//     rows past N zero, if dK / dV are not null;
//   dalpha [H] (mode 2 only, summed over every row of every head) if not null.
// Every query row that feeds a requested output is visited (for dK / dV:
// the rows whose block keeps J, plus every row of the head in modes 1 and 2).
// ===========================================================================
extern "C" {

int oracle_attention_bwd(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* dO, int64_t BH,
                         int64_t N, int d, int bq, int bk, const int32_t* kv_idx, const int32_t* kv_cnt,
                         const float* alpha, int64_t H, int mode, const int64_t* q_rows, int64_t n_rows,
                         const int64_t* k_blocks, int64_t n_blocks, double* dQ, double* dK, double* dV,
                         double* dalpha) {
  if (!Q || !K || !V || !dO || !shape_ok(BH, N, d, bq) || bk <= 0) return ERR_ARG;
  if (mode < 0 || mode > 3) return ERR_ARG;
  if (mode != 3 && (!kv_idx || !kv_cnt)) return ERR_ARG;
  if (mode == 2 && (!alpha || H <= 0 || BH % H != 0)) return ERR_ARG;
  if (dalpha && mode != 2) return ERR_ARG;
  if ((n_rows > 0 && (!q_rows || !dQ)) || (n_blocks > 0 && (!k_blocks || (!dK && !dV)))) return ERR_ARG;
  const int64_t Nqb = ceil_div(N, bq), Nkb = ceil_div(N, bk);
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  const bool use_s = mode != 1, use_l = mode == 1 || mode == 2;
  for (int64_t t = 0; t < n_rows; ++t)
    if (q_rows[t] < 0 || q_rows[t] >= BH * N) return ERR_ARG;
  for (int64_t t = 0; t < n_blocks; ++t)
    if (k_blocks[t] < 0 || k_blocks[t] >= BH * Nkb) return ERR_ARG;
  if (dQ) std::fill(dQ, dQ + n_rows * d, 0.0);
  if (dK) std::fill(dK, dK + n_blocks * bk * d, 0.0);
  if (dV) std::fill(dV, dV + n_blocks * bk * d, 0.0);
  if (dalpha) std::fill(dalpha, dalpha + H, 0.0);

  // kept[J] of query block I of head bh.
  auto kept_row = [&](int64_t bh, int64_t I, std::vector<char>& kept) -> bool {
    if (mode == 3) {
      std::fill(kept.begin(), kept.end(), 1);
      return true;
    }
    std::fill(kept.begin(), kept.end(), 0);
    const int64_t cnt = kv_cnt[bh * Nqb + I];
    if (cnt < 0 || cnt > Nkb) return false;
    for (int64_t e = 0; e < cnt; ++e) {
      const int32_t J = kv_idx[(bh * Nqb + I) * Nkb + e];
      if (J < 0 || J >= Nkb) return false;
      kept[J] = 1;
    }
    return true;
  };

  std::vector<double> Kd, Vd, phiK, q(d), phiq(d), g(d), hl(d), s, w, Os(d), Ol(d), dq(d), dphiq(d);
  std::vector<char> kept(Nkb), qkeep(Nkb);
  std::vector<int64_t> qslot, kslot;
  for (int64_t bh = 0; bh < BH; ++bh) {
    // Requested outputs of this head.
    qslot.assign(static_cast<size_t>(N), -1);
    kslot.assign(static_cast<size_t>(Nkb), -1);
    bool any = dalpha != nullptr;
    for (int64_t t = 0; t < n_rows; ++t)
      if (q_rows[t] / N == bh) qslot[q_rows[t] % N] = t, any = true;
    for (int64_t t = 0; t < n_blocks; ++t)
      if (k_blocks[t] / Nkb == bh) kslot[k_blocks[t] % Nkb] = t, any = true;
    if (!any) continue;
    Kd.assign(static_cast<size_t>(N * d), 0.0);
    Vd.assign(static_cast<size_t>(N * d), 0.0);
    phiK.assign(static_cast<size_t>(N * d), 0.0);
    for (int64_t e = 0; e < N * d; ++e) {
      Kd[e] = widen(K[bh * N * d + e]);
      Vd[e] = widen(V[bh * N * d + e]);
      phiK[e] = phi(Kd[e]);
    }
    const double a = mode == 2 ? static_cast<double>(alpha[bh % H]) : 1.0;
    for (int64_t i = 0; i < N; ++i) {
      const int64_t I = i / bq;
      if (!kept_row(bh, I, kept)) return ERR_ARG;
      // Does this row feed anything requested?
      bool feeds = dalpha != nullptr || qslot[i] >= 0;
      for (int64_t J = 0; J < Nkb && !feeds; ++J)
        if (kslot[J] >= 0 && ((use_s && kept[J]) || (use_l && !kept[J]))) feeds = true;
      if (!feeds) continue;
      for (int c = 0; c < d; ++c) {
        q[c] = widen(Q[(bh * N + i) * d + c]);
        phiq[c] = phi(q[c]);
        const double go = widen(dO[(bh * N + i) * d + c]);
        g[c] = mode == 2 ? a * go : go;
        hl[c] = mode == 2 ? (1.0 - a) * go : go;
      }
      std::fill(dq.begin(), dq.end(), 0.0);
      std::fill(Os.begin(), Os.end(), 0.0);
      std::fill(Ol.begin(), Ol.end(), 0.0);
      // Sparse branch: forward (two passes), then its gradients.
      if (use_s) {
        double mx = -std::numeric_limits<double>::infinity();
        s.assign(static_cast<size_t>(N), 0.0);
        for (int64_t j = 0; j < N; ++j) {
          if (!kept[j / bk]) continue;
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += q[c] * Kd[j * d + c];
          s[j] = dot * scale;
          mx = std::max(mx, s[j]);
        }
        if (mx > -std::numeric_limits<double>::infinity()) {
          double l = 0.0;
          for (int64_t j = 0; j < N; ++j)
            if (kept[j / bk]) l += std::exp(s[j] - mx);
          for (int64_t j = 0; j < N; ++j) {
            if (!kept[j / bk]) continue;
            s[j] = std::exp(s[j] - mx) / l;  // s now holds P_ij
            for (int c = 0; c < d; ++c) Os[c] += s[j] * Vd[j * d + c];
          }
          double gO = 0.0;
          for (int c = 0; c < d; ++c) gO += g[c] * Os[c];
          for (int64_t j = 0; j < N; ++j) {
            if (!kept[j / bk]) continue;
            double dP = 0.0;
            for (int c = 0; c < d; ++c) dP += g[c] * Vd[j * d + c];
            const double dS = s[j] * (dP - gO);
            for (int c = 0; c < d; ++c) dq[c] += dS * Kd[j * d + c] * scale;
            const int64_t ks = kslot[j / bk];
            if (ks >= 0) {
              const int64_t r = (ks * bk + j % bk) * d;
              for (int c = 0; c < d; ++c) {
                if (dK) dK[r + c] += dS * q[c] * scale;
                if (dV) dV[r + c] += s[j] * g[c];
              }
            }
          }
        }
      }
      // Linear branch over the complement: forward, then its gradients.
      if (use_l) {
        w.assign(static_cast<size_t>(N), 0.0);
        double den = 0.0;
        for (int64_t j = 0; j < N; ++j) {
          if (kept[j / bk]) continue;
          double x = 0.0;
          for (int c = 0; c < d; ++c) x += phiq[c] * phiK[j * d + c];
          w[j] = x;
          den += x;
        }
        if (den > 0.0) {
          for (int64_t j = 0; j < N; ++j) {
            if (kept[j / bk]) continue;
            for (int c = 0; c < d; ++c) Ol[c] += w[j] * Vd[j * d + c];
          }
          for (int c = 0; c < d; ++c) Ol[c] /= den;
          double hO = 0.0;
          for (int c = 0; c < d; ++c) hO += hl[c] * Ol[c];
          std::fill(dphiq.begin(), dphiq.end(), 0.0);
          for (int64_t j = 0; j < N; ++j) {
            if (kept[j / bk]) continue;
            double hv = 0.0;
            for (int c = 0; c < d; ++c) hv += hl[c] * Vd[j * d + c];
            const double dw = (hv - hO) / den;
            for (int c = 0; c < d; ++c) dphiq[c] += dw * phiK[j * d + c];
            const int64_t ks = kslot[j / bk];
            if (ks >= 0) {
              const int64_t r = (ks * bk + j % bk) * d;
              for (int c = 0; c < d; ++c) {
                const double kc = Kd[j * d + c];
                if (dK) dK[r + c] += dw * phiq[c] * (kc > 0.0 ? 1.0 : std::exp(kc));
                if (dV) dV[r + c] += (w[j] / den) * hl[c];
              }
            }
          }
          for (int c = 0; c < d; ++c) dq[c] += dphiq[c] * (q[c] > 0.0 ? 1.0 : std::exp(q[c]));
        }
      }
      if (qslot[i] >= 0)
        for (int c = 0; c < d; ++c) dQ[qslot[i] * d + c] = dq[c];
      if (dalpha) {
        double x = 0.0;
        for (int c = 0; c < d; ++c) x += widen(dO[(bh * N + i) * d + c]) * (Os[c] - Ol[c]);
        dalpha[bh % H] += x;
      }
    }
  }
  return OK;
}

}  // extern "C"
