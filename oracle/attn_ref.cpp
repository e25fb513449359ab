// Plain fp64 reference for exact softmax attention (forward + backward).
//
// TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA kernels are checked
// against. Only the tests, the package's smoke check and the benchmark's CPU-baseline
// leg may load it. It shares no code, header, table or constant with the CUDA path.
//
// Sources (web pages on FlashAttention, cited by title and section):
//   [P1] "FlashAttention-2 的前世今生" overview, jishu.shishitao.com/detail/60083.html
//   [P2] "Attention 为什么慢" / Flash Attention explainer, ds6.com.cn/news/67428.html
//   [P3] FlashAttention V1 lecture summary, spark.aweffr.cn/summary/0684ec99-...
//
// What is computed (per batch b and head h, every tensor row-major N x d):
//   S_ij = scale * <q_i, k_j>                 for allowed (i, j)         [P3 §2.1, §2.2 step 1]
//   m_i  = max_j S_ij                          (safe softmax pass 1)      [P2 "时间复杂度"; P3 §3.2]
//   l_i  = sum_j exp(S_ij - m_i)               (pass 2)
//   P_ij = exp(S_ij - m_i) / l_i               (pass 3)
//   O_i  = sum_j P_ij v_j                                                  [P3 §2.2 step 3]
//   LSE_i = m_i + ln l_i   -- the single per-row statistic the FA2 backward keeps  [P1 §主要操作, backward]
// allowed(i, j) = (!causal || j <= i) && (mask == null || mask[i/bs][j/bs] != 0)
//   (causal: [P1] benchmark setting "with or without causal mask"; block mask: [P1] §Block-Sparse).
// A row with no allowed key has O_i = 0 and LSE_i = -inf (a reading; the pages are silent).
//
// General shapes (oracle_fwd_qk): N_q query rows against N_k keys per head. The pages only
// treat N_q = N_k; the reading taken is the bottom-right alignment, where the last query row
// sees every key: causal allows j <= i + (N_k - N_q), which is j <= i when N_q = N_k.
//
// Backward with upstream gradient dO. The pages only say that the backward recomputes S and
// P from the saved statistics and goes through the softmax Jacobian ([P3] §4.1, §4.2); the
// formulas below are the textbook chain rule through steps above:
//   dV_j = sum_i P_ij dO_i
//   dP_ij = <dO_i, v_j>
//   D_i  = sum_j P_ij dP_ij
//   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i = scale * sum_j dS_ij k_j ,   dK_j = scale * sum_i dS_ij q_i
//
// The online variant (oracle_online_fwd) walks the keys block by block with a running
// maximum, running normaliser and running output, in either the per-step-normalised form of
// [P3] §3.2 (recurrence steps 1-3) and §3.4, or the deferred form (keep the output
// unnormalised, divide once at the end), which is how [P1] §主要操作 cuts non-matmul work.
// It exists only to check that the running recurrence reproduces three-pass softmax.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

struct Mask {
  int causal;
  const uint8_t* blocks;  // nullable, [nb][nb] row-major
  int nb;                 // blocks per side
  int bs;                 // block size in rows/keys
  int off = 0;            // causal alignment: key j visible to query i iff j <= i + off
  bool allowed(int i, int j) const {
    if (causal && j > i + off) return false;
    if (blocks && blocks[(int64_t)(i / bs) * nb + (j / bs)] == 0) return false;
    return true;
  }
};

Mask make_mask(int N, int causal, const uint8_t* blocks, int bs) {
  Mask m;
  m.causal = causal;
  m.blocks = blocks;
  m.bs = bs > 0 ? bs : 128;
  m.nb = (N + m.bs - 1) / m.bs;
  return m;
}

double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int t = 0; t < d; ++t) s += a[t] * b[t];
  return s;
}

// Three-pass softmax of one query row. Fills s_row[j] with scale*q.k_j for allowed j and
// p_row[j] with the probability (0 where not allowed). Returns LSE (or -inf if no key is
// allowed).
double softmax_row(const double* qi, const double* k, int N, int d, double scale, const Mask& mk,
                   int i, double* s_row, double* p_row) {
  const double NEG_INF = -std::numeric_limits<double>::infinity();
  // S_ij for allowed keys.
  double m = NEG_INF;
  for (int j = 0; j < N; ++j) {
    if (mk.allowed(i, j)) {
      s_row[j] = scale * dot(qi, k + (int64_t)j * d, d);
      if (s_row[j] > m) m = s_row[j];  // pass 1: row maximum
    }
  }
  if (m == NEG_INF) {
    for (int j = 0; j < N; ++j) p_row[j] = 0.0;
    return NEG_INF;
  }
  double l = 0.0;  // pass 2: normaliser with the maximum subtracted
  for (int j = 0; j < N; ++j)
    if (mk.allowed(i, j)) l += std::exp(s_row[j] - m);
  for (int j = 0; j < N; ++j)  // pass 3: probabilities
    p_row[j] = mk.allowed(i, j) ? std::exp(s_row[j] - m) / l : 0.0;
  return m + std::log(l);
}

int nthreads_used() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // namespace

extern "C" {

int oracle_num_threads() { return nthreads_used(); }

// Forward for all BH = B*H heads. q, k, v, o: [BH][N][d]; lse: [BH][N].
void oracle_fwd(const double* q, const double* k, const double* v, int64_t BH, int N, int d,
                double scale, int causal, const uint8_t* mask, int mask_bs, double* o, double* lse) {
  const Mask mk = make_mask(N, causal, mask, mask_bs);
  for (int64_t bh = 0; bh < BH; ++bh) {
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    double* oh = o + bh * N * d;
    double* lh = lse + bh * N;
#pragma omp parallel
    {
      std::vector<double> s_row(N), p_row(N);
#pragma omp for schedule(dynamic, 4)
      for (int i = 0; i < N; ++i) {
        lh[i] = softmax_row(qh + (int64_t)i * d, kh, N, d, scale, mk, i, s_row.data(), p_row.data());
        double* oi = oh + (int64_t)i * d;
        for (int t = 0; t < d; ++t) oi[t] = 0.0;
        for (int j = 0; j < N; ++j) {
          if (p_row[j] == 0.0) continue;
          const double* vj = vh + (int64_t)j * d;
          for (int t = 0; t < d; ++t) oi[t] += p_row[j] * vj[t];
        }
      }
    }
  }
}

// Forward for general shapes: q, o: [BH][Nq][d]; k, v: [BH][Nk][d]; lse: [BH][Nq]. No block
// mask; causal uses the bottom-right alignment described at the top of this file.
void oracle_fwd_qk(const double* q, const double* k, const double* v, int64_t BH, int Nq, int Nk, int d,
                   double scale, int causal, double* o, double* lse) {
  Mask mk = make_mask(Nk, causal, nullptr, 128);
  mk.off = Nk - Nq;
  for (int64_t bh = 0; bh < BH; ++bh) {
    const double* qh = q + bh * Nq * d;
    const double* kh = k + bh * Nk * d;
    const double* vh = v + bh * Nk * d;
    double* oh = o + bh * Nq * d;
    double* lh = lse + bh * Nq;
#pragma omp parallel
    {
      std::vector<double> s_row(Nk), p_row(Nk);
#pragma omp for schedule(dynamic, 4)
      for (int i = 0; i < Nq; ++i) {
        lh[i] = softmax_row(qh + (int64_t)i * d, kh, Nk, d, scale, mk, i, s_row.data(), p_row.data());
        double* oi = oh + (int64_t)i * d;
        for (int t = 0; t < d; ++t) oi[t] = 0.0;
        for (int j = 0; j < Nk; ++j) {
          if (p_row[j] == 0.0) continue;
          const double* vj = vh + (int64_t)j * d;
          for (int t = 0; t < d; ++t) oi[t] += p_row[j] * vj[t];
        }
      }
    }
  }
}

// Forward restricted to the listed query rows of ONE head (qh, kh, vh: [N][d]).
// o_rows: [nrows][d]; lse_rows: [nrows].
void oracle_fwd_rows(const double* qh, const double* kh, const double* vh, int N, int d, double scale,
                     int causal, const uint8_t* mask, int mask_bs, const int* rows, int nrows,
                     double* o_rows, double* lse_rows) {
  const Mask mk = make_mask(N, causal, mask, mask_bs);
#pragma omp parallel
  {
    std::vector<double> s_row(N), p_row(N);
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
      const int i = rows[r];
      lse_rows[r] = softmax_row(qh + (int64_t)i * d, kh, N, d, scale, mk, i, s_row.data(), p_row.data());
      double* oi = o_rows + (int64_t)r * d;
      for (int t = 0; t < d; ++t) oi[t] = 0.0;
      for (int j = 0; j < N; ++j) {
        if (p_row[j] == 0.0) continue;
        for (int t = 0; t < d; ++t) oi[t] += p_row[j] * vh[(int64_t)j * d + t];
      }
    }
  }
}

}  // extern "C"

namespace {

// Backward of one head: Nq query rows (qh, doh, dqh: [Nq][d]) against Nk keys (kh, vh, dkh,
// dvh: [Nk][d]); mk decides which (i, j) are allowed. dK and dV are summed over query rows,
// so each thread accumulates its own partial copy (dk_part, dv_part: T x Nk x d) and the
// copies are added at the end. Dh (nullable): [Nq], D_i from its definition.
void bwd_head(const double* qh, const double* kh, const double* vh, const double* doh, int Nq, int Nk, int d,
              double scale, const Mask& mk, int T, std::vector<double>& dk_part, std::vector<double>& dv_part,
              double* dqh, double* dkh, double* dvh, double* Dh) {
  std::fill(dk_part.begin(), dk_part.end(), 0.0);
  std::fill(dv_part.begin(), dv_part.end(), 0.0);
#pragma omp parallel num_threads(T)
  {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    double* dk_t = dk_part.data() + (size_t)tid * Nk * d;
    double* dv_t = dv_part.data() + (size_t)tid * Nk * d;
    std::vector<double> s_row(Nk), p_row(Nk), dp_row(Nk);
#pragma omp for schedule(dynamic, 4)
    for (int i = 0; i < Nq; ++i) {
      const double* qi = qh + (int64_t)i * d;
      const double* doi = doh + (int64_t)i * d;
      softmax_row(qi, kh, Nk, d, scale, mk, i, s_row.data(), p_row.data());
      double Di = 0.0;
      for (int j = 0; j < Nk; ++j) {
        if (p_row[j] == 0.0) { dp_row[j] = 0.0; continue; }
        dp_row[j] = dot(doi, vh + (int64_t)j * d, d);  // dP_ij = dO_i . v_j
        Di += p_row[j] * dp_row[j];
      }
      if (Dh) Dh[i] = Di;
      double* dqi = dqh + (int64_t)i * d;
      for (int t = 0; t < d; ++t) dqi[t] = 0.0;
      for (int j = 0; j < Nk; ++j) {
        const double pij = p_row[j];
        if (pij == 0.0) continue;
        const double dsij = pij * (dp_row[j] - Di);  // dS_ij = P_ij (dP_ij - D_i)
        const double* kj = kh + (int64_t)j * d;
        double* dkj = dk_t + (int64_t)j * d;
        double* dvj = dv_t + (int64_t)j * d;
        for (int t = 0; t < d; ++t) {
          dqi[t] += scale * dsij * kj[t];
          dkj[t] += scale * dsij * qi[t];
          dvj[t] += pij * doi[t];
        }
      }
    }
  }
  // Sum the per-thread partial dK, dV.
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < (int64_t)Nk * d; ++e) {
    double a = 0.0, b = 0.0;
    for (int t = 0; t < T; ++t) {
      a += dk_part[(size_t)t * Nk * d + e];
      b += dv_part[(size_t)t * Nk * d + e];
    }
    dkh[e] = a;
    dvh[e] = b;
  }
}

}  // namespace

extern "C" {

// Backward for all BH heads. Outputs dq, dk, dv: [BH][N][d]; Dvec: [BH][N] holds
// D_i = sum_j P_ij dP_ij computed from that definition.
void oracle_bwd(const double* q, const double* k, const double* v, const double* dout, int64_t BH,
                int N, int d, double scale, int causal, const uint8_t* mask, int mask_bs, double* dq,
                double* dk, double* dv, double* Dvec) {
  const Mask mk = make_mask(N, causal, mask, mask_bs);
  const int T = nthreads_used();
  std::vector<double> dk_part((size_t)T * N * d), dv_part((size_t)T * N * d);
  for (int64_t bh = 0; bh < BH; ++bh) {
    const int64_t off = bh * N * d;
    bwd_head(q + off, k + off, v + off, dout + off, N, N, d, scale, mk, T, dk_part, dv_part, dq + off, dk + off,
             dv + off, Dvec ? Dvec + bh * N : nullptr);
  }
}

// Backward for general shapes (the gradient of oracle_fwd_qk): q, dout, dq: [BH][Nq][d];
// k, v, dk, dv: [BH][Nk][d]; Dvec: [BH][Nq]. Causal uses the bottom-right alignment; no mask.
void oracle_bwd_qk(const double* q, const double* k, const double* v, const double* dout, int64_t BH, int Nq,
                   int Nk, int d, double scale, int causal, double* dq, double* dk, double* dv, double* Dvec) {
  Mask mk = make_mask(Nk, causal, nullptr, 128);
  mk.off = Nk - Nq;
  const int T = nthreads_used();
  std::vector<double> dk_part((size_t)T * Nk * d), dv_part((size_t)T * Nk * d);
  for (int64_t bh = 0; bh < BH; ++bh) {
    bwd_head(q + bh * Nq * d, k + bh * Nk * d, v + bh * Nk * d, dout + bh * Nq * d, Nq, Nk, d, scale, mk, T,
             dk_part, dv_part, dq + bh * Nq * d, dk + bh * Nk * d, dv + bh * Nk * d, Dvec ? Dvec + bh * Nq : nullptr);
  }
}

// Online (single sweep over key blocks) forward, for the equivalence check only.
// deferred = 0: output renormalised at every block ([P3] §3.2 steps 1-3, §3.4).
// deferred = 1: output kept unnormalised and divided by the normaliser once at the end.
void oracle_online_fwd(const double* q, const double* k, const double* v, int64_t BH, int N, int d,
                       double scale, int causal, const uint8_t* mask, int mask_bs, int block,
                       int deferred, double* o, double* lse) {
  const Mask mk = make_mask(N, causal, mask, mask_bs);
  const double NEG_INF = -std::numeric_limits<double>::infinity();
  if (block < 1) block = 1;
  for (int64_t bh = 0; bh < BH; ++bh) {
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
#pragma omp parallel
    {
      std::vector<double> s(block), acc(d);
#pragma omp for schedule(dynamic, 4)
      for (int i = 0; i < N; ++i) {
        const double* qi = qh + (int64_t)i * d;
        double m = NEG_INF;  // running maximum m_i
        double l = 0.0;      // running normaliser l~_i
        for (int t = 0; t < d; ++t) acc[t] = 0.0;  // running output o~_i
        for (int j0 = 0; j0 < N; j0 += block) {
          const int j1 = j0 + block < N ? j0 + block : N;
          double mb = NEG_INF;  // maximum over this block's allowed scores
          for (int j = j0; j < j1; ++j) {
            if (mk.allowed(i, j)) {
              s[j - j0] = scale * dot(qi, kh + (int64_t)j * d, d);
              if (s[j - j0] > mb) mb = s[j - j0];
            }
          }
          if (mb == NEG_INF) continue;  // nothing allowed in this block
          const double m_new = mb > m ? mb : m;
          const double alpha = (m == NEG_INF) ? 0.0 : std::exp(m - m_new);  // e^{m_{i-1} - m_i}
          double blk_sum = 0.0;
          for (int t = 0; t < d; ++t) {
            double pv = 0.0;
            for (int j = j0; j < j1; ++j)
              if (mk.allowed(i, j)) pv += std::exp(s[j - j0] - m_new) * vh[(int64_t)j * d + t];
            if (deferred) {
              acc[t] = acc[t] * alpha + pv;
            } else {
              // o~_{i-1} l~_{i-1} e^{m_{i-1}-m_i} + sum e^{s-m_i} v; divided by l~_i below.
              acc[t] = acc[t] * (l * alpha) + pv;
            }
          }
          for (int j = j0; j < j1; ++j)
            if (mk.allowed(i, j)) blk_sum += std::exp(s[j - j0] - m_new);
          const double l_new = l * alpha + blk_sum;  // l~_i = l~_{i-1} e^{m_{i-1}-m_i} + sum e^{s-m_i}
          if (!deferred)
            for (int t = 0; t < d; ++t) acc[t] /= l_new;  // o~_i is normalised at every step
          m = m_new;
          l = l_new;
        }
        double* oi = o + bh * N * d + (int64_t)i * d;
        if (m == NEG_INF) {
          for (int t = 0; t < d; ++t) oi[t] = 0.0;
          lse[bh * N + i] = NEG_INF;
          continue;
        }
        for (int t = 0; t < d; ++t) oi[t] = deferred ? acc[t] / l : acc[t];
        lse[bh * N + i] = m + std::log(l);
      }
    }
  }
}

}  // extern "C"
