// Test infrastructure, not product code.
//
// Plain, slow, fp64 reference for the exact attention forward that the CUDA
// library computes. Only the test suite, the smoke check and the bench's
// CPU-baseline leg may load this library; the product path never does.
//
// What it computes (the plain definition, written out):
//   * "Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V" and its four steps
//     (similarity, scaling, softmax, weighted sum of V): llmtrend.com,
//     "FlashAttention: ...", section on the self-attention bottleneck.
//   * the same computation written as matmul / divide / softmax / matmul on
//     [batch, heads, seq, seq] scores: the tuning handbook chapter 3
//     ("MHA performance tuning"), section "where the MHA memory bottleneck is".
//   * causal attention skips future key positions: same chapter, section
//     "practical notes" (causal mask bullet).
//   * max subtraction before exp (the log-sum-exp trick) and a per-row
//     log-sum-exp: llmtrend.com page, "numerical stability" bullet; the
//     handbook's tiled routine keeps lse[B,H,N] and updates it with log().
//
// For each (b, h, i), with vis(i) = { j : 0 <= j < N and (j <= i if causal) }:
//   s_j   = scale * sum_d q[b,i,h,d] * k[b,j,h,d]      (d ascending)
//   m     = max_{j in vis} s_j
//   l     = sum_{j in vis} exp(s_j - m)                  (j ascending)
//   O_d   = (sum_{j in vis} exp(s_j - m) * v[b,j,h,d]) / l
//   LSE   = m + log(l)                                    (natural log)
//
// Inputs are the raw 16-bit patterns (bf16 or fp16) of Q, K, V in
// [B, N, H, D] order; they are widened to double exactly. Outputs are double:
// O in [B, N, H, D], LSE in [B, H, N].
//
// A second, algorithmically different statement is also here: the tiled
// online-softmax routine printed in the handbook chapter (section "engineering
// implementation"), restated in fp64 with two readings: the block max is taken
// with keepdim (the printed code mixes a [B,H,bs] lse slice with a
// [B,H,bs,1] max), and the routine returns its lse as well as its output.
// Its algebra is exact, so it must agree with the plain definition to
// rounding; the tests use that as an independent pin.

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
double decode_fp16(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int e = (h >> 10) & 0x1f;
  const int f = h & 0x3ff;
  double mag;
  if (e == 0) {
    mag = std::ldexp(static_cast<double>(f), -24);  // subnormal: f * 2^-24
  } else if (e == 31) {
    mag = f ? std::numeric_limits<double>::quiet_NaN()
            : std::numeric_limits<double>::infinity();
  } else {
    mag = std::ldexp(static_cast<double>(1024 + f), e - 25);  // (1.f) * 2^(e-15)
  }
  return sign ? -mag : mag;
}

// bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits.
double decode_bf16(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int e = (h >> 7) & 0xff;
  const int f = h & 0x7f;
  double mag;
  if (e == 0) {
    mag = std::ldexp(static_cast<double>(f), -133);  // subnormal: f * 2^-133
  } else if (e == 255) {
    mag = f ? std::numeric_limits<double>::quiet_NaN()
            : std::numeric_limits<double>::infinity();
  } else {
    mag = std::ldexp(static_cast<double>(128 + f), e - 134);  // (1.f) * 2^(e-127)
  }
  return sign ? -mag : mag;
}

double decode(uint16_t h, int dtype) { return dtype == 0 ? decode_bf16(h) : decode_fp16(h); }

struct Problem {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  int64_t B, N, H, D;
  double scale;
  int causal;
  int dtype;
};

// Index of element (b, n, h, d) in a contiguous [B, N, H, D] tensor.
inline int64_t at(const Problem& p, int64_t b, int64_t n, int64_t h, int64_t d) {
  return ((b * p.N + n) * p.H + h) * p.D + d;
}

// Widen the (b, h) head of a [B,N,H,D] tensor to a dense [N][D] double block.
void widen_head(const Problem& p, const uint16_t* src, int64_t b, int64_t h, std::vector<double>& dst) {
  dst.resize(static_cast<size_t>(p.N * p.D));
  for (int64_t n = 0; n < p.N; ++n)
    for (int64_t d = 0; d < p.D; ++d) dst[n * p.D + d] = decode(src[at(p, b, n, h, d)], p.dtype);
}

int64_t visible_count(const Problem& p, int64_t i) { return p.causal ? (i + 1) : p.N; }

// One query row of the definition, given that row's materialised scores
// s[0 .. nvis-1]. Writes O[0..D-1] and returns LSE.
double finish_row(const Problem& p, const double* s, int64_t nvis, const std::vector<double>& V,
                  double* o_out) {
  double m = -std::numeric_limits<double>::infinity();
  for (int64_t j = 0; j < nvis; ++j) m = s[j] > m ? s[j] : m;
  // the unnormalised weights exp(s_j - m), each evaluated once
  std::vector<double> e(static_cast<size_t>(nvis));
  double l = 0.0;
  for (int64_t j = 0; j < nvis; ++j) {
    e[j] = std::exp(s[j] - m);
    l += e[j];
  }
  // O_d = sum_j e_j V_jd / l, each sum taken over j in ascending order
  std::vector<double> acc(static_cast<size_t>(p.D), 0.0);
  for (int64_t j = 0; j < nvis; ++j) {
    const double ej = e[j];
    const double* vj = &V[j * p.D];
    for (int64_t d = 0; d < p.D; ++d) acc[d] += ej * vj[d];
  }
  for (int64_t d = 0; d < p.D; ++d) o_out[d] = acc[d] / l;
  return m + std::log(l);
}

// s_j for one query row i against all keys j < nvis.
void score_row(const Problem& p, const std::vector<double>& Q, const std::vector<double>& K, int64_t i,
               int64_t nvis, double* s) {
  const double* qi = &Q[i * p.D];
  for (int64_t j = 0; j < nvis; ++j) {
    const double* kj = &K[j * p.D];
    double dot = 0.0;
    for (int64_t d = 0; d < p.D; ++d) dot += qi[d] * kj[d];
    s[j] = p.scale * dot;
  }
}

template <class F>
void parallel_for(int64_t n, int nthreads, F&& fn) {
  if (nthreads <= 1 || n <= 1) {
    fn(0, n);
    return;
  }
  const int64_t nt = nthreads < n ? nthreads : n;
  std::vector<std::thread> pool;
  for (int64_t t = 0; t < nt; ++t) {
    const int64_t lo = n * t / nt, hi = n * (t + 1) / nt;
    pool.emplace_back([&fn, lo, hi] { fn(lo, hi); });
  }
  for (auto& th : pool) th.join();
}

bool valid(const Problem& p) {
  return p.q && p.k && p.v && p.B >= 0 && p.N >= 0 && p.H >= 0 && p.D >= 1 && (p.dtype == 0 || p.dtype == 1);
}

}  // namespace

extern "C" {

// Widen n 16-bit patterns to double (dtype 0 = bf16, 1 = fp16).
int oracle_decode16(const uint16_t* src, int64_t n, int dtype, double* dst) {
  if (!src || !dst || n < 0 || (dtype != 0 && dtype != 1)) return 1;
  for (int64_t i = 0; i < n; ++i) dst[i] = decode(src[i], dtype);
  return 0;
}

// The definition with the whole N x N score matrix of one (b, h) materialised
// in memory (rows filled by `nthreads` threads). O: [B,N,H,D], LSE: [B,H,N].
int oracle_attention_full(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t B, int64_t N,
                          int64_t H, int64_t D, double scale, int causal, int dtype, double* o, double* lse,
                          int nthreads) {
  Problem p{q, k, v, B, N, H, D, scale, causal, dtype};
  if (!valid(p) || !o || !lse) return 1;
  std::vector<double> Q, K, V;
  std::vector<double> S(static_cast<size_t>(N) * static_cast<size_t>(N));
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      widen_head(p, q, b, h, Q);
      widen_head(p, k, b, h, K);
      widen_head(p, v, b, h, V);
      parallel_for(N, nthreads, [&](int64_t lo, int64_t hi) {
        for (int64_t i = lo; i < hi; ++i) score_row(p, Q, K, i, visible_count(p, i), &S[i * N]);
      });
      parallel_for(N, nthreads, [&](int64_t lo, int64_t hi) {
        std::vector<double> orow(static_cast<size_t>(D));
        for (int64_t i = lo; i < hi; ++i) {
          const double L = finish_row(p, &S[i * N], visible_count(p, i), V, orow.data());
          for (int64_t d = 0; d < D; ++d) o[at(p, b, i, h, d)] = orow[d];
          lse[(b * H + h) * N + i] = L;
        }
      });
    }
  }
  return 0;
}

// The same definition for a list of (b, h, i) triples, one score row at a
// time. rows: [nrows][3]; o_rows: [nrows][D]; lse_rows: [nrows]. Rows are
// independent, so this is bit-identical to oracle_attention_full on them. The
// rows of one (b, h) share that head's K and V widened to double once
// (decoding is exact, so this changes no value).
int oracle_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t B, int64_t N,
                          int64_t H, int64_t D, double scale, int causal, int dtype, const int64_t* rows,
                          int64_t nrows, double* o_rows, double* lse_rows, int nthreads) {
  Problem p{q, k, v, B, N, H, D, scale, causal, dtype};
  if (!valid(p) || !rows || nrows < 0 || (nrows > 0 && (!o_rows || !lse_rows))) return 1;
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= N) return 2;
  }
  // the requested rows grouped by head (b, h), in request order within a head
  std::vector<int64_t> order(static_cast<size_t>(nrows));
  for (int64_t r = 0; r < nrows; ++r) order[r] = r;
  std::stable_sort(order.begin(), order.end(), [&](int64_t x, int64_t y) {
    return rows[3 * x] * H + rows[3 * x + 1] < rows[3 * y] * H + rows[3 * y + 1];
  });
  std::vector<double> K, V;
  for (int64_t g0 = 0; g0 < nrows;) {
    const int64_t b = rows[3 * order[g0]], h = rows[3 * order[g0] + 1];
    int64_t g1 = g0;
    while (g1 < nrows && rows[3 * order[g1]] == b && rows[3 * order[g1] + 1] == h) ++g1;
    widen_head(p, k, b, h, K);
    widen_head(p, v, b, h, V);
    parallel_for(g1 - g0, nthreads, [&](int64_t lo, int64_t hi) {
      std::vector<double> qrow(static_cast<size_t>(D));
      std::vector<double> s;
      for (int64_t t = g0 + lo; t < g0 + hi; ++t) {
        const int64_t r = order[t], i = rows[3 * r + 2];
        const int64_t nvis = visible_count(p, i);
        s.assign(static_cast<size_t>(nvis), 0.0);
        for (int64_t d = 0; d < D; ++d) qrow[d] = decode(q[at(p, b, i, h, d)], dtype);
        // s_j = scale * sum_d q_d k_jd, each sum over d in ascending order;
        // four keys at a time only to give the CPU independent chains
        int64_t j = 0;
        for (; j + 4 <= nvis; j += 4) {
          const double* k0 = &K[j * D];
          double dot0 = 0.0, dot1 = 0.0, dot2 = 0.0, dot3 = 0.0;
          for (int64_t d = 0; d < D; ++d) {
            dot0 += qrow[d] * k0[d];
            dot1 += qrow[d] * k0[D + d];
            dot2 += qrow[d] * k0[2 * D + d];
            dot3 += qrow[d] * k0[3 * D + d];
          }
          s[j] = scale * dot0;
          s[j + 1] = scale * dot1;
          s[j + 2] = scale * dot2;
          s[j + 3] = scale * dot3;
        }
        for (; j < nvis; ++j) {
          double dot = 0.0;
          for (int64_t d = 0; d < D; ++d) dot += qrow[d] * K[j * D + d];
          s[j] = scale * dot;
        }
        lse_rows[r] = finish_row(p, s.data(), nvis, V, &o_rows[r * D]);
      }
    });
    g0 = g1;
  }
  return 0;
}

// The definition for a batch of sequences packed without padding, with
// grouped-query heads and queries and keys of different lengths:
//   q, o : [total_q, Hq, D]; k, v : [total_k, Hkv, D]; lse : [Hq, total_q]
//   sequence b owns query rows cu_q[b] .. cu_q[b+1]-1 and key rows
//   cu_k[b] .. cu_k[b+1]-1 (nq and nk rows); query head h reads key/value head
//   h / (Hq / Hkv);
//   vis(i) = { j < nk : (j <= i + nk - nq if causal) }  (causal aligned at the
//   bottom-right corner, which is the square mask when nq == nk);
//   a query with no visible key has O = 0 and LSE = -inf (an empty sum).
// Rows are computed one at a time with the same arithmetic as finish_row.
int oracle_attention_varlen(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int64_t* cu_q,
                            const int64_t* cu_k, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, double scale,
                            int causal, int dtype, double* o, double* lse, int nthreads) {
  if (!q || !k || !v || !cu_q || !cu_k || !o || !lse || B < 0 || Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv != 0 ||
      (dtype != 0 && dtype != 1))
    return 1;
  for (int64_t b = 0; b < B; ++b)
    if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b] || cu_q[0] != 0 || cu_k[0] != 0) return 2;
  const int64_t total_q = cu_q[B];
  const int64_t group = Hq / Hkv;
  // one task per (b, h, i)
  std::vector<int64_t> task_b;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t i = cu_q[b]; i < cu_q[b + 1]; ++i) task_b.push_back(b);
  const int64_t n_rows = static_cast<int64_t>(task_b.size());
  parallel_for(n_rows * Hq, nthreads, [&](int64_t lo, int64_t hi) {
    std::vector<double> s, Vvis, qrow(static_cast<size_t>(D));
    for (int64_t t = lo; t < hi; ++t) {
      const int64_t row = t / Hq, h = t % Hq, b = task_b[row];
      const int64_t nq = cu_q[b + 1] - cu_q[b], nk = cu_k[b + 1] - cu_k[b];
      const int64_t i = row - cu_q[b];
      const int64_t hk = h / group;
      int64_t nvis = nk;
      if (causal) nvis = std::min(nk, std::max<int64_t>(0, i + nk - nq + 1));
      double* orow = &o[(row * Hq + h) * D];
      if (nvis == 0) {
        for (int64_t d = 0; d < D; ++d) orow[d] = 0.0;
        lse[h * total_q + row] = -std::numeric_limits<double>::infinity();
        continue;
      }
      for (int64_t d = 0; d < D; ++d) qrow[d] = decode(q[(row * Hq + h) * D + d], dtype);
      s.assign(static_cast<size_t>(nvis), 0.0);
      Vvis.assign(static_cast<size_t>(nvis * D), 0.0);
      for (int64_t j = 0; j < nvis; ++j) {
        const int64_t krow = cu_k[b] + j;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qrow[d] * decode(k[(krow * Hkv + hk) * D + d], dtype);
        s[j] = scale * dot;
        for (int64_t d = 0; d < D; ++d) Vvis[j * D + d] = decode(v[(krow * Hkv + hk) * D + d], dtype);
      }
      Problem p{q, k, v, 1, nk, 1, D, scale, causal, dtype};
      lse[h * total_q + row] = finish_row(p, s.data(), nvis, Vvis, orow);
    }
  });
  return 0;
}

// Backward of the definition: the gradients of a scalar loss L through O,
// given dO = dL/dO (the recomputation-based backward the jsqmd page describes
// needs exactly these quantities; the weights are recomputed from Q, K and the
// row's log-sum-exp rather than stored). For each (b, h), with
// P_ij = exp(s_ij - LSE_i) over the visible j (0 elsewhere):
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . V_j
//   D_i   = dO_i . O_i              (= sum_j P_ij dP_ij)
//   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i  = scale * sum_j dS_ij K_j
//   dK_j  = scale * sum_i dS_ij Q_i
// O and LSE are the fp64 forward of this file. Inputs are 16-bit patterns in
// [B, N, H, D] (dO too); gradients are double in [B, N, H, D].
int oracle_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                              int64_t B, int64_t N, int64_t H, int64_t D, double scale, int causal, int dtype,
                              double* dq, double* dk, double* dv, int nthreads) {
  Problem p{q, k, v, B, N, H, D, scale, causal, dtype};
  if (!valid(p) || !dout || !dq || !dk || !dv) return 1;
  std::vector<double> Q, K, V, dO;
  std::vector<double> P(static_cast<size_t>(N) * static_cast<size_t>(N));
  std::vector<double> dS(static_cast<size_t>(N) * static_cast<size_t>(N));
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      widen_head(p, q, b, h, Q);
      widen_head(p, k, b, h, K);
      widen_head(p, v, b, h, V);
      widen_head(p, dout, b, h, dO);
      // rows: P, O, D, dP, dS
      parallel_for(N, nthreads, [&](int64_t lo, int64_t hi) {
        std::vector<double> s(static_cast<size_t>(N)), orow(static_cast<size_t>(D));
        for (int64_t i = lo; i < hi; ++i) {
          const int64_t nvis = visible_count(p, i);
          score_row(p, Q, K, i, nvis, s.data());
          const double lse = finish_row(p, s.data(), nvis, V, orow.data());
          double Di = 0.0;
          for (int64_t d = 0; d < D; ++d) Di += dO[i * D + d] * orow[d];
          for (int64_t j = 0; j < N; ++j) {
            if (j < nvis) {
              const double pij = std::exp(s[j] - lse);
              double dpij = 0.0;
              for (int64_t d = 0; d < D; ++d) dpij += dO[i * D + d] * V[j * D + d];
              P[i * N + j] = pij;
              dS[i * N + j] = pij * (dpij - Di);
            } else {
              P[i * N + j] = 0.0;
              dS[i * N + j] = 0.0;
            }
          }
        }
      });
      // dQ rows
      parallel_for(N, nthreads, [&](int64_t lo, int64_t hi) {
        for (int64_t i = lo; i < hi; ++i)
          for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t j = 0; j < N; ++j) acc += dS[i * N + j] * K[j * D + d];
            dq[at(p, b, i, h, d)] = scale * acc;
          }
      });
      // dK, dV rows
      parallel_for(N, nthreads, [&](int64_t lo, int64_t hi) {
        for (int64_t j = lo; j < hi; ++j)
          for (int64_t d = 0; d < D; ++d) {
            double ak = 0.0, av = 0.0;
            for (int64_t i = 0; i < N; ++i) {
              ak += dS[i * N + j] * Q[i * D + d];
              av += P[i * N + j] * dO[i * D + d];
            }
            dk[at(p, b, j, h, d)] = scale * ak;
            dv[at(p, b, j, h, d)] = av;
          }
      });
    }
  }
  return 0;
}

// Backward of oracle_attention_varlen (packed sequences, grouped-query heads,
// causal mask aligned at the bottom-right corner), the same gradients as
// oracle_attention_backward, per sequence b and query head h:
//   P_ij, dP_ij, D_i, dS_ij  as there, over the keys visible to query i
//                            (P_ij = dS_ij = 0 elsewhere; a query with no
//                            visible key has P = 0 and dQ = 0)
//   dQ_i  (head h)           = scale * sum_j dS_ij K_j
//   dK_j  (K/V head hk)      = scale * sum_{h in group(hk)} sum_i dS^h_ij Q^h_i
//   dV_j  (K/V head hk)      = sum_{h in group(hk)} sum_i P^h_ij dO^h_i
// where group(hk) are the query heads hk G .. hk G + G - 1 (G = Hq / Hkv)
// that read K/V head hk: each K/V element serves every head of its group, so
// its gradient is the sum over them (taken in ascending h, each head's sum
// over i first). Layouts as oracle_attention_varlen: q, dout, dq
// [total_q, Hq, D]; k, v, dk, dv [total_k, Hkv, D]; gradients in double.
int oracle_attention_backward_varlen(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                                     const int64_t* cu_q, const int64_t* cu_k, int64_t B, int64_t Hq, int64_t Hkv,
                                     int64_t D, double scale, int causal, int dtype, double* dq, double* dk,
                                     double* dv, int nthreads) {
  if (!q || !k || !v || !dout || !cu_q || !cu_k || !dq || !dk || !dv || B < 0 || Hq < 1 || Hkv < 1 || D < 1 ||
      Hq % Hkv != 0 || (dtype != 0 && dtype != 1))
    return 1;
  for (int64_t b = 0; b < B; ++b)
    if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b] || cu_q[0] != 0 || cu_k[0] != 0) return 2;
  const int64_t group = Hq / Hkv;
  // widen rows r0 .. r0+n-1 of head h of a [total, heads, D] tensor to [n][D]
  auto widen = [&](const uint16_t* src, int64_t heads, int64_t h, int64_t r0, int64_t n, std::vector<double>& dst) {
    dst.resize(static_cast<size_t>(n * D));
    for (int64_t r = 0; r < n; ++r)
      for (int64_t d = 0; d < D; ++d) dst[r * D + d] = decode(src[((r0 + r) * heads + h) * D + d], dtype);
  };
  std::vector<double> Q, K, V, dO, P, dS, dKacc, dVacc;
  for (int64_t b = 0; b < B; ++b) {
    const int64_t q0 = cu_q[b], nq = cu_q[b + 1] - q0, k0 = cu_k[b], nk = cu_k[b + 1] - k0;
    for (int64_t hk = 0; hk < Hkv; ++hk) {
      widen(k, Hkv, hk, k0, nk, K);
      widen(v, Hkv, hk, k0, nk, V);
      dKacc.assign(static_cast<size_t>(nk * D), 0.0);
      dVacc.assign(static_cast<size_t>(nk * D), 0.0);
      for (int64_t h = hk * group; h < (hk + 1) * group; ++h) {
        widen(q, Hq, h, q0, nq, Q);
        widen(dout, Hq, h, q0, nq, dO);
        P.assign(static_cast<size_t>(nq * nk), 0.0);
        dS.assign(static_cast<size_t>(nq * nk), 0.0);
        // rows: P, O, D, dP, dS, then dQ
        parallel_for(nq, nthreads, [&](int64_t lo, int64_t hi) {
          std::vector<double> s(static_cast<size_t>(nk)), orow(static_cast<size_t>(D));
          for (int64_t i = lo; i < hi; ++i) {
            int64_t nvis = nk;
            if (causal) nvis = std::min(nk, std::max<int64_t>(0, i + nk - nq + 1));
            double* dqrow = &dq[((q0 + i) * Hq + h) * D];
            if (nvis == 0) {
              for (int64_t d = 0; d < D; ++d) dqrow[d] = 0.0;
              continue;
            }
            for (int64_t j = 0; j < nvis; ++j) {
              double dot = 0.0;
              for (int64_t d = 0; d < D; ++d) dot += Q[i * D + d] * K[j * D + d];
              s[j] = scale * dot;
            }
            Problem p{q, k, v, 1, nk, 1, D, scale, causal, dtype};
            const double lse = finish_row(p, s.data(), nvis, V, orow.data());
            double Di = 0.0;
            for (int64_t d = 0; d < D; ++d) Di += dO[i * D + d] * orow[d];
            for (int64_t j = 0; j < nvis; ++j) {
              const double pij = std::exp(s[j] - lse);
              double dpij = 0.0;
              for (int64_t d = 0; d < D; ++d) dpij += dO[i * D + d] * V[j * D + d];
              P[i * nk + j] = pij;
              dS[i * nk + j] = pij * (dpij - Di);
            }
            for (int64_t d = 0; d < D; ++d) {
              double acc = 0.0;
              for (int64_t j = 0; j < nk; ++j) acc += dS[i * nk + j] * K[j * D + d];
              dqrow[d] = scale * acc;
            }
          }
        });
        // this head's share of dK, dV
        parallel_for(nk, nthreads, [&](int64_t lo, int64_t hi) {
          for (int64_t j = lo; j < hi; ++j)
            for (int64_t d = 0; d < D; ++d) {
              double ak = 0.0, av = 0.0;
              for (int64_t i = 0; i < nq; ++i) {
                ak += dS[i * nk + j] * Q[i * D + d];
                av += P[i * nk + j] * dO[i * D + d];
              }
              dKacc[j * D + d] += ak;
              dVacc[j * D + d] += av;
            }
        });
      }
      for (int64_t j = 0; j < nk; ++j)
        for (int64_t d = 0; d < D; ++d) {
          dk[((k0 + j) * Hkv + hk) * D + d] = scale * dKacc[j * D + d];
          dv[((k0 + j) * Hkv + hk) * D + d] = dVacc[j * D + d];
        }
    }
  }
  return 0;
}

// The handbook's tiled online-softmax routine, in fp64, one (b, h) at a time.
// For every query block [qs, qe) and every key block [ks, ke) (both cut at
// block_size, the last one truncated at N):
//   scores    = scale * Q_blk K_blk^T            (future keys = -inf if causal)
//   blk_max   = row max of scores                (keepdim reading)
//   mu        = max(lse, blk_max)
//   e_new     = exp(scores - mu),  e_old = exp(lse - mu)
//   out       = (out * e_old + e_new V_blk) / (e_old + rowsum(e_new))
//   lse       = mu + log(e_old + rowsum(e_new))
// Key blocks that lie wholly in the future of every row of the query block
// are skipped (the causal reading); key block 0 always holds a visible key,
// so lse is finite after it and mu never subtracts -inf from -inf.
int oracle_tiled_reference(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t B, int64_t N,
                           int64_t H, int64_t D, double scale, int causal, int dtype, int64_t block_size,
                           double* o, double* lse) {
  Problem p{q, k, v, B, N, H, D, scale, causal, dtype};
  if (!valid(p) || !o || !lse || block_size < 1) return 1;
  const double ninf = -std::numeric_limits<double>::infinity();
  std::vector<double> Q, K, V;
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      widen_head(p, q, b, h, Q);
      widen_head(p, k, b, h, K);
      widen_head(p, v, b, h, V);
      for (int64_t qs = 0; qs < N; qs += block_size) {
        const int64_t qe = qs + block_size < N ? qs + block_size : N;
        const int64_t nq = qe - qs;
        std::vector<double> out(static_cast<size_t>(nq * D), 0.0);
        std::vector<double> run_lse(static_cast<size_t>(nq), ninf);
        for (int64_t ks = 0; ks < N; ks += block_size) {
          if (causal && ks > qe - 1) break;  // every key of this block is in every row's future
          const int64_t ke = ks + block_size < N ? ks + block_size : N;
          const int64_t nk = ke - ks;
          for (int64_t r = 0; r < nq; ++r) {
            const int64_t i = qs + r;
            std::vector<double> sc(static_cast<size_t>(nk));
            double bmax = ninf;
            for (int64_t c = 0; c < nk; ++c) {
              const int64_t j = ks + c;
              if (causal && j > i) {
                sc[c] = ninf;
              } else {
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d) dot += Q[i * D + d] * K[j * D + d];
                sc[c] = scale * dot;
              }
              bmax = sc[c] > bmax ? sc[c] : bmax;
            }
            const double mu = run_lse[r] > bmax ? run_lse[r] : bmax;
            const double e_old = std::exp(run_lse[r] - mu);
            double e_sum = 0.0;
            std::vector<double> e(static_cast<size_t>(nk));
            for (int64_t c = 0; c < nk; ++c) {
              e[c] = std::exp(sc[c] - mu);
              e_sum += e[c];
            }
            for (int64_t d = 0; d < D; ++d) {
              double pv = 0.0;
              for (int64_t c = 0; c < nk; ++c) pv += e[c] * V[(ks + c) * D + d];
              out[r * D + d] = (out[r * D + d] * e_old + pv) / (e_old + e_sum);
            }
            run_lse[r] = mu + std::log(e_old + e_sum);
          }
        }
        for (int64_t r = 0; r < nq; ++r) {
          for (int64_t d = 0; d < D; ++d) o[at(p, b, qs + r, h, d)] = out[r * D + d];
          lse[(b * H + h) * N + qs + r] = run_lse[r];
        }
      }
    }
  }
  return 0;
}

}  // extern "C"
