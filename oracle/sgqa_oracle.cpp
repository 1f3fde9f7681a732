// Sparse GQA oracle: plain, slow, obviously correct CPU implementation in fp64.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load this code:
// only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg use it.
// It shares no code, header, table or helper with the CUDA library.
//
// What it computes (Step 5 Preview's full-context attention layer, "Sparse GQA"):
//   mo.ai.kr, "Step 5 Preview agentic work design", section "model structure and training
//   stability": shared index keys are compressed per block, block size 8, and each KV group
//   picks its own relevant past context; the final setting is B = 8, k = 4096 tokens, i.e.
//   512 blocks; the full-context layer is Sparse GQA built on Gated GQA.
//   ai.info, "StepFun illustrates the 92-block architecture of Step 5 Preview", section
//   "Sparse GQA aims at a 1 million token context": relevant past blocks are selected instead
//   of attending to the whole history; blocks of eight tokens cut indexing and selection cost.
//
// The pages give no formula. The readings taken (each is stated where it is used):
//   compress   kbar[b,j,:] = (1/B) * sum_{i<B} k_idx[b, jB+i, :]          complete blocks only
//   score      s[t,g,j]   = q_idx[t,g,:] . kbar[j,:]                          j < c(t) = floor(t/B)
//   select     S(t,g) = top m(t) = min(K_b - 1, c(t)) candidates by (s desc, j asc),
//              plus the own block c(t); ascending; K_b = k / B
//   attend     U = {u <= t : floor(u/B) in S(t,g)}, for each head h of group g = floor(h/R):
//              o = softmax_U(q[t,h] . k[u,g] / sqrt(d)) . v[u,g]
//   gate       out = o * sigmoid(gate_logits[t,h])   (elementwise)
// All arithmetic is fp64; bf16 inputs arrive as uint16 bit patterns.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

struct Dims {
  int batch, T, Hq, G, d, d_idx, B, k;
};

double bf16_to_f64(uint16_t u) {
  uint32_t x = (uint32_t)u << 16;
  float f;
  std::memcpy(&f, &x, sizeof f);
  return (double)f;
}

bool dims_ok(const Dims* dm) {
  return dm && dm->batch > 0 && dm->T > 0 && dm->Hq > 0 && dm->G > 0 && dm->Hq % dm->G == 0 &&
         dm->d > 0 && dm->d_idx > 0 && dm->B > 0 && dm->k > 0 && dm->k % dm->B == 0;
}

void set_threads(int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
}

// Candidate ranking: higher score first, equal scores go to the lower block index.
struct Cand {
  double s;
  int j;
};
inline bool ranks_before(const Cand& a, const Cand& b) {
  return a.s > b.s || (a.s == b.s && a.j < b.j);
}

}  // namespace

extern "C" {

int oracle_max_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Block-key compression: kbar[b, j, i] = mean of the B index keys of block j (fp64; exact for
// bf16 inputs). Only complete blocks j < floor(T / B) exist. kbar: [batch, T/B, d_idx].
int oracle_compress(const Dims* dm, const uint16_t* k_idx, double* kbar, int n_threads) {
  if (!dims_ok(dm)) return -1;
  set_threads(n_threads);
  const int nblk = dm->T / dm->B;
  const long total = (long)dm->batch * nblk;
#pragma omp parallel for schedule(static)
  for (long bj = 0; bj < total; ++bj) {
    const long b = bj / nblk, j = bj % nblk;
    for (int i = 0; i < dm->d_idx; ++i) {
      double sum = 0.0;
      for (int r = 0; r < dm->B; ++r)
        sum += bf16_to_f64(k_idx[((b * dm->T) + j * dm->B + r) * dm->d_idx + i]);
      kbar[bj * dm->d_idx + i] = sum / (double)dm->B;
    }
  }
  return 0;
}

// Indexer scores of one (token, group) row against candidate blocks j < n:
// s[j] = q_idx_row . kbar[b, j]. kbar_b points at kbar[b, 0, 0].
int oracle_scores(const Dims* dm, const double* kbar_b, const uint16_t* q_idx_row, int n, double* s) {
  if (!dims_ok(dm) || n < 0) return -1;
  for (int j = 0; j < n; ++j) {
    double acc = 0.0;
    for (int i = 0; i < dm->d_idx; ++i) acc += bf16_to_f64(q_idx_row[i]) * kbar_b[(long)j * dm->d_idx + i];
    s[j] = acc;
  }
  return 0;
}

// Block selection for a list of query rows.
//   rows_bt   [n_rows][2]  (b, t) of each query row
//   q_idx     [n_rows, G, d_idx] bf16 bits: the rows' indexer queries
//   kbar      [batch, T/B, d_idx] fp64 from oracle_compress
//   sel       [n_rows, G, K_b] out: ascending block ids, own block included, -1 padded
//   s_m, s_m1 [n_rows, G] out: the m-th and (m+1)-th best candidate scores (NaN if absent)
int oracle_select(const Dims* dm, const double* kbar, int n_rows, const int32_t* rows_bt,
                  const uint16_t* q_idx, int32_t* sel, double* s_m, double* s_m1, int n_threads) {
  if (!dims_ok(dm)) return -1;
  set_threads(n_threads);
  const int Kb = dm->k / dm->B, nblk = dm->T / dm->B;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (long rg = 0; rg < (long)n_rows * dm->G; ++rg) {
    const long row = rg / dm->G;
    const int g = (int)(rg % dm->G);
    const int b = rows_bt[2 * row], t = rows_bt[2 * row + 1];
    int32_t* out = sel + rg * Kb;
    if (b < 0 || b >= dm->batch || t < 0 || t >= dm->T) {
      bad = 1;
      continue;
    }
    const int c = t / dm->B;                  // own block; candidates are the complete past blocks
    const int m = std::min(Kb - 1, c);        // the own block counts toward the budget
    std::vector<double> s(c);
    oracle_scores(dm, kbar + (long)b * nblk * dm->d_idx, q_idx + rg * dm->d_idx, c, s.data());
    std::vector<Cand> cand(c);
    for (int j = 0; j < c; ++j) cand[j] = Cand{s[j], j};
    if (m < c) std::nth_element(cand.begin(), cand.begin() + m, cand.end(), ranks_before);
    double sm = NAN, sm1 = NAN;
    if (m > 0) sm = std::max_element(cand.begin(), cand.begin() + m, ranks_before)->s;
    if (m < c) sm1 = cand[m].s;
    std::vector<int> pick(m + 1);
    for (int i = 0; i < m; ++i) pick[i] = cand[i].j;
    pick[m] = c;
    std::sort(pick.begin(), pick.end());
    for (int i = 0; i < Kb; ++i) out[i] = i <= m ? pick[i] : -1;
    s_m[rg] = sm;
    s_m1[rg] = sm1;
  }
  return bad ? -2 : 0;
}

// Gated attention over the selected tokens, for a list of query rows.
//   q, gate   [n_rows, Hq, d] bf16 bits (the rows' queries and gate logits)
//   k, v      [batch, T, G, d] bf16 bits (whole sequences)
//   sel       [n_rows, G, K_b] block ids (any order, -1 = unused slot)
//   out       [n_rows, Hq, d] fp64
// Returns -3 if a selection names a block that is not the own block or a complete past block.
int oracle_attend(const Dims* dm, int n_rows, const int32_t* rows_bt, const uint16_t* q,
                  const uint16_t* k, const uint16_t* v, const uint16_t* gate, const int32_t* sel,
                  double* out, int n_threads) {
  if (!dims_ok(dm)) return -1;
  set_threads(n_threads);
  const int Kb = dm->k / dm->B, R = dm->Hq / dm->G, d = dm->d;
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (long rh = 0; rh < (long)n_rows * dm->Hq; ++rh) {
    const long row = rh / dm->Hq;
    const int h = (int)(rh % dm->Hq), g = h / R;
    const long b = rows_bt[2 * row];
    const int t = rows_bt[2 * row + 1];
    const int32_t* S = sel + (row * dm->G + g) * Kb;
    const uint16_t* qv = q + rh * d;
    std::vector<int> U;
    for (int i = 0; i < Kb; ++i) {
      const int j = S[i];
      if (j < 0) continue;
      if (j > t / dm->B) { bad = 1; continue; }
      for (int u = j * dm->B; u < (j + 1) * dm->B && u <= t; ++u) U.push_back(u);
    }
    std::vector<double> z(U.size());
    double zmax = -INFINITY;
    for (size_t n = 0; n < U.size(); ++n) {
      const uint16_t* kv = k + ((b * dm->T + U[n]) * dm->G + g) * d;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += bf16_to_f64(qv[e]) * bf16_to_f64(kv[e]);
      z[n] = dot * inv_sqrt_d;
      zmax = std::max(zmax, z[n]);
    }
    std::vector<double> o(d, 0.0);
    double l = 0.0;
    for (size_t n = 0; n < U.size(); ++n) {
      const double p = std::exp(z[n] - zmax);
      l += p;
      const uint16_t* vv = v + ((b * dm->T + U[n]) * dm->G + g) * d;
      for (int e = 0; e < d; ++e) o[e] += p * bf16_to_f64(vv[e]);
    }
    for (int e = 0; e < d; ++e) {
      const double gl = bf16_to_f64(gate[rh * d + e]);
      const double oe = U.empty() ? 0.0 : o[e] / l;
      out[rh * d + e] = oe * (1.0 / (1.0 + std::exp(-gl)));
    }
  }
  return bad ? -3 : 0;
}

// Gated SWA, the efficient layer that alternates 3:1 with the full-context layer (mo.ai.kr,
// "Step 5 Preview agentic work design", section "model structure and training stability"): the
// same gated softmax attention over the keys of a sliding window, U = {u : t - window < u <= t}.
// The pages give no window size; it is a parameter. Shapes as for oracle_attend; out [n_rows,
// Hq, d] fp64. Returns -1 for window < 1.
int oracle_swa(const Dims* dm, int n_rows, const int32_t* rows_bt, const uint16_t* q, const uint16_t* k,
               const uint16_t* v, const uint16_t* gate, int window, double* out, int n_threads) {
  if (!dims_ok(dm) || window < 1) return -1;
  set_threads(n_threads);
  const int R = dm->Hq / dm->G, d = dm->d;
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
  for (long rh = 0; rh < (long)n_rows * dm->Hq; ++rh) {
    const long row = rh / dm->Hq;
    const int h = (int)(rh % dm->Hq), g = h / R;
    const long b = rows_bt[2 * row];
    const int t = rows_bt[2 * row + 1];
    const int u_lo = std::max(0, t - window + 1);
    const uint16_t* qv = q + rh * d;
    std::vector<double> z(t - u_lo + 1);
    double zmax = -INFINITY;
    for (int u = u_lo; u <= t; ++u) {
      const uint16_t* kv = k + ((b * dm->T + u) * dm->G + g) * d;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += bf16_to_f64(qv[e]) * bf16_to_f64(kv[e]);
      z[u - u_lo] = dot * inv_sqrt_d;
      zmax = std::max(zmax, z[u - u_lo]);
    }
    std::vector<double> o(d, 0.0);
    double l = 0.0;
    for (int u = u_lo; u <= t; ++u) {
      const double p = std::exp(z[u - u_lo] - zmax);
      l += p;
      const uint16_t* vv = v + ((b * dm->T + u) * dm->G + g) * d;
      for (int e = 0; e < d; ++e) o[e] += p * bf16_to_f64(vv[e]);
    }
    for (int e = 0; e < d; ++e) {
      const double gl = bf16_to_f64(gate[rh * d + e]);
      out[rh * d + e] = (o[e] / l) * (1.0 / (1.0 + std::exp(-gl)));
    }
  }
  return 0;
}

// Token coverage of a selection (the ablation's quality metric): for each (row, head), the
// fraction of the top-`ktop` tokens u <= t by exact q[t,h] . k[u,g] (ties to the lower u)
// that lie in the selected token set U(t, g). cov: [n_rows, Hq].
int oracle_coverage(const Dims* dm, int n_rows, const int32_t* rows_bt, const uint16_t* q,
                    const uint16_t* k, const int32_t* sel, int ktop, double* cov, int n_threads) {
  if (!dims_ok(dm) || ktop <= 0) return -1;
  set_threads(n_threads);
  const int Kb = dm->k / dm->B, R = dm->Hq / dm->G, d = dm->d;
#pragma omp parallel for schedule(dynamic, 1)
  for (long rh = 0; rh < (long)n_rows * dm->Hq; ++rh) {
    const long row = rh / dm->Hq;
    const int h = (int)(rh % dm->Hq), g = h / R;
    const long b = rows_bt[2 * row];
    const int t = rows_bt[2 * row + 1];
    std::vector<char> in_sel(t / dm->B + 1, 0);
    const int32_t* S = sel + (row * dm->G + g) * Kb;
    for (int i = 0; i < Kb; ++i)
      if (S[i] >= 0 && S[i] <= t / dm->B) in_sel[S[i]] = 1;
    std::vector<Cand> z(t + 1);
    for (int u = 0; u <= t; ++u) {
      const uint16_t* kv = k + ((b * dm->T + u) * dm->G + g) * d;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += bf16_to_f64(q[rh * d + e]) * bf16_to_f64(kv[e]);
      z[u] = Cand{dot, u};
    }
    const int n = std::min(ktop, t + 1);
    if (n < t + 1) std::nth_element(z.begin(), z.begin() + n, z.end(), ranks_before);
    int hit = 0;
    for (int i = 0; i < n; ++i) hit += in_sel[z[i].j / dm->B];
    cov[rh] = (double)hit / (double)n;
  }
  return 0;
}


// FP8 KV cache (mo.ai.kr, "Step 5 Preview agentic work design", section "long-horizon RL and run
// cost": the KV cache is trained for FP8 storage). The pages give no format details; the reading
// taken: every (token, group) row of K or V (d values) is stored as FP8 E4M3 values (1 sign, 4
// exponent bits with bias 7, 3 mantissa bits; largest finite value 448 = 1.75 * 2^8; subnormals
// in steps of 2^-9) with one power-of-two scale s = 2^e per row, e the smallest integer with
// max_i |x_i| <= 448 * 2^e (e = 0 for an all-zero row). Each value is x_i / s (exact) rounded to
// the nearest E4M3 value, ties to the even mantissa. The dequantized value q_i * s has at most 4
// significant bits, so it is exact in bf16: attention then runs on those values.
//
// e4m3 code of a finite |y| <= 448 (sign separately): the representable magnitudes are k * 2^-9
// (k = 0..7, subnormal) and (8 + m) * 2^(E-3) (E = -6..8, m = 0..7, except E = 8, m = 7 ... 448 is
// E = 8, m = 6; the all-ones code is NaN). Rounding: quantum 2^(E-3) for the binade of |y|
// (E = -6 below 2^-6), n = |y| / quantum exact, round half to even.
static uint8_t e4m3_encode(double y) {
  const uint8_t sign = std::signbit(y) ? 0x80 : 0x00;
  const double a = std::fabs(y);
  if (a == 0.0) return sign;
  int E = (int)std::floor(std::log2(a));
  // guard the floor(log2) against rounding at exact powers of two
  while (std::ldexp(1.0, E) > a) --E;
  while (std::ldexp(1.0, E + 1) <= a) ++E;
  if (E < -6) E = -6;
  const double quantum = std::ldexp(1.0, E - 3);
  const double n = a / quantum;                 // exact: a has a short significand here
  double r = std::floor(n);
  const double frac = n - r;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
  const double v = r * quantum;                 // the rounded magnitude
  if (v == 0.0) return sign;
  if (v < std::ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(v / std::ldexp(1.0, -9)));  // subnormal
  int Ev = (int)std::floor(std::log2(v));
  while (std::ldexp(1.0, Ev) > v) --Ev;
  while (std::ldexp(1.0, Ev + 1) <= v) ++Ev;
  const int m = (int)(v / std::ldexp(1.0, Ev - 3)) - 8;
  return (uint8_t)(sign | (uint8_t)((Ev + 7) << 3) | (uint8_t)m);
}

static double e4m3_decode(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  const double mag = e == 0 ? m * std::ldexp(1.0, -9) : (8 + m) * std::ldexp(1.0, e - 7 - 3);
  return (c & 0x80) ? -mag : mag;
}

// Quantize n_rows rows of d bf16 values: q [n_rows, d] e4m3 codes, scale [n_rows] (powers of 2).
int oracle_quantize_fp8(int n_rows, int d, const uint16_t* x, uint8_t* q, double* scale) {
  if (n_rows < 0 || d <= 0) return -1;
  for (long r = 0; r < n_rows; ++r) {
    double amax = 0.0;
    for (int i = 0; i < d; ++i) amax = std::max(amax, std::fabs(bf16_to_f64(x[r * d + i])));
    int e = 0;
    if (amax > 0.0) {
      // smallest e with amax <= 448 * 2^e
      e = (int)std::ceil(std::log2(amax / 448.0));
      while (amax > 448.0 * std::ldexp(1.0, e)) ++e;
      while (amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;
    }
    scale[r] = std::ldexp(1.0, e);
    for (int i = 0; i < d; ++i) q[r * d + i] = e4m3_encode(bf16_to_f64(x[r * d + i]) / scale[r]);
  }
  return 0;
}

// Dequantize: out [n_rows, d] fp64 = e4m3 value * scale.
int oracle_dequantize_fp8(int n_rows, int d, const uint8_t* q, const double* scale, double* out) {
  if (n_rows < 0 || d <= 0) return -1;
  for (long r = 0; r < n_rows; ++r)
    for (int i = 0; i < d; ++i) out[r * d + i] = e4m3_decode(q[r * d + i]) * scale[r];
  return 0;
}


// Backward of steps (3) and (4) through a given selection (the selection is a discrete choice and
// carries no gradient; the pages train the 1M-context model with this layer: mo.ai.kr, "Step 5
// Preview agentic work design", section "model structure and training stability"). For every
// query row (b, t) and head h of group g, with U the selected tokens u <= t:
//   z_u = q . k_u / sqrt(d),  p = softmax_U(z),  o = sum_u p_u v_u,  s = sigmoid(gate),  y = o * s
// and dy the gradient of y:
//   dgate = dy * o * s * (1 - s)          do = dy * s
//   dv_u += p_u do                         dp_u = do . v_u
//   dz_u = p_u (dp_u - sum_w p_w dp_w)     dq = sum_u dz_u k_u / sqrt(d)     dk_u += dz_u q / sqrt(d)
// dq, dgate [n_rows, Hq, d] (the listed rows); dk, dv [batch, T, G, d] accumulate over all listed
// rows (zeroed here). All fp64; rows are processed one after another.
int oracle_attend_backward(const Dims* dm, int n_rows, const int32_t* rows_bt, const uint16_t* q,
                           const uint16_t* k, const uint16_t* v, const uint16_t* gate, const int32_t* sel,
                           const uint16_t* dy, double* dq, double* dk, double* dv, double* dgate) {
  if (!dims_ok(dm)) return -1;
  const int Kb = dm->k / dm->B, R = dm->Hq / dm->G, d = dm->d;
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  const long kv_elems = (long)dm->batch * dm->T * dm->G * d;
  std::fill(dk, dk + kv_elems, 0.0);
  std::fill(dv, dv + kv_elems, 0.0);
  for (long rh = 0; rh < (long)n_rows * dm->Hq; ++rh) {
    const long row = rh / dm->Hq;
    const int h = (int)(rh % dm->Hq), g = h / R;
    const long b = rows_bt[2 * row];
    const int t = rows_bt[2 * row + 1];
    const int32_t* S = sel + (row * dm->G + g) * Kb;
    std::vector<int> U;
    for (int i = 0; i < Kb; ++i) {
      const int j = S[i];
      if (j < 0) continue;
      if (j > t / dm->B) return -3;
      for (int u = j * dm->B; u < (j + 1) * dm->B && u <= t; ++u) U.push_back(u);
    }
    const uint16_t* qv = q + rh * d;
    auto kat = [&](int u, int e) { return bf16_to_f64(k[((b * dm->T + u) * dm->G + g) * d + e]); };
    auto vat = [&](int u, int e) { return bf16_to_f64(v[((b * dm->T + u) * dm->G + g) * d + e]); };
    std::vector<double> z(U.size()), p(U.size()), o(d, 0.0), dov(d), dp(U.size());
    double zmax = -INFINITY;
    for (size_t n = 0; n < U.size(); ++n) {
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += bf16_to_f64(qv[e]) * kat(U[n], e);
      z[n] = dot * inv_sqrt_d;
      zmax = std::max(zmax, z[n]);
    }
    double l = 0.0;
    for (size_t n = 0; n < U.size(); ++n) l += (p[n] = std::exp(z[n] - zmax));
    for (size_t n = 0; n < U.size(); ++n) {
      p[n] /= l;
      for (int e = 0; e < d; ++e) o[e] += p[n] * vat(U[n], e);
    }
    for (int e = 0; e < d; ++e) {
      const double s = 1.0 / (1.0 + std::exp(-bf16_to_f64(gate[rh * d + e])));
      const double dye = bf16_to_f64(dy[rh * d + e]);
      dgate[rh * d + e] = dye * o[e] * s * (1.0 - s);
      dov[e] = dye * s;
    }
    double sum_pdp = 0.0;
    for (size_t n = 0; n < U.size(); ++n) {
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += dov[e] * vat(U[n], e);
      dp[n] = dot;
      sum_pdp += p[n] * dot;
    }
    for (int e = 0; e < d; ++e) dq[rh * d + e] = 0.0;
    for (size_t n = 0; n < U.size(); ++n) {
      const double dz = p[n] * (dp[n] - sum_pdp);
      const long kvrow = ((b * dm->T + U[n]) * dm->G + g) * d;
      for (int e = 0; e < d; ++e) {
        dq[rh * d + e] += dz * kat(U[n], e) * inv_sqrt_d;
        dk[kvrow + e] += dz * bf16_to_f64(qv[e]) * inv_sqrt_d;
        dv[kvrow + e] += p[n] * dov[e];
      }
    }
  }
  return 0;
}

}  // extern "C"
